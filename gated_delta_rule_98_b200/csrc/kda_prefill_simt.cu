// kda_prefill_simt.cu -- chunkwise KDA prefill on CUDA cores in fp32.
//
// This path serves every supported size and dtype.  It is the path for fp32
// inputs, whose max-abs tolerance of 1e-4 TF32/bf16 tensor-core operands
// cannot meet.  Two kernels:
//
//   prep  (one CTA per chunk and head, all chunks in parallel)
//         gate, unit-length q/k, chunk-local cumulative log-decay Gam,
//         A_kk / A_qk, T = (I + A_kk)^{-1} by forward substitution on 16x16
//         diagonal blocks plus block combination, W = T Diag(beta)(K e^Gam),
//         U~ = T Diag(beta) V, Q' = Q e^Gam, K' = K e^{Gam_last - Gam},
//         gamma = e^{Gam_last}; results go to the workspace.
//   state (one CTA per sequence, head and 32-column slice of the state)
//         sequential over the sequence's chunks:
//           U = U~ - W S;  O = Q' S + A_qk U;  S = Diag(gamma) S + K'^T U.
//
// Chunk algebra: Kimi Linear summary §3.1 (WY representation, UT transform,
// forward-substitution inverse; output = incoming-state term + causal
// intra-chunk term) and Appendix C (cumulative log-decay per chunk), written
// out from the recurrence of §3 with the decay applied first.  The columns of
// S never mix in the recurrence, so the state is split by value columns.
//
// The intra-chunk decay factors exp(Gam_r - Gam_i), i <= r, are evaluated
// directly per pair here (always <= 1, no rescaling needed in fp32).
#include "kda_common.cuh"
#include "kda_launch.h"

namespace kda {
namespace {

struct SimtLayout {
  size_t W, Ut, Qp, Kp, Aqk, gam, total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

SimtLayout simt_layout(int N, int T, int H, int dk, int dv, int C) {
  SimtLayout L;
  const size_t th = (size_t)T * H;
  size_t off = sizeof(WsHeader);
  L.W = off;   off = align256(off + th * dk * 4);
  L.Ut = off;  off = align256(off + th * dv * 4);
  L.Qp = off;  off = align256(off + th * dk * 4);
  L.Kp = off;  off = align256(off + th * dk * 4);
  L.Aqk = off; off = align256(off + th * C * 4);
  const size_t nc = (size_t)T / C + N + 1;  // chunk ids cu[n]/C + n + j are unique below this
  L.gam = off; off = align256(off + nc * H * dk * 4);
  L.total = off;
  return L;
}

struct SimtParams {
  const void *q, *k, *v, *z, *beta;
  const float *A, *g, *S0;
  const float* gs;  // scalar log-decay [T, H] (one per token and head), or null
  const int32_t* cu;
  void* o;
  float* S_final;
  float* S_ckpt;  // checkpoints every ckpt_every chunks (ckpt_count per sequence and head)
  int ckpt_every, ckpt_count;
  const void* og;  // output epilogue: sigmoid gate input [T, H, DV] (input dtype), or null
  const float* ow;  // RMSNorm gain [DV], or null (ones)
  float oeps;
  int N, T, max_len, H, max_cps;
  float *W, *Ut, *Qp, *Kp, *Aqk, *gam;
  WsHeader* hdr;
};

template <int DK, int DV, int C>
constexpr size_t prep_smem_floats() {
  return 3 * C * (DK + 1) + C * (DV + 1) + 3 * C * (C + 1) + C + (C / kSubTile) * 256;
}

template <int DK, int DV, int C, typename T>
__global__ void __launch_bounds__(256) simt_prep_kernel(SimtParams p) {
  constexpr int NT = 256;
  constexpr int NB = C / kSubTile;
  constexpr int LK = DK + 1, LV = DV + 1, LC = C + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.y;
  const int n = blockIdx.x / p.max_cps, j = blockIdx.x % p.max_cps;
  const int H = p.H;

  const bool ok = seqlens_valid(p.cu, p.N, p.T, p.max_len);
  if (!ok && blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) atomicOr(&p.hdr->err, kErrBadSeqlens);
  if (!ok) return;
  int a, b;
  seq_bounds(p.cu, n, p.max_len, a, b);
  const int tok0 = a + j * C;
  if (tok0 >= b) return;
  const int len = min(C, b - tok0);
  const int cid = a / C + n + j;

  extern __shared__ float sm[];
  float* qh = sm;              // [C][LK] unit q
  float* kh = qh + C * LK;     // [C][LK] unit k
  float* G = kh + C * LK;      // [C][LK] log-decay, then its chunk-local cumsum
  float* vv = G + C * LK;      // [C][LV]
  float* Akk = vv + C * LV;    // [C][LC]
  float* Aq = Akk + C * LC;    // [C][LC]
  float* Tm = Aq + C * LC;     // [C][LC]
  float* bet = Tm + C * LC;    // [C]
  float* X = bet + C;          // [NB][16][16] block-combination scratch

  const T* qg = (const T*)p.q;
  const T* kg = (const T*)p.k;
  const T* vg = (const T*)p.v;
  const T* zg = (const T*)p.z;
  const T* bg = (const T*)p.beta;
  const float expA = p.z ? expf(p.A[h]) : 0.f;

  // ---- load (rows past the chunk end are zero: q = k = v = 0, g = 0, beta = 0)
  for (int e = tid; e < C * DK; e += NT) {
    const int r = e / DK, c = e % DK;
    float qv = 0.f, kv = 0.f, gv = 0.f;
    if (r < len) {
      const size_t idx = ((size_t)(tok0 + r) * H + h) * DK + c;
      qv = to_f(qg[idx]);
      kv = to_f(kg[idx]);
      gv = p.g    ? p.g[idx]
           : p.gs ? p.gs[(size_t)(tok0 + r) * H + h]
                  : gate_logdecay(to_f(zg[idx]), expA);
    }
    qh[r * LK + c] = qv;
    kh[r * LK + c] = kv;
    G[r * LK + c] = gv;
  }
  for (int e = tid; e < C * DV; e += NT) {
    const int r = e / DV, c = e % DV;
    vv[r * LV + c] = r < len ? to_f(vg[((size_t)(tok0 + r) * H + h) * DV + c]) : 0.f;
  }
  for (int r = tid; r < C; r += NT) bet[r] = r < len ? to_f(bg[(size_t)(tok0 + r) * H + h]) : 0.f;
  for (int e = tid; e < C * LC; e += NT) Tm[e] = 0.f;
  __syncthreads();

  // ---- unit-length q, k (one warp per row)
  for (int r = warp; r < C; r += NT / 32) {
    float sk = 0.f, sq = 0.f;
    for (int c = lane; c < DK; c += 32) {
      sk += kh[r * LK + c] * kh[r * LK + c];
      sq += qh[r * LK + c] * qh[r * LK + c];
    }
    sk = warp_sum(sk);
    sq = warp_sum(sq);
    const float ik = 1.0f / sqrtf(sk + kNormEps), iq = 1.0f / sqrtf(sq + kNormEps);
    for (int c = lane; c < DK; c += 32) {
      kh[r * LK + c] *= ik;
      qh[r * LK + c] *= iq;
    }
  }
  // ---- chunk-local inclusive cumsum of g per channel
  for (int c = tid; c < DK; c += NT) {
    float acc = 0.f;
    for (int r = 0; r < C; ++r) {
      acc += G[r * LK + c];
      G[r * LK + c] = acc;
    }
  }
  __syncthreads();

  // ---- A_kk (strictly lower, rows scaled by beta) and A_qk (lower incl. diagonal)
  for (int e = tid; e < C * C; e += NT) {
    const int r = e / C, i = e % C;
    float ak = 0.f, aq = 0.f;
    if (i <= r && r < len) {
      for (int c = 0; c < DK; ++c) {
        const float kd = kh[i * LK + c] * expf(G[r * LK + c] - G[i * LK + c]);
        ak += kh[r * LK + c] * kd;
        aq += qh[r * LK + c] * kd;
      }
    }
    Akk[r * LC + i] = (i < r) ? bet[r] * ak : 0.f;
    Aq[r * LC + i] = aq;
  }
  __syncthreads();

  // ---- T = (I + A_kk)^{-1}: forward substitution inside each 16x16 diagonal block
  if (tid < C) {
    const int r0 = (tid / kSubTile) * kSubTile, col = tid;
    for (int r = r0; r < r0 + kSubTile; ++r) {
      float x = (r == col) ? 1.f : 0.f;
      if (r > col)
        for (int i = col; i < r; ++i) x -= Akk[r * LC + i] * Tm[i * LC + col];
      Tm[r * LC + col] = x;
    }
  }
  __syncthreads();
  // ---- block rows below the diagonal: T_ba = -T_bb sum_{a<=c<b} A_bc T_ca
  for (int dist = 1; dist < NB; ++dist) {
    const int npairs = NB - dist;
    for (int e = tid; e < npairs * 256; e += NT) {
      const int pr = e / 256, rr = (e % 256) / 16, cc = e % 16;
      const int bb = pr + dist, aa = pr;
      float x = 0.f;
      for (int m = aa * kSubTile; m < bb * kSubTile; ++m)
        x += Akk[(bb * kSubTile + rr) * LC + m] * Tm[m * LC + aa * kSubTile + cc];
      X[e] = x;
    }
    __syncthreads();
    for (int e = tid; e < npairs * 256; e += NT) {
      const int pr = e / 256, rr = (e % 256) / 16, cc = e % 16;
      const int bb = pr + dist, aa = pr;
      float y = 0.f;
      for (int m = 0; m < kSubTile; ++m)
        y -= Tm[(bb * kSubTile + rr) * LC + bb * kSubTile + m] * X[pr * 256 + m * 16 + cc];
      Tm[(bb * kSubTile + rr) * LC + aa * kSubTile + cc] = y;
    }
    __syncthreads();
  }

  // ---- Q', K', gamma, A_qk out
  for (int e = tid; e < len * DK; e += NT) {
    const int r = e / DK, c = e % DK;
    const size_t idx = ((size_t)(tok0 + r) * H + h) * DK + c;
    p.Qp[idx] = qh[r * LK + c] * expf(G[r * LK + c]);
    p.Kp[idx] = kh[r * LK + c] * expf(G[(len - 1) * LK + c] - G[r * LK + c]);
  }
  for (int c = tid; c < DK; c += NT)
    p.gam[((size_t)cid * H + h) * DK + c] = expf(G[(len - 1) * LK + c]);
  for (int e = tid; e < len * C; e += NT) {
    const int r = e / C, i = e % C;
    p.Aqk[((size_t)(tok0 + r) * H + h) * C + i] = Aq[r * LC + i];
  }
  __syncthreads();
  // ---- WY blocks: rows of Diag(beta)(K e^Gam) and Diag(beta) V, then multiply by T
  for (int e = tid; e < C * DK; e += NT) {
    const int r = e / DK, c = e % DK;
    kh[r * LK + c] *= bet[r] * expf(G[r * LK + c]);
  }
  for (int e = tid; e < C * DV; e += NT) {
    const int r = e / DV, c = e % DV;
    vv[r * LV + c] *= bet[r];
  }
  __syncthreads();
  for (int e = tid; e < len * DK; e += NT) {
    const int r = e / DK, c = e % DK;
    float acc = 0.f;
    for (int i = 0; i <= r; ++i) acc += Tm[r * LC + i] * kh[i * LK + c];
    p.W[((size_t)(tok0 + r) * H + h) * DK + c] = acc;
  }
  for (int e = tid; e < len * DV; e += NT) {
    const int r = e / DV, c = e % DV;
    float acc = 0.f;
    for (int i = 0; i <= r; ++i) acc += Tm[r * LC + i] * vv[i * LV + c];
    p.Ut[((size_t)(tok0 + r) * H + h) * DV + c] = acc;
  }
}

constexpr int kBV = 32;  // state columns per CTA

template <int DK, int C>
constexpr size_t state_smem_floats() {
  return DK * kBV + 3 * C * (DK + 1) + C * kBV + C * (C + 1) + DK;
}

template <int DK, int DV, int C, typename T>
__global__ void __launch_bounds__(256) simt_state_kernel(SimtParams p) {
  constexpr int NT = 256;
  constexpr int BV = kBV;
  constexpr int LK = DK + 1, LC = C + 1;
  const int tid = threadIdx.x;
  const int n = blockIdx.x, h = blockIdx.y, c0 = blockIdx.z * BV;
  const int H = p.H;
  const bool ok = seqlens_valid(p.cu, p.N, p.T, p.max_len);
  // Also reported by the prep kernel; repeated here for calls where every
  // sequence is empty and prep is not launched.  The host cleared the word.
  if (!ok && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && tid == 0)
    atomicOr(&p.hdr->err, kErrBadSeqlens);
  if (!ok) return;
  int a, b;
  seq_bounds(p.cu, n, p.max_len, a, b);

  extern __shared__ float sm[];
  float* S = sm;              // [DK][BV]
  float* Ws = S + DK * BV;    // [C][LK]
  float* Qs = Ws + C * LK;    // [C][LK]
  float* Ks = Qs + C * LK;    // [C][LK]
  float* Us = Ks + C * LK;    // [C][BV]
  float* As = Us + C * BV;    // [C][LC]
  float* gs = As + C * LC;    // [DK]

  const size_t sbase = ((size_t)n * H + h) * DK * DV;
  for (int e = tid; e < DK * BV; e += NT) {
    const int i = e / BV, c = e % BV;
    S[e] = p.S0 ? p.S0[sbase + (size_t)i * DV + c0 + c] : 0.f;
  }
  T* og = (T*)p.o;
  const int nchunks = (b - a + C - 1) / C;
  for (int j = 0; j < nchunks; ++j) {
    const int tok0 = a + j * C, len = min(C, b - tok0), cid = a / C + n + j;
    __syncthreads();
    for (int e = tid; e < len * DK; e += NT) {
      const int r = e / DK, i = e % DK;
      const size_t idx = ((size_t)(tok0 + r) * H + h) * DK + i;
      Ws[r * LK + i] = p.W[idx];
      Qs[r * LK + i] = p.Qp[idx];
      Ks[r * LK + i] = p.Kp[idx];
    }
    for (int e = tid; e < len * C; e += NT) {
      const int r = e / C, i = e % C;
      As[r * LC + i] = p.Aqk[((size_t)(tok0 + r) * H + h) * C + i];
    }
    for (int i = tid; i < DK; i += NT) gs[i] = p.gam[((size_t)cid * H + h) * DK + i];
    __syncthreads();
    // U = U~ - W S
    for (int e = tid; e < len * BV; e += NT) {
      const int r = e / BV, c = e % BV;
      float acc = p.Ut[((size_t)(tok0 + r) * H + h) * DV + c0 + c];
      for (int i = 0; i < DK; ++i) acc -= Ws[r * LK + i] * S[i * BV + c];
      Us[r * BV + c] = acc;
    }
    __syncthreads();
    // O = Q' S + A_qk U (causal incl. diagonal)
    for (int e = tid; e < len * BV; e += NT) {
      const int r = e / BV, c = e % BV;
      float acc = 0.f;
      for (int i = 0; i < DK; ++i) acc += Qs[r * LK + i] * S[i * BV + c];
      for (int i = 0; i <= r; ++i) acc += As[r * LC + i] * Us[i * BV + c];
      og[((size_t)(tok0 + r) * H + h) * DV + c0 + c] = from_f<T>(acc);
    }
    __syncthreads();
    // S = Diag(gamma) S + K'^T U; a checkpoint after every ckpt_every full chunks
    const bool ckpt = p.S_ckpt && (j + 1) % p.ckpt_every == 0 && (j + 1) * C <= b - a;
    float* Sc = ckpt ? p.S_ckpt + (((size_t)n * H + h) * p.ckpt_count + (j + 1) / p.ckpt_every - 1) *
                                      DK * DV
                     : nullptr;
    for (int e = tid; e < DK * BV; e += NT) {
      const int i = e / BV, c = e % BV;
      float acc = gs[i] * S[e];
      for (int r = 0; r < len; ++r) acc += Ks[r * LK + i] * Us[r * BV + c];
      S[e] = acc;
      if (ckpt) Sc[(size_t)i * DV + c0 + c] = acc;
    }
  }
  __syncthreads();
  if (p.S_final)
    for (int e = tid; e < DK * BV; e += NT) {
      const int i = e / BV, c = e % BV;
      p.S_final[sbase + (size_t)i * DV + c0 + c] = S[e];
    }
}

// Output epilogue (Kimi Linear summary, §4: head-wise RMSNorm of o, then a
// data-dependent sigmoid gate), in place on o after the state pass.  The state
// kernel splits a head's DV features over DV / 32 CTAs, so the row reduction
// runs here: one warp per (token, head) row of DV features.
template <int DV, typename T>
__global__ void __launch_bounds__(256) simt_norm_gate_kernel(SimtParams p) {
  constexpr int PER = DV / 32;
  if (p.hdr->err != kErrNone) return;  // invalid cu_seqlens: o was not written
  const int lane = threadIdx.x & 31;
  const size_t row = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= (size_t)p.T * p.H) return;
  T* o = (T*)p.o + row * DV;
  const T* r = (const T*)p.og + row * DV;
  float x[PER], ss = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    x[i] = to_f(o[lane + 32 * i]);
    ss += x[i] * x[i];
  }
  ss = warp_sum(ss);
  const float inv = rsqrtf(ss * (1.0f / DV) + p.oeps);
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int j = lane + 32 * i;
    const float w = p.ow ? p.ow[j] : 1.f;
    o[j] = from_f<T>(x[i] * inv * w * out_sigmoid(to_f(r[j])));
  }
}

template <int DK, int DV, int C, typename T>
cudaError_t launch_t(const ForwardArgs& a, const SimtParams& p) {
  cudaError_t err;
  if (p.max_cps > 0 && a.N > 0) {
    const size_t smem = prep_smem_floats<DK, DV, C>() * sizeof(float);
    err = cudaFuncSetAttribute(simt_prep_kernel<DK, DV, C, T>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    dim3 grid(a.N * p.max_cps, a.H);
    simt_prep_kernel<DK, DV, C, T><<<grid, 256, smem, a.stream>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  if (a.N > 0) {
    const size_t smem = state_smem_floats<DK, C>() * sizeof(float);
    err = cudaFuncSetAttribute(simt_state_kernel<DK, DV, C, T>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    dim3 grid(a.N, a.H, DV / kBV);
    simt_state_kernel<DK, DV, C, T><<<grid, 256, smem, a.stream>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  if (p.og && a.T > 0) {
    const unsigned rows = (unsigned)((size_t)a.T * a.H);
    simt_norm_gate_kernel<DV, T><<<(rows + 7) / 8, 256, 0, a.stream>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  return cudaSuccess;
}

template <int DK, int DV, int C>
cudaError_t launch_c(const ForwardArgs& a, const SimtParams& p) {
  return a.bf16 ? launch_t<DK, DV, C, __nv_bfloat16>(a, p) : launch_t<DK, DV, C, float>(a, p);
}
template <int DK, int DV>
cudaError_t launch_v(const ForwardArgs& a, const SimtParams& p) {
  return a.chunk == 16 ? launch_c<DK, DV, 16>(a, p) : launch_c<DK, DV, 64>(a, p);
}
template <int DK>
cudaError_t launch_k(const ForwardArgs& a, const SimtParams& p) {
  switch (a.dv) {
    case 32: return launch_v<DK, 32>(a, p);
    case 64: return launch_v<DK, 64>(a, p);
    case 128: return launch_v<DK, 128>(a, p);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

size_t simt_workspace_bytes(int N, int T, int H, int dk, int dv, int chunk) {
  return simt_layout(N, T, H, dk, dv, chunk).total;
}

int simt_launches(int N, int max_len, int chunk) {
  if (N <= 0) return 0;
  return (max_len + chunk - 1) / chunk > 0 ? 2 : 1;
}

cudaError_t launch_forward_simt(const ForwardArgs& a) {
  const SimtLayout L = simt_layout(a.N, a.T, a.H, a.dk, a.dv, a.chunk);
  char* base = (char*)a.ws;
  SimtParams p;
  p.q = a.q; p.k = a.k; p.v = a.v; p.z = a.z; p.beta = a.beta;
  p.A = a.A; p.g = a.g; p.gs = a.g_head; p.S0 = a.S0; p.cu = a.cu; p.o = a.o; p.S_final = a.S_final;
  p.S_ckpt = a.S_ckpt; p.ckpt_every = a.ckpt_every; p.ckpt_count = a.ckpt_count;
  p.og = a.out_gate; p.ow = a.norm_w; p.oeps = a.norm_eps;
  p.N = a.N; p.T = a.T; p.max_len = a.max_len; p.H = a.H;
  p.max_cps = (a.max_len + a.chunk - 1) / a.chunk;
  p.W = (float*)(base + L.W);
  p.Ut = (float*)(base + L.Ut);
  p.Qp = (float*)(base + L.Qp);
  p.Kp = (float*)(base + L.Kp);
  p.Aqk = (float*)(base + L.Aqk);
  p.gam = (float*)(base + L.gam);
  p.hdr = (WsHeader*)base;
  switch (a.dk) {
    case 32: return launch_k<32>(a, p);
    case 64: return launch_k<64>(a, p);
    case 128: return launch_k<128>(a, p);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kda
