// kda_prefill_tc.cu -- chunkwise KDA prefill on the sm_100a tensor cores
// (tcgen05.mma, TMEM accumulators), bf16 inputs, dk = dv = 128, chunk = 64.
//
// One CTA of 256 threads runs one (sequence, head) over its chunks in order
// (Kimi Linear summary §3.1: chunkwise WY / UT form with an inter-chunk state
// carry; §3.2: sub-chunking keeps the channel-wise decay factors in range;
// Appendix C: per-chunk cumulative log-decay, forward-substitution inverse).
// The fp32 state S [dk x dv] lives in Tensor Memory for the whole sequence.
// Per 64-token chunk, with Gam = chunk-local inclusive cumsum of the gate g:
//
//   products  A_kk = StrictTril(Diag(beta) K K^T (decayed)), A_qk = Tril(Q K^T
//             (decayed)), from four M=64 MMAs: for row sub-tile b (16 tokens,
//             reference rho_b = Gam at its first token) the rows carry
//             E = e^{Gam_r - rho_b} <= 1 and the column operand C_b carries
//             e^{rho_b - Gam_i} (<= e^75 on the diagonal sub-tile, <= 1 before)
//   inverse   T = (I + A_kk)^{-1} by forward substitution on 16x16 diagonal
//             blocks plus block combination (fp32, CUDA cores)
//   WY        [W | U~] = T [Diag(beta)(K e^Gam) | Diag(beta) V]   (one MMA)
//   chain     D1 = [W ; Q e^Gam] S      (rows 0-63: W S, rows 64-127: Q' S)
//             U  = U~ - D1[0:64]
//             S  = Diag(e^{Gam_last}) S + (K e^{Gam_last - Gam})^T U
//             O  = D1[64:128] + A_qk U
//
// MMA operands are bf16 in shared memory (no swizzle, 8x16-byte core
// matrices); every accumulator is fp32 in TMEM.  Rows of a partial chunk past
// the sequence end are zero, so they contribute nothing.
//
// Segments: with P > 1 a sequence is cut into P runs of chunks.  The
// transition pass (mode 1) runs each segment but the last from a zero state
// and from the identity, giving the affine map S_out = M S_in + N of the
// segment; a small kernel composes the maps into every segment's incoming
// state; the full pass (mode 0) then runs every segment from its true
// incoming state and writes the outputs.  This is the single-GPU form of the
// prefix scan over per-segment state updates (Kimi K3 architecture summary,
// KDA context parallelism).
#include "kda_common.cuh"
#include "kda_launch.h"
#include "tc_sm100.cuh"

namespace kda {
namespace {

using namespace tc;

constexpr int kC = 64;    // chunk tokens
constexpr int kD = 128;   // dk = dv
constexpr int kNT = 256;  // threads

// ---- shared memory map (bytes) ----
// Region P is reused through a chunk: R + C (products) | A_kk, T (fp32) |
// [X_K | X_V] (WY operand) | U (chain operand).
constexpr int kOffR = 0;               // 128 rows x 128 (K-major): sub-tile b rows 32b..32b+15 = K, +16..31 = Q
constexpr int kOffC = 32768;           // 160 rows x 128 (K-major): C_b at rows 0,16,48,96
constexpr int kOffAkk = 0;             // fp32 [64][65]
constexpr int kOffT = 16640;           // fp32 [64][65]
constexpr int kOffX = 0;               // 256 (N) x 64 (K) MN-major bf16
constexpr int kOffU = 0;               // 128 (N) x 64 (K) MN-major bf16 (transition pass: 256 x 64)
constexpr int kSizeP = 73728;
constexpr int kOffA3 = kSizeP;         // 128 x 64 K-major: rows 0-63 zero, 64-127 A_qk
constexpr int kOffTp = kOffA3 + 16384; // 128 x 64 K-major: rows 0-63 T, 64-127 zero
constexpr int kOffA1 = kOffTp + 16384; // 128 x 128 K-major: rows 0-63 W, 64-127 Q'
constexpr int kOffKp = kOffA1 + 32768; // K': M=128 (dk) x K=64 (tok) MN-major
constexpr int kOffSb = kOffKp + 16384; // S bf16: N=128 (dv) x K=128 (dk) MN-major (transition: N=256)
constexpr int kSizeSb = 65536;
constexpr int kOffVec = kOffSb + kSizeSb;
// vectors (floats)
constexpr int kVecIq = 0, kVecIk = 64, kVecBeta = 128, kVecGam = 192, kVecRho = 320,
              kVecTot = 832, kVecGlast = 960, kVecX = 1088, kVecEnd = 1088 + 1024;
constexpr int kSmemBytes = kOffVec + kVecEnd * 4 + 64;

// TMEM columns
constexpr uint32_t kTmWU = 0;    // [W | U~] (256 columns, rows 0-63 valid)
constexpr uint32_t kTmD1 = 256;  // chain product (128 columns); A products during prep
constexpr uint32_t kTmS = 384;   // fp32 state (128 columns)
// transition pass: the identity-propagated block X uses columns 384..511 as
// the state's partner, and the state moves to 256..383; see tc_kernel.

constexpr long long kWaitCycles = 4000000000LL;  // ~2 s: a wait this long is a fault

__device__ __forceinline__ uint32_t km128(int row, int k) {
  return (row >> 3) * 2048 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
}
__device__ __forceinline__ uint32_t km64(int row, int k) {
  return (row >> 3) * 1024 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
}
template <int E>
__device__ __forceinline__ uint32_t mnm(int m, int k) {
  return (m >> 3) * 128 + (k >> 3) * (E / 8 * 128) + (k & 7) * 16 + (m & 7) * 2;
}

__device__ __forceinline__ void st_bf16(unsigned char* base, uint32_t off, float x) {
  *reinterpret_cast<__nv_bfloat16*>(base + off) = __float2bfloat16_rn(x);
}
__device__ __forceinline__ uint4 pack8(const float* v) {
  uint4 u;
  __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]),
                  c = __floats2bfloat162_rn(v[4], v[5]), d = __floats2bfloat162_rn(v[6], v[7]);
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  u.z = *reinterpret_cast<uint32_t*>(&c);
  u.w = *reinterpret_cast<uint32_t*>(&d);
  return u;
}

struct TcParams {
  const __nv_bfloat16 *q, *k, *v, *z, *beta;
  const float *A, *g, *S0;
  const int32_t* cu;
  __nv_bfloat16* o;
  float* S_final;
  int N, T, max_len, H, P;
  float* seg;  // per (n, h, p): transition M [dk][dk] and offset N [dk][dv] (mode 1 output),
               // incoming state S_in [dk][dv] (composition output, mode 0 input)
  WsHeader* hdr;
};

// Segment p of a sequence with nch chunks: chunks [c0, c1).
__device__ __forceinline__ void segment_chunks(int nch, int P, int p, int& c0, int& c1) {
  const int G = (nch + P - 1) / P;
  c0 = min(nch, p * G);
  c1 = min(nch, c0 + G);
}

// Layout of the segment workspace (floats), per (n, h):
//   trans[p] (p < P-1): M then N, 2 * dk * dv each
//   sin[p]   (p >= 1) : dk * dv
__device__ __forceinline__ float* seg_trans(float* seg, int n, int h, int H, int P, int p) {
  const size_t per = (size_t)(P - 1) * 2 * kD * kD + (size_t)P * kD * kD;
  return seg + ((size_t)n * H + h) * per + (size_t)p * 2 * kD * kD;
}
__device__ __forceinline__ float* seg_sin(float* seg, int n, int h, int H, int P, int p) {
  const size_t per = (size_t)(P - 1) * 2 * kD * kD + (size_t)P * kD * kD;
  return seg + ((size_t)n * H + h) * per + (size_t)(P - 1) * 2 * kD * kD + (size_t)p * kD * kD;
}

// ---------------------------------------------------------------------------
// MODE 0: full pass from the true incoming state, writes o and S_final.
// MODE 1: transition pass of segments 0..P-2: from S = 0 (N) and X = I (M).
template <int MODE>
__global__ void __launch_bounds__(kNT, 1) tc_kernel(TcParams p) {
  extern __shared__ __align__(1024) unsigned char sm[];
  __shared__ uint64_t s_bar;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  float* vec = reinterpret_cast<float*>(sm + kOffVec);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x, h = blockIdx.y, seg = blockIdx.z;
  const int H = p.H;

  const bool ok = seqlens_valid(p.cu, p.N, p.T, p.max_len);
  if (MODE == 0 && n == 0 && h == 0 && seg == 0 && tid == 0)
    p.hdr->err = ok ? kErrNone : kErrBadSeqlens;
  if (!ok) return;
  int a, b;
  seq_bounds(p.cu, n, p.max_len, a, b);
  const int nch = (b - a + kC - 1) / kC;
  int c0, c1;
  segment_chunks(nch, p.P, seg, c0, c1);
  // MODE 1: the last segment needs no transition; empty segments have M = I, N = 0
  if (MODE == 1 && seg >= p.P - 1) return;

  // ---- set-up: TMEM, barrier, constant zero blocks
  if (warp == 0) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&s_bar, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  for (int e = tid * 16; e < 16384; e += kNT * 16) {
    *reinterpret_cast<uint4*>(sm + kOffA3 + e) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(sm + kOffTp + e) = make_uint4(0, 0, 0, 0);
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = s_tmem;
  uint32_t phase = 0;

  // MODE 0: S lives in TMEM columns [384, 512).  MODE 1: the zero-start state
  // S in [256, 384) and the identity-start block X in [384, 512); the chain
  // product then uses [0, 256) after W/U~ have been read out.
  constexpr uint32_t tmS = MODE == 0 ? kTmS : 256;
  constexpr uint32_t tmA = MODE == 0 ? kTmD1 : 0;  // A products (free columns during prep)
  const int q4 = warp & 3, ch = warp >> 2;  // TMEM lane quarter, column half
  const int srow = 32 * q4 + lane;          // dk row held by this thread

  // ---- initial state
  {
    const float* S0 = nullptr;
    if (MODE == 0)
      S0 = seg > 0 ? seg_sin(p.seg, n, h, H, p.P, seg)
                   : (p.S0 ? p.S0 + ((size_t)n * H + h) * kD * kD : nullptr);
    for (int c16 = 0; c16 < 64; c16 += 16) {
      float v16[16];
      const int col = 64 * ch + c16;
#pragma unroll
      for (int i = 0; i < 16; ++i) v16[i] = S0 ? S0[(size_t)srow * kD + col + i] : 0.f;
      tmem_st16(tmem_addr(tm, 32 * q4, tmS + col), v16);
#pragma unroll
      for (int i = 0; i < 16; i += 8)
        *reinterpret_cast<uint4*>(sm + kOffSb + mnm<(MODE == 0 ? 128 : 256)>(col + i, srow)) =
            pack8(v16 + i);
      if (MODE == 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) v16[i] = (col + i == srow) ? 1.f : 0.f;
        tmem_st16(tmem_addr(tm, 32 * q4, 384 + col), v16);
#pragma unroll
        for (int i = 0; i < 16; i += 8)
          *reinterpret_cast<uint4*>(sm + kOffSb + mnm<256>(128 + col + i, srow)) = pack8(v16 + i);
      }
    }
    tmem_st_wait();
  }

  const float expA = p.g ? 0.f : expf(p.A[h]);
  const int j = tid & 127, hf = tid >> 7;  // prep ownership: channel j, rows 32hf..32hf+31

  for (int c = c0; c < c1; ++c) {
    const int tok0 = a + c * kC;
    const int len = min(kC, b - tok0);
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    // ---- row norms, beta (one warp per 8 rows)
    for (int r = warp; r < kC; r += 8) {
      float sq = 0.f, sk = 0.f;
      if (r < len) {
        const size_t base = ((size_t)(tok0 + r) * H + h) * kD + 4 * lane;
        const uint2 qq = *reinterpret_cast<const uint2*>(p.q + base);
        const uint2 kk = *reinterpret_cast<const uint2*>(p.k + base);
        const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&qq);
        const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kk);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const float2 fq = __bfloat1622float2(q2[i]), fk = __bfloat1622float2(k2[i]);
          sq += fq.x * fq.x + fq.y * fq.y;
          sk += fk.x * fk.x + fk.y * fk.y;
        }
      }
      sq = warp_sum(sq);
      sk = warp_sum(sk);
      if (lane == 0) {
        vec[kVecIq + r] = r < len ? 1.0f / sqrtf(sq + kNormEps) : 0.f;
        vec[kVecIk + r] = r < len ? 1.0f / sqrtf(sk + kNormEps) : 0.f;
        vec[kVecBeta + r] = r < len ? __bfloat162float(p.beta[(size_t)(tok0 + r) * H + h]) : 0.f;
      }
    }
    // ---- gate and chunk-local cumsum for channel j, rows 32hf..32hf+31
    float E[32], kh[32], qh[32];
    {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int r = 32 * hf + i;
        float gv = 0.f;
        if (r < len) {
          const size_t idx = ((size_t)(tok0 + r) * H + h) * kD + j;
          gv = p.g ? p.g[idx] : gate_logdecay(__bfloat162float(p.z[idx]), expA);
          kh[i] = __bfloat162float(p.k[idx]);
          qh[i] = __bfloat162float(p.q[idx]);
        } else {
          kh[i] = 0.f;
          qh[i] = 0.f;
        }
        acc += gv;
        E[i] = acc;  // Gam (local to this half for now)
      }
      if (hf == 0) vec[kVecTot + j] = acc;
    }
    __syncthreads();
    {
      const float off = hf ? vec[kVecTot + j] : 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) E[i] += off;
      vec[kVecRho + (2 * hf) * 128 + j] = E[0];
      vec[kVecRho + (2 * hf + 1) * 128 + j] = E[16];
      if (hf == 1) vec[kVecGlast + j] = E[31];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int r = 32 * hf + i;
        kh[i] *= vec[kVecIk + r];
        qh[i] *= vec[kVecIq + r];
      }
    }
    __syncthreads();
    // E = e^{Gam_r - rho_b(r)}; per-channel factors
    float rho[4];
#pragma unroll
    for (int bb = 0; bb < 4; ++bb) rho[bb] = vec[kVecRho + bb * 128 + j];
    const float glast = vec[kVecGlast + j];
#pragma unroll
    for (int i = 0; i < 32; ++i) E[i] = expf(E[i] - (hf ? rho[2 + (i >> 4)] : rho[i >> 4]));

    // ---- product operands: R (rows) and C_b (columns per row sub-tile b)
    {
      unsigned char* R = sm + kOffR;
      unsigned char* Cm = sm + kOffC;
      const int cbase[4] = {0, 16, 48, 96};
      // F[t2][bb] = e^{rho_bb - rho_bt} for this half's sub-tiles bt = 2hf + t2
      float F[2][4];
#pragma unroll
      for (int t2 = 0; t2 < 2; ++t2)
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
          const float rb = hf ? rho[2 + t2] : rho[t2];
          F[t2][bb] = expf(rho[bb] - rb);
        }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int t2 = i >> 4, r = 32 * hf + i, bt = r >> 4, rr = r & 15;
        st_bf16(R, km128(32 * bt + rr, j), kh[i] * E[i]);
        st_bf16(R, km128(32 * bt + 16 + rr, j), qh[i] * E[i]);
        const float kinv = kh[i] / E[i];
#pragma unroll
        for (int bb = 0; bb < 4; ++bb)
          if (bb >= bt) st_bf16(Cm, km128(cbase[bb] + r, j), bb == bt ? kinv : kinv * F[t2][bb]);
      }
    }
    fence_async_smem();
    __syncthreads();
    {
      // ---- M1: four M=64 MMAs -> TMEM [256 + 32b, +32): cols 0-15 A_kk^T, 16-31 A_qk^T
      if (tid == 0) {
        fence_after_sync();
        constexpr uint32_t id = instr_desc(kFmtBF16, 64, 32, false, false);
        const int cbase[4] = {0, 16, 48, 96};
        for (int bb = 0; bb < 4; ++bb) {
          const uint32_t abase = smem_u32(sm + kOffC) + (cbase[bb] >> 3) * 2048;
          const uint32_t bbase = smem_u32(sm + kOffR) + (32 * bb >> 3) * 2048;
          for (int k = 0; k < 8; ++k)
            mma_bf16(tm + tmA + 32 * bb, smem_desc(abase + 256 * k, 128, 2048),
                     smem_desc(bbase + 256 * k, 128, 2048), id, k > 0);
        }
        mma_commit(&s_bar);
      }
      const bool got = mbar_wait_cycles(&s_bar, phase, kWaitCycles);
      phase ^= 1;
      if (__syncthreads_or(!got)) {
        if (tid == 0) { s_abort = 1; atomicOr(&p.hdr->err, kErrTimeout); }
        break;
      }
      fence_after_sync();
    }
    // ---- A_kk (fp32 smem, beta-scaled, strictly lower) and A_qk (bf16 into A3)
    float* Akk = reinterpret_cast<float*>(sm + kOffAkk);
    if (warp < 4) {
      const int i = 16 * warp + lane;  // valid for lane < 16
#pragma unroll 1
      for (int bb = 0; bb < 4; ++bb) {
        float va[16], vq[16];
        tmem_ld16(tmem_addr(tm, 32 * warp, tmA + 32 * bb), va);
        tmem_ld16(tmem_addr(tm, 32 * warp, tmA + 32 * bb + 16), vq);
        tmem_ld_wait();
        if (lane < 16) {
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) {
            const int r = 16 * bb + cc;
            Akk[r * 65 + i] = (i < r) ? vec[kVecBeta + r] * va[cc] : 0.f;
            if (MODE == 0) st_bf16(sm + kOffA3, km64(64 + r, i), (i <= r) ? vq[cc] : 0.f);
          }
        }
      }
    }
    fence_before_sync();
    __syncthreads();
    // ---- T = (I + A_kk)^{-1}: forward substitution on 16x16 diagonal blocks
    float* Tm = reinterpret_cast<float*>(sm + kOffT);
    float* Xs = vec + kVecX;
    for (int e = tid; e < kC * 65; e += kNT) Tm[e] = 0.f;
    __syncthreads();
    if (tid < kC) {
      const int r0 = (tid >> 4) << 4, col = tid;
      for (int r = r0; r < r0 + 16; ++r) {
        float x = (r == col) ? 1.f : 0.f;
        if (r > col)
          for (int i = col; i < r; ++i) x -= Akk[r * 65 + i] * Tm[i * 65 + col];
        Tm[r * 65 + col] = x;
      }
    }
    __syncthreads();
    // block rows below the diagonal: T_ba = -T_bb sum_{a<=c<b} A_bc T_ca
    for (int dist = 1; dist < 4; ++dist) {
      const int npairs = 4 - dist;
      for (int e = tid; e < npairs * 256; e += kNT) {
        const int pr = e >> 8, rr = (e >> 4) & 15, cc = e & 15, bb = pr + dist, aa = pr;
        float x = 0.f;
        for (int m = aa * 16; m < bb * 16; ++m) x += Akk[(bb * 16 + rr) * 65 + m] * Tm[m * 65 + aa * 16 + cc];
        Xs[e] = x;
      }
      __syncthreads();
      for (int e = tid; e < npairs * 256; e += kNT) {
        const int pr = e >> 8, rr = (e >> 4) & 15, cc = e & 15, bb = pr + dist, aa = pr;
        float y = 0.f;
        for (int m = 0; m < 16; ++m) y -= Tm[(bb * 16 + rr) * 65 + bb * 16 + m] * Xs[pr * 256 + m * 16 + cc];
        Tm[(bb * 16 + rr) * 65 + aa * 16 + cc] = y;
      }
      __syncthreads();
    }
    for (int e = tid; e < kC * kC; e += kNT) {
      const int r = e >> 6, i = e & 63;
      st_bf16(sm + kOffTp, km64(r, i), Tm[r * 65 + i]);
    }
    __syncthreads();  // T (fp32) is dead from here: region P holds [X_K | X_V] next

    // ---- WY / chain operands from registers: X_K, X_V, Q', K', gamma
    {
      float erho[2], elast[2];
#pragma unroll
      for (int t2 = 0; t2 < 2; ++t2) {
        const float rb = hf ? rho[2 + t2] : rho[t2];
        erho[t2] = expf(rb);
        elast[t2] = expf(glast - rb);
      }
      if (hf == 0) vec[kVecGam + j] = expf(glast);
      unsigned char* X = sm + kOffX;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int r = 32 * hf + i, t2 = i >> 4;
        const float bet = vec[kVecBeta + r];
        const float eg = E[i] * erho[t2];
        st_bf16(X, mnm<256>(j, r), bet * kh[i] * eg);
        const float vv = r < len ? __bfloat162float(p.v[((size_t)(tok0 + r) * H + h) * kD + j]) : 0.f;
        st_bf16(X, mnm<256>(128 + j, r), bet * vv);
        if (MODE == 0) st_bf16(sm + kOffA1, km128(64 + r, j), qh[i] * eg);
        st_bf16(sm + kOffKp, mnm<128>(j, r), (kh[i] / E[i]) * elast[t2]);
      }
    }
    fence_async_smem();
    __syncthreads();
    // ---- M2: [W | U~] = T_pad [X_K | X_V]  (M=128, N=256, K=64) -> TMEM [0, 256)
    if (tid == 0) {
      fence_after_sync();
      constexpr uint32_t id = instr_desc(kFmtBF16, 128, 256, false, true);
      const uint32_t abase = smem_u32(sm + kOffTp), bbase = smem_u32(sm + kOffX);
      for (int k = 0; k < 4; ++k)
        mma_bf16(tm + kTmWU, smem_desc(abase + 256 * k, 128, 1024),
                 smem_desc(bbase + 2 * 4096 * k, 4096, 128), id, k > 0);
      mma_commit(&s_bar);
    }
    {
      const bool got = mbar_wait_cycles(&s_bar, phase, kWaitCycles);
      phase ^= 1;
      if (__syncthreads_or(!got)) {
        if (tid == 0) { s_abort = 1; atomicOr(&p.hdr->err, kErrTimeout); }
        break;
      }
      fence_after_sync();
    }
    // ---- W -> bf16 A1 rows 0-63 (warps 0,1,4,5 hold TMEM lanes 0-63);
    //      U~ stays in TMEM columns [128, 256)
    float ut[64];
    if (q4 < 2) {
      const int r = srow;
#pragma unroll
      for (int c16 = 0; c16 < 64; c16 += 16) {
        float w16[16];
        tmem_ld16(tmem_addr(tm, 32 * q4, kTmWU + 64 * ch + c16), w16);
        float u16[16];
        tmem_ld16(tmem_addr(tm, 32 * q4, kTmWU + 128 + 64 * ch + c16), u16);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) ut[c16 + i] = u16[i];
#pragma unroll
        for (int i = 0; i < 16; i += 8)
          *reinterpret_cast<uint4*>(sm + kOffA1 + km128(r, 64 * ch + c16 + i)) = pack8(w16 + i);
      }
    }
    // ---- decay the state(s) by gamma = e^{Gam_last} (rows = dk = TMEM lanes)
    {
      const float gm = vec[kVecGam + srow];
      constexpr int NB = MODE == 0 ? 1 : 2;
#pragma unroll
      for (int blk = 0; blk < NB; ++blk)
#pragma unroll
        for (int c16 = 0; c16 < 64; c16 += 16) {
          float s16[16];
          const uint32_t col = tmS + 128 * blk + 64 * ch + c16;
          tmem_ld16(tmem_addr(tm, 32 * q4, col), s16);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) s16[i] *= gm;
          tmem_st16(tmem_addr(tm, 32 * q4, col), s16);
        }
      tmem_st_wait();
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    // ---- C1: D1 = A1 S  (M=128 [W;Q'] or M=64 W, K=128)
    //      MODE 0: N=128 -> TMEM [256, 384);  MODE 1: N=256 ([S|X]) -> TMEM [0, 256)
    if (tid == 0) {
      fence_after_sync();
      const uint32_t abase = smem_u32(sm + kOffA1), bbase = smem_u32(sm + kOffSb);
      if (MODE == 0) {
        constexpr uint32_t id = instr_desc(kFmtBF16, 128, 128, false, true);
        for (int k = 0; k < 8; ++k)
          mma_bf16(tm + kTmD1, smem_desc(abase + 256 * k, 128, 2048),
                   smem_desc(bbase + 2 * 2048 * k, 2048, 128), id, k > 0);
      } else {
        constexpr uint32_t id = instr_desc(kFmtBF16, 128, 256, false, true);
        for (int k = 0; k < 8; ++k)
          mma_bf16(tm + 0, smem_desc(abase + 256 * k, 128, 2048),
                   smem_desc(bbase + 2 * 4096 * k, 4096, 128), id, k > 0);
      }
      mma_commit(&s_bar);
    }
    {
      const bool got = mbar_wait_cycles(&s_bar, phase, kWaitCycles);
      phase ^= 1;
      if (__syncthreads_or(!got)) {
        if (tid == 0) { s_abort = 1; atomicOr(&p.hdr->err, kErrTimeout); }
        break;
      }
      fence_after_sync();
    }
    // ---- U = U~ - W S  (MODE 1: [U_S | U_X] = [U~ | 0] - W [S | X])
    if (q4 < 2) {
      const int r = srow;
      constexpr int NB = MODE == 0 ? 1 : 2;
#pragma unroll
      for (int blk = 0; blk < NB; ++blk)
#pragma unroll
        for (int c16 = 0; c16 < 64; c16 += 16) {
          float d16[16];
          const uint32_t col = (MODE == 0 ? kTmD1 : 0) + 128 * blk + 64 * ch + c16;
          tmem_ld16(tmem_addr(tm, 32 * q4, col), d16);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) d16[i] = (blk == 0 ? ut[c16 + i] : 0.f) - d16[i];
#pragma unroll
          for (int i = 0; i < 16; i += 8) {
            const int n = 128 * blk + 64 * ch + c16 + i;
            const uint32_t off = MODE == 0 ? mnm<128>(n, r) : mnm<256>(n, r);
            *reinterpret_cast<uint4*>(sm + kOffU + off) = pack8(d16 + i);
          }
        }
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    // ---- C2: S += K'^T U  (and O += A_qk U in MODE 0)
    if (tid == 0) {
      fence_after_sync();
      const uint32_t kb = smem_u32(sm + kOffKp), ub = smem_u32(sm + kOffU);
      if (MODE == 0) {
        constexpr uint32_t id = instr_desc(kFmtBF16, 128, 128, true, true);
        for (int k = 0; k < 4; ++k)
          mma_bf16(tm + kTmS, smem_desc(kb + 2 * 2048 * k, 2048, 128),
                   smem_desc(ub + 2 * 2048 * k, 2048, 128), id, 1);
        constexpr uint32_t id2 = instr_desc(kFmtBF16, 128, 128, false, true);
        const uint32_t a3 = smem_u32(sm + kOffA3);
        for (int k = 0; k < 4; ++k)
          mma_bf16(tm + kTmD1, smem_desc(a3 + 256 * k, 128, 1024),
                   smem_desc(ub + 2 * 2048 * k, 2048, 128), id2, 1);
      } else {
        constexpr uint32_t id = instr_desc(kFmtBF16, 128, 256, true, true);
        for (int k = 0; k < 4; ++k)
          mma_bf16(tm + 256, smem_desc(kb + 2 * 2048 * k, 2048, 128),
                   smem_desc(ub + 2 * 4096 * k, 4096, 128), id, 1);
      }
      mma_commit(&s_bar);
    }
    {
      const bool got = mbar_wait_cycles(&s_bar, phase, kWaitCycles);
      phase ^= 1;
      if (__syncthreads_or(!got)) {
        if (tid == 0) { s_abort = 1; atomicOr(&p.hdr->err, kErrTimeout); }
        break;
      }
      fence_after_sync();
    }
    // ---- S (and X) -> bf16 operand for the next chunk; O -> global
    {
      constexpr int NB = MODE == 0 ? 1 : 2;
#pragma unroll
      for (int blk = 0; blk < NB; ++blk)
#pragma unroll
        for (int c16 = 0; c16 < 64; c16 += 16) {
          float s16[16];
          const int col = 128 * blk + 64 * ch + c16;
          tmem_ld16(tmem_addr(tm, 32 * q4, tmS + col), s16);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; i += 8) {
            const uint32_t off = MODE == 0 ? mnm<128>(col + i, srow) : mnm<256>(col + i, srow);
            *reinterpret_cast<uint4*>(sm + kOffSb + off) = pack8(s16 + i);
          }
        }
      if (MODE == 0 && q4 >= 2) {
        const int r = srow - 64;
#pragma unroll
        for (int c16 = 0; c16 < 64; c16 += 16) {
          float o16[16];
          tmem_ld16(tmem_addr(tm, 32 * q4, kTmD1 + 64 * ch + c16), o16);
          tmem_ld_wait();
          if (r < len) {
            uint4* dst = reinterpret_cast<uint4*>(p.o + ((size_t)(tok0 + r) * H + h) * kD + 64 * ch + c16);
            dst[0] = pack8(o16);
            dst[1] = pack8(o16 + 8);
          }
        }
      }
    }
  }

  // ---- results
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (!s_abort) {
    if (MODE == 0) {
      if (p.S_final && seg == p.P - 1) {
        float* dst = p.S_final + ((size_t)n * H + h) * kD * kD + (size_t)srow * kD;
#pragma unroll
        for (int c16 = 0; c16 < 64; c16 += 16) {
          float s16[16];
          tmem_ld16(tmem_addr(tm, 32 * q4, tmS + 64 * ch + c16), s16);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(dst + 64 * ch + c16 + i) = make_float4(s16[i], s16[i + 1], s16[i + 2], s16[i + 3]);
        }
      }
    } else {
      // transition: M (from X, columns 384..511) and N (from S, columns 256..383)
      float* Mt = seg_trans(p.seg, n, h, H, p.P, seg);
      float* Nt = Mt + kD * kD;
#pragma unroll
      for (int blk = 0; blk < 2; ++blk)
#pragma unroll
        for (int c16 = 0; c16 < 64; c16 += 16) {
          float s16[16];
          tmem_ld16(tmem_addr(tm, 32 * q4, 256 + 128 * blk + 64 * ch + c16), s16);
          tmem_ld_wait();
          float* dst = (blk == 0 ? Nt : Mt) + (size_t)srow * kD + 64 * ch + c16;
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(dst + i) = make_float4(s16[i], s16[i + 1], s16[i + 2], s16[i + 3]);
        }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, 512);
}

// Incoming state of every segment: S_in(0) = S0, S_in(p+1) = M_p S_in(p) + N_p.
// One CTA per (n, h, 16-column block of the state); fp32 on CUDA cores.
__global__ void __launch_bounds__(256) compose_kernel(TcParams p) {
  const int n = blockIdx.x, h = blockIdx.y, cb = blockIdx.z * 16;
  const int H = p.H;
  if (!seqlens_valid(p.cu, p.N, p.T, p.max_len)) return;
  __shared__ float Sc[kD][16];
  __shared__ float Mrow[8][kD];
  const int tid = threadIdx.x;
  for (int e = tid; e < kD * 16; e += 256) {
    const int r = e >> 4, c = e & 15;
    Sc[r][c] = p.S0 ? p.S0[((size_t)n * H + h) * kD * kD + (size_t)r * kD + cb + c] : 0.f;
  }
  __syncthreads();
  for (int sg = 0; sg + 1 < p.P; ++sg) {
    const float* Mt = seg_trans(p.seg, n, h, H, p.P, sg);
    const float* Nt = Mt + kD * kD;
    // thread: column c = tid & 15, rows r = tid >> 4 + 16 m
    float acc[8];
    const int c = tid & 15, r0 = tid >> 4;
#pragma unroll
    for (int m = 0; m < 8; ++m) acc[m] = Nt[(size_t)(r0 + 16 * m) * kD + cb + c];
    for (int k0 = 0; k0 < kD; k0 += 8) {
      __syncthreads();
      for (int e = tid; e < 8 * kD; e += 256) {
        const int kk = e >> 7, r = e & 127;
        Mrow[kk][r] = Mt[(size_t)r * kD + k0 + kk];  // column k0+kk of M
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const float s = Sc[k0 + kk][c];
#pragma unroll
        for (int m = 0; m < 8; ++m) acc[m] += Mrow[kk][r0 + 16 * m] * s;
      }
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < 8; ++m) Sc[r0 + 16 * m][c] = acc[m];
    __syncthreads();
    float* Sin = seg_sin(p.seg, n, h, H, p.P, sg + 1);
    for (int e = tid; e < kD * 16; e += 256) {
      const int r = e >> 4, cc = e & 15;
      Sin[(size_t)r * kD + cb + cc] = Sc[r][cc];
    }
  }
}

}  // namespace

bool tc_supported(const ForwardArgs& a) {
  return a.bf16 && a.dk == kD && a.dv == kD && a.chunk == kC;
}

int tc_segments(int N, int H, int max_len) {
  // enough (sequence, head, segment) CTAs to fill the 148 SMs; long sequences only
  const int pairs = N * H;
  int P = pairs >= 128 ? 1 : 148 / pairs;
  const int nch = (max_len + kC - 1) / kC;
  if (P > nch / 2) P = nch / 2;
  if (P < 1) P = 1;
  if (P > 16) P = 16;
  return P;
}

size_t tc_workspace_bytes(int N, int T, int H, int max_len) {
  const int P = tc_segments(N, H, max_len);
  size_t per = (size_t)(P - 1) * 2 * kD * kD + (size_t)P * kD * kD;
  return sizeof(WsHeader) + (size_t)N * H * per * sizeof(float);
}

int tc_launches(int N, int H, int max_len) {
  if (N <= 0) return 0;
  return tc_segments(N, H, max_len) > 1 ? 3 : 1;
}

cudaError_t launch_forward_tc(const ForwardArgs& a) {
  TcParams p;
  p.q = (const __nv_bfloat16*)a.q;
  p.k = (const __nv_bfloat16*)a.k;
  p.v = (const __nv_bfloat16*)a.v;
  p.z = (const __nv_bfloat16*)a.z;
  p.beta = (const __nv_bfloat16*)a.beta;
  p.A = a.A;
  p.g = a.g;
  p.S0 = a.S0;
  p.cu = a.cu;
  p.o = (__nv_bfloat16*)a.o;
  p.S_final = a.S_final;
  p.N = a.N;
  p.T = a.T;
  p.max_len = a.max_len;
  p.H = a.H;
  p.P = tc_segments(a.N, a.H, a.max_len);
  p.hdr = (WsHeader*)a.ws;
  p.seg = (float*)((char*)a.ws + sizeof(WsHeader));
  cudaError_t err;
  if (p.P > 1) {
    err = cudaFuncSetAttribute(tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    tc_kernel<1><<<dim3(a.N, a.H, p.P - 1), kNT, kSmemBytes, a.stream>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    compose_kernel<<<dim3(a.N, a.H, kD / 16), 256, 0, a.stream>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  err = cudaFuncSetAttribute(tc_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (err != cudaSuccess) return err;
  tc_kernel<0><<<dim3(a.N, a.H, p.P), kNT, kSmemBytes, a.stream>>>(p);
  return cudaGetLastError();
}

}  // namespace kda
