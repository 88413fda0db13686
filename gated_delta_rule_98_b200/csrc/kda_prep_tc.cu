// kda_prep_tc.cu -- chunk preparation of the tensor-core KDA prefill (sm_100a):
// everything of one (chunk, head) that does not depend on the state, left in
// the chunk's slot for the chain passes (kda_prefill_tc.cu).
//
// Kimi Linear summary §3.1 (chunkwise WY / UT form: per-chunk cumulative
// log-decay, the lower-triangular inverse by forward substitution, W and U~),
// §3.2 (16-token sub-chunks keep the channel-wise decay factors in range).
// Per 64-token chunk, with alpha = e^g the per-token, per-channel decay and
// Gam the chunk-local inclusive cumulative log-decay:
//
//   A_kk[r][i] = beta_r sum_j k^_rj k^_ij e^{Gam_rj - Gam_ij}   (i < r)
//   A_qk[r][i] =        sum_j q_rj  k^_ij e^{Gam_rj - Gam_ij}   (i <= r)
//   T   = (I + A_kk)^{-1}
//   W   = T (Diag(beta) K^ e^{Gam})       U~ = T Diag(beta) V
//   Q'  = q e^{Gam},  K' = k^ e^{Gam_last - Gam},  gamma = e^{Gam_last}
//
// (k^ = k / |k|; q stays unnormalised and 1/|q| scales the output rows.)
// The products are formed per 16-token row sub-tile b with the reference
// rho_b = Gam at the sub-tile's first token: the row operand carries
// E = e^{Gam_r - rho_b} <= 1, the column operand ("window" b, every token up
// to the end of sub-tile b) carries e^{rho_b - Gam_i} (<= e^75 on the diagonal
// sub-tile, <= 1 before it).  The decay factors are cumulative products of
// alpha inside a sub-tile (16 tokens x alpha >= e^-5 stays above e^-80).
//
// Thread layout of the elementwise phases: thread (channel j, sub-tile b),
// 512 threads; the 16 tokens of a sub-tile are a serial product in registers
// and every operand image unit (8 consecutive tokens of one channel) is one
// 16-byte store.  Persistent: one CTA per SM walks (chunk, sequence, head)
// items.  q, k, z rows are double-buffered: an item's rows are requested two
// items ahead, as soon as the buffer's previous item has read them (one item
// ahead, single-buffered, with the input prologue); v rows are requested as
// soon as the WY product that reads them has completed.
#include <type_traits>

#include "kda_tc_common.cuh"

namespace kda {
namespace tcp {
namespace {

constexpr int kLd = 68;  // row stride (floats) of the fp32 work matrices of the inverse

// Windows: window w (the column operand of row sub-tile w) holds the 16 (w + 1)
// tokens of sub-tiles 0 .. w and starts at row 8 w (w + 1) of one 160-row image.
__host__ __device__ constexpr int win_row0(int w) { return 8 * w * (w + 1); }
constexpr int kWinRows = 160;

// CV: the input prologue runs here (q, k, v arrive before their short
// convolution and Swish).  Their boxes then start 8 tokens before the chunk,
// so box row 8 + t holds token t and rows 5 .. 7 the convolution's history.
template <bool CV>
struct PrepSmem {
  // staged rows: per tensor two 64-channel boxes of kRows tokens, 128-byte swizzle.
  // q, k, z rows are double-buffered (kNQ buffers of kQKZ bytes: an item's rows
  // are requested two items ahead) where shared memory allows, i.e. without the
  // prologue; v rows have one buffer.
  static constexpr int kRows = CV ? kC + 8 : kC;
  static constexpr int kBox = kRows * 128;
  static constexpr int kNQ = CV ? 1 : 2;
  static constexpr int kQKZ = 4 * kBox + 16384;
  static constexpr int kQ = 0, kK = 2 * kBox, kZ = 4 * kBox;  // in buffer 0 (+ kQKZ: buffer 1)
  static constexpr int kV = kNQ * kQKZ;
  static constexpr int kWB = kV + 2 * kBox;        // windows, 160-row image: the B operand of M1
  static constexpr int kR = kWB + kWinRows * 256; // R: 128-row image (sub-tile b: k rows 32b..,
                                                  //   q rows 32b+16..), the A operand of M1
  // after M1 the window / R region holds the inverse's work and the T images
  static constexpr int kAf = kWB;                 // A_kk fp32 [64][kLd], row r, column i
  static constexpr int kAT = kAf + 64 * kLd * 4;  // merge products, transposed [64][kLd]
  static constexpr int kTf = kAT + 64 * kLd * 4;  // T fp32 [64][kLd]
  static constexpr int kTT = kTf + 64 * kLd * 4;  // T^T fp32 [64][kLd]
  static constexpr int kTb = kTT + 64 * kLd * 4;  // T, the B operand T^T of M2 (64-row f16 image)
  static constexpr int kTbb = kTb + 8192;         // T Diag(beta), the same for U~ (bf16, with V)
  static constexpr int kXK = kTbb + 8192;         // X_K: 64-row f16 image, the A operand X_K^T of M2
  static constexpr int kNrm = kXK + 16384;        // 1/|q| (64), 1/|k| (64)
  static constexpr int kBeta = kNrm + 512;        // beta (64)
  static constexpr int kGh = kBeta + 256;         // the scalar gate's log-decay of each token (64)
  static constexpr int kEx = kGh + 256;           // [4][128] alpha at each sub-tile's first token,
                                                  // then [4][128] E at its last token
  // CV: the prologue's taps (x 1/2) of the item's head and of the next item's,
  // [2][q, k, v][128 channels] float4 (right-aligned: the last on the current token)
  static constexpr int kTaps = kEx + 4096;
  // CV: a 16 x 16 bf16 block of ones, the B operand of the norm product
  static constexpr int kOnes = kTaps + (CV ? 12288 : 0);
  // CV: Swish(conv(v)) as a 64-row bf16 image, the A operand V^T of M2 (K-major)
  static constexpr int kVc = kOnes + (CV ? 512 : 0);
  static constexpr int kBar = kVc + (CV ? 16384 : 0);  // four mbarriers, then the TMEM base
  static constexpr int kBytes = kBar + 64;
  // CV, before M1: squares of q, k (hi and lo bf16 parts), a 128-row image with
  // 256 channels over the window / R region: the A operand of the norm product
  static constexpr int kSq = kWB;
  static_assert(kSq + 65536 <= kXK, "norm operand overlaps X_K");
  static_assert(kR + 32768 <= kXK, "M1 operands overlap X_K");
  static_assert(kBox % 1024 == 0 && kQKZ % 1024 == 0 && kV % 1024 == 0,
                "swizzled boxes need 1024-byte alignment");
  static_assert(kBytes <= 232448, "shared memory per CTA");
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
constexpr float kLog2e = 1.4426950408889634f;
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Shared-memory matrix descriptor with the 128-byte swizzle (the layout TMA
// writes with CU_TENSOR_MAP_SWIZZLE_128B into a 1024-byte aligned buffer).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return smem_desc(saddr, lbo, sbo) | ((uint64_t)2u << 61);
}

// y = a * b and y = a * s over 16 values, in packed fp32x2 pairs
__device__ __forceinline__ void mul16(float* y, const float* a, const float* b) {
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const float2 r = __fmul2_rn(make_float2(a[i], a[i + 1]), make_float2(b[i], b[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  }
}
__device__ __forceinline__ void scale16(float* y, const float* a, float s) {
  const float2 s2 = make_float2(s, s);
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const float2 r = __fmul2_rn(make_float2(a[i], a[i + 1]), s2);
    y[i] = r.x;
    y[i + 1] = r.y;
  }
}
// 16 consecutive fp32 from shared memory (64-byte aligned)
__device__ __forceinline__ void lds16(const float* p, float* y) {
#pragma unroll
  for (int i = 0; i < 16; i += 4) {
    const float4 v = *reinterpret_cast<const float4*>(p + i);
    y[i] = v.x; y[i + 1] = v.y; y[i + 2] = v.z; y[i + 3] = v.w;
  }
}

// 16 fp32 values of 16 consecutive tokens -> two units of a bf16 operand image
__device__ __forceinline__ void put16(unsigned char* base, uint32_t unit0, uint32_t unit1,
                                      const float* v) {
  *reinterpret_cast<uint4*>(base + unit0) = pack8(v);
  *reinterpret_cast<uint4*>(base + unit1) = pack8(v + 8);
}
// the same for an f16 image (the chain operands)
__device__ __forceinline__ void put16h(unsigned char* base, uint32_t unit0, uint32_t unit1,
                                       const float* v) {
  *reinterpret_cast<uint4*>(base + unit0) = pack8h(v);
  *reinterpret_cast<uint4*>(base + unit1) = pack8h(v + 8);
}

template <int GS, bool CV>
__global__ void __launch_bounds__(kNT, 1) prep_kernel(const __grid_constant__ TcParams p) {
  using L = PrepSmem<CV>;
  extern __shared__ __align__(1024) unsigned char sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* nrm = reinterpret_cast<float*>(sm + L::kNrm);
  float* bvec = reinterpret_cast<float*>(sm + L::kBeta);
  float* ghv = reinterpret_cast<float*>(sm + L::kGh);
  float* exf = reinterpret_cast<float*>(sm + L::kEx);
  float* exl = exf + 512;
  uint64_t* bar_qkz = reinterpret_cast<uint64_t*>(sm + L::kBar);  // one per q, k, z buffer
  uint64_t* bar_v = bar_qkz + 2;
  uint64_t* bar_mma = bar_qkz + 3;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bar_qkz + 4);
  const int H = p.H;

  if (!seqlens_valid(p.cu, p.N, p.T, p.max_len)) {
    if (blockIdx.x == 0 && tid == 0) atomicOr(&p.hdr->err, kErrBadSeqlens);
    return;
  }
  // the 128-byte swizzle needs 1024-byte aligned destinations
  if (smem_u32(sm) & 1023u) {
    if (tid == 0) atomicOr(&p.hdr->err, kErrTimeout);
    return;
  }
  if (warp == 0) {
    tmem_alloc(s_tmem, 256);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_qkz, 1);
    mbar_init(bar_qkz + 1, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = *s_tmem;
  uint32_t ph_qkz = 0, ph_v = 0, ph_mma = 0;  // ph_qkz bit s: parity of buffer s's next load
  uint32_t qkz_pending = 0;                    // bit s: buffer s being filled
  bool ok = true, v_pending = false, mma_pending = false;

  // elementwise phases: channel j, sub-tile b (tokens 16 b .. 16 b + 15)
  const int j = tid & 127, b = tid >> 7;
  // TMEM phases: lane quarter q4, column group cq
  const int q4 = warp & 3, cq = warp >> 2;
  // byte offset of (token 16 b + i, channel j) in a staged swizzled tile: box
  // j / 64, row t, 16-byte unit ((j % 64) / 8) ^ (t % 8), element j % 8
  const uint32_t jbox = (uint32_t)(j >> 6) * 8192u + (uint32_t)(j & 7) * 2u;
  const uint32_t junit = (uint32_t)((j & 63) >> 3);
  auto raw_off = [&](int i) -> uint32_t {
    return jbox + (uint32_t)(16 * b + i) * 128u + ((junit ^ (uint32_t)(i & 7)) << 4);
  };
  auto raw_f = [&](int base, int i) -> float {
    const uint32_t u = *reinterpret_cast<const uint16_t*>(sm + base + raw_off(i));
    return __uint_as_float(u << 16);
  };
  // CV: input prologue of channel j, tokens 16 b .. 16 b + 15 (box row 8 + t holds token t):
  // y_i = Swish(sum_m w4[m] x[16 b + i - 3 + m]), the taps w4 right-aligned (w4[3] on
  // the current token); history before the sequence's first token reads as zero
  // (first: this chunk is its sequence's first), tokens from len on give zero
  // Token pairs (16 b + 2 p, 16 b + 2 p + 1) go through packed fp32x2 arithmetic;
  // the taps hw are halved, so the sum is h = u / 2 and, with sigmoid(u) =
  // (1 + tanh(u / 2)) / 2, Swish(u) = u sigmoid(u) = h + h tanh(h).
  const uint32_t jboxc = (uint32_t)(j >> 6) * (uint32_t)L::kBox + (uint32_t)(j & 7) * 2u;
  auto conv16 = [&](int base, const float4 hw, bool first, int len, float* y) {
    float x[19];  // tokens 16 b - 3 .. 16 b + 15
#pragma unroll
    for (int i = 0; i < 19; ++i) {
      const int r = 16 * b + 5 + i;
      const uint32_t off = jboxc + (uint32_t)r * 128u + ((junit ^ (uint32_t)(r & 7)) << 4);
      x[i] = __uint_as_float((uint32_t)*reinterpret_cast<const uint16_t*>(sm + base + off) << 16);
    }
    if (first && b == 0) x[0] = x[1] = x[2] = 0.f;
    const float2 w0 = make_float2(hw.x, hw.x), w1 = make_float2(hw.y, hw.y),
                 w2 = make_float2(hw.z, hw.z), w3 = make_float2(hw.w, hw.w);
#pragma unroll
    for (int q2 = 0; q2 < 8; ++q2) {
      const int i = 2 * q2;
      float2 h = __fmul2_rn(w0, make_float2(x[i], x[i + 1]));
      h = __ffma2_rn(w1, make_float2(x[i + 1], x[i + 2]), h);
      h = __ffma2_rn(w2, make_float2(x[i + 2], x[i + 3]), h);
      h = __ffma2_rn(w3, make_float2(x[i + 3], x[i + 4]), h);
      const float2 s = __ffma2_rn(h, make_float2(tanh_approx(h.x), tanh_approx(h.y)), h);
      y[i] = s.x;
      y[i + 1] = s.y;
    }
    if (len < kC) {
#pragma unroll
      for (int i = 0; i < 16; ++i) y[i] = 16 * b + i < len ? y[i] : 0.f;
    }
  };
  // CV: Swish(conv(v)) of channel j, tokens t0 .. t0 + N - 1 (t0 a multiple of 8)
  // into the bf16 image V^T of M2, from the staged rows (history and tail as in
  // conv16); run by the warps that the diagonal solve leaves idle, in three token
  // groups of 24, 24 and 16
  auto conv_v = [&](auto n_tokens, int t0, const float4 hw, bool first, int len) {
    constexpr int N = decltype(n_tokens)::value;
    float x[N + 3];
#pragma unroll
    for (int i = 0; i < N + 3; ++i) {
      const int r = t0 + 5 + i;
      const uint32_t off = jboxc + (uint32_t)r * 128u + ((junit ^ (uint32_t)(r & 7)) << 4);
      x[i] = __uint_as_float((uint32_t)*reinterpret_cast<const uint16_t*>(sm + L::kV + off) << 16);
    }
    if (first && t0 == 0) x[0] = x[1] = x[2] = 0.f;
    float y[N];
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const float h = fmaf(hw.w, x[i + 3], fmaf(hw.z, x[i + 2], fmaf(hw.y, x[i + 1], hw.x * x[i])));
      y[i] = t0 + i < len ? fmaf(h, tanh_approx(h), h) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < N / 8; ++u)
      *reinterpret_cast<uint4*>(sm + L::kVc + img_unit(t0 + 8 * u, j, 64)) = pack8(y + 8 * u);
  };
  // CV: taps of head hh for thread (j, b < 3): tensor b (q, k, v), channel j; the
  // loads are not waited for until the taps are stored, halved (store_taps)
  float4* tapbuf = reinterpret_cast<float4*>(sm + L::kTaps);
  auto load_taps = [&](int hh) -> float4 {
    const float* wc = (b == 0 ? p.cwq : b == 1 ? p.cwk : p.cwv) + (size_t)(hh * kD + j) * p.cw;
    float w[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) w[m] = m >= 4 - p.cw ? wc[m - (4 - p.cw)] : 0.f;
    return make_float4(w[0], w[1], w[2], w[3]);
  };
  auto store_taps = [&](int buf, float4 w) {
    tapbuf[buf * 384 + b * 128 + j] = make_float4(0.5f * w.x, 0.5f * w.y, 0.5f * w.z, 0.5f * w.w);
  };
  // CV: squares of y (16 tokens of channel j at rows r0 ..) as hi and lo bf16
  // parts (hi = bf16(y^2), lo = bf16(y^2 - hi)) into the norm operand: hi at
  // channel j, lo at channel 128 + j
  auto put_squares = [&](const float* y, int r0) {
    float s[16], lo[16];
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const float2 q2 = __fmul2_rn(make_float2(y[i], y[i + 1]), make_float2(y[i], y[i + 1]));
      s[i] = q2.x;
      s[i + 1] = q2.y;
    }
    const uint4 h0 = pack8(s), h1 = pack8(s + 8);
    float hf[16];
    unpack8(h0, hf);
    unpack8(h1, hf + 8);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const float2 d = __fadd2_rn(make_float2(s[i], s[i + 1]), make_float2(-hf[i], -hf[i + 1]));
      lo[i] = d.x;
      lo[i + 1] = d.y;
    }
    *reinterpret_cast<uint4*>(sm + L::kSq + img_unit(r0, j, 128)) = h0;
    *reinterpret_cast<uint4*>(sm + L::kSq + img_unit(r0 + 8, j, 128)) = h1;
    *reinterpret_cast<uint4*>(sm + L::kSq + img_unit(r0, 128 + j, 128)) = pack8(lo);
    *reinterpret_cast<uint4*>(sm + L::kSq + img_unit(r0 + 8, 128 + j, 128)) = pack8(lo + 8);
  };

  // items (chunk c, sequence n, head h), heads fastest; the CTA takes every
  // gridDim.x-th one, stepping the mixed-radix index without divisions
  const int maxch = (p.max_len + kC - 1) / kC;
  const long long it0 = blockIdx.x, stride = gridDim.x;
  const int sh = (int)(stride % H), sn = (int)((stride / H) % p.N);
  const int sc = (int)(stride / ((long long)H * p.N));
  struct Item { int h, n, c, a, e; };  // head, sequence, chunk; token range [a, e) of n
  auto step = [&](Item& s) {
    s.h += sh;
    if (s.h >= H) { s.h -= H; ++s.n; }
    s.n += sn;
    if (s.n >= p.N) { s.n -= p.N; ++s.c; }
    s.c += sc;
  };
  auto seek = [&](Item& s) -> bool {  // the first item from s on that holds tokens
    for (; s.c < maxch;) {
      seq_bounds(p.cu, s.n, p.max_len, s.a, s.e);
      if (s.a + s.c * kC < s.e) return true;
      step(s);
    }
    return false;
  };
  constexpr int kHist = CV ? 8 : 0;  // box rows before the chunk
  auto stage_qkz = [&](int s, int tok, int hh) {  // one thread; buffer s
    unsigned char* d = sm + s * L::kQKZ;
    mbar_arrive_expect_tx(bar_qkz + s, 4 * L::kBox + (GS == kGateZ ? 16384 : 0));
    tma_box_x(d + L::kQ, &p.sq, 0, hh, tok - kHist, bar_qkz + s);
    tma_box_x(d + L::kQ + L::kBox, &p.sq, 64, hh, tok - kHist, bar_qkz + s);
    tma_box_x(d + L::kK, &p.sk, 0, hh, tok - kHist, bar_qkz + s);
    tma_box_x(d + L::kK + L::kBox, &p.sk, 64, hh, tok - kHist, bar_qkz + s);
    if (GS == kGateZ) {
      tma_box_x(d + L::kZ, &p.sz, 0, hh, tok, bar_qkz + s);
      tma_box_x(d + L::kZ + 8192, &p.sz, 64, hh, tok, bar_qkz + s);
    }
  };
  auto stage_v = [&](int tok, int hh) {  // one thread
    mbar_arrive_expect_tx(bar_v, 2 * L::kBox);
    tma_box_x(sm + L::kV, &p.sv, 0, hh, tok - kHist, bar_v);
    tma_box_x(sm + L::kV + L::kBox, &p.sv, 64, hh, tok - kHist, bar_v);
  };
  // beta of an item's token t = tid < 64 as raw bf16 bits (converted when used, so
  // the load is not waited for until the next item)
  auto load_beta = [&](int tok, int end, int hh) -> uint32_t {
    return (tid < kC && tok + tid < end)
               ? (uint32_t)reinterpret_cast<const uint16_t*>(p.beta)[(size_t)(tok + tid) * H + hh]
               : 0u;
  };

  // the current item, the next one and (two buffers) the one after
  Item cur{(int)(it0 % H), (int)((it0 / H) % p.N), (int)(it0 / ((long long)H * p.N)), 0, 0};
  bool have = seek(cur);
  Item nx = cur;
  bool have_nx = false;
  if (have) {
    step(nx);
    have_nx = seek(nx);
  }
  uint32_t beta_nx = 0u;
  // the scalar gate of an item's token tid < 64, loaded an item ahead like beta
  auto load_gh = [&](int tok, int end, int hh) -> float {
    return (GS == kGateHead && tid < kC && tok + tid < end) ? p.g[(size_t)(tok + tid) * H + hh] : 0.f;
  };
  float gh_nx = 0.f;
  // A_h of the next item's head, loaded an item ahead
  float a_nx = (GS == kGateZ && have) ? p.A[cur.h] : 0.f;
  if (have) {
    if (tid == 0) {
      stage_qkz(0, cur.a + cur.c * kC, cur.h);
      if (L::kNQ == 2 && have_nx) stage_qkz(1, nx.a + nx.c * kC, nx.h);
      stage_v(cur.a + cur.c * kC, cur.h);
    }
    qkz_pending = (L::kNQ == 2 && have_nx) ? 3u : 1u;
    v_pending = true;
    beta_nx = load_beta(cur.a + cur.c * kC, cur.e, cur.h);
    gh_nx = load_gh(cur.a + cur.c * kC, cur.e, cur.h);
  }
  int qs = 0;  // the q, k, z buffer of the current item
  int tbuf = 0;  // CV: the taps buffer of the current item
  if constexpr (CV) {
    // the ones block (bf16 1.0) and the first item's taps; published by the
    // first item's first block-wide wait
    if (tid < 128) reinterpret_cast<uint32_t*>(sm + L::kOnes)[tid] = 0x3F803F80u;
    if (have && b < 3) store_taps(0, load_taps(cur.h));
  }
  while (have) {
    const int hc = cur.h, nc = cur.n, ac = cur.a, ec = cur.e, cc0 = cur.c;
    // the item after the next: its q, k, z rows go to this item's buffer
    Item nx2 = nx;
    bool have_nx2 = false;
    if (L::kNQ == 2 && have_nx) {
      step(nx2);
      have_nx2 = seek(nx2);
    }
    const int tok0 = ac + cc0 * kC;
    const int len = min(kC, ec - tok0);
    const int tokn = have_nx ? nx.a + nx.c * kC : 0, hn = nx.h;
    const int qb = qs * L::kQKZ;  // byte offset of this item's q, k, z buffer
    unsigned char* slot = chunk_slot(p.prep, ac, nc, cc0, hc, H);
    if (tid < kC) bvec[tid] = __uint_as_float(beta_nx << 16);
    if (GS == kGateHead && tid < kC) ghv[tid] = gh_nx;
    if (have_nx) {
      beta_nx = load_beta(tokn, nx.e, hn);
      gh_nx = load_gh(tokn, nx.e, hn);
    }

    // per-channel gate input, issued before the wait
    float al[16];  // alpha of tokens 16 b + i (then 1 / E)
    if constexpr (GS == kGateChannel) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = 16 * b + i;
        al[i] = t < len ? p.g[((size_t)(tok0 + t) * H + hc) * kD + j] : 0.f;
      }
    }
    const float expA_l2 = GS == kGateZ ? expf(a_nx) * kLog2e : 0.f;
    if (GS == kGateZ && have_nx) a_nx = p.A[hn];

    {
      uint32_t ph = (ph_qkz >> qs) & 1u;
      if (!block_wait(bar_qkz + qs, ph, p.hdr, p.wait_limit)) { ok = false; break; }
      ph_qkz ^= 1u << qs;
      qkz_pending &= ~(1u << qs);
    }

    float qv[16], kv[16];  // q, k of the thread's tokens (zero past the sequence end)
    if constexpr (CV) {
      // ---- A0: input prologue on q and k; their squares (hi + lo bf16 parts)
      //      go to one product with a block of ones, D[row][.] = sum over the
      //      channels (rows 0-63 q, 64-127 k), read after the gate
      const float4* tq = tapbuf + tbuf * 384;
      conv16(L::kQ + qb, tq[j], cc0 == 0, len, qv);
      put_squares(qv, 16 * b);
      conv16(L::kK + qb, tq[128 + j], cc0 == 0, len, kv);
      put_squares(kv, 64 + 16 * b);
      sync_for_mma();
      if (tid == 0) {
        constexpr uint32_t id = instr_desc(kFmtBF16, 128, 16, true, true);
        const uint64_t bd = smem_desc(smem_u32(sm + L::kOnes), 256, 128);
#pragma unroll
        for (int k = 0; k < 16; ++k)
          mma_bf16(tm + 160, smem_desc(smem_u32(sm + L::kSq + k * 4096), 2048, 128), bd, id, k > 0);
        mma_commit(bar_mma);
      }
      mma_pending = true;
    } else {
      // ---- A1: row norms (thread: row tid / 4 of [q ; k], 32 channels)
      const int r = tid >> 2, qt = tid & 3, t = r & 63;
      const unsigned char* rowp =
          sm + qb + (r < 64 ? L::kQ : L::kK) + (qt >> 1) * 8192 + t * 128;
      float ss = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t un = (uint32_t)(4 * (qt & 1) + u) ^ (uint32_t)(t & 7);
        float f[8];
        unpack8(*reinterpret_cast<const uint4*>(rowp + (un << 4)), f);
#pragma unroll
        for (int x = 0; x < 8; ++x) ss = fmaf(f[x], f[x], ss);
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      ss += __shfl_xor_sync(0xffffffffu, ss, 2);
      if (qt == 0) nrm[r] = t < len ? rsqrtf(ss + kNormEps) : 0.f;
    }
    // ---- A2: gate -> alpha; E = e^{Gam - rho_b} (E = 1 at the sub-tile's first token)
    if constexpr (GS == kGateZ) {
      const float2 nA = make_float2(-expA_l2, -expA_l2), one = make_float2(1.0f, 1.0f),
                   c5 = make_float2(kGateMin * kLog2e, kGateMin * kLog2e);
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        const float2 m = __fmul2_rn(make_float2(raw_f(L::kZ + qb, i), raw_f(L::kZ + qb, i + 1)), nA);
        const float2 d = __fadd2_rn(make_float2(ex2(m.x), ex2(m.y)), one);  // 1 + e^{-e^A z}
        const float2 s = __fmul2_rn(make_float2(rcp(d.x), rcp(d.y)), c5);   // -5 log2e sigmoid
        al[i] = ex2(s.x);                                                   // e^{-5 sigmoid}
        al[i + 1] = ex2(s.y);
      }
      if (len < kC) {
#pragma unroll
        for (int i = 0; i < 16; ++i) al[i] = 16 * b + i < len ? al[i] : 1.0f;
      }
    } else {
      if constexpr (GS == kGateHead) lds16(ghv + 16 * b, al);  // zero past the sequence end
#pragma unroll
      for (int i = 0; i < 16; ++i) al[i] = ex2(al[i] * kLog2e);  // masked tokens: g = 0
    }
    float E[16];
    E[0] = 1.0f;
#pragma unroll
    for (int i = 1; i < 16; ++i) E[i] = E[i - 1] * al[i];
    exf[b * 128 + j] = al[0];
    exl[b * 128 + j] = E[15];
    if constexpr (CV) {
      if (!block_wait(bar_mma, ph_mma, p.hdr, p.wait_limit)) { ok = false; break; }
      mma_pending = false;
      if (warp < 4) {  // row 32 warp + lane of the norm product
        const float ss = tmem_ld1(tmem_addr(tm, 32 * warp, 160));
        tmem_ld_wait();
        const int r = 32 * warp + lane;
        nrm[r] = (r & 63) < len ? rsqrtf(ss + kNormEps) : 0.f;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const bool in = 16 * b + i < len;
        qv[i] = in ? raw_f(L::kQ + qb, i) : 0.f;
        kv[i] = in ? raw_f(L::kK + qb, i) : 0.f;
      }
    }
    __syncthreads();
    // the staged q, k, z rows are consumed: load the rows of the item kNQ ahead
    {
      const bool more = L::kNQ == 2 ? have_nx2 : have_nx;
      const Item& ld = L::kNQ == 2 ? nx2 : nx;
      if (more && tid == 0) stage_qkz(qs, ld.a + ld.c * kC, ld.h);
      if (more) qkz_pending |= 1u << qs;
    }

    // ---- B: decay factors of (channel j, sub-tile b)
    float Pb, Lb, F1 = 0.f, F2 = 0.f, F3 = 0.f;  // e^{rho_b}, e^{Gam_last - rho_b}, e^{rho_{b+s} - rho_b}
    {
      float a0[4], e15[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        a0[x] = exf[x * 128 + j];
        e15[x] = exl[x * 128 + j];
      }
      float u[3];  // e^{rho_{x+1} - rho_x}
#pragma unroll
      for (int x = 0; x < 3; ++x) u[x] = e15[x] * a0[x + 1];
      Pb = a0[0];
#pragma unroll
      for (int x = 0; x < 3; ++x)
        if (x < b) Pb *= u[x];
      Lb = b == 0 ? e15[0] : b == 1 ? e15[1] : b == 2 ? e15[2] : e15[3];
#pragma unroll
      for (int x = 1; x < 4; ++x)
        if (x > b) Lb *= a0[x] * e15[x];
      // F_s = e^{rho_{b+s} - rho_b} = u[b] ... u[b+s-1]
      const float ub0 = b == 0 ? u[0] : b == 1 ? u[1] : u[2];
      const float ub1 = b == 0 ? u[1] : u[2];
      F1 = ub0;
      F2 = ub0 * ub1;
      F3 = ub0 * ub1 * u[2];
      if (b == 0) reinterpret_cast<float*>(slot + kSlotGam)[j] = Pb * Lb;  // gamma = e^{Gam_last}
      if (tid < kC) reinterpret_cast<float*>(slot + kSlotIq)[tid] = nrm[tid];
    }
    // 1 / E by the reverse product: e^{rho_b - Gam_i} = (prod_{s > i} alpha_s) / E_15
    {
      float rv = rcp(E[15]);
#pragma unroll
      for (int i = 15; i >= 0; --i) {
        const float ai = al[i];
        al[i] = rv;
        rv *= ai;
      }
    }
    float* Ei = al;
    // k / |k|
    {
      float t[16];
      lds16(nrm + 64 + 16 * b, t);
      mul16(kv, kv, t);
    }

    // ---- C: M1 operands.  R rows (beta k^ E, then q E), windows (k^ / E times
    //      e^{rho_c - rho_b} for the later row sub-tiles c)
    {
      float x[16], bke[16], qe[16], cd[16];
      lds16(bvec + 16 * b, x);
      mul16(bke, kv, E);
      mul16(bke, bke, x);   // beta k^ E
      put16(sm + L::kR, img_unit(32 * b, j, 128), img_unit(32 * b + 8, j, 128), bke);
      mul16(qe, qv, E);     // q E
      put16(sm + L::kR, img_unit(32 * b + 16, j, 128), img_unit(32 * b + 24, j, 128), qe);
      mul16(cd, kv, Ei);    // k^ / E
      {
        const int r0 = win_row0(b) + 16 * b;
        put16(sm + L::kWB, img_unit(r0, j, kWinRows), img_unit(r0 + 8, j, kWinRows), cd);
      }
#pragma unroll
      for (int s = 1; s < 4; ++s) {
        const int cw = b + s;  // window of row sub-tile cw
        if (cw < 4) {
          const float f = s == 1 ? F1 : s == 2 ? F2 : F3;
          scale16(x, cd, f);
          const int r0 = win_row0(cw) + 16 * b;
          put16(sm + L::kWB, img_unit(r0, j, kWinRows), img_unit(r0 + 8, j, kWinRows), x);
        }
      }
      sync_for_mma();
      // M1: D[R row][window row] = R W^T, per K step (16 channels) one M=128 x
      // N=160 MMA (both operands MN-major: 8 tokens of a channel per 16 bytes)
      if (tid == 0) {
        constexpr uint32_t id = instr_desc(kFmtBF16, 128, kWinRows, true, true);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t ad = smem_desc(smem_u32(sm + L::kR + k * 4096), 2048, 128);
          const uint64_t bd = smem_desc(smem_u32(sm + L::kWB + k * 2 * kWinRows * 16), kWinRows * 16, 128);
          mma_bf16(tm, ad, bd, id, k > 0);
        }
        mma_commit(bar_mma);
      }
      mma_pending = true;
      // meanwhile: X_K = beta k^ e^{Gam} (M2 operand), Q' = q e^{Gam} and
      // K' = k^ e^{Gam_last - Gam} (slot)
      scale16(x, bke, Pb);
      put16h(sm + L::kXK, img_unit(16 * b, j, 64), img_unit(16 * b + 8, j, 64), x);
      scale16(x, qe, Pb);
      put16h(slot + kSlotWQ, img_tg(16 * b, j), img_tg(16 * b + 8, j), x);
      scale16(x, cd, Lb);
      put16h(slot + kSlotK, img_unit(16 * b, j, 64), img_unit(16 * b + 8, j, 64), x);
    }
    if (!block_wait(bar_mma, ph_mma, p.hdr, p.wait_limit)) { ok = false; break; }
    mma_pending = false;

    // ---- D: products -> A_kk (fp32, strictly lower) and A_qk (f16 slot image,
    //      lower with the diagonal).  Warp (q4, cq): R rows 32 q4 + lane, i.e. row sub-tile q4 (lanes
    //      0-15 its k rows, 16-31 its q rows); key tokens i = 16 cq .. 16 cq + 15 from
    //      window q4 (cq <= q4).
    float* Af = reinterpret_cast<float*>(sm + L::kAf);
    {
      const bool krow = lane < 16;
      const int r = 16 * q4 + (lane & 15), i0 = 16 * cq;
      float v[16];
      if (cq <= q4) {
        tmem_ld16(tmem_addr(tm, 32 * q4, win_row0(q4) + i0), v);
        tmem_ld_wait();
      }
      if (krow) {
        if (cq <= q4) {
#pragma unroll
          for (int x = 0; x < 16; ++x) v[x] = i0 + x < r ? v[x] : 0.f;
#pragma unroll
          for (int x = 0; x < 16; x += 4)
            *reinterpret_cast<float4*>(Af + r * kLd + i0 + x) = make_float4(v[x], v[x + 1], v[x + 2], v[x + 3]);
        }
      } else {
#pragma unroll
        for (int x = 0; x < 16; ++x) v[x] = (cq <= q4 && i0 + x <= r) ? v[x] : 0.f;
        put16h(slot + kSlotA, img_unit(i0, r, 64), img_unit(i0 + 8, r, 64), v);
      }
    }
    fence_before_sync();
    __syncthreads();
    // CV: the next item's taps, loaded during the inverse and stored after it
    float4 tnext = make_float4(0.f, 0.f, 0.f, 0.f);
    if (CV && have_nx && b < 3) tnext = load_taps(hn);
    bool v_got = true;  // CV: this thread's wait for the v rows succeeded

    // ---- E: T = (I + A_kk)^{-1} in fp32.  Diagonal 16x16 blocks by forward
    //      substitution (one warp per block, lane = column), then the blocks below
    //      them by merging, 16 -> 32 -> 64: [[P,0],[B,Q]]^{-1} has lower-left
    //      block -Q^{-1} B P^{-1}.
    float* Tf = reinterpret_cast<float*>(sm + L::kTf);
    float* TT = reinterpret_cast<float*>(sm + L::kTT);
    float* Yb = reinterpret_cast<float*>(sm + L::kAT);  // merge products, transposed
    if (warp < 4) {
      const int base = 16 * warp, cc = lane & 15;
      float x[16];
#pragma unroll
      for (int rr = 0; rr < 16; ++rr) x[rr] = rr == cc ? 1.f : 0.f;
#pragma unroll
      for (int m = 0; m < 15; ++m)
#pragma unroll
        for (int rr = m + 1; rr < 16; ++rr)
          x[rr] = fmaf(-Af[(base + rr) * kLd + base + m], x[m], x[rr]);
      if (lane < 16) {
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) Tf[(base + rr) * kLd + base + cc] = x[rr];
#pragma unroll
        for (int rr = 0; rr < 16; rr += 4)
          *reinterpret_cast<float4*>(TT + (base + cc) * kLd + base + rr) =
              make_float4(x[rr], x[rr + 1], x[rr + 2], x[rr + 3]);
      }
    } else {
      // zero the upper blocks T[0:16][16:32], T[32:48][48:64] (and in T^T)
      for (int u = tid - 128; u < 512; u += 384) {
        const int blk = u >> 8, rr = (u >> 4) & 15, c2 = u & 15;
        const int r = 32 * blk + rr, col = 32 * blk + 16 + c2;
        Tf[r * kLd + col] = 0.f;
        TT[col * kLd + r] = 0.f;
      }
      if constexpr (CV) {
        // meanwhile the input prologue on v (its rows were requested an item ago)
        v_got = mbar_wait_cycles(bar_v, ph_v, p.wait_limit);
        if (v_got) {
          const float4 hw = tapbuf[tbuf * 384 + 256 + j];
          const int g = b - 1;  // token group: 0..23, 24..47, 48..63
          if (g < 2) conv_v(std::integral_constant<int, 24>{}, 24 * g, hw, cc0 == 0, len);
          else conv_v(std::integral_constant<int, 16>{}, 48, hw, cc0 == 0, len);
          fence_async_smem();
        }
      }
    }
    // (every thread reaches the barrier; a v wait that gave up is reported by the
    // block-wide wait on the same rows below)
    __syncthreads();
    // 16 -> 32 for the pairs (0, 1) and (2, 3): Y = A[hi][lo] T[lo][lo]
    {
      const int pr = tid >> 8, r = (tid >> 4) & 15, c2 = tid & 15;
      const int lo = 32 * pr, hi = lo + 16;
      const float* ar = Af + (hi + r) * kLd + lo;
      const float* tr = TT + (lo + c2) * kLd + lo;
      float y = 0.f;
#pragma unroll
      for (int m = 0; m < 16; m += 4) {
        const float4 x4 = *reinterpret_cast<const float4*>(ar + m);
        const float4 t4 = *reinterpret_cast<const float4*>(tr + m);
        y = fmaf(x4.x, t4.x, fmaf(x4.y, t4.y, fmaf(x4.z, t4.z, fmaf(x4.w, t4.w, y))));
      }
      Yb[(lo + c2) * kLd + r] = y;  // Y^T
    }
    __syncthreads();
    // T[hi][lo] = -T[hi][hi] Y
    {
      const int pr = tid >> 8, r = (tid >> 4) & 15, c2 = tid & 15;
      const int lo = 32 * pr, hi = lo + 16;
      const float* tr = Tf + (hi + r) * kLd + hi;
      const float* yr = Yb + (lo + c2) * kLd;
      float t = 0.f;
#pragma unroll
      for (int m = 0; m < 16; m += 4) {
        const float4 x4 = *reinterpret_cast<const float4*>(tr + m);
        const float4 y4 = *reinterpret_cast<const float4*>(yr + m);
        t = fmaf(x4.x, y4.x, fmaf(x4.y, y4.y, fmaf(x4.z, y4.z, fmaf(x4.w, y4.w, t))));
      }
      Tf[(hi + r) * kLd + lo + c2] = -t;
      TT[(lo + c2) * kLd + hi + r] = -t;
    }
    __syncthreads();
    // T -> the M2 operands, 8 columns k0 .. k0+7 of row r per 16-byte unit (upper
    // triangle zero): T (f16) and T Diag(beta) (bf16, with the bf16 v rows)
    auto put_t = [&](int r, int k0) {
      float t8[8], tb8[8];
      ld8f(Tf + r * kLd + k0, t8);
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        t8[x] = k0 + x <= r ? t8[x] : 0.f;
        tb8[x] = t8[x] * bvec[k0 + x];
      }
      *reinterpret_cast<uint4*>(sm + L::kTb + img_unit(k0, r, 64)) = pack8h(t8);
      *reinterpret_cast<uint4*>(sm + L::kTbb + img_unit(k0, r, 64)) = pack8(tb8);
    };
    // 32 -> 64 on threads 0..255 (2 x 2 tiles: rows 2 rp, 2 rp + 1 and columns
    // 2 cp, 2 cp + 1 of the lower-left 32 x 32 block); meanwhile threads 256..511
    // convert the final blocks T[0:32][0:64] and T[32:64][32:64]
    const int rp = ((tid >> 5) & 3) * 4 + (lane & 3), cp = (tid >> 7) * 8 + ((lane >> 2) & 7);
    if (tid < 256) {
      // Y = A[32:64][0:32] T[0:32][0:32]
      const float* a0 = Af + (32 + 2 * rp) * kLd;
      const float* a1 = a0 + kLd;
      const float* t0 = TT + (2 * cp) * kLd;
      const float* t1 = t0 + kLd;
      float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll
      for (int m = 0; m < 32; m += 4) {
        const float4 x0 = *reinterpret_cast<const float4*>(a0 + m);
        const float4 x1 = *reinterpret_cast<const float4*>(a1 + m);
        const float4 u0 = *reinterpret_cast<const float4*>(t0 + m);
        const float4 u1 = *reinterpret_cast<const float4*>(t1 + m);
        y00 = fmaf(x0.x, u0.x, fmaf(x0.y, u0.y, fmaf(x0.z, u0.z, fmaf(x0.w, u0.w, y00))));
        y01 = fmaf(x0.x, u1.x, fmaf(x0.y, u1.y, fmaf(x0.z, u1.z, fmaf(x0.w, u1.w, y01))));
        y10 = fmaf(x1.x, u0.x, fmaf(x1.y, u0.y, fmaf(x1.z, u0.z, fmaf(x1.w, u0.w, y10))));
        y11 = fmaf(x1.x, u1.x, fmaf(x1.y, u1.y, fmaf(x1.z, u1.z, fmaf(x1.w, u1.w, y11))));
      }
      *reinterpret_cast<float2*>(Yb + (2 * cp) * kLd + 2 * rp) = make_float2(y00, y10);      // Y^T
      *reinterpret_cast<float2*>(Yb + (2 * cp + 1) * kLd + 2 * rp) = make_float2(y01, y11);
    } else {
      for (int u = tid - 256; u < 384; u += 256) {
        // units 0..255: rows 0..31, k0 = 0..56; units 256..383: rows 32..63, k0 = 32..56
        const int r = u < 256 ? (u & 31) : 32 + (u & 31);
        const int k0 = u < 256 ? (u >> 5) * 8 : 32 + ((u - 256) >> 5) * 8;
        put_t(r, k0);
      }
    }
    if (tid < 256) {
      asm volatile("bar.sync 1, 256;" ::: "memory");  // threads 0..255 only: Y is complete
      // T[32:64][0:32] = -T[32:64][32:64] Y
      const float* r0 = Tf + (32 + 2 * rp) * kLd + 32;
      const float* r1 = r0 + kLd;
      const float* y0 = Yb + (2 * cp) * kLd;
      const float* y1 = y0 + kLd;
      float t00 = 0.f, t01 = 0.f, t10 = 0.f, t11 = 0.f;
#pragma unroll
      for (int m = 0; m < 32; m += 4) {
        const float4 x0 = *reinterpret_cast<const float4*>(r0 + m);
        const float4 x1 = *reinterpret_cast<const float4*>(r1 + m);
        const float4 u0 = *reinterpret_cast<const float4*>(y0 + m);
        const float4 u1 = *reinterpret_cast<const float4*>(y1 + m);
        t00 = fmaf(x0.x, u0.x, fmaf(x0.y, u0.y, fmaf(x0.z, u0.z, fmaf(x0.w, u0.w, t00))));
        t01 = fmaf(x0.x, u1.x, fmaf(x0.y, u1.y, fmaf(x0.z, u1.z, fmaf(x0.w, u1.w, t01))));
        t10 = fmaf(x1.x, u0.x, fmaf(x1.y, u0.y, fmaf(x1.z, u0.z, fmaf(x1.w, u0.w, t10))));
        t11 = fmaf(x1.x, u1.x, fmaf(x1.y, u1.y, fmaf(x1.z, u1.z, fmaf(x1.w, u1.w, t11))));
      }
      *reinterpret_cast<float2*>(Tf + (32 + 2 * rp) * kLd + 2 * cp) = make_float2(-t00, -t01);
      *reinterpret_cast<float2*>(Tf + (33 + 2 * rp) * kLd + 2 * cp) = make_float2(-t10, -t11);
    }
    __syncthreads();
    // the merged block T[32:64][0:32]
    if (tid < 128) put_t(32 + (tid & 31), (tid >> 5) * 8);
    if (CV && have_nx && b < 3) store_taps(tbuf ^ 1, tnext);
    // the v rows must have landed (a block-wide wait that also orders the T images)
    fence_async_smem();
    fence_before_sync();
    if (!block_wait(bar_v, ph_v, p.hdr, p.wait_limit)) { ok = false; break; }
    v_pending = false;
    if constexpr (CV) {
      // the v image was made during the diagonal solve (and published by the
      // barriers since): the raw rows are consumed, request the next item's
      if (!__syncthreads_or(!v_got)) {
        if (have_nx && tid == 0) stage_v(tokn, hn);
        v_pending = have_nx;
      } else {
        if (tid == 0) atomicOr(&p.hdr->err, kErrTimeout);
        ok = false;
        break;
      }
    }
    // ---- M2: W^T = X_K^T T^T -> TMEM columns 0-63 and U~^T = V^T (T Diag(beta))^T
    //      -> 64-127 (M = 128 channels, N = 64 tokens; V read in place from its
    //      swizzled tile as an MN-major operand)
    if (tid == 0) {
      constexpr uint32_t idw = instr_desc(kFmtF16, 128, 64, false, false);
      // V^T: MN-major from the swizzled rows as staged, or K-major from the CV image
      constexpr uint32_t idu = instr_desc(kFmtBF16, 128, 64, !CV, false);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t xd = smem_desc(smem_u32(sm + L::kXK + k * 256), 128, 1024);
        const uint64_t tb = smem_desc(smem_u32(sm + L::kTb + k * 256), 128, 1024);
        const uint64_t vd = CV ? smem_desc(smem_u32(sm + L::kVc + k * 256), 128, 1024)
                               : smem_desc_sw128(smem_u32(sm + L::kV + k * 2048), 8192, 1024);
        const uint64_t tbb = smem_desc(smem_u32(sm + L::kTbb + k * 256), 128, 1024);
        mma_bf16(tm, xd, tb, idw, k > 0);
        mma_bf16(tm + 64, vd, tbb, idu, k > 0);
      }
      mma_commit(bar_mma);
    }
    mma_pending = true;
    if (!block_wait(bar_mma, ph_mma, p.hdr, p.wait_limit)) { ok = false; break; }
    mma_pending = false;
    if constexpr (!CV) {
      // v is consumed: load the next item's
      if (have_nx && tid == 0) stage_v(tokn, hn);
      v_pending = have_nx;
    }
    // ---- F: W (the second half of the [Q' ; W] image) and U~^T -> slot
    {
      const int ch = 32 * q4 + lane;
      float w16[16], u16[16];
      tmem_ld16(tmem_addr(tm, 32 * q4, 16 * cq), w16);
      tmem_ld16(tmem_addr(tm, 32 * q4, 64 + 16 * cq), u16);
      tmem_ld_wait();
      put16h(slot + kSlotWQ, img_tg(64 + 16 * cq, ch), img_tg(72 + 16 * cq, ch), w16);
      uint4* ug = reinterpret_cast<uint4*>(slot + kSlotU);
      ug[ut_index(q4, cq, 0, lane)] = pack8h(u16);
      ug[ut_index(q4, cq, 1, lane)] = pack8h(u16 + 8);
    }
    fence_before_sync();
    tbuf ^= 1;
    qs = L::kNQ == 2 ? qs ^ 1 : 0;
    cur = nx;
    have = have_nx;
    if (L::kNQ == 2) {
      nx = nx2;
      have_nx = have_nx2;
    } else if (have) {  // one buffer: the item after the new current one is found here
      nx = cur;
      step(nx);
      have_nx = seek(nx);
    } else {
      have_nx = false;
    }
  }
  if (tid == 0) {
    // a wait gave up: let the row loads and the products still in flight land
    // before the CTA frees its Tensor Memory and leaves (at most ~2 s each)
    for (int q = 0; q < 2; ++q)
      if (qkz_pending & (1u << q)) (void)mbar_wait_cycles(bar_qkz + q, (ph_qkz >> q) & 1u, kWaitCycles);
    if (v_pending) (void)mbar_wait_cycles(bar_v, ph_v, kWaitCycles);
    if (mma_pending) (void)mbar_wait_cycles(bar_mma, ph_mma, kWaitCycles);
  }
  (void)ok;
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, 256);
}

}  // namespace

size_t prep_tc_smem_bytes() { return PrepSmem<true>::kBytes; }

cudaError_t launch_prep_tc(const TcParams& p, int gs, cudaStream_t st) {
  // the input prologue comes with the KDA gate only
  if (p.cw > 0 && gs != kGateZ) return cudaErrorInvalidValue;
  auto prep = p.cw > 0 ? prep_kernel<kGateZ, true>
            : gs == kGateHead ? prep_kernel<kGateHead, false>
            : gs == kGateChannel ? prep_kernel<kGateChannel, false> : prep_kernel<kGateZ, false>;
  const int bytes = p.cw > 0 ? PrepSmem<true>::kBytes : PrepSmem<false>::kBytes;
  cudaError_t err = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err != cudaSuccess) return err;
  int sms = 0, dev = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  prep<<<sms, kNT, bytes, st>>>(p);
  return cudaGetLastError();
}

}  // namespace tcp
}  // namespace kda
