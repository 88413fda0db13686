// kda_prefill_tc.cu -- chunkwise KDA prefill on the sm_100a tensor cores
// (tcgen05.mma, TMEM accumulators), bf16 inputs, dk = dv = 128, chunk = 64.
//
// One CTA of 512 threads runs one (sequence, head, segment) over its chunks in
// order (Kimi Linear summary §3.1: chunkwise WY / UT form with an inter-chunk
// state carry; §3.2: sub-chunking keeps the channel-wise decay factors in
// range; Appendix C: per-chunk cumulative log-decay, forward-substitution
// inverse).  The fp32 state S [dk x dv] stays in Tensor Memory.  Per 64-token
// chunk, with Gam = chunk-local inclusive cumsum of the gate g:
//
//   products  A_kk = StrictTril(Diag(beta) K K^T (decayed)), A_qk = Tril(Q K^T
//             (decayed)), from four M=64 MMAs: for row sub-tile b (16 tokens,
//             reference rho_b = Gam at its first token) the rows carry
//             E = e^{Gam_r - rho_b} <= 1 and the column operand C_b carries
//             e^{rho_b - Gam_i} (<= e^75 on the diagonal sub-tile, <= 1 before)
//   inverse   T = (I + A_kk)^{-1}: forward substitution in registers on the
//             16x16 diagonal blocks, then the blocks below the diagonal by
//             T_ba = -T_bb sum_{a<=c<b} A_bc T_ca (fp32, CUDA cores)
//   WY        [W | U~] = T [Diag(beta)(K e^Gam) | Diag(beta) V]   (one MMA)
//   chain     D_W = W S, D_Q = (Q e^Gam) S, U = U~ - D_W,
//             S = Diag(e^{Gam_last}) S + (K e^{Gam_last - Gam})^T U,
//             O = D_Q + A_qk U
//
// Inputs arrive by TMA (3-D tensor maps over [T, H, 128], one 64x128 box per
// tensor and chunk), prefetched one chunk ahead.  MMA operands are bf16 in
// shared memory (no swizzle, 8 x 16-byte core matrices); each operand's major
// order is chosen so that the threads that produce it store 16-byte vectors of
// 8 consecutive tokens.  Accumulators are fp32 in TMEM.  Rows of a partial
// chunk past the sequence end are zero, so they contribute nothing.
//
// Segments: with P > 1 a sequence is cut into P runs of chunks.  The
// transition pass (mode 1) runs each segment but the last from a zero state
// and from the identity, giving the affine map S_out = M S_in + N of the
// segment; a small kernel composes the maps into every segment's incoming
// state; the full pass (mode 0) then runs every segment from its true
// incoming state and writes the outputs.  This is the single-GPU form of the
// prefix scan over per-segment state updates (Kimi K3 architecture summary,
// KDA context parallelism).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kda_common.cuh"
#include "kda_launch.h"
#include "tc_sm100.cuh"

namespace kda {
namespace {

using namespace tc;

constexpr int kC = 64;    // chunk tokens
constexpr int kD = 128;   // dk = dv
constexpr int kNT = 512;  // threads (16 warps)

// ---- shared memory map (bytes), per pass ----
struct FusedSmem {
  static constexpr int kSb = 0;                                 // S bf16, B operand, MN-major
  static constexpr int kRaw = kSb + 32768;                      // q | k | z | v, [64][128] bf16
  static constexpr int kP = kRaw + 65536;                       // region P, reused through a chunk:
  static constexpr int kR = kP;                                 //   R   B op (N=128, K=128) MN-major
  static constexpr int kCc = kP + 32768;                        //   C   A op (M=160, K=128) MN-major
  static constexpr int kAkk = kP;                               //   A_kk fp32 [64][68]
  static constexpr int kTf = kP + 17408;                        //   T    fp32 [64][68]
  static constexpr int kX = kP;                                 //   X   B op (N=256, K=64) K-major
  static constexpr int kQp = kP + 32768;                        //   Q'  A op (M=64, K=128) MN-major
  static constexpr int kKp = kP + 49152;                        //   K'  A op (M=128, K=64) K-major
  static constexpr int kW = kP;                                 //   W   A op (M=64, K=128) K-major
  static constexpr int kU = kP;                                 //   U   B op (N=128, K=64) MN-major
  static constexpr int kTop = kP + 73728;                       // T   A op (M=64, K=64) K-major
  static constexpr int kA3 = kTop + 8192;                       // A_qk A op (M=64, K=64) MN-major
  static constexpr int kVec = kA3 + 8192;
  static constexpr int kBytes = kVec + 2304 * 4 + 64;
};
// vectors (floats) at Smem::kVec
constexpr int kVecIq = 0, kVecIk = 64, kVecBeta = 128, kVecGam = 192, kVecRho = 320,
              kVecTot = 832, kVecY = 1088;  // Y: up to 32 x 36 floats

// TMEM columns.  M=64 accumulators put row r in lane 32 (r / 16) + r % 16.
constexpr uint32_t kTmA = 0;     // A products, 4 x 32 columns (prep)
constexpr uint32_t kTmWU = 0;    // [W | U~]: 256 columns (after the products are read)
constexpr uint32_t kTmW = 0;     // D_W = W S (128, or 256 for W [S | X])
constexpr uint32_t kTmQ = 128;   // D_Q = Q' S (+ A_qk U)
constexpr uint32_t kTmS = 256;   // fp32 state; identity-started block X at 384 (transition)

constexpr int kLd = 68;  // row stride (floats) of the fp32 A_kk / T tiles

// Chain operands of one (chunk, head), written by the preparation kernel and
// read by the chain passes with bulk copies.  The bf16 images have exactly the
// shared-memory layouts the MMAs read: W and Q' (K-major [token][dk], adjacent
// so that [W ; Q'] is one N=128 operand), K' (MN-major [token][dk]), A_qk
// (MN-major, N = query row, K = key row); U~^T is bf16 [dv][token] in the
// order the chain threads read it (see ut_index); then gamma (128 fp32) and the
// query row scales (64 fp32).
constexpr int kSlotW = 0, kSlotQ = 16384, kSlotK = 32768, kSlotA3 = 49152, kSlotU = 57344,
              kSlotGam = 73728, kSlotIq = 74240, kSlotBytes = 74496;
// Chunk c of sequence n (first token a) has slot a / C + n + c: distinct for
// every chunk of every sequence and below T / C + N.
__device__ __forceinline__ unsigned char* chunk_slot(const unsigned char* prep_base, int a, int n,
                                                     int c, int h, int H) {
  return const_cast<unsigned char*>(prep_base) +
         ((size_t)(a / 64 + n + c) * H + h) * (size_t)kSlotBytes;
}
// 16-byte unit of U~^T (value column 32 q4 + l; tokens 16 cq + 8 half .. +7, bf16)
// in a slot: each warp reads 512 consecutive bytes per vector.
__device__ __forceinline__ int ut_index(int q4, int cq, int half, int l) {
  return ((cq * 4 + q4) * 2 + half) * 32 + l;
}

constexpr long long kWaitCycles = 4000000000LL;  // ~2 s: a wait this long is a fault

// 16-byte-vector layouts of bf16 operands
__device__ __forceinline__ uint32_t kmaj(int row, int k, int sbo) {
  return (row >> 3) * sbo + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
}
__device__ __forceinline__ uint32_t mnmaj(int mn, int k, int lbo) {
  return (mn >> 3) * 128 + (k >> 3) * lbo + (k & 7) * 16 + (mn & 7) * 2;
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
// 8 bf16 (one 16-byte vector) -> fp32, exactly
__device__ __forceinline__ void unpack8(const uint4 u, float* f) {
  f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
  f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
  f[4] = __uint_as_float(u.z << 16); f[5] = __uint_as_float(u.z & 0xffff0000u);
  f[6] = __uint_as_float(u.w << 16); f[7] = __uint_as_float(u.w & 0xffff0000u);
}
__device__ __forceinline__ void ld8f(const float* p, float* f) {  // 8 fp32, 16-byte aligned
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void st16(unsigned char* base, uint32_t off, const float* v) {
  *reinterpret_cast<uint4*>(base + off) = pack8(v);
}

// c += A B for a 2 x 2 tile: A rows a0, a1 (16-byte aligned, read as float4),
// B rows ldb floats apart (float2 at the tile's column); NK a multiple of 4.
template <int NK>
__device__ __forceinline__ void mm2x2(const float* a0, const float* a1, const float* b, int ldb,
                                      float (&c)[4]) {
#pragma unroll
  for (int i = 0; i < NK; i += 4) {
    const float4 x = *reinterpret_cast<const float4*>(a0 + i);
    const float4 y = *reinterpret_cast<const float4*>(a1 + i);
    const float xa[4] = {x.x, x.y, x.z, x.w}, ya[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 t = *reinterpret_cast<const float2*>(b + (i + u) * ldb);
      c[0] += xa[u] * t.x;
      c[1] += xa[u] * t.y;
      c[2] += ya[u] * t.x;
      c[3] += ya[u] * t.y;
    }
  }
}

struct alignas(64) TcParams {
  CUtensorMap tq, tk, tz, tv;  // [T, H, 128] bf16, box 64 tokens x 1 x 128 channels
  CUtensorMap sq, sk, sz, sv;  // the same, box 64 tokens x 1 x 64 channels, 128-byte swizzle
  const __nv_bfloat16 *q, *k, *beta, *z, *v;
  // g: the log-decay given directly, [T, H, 128], or the scalar gate's [T, H]
  // (one value per token and head); null when it is computed from z and A.
  const float *A, *g, *S0;
  const int32_t* cu;
  __nv_bfloat16* o;
  float* S_final;
  float* S_ckpt;  // checkpoints every ckpt_every chunks (ckpt_count per sequence and head)
  int ckpt_every, ckpt_count;
  const __nv_bfloat16* og;  // output epilogue: sigmoid gate input [T, H, 128], or null (no epilogue)
  const float* ow;          // RMSNorm gain [128], or null (ones)
  float oeps;
  int N, T, max_len, H, P;
  float* seg;  // per (n, h): transitions (M, N) of segments 0..P-2, incoming states of 0..P-1
  unsigned char* prep;  // per (chunk slot, h): chain operands left by the transition pass
  WsHeader* hdr;
  // Context parallelism: the segment buffers are laid out for Pseg segments
  // (P, or P + 1 so that all P transitions fit); M_out, N_out receive the
  // folded transition of each (sequence, head) when set.
  int Pseg;
  float *M_out, *N_out;
};

// Checkpoint slot of the state after sequence-relative chunk c (n_tok tokens in
// the sequence), or null when no checkpoint falls there.
__device__ __forceinline__ float* ckpt_state(const TcParams& p, int n, int h, int c, int n_tok) {
  if (!p.S_ckpt || (c + 1) % p.ckpt_every != 0 || (c + 1) * 64 > n_tok) return nullptr;
  return p.S_ckpt + (((size_t)n * p.H + h) * p.ckpt_count + (c + 1) / p.ckpt_every - 1) * 128 * 128;
}

// Output epilogue (Kimi Linear summary, §4: head-wise RMSNorm of o, then a
// data-dependent sigmoid gate) on x[0..NX) of one token's 128 features, given
// the sum of squares over all 128: x * rsqrt(mean + eps) * w * sigmoid(r).
// r: the gate input at the same features (16-byte aligned); w: the gain or null.
__device__ __forceinline__ void norm_gate8(float* x, float inv, uint4 r8, const float* w) {
  float rv[8], wv[8];
  unpack8(r8, rv);
  if (w) {
    ld8f(w, wv);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) wv[e] = 1.f;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = x[e] * inv * wv[e] * out_sigmoid(rv[e]);
}
template <int NX>
__device__ __forceinline__ void norm_gate(float* x, float sumsq, const __nv_bfloat16* r,
                                          const float* w, float eps) {
  const float inv = rsqrtf(sumsq * (1.0f / 128) + eps);
#pragma unroll
  for (int i = 0; i < NX; i += 8)
    norm_gate8(x + i, inv, *reinterpret_cast<const uint4*>(r + i), w ? w + i : nullptr);
}

// Segment p of a sequence with nch chunks: chunks [c0, c1).
__device__ __forceinline__ void segment_chunks(int nch, int P, int p, int& c0, int& c1) {
  const int G = (nch + P - 1) / P;
  c0 = min(nch, p * G);
  c1 = min(nch, c0 + G);
}

__device__ __forceinline__ float* seg_trans(float* seg, int n, int h, int H, int P, int p) {
  const size_t per = (size_t)(P - 1) * 2 * kD * kD + (size_t)P * kD * kD;
  return seg + ((size_t)n * H + h) * per + (size_t)p * 2 * kD * kD;
}
__device__ __forceinline__ float* seg_sin(float* seg, int n, int h, int H, int P, int p) {
  const size_t per = (size_t)(P - 1) * 2 * kD * kD + (size_t)P * kD * kD;
  return seg + ((size_t)n * H + h) * per + (size_t)(P - 1) * 2 * kD * kD + (size_t)p * kD * kD;
}

// One TMA box (64 tokens x 1 head x 128 channels) of a [T, H, 128] tensor.
__device__ __forceinline__ void tma_box(void* dst, const CUtensorMap* map, int h, int tok0,
                                        uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(h), "r"(tok0), "r"(smem_u32(bar))
      : "memory");
}

// One TMA box at channel offset x (a multiple of 64) of a [T, H, 128] tensor.
__device__ __forceinline__ void tma_box_x(void* dst, const CUtensorMap* map, int x, int h, int tok0,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(h), "r"(tok0), "r"(smem_u32(bar))
      : "memory");
}

// Where the log-decay comes from (a template parameter of the kernels that
// compute it, so each variant carries only its own code): the KDA gate from z
// and A; given per channel (g [T, H, 128]); given once per token and head
// (g [T, H], the scalar gate of Gated DeltaNet, broadcast over the channels).
enum GateSrc : int { kGateZ = 0, kGateChannel = 1, kGateHead = 2 };

// q, k, z, v rows of the chunk starting at tok0 (single thread); z only when
// the gate is computed from it.
template <int GS>
__device__ __forceinline__ void stage_chunk(const TcParams& p, unsigned char* raw, uint64_t* bar,
                                            int tok0, int h) {
  mbar_arrive_expect_tx(bar, (GS == kGateZ ? 4 : 3) * 16384);
  tma_box(raw + 0 * 16384, &p.tq, h, tok0, bar);
  tma_box(raw + 1 * 16384, &p.tk, h, tok0, bar);
  if (GS == kGateZ) tma_box(raw + 2 * 16384, &p.tz, h, tok0, bar);
  tma_box(raw + 3 * 16384, &p.tv, h, tok0, bar);
}

__device__ __forceinline__ float raw_at(const unsigned char* raw, int t, int r, int c) {
  return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(raw + t * 16384 + r * 256)[c]);
}

// Block-wide bounded wait on an mbarrier phase; false if it timed out (the
// error word then carries kErrTimeout).
__device__ __forceinline__ bool block_wait(uint64_t* bar, uint32_t& phase, WsHeader* hdr) {
  const bool got = mbar_wait_cycles(bar, phase, kWaitCycles);
  phase ^= 1;
  if (__syncthreads_or(!got)) {
    if (threadIdx.x == 0) atomicOr(&hdr->err, kErrTimeout);
    return false;
  }
  fence_after_sync();
  return true;
}

__device__ __forceinline__ void sync_for_mma() {
  fence_async_smem();
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
}

// ---------------------------------------------------------------------------
// Fused pass for sequences that are not split into segments: one CTA per
// (sequence, head) prepares each chunk and advances the state through it,
// chunk after chunk (incoming state S0 or S_in of its segment); o, S_final.
template <int GS>
__global__ void __launch_bounds__(kNT, 1) fused_kernel(const __grid_constant__ TcParams p) {
  using L = FusedSmem;
  extern __shared__ __align__(1024) unsigned char sm[];
  __shared__ uint64_t s_bar, s_bar_raw;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  float* vec = reinterpret_cast<float*>(sm + L::kVec);
  unsigned char* raw = sm + L::kRaw;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x, h = blockIdx.y, seg = blockIdx.z;
  const int H = p.H;

  const bool ok = seqlens_valid(p.cu, p.N, p.T, p.max_len);
  if (!ok && n == 0 && h == 0 && seg == 0 && tid == 0) atomicOr(&p.hdr->err, kErrBadSeqlens);
  if (!ok) return;
  int a, b;
  seq_bounds(p.cu, n, p.max_len, a, b);
  const int nch = (b - a + kC - 1) / kC;
  int c0, c1;
  segment_chunks(nch, p.P, seg, c0, c1);

  // ---- set-up: TMEM, barriers, first chunk's rows
  if (warp == 0) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&s_bar, 1);
    mbar_init(&s_bar_raw, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = s_tmem;
  uint32_t phase = 0, phase_raw = 0;
  bool raw_pending = c0 < c1;  // a TMA load into the staging area is in flight
  if (tid == 0 && c0 < c1) stage_chunk<GS>(p, raw, &s_bar_raw, a + c0 * kC, h);

  constexpr int SbN = 128;                    // N extent of the bf16 state operand
  constexpr int SbL = SbN * 16;               // its K-group stride (LBO)
  const int q4 = warp & 3, cq = warp >> 2;    // TMEM lane quarter, 32-column quarter
  const int srow = 32 * q4 + lane;            // dk row (M=128 accumulators)
  const int r64 = 16 * q4 + lane;             // token row of M=64 accumulators (lane < 16)
  const bool m64 = lane < 16;

  // ---- initial state: S0 (or the composed incoming state)
  {
    const float* S0 = seg > 0 ? seg_sin(p.seg, n, h, H, p.Pseg, seg)
                              : (p.S0 ? p.S0 + ((size_t)n * H + h) * kD * kD : nullptr);
#pragma unroll
    for (int c16 = 0; c16 < 32; c16 += 16) {
      float v16[16];
      const int col = 32 * cq + c16;
      if (S0) {
        const float4* src = reinterpret_cast<const float4*>(S0 + (size_t)srow * kD + col);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 f = src[i];
          v16[4 * i] = f.x; v16[4 * i + 1] = f.y; v16[4 * i + 2] = f.z; v16[4 * i + 3] = f.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v16[i] = 0.f;
      }
      tmem_st16(tmem_addr(tm, 32 * q4, kTmS + col), v16);
      st16(sm + L::kSb, mnmaj(col, srow, SbL), v16);
      st16(sm + L::kSb, mnmaj(col + 8, srow, SbL), v16 + 8);
    }
    tmem_st_wait();
  }

  const float expA = GS == kGateZ ? expf(p.A[h]) : 0.f;
  // prep ownership: channel j, row sub-tile qq (rows 16qq .. 16qq+15)
  const int j = tid & 127, qq = tid >> 7;
  // C_b window of row sub-tile b starts at row 8 b (b + 1) of C: 0, 16, 48, 96

  // beta of the chunk, loaded one chunk ahead (thread t < 64 holds token t)
  auto load_beta = [&](int cc) -> float {
    const int t0 = a + cc * kC;
    return (tid < kC && cc < c1 && tid < b - t0) ? __bfloat162float(p.beta[(size_t)(t0 + tid) * H + h]) : 0.f;
  };
  float beta_next = load_beta(c0);
  for (int c = c0; c < c1; ++c) {
    const int tok0 = a + c * kC;
    const int len = min(kC, b - tok0);
    sync_for_mma();
    if (tid < kC) vec[kVecBeta + tid] = beta_next;
    beta_next = load_beta(c + 1);
    if (!block_wait(&s_bar_raw, phase_raw, p.hdr)) { s_abort = 1; break; }
    raw_pending = false;

    // ---- inverse row norms of q and k (warp w: rows w, w+16, w+32, w+48); the
    //      query norm scales the output row at the end
    {
      float sq[8];  // q rows, then k rows
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int r = warp + 16 * (m & 3);
        const uint2 uq = *reinterpret_cast<const uint2*>(raw + (m >> 2) * 16384 + r * 256 + 8 * lane);
        const float2 q0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uq.x));
        const float2 q1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uq.y));
        sq[m] = q0.x * q0.x + q0.y * q0.y + q1.x * q1.x + q1.y * q1.y;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int m = 0; m < 8; ++m) sq[m] += __shfl_xor_sync(0xffffffffu, sq[m], o);
      if (lane < 8) {
        const int r = warp + 16 * (lane & 3);
        float v = sq[0];
#pragma unroll
        for (int m = 1; m < 8; ++m)
          if (lane == m) v = sq[m];
        vec[(lane < 4 ? kVecIq : kVecIk) + r] = r < len ? rsqrtf(v + kNormEps) : 0.f;
      }
    }
    // ---- gate and cumsum of channel j over sub-tile qq; E = e^{Gam_r - rho_qq}
    //      depends only on this sub-tile's own partial sums
    float E[16], Ei[16];
    {
      if constexpr (GS == kGateChannel) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = 16 * qq + i;
          E[i] = r < len ? p.g[((size_t)(tok0 + r) * H + h) * kD + j] : 0.f;
        }
      } else if constexpr (GS == kGateHead) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = 16 * qq + i;
          E[i] = r < len ? p.g[(size_t)(tok0 + r) * H + h] : 0.f;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) E[i] = raw_at(raw, 2, 16 * qq + i, j);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          E[i] = (16 * qq + i < len) ? __fdividef(kGateMin, 1.0f + __expf(-expA * E[i])) : 0.f;
      }
#pragma unroll
      for (int i = 1; i < 16; ++i) E[i] += E[i - 1];
      vec[kVecTot + qq * 128 + j] = E[15];
      vec[kVecRho + qq * 128 + j] = E[0];  // sub-tile-local; the offsets are added below
#pragma unroll
      for (int i = 15; i >= 0; --i) {
        E[i] = __expf(E[i] - E[0]);
        Ei[i] = __fdividef(1.0f, E[i]);
      }
    }
    __syncthreads();
    // rho_b = Gam at the first token of sub-tile b; Gam_last = Gam at row 63
    float rho[4], glast;
    {
      float acc = 0.f;
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) {
        rho[bb] = acc + vec[kVecRho + bb * 128 + j];
        acc += vec[kVecTot + bb * 128 + j];
      }
      glast = acc;
    }
    const float rq = qq == 0 ? rho[0] : qq == 1 ? rho[1] : qq == 2 ? rho[2] : rho[3];

    // ---- product operands R (rows, MN-major) and C_b (columns, MN-major)
    {
#pragma unroll
      for (int g8 = 0; g8 < 2; ++g8) {
        const int r0 = 16 * qq + 8 * g8;
        float kv[8], qv[8], cv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = r0 + i;
          const float kh = r < len ? raw_at(raw, 1, r, j) : 0.f;
          const float qh = r < len ? raw_at(raw, 0, r, j) : 0.f;
          kv[i] = kh * E[8 * g8 + i];
          qv[i] = qh * E[8 * g8 + i];
          cv[i] = kh * Ei[8 * g8 + i];
        }
        st16(sm + L::kR, mnmaj(32 * qq + 8 * g8, j, 2048), kv);
        st16(sm + L::kR, mnmaj(32 * qq + 16 + 8 * g8, j, 2048), qv);
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
          if (bb < qq) continue;
          float w8[8];
          const float f = bb == qq ? 1.f : __expf(rho[bb] - rq);
#pragma unroll
          for (int i = 0; i < 8; ++i) w8[i] = cv[i] * f;
          st16(sm + L::kCc, mnmaj(8 * bb * (bb + 1) + r0, j, 2560), w8);
        }
      }
    }
    sync_for_mma();
    // ---- M1: four M=64 MMAs -> TMEM [32b, +32): cols 0-15 A_kk^T, 16-31 A_qk^T
    if (tid == 0) {
      constexpr uint32_t id = instr_desc(kFmtBF16, 64, 32, true, true);
      const uint64_t ad = smem_desc(smem_u32(sm + L::kCc), 2560, 128);
      const uint64_t bd = smem_desc(smem_u32(sm + L::kR), 2048, 128);
#pragma unroll
      for (int bb = 0; bb < 4; ++bb)
#pragma unroll
        for (int k = 0; k < 8; ++k)  // descriptor addresses count 16-byte units
          mma_bf16(tm + kTmA + 32 * bb, ad + ((bb * (bb + 1) * 128 + 2 * 2560 * k) >> 4),
                   bd + ((32 * bb * 16 + 2 * 2048 * k) >> 4), id, k > 0);
      mma_commit(&s_bar);
    }
    if (!block_wait(&s_bar, phase, p.hdr)) { s_abort = 1; break; }
    // ---- A products -> A_kk (fp32 smem, beta- and norm-scaled, strictly
    //      lower) and A_qk (bf16 A3, MN-major)
    float* Akk = reinterpret_cast<float*>(sm + L::kAkk);
    {
      const int i = r64, bb = cq;  // warp: lane quarter q4, row block bb
      float va[16], vq[16];
      tmem_ld16(tmem_addr(tm, 32 * q4, kTmA + 32 * bb), va);
      tmem_ld16(tmem_addr(tm, 32 * q4, kTmA + 32 * bb + 16), vq);
      tmem_ld_wait();
      if (m64) {
        const float ki = vec[kVecIk + i];
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) {
          const int r = 16 * bb + cc;
          Akk[r * kLd + i] = (i < r) ? vec[kVecBeta + r] * vec[kVecIk + r] * ki * va[cc] : 0.f;
          vq[cc] = (i <= r) ? vq[cc] * ki : 0.f;
        }
        st16(sm + L::kA3, mnmaj(16 * bb, i, 1024), vq);
        st16(sm + L::kA3, mnmaj(16 * bb + 8, i, 1024), vq + 8);
      }
    }
    fence_before_sync();
    __syncthreads();
    // ---- T = (I + A_kk)^{-1}
    // diagonal 16x16 blocks by forward substitution (registers), then the
    // blocks below them by merging: [[P,0],[B,Q]]^{-1} has lower-left block
    // -Q^{-1} B P^{-1}; first 16 -> 32 (block pairs 0|1 and 2|3), then 32 -> 64.
    // The merges use 2x2 register tiles; the two upper blocks they read are
    // zeroed first.
    float* Tf = reinterpret_cast<float*>(sm + L::kTf);
    float* Y = vec + kVecY;  // scratch, 32 x 36
    if (tid < kC) {
      const int bk = tid >> 4, cc = tid & 15, base = 16 * bk;
      float x[16];
#pragma unroll
      for (int rr = 0; rr < 16; ++rr) {
        float acc = (rr == cc) ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < rr; ++i) acc -= Akk[(base + rr) * kLd + base + i] * x[i];
        x[rr] = (rr < cc) ? 0.f : acc;
      }
#pragma unroll
      for (int rr = 0; rr < 16; ++rr) Tf[(base + rr) * kLd + base + cc] = x[rr];
    } else {
      // zero T[0:16][16:32] and T[32:48][48:64]
      const int e = tid - kC;  // 0..447
      if (e < 512 - kC) {
        for (int f = e; f < 512; f += 512 - kC) {
          const int blk = f >> 8, rr = (f >> 4) & 15, cc = f & 15;
          Tf[(32 * blk + rr) * kLd + 32 * blk + 16 + cc] = 0.f;
        }
      }
    }
    __syncthreads();
    if (tid < 128) {
      // 16 -> 32, pair pr: Y = A[hi][lo] T[lo][lo]; T[hi][lo] = -T[hi][hi] Y (2x2 tiles)
      const int pr = tid >> 6, r2 = ((tid >> 3) & 7) * 2, c2 = (tid & 7) * 2;
      const int lo = 32 * pr, hi = lo + 16;
      float y[4] = {0.f, 0.f, 0.f, 0.f};
      mm2x2<16>(Akk + (hi + r2) * kLd + lo, Akk + (hi + r2 + 1) * kLd + lo, Tf + lo * kLd + lo + c2,
                kLd, y);
      float* Yp = Y + pr * 16 * 34;
      *reinterpret_cast<float2*>(Yp + r2 * 34 + c2) = make_float2(y[0], y[1]);
      *reinterpret_cast<float2*>(Yp + (r2 + 1) * 34 + c2) = make_float2(y[2], y[3]);
      __syncwarp();
      // all of this pair's Y rows come from the same two warps: sync those
      asm volatile("bar.sync %0, %1;" ::"r"(1 + pr), "r"(64) : "memory");
      float t[4] = {0.f, 0.f, 0.f, 0.f};
      mm2x2<16>(Tf + (hi + r2) * kLd + hi, Tf + (hi + r2 + 1) * kLd + hi, Yp + c2, 34, t);
      *reinterpret_cast<float2*>(Tf + (hi + r2) * kLd + lo + c2) = make_float2(-t[0], -t[1]);
      *reinterpret_cast<float2*>(Tf + (hi + r2 + 1) * kLd + lo + c2) = make_float2(-t[2], -t[3]);
    }
    __syncthreads();
    if (tid < 256) {
      // 32 -> 64: Y = A[32:64][0:32] T[0:32][0:32]; T[32:64][0:32] = -T[32:64][32:64] Y
      const int r2 = (tid >> 4) * 2, c2 = (tid & 15) * 2;
      float y[4] = {0.f, 0.f, 0.f, 0.f};
      mm2x2<32>(Akk + (32 + r2) * kLd, Akk + (33 + r2) * kLd, Tf + c2, kLd, y);
      *reinterpret_cast<float2*>(Y + r2 * 34 + c2) = make_float2(y[0], y[1]);
      *reinterpret_cast<float2*>(Y + (r2 + 1) * 34 + c2) = make_float2(y[2], y[3]);
      asm volatile("bar.sync %0, %1;" ::"r"(3), "r"(256) : "memory");
      float t[4] = {0.f, 0.f, 0.f, 0.f};
      mm2x2<32>(Tf + (32 + r2) * kLd + 32, Tf + (33 + r2) * kLd + 32, Y + c2, 34, t);
      *reinterpret_cast<float2*>(Tf + (32 + r2) * kLd + c2) = make_float2(-t[0], -t[1]);
      *reinterpret_cast<float2*>(Tf + (33 + r2) * kLd + c2) = make_float2(-t[2], -t[3]);
    }
    __syncthreads();
    // T -> bf16 A operand (K-major), upper triangle zero; 8 consecutive threads
    // take 8 consecutive rows so each 16-byte store phase is conflict-free
    {
      const int r = (tid >> 6) * 8 + (tid & 7), i0 = ((tid >> 3) & 7) * 8;
      float t8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) t8[i] = (i0 + i <= r) ? Tf[r * kLd + i0 + i] : 0.f;
      st16(sm + L::kTop, kmaj(r, i0, 1024), t8);
    }
    __syncthreads();  // A_kk / T (fp32) are dead from here: region P takes X, Q', K'

    // ---- WY / chain operands: X_K, X_V (K-major), Q' (MN-major), K' (K-major), gamma
    {
      const float er = __expf(rq), el = __expf(glast - rq);
      if (qq == 0) vec[kVecGam + j] = __expf(glast);
#pragma unroll
      for (int g8 = 0; g8 < 2; ++g8) {
        const int r0 = 16 * qq + 8 * g8;
        float xk[8], xv[8], qp[8], kp[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = r0 + i;
          const bool in = r < len;
          const float kh = in ? raw_at(raw, 1, r, j) * vec[kVecIk + r] : 0.f;
          const float bet = vec[kVecBeta + r];
          xk[i] = bet * kh * E[8 * g8 + i] * er;
          xv[i] = in ? bet * raw_at(raw, 3, r, j) : 0.f;
          kp[i] = kh * Ei[8 * g8 + i] * el;
          qp[i] = in ? raw_at(raw, 0, r, j) * E[8 * g8 + i] * er : 0.f;
        }
        st16(sm + L::kX, kmaj(j, r0, 1024), xk);
        st16(sm + L::kX, kmaj(128 + j, r0, 1024), xv);
        st16(sm + L::kKp, kmaj(j, r0, 1024), kp);
        st16(sm + L::kQp, mnmaj(r0, j, 1024), qp);
      }
    }
    sync_for_mma();
    // the staged rows are consumed: prefetch the next chunk
    if (c + 1 < c1) {
      raw_pending = true;
      if (tid == 0) stage_chunk<GS>(p, raw, &s_bar_raw, a + (c + 1) * kC, h);
    }
    // ---- M2: [W | U~] = T [X_K | X_V]  (M=64, N=256, K=64)
    if (tid == 0) {
      constexpr uint32_t id = instr_desc(kFmtBF16, 64, 256, false, false);
      const uint64_t ad = smem_desc(smem_u32(sm + L::kTop), 128, 1024);
      const uint64_t bd = smem_desc(smem_u32(sm + L::kX), 128, 1024);
#pragma unroll
      for (int k = 0; k < 4; ++k) mma_bf16(tm + kTmWU, ad + 16 * k, bd + 16 * k, id, k > 0);
      mma_commit(&s_bar);
    }
    if (!block_wait(&s_bar, phase, p.hdr)) { s_abort = 1; break; }
    // ---- W -> bf16 A operand (K-major); U~ -> registers (M=64 rows, lane < 16)
    float ut[32];
#pragma unroll
    for (int c16 = 0; c16 < 32; c16 += 16) {
      float w16[16], u16[16];
      tmem_ld16(tmem_addr(tm, 32 * q4, kTmWU + 32 * cq + c16), w16);
      tmem_ld16(tmem_addr(tm, 32 * q4, kTmWU + 128 + 32 * cq + c16), u16);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) ut[c16 + i] = u16[i];
      if (m64) {
        st16(sm + L::kW, kmaj(r64, 32 * cq + c16, 2048), w16);
        st16(sm + L::kW, kmaj(r64, 32 * cq + c16 + 8, 2048), w16 + 8);
      }
    }
    sync_for_mma();
    // ---- C1: D_W = W S, D_Q = Q' S (M=64, N=128, K=128)
    if (tid == 0) {
      const uint64_t sd = smem_desc(smem_u32(sm + L::kSb), SbL, 128);
      const uint64_t wd = smem_desc(smem_u32(sm + L::kW), 128, 2048);
      const uint64_t qd = smem_desc(smem_u32(sm + L::kQp), 1024, 128);
      constexpr uint32_t idw = instr_desc(kFmtBF16, 64, SbN, false, true);
      constexpr uint32_t idq = instr_desc(kFmtBF16, 64, 128, true, true);
#pragma unroll
      for (int k = 0; k < 8; ++k) mma_bf16(tm + kTmW, wd + 16 * k, sd + (2 * SbL >> 4) * k, idw, k > 0);
#pragma unroll
      for (int k = 0; k < 8; ++k) mma_bf16(tm + kTmQ, qd + 128 * k, sd + (2 * SbL >> 4) * k, idq, k > 0);
      mma_commit(&s_bar);
    }
    // ---- meanwhile decay the fp32 state by gamma = e^{Gam_last} (rows = dk =
    //      TMEM lanes); C1 reads the bf16 copy
    {
      const float gm = vec[kVecGam + srow];
      float s0[16], s1[16];
      const uint32_t col = kTmS + 32 * cq;
      tmem_ld16(tmem_addr(tm, 32 * q4, col), s0);
      tmem_ld16(tmem_addr(tm, 32 * q4, col + 16), s1);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) { s0[i] *= gm; s1[i] *= gm; }
      tmem_st16(tmem_addr(tm, 32 * q4, col), s0);
      tmem_st16(tmem_addr(tm, 32 * q4, col + 16), s1);
      tmem_st_wait();
    }
    if (!block_wait(&s_bar, phase, p.hdr)) { s_abort = 1; break; }
    // ---- U = U~ - W S -> B operand (MN-major)
    {
      float d0[16], d1[16];
      const int col = 32 * cq;
      tmem_ld16(tmem_addr(tm, 32 * q4, kTmW + col), d0);
      tmem_ld16(tmem_addr(tm, 32 * q4, kTmW + col + 16), d1);
      tmem_ld_wait();
      if (m64) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          d0[i] = ut[i] - d0[i];
          d1[i] = ut[16 + i] - d1[i];
        }
        st16(sm + L::kU, mnmaj(col, r64, SbL), d0);
        st16(sm + L::kU, mnmaj(col + 8, r64, SbL), d0 + 8);
        st16(sm + L::kU, mnmaj(col + 16, r64, SbL), d1);
        st16(sm + L::kU, mnmaj(col + 24, r64, SbL), d1 + 8);
      }
    }
    sync_for_mma();
    // ---- C2: S += K'^T U (M=128); D_Q += A_qk U (M=64)
    if (tid == 0) {
      const uint64_t kd = smem_desc(smem_u32(sm + L::kKp), 128, 1024);
      const uint64_t ud = smem_desc(smem_u32(sm + L::kU), SbL, 128);
      const uint64_t a3 = smem_desc(smem_u32(sm + L::kA3), 1024, 128);
      constexpr uint32_t ids = instr_desc(kFmtBF16, 128, SbN, false, true);
      constexpr uint32_t ido = instr_desc(kFmtBF16, 64, 128, true, true);
#pragma unroll
      for (int k = 0; k < 4; ++k) mma_bf16(tm + kTmS, kd + 16 * k, ud + (2 * SbL >> 4) * k, ids, 1);
#pragma unroll
      for (int k = 0; k < 4; ++k) mma_bf16(tm + kTmQ, a3 + 128 * k, ud + (2 * SbL >> 4) * k, ido, 1);
      mma_commit(&s_bar);
    }
    if (!block_wait(&s_bar, phase, p.hdr)) { s_abort = 1; break; }
    // ---- S -> bf16 operand for the next chunk (and the fp32 checkpoint, if one
    //      falls after this chunk); O -> global
    {
      float s0[16], s1[16];
      const int col = 32 * cq;
      tmem_ld16(tmem_addr(tm, 32 * q4, kTmS + col), s0);
      tmem_ld16(tmem_addr(tm, 32 * q4, kTmS + col + 16), s1);
      tmem_ld_wait();
      if (float* ck = ckpt_state(p, n, h, c, b - a)) {
        float4* d4 = reinterpret_cast<float4*>(ck + (size_t)srow * kD + col);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          d4[i] = make_float4(s0[4 * i], s0[4 * i + 1], s0[4 * i + 2], s0[4 * i + 3]);
          d4[4 + i] = make_float4(s1[4 * i], s1[4 * i + 1], s1[4 * i + 2], s1[4 * i + 3]);
        }
      }
      st16(sm + L::kSb, mnmaj(col, srow, SbL), s0);
      st16(sm + L::kSb, mnmaj(col + 8, srow, SbL), s0 + 8);
      st16(sm + L::kSb, mnmaj(col + 16, srow, SbL), s1);
      st16(sm + L::kSb, mnmaj(col + 24, srow, SbL), s1 + 8);
      float o0[16], o1[16];
      tmem_ld16(tmem_addr(tm, 32 * q4, kTmQ + col), o0);
      tmem_ld16(tmem_addr(tm, 32 * q4, kTmQ + col + 16), o1);
      tmem_ld_wait();
      const size_t orow = ((size_t)(tok0 + r64) * H + h) * kD;
      if (m64) {
        const float iq = vec[kVecIq + r64];
#pragma unroll
        for (int i = 0; i < 16; ++i) { o0[i] *= iq; o1[i] *= iq; }
      }
      if (p.og) {
        // output epilogue: a token's 128 features lie in the four column quarters
        float* red = vec + kVecY;  // [4 quarters][64 tokens] partial sums of squares
        if (m64) {
          float ss = 0.f;
#pragma unroll
          for (int i = 0; i < 16; ++i) ss += o0[i] * o0[i] + o1[i] * o1[i];
          red[cq * 64 + r64] = ss;
        }
        __syncthreads();
        if (m64 && r64 < len) {
          const float ss = red[r64] + red[64 + r64] + red[128 + r64] + red[192 + r64];
          norm_gate<16>(o0, ss, p.og + orow + col, p.ow ? p.ow + col : nullptr, p.oeps);
          norm_gate<16>(o1, ss, p.og + orow + col + 16, p.ow ? p.ow + col + 16 : nullptr, p.oeps);
        }
      }
      if (m64 && r64 < len) {
        uint4* dst = reinterpret_cast<uint4*>(p.o + orow + col);
        dst[0] = pack8(o0);
        dst[1] = pack8(o0 + 8);
        dst[2] = pack8(o1);
        dst[3] = pack8(o1 + 8);
      }
    }
  }

  // ---- results
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (!s_abort) {
    if (p.S_final && seg == p.P - 1) {
      float* dst = p.S_final + ((size_t)n * H + h) * kD * kD + (size_t)srow * kD;
#pragma unroll
      for (int c16 = 0; c16 < 32; c16 += 16) {
        float s16[16];
        tmem_ld16(tmem_addr(tm, 32 * q4, kTmS + 32 * cq + c16), s16);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; i += 4)
          *reinterpret_cast<float4*>(dst + 32 * cq + c16 + i) = make_float4(s16[i], s16[i + 1], s16[i + 2], s16[i + 3]);
      }
    }
  } else if (raw_pending) {
    // a wait gave up: let the TMA load still in flight land before leaving
    mbar_wait_cycles(&s_bar_raw, phase_raw, kWaitCycles);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, 512);
}

// ---------------------------------------------------------------------------
// Chunk preparation: everything of one (chunk, head) that does not depend on
// the state, left in the chunk's slot for the chain passes.  Persistent: each
// CTA (one per SM; a kernel that uses Tensor Memory gets one CTA per SM) walks
// its share of the (chunk, sequence, head) items, loading the next item's q,
// k, z, v rows by TMA while it finishes the current one.  The 512 threads form
// one group with its own named barriers (the layout allows more groups per CTA
// when registers and shared memory permit).  Warp w covers sub-tile w / 4 and
// 32 channels; each lane owns 8 channels of a token pair, so every row access
// is one 16-byte vector and every operand image is K-major or MN-major such
// that each such vector is one 16-byte row of a core matrix.
// Per (chunk, head): gate and cumulative log-decay (scans within 16-token
// sub-tiles); q/k row norms; sub-tile decay factors; product operands R, C
// and Q', K'; M1 (A products); X_K, X_V; A_kk and A_qk; T = (I + A_kk)^{-1};
// M2 ([W | U~] = T [X_K | X_V]); bulk stores.
constexpr int kPrepGroups = 1;  // 512-thread groups per CTA (each with its own smem part)
constexpr int kPrepThreads = kNT * kPrepGroups;
struct PrepSmem {  // one group's part
  static constexpr int kP = 0;               // region P, reused through the chunk:
  static constexpr int kR = kP;              //   R   B op (N=128 rows, K=128) K-major
  static constexpr int kCc = kP + 32768;     //   C   A op, window b at rows 64 b (K=128) K-major
  static constexpr int kAkk = kP;            //   A_kk fp32 [64][68]  (after M1)
  static constexpr int kTf = kP + 17408;     //   T    fp32 [64][68]
  static constexpr int kY = kP + 34816;      //   merge scratch fp32 [32][34]
  static constexpr int kW = kP;              //   W   slot image   (after M2)
  static constexpr int kUt = kP + 16384;     //   U~  slot image
  static constexpr int kTop = kP + 98304;    // sub-tile sums and first gates, then T (A op, K-major)
  static constexpr int kFac = kTop + 8192;   // decay factors [4 sub-tiles][5][128] fp32
  static constexpr int kNrm = kFac + 10240;  // squared-norm partials [16 channel groups][64][2]
  static constexpr int kVec = kNrm + 8192;   // 1/|q|, 1/|k|, beta (64 floats each)
  static constexpr int kRaw = 125952;        // q | k | z | v, [64 tokens][2 x 64 channels] bf16,
                                             //   128-byte swizzled (TMA), 16 KB each
  static constexpr int kX = kRaw + 65536;    // X B op (N=256, K=64 tokens) MN-major: written
                                             //   while M1 runs
  static constexpr int kGroup = kX + 32768;  // bytes per group
  static constexpr int kBar = kPrepGroups * kGroup;  // per group: two mbarriers; then the TMEM base
  static constexpr int kBytes = kBar + 48;
};
// decay factor rows of sub-tile b (128 channels each): e^{rho_b}, e^{Gam_last - rho_b},
// then e^{rho_c - rho_b} for the later sub-tiles c = b+1 .. 3
constexpr int kFacEr = 0, kFacEl = 1, kFacWin = 2;

// Barrier of one 512-thread group (ids 1 + 4 g .. 4 + 4 g are the group's).
__device__ __forceinline__ void group_sync(int id) {
  asm volatile("bar.sync %0, 512;" ::"r"(id) : "memory");
}
__device__ __forceinline__ bool group_sync_or(int id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 512, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void group_sync_for_mma(int id) {
  fence_async_smem();
  fence_before_sync();
  group_sync(id);
  fence_after_sync();
}
// Group-wide bounded wait on an mbarrier phase; false if it timed out.
__device__ __forceinline__ bool group_wait(uint64_t* bar, uint32_t& phase, WsHeader* hdr, int id,
                                           int gtid) {
  const bool got = mbar_wait_cycles(bar, phase, kWaitCycles);
  phase ^= 1;
  if (group_sync_or(id, !got)) {
    if (gtid == 0) atomicOr(&hdr->err, kErrTimeout);
    return false;
  }
  fence_after_sync();
  return true;
}

__device__ __forceinline__ void st8f(float* p, const float* f) {
  *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(f[4], f[5], f[6], f[7]);
}

template <int GS>
__global__ void __launch_bounds__(kPrepThreads, 1) prep_kernel(const __grid_constant__ TcParams p) {
  using L = PrepSmem;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x;
  const int grp = tid >> 9, gtid = tid & 511;  // group, thread within it
  const int warp = gtid >> 5, lane = tid & 31;
  unsigned char* sm = smem + grp * L::kGroup;
  float* vec = reinterpret_cast<float*>(sm + L::kVec);
  float* fac = reinterpret_cast<float*>(sm + L::kFac);
  uint64_t* bar_mma = reinterpret_cast<uint64_t*>(smem + L::kBar) + 2 * grp;
  uint64_t* bar_raw = bar_mma + 1;
  const unsigned char* raw = sm + L::kRaw;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::kBar + 32);
  const int bid = 1 + 4 * grp;  // the group's barrier: bid; merges: bid + 1, bid + 2, bid + 3
  const int H = p.H;

  if (!seqlens_valid(p.cu, p.N, p.T, p.max_len)) {
    if (blockIdx.x == 0 && tid == 0) atomicOr(&p.hdr->err, kErrBadSeqlens);
    return;
  }
  // the 128-byte swizzle needs 1024-byte aligned destinations
  if (smem_u32(smem) & 1023u) {
    if (tid == 0) atomicOr(&p.hdr->err, kErrTimeout);
    return;
  }
  if (tid < 32) {
    tmem_alloc(s_tmem, 256 * kPrepGroups);
    tmem_relinquish();
  }
  if (gtid == 0) {
    mbar_init(bar_mma, 1);
    mbar_init(bar_raw, 1);
    fence_mbar_init();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = *s_tmem + 256 * grp;  // this group's 256 columns
  uint32_t ph_mma = 0, ph_raw = 0;          // next parity of each barrier
  bool ok = true, raw_pending = false;

  // warp: sub-tile qq (tokens 16 qq ..) and 32 channels; lane: 8 of those
  // channels (group cg) and a token pair of the sub-tile (lanes 8 m .. 8 m + 7
  // share a channel group and scan its 16 tokens)
  const int qq = warp >> 2, pr = lane & 7;
  const int cg = 4 * (warp & 3) + (lane >> 3), c0 = 8 * cg;
  const int t0 = 16 * qq + 2 * pr;          // tokens t0, t0 + 1
  const int sw = pr >> 2;                   // row-store order: conflict-free 16-byte stores
  const int q4 = warp & 3, cq = warp >> 2;  // TMEM lane quarter, 32-column quarter
  const int r64 = 16 * q4 + lane;           // token row of M=64 accumulators (lane < 16)
  const bool m64 = lane < 16;

  // items (chunk c, sequence n, head h), heads fastest; each group takes every
  // (2 * gridDim.x)-th one, stepping the mixed-radix index without divisions
  const int maxch = (p.max_len + kC - 1) / kC;
  const long long it0 = (long long)kPrepGroups * blockIdx.x + grp;
  const long long stride = (long long)kPrepGroups * gridDim.x;
  int h = (int)(it0 % H), n = (int)((it0 / H) % p.N), c = (int)(it0 / ((long long)H * p.N));
  const int sh = (int)(stride % H), sn = (int)((stride / H) % p.N);
  const int sc = (int)(stride / ((long long)H * p.N));
  int a = 0, b = 0;
  // the group's next item that holds tokens, from (c, n, h) on
  auto next_item = [&]() -> bool {
    for (; c < maxch;) {
      seq_bounds(p.cu, n, p.max_len, a, b);
      if (a + c * kC < b) return true;
      h += sh;
      if (h >= H) { h -= H; ++n; }
      n += sn;
      if (n >= p.N) { n -= p.N; ++c; }
      c += sc;
    }
    return false;
  };
  // q, k, z, v rows of an item -> the staging tile (two 64-channel boxes each)
  auto stage = [&](int tok, int hh) {
    mbar_arrive_expect_tx(bar_raw, (GS == kGateZ ? 4 : 3) * 16384);
    tma_box_x(sm + L::kRaw, &p.sq, 0, hh, tok, bar_raw);
    tma_box_x(sm + L::kRaw + 8192, &p.sq, 64, hh, tok, bar_raw);
    tma_box_x(sm + L::kRaw + 16384, &p.sk, 0, hh, tok, bar_raw);
    tma_box_x(sm + L::kRaw + 24576, &p.sk, 64, hh, tok, bar_raw);
    if (GS == kGateZ) {  // z only when the gate is computed from it
      tma_box_x(sm + L::kRaw + 32768, &p.sz, 0, hh, tok, bar_raw);
      tma_box_x(sm + L::kRaw + 40960, &p.sz, 64, hh, tok, bar_raw);
    }
    tma_box_x(sm + L::kRaw + 49152, &p.sv, 0, hh, tok, bar_raw);
    tma_box_x(sm + L::kRaw + 57344, &p.sv, 64, hh, tok, bar_raw);
  };
  // 16-byte row vector (token t, channels c0 .. c0+7) of staged tensor ti
  auto rawv = [&](int ti, int t) -> uint4 {
    return *reinterpret_cast<const uint4*>(raw + ti * 16384 + (cg >> 3) * 8192 + t * 128 +
                                           (((cg & 7) ^ (t & 7)) << 4));
  };
  // beta of an item (thread t < 64: token t), loaded one item ahead
  auto load_beta = [&](int tok, int end, int hh) -> float {
    return (gtid < kC && tok + gtid < end) ? __bfloat162float(p.beta[(size_t)(tok + gtid) * H + hh])
                                           : 0.f;
  };
  bool have = next_item();
  float beta_nx = 0.f;
  if (have) {
    if (gtid == 0) stage(a + c * kC, h);
    raw_pending = true;
    beta_nx = load_beta(a + c * kC, b, h);
  }
  while (ok && have) {
    const int hc = h, nc = n, cc0 = c, ac = a, bc = b;
    h += sh;
    if (h >= H) { h -= H; ++n; }
    n += sn;
    if (n >= p.N) { n -= p.N; ++c; }
    c += sc;
    have = next_item();  // the item after this one (its rows are loaded during this one)
    const int tok0 = ac + cc0 * kC;
    const int len = min(kC, bc - tok0);
    if (gtid < kC) vec[kVecBeta + gtid] = beta_nx;
    if (have) beta_nx = load_beta(a + c * kC, b, h);
    unsigned char* slot = chunk_slot(p.prep, ac, nc, cc0, hc, H);
    const bool in0 = t0 < len, in1 = t0 + 1 < len;
    const size_t row0 = ((size_t)(tok0 + t0) * H + hc) * kD + c0;  // element offset of (t0, c0)
    const size_t rstep = (size_t)H * kD;                          // next token
    const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);

    if (!group_wait(bar_raw, ph_raw, p.hdr, bid, gtid)) {
      ph_raw ^= 1;  // the load is still pending in this phase
      ok = false;
      break;
    }
    raw_pending = false;
    // ---- rows of q and k (16-byte vectors; the token order of the two reads
    //      keeps each 8-lane phase on distinct banks)
    uint4 qa, qb, ka, kb;
    {
      const int ta = t0 + sw, tb = t0 + 1 - sw;
      const uint4 q1 = rawv(0, ta), q2 = rawv(0, tb), k1 = rawv(1, ta), k2 = rawv(1, tb);
      qa = sw ? q2 : q1; qb = sw ? q1 : q2;
      ka = sw ? k2 : k1; kb = sw ? k1 : k2;
      if (!in0) { qa = zero4; ka = zero4; }
      if (!in1) { qb = zero4; kb = zero4; }
    }

    // ---- log-decay gate g of the 16 elements; E[8 s + i]: token t0 + s, channel c0 + i
    float E[16];
    if constexpr (GS == kGateChannel) {
      const float* g0 = p.g + row0;
      if (in0) { ld8f(g0, E); } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) E[i] = 0.f;
      }
      if (in1) { ld8f(g0 + rstep, E + 8); } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) E[8 + i] = 0.f;
      }
    } else if constexpr (GS == kGateHead) {  // one log-decay per token and head
      const float* g0 = p.g + (size_t)(tok0 + t0) * H + hc;
      const float ga = in0 ? g0[0] : 0.f, gb = in1 ? g0[H] : 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) { E[i] = ga; E[8 + i] = gb; }
    } else {
      const float expA = expf(p.A[hc]);
      const uint4 z1 = rawv(2, t0 + sw), z2 = rawv(2, t0 + 1 - sw);
      unpack8(sw ? z2 : z1, E);
      unpack8(sw ? z1 : z2, E + 8);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const bool in = i < 8 ? in0 : in1;
        E[i] = in ? __fdividef(kGateMin, 1.0f + __expf(-expA * E[i])) : 0.f;
      }
    }
    // ---- cumulative log-decay within the sub-tile: scan over its 8 lanes
    float gf[8];  // g of the sub-tile's first token (lane 8 qq, token t0)
    {
      float x[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = E[i] + E[8 + i];  // pair sums
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float y = __shfl_up_sync(0xffffffffu, x[i], off);
          if ((lane & 7) >= off) x[i] += y;
        }
      }
      // x = inclusive sum of the sub-tile through token t0 + 1
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        gf[i] = __shfl_sync(0xffffffffu, E[i], lane & ~7);
        const float g1 = E[8 + i];
        E[8 + i] = x[i];       // through t0 + 1
        E[i] = x[i] - g1;      // through t0
      }
      float* tot = reinterpret_cast<float*>(sm + L::kTop);  // [4][128] sub-tile sums
      float* fst = tot + 512;                               // [4][128] first gates
      if ((lane & 7) == 7) st8f(tot + qq * 128 + c0, x);
      if ((lane & 7) == 0) st8f(fst + qq * 128 + c0, gf);
    }
    // E = e^{Gam_r - rho_qq}, rho_qq = Gam at the sub-tile's first token
#pragma unroll
    for (int i = 0; i < 16; ++i) E[i] = __expf(E[i] - gf[i & 7]);
    // ---- squared row norms of q and k: partial sums over this channel group
    {
      float qf[8], kf[8];
      float4 part;
      unpack8(qa, qf); unpack8(ka, kf);
      part.x = 0.f; part.y = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) { part.x += qf[i] * qf[i]; part.y += kf[i] * kf[i]; }
      unpack8(qb, qf); unpack8(kb, kf);
      part.z = 0.f; part.w = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) { part.z += qf[i] * qf[i]; part.w += kf[i] * kf[i]; }
      *reinterpret_cast<float4*>(sm + L::kNrm + (cg * 64 + t0) * 8) = part;
    }
    // region P is rewritten from here on: the previous item's bulk stores must have read it
    if (gtid == 0) bulk_wait_read();
    group_sync(bid);
    // ---- decay factors of (sub-tile b, channel ch); 1/|q|, 1/|k|; gamma
    {
      const float* tot = reinterpret_cast<const float*>(sm + L::kTop);
      const float* fst = tot + 512;
      const int ch = gtid & 127, bq = gtid >> 7;
      float rho[4], acc = 0.f;
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) {
        rho[bb] = acc + fst[bb * 128 + ch];
        acc += tot[bb * 128 + ch];
      }
      const float rb = bq == 0 ? rho[0] : bq == 1 ? rho[1] : bq == 2 ? rho[2] : rho[3];
      fac[(bq * 5 + kFacEr) * 128 + ch] = __expf(rb);
      fac[(bq * 5 + kFacEl) * 128 + ch] = __expf(acc - rb);
#pragma unroll
      for (int bb = 1; bb < 4; ++bb)
        if (bb > bq) fac[(bq * 5 + kFacWin + bb - bq - 1) * 128 + ch] = __expf(rho[bb] - rb);
      if (bq == 0) reinterpret_cast<float*>(slot + kSlotGam)[ch] = __expf(acc);
      if (gtid < 128) {
        const int t = gtid & 63, w = gtid >> 6;  // token, q (0) or k (1)
        const float* np = reinterpret_cast<const float*>(sm + L::kNrm) + 2 * t + w;
        float ss = 0.f;
#pragma unroll
        for (int g = 0; g < 16; ++g) ss += np[g * 128];
        const float inv = t < len ? rsqrtf(ss + kNormEps) : 0.f;
        vec[(w == 0 ? kVecIq : kVecIk) + t] = inv;
        if (w == 0) reinterpret_cast<float*>(slot + kSlotIq)[t] = inv;
      }
    }
    group_sync(bid);
    // ---- R rows (k e, q e; K-major), Q' = q e^{Gam_r} (norm applied to o), C_b
    //      windows (k e^{rho_b - Gam_r}; K-major)
    {
      const float* fq = fac + qq * 5 * 128 + c0;
      float er[8];
      ld8f(fq + kFacEr * 128, er);
#pragma unroll
      for (int s2 = 0; s2 < 2; ++s2) {
        const int s = s2 ^ sw, t = t0 + s;
        float qf[8], kf[8], w8[8];
        unpack8(s ? qb : qa, qf);
        unpack8(s ? kb : ka, kf);
#pragma unroll
        for (int i = 0; i < 8; ++i) { qf[i] *= (sw ? E[8 * (s2 ^ 1) + i] : E[8 * s2 + i]); w8[i] = kf[i] * (sw ? E[8 * (s2 ^ 1) + i] : E[8 * s2 + i]); }
        const int rr = 32 * qq + (t & 15);  // R row: k rows then q rows of the sub-tile
        st16(sm + L::kR, kmaj(rr, c0, 2048), w8);
        st16(sm + L::kR, kmaj(rr + 16, c0, 2048), qf);
#pragma unroll
        for (int i = 0; i < 8; ++i) qf[i] *= er[i];
        st16(slot + kSlotQ, kmaj(t, c0, 2048), qf);
      }
      // k e^{rho_qq - Gam_r}: window qq as is, later windows times e^{rho_b - rho_qq};
      // K' = k / |k| e^{Gam_last - Gam_r} -> slot (MN-major)
      float el[8];
      ld8f(fq + kFacEl * 128, el);
#pragma unroll
      for (int s2 = 0; s2 < 2; ++s2) {
        const int s = s2 ^ sw, t = t0 + s;
        const float ik = vec[kVecIk + t];
        float kf[8], w8[8];
        unpack8(s ? kb : ka, kf);
#pragma unroll
        for (int i = 0; i < 8; ++i) kf[i] = __fdividef(kf[i], (sw ? E[8 * (s2 ^ 1) + i] : E[8 * s2 + i]));
        st16(sm + L::kCc, kmaj(64 * qq + t, c0, 2048), kf);
        for (int bb = qq + 1; bb < 4; ++bb) {  // warp-uniform
          float f[8];
          ld8f(fq + (kFacWin + bb - qq - 1) * 128, f);
#pragma unroll
          for (int i = 0; i < 8; ++i) w8[i] = kf[i] * f[i];
          st16(sm + L::kCc, kmaj(64 * bb + t, c0, 2048), w8);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) kf[i] *= ik * el[i];
        st16(slot + kSlotK, mnmaj(c0, t, 2048), kf);
      }
    }
    group_sync_for_mma(bid);
    // ---- M1: per K step two M=128, N=64 MMAs (K-major operands): windows (0, 1)
    //      against R sub-tiles (0, 1) -> TMEM columns 0-63, windows (2, 3) against
    //      sub-tiles (2, 3) -> 64-127.  Lanes 0-63 hold window 2 P's rows, 64-127
    //      window 2 P + 1's; of each sub-tile's 32 columns 0-15 are A_kk^T, 16-31
    //      A_qk^T.  Window b is needed against sub-tile b only.
    if (gtid == 0) {
      constexpr uint32_t id = instr_desc(kFmtBF16, 128, 64, false, false);
      const uint64_t ad = smem_desc(smem_u32(sm + L::kCc), 128, 2048);
      const uint64_t bd = smem_desc(smem_u32(sm + L::kR), 128, 2048);
#pragma unroll
      for (int k = 0; k < 8; ++k)  // descriptor addresses count 16-byte units
#pragma unroll
        for (int pr = 0; pr < 2; ++pr)  // two independent accumulators back to back
          mma_bf16(tm + kTmA + 64 * pr, ad + 2048 * pr + 16 * k, bd + 1024 * pr + 16 * k, id, k > 0);
      mma_commit(bar_mma);
    }
    // ---- while M1 runs: X_K = beta k / |k| e^{Gam_r}, X_V = beta v (MN-major)
    {
      const float* fq = fac + qq * 5 * 128 + c0;
      const uint4 v1 = rawv(3, t0 + sw), v2 = rawv(3, t0 + 1 - sw);
      const uint4 va = in0 ? (sw ? v2 : v1) : zero4, vb = in1 ? (sw ? v1 : v2) : zero4;
      float er[8];
      ld8f(fq + kFacEr * 128, er);
#pragma unroll
      for (int s2 = 0; s2 < 2; ++s2) {
        const int s = s2 ^ sw, t = t0 + s;
        const float bet = vec[kVecBeta + t], bik = bet * vec[kVecIk + t];
        float kf[8], vf[8];
        unpack8(s ? kb : ka, kf);
        unpack8(s ? vb : va, vf);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          kf[i] *= bik * (sw ? E[8 * (s2 ^ 1) + i] : E[8 * s2 + i]) * er[i];
          vf[i] *= bet;
        }
        st16(sm + L::kX, mnmaj(c0, t, 4096), kf);
        st16(sm + L::kX, mnmaj(128 + c0, t, 4096), vf);
      }
    }
    if (!group_wait(bar_mma, ph_mma, p.hdr, bid, gtid)) { ok = false; break; }
    // ---- A products -> A_kk (fp32, beta- and norm-scaled, strictly lower) and
    //      A_qk (bf16 slot image, MN-major).  Warp (q4, cq): window bb = 2 (cq / 2) +
    //      q4 / 2, key row i = 32 (q4 % 2) + lane; cq % 2 selects A_kk or A_qk.
    float* Akk = reinterpret_cast<float*>(sm + L::kAkk);
    {
      const int pr = cq >> 1, part = cq & 1, bb = 2 * pr + (q4 >> 1), i = 32 * (q4 & 1) + lane;
      float va[16];
      tmem_ld16(tmem_addr(tm, 32 * q4, kTmA + 64 * pr + 32 * (q4 >> 1) + 16 * part), va);
      tmem_ld_wait();
      const float ki = vec[kVecIk + i];
      if (part == 0) {
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) {
          const int r = 16 * bb + cc;
          Akk[r * kLd + i] = (i < r) ? vec[kVecBeta + r] * vec[kVecIk + r] * ki * va[cc] : 0.f;
        }
      } else {
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) va[cc] = (i <= 16 * bb + cc) ? va[cc] * ki : 0.f;
        st16(slot + kSlotA3, mnmaj(16 * bb, i, 1024), va);
        st16(slot + kSlotA3, mnmaj(16 * bb + 8, i, 1024), va + 8);
      }
    }
    fence_before_sync();
    group_sync(bid);
    // the staged rows are consumed: load the next item's
    if (have) {
      if (gtid == 0) stage(a + c * kC, h);
      raw_pending = true;
    }
    // ---- T = (I + A_kk)^{-1}: 16x16 diagonal blocks by forward substitution,
    //      then merges 16 -> 32 -> 64 ([[P,0],[B,Q]]^{-1} has lower-left block
    //      -Q^{-1} B P^{-1}) on 2x2 register tiles; upper blocks zeroed first.
    float* Tf = reinterpret_cast<float*>(sm + L::kTf);
    float* Y = reinterpret_cast<float*>(sm + L::kY);
    if (gtid < kC) {
      // column cc of block bk: x = e_cc, then x_r -= A[r][m] x_m for m < r (right-looking)
      const int bk = gtid >> 4, cc = gtid & 15, base = 16 * bk;
      float x[16];
#pragma unroll
      for (int rr = 0; rr < 16; ++rr) x[rr] = (rr == cc) ? 1.f : 0.f;
#pragma unroll
      for (int m = 0; m < 15; ++m)
#pragma unroll
        for (int rr = m + 1; rr < 16; ++rr) x[rr] -= Akk[(base + rr) * kLd + base + m] * x[m];
#pragma unroll
      for (int rr = 0; rr < 16; ++rr) Tf[(base + rr) * kLd + base + cc] = x[rr];
    } else {
      // zero T[0:16][16:32] and T[32:48][48:64]
      for (int e = gtid - kC; e < 512; e += kNT - kC) {
        const int blk = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
        Tf[(32 * blk + rr) * kLd + 32 * blk + 16 + cc] = 0.f;
      }
    }
    group_sync(bid);
    if (gtid < 128) {
      // 16 -> 32, pair pr: Y = A[hi][lo] T[lo][lo]; T[hi][lo] = -T[hi][hi] Y (2x2 tiles;
      // the merges are bound by shared-memory loads, which larger tiles reuse)
      const int pr = gtid >> 6, r2 = ((gtid >> 3) & 7) * 2, c2 = (gtid & 7) * 2;
      const int lo = 32 * pr, hi = lo + 16;
      float y[4] = {0.f, 0.f, 0.f, 0.f};
      mm2x2<16>(Akk + (hi + r2) * kLd + lo, Akk + (hi + r2 + 1) * kLd + lo, Tf + lo * kLd + lo + c2,
                kLd, y);
      float* Yp = Y + pr * 16 * 34;
      *reinterpret_cast<float2*>(Yp + r2 * 34 + c2) = make_float2(y[0], y[1]);
      *reinterpret_cast<float2*>(Yp + (r2 + 1) * 34 + c2) = make_float2(y[2], y[3]);
      __syncwarp();
      // this pair's Y rows come from the same two warps: sync those
      asm volatile("bar.sync %0, 64;" ::"r"(bid + 1 + pr) : "memory");
      float t[4] = {0.f, 0.f, 0.f, 0.f};
      mm2x2<16>(Tf + (hi + r2) * kLd + hi, Tf + (hi + r2 + 1) * kLd + hi, Yp + c2, 34, t);
      *reinterpret_cast<float2*>(Tf + (hi + r2) * kLd + lo + c2) = make_float2(-t[0], -t[1]);
      *reinterpret_cast<float2*>(Tf + (hi + r2 + 1) * kLd + lo + c2) = make_float2(-t[2], -t[3]);
    }
    group_sync(bid);
    if (gtid < 256) {
      // 32 -> 64: Y = A[32:64][0:32] T[0:32][0:32]; T[32:64][0:32] = -T[32:64][32:64] Y
      const int r2 = (gtid >> 4) * 2, c2 = (gtid & 15) * 2;
      float y[4] = {0.f, 0.f, 0.f, 0.f};
      mm2x2<32>(Akk + (32 + r2) * kLd, Akk + (33 + r2) * kLd, Tf + c2, kLd, y);
      *reinterpret_cast<float2*>(Y + r2 * 34 + c2) = make_float2(y[0], y[1]);
      *reinterpret_cast<float2*>(Y + (r2 + 1) * 34 + c2) = make_float2(y[2], y[3]);
      asm volatile("bar.sync %0, 256;" ::"r"(bid + 3) : "memory");
      float t[4] = {0.f, 0.f, 0.f, 0.f};
      mm2x2<32>(Tf + (32 + r2) * kLd + 32, Tf + (33 + r2) * kLd + 32, Y + c2, 34, t);
      *reinterpret_cast<float2*>(Tf + (32 + r2) * kLd + c2) = make_float2(-t[0], -t[1]);
      *reinterpret_cast<float2*>(Tf + (33 + r2) * kLd + c2) = make_float2(-t[2], -t[3]);
    } else {
      // meanwhile: the final diagonal halves T[0:32][0:32], T[32:64][32:64] and the
      // zero block T[0:32][32:64] -> bf16 A operand (K-major), 8 columns per vector
      for (int u = gtid - 256; u < 384; u += 256) {
        const int blk = u >> 7, r = (u >> 2) & 31, i0 = (u & 3) * 8;  // blk 0: T11, 1: T22, 2: T12
        const int row = blk == 1 ? 32 + r : r, col = blk == 0 ? i0 : 32 + i0;
        float t8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          t8[i] = (blk < 2 && col + i <= row) ? Tf[row * kLd + col + i] : 0.f;
        st16(sm + L::kTop, kmaj(row, col, 1024), t8);
      }
    }
    group_sync(bid);
    // the merged block T[32:64][0:32] -> bf16 A operand
    if (gtid < 128) {
      const int r = 32 + (gtid >> 2), i0 = (gtid & 3) * 8;
      float t8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) t8[i] = Tf[r * kLd + i0 + i];
      st16(sm + L::kTop, kmaj(r, i0, 1024), t8);
    }
    group_sync_for_mma(bid);
    // ---- M2: W = T X_K (M=64, N=128, K=64; X MN-major) -> columns 0-127, and
    //      U~^T = X_V^T T^T (M=128 value columns, N=64 tokens) -> columns 128-191
    if (gtid == 0) {
      constexpr uint32_t id = instr_desc(kFmtBF16, 64, 128, false, true);
      constexpr uint32_t idu = instr_desc(kFmtBF16, 128, 64, true, false);
      const uint64_t ad = smem_desc(smem_u32(sm + L::kTop), 128, 1024);
      const uint64_t bd = smem_desc(smem_u32(sm + L::kX), 4096, 128);
      const uint64_t xv = smem_desc(smem_u32(sm + L::kX + 2048), 4096, 128);  // X_V, M = value column
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        mma_bf16(tm + kTmWU, ad + 16 * k, bd + 512 * k, id, k > 0);
        mma_bf16(tm + kTmWU + 128, xv + 512 * k, ad + 16 * k, idu, k > 0);
      }
      mma_commit(bar_mma);
    }
    if (!group_wait(bar_mma, ph_mma, p.hdr, bid, gtid)) { ok = false; break; }
    // ---- W and U~^T (bf16 images) -> shared memory -> slot
#pragma unroll
    for (int c16 = 0; c16 < 32; c16 += 16) {
      float w16[16];
      tmem_ld16(tmem_addr(tm, 32 * q4, kTmWU + 32 * cq + c16), w16);
      tmem_ld_wait();
      if (m64) {
        st16(sm + L::kW, kmaj(r64, 32 * cq + c16, 2048), w16);
        st16(sm + L::kW, kmaj(r64, 32 * cq + c16 + 8, 2048), w16 + 8);
      }
    }
    {
      float u16[16];  // U~^T: value column 32 q4 + lane, tokens 16 cq .. 16 cq + 15
      tmem_ld16(tmem_addr(tm, 32 * q4, kTmWU + 128 + 16 * cq), u16);
      tmem_ld_wait();
      uint4* ug = reinterpret_cast<uint4*>(sm + L::kUt);
      ug[ut_index(q4, cq, 0, lane)] = pack8(u16);
      ug[ut_index(q4, cq, 1, lane)] = pack8(u16 + 8);
    }
    group_sync_for_mma(bid);
    if (gtid == 0) {
      bulk_s2g(slot + kSlotW, sm + L::kW, 16384);
      bulk_s2g(slot + kSlotU, sm + L::kUt, 16384);
      bulk_commit();
    }
  }
  if (gtid == 0) {
    bulk_wait_all();
    // a wait gave up: let the row load still in flight land before leaving
    if (raw_pending) (void)mbar_wait_cycles(bar_raw, ph_raw, kWaitCycles);
  }
  fence_before_sync();
  __syncthreads();
  if (tid < 32) tmem_dealloc(*s_tmem, 256 * kPrepGroups);
}

// ---------------------------------------------------------------------------
// Chain passes of a segmented sequence: the state-dependent half of each chunk,
// from the operands in its slot, in transposed form so that the state's value
// columns are the M=128 dimension of the MMAs.  Per chunk:
//   C1: [D_W^T | D_Q^T] = S^T [W ; Q']^T   (M=128 value columns, N=128 tokens),
//       while S <- gamma S (fp32, TMEM) and the previous chunk's o is staged;
//   U^T = U~^T - D_W^T  (bf16, K-major [value column][token]);
//   C2: S += K'^T U  (M=128, N=128);  D_Q^T += U^T A_qk^T  (N=64);
//   o = (D_Q^T)^T / |q|, staged through shared memory during the next C1.
//   TRANS = false: full pass of segment p from its true incoming state; o, S_final.
//   TRANS = true : transition of segments 0..P-2 on [S | X] (256 columns) from
//                  S = 0 (-> N_p) and X = I (-> M_p); C1 is two M=128, N=64 MMAs
//                  per K step (S and X against W); no Q', no output.
// Slot parts are bulk-copied two chunks ahead into two stages.
template <bool TRANS>
struct ChainSmem {
  static constexpr int kSbN = TRANS ? 256 : 128;   // state columns
  static constexpr int kSb = 0;                    // [S | X] bf16, MN-major (M = column, K = dk)
  static constexpr int kU = kSbN * 256;            // U^T bf16, K-major [column][token]
  static constexpr int kO = kU + kSbN * 128;       // o staging [64 tokens][128] bf16 (full pass)
  static constexpr int kIqs = kO + (TRANS ? 0 : 16384);     // 1/|q| of the staged chunk
  static constexpr int kStage = kIqs + (TRANS ? 0 : 256);   // two stages
  // stage layout: the slot (full pass), or W | K' | U~^T | gamma (transition)
  static constexpr int kW = 0, kQ = kSlotQ, kA3 = kSlotA3, kIq = kSlotIq;
  static constexpr int kK = TRANS ? 16384 : kSlotK;
  static constexpr int kUt = TRANS ? 32768 : kSlotU;
  static constexpr int kGam = TRANS ? 32768 + 16384 : kSlotGam;
  static constexpr int kStageBytes = TRANS ? 32768 + 16384 + 512 : kSlotBytes;
  static constexpr int kBytes = kStage + 2 * kStageBytes;
};

template <bool TRANS>
__global__ void __launch_bounds__(kNT, 1) chain_kernel(const __grid_constant__ TcParams p) {
  using L = ChainSmem<TRANS>;
  constexpr int SbN = L::kSbN, SbL = SbN * 16;  // state columns, K-group stride of their copy
  constexpr int NB = SbN / 128;                 // 128-column blocks
  extern __shared__ __align__(1024) unsigned char sm[];
  __shared__ uint64_t s_bar, s_ld[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x, h = blockIdx.y, seg = blockIdx.z;
  const int H = p.H;
  if (!seqlens_valid(p.cu, p.N, p.T, p.max_len)) return;  // the error word is already set
  int a, b;
  seq_bounds(p.cu, n, p.max_len, a, b);
  const int nch = (b - a + kC - 1) / kC;
  int c0, c1;
  segment_chunks(nch, p.P, seg, c0, c1);

  if (warp == 0) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&s_bar, 1);
    mbar_init(&s_ld[0], 1);
    mbar_init(&s_ld[1], 1);
    fence_mbar_init();
    s_abort = 0;
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = s_tmem;
  auto load_slot = [&](int c) {  // single thread
    const int s = (c - c0) & 1;
    unsigned char* dst = sm + L::kStage + s * L::kStageBytes;
    const unsigned char* src = chunk_slot(p.prep, a, n, c, h, H);
    mbar_arrive_expect_tx(&s_ld[s], L::kStageBytes);
    if (TRANS) {
      bulk_g2s(dst, src + kSlotW, 16384, &s_ld[s]);                     // W
      bulk_g2s(dst + L::kK, src + kSlotK, 16384, &s_ld[s]);             // K'
      bulk_g2s(dst + L::kUt, src + kSlotU, 16384 + 512, &s_ld[s]);      // U~^T | gamma
    } else {
      bulk_g2s(dst, src, kSlotBytes, &s_ld[s]);
    }
  };
  if (tid == 0) {
    if (c0 < c1) load_slot(c0);
    if (c0 + 1 < c1) load_slot(c0 + 1);
  }
  uint32_t phase = 0, ph_ld = 0;  // ph_ld bit s: parity of stage s's next completion
  uint32_t inflight = (c0 < c1 ? 1u : 0u) | (c0 + 1 < c1 ? 2u : 0u);  // stages being filled

  const int q4 = warp & 3, cq = warp >> 2;  // TMEM lane quarter, column quarter
  const int srow = 32 * q4 + lane;          // TMEM lane: dk row of S, value column of D^T

  // ---- initial state -> TMEM (fp32) and the bf16 copy: S_in (full pass),
  //      or S = 0 and X = I (transition)
  {
    const float* S0 = nullptr;
    if (!TRANS)
      S0 = seg > 0 ? seg_sin(p.seg, n, h, H, p.Pseg, seg)
                   : (p.S0 ? p.S0 + ((size_t)n * H + h) * kD * kD : nullptr);
#pragma unroll
    for (int blk = 0; blk < NB; ++blk)
#pragma unroll
      for (int c16 = 0; c16 < 32; c16 += 16) {
        float v16[16];
        const int col = 32 * cq + c16;
        if (S0) {
          const float4* src = reinterpret_cast<const float4*>(S0 + (size_t)srow * kD + col);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 f = src[i];
            v16[4 * i] = f.x; v16[4 * i + 1] = f.y; v16[4 * i + 2] = f.z; v16[4 * i + 3] = f.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) v16[i] = (blk == 1 && col + i == srow) ? 1.f : 0.f;
        }
        tmem_st16(tmem_addr(tm, 32 * q4, kTmS + 128 * blk + col), v16);
        st16(sm + L::kSb, mnmaj(128 * blk + col, srow, SbL), v16);
        st16(sm + L::kSb, mnmaj(128 * blk + col + 8, srow, SbL), v16 + 8);
      }
    tmem_st_wait();
  }

  // o of a chunk: D_Q^T (columns dcol + 64 .. dcol + 127) / |q| -> staging [token][value]
  float* iqs = reinterpret_cast<float*>(sm + L::kIqs);
  __nv_bfloat16* ost = reinterpret_cast<__nv_bfloat16*>(sm + L::kO);
  auto stage_o = [&](uint32_t dcol) {
    float v[16];
    tmem_ld16(tmem_addr(tm, 32 * q4, dcol + 64 + 16 * cq), v);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int t = 16 * cq + i;
      ost[t * kD + srow] = __float2bfloat16_rn(v[i] * iqs[t]);
    }
  };
  // o rows of a chunk: 16 lanes per token, 8 features each, kC * kD / 8 / kNT = 2 per thread
  static_assert(kC * kD / 8 == 2 * kNT, "two o vectors per thread");
  uint4 rg[2];  // output-epilogue gate inputs of the rows write_o stores next
  auto load_gate = [&](int cc) {  // issued early; used by write_o(cc)
    if (!p.og) return;
    const int t0c = a + cc * kC, lenc = min(kC, b - t0c);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int u = tid + k * kNT, t = u >> 4, d8 = (u & 15) * 8;
      rg[k] = t < lenc ? *reinterpret_cast<const uint4*>(p.og + ((size_t)(t0c + t) * H + h) * kD + d8)
                       : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  auto write_o = [&](int cc) {  // staging -> o rows of chunk cc (after a barrier)
    const int t0c = a + cc * kC, lenc = min(kC, b - t0c);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int u = tid + k * kNT, t = u >> 4, d8 = (u & 15) * 8;
      const size_t off = ((size_t)(t0c + t) * H + h) * kD + d8;
      uint4 w8 = *reinterpret_cast<const uint4*>(ost + t * kD + d8);
      if (p.og) {  // output epilogue (uniform branch: every lane takes part in the sums)
        float x[8];
        unpack8(w8, x);
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss += x[e] * x[e];
#pragma unroll
        for (int m = 8; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
        norm_gate8(x, rsqrtf(ss * (1.0f / kD) + p.oeps), rg[k], p.ow ? p.ow + d8 : nullptr);
        w8 = pack8(x);
      }
      if (t < lenc) *reinterpret_cast<uint4*>(p.o + off) = w8;
    }
  };

  for (int c = c0; c < c1; ++c) {
    const int s = (c - c0) & 1;
    const uint32_t dcol = (!TRANS && s) ? 128u : 0u;  // this chunk's products (two buffers)
    unsigned char* st = sm + L::kStage + s * L::kStageBytes;
    if (!TRANS && c > c0) load_gate(c - 1);  // in flight until write_o(c - 1) below
    sync_for_mma();
    {
      const bool got = mbar_wait_cycles(&s_ld[s], (ph_ld >> s) & 1, kWaitCycles);
      if (__syncthreads_or(!got)) {
        if (tid == 0) atomicOr(&p.hdr->err, kErrTimeout);
        s_abort = 1;
        break;
      }
      ph_ld ^= 1u << s;
      inflight &= ~(1u << s);
    }
    // ---- C1 (copy of S as the MN-major A operand; W, Q' as the K-major B operand)
    if (tid == 0) {
      const uint64_t bd = smem_desc(smem_u32(st + L::kW), 128, 2048);
      const uint64_t sd = smem_desc(smem_u32(sm + L::kSb), SbL, 128);
      if (!TRANS) {
        constexpr uint32_t id = instr_desc(kFmtBF16, 128, 128, true, false);
#pragma unroll
        for (int k = 0; k < 8; ++k) mma_bf16(tm + dcol, sd + (2 * SbL >> 4) * k, bd + 16 * k, id, k > 0);
      } else {
        constexpr uint32_t id = instr_desc(kFmtBF16, 128, 64, true, false);
        const uint64_t xd = smem_desc(smem_u32(sm + L::kSb + 2048), SbL, 128);  // X columns
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          mma_bf16(tm, sd + (2 * SbL >> 4) * k, bd + 16 * k, id, k > 0);
          mma_bf16(tm + 64, xd + (2 * SbL >> 4) * k, bd + 16 * k, id, k > 0);
        }
      }
      mma_commit(&s_bar);
    }
    // ---- meanwhile: decay the fp32 state by gamma; stage the previous chunk's o
    {
      const float gm = reinterpret_cast<const float*>(st + L::kGam)[srow];
#pragma unroll
      for (int blk = 0; blk < NB; ++blk) {
        float s0[16], s1[16];
        const uint32_t col = kTmS + 128 * blk + 32 * cq;
        tmem_ld16(tmem_addr(tm, 32 * q4, col), s0);
        tmem_ld16(tmem_addr(tm, 32 * q4, col + 16), s1);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) { s0[i] *= gm; s1[i] *= gm; }
        tmem_st16(tmem_addr(tm, 32 * q4, col), s0);
        tmem_st16(tmem_addr(tm, 32 * q4, col + 16), s1);
      }
      tmem_st_wait();
    }
    if (!TRANS && c > c0) stage_o(dcol ^ 128u);
    if (!block_wait(&s_bar, phase, p.hdr)) { s_abort = 1; break; }
    // ---- U^T = U~^T - D_W^T (transition: [U~^T - D_S^T ; -D_X^T]) -> K-major
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
      float d[16];
      tmem_ld16(tmem_addr(tm, 32 * q4, dcol + 64 * blk + 16 * cq), d);
      tmem_ld_wait();
      if (blk == 0) {
        const uint4* ug = reinterpret_cast<const uint4*>(st + L::kUt);
        float u0[8], u1[8];
        unpack8(ug[ut_index(q4, cq, 0, lane)], u0);
        unpack8(ug[ut_index(q4, cq, 1, lane)], u1);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          d[e] = u0[e] - d[e];
          d[8 + e] = u1[e] - d[8 + e];
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) d[e] = -d[e];
      }
      st16(sm + L::kU, kmaj(128 * blk + srow, 16 * cq, 1024), d);
      st16(sm + L::kU, kmaj(128 * blk + srow, 16 * cq + 8, 1024), d + 8);
    }
    sync_for_mma();
    // ---- C2: [S | X] += K'^T U (K' MN-major A, U K-major B); D_Q^T += U^T A_qk^T
    if (tid == 0) {
      const uint64_t kd = smem_desc(smem_u32(st + L::kK), 2048, 128);
      const uint64_t ud = smem_desc(smem_u32(sm + L::kU), 128, 1024);
      constexpr uint32_t ids = instr_desc(kFmtBF16, 128, SbN, true, false);
      const uint64_t a3 = smem_desc(smem_u32(st + L::kA3), 1024, 128);
      constexpr uint32_t ido = instr_desc(kFmtBF16, 128, 64, false, true);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        mma_bf16(tm + kTmS, kd + 256 * k, ud + 16 * k, ids, 1);
        if (!TRANS) mma_bf16(tm + dcol + 64, ud + 16 * k, a3 + 128 * k, ido, 1);
      }
      mma_commit(&s_bar);
    }
    // the previous chunk's o rows (staged before the last barrier) go out while C2 runs
    if (!TRANS && c > c0) write_o(c - 1);
    // the query row scales of this chunk (read before the barrier below, which
    // orders them before the stage's refill)
    if (!TRANS && tid < kC) iqs[tid] = reinterpret_cast<const float*>(st + L::kIq)[tid];
    if (!block_wait(&s_bar, phase, p.hdr)) { s_abort = 1; break; }
    // the stage is consumed (its reads ended before the barrier above): refill it
    if (c + 2 < c1) {
      inflight |= 1u << s;
      if (tid == 0) load_slot(c + 2);
    }
    // ---- [S | X] -> bf16 copy for the next chunk (and the fp32 checkpoint, if one
    //      falls after this chunk)
    float* ck = TRANS ? nullptr : ckpt_state(p, n, h, c, b - a);
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
      float s0[16], s1[16];
      const int col = 128 * blk + 32 * cq;
      tmem_ld16(tmem_addr(tm, 32 * q4, kTmS + col), s0);
      tmem_ld16(tmem_addr(tm, 32 * q4, kTmS + col + 16), s1);
      tmem_ld_wait();
      if (ck) {
        float4* d4 = reinterpret_cast<float4*>(ck + (size_t)srow * kD + col);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          d4[i] = make_float4(s0[4 * i], s0[4 * i + 1], s0[4 * i + 2], s0[4 * i + 3]);
          d4[4 + i] = make_float4(s1[4 * i], s1[4 * i + 1], s1[4 * i + 2], s1[4 * i + 3]);
        }
      }
      st16(sm + L::kSb, mnmaj(col, srow, SbL), s0);
      st16(sm + L::kSb, mnmaj(col + 8, srow, SbL), s0 + 8);
      st16(sm + L::kSb, mnmaj(col + 16, srow, SbL), s1);
      st16(sm + L::kSb, mnmaj(col + 24, srow, SbL), s1 + 8);
    }
  }
  // o of the last chunk
  if (!TRANS && !s_abort && c1 > c0) {
    load_gate(c1 - 1);
    stage_o(((c1 - 1 - c0) & 1) ? 128u : 0u);
    __syncthreads();
    write_o(c1 - 1);
  }

  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (!s_abort) {
    float* dst0 = nullptr;
    if (TRANS)
      dst0 = seg_trans(p.seg, n, h, H, p.Pseg, seg);  // M_p, then N_p
    else if (p.S_final && seg == p.P - 1)
      dst0 = p.S_final + ((size_t)n * H + h) * kD * kD;
    if (dst0) {
#pragma unroll
      for (int blk = 0; blk < NB; ++blk)
#pragma unroll
        for (int c16 = 0; c16 < 32; c16 += 16) {
          float s16[16];
          tmem_ld16(tmem_addr(tm, 32 * q4, kTmS + 128 * blk + 32 * cq + c16), s16);
          tmem_ld_wait();
          // transition: S (block 0) is N_p, X (block 1) is M_p
          float* dst = (TRANS ? dst0 + (blk == 0 ? kD * kD : 0) : dst0) + (size_t)srow * kD + 32 * cq + c16;
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(dst + i) = make_float4(s16[i], s16[i + 1], s16[i + 2], s16[i + 3]);
        }
    }
  } else if (tid == 0) {
    // a wait gave up: let the slot copies still in flight land before leaving
    for (int s = 0; s < 2; ++s)
      if (inflight & (1u << s)) (void)mbar_wait_cycles(&s_ld[s], (ph_ld >> s) & 1, kWaitCycles);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, 512);
}

// Incoming state of every segment: S_in(0) = S0, S_in(p+1) = M_p S_in(p) + N_p.
// One CTA per (n, h, 16-column block of the state); fp32 on CUDA cores.  Each
// M_p (64 KB) is bulk-copied into shared memory one step ahead; the state
// columns are kept transposed so both operands are read as float4.
constexpr int kComposeThreads = 256;
constexpr int kSct = kD + 4;  // row stride (floats) of the transposed state columns
struct ComposeSmem {
  static constexpr int kM = 0;                        // two M_p buffers, [128][128] fp32
  static constexpr int kS = 2 * kD * kD * 4;          // state columns, [16][kSct] fp32
  static constexpr int kBar = kS + 16 * kSct * 4;     // two mbarriers
  static constexpr int kBytes = kBar + 16;
};

// FOLD = false: incoming states S_in(p + 1) = M_p S_in(p) + N_p of segments
// 1 .. P-1 from S_in(0) = S0 (16 state columns per CTA).
// FOLD = true: the transition of the whole sequence, [N | M] = fold over all
// P segments of [N | M] <- M_p [N | M] + [N_p | 0] from [0 | I], written to
// N_out and M_out (16 of the 256 columns of [N | M] per CTA).
template <bool FOLD>
__global__ void __launch_bounds__(kComposeThreads) compose_kernel(const __grid_constant__ TcParams p) {
  using L = ComposeSmem;
  extern __shared__ __align__(1024) unsigned char sm[];
  const int n = blockIdx.x, h = blockIdx.y, cb = blockIdx.z * 16;
  const int H = p.H, tid = threadIdx.x;
  if (!seqlens_valid(p.cu, p.N, p.T, p.max_len)) return;
  float* Sct = reinterpret_cast<float*>(sm + L::kS);  // Sct[cc][r] = S[r][cb + cc]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::kBar);
  const int steps = FOLD ? p.P : p.P - 1;
  const bool addn = !FOLD || cb < kD;  // columns of N take N_p; columns of M do not
  auto load_m = [&](int sg) {  // single thread
    mbar_arrive_expect_tx(&bar[sg & 1], kD * kD * 4);
    bulk_g2s(sm + L::kM + (sg & 1) * kD * kD * 4, seg_trans(p.seg, n, h, H, p.Pseg, sg), kD * kD * 4,
             &bar[sg & 1]);
  };
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0 && steps > 0) load_m(0);
  for (int e = tid; e < kD * 16; e += kComposeThreads) {
    const int r = e >> 4, cc = e & 15;
    if (FOLD)
      Sct[cc * kSct + r] = (cb >= kD && r == cb - kD + cc) ? 1.f : 0.f;
    else
      Sct[cc * kSct + r] = p.S0 ? p.S0[((size_t)n * H + h) * kD * kD + (size_t)r * kD + cb + cc] : 0.f;
  }
  const int c = tid & 15, r0 = tid >> 4;  // column c, rows r0 + 16 m
  uint32_t inflight = steps > 0 ? 1u : 0u;  // buffers being filled
  uint32_t ph = 0;                            // bit b: parity of buffer b's next completion
  bool ok = true;
  // N_p columns, loaded one step ahead
  auto load_n = [&](int sg, float (&v)[8]) {
    const float* Nt = seg_trans(p.seg, n, h, H, p.Pseg, sg) + kD * kD;
#pragma unroll
    for (int m = 0; m < 8; ++m) v[m] = addn ? Nt[(size_t)(r0 + 16 * m) * kD + cb + c] : 0.f;
  };
  float nxt[8];
  if (steps > 0) load_n(0, nxt);
  for (int sg = 0; sg < steps; ++sg) {
    const int buf = sg & 1;
    // M_{sg+1} into the other buffer (its readers finished before the last barrier)
    if (sg + 1 < steps) {
      if (tid == 0) load_m(sg + 1);
      inflight |= 1u << (buf ^ 1);
    }
    float acc[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) acc[m] = nxt[m];
    if (sg + 1 < steps) load_n(sg + 1, nxt);
    const bool got = mbar_wait_cycles(&bar[buf], (ph >> buf) & 1, kWaitCycles);
    if (__syncthreads_or(!got)) {
      if (tid == 0) atomicOr(&p.hdr->err, kErrTimeout);
      ok = false;
      break;
    }
    ph ^= 1u << buf;
    inflight &= ~(1u << buf);
    const float* Ms = reinterpret_cast<const float*>(sm + L::kM + buf * kD * kD * 4);
#pragma unroll 4
    for (int k = 0; k < kD; k += 4) {
      const float4 sv = *reinterpret_cast<const float4*>(Sct + c * kSct + k);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float4 mv = *reinterpret_cast<const float4*>(Ms + (r0 + 16 * m) * kD + k);
        acc[m] += mv.x * sv.x + mv.y * sv.y + mv.z * sv.z + mv.w * sv.w;
      }
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < 8; ++m) Sct[c * kSct + r0 + 16 * m] = acc[m];
    __syncthreads();
    if (!FOLD) {
      float* Sin = seg_sin(p.seg, n, h, H, p.Pseg, sg + 1);
      for (int e = tid; e < kD * 16; e += kComposeThreads) {
        const int r = e >> 4, cc = e & 15;
        Sin[(size_t)r * kD + cb + cc] = Sct[cc * kSct + r];
      }
    }
  }
  if (FOLD && ok) {
    float* dst = (cb < kD ? p.N_out + cb : p.M_out + (cb - kD)) + ((size_t)n * H + h) * kD * kD;
    for (int e = tid; e < kD * 16; e += kComposeThreads) {
      const int r = e >> 4, cc = e & 15;
      dst[(size_t)r * kD + cc] = Sct[cc * kSct + r];
    }
  }
  if (!ok && tid == 0) {
    // a wait gave up: let the copies still in flight land before leaving
    for (int b2 = 0; b2 < 2; ++b2)
      if (inflight & (1u << b2)) (void)mbar_wait_cycles(&bar[b2], (ph >> b2) & 1, kWaitCycles);
  }
}

// cuTensorMapEncodeTiled from the driver, looked up once (no link to libcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

// [T, H, 128] bf16 tensor, box 64 tokens x 1 head x 128 channels; rows past T
// read as zero.
// [T, H, 128] bf16 tensor; box 64 tokens x 1 head x 128 channels, or (swizzled)
// x 64 channels with the 128-byte swizzle
bool make_map(CUtensorMap* map, const void* base, int T, int H, bool swizzled = false) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2};
  const cuuint32_t box[3] = {(cuuint32_t)(swizzled ? kD / 2 : kD), 1, (cuuint32_t)kC};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzled ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_supported(const ForwardArgs& a) {
  return a.bf16 && a.dk == kD && a.dv == kD && a.chunk == kC;
}

int tc_segments(int N, int H, int max_len) {
  // enough (sequence, head, segment) CTAs to fill the 148 SMs; long sequences only
  if (N <= 0 || H <= 0) return 1;
  const long long pairs = (long long)N * H;
  int P = pairs >= 128 ? 1 : (int)(148 / pairs);
  const int nch = (max_len + kC - 1) / kC;
  if (P > nch / 2) P = nch / 2;
  if (P < 1) P = 1;
  if (P > 16) P = 16;
  return P;
}

// Workspace: header | per (n, h) segment transitions and incoming states |
// (segmented only) one chain-operand slot per (chunk, head), 1 KB aligned.
static size_t seg_bytes(int N, int H, int P) {
  const size_t per = (size_t)(P - 1) * 2 * kD * kD + (size_t)P * kD * kD;
  return sizeof(WsHeader) + (size_t)N * H * per * sizeof(float);
}
static size_t prep_offset(int N, int H, int P) { return (seg_bytes(N, H, P) + 1023) & ~(size_t)1023; }

size_t tc_workspace_bytes(int N, int T, int H, int max_len) {
  const int P = tc_segments(N, H, max_len);
  if (P == 1) return seg_bytes(N, H, P);
  const size_t slots = (size_t)T / kC + (size_t)N;
  return prep_offset(N, H, P) + slots * H * kSlotBytes;
}

int tc_launches(int N, int H, int max_len) {
  if (N <= 0) return 0;
  return tc_segments(N, H, max_len) > 1 ? 4 : 1;
}

namespace {

// Kernel parameters of a call; tensor maps only when the call stages inputs.
cudaError_t fill_params(const ForwardArgs& a, TcParams& p, bool maps) {
  memset(&p, 0, sizeof(p));
  if (maps && a.T > 0) {
    const void* zz = a.z ? a.z : a.k;
    if (!make_map(&p.tq, a.q, a.T, a.H) || !make_map(&p.tk, a.k, a.T, a.H) ||
        !make_map(&p.tz, zz, a.T, a.H) || !make_map(&p.tv, a.v, a.T, a.H) ||
        !make_map(&p.sq, a.q, a.T, a.H, true) || !make_map(&p.sk, a.k, a.T, a.H, true) ||
        !make_map(&p.sz, zz, a.T, a.H, true) || !make_map(&p.sv, a.v, a.T, a.H, true))
      return cudaErrorInvalidValue;
  }
  p.beta = (const __nv_bfloat16*)a.beta;
  p.q = (const __nv_bfloat16*)a.q;
  p.k = (const __nv_bfloat16*)a.k;
  p.z = (const __nv_bfloat16*)a.z;
  p.v = (const __nv_bfloat16*)a.v;
  p.A = a.A;
  p.g = a.g_head ? a.g_head : a.g;
  p.S0 = a.S0;
  p.cu = a.cu;
  p.o = (__nv_bfloat16*)a.o;
  p.S_final = a.S_final;
  p.S_ckpt = a.S_ckpt;
  p.ckpt_every = a.ckpt_every;
  p.ckpt_count = a.ckpt_count;
  p.og = (const __nv_bfloat16*)a.out_gate;
  p.ow = a.norm_w;
  p.oeps = a.norm_eps;
  p.N = a.N;
  p.T = a.T;
  p.max_len = a.max_len;
  p.H = a.H;
  p.P = tc_segments(a.N, a.H, a.max_len);
  p.Pseg = p.P;
  p.hdr = (WsHeader*)a.ws;
  p.seg = (float*)((char*)a.ws + sizeof(WsHeader));
  return cudaSuccess;
}

int gate_src(const ForwardArgs& a) {
  return a.g_head ? kGateHead : a.g ? kGateChannel : kGateZ;
}

cudaError_t launch_prep(const TcParams& p, int gs, cudaStream_t st) {
  auto prep = gs == kGateHead ? prep_kernel<kGateHead>
            : gs == kGateChannel ? prep_kernel<kGateChannel> : prep_kernel<kGateZ>;
  cudaError_t err = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         PrepSmem::kBytes);
  if (err != cudaSuccess) return err;
  int sms = 0, dev = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  prep<<<sms, kPrepThreads, PrepSmem::kBytes, st>>>(p);
  return cudaGetLastError();
}

template <bool TRANS>
cudaError_t launch_chain(const TcParams& p, int segments, cudaStream_t st) {
  cudaError_t err = cudaFuncSetAttribute(chain_kernel<TRANS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         ChainSmem<TRANS>::kBytes);
  if (err != cudaSuccess) return err;
  chain_kernel<TRANS><<<dim3(p.N, p.H, segments), kNT, ChainSmem<TRANS>::kBytes, st>>>(p);
  return cudaGetLastError();
}

template <bool FOLD>
cudaError_t launch_compose(const TcParams& p, cudaStream_t st) {
  cudaError_t err = cudaFuncSetAttribute(compose_kernel<FOLD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         ComposeSmem::kBytes);
  if (err != cudaSuccess) return err;
  const int blocks = (FOLD ? 2 * kD : kD) / 16;
  compose_kernel<FOLD><<<dim3(p.N, p.H, blocks), kComposeThreads, ComposeSmem::kBytes, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_forward_tc(const ForwardArgs& a) {
  TcParams p;
  cudaError_t err = fill_params(a, p, true);
  if (err != cudaSuccess) return err;
  const int gs = gate_src(a);
  if (p.P > 1) {
    // chunk preparation -> segment transitions -> incoming states -> chain pass
    p.prep = (unsigned char*)a.ws + prep_offset(a.N, a.H, p.Pseg);
    if ((err = launch_prep(p, gs, a.stream)) != cudaSuccess) return err;
    if ((err = launch_chain<true>(p, p.P - 1, a.stream)) != cudaSuccess) return err;
    if ((err = launch_compose<false>(p, a.stream)) != cudaSuccess) return err;
    return launch_chain<false>(p, p.P, a.stream);
  }
  auto fused = gs == kGateHead ? fused_kernel<kGateHead>
               : gs == kGateChannel ? fused_kernel<kGateChannel> : fused_kernel<kGateZ>;
  err = cudaFuncSetAttribute(fused, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             FusedSmem::kBytes);
  if (err != cudaSuccess) return err;
  fused<<<dim3(a.N, a.H, p.P), kNT, FusedSmem::kBytes, a.stream>>>(p);
  return cudaGetLastError();
}

// Context parallelism.  The workspace holds the segment buffers for P + 1
// segments (room for all P transitions) and the chunk slots, and it carries
// the slots and transitions from the local pass to the finishing pass.
size_t tc_cp_workspace_bytes(int N, int T, int H, int max_len) {
  const int P = tc_segments(N, H, max_len);
  const size_t slots = (size_t)T / kC + (size_t)N;
  return prep_offset(N, H, P + 1) + slots * H * kSlotBytes;
}

int tc_cp_local_launches() { return 3; }
int tc_cp_finish_launches(int N, int H, int max_len) {
  return tc_segments(N, H, max_len) > 1 ? 2 : 1;
}

cudaError_t launch_cp_local_tc(const ForwardArgs& a, float* M_out, float* N_out) {
  TcParams p;
  cudaError_t err = fill_params(a, p, true);
  if (err != cudaSuccess) return err;
  p.Pseg = p.P + 1;
  p.prep = (unsigned char*)a.ws + prep_offset(a.N, a.H, p.Pseg);
  p.M_out = M_out;
  p.N_out = N_out;
  if ((err = launch_prep(p, gate_src(a), a.stream)) != cudaSuccess) return err;
  if ((err = launch_chain<true>(p, p.P, a.stream)) != cudaSuccess) return err;
  return launch_compose<true>(p, a.stream);
}

cudaError_t launch_cp_finish_tc(const ForwardArgs& a) {
  TcParams p;
  cudaError_t err = fill_params(a, p, false);
  if (err != cudaSuccess) return err;
  p.Pseg = p.P + 1;
  p.prep = (unsigned char*)a.ws + prep_offset(a.N, a.H, p.Pseg);
  if (p.P > 1 && (err = launch_compose<false>(p, a.stream)) != cudaSuccess) return err;
  return launch_chain<false>(p, p.P, a.stream);
}

}  // namespace kda
