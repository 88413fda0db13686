// kda_tc_common.cuh -- pieces shared by the tensor-core prefill kernels
// (chunk preparation in kda_prep_tc.cu; chain passes and composition in
// kda_prefill_tc.cu): kernel parameters, the chunk-slot format the
// preparation leaves for the chain passes, bf16 operand-image addressing, TMA
// box loads and bounded block-wide waits.  Internal; not part of the C ABI.
//
// Operand images.  Every MMA operand the kernels build is an "image" of 16-byte
// units, each unit holding 8 consecutive tokens of one channel (or 8
// consecutive query rows of one key column).  An image of R token rows and 128
// channels places (token t, channel c) at
//   (c / 8) * (R * 16) + (t / 8) * 128 + (c % 8) * 16 + (t % 8) * 2
// so that, in the no-swizzle core-matrix form of the tcgen05 descriptors, the
// same bytes serve as an MN-major operand with the tokens as M or N
// (SBO = 128, LBO = R * 16) and as a K-major operand with the tokens as K
// (LBO = 128, SBO = R * 16).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cuda_fp16.h>

#include "kda_common.cuh"
#include "kda_launch.h"
#include "tc_sm100.cuh"

namespace kda {
namespace tcp {

using namespace tc;

constexpr int kC = 64;    // chunk tokens
constexpr int kD = 128;   // dk = dv
constexpr int kNT = 512;  // threads of the preparation and chain kernels (16 warps)

constexpr long long kWaitCycles = 4000000000LL;  // ~2 s: a wait this long is a fault

// Byte offset of (token t, channel c) in an operand image of `rows` token rows.
__host__ __device__ constexpr uint32_t img(int t, int c, int rows) {
  return (uint32_t)((c >> 3) * (rows * 16) + (t >> 3) * 128 + (c & 7) * 16 + (t & 7) * 2);
}
// Byte offset of the 16-byte unit holding tokens t0 .. t0+7 (t0 % 8 == 0) of channel c.
__host__ __device__ constexpr uint32_t img_unit(int t0, int c, int rows) {
  return (uint32_t)((c >> 3) * (rows * 16) + (t0 >> 3) * 128 + (c & 7) * 16);
}
// The same units ordered token group first (a 128-channel image): group t0 / 8
// of 8 tokens occupies 2 KB, so any run of token groups is contiguous; as an
// MN-major operand with the tokens as N: LBO = 128 (channel groups), SBO = 2048.
__host__ __device__ constexpr uint32_t img_tg(int t0, int c) {
  return (uint32_t)((t0 >> 3) * 2048 + (c >> 3) * 128 + (c & 7) * 16);
}

// Chain operands of one (chunk, head), written by the preparation kernel and
// read by the chain passes with bulk copies.  The images are f16 (10-bit
// mantissa): every chain operand is bounded (the decay factors are at most 1
// and the state is non-expansive), so f16 holds them with 8x less rounding
// than bf16; values below the f16 range flush towards zero (absolute error
// under 1e-7) and out-of-range ones would saturate.
//   WQ   [Q' ; W] as one 128-row token-group-first image (img_tg: Q' tokens
//        0..63 in the first 16 KB, W tokens 64..127 in the next), the B operand
//        of C1 (N = 128 tokens, K = dk; the transition pass reads the W half), MN-major.
//   K    K' (64-row image): the B operand of the state update in C2 (N = key
//        channel, K = token), K-major; directly followed by A, so that
//        [K' | A_qk^T] is one B operand with N = 192.
//   A    A_qk with key column i as the "token" and query row r as the channel
//        (64 x 64): the B operand A_qk^T of the output update (N = r, K = i),
//        K-major.
//   U    U~^T (bf16 [dv][token]) in the order the chain threads read it (ut_index).
//   Gam  gamma = e^{Gam_last} per key channel (128 fp32); Iq 1/|q| per token (64 fp32).
constexpr int kSlotWQ = 0, kSlotK = 32768, kSlotA = 49152, kSlotU = 57344, kSlotGam = 73728,
              kSlotIq = 74240, kSlotBytes = 74496;
static_assert(kSlotU + 16384 == kSlotGam && kSlotGam + 512 == kSlotIq, "slot layout");
static_assert(kSlotK + 16384 == kSlotA, "[K' | A_qk^T] is one operand");

// 16-byte unit of U~^T (value column 32 q4 + l; tokens 16 cq + 8 half .. +7) in
// a slot: warp (q4, cq) reads 512 consecutive bytes per vector.
__host__ __device__ constexpr int ut_index(int q4, int cq, int half, int l) {
  return ((cq * 4 + q4) * 2 + half) * 32 + l;
}

// Chunk c of sequence n (first token a) has slot a / C + n + c: distinct for
// every chunk of every sequence and below T / C + N.
__device__ __forceinline__ unsigned char* chunk_slot(const unsigned char* prep_base, int a, int n,
                                                     int c, int h, int H) {
  return const_cast<unsigned char*>(prep_base) +
         ((size_t)(a / 64 + n + c) * H + h) * (size_t)kSlotBytes;
}

struct alignas(64) TcParams {
  // [T, H, 128] bf16, box 64 tokens x 1 x 64 channels, 128-byte swizzle (q, k,
  // v: 72 tokens from 8 before the chunk when the input prologue runs in the preparation)
  CUtensorMap sq, sk, sz, sv;
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
  float* seg;           // per (n, h): transitions (M, N) of segments 0..P-2, incoming states of 0..P-1
  unsigned char* prep;  // per (chunk slot, h): chain operands left by the preparation
  WsHeader* hdr;
  // Context parallelism: the segment buffers are laid out for Pseg segments
  // (P, or P + 1 so that all P transitions fit); M_out, N_out receive the
  // folded transition of each (sequence, head) when set.
  int Pseg;
  float *M_out, *N_out;
  // Limit (SM cycles) of the waits that can give up first; the waits that let
  // in-flight copies and MMAs land before a kernel leaves use kWaitCycles.
  long long wait_limit;
  // Input prologue in the preparation (cw > 0): q, k, v are the inputs of the
  // short convolution, cwq, cwk [H * 128, cw] and cwv [H * 128, cw] its taps.
  const float *cwq, *cwk, *cwv;
  int cw;
};

// Where the log-decay comes from (a template parameter of the preparation, so
// each variant carries only its own code): the KDA gate from z and A; given per
// channel (g [T, H, 128]); given once per token and head (g [T, H], the scalar
// gate of Gated DeltaNet, broadcast over the channels).
enum GateSrc : int { kGateZ = 0, kGateChannel = 1, kGateHead = 2 };

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

// One TMA box at channel offset x (a multiple of 64) of a [T, H, 128] tensor.
__device__ __forceinline__ void tma_box_x(void* dst, const CUtensorMap* map, int x, int h, int tok0,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(h), "r"(tok0), "r"(smem_u32(bar))
      : "memory");
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
// Two fp32 -> one f16x2 word (lo in the low half), rounded to nearest, values
// beyond the f16 range clamped to +-65504.
__device__ __forceinline__ uint32_t h2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint4 pack8h(const float* v) {
  return make_uint4(h2(v[0], v[1]), h2(v[2], v[3]), h2(v[4], v[5]), h2(v[6], v[7]));
}
// 8 f16 (one 16-byte vector) -> fp32, exactly
__device__ __forceinline__ void unpack8h(const uint4 u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    f[2 * i] = x.x;
    f[2 * i + 1] = x.y;
  }
}
__device__ __forceinline__ void ld8f(const float* p, float* f) {  // 8 fp32, 16-byte aligned
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// Block-wide bounded wait on an mbarrier phase (at most `limit` SM cycles); false
// if it timed out (the error word then carries kErrTimeout and `phase` still
// names the pending phase, for the drain before the kernel leaves).
__device__ __forceinline__ bool block_wait(uint64_t* bar, uint32_t& phase, WsHeader* hdr,
                                           long long limit) {
  const bool got = mbar_wait_cycles(bar, phase, limit);
  if (__syncthreads_or(!got)) {
    if (threadIdx.x == 0) atomicOr(&hdr->err, kErrTimeout);
    return false;
  }
  phase ^= 1;
  fence_after_sync();
  return true;
}

__device__ __forceinline__ void sync_for_mma() {
  fence_async_smem();
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
}

// Launcher of the preparation kernel (kda_prep_tc.cu): one persistent CTA per SM.
cudaError_t launch_prep_tc(const TcParams& p, int gate_src, cudaStream_t st);
size_t prep_tc_smem_bytes();

}  // namespace tcp
}  // namespace kda
