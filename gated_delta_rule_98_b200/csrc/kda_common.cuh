// kda_common.cuh -- device helpers shared by the KDA kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// Lower bound of the log-decay gate (Kimi K3 architecture summary: g_min = -5).
constexpr float kGateMin = -5.0f;
// Epsilon inside the root of the unit-length normalisation of q and k.
constexpr float kNormEps = 1e-6f;
// Token sub-tile of the chunkwise algorithm: 16 tokens x (g >= -5) keeps the
// cumulative log-decay of a sub-tile within [-80, 0].
constexpr int kSubTile = 16;

// Device error word values (workspace offset 0).
constexpr uint32_t kErrNone = 0u;
constexpr uint32_t kErrBadSeqlens = 1u;
constexpr uint32_t kErrTimeout = 2u;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// g = g_min * sigmoid(e^{A} z) = g_min / (1 + exp(-e^{A} z)); expA = exp(A_h).
__device__ __forceinline__ float gate_logdecay(float z, float expA) {
  return kGateMin / (1.0f + expf(-expA * z));
}

// Output gate of the epilogue: sigmoid(x) = 1 / (1 + e^{-x}), with the fast
// exponential and division (a few ulp; 0 once e^{-x} overflows).
__device__ __forceinline__ float out_sigmoid(float x) {
  return __fdividef(1.0f, 1.0f + __expf(-x));
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Chunk table entry: one chunk of one sequence.
struct ChunkInfo {
  int32_t tok0;   // first token (packed index)
  int32_t len;    // tokens in this chunk, 1..C
  int32_t seq;    // sequence index
  int32_t first;  // 1 if this is the sequence's first chunk
};

// Token range [a, b) of sequence n: from cu_seqlens, or n * L for equal lengths.
__device__ __forceinline__ void seq_bounds(const int32_t* cu, int n, int L, int& a, int& b) {
  if (cu) {
    a = cu[n];
    b = cu[n + 1];
  } else {
    a = n * L;
    b = a + L;
  }
}

// Every CTA checks the whole cu_seqlens (0 = cu[0] <= ... <= cu[N] = T, every
// length <= max_len), so all CTAs of a launch agree on skipping.  Block-wide.
__device__ __forceinline__ bool seqlens_valid(const int32_t* cu, int N, int T, int max_len) {
  if (!cu) return true;
  int bad = 0;
  for (int n = threadIdx.x; n < N; n += blockDim.x) {
    const int a = cu[n], b = cu[n + 1];
    if (b < a || b - a > max_len) bad = 1;
  }
  if (threadIdx.x == 0 && (cu[0] != 0 || cu[N] != T)) bad = 1;
  return __syncthreads_or(bad) == 0;
}

// Workspace header (offset 0, 256 bytes).
struct WsHeader {
  uint32_t err;
  int32_t num_chunks;
  int32_t pad[62];
};

}  // namespace kda
