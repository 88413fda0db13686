// kda_prologue.cu -- the layer's input prologue: a causal depthwise short
// convolution along the tokens of each sequence, then Swish, on the q, k and v
// inputs of KDA (Kimi Linear summary, §4 "The Kimi Linear Model Architecture":
// a short convolution for neighbouring-token dependencies and a Swish
// nonlinearity on queries, keys and values; the unit-length normalisation of
// q and k that follows is part of the operator).
//
//   u[t,c] = sum_{i<W} w[c,i] * x[t-(W-1)+i, c]   (x = 0 before the sequence's first token)
//   y[t,c] = u[t,c] * sigmoid(u[t,c])
//
// HBM-bound: one read and one write of each element.  A thread owns 8
// consecutive channels (one 16-byte bf16 vector) of a run of kTokens tokens
// and slides a W-1 token window along them in registers, so each input row is
// read once per run plus W-1 halo rows; a warp covers 256 consecutive channels
// of one token (512 contiguous bytes in bf16).  The three tensors are one
// launch (blockIdx.z).
#include "kda_common.cuh"
#include "kda_launch.h"

namespace kda {

namespace {

constexpr int kTokens = 64;  // tokens per thread run
constexpr int kGroup = 4;    // token rows loaded together
constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ void ld8(const T* p, float* f);
template <>
__device__ __forceinline__ void ld8<__nv_bfloat16>(const __nv_bfloat16* p, float* f) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
  f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
  f[4] = __uint_as_float(u.z << 16); f[5] = __uint_as_float(u.z & 0xffff0000u);
  f[6] = __uint_as_float(u.w << 16); f[7] = __uint_as_float(u.w & 0xffff0000u);
}
template <>
__device__ __forceinline__ void ld8<float>(const float* p, float* f) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

template <typename T>
__device__ __forceinline__ void st8(T* p, const float* f);
template <>
__device__ __forceinline__ void st8<__nv_bfloat16>(__nv_bfloat16* p, const float* f) {
  uint4 u;
  __nv_bfloat162 a = __floats2bfloat162_rn(f[0], f[1]), b = __floats2bfloat162_rn(f[2], f[3]),
                  c = __floats2bfloat162_rn(f[4], f[5]), d = __floats2bfloat162_rn(f[6], f[7]);
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  u.z = *reinterpret_cast<uint32_t*>(&c);
  u.w = *reinterpret_cast<uint32_t*>(&d);
  *reinterpret_cast<uint4*>(p) = u;
}
template <>
__device__ __forceinline__ void st8<float>(float* p, const float* f) {
  *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(f[4], f[5], f[6], f[7]);
}

// First token of the sequence holding token t, clamped into [0, t] so every
// read stays inside the tensor even when cu_seqlens is malformed (the forward
// reports that case; the prologue's output is then unused).
__device__ __forceinline__ int seq_start(const int32_t* cu, int N, int L, int t) {
  if (!cu) return L > 0 ? (t / L) * L : 0;
  int lo = 0, hi = N - 1;  // largest s in [0, N-1] with cu[s] <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return min(max(cu[lo], 0), t);
}

// First sequence boundary after token t (the first cu entry above t), clamped
// into [t + 1, T].
__device__ __forceinline__ int next_boundary(const int32_t* cu, int N, int L, int T, int start,
                                             int t) {
  if (!cu) return L > 0 ? min(start + L, T) : T;
  int lo = 0, hi = N;  // first m in [0, N) with cu[m] > t, else N
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (cu[mid] > t) hi = mid; else lo = mid + 1;
  }
  return min(max(cu[lo], t + 1), T);
}

// Swish u * sigmoid(u).  For bf16 outputs as u * (1/2 + tanh(u/2)/2) with the
// hardware tanh approximation (one MUFU operation instead of an exponential
// and a division; its relative error, about 2^-11, is below bf16's 2^-9); for
// fp32 outputs with the exponential and division.
template <typename T>
__device__ __forceinline__ float swish(float u);
template <>
__device__ __forceinline__ float swish<__nv_bfloat16>(float u) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * u));
  return fmaf(0.5f * u, t, 0.5f * u);
}
template <>
__device__ __forceinline__ float swish<float>(float u) {
  return u * out_sigmoid(u);
}

template <typename T, int W>
__global__ void __launch_bounds__(kThreads) conv_swish_kernel(ConvArgs a) {
  const ConvTensor& ct = a.t[blockIdx.z];
  const int nvec = ct.channels / 8;
  const int vec = blockIdx.x * kThreads + threadIdx.x;
  const int t0 = blockIdx.y * kTokens;
  if (vec >= nvec || t0 >= a.T) return;
  const int t1 = min(t0 + kTokens, a.T);
  const size_t C = (size_t)ct.channels;
  const T* x = (const T*)ct.x + (size_t)vec * 8;
  T* y = (T*)ct.y + (size_t)vec * 8;

  float w[8][W];
#pragma unroll
  for (int e = 0; e < 8; ++e)
#pragma unroll
    for (int i = 0; i < W; ++i) w[e][i] = ct.w[((size_t)vec * 8 + e) * W + i];

  // window: win[j] = x of token t-(W-1)+j for the next token t (zeros before the start)
  float win[W > 1 ? W - 1 : 1][8];
  int start = seq_start(a.cu, a.N, a.L, t0);
#pragma unroll
  for (int j = 0; j < W - 1; ++j) {
    const int s = t0 - (W - 1) + j;
    if (s >= start) {
      ld8<T>(x + (size_t)s * C, win[j]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) win[j][e] = 0.f;
    }
  }
  int next = next_boundary(a.cu, a.N, a.L, a.T, start, t0);

  // groups of kGroup tokens: their rows are loaded together (independent
  // loads in flight) before the window slides over them
  for (int tg = t0; tg < t1; tg += kGroup) {
    float xr[kGroup][8];
#pragma unroll
    for (int j = 0; j < kGroup; ++j) {
      if (tg + j < t1) {
        ld8<T>(x + (size_t)(tg + j) * C, xr[j]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) xr[j][e] = 0.f;
      }
    }
#pragma unroll
    for (int j = 0; j < kGroup; ++j) {
      const int t = tg + j;
      if (t >= t1) break;
      if (t >= next) {  // a new sequence starts at t: the window restarts from zeros
#pragma unroll
        for (int i = 0; i < W - 1; ++i)
#pragma unroll
          for (int e = 0; e < 8; ++e) win[i][e] = 0.f;
        start = seq_start(a.cu, a.N, a.L, t);
        next = next_boundary(a.cu, a.N, a.L, a.T, start, t);
      }
      float u[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float acc = w[e][W - 1] * xr[j][e];
#pragma unroll
        for (int i = 0; i < W - 1; ++i) acc = fmaf(w[e][i], win[i][e], acc);
        u[e] = swish<T>(acc);
      }
      st8<T>(y + (size_t)t * C, u);
      // slide the window by one token
#pragma unroll
      for (int i = 0; i < W - 1; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) win[i][e] = (i + 1 < W - 1) ? win[i + 1][e] : xr[j][e];
    }
  }
}

template <typename T>
cudaError_t launch_t(const ConvArgs& a) {
  int maxc = 0;
  for (int i = 0; i < a.ntensors; ++i) maxc = max(maxc, a.t[i].channels);
  dim3 grid((maxc / 8 + kThreads - 1) / kThreads, (a.T + kTokens - 1) / kTokens, a.ntensors);
  switch (a.width) {
    case 1: conv_swish_kernel<T, 1><<<grid, kThreads, 0, a.stream>>>(a); break;
    case 2: conv_swish_kernel<T, 2><<<grid, kThreads, 0, a.stream>>>(a); break;
    case 3: conv_swish_kernel<T, 3><<<grid, kThreads, 0, a.stream>>>(a); break;
    case 4: conv_swish_kernel<T, 4><<<grid, kThreads, 0, a.stream>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_conv_swish(const ConvArgs& a) {
  if (a.T <= 0 || a.ntensors <= 0) return cudaSuccess;
  return a.bf16 ? launch_t<__nv_bfloat16>(a) : launch_t<float>(a);
}

}  // namespace kda
