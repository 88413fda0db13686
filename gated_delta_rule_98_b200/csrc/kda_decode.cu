// kda_decode.cu -- one recurrent KDA step per (sequence, head), in place.
//
// Kimi Linear summary, §6.3: token generation uses the recurrent update; §3:
//   S' = Diag(alpha) S,  u = beta (v - S'^T k^),  S = S' + k^ u^T,  o = S^T q^.
// The output is taken as o = S'^T q^ + (k^ . q^) u, which equals S^T q^ for the
// updated S, so the state is read once and written once: the step is bound by
// the 2 * dk * dv * 4 bytes of state traffic per (sequence, head).
//
// One CTA of 256 threads owns one (b, h) state.  Threads tile the state as
// (row group, float4 column group) so every warp reads and writes whole
// contiguous 512-byte rows; the state lives in registers between the load and
// the store.  Column sums are reduced across row groups through shared memory
// in a fixed order (deterministic, no atomics).
//
// With the input prologue (Kimi Linear summary §4: short convolution and Swish
// on q, k, v) the step also carries each sequence's rolling window of the last
// width - 1 inputs per channel: the convolution of this token reads the window
// and the token's own input, and the window then shifts by one.
#include "kda_common.cuh"
#include "kda_launch.h"

namespace kda {

// Rolling input window of the decode-side prologue (width 0: none).
struct DecodeConv {
  const float *wq, *wk, *wv;  // taps [channels, width], w[c][width - 1] on the current token
  void* state;                // [B, H * (2 dk + dv), width - 1], input dtype
  int width;
};

// Swish(conv) of one channel (taps wc[0 .. W-1]) for this token's input x; the
// window win[0 .. W-2] holds the earlier inputs, oldest first, and is shifted.
template <typename T>
__device__ __forceinline__ float conv_step(const float* wc, T* win, int W, float x) {
  float u = wc[W - 1] * x;
  for (int m = 0; m < W - 1; ++m) u = fmaf(wc[m], to_f(win[m]), u);
  for (int m = 0; m + 1 < W - 1; ++m) win[m] = win[m + 1];
  if (W > 1) win[W - 2] = from_f<T>(x);
  return u / (1.0f + expf(-u));
}

template <int DK, int DV, typename T>
__global__ void __launch_bounds__(256)
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k,
                   const T* __restrict__ v, const T* __restrict__ z,
                   const float* __restrict__ A, const T* __restrict__ beta,
                   float* __restrict__ S, int H, T* __restrict__ o,
                   const T* __restrict__ og, const float* __restrict__ ow, float oeps,
                   const DecodeConv cv) {
  constexpr int NT = 256;
  constexpr int CG = DV / 4;   // float4 column groups per state row
  constexpr int RG = NT / CG;  // row groups
  constexpr int RPT = DK / RG; // state rows held by one thread
  static_assert(RG * CG == NT && RPT * RG == DK, "tiling");

  __shared__ __align__(16) float s_k[DK], s_q[DK], s_a[DK], s_v[DV];
  __shared__ __align__(16) float s_p[RG][DV + 4], s_r[RG][DV + 4];
  __shared__ __align__(16) float s_u[DV];
  __shared__ float s_scal[4];
  __shared__ float s_ss[DV / 32];

  const int bh = blockIdx.x;
  const int h = bh % H;
  const int tid = threadIdx.x;
  const int cg = tid % CG, rg = tid / CG;

  // Issue the state loads first: they are the whole cost of the step.
  float4* Sp = reinterpret_cast<float4*>(S + (size_t)bh * DK * DV);
  float4 s[RPT];
#pragma unroll
  for (int m = 0; m < RPT; ++m) s[m] = __ldcs(&Sp[(rg + m * RG) * CG + cg]);

  const float expA = expf(A[h]);
  if (cv.width > 0) {
    // prologue: the window's channels of (b, h) are q h*DK+i, k H*DK+h*DK+i, v 2*H*DK+h*DV+j
    const int W = cv.width, b = bh / H;
    T* win = reinterpret_cast<T*>(cv.state) + (size_t)b * H * (2 * DK + DV) * (W - 1);
    for (int i = tid; i < DK; i += NT) {
      const int cq = h * DK + i, ck = H * DK + h * DK + i;
      s_q[i] = conv_step(cv.wq + (size_t)cq * W, win + (size_t)cq * (W - 1), W,
                         to_f(q[(size_t)bh * DK + i]));
      s_k[i] = conv_step(cv.wk + (size_t)cq * W, win + (size_t)ck * (W - 1), W,
                         to_f(k[(size_t)bh * DK + i]));
      s_a[i] = expf(gate_logdecay(to_f(z[(size_t)bh * DK + i]), expA));
    }
    for (int j = tid; j < DV; j += NT) {
      const int cvh = h * DV + j, cvw = 2 * H * DK + h * DV + j;
      s_v[j] = conv_step(cv.wv + (size_t)cvh * W, win + (size_t)cvw * (W - 1), W,
                         to_f(v[(size_t)bh * DV + j]));
    }
  } else {
    for (int i = tid; i < DK; i += NT) {
      s_k[i] = to_f(k[(size_t)bh * DK + i]);
      s_q[i] = to_f(q[(size_t)bh * DK + i]);
      s_a[i] = expf(gate_logdecay(to_f(z[(size_t)bh * DK + i]), expA));
    }
    for (int j = tid; j < DV; j += NT) s_v[j] = to_f(v[(size_t)bh * DV + j]);
  }
  __syncthreads();
  if (tid < 32) {
    float kk = 0.f, qq = 0.f, kq = 0.f;
    for (int i = tid; i < DK; i += 32) {
      kk += s_k[i] * s_k[i];
      qq += s_q[i] * s_q[i];
      kq += s_k[i] * s_q[i];
    }
    kk = warp_sum(kk);
    qq = warp_sum(qq);
    kq = warp_sum(kq);
    if (tid == 0) {
      const float ik = 1.0f / sqrtf(kk + kNormEps);
      const float iq = 1.0f / sqrtf(qq + kNormEps);
      s_scal[0] = ik;
      s_scal[1] = iq;
      s_scal[2] = kq * ik * iq;  // k^ . q^
    }
  }
  __syncthreads();
  const float ik = s_scal[0], iq = s_scal[1], kq = s_scal[2];

  // Decay and the two column reductions over this thread's rows.
  float4 p = make_float4(0.f, 0.f, 0.f, 0.f), r = p;
#pragma unroll
  for (int m = 0; m < RPT; ++m) {
    const int i = rg + m * RG;
    const float a = s_a[i], kh = s_k[i] * ik, qh = s_q[i] * iq;
    s[m].x *= a; s[m].y *= a; s[m].z *= a; s[m].w *= a;
    p.x += kh * s[m].x; p.y += kh * s[m].y; p.z += kh * s[m].z; p.w += kh * s[m].w;
    r.x += qh * s[m].x; r.y += qh * s[m].y; r.z += qh * s[m].z; r.w += qh * s[m].w;
  }
  *reinterpret_cast<float4*>(&s_p[rg][4 * cg]) = p;
  *reinterpret_cast<float4*>(&s_r[rg][4 * cg]) = r;
  __syncthreads();
  const float b = to_f(beta[bh]);
  static_assert(DV <= NT, "one output feature per thread");
  float oj = 0.f;
  if (tid < DV) {
    float pj = 0.f, rj = 0.f;
#pragma unroll
    for (int g2 = 0; g2 < RG; ++g2) {
      pj += s_p[g2][tid];
      rj += s_r[g2][tid];
    }
    const float u = b * (s_v[tid] - pj);
    s_u[tid] = u;
    oj = rj + kq * u;
  }
  if (og) {
    // output epilogue (Kimi Linear summary, §4): head-wise RMSNorm over the DV
    // outputs, gain, sigmoid gate; the sum of squares is reduced over the DV / 32 warps
    const float ss = warp_sum(oj * oj);  // zero beyond DV
    if (tid < DV && (tid & 31) == 0) s_ss[tid >> 5] = ss;
    __syncthreads();
    if (tid < DV) {
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < DV / 32; ++w) tot += s_ss[w];
      const float wj = ow ? ow[tid] : 1.f;
      oj = oj * rsqrtf(tot * (1.0f / DV) + oeps) * wj * out_sigmoid(to_f(og[(size_t)bh * DV + tid]));
    }
  }
  if (tid < DV) o[(size_t)bh * DV + tid] = from_f<T>(oj);
  __syncthreads();
  const float4 u4 = *reinterpret_cast<const float4*>(&s_u[4 * cg]);
#pragma unroll
  for (int m = 0; m < RPT; ++m) {
    const int i = rg + m * RG;
    const float kh = s_k[i] * ik;
    float4 w = s[m];
    w.x += kh * u4.x; w.y += kh * u4.y; w.z += kh * u4.z; w.w += kh * u4.w;
    __stcs(&Sp[i * CG + cg], w);
  }
}

template <int DK, int DV, typename T>
static cudaError_t launch_decode_t(const DecodeArgs& a) {
  decode_step_kernel<DK, DV, T><<<a.B * a.H, 256, 0, a.stream>>>(
      (const T*)a.q, (const T*)a.k, (const T*)a.v, (const T*)a.z, a.A,
      (const T*)a.beta, a.S, a.H, (T*)a.o, (const T*)a.out_gate, a.norm_w, a.norm_eps,
      DecodeConv{a.conv_wq, a.conv_wk, a.conv_wv, a.conv_state, a.conv_width});
  return cudaGetLastError();
}

template <int DK, int DV>
static cudaError_t launch_decode_d(const DecodeArgs& a) {
  return a.bf16 ? launch_decode_t<DK, DV, __nv_bfloat16>(a) : launch_decode_t<DK, DV, float>(a);
}

template <int DK>
static cudaError_t launch_decode_k(const DecodeArgs& a) {
  switch (a.dv) {
    case 32: return launch_decode_d<DK, 32>(a);
    case 64: return launch_decode_d<DK, 64>(a);
    case 128: return launch_decode_d<DK, 128>(a);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const DecodeArgs& a) {
  switch (a.dk) {
    case 32: return launch_decode_k<32>(a);
    case 64: return launch_decode_k<64>(a);
    case 128: return launch_decode_k<128>(a);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kda
