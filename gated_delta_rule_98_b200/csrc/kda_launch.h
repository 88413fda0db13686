// kda_launch.h -- host-side launch descriptors shared by the API layer and the
// kernel translation units (internal; not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kda {

struct DecodeArgs {
  const void *q, *k, *v, *z, *beta;
  const float* A;
  float* S;
  void* o;
  int B, H, dk, dv;
  bool bf16;
  cudaStream_t stream;
  const void* out_gate = nullptr;  // [B, H, dv] sigmoid output-gate input (input dtype), or null
  const float* norm_w = nullptr;   // [dv] RMSNorm gain, or null (ones)
  float norm_eps = 0.f;
  // Input prologue (conv_width > 0): q, k, v are the convolution's inputs of
  // this token, conv_wq/wk/wv [channels, conv_width] its taps and conv_state
  // [B, H * (2 dk + dv), conv_width - 1] (input dtype) the rolling window of
  // earlier inputs, updated in place.
  const float *conv_wq = nullptr, *conv_wk = nullptr, *conv_wv = nullptr;
  void* conv_state = nullptr;
  int conv_width = 0;
};

struct ForwardArgs {
  const void *q, *k, *v, *z, *beta;
  const float* A;        // with z
  const float* g;        // log-decay input (instead of z, A) or nullptr
  const float* S0;       // nullptr = zeros
  const int32_t* cu;     // nullptr = equal lengths
  void* o;
  float* S_final;        // nullptr = skip
  int N, T, max_len, H, dk, dv, chunk;
  bool bf16;
  void* ws;              // workspace base (header at offset 0)
  size_t ws_bytes;
  cudaStream_t stream;
  float* S_ckpt = nullptr;  // [N, H, ckpt_count, dk, dv] states every ckpt_every chunks, or null
  int ckpt_every = 0;       // chunks between checkpoints
  int ckpt_count = 0;       // checkpoints per (sequence, head): max_len / interval
  // Output epilogue (head-wise RMSNorm over dv, gain, sigmoid gate) on o, when out_gate is set.
  const void* out_gate = nullptr;  // [T, H, dv] gate input (input dtype)
  const float* norm_w = nullptr;   // [dv] gain, or null (ones)
  float norm_eps = 0.f;
  // Scalar gate (Gated DeltaNet): [T, H] fp32 log-decay shared by a head's dk
  // channels, instead of z, A and g.
  const float* g_head = nullptr;
  // Input prologue fused into the chunk preparation (tensor-core path, KDA
  // gate): q, k, v are the short convolution's inputs and these its
  // [channels, conv_width] fp32 taps.  conv_width 0: q, k, v as given.
  const float *conv_wq = nullptr, *conv_wk = nullptr, *conv_wv = nullptr;
  int conv_width = 0;
};

// Input prologue: causal depthwise short convolution per sequence + Swish.
struct ConvTensor {
  const void* x;   // [T, channels] input (dtype of the call)
  const float* w;  // [channels, width] taps, w[c][width-1] on the current token
  void* y;         // [T, channels] output
  int channels;    // a multiple of 8
};
struct ConvArgs {
  ConvTensor t[3];
  int ntensors;
  const int32_t* cu;  // nullptr = N equal sequences of L tokens
  int N, T, L, width;
  bool bf16;
  cudaStream_t stream;
};
cudaError_t launch_conv_swish(const ConvArgs& a);

cudaError_t launch_decode(const DecodeArgs& a);

// SIMT (CUDA-core, fp32) chunkwise path: any supported size and dtype.
size_t simt_workspace_bytes(int N, int T, int H, int dk, int dv, int chunk);
cudaError_t launch_forward_simt(const ForwardArgs& a);
int simt_launches(int N, int max_len, int chunk);

// Tensor-core (tcgen05) chunkwise path: bf16, dk = dv = 128, chunk = 64.
bool tc_supported(const ForwardArgs& a);
int tc_segments(int N, int H, int max_len);
size_t tc_workspace_bytes(int N, int T, int H, int max_len);
int tc_launches(int N, int H, int max_len);
cudaError_t launch_forward_tc(const ForwardArgs& a);
// Limit (SM cycles) of the tensor-core kernels' first-giving-up waits; <= 0
// restores the default (about 2 s).  A test hook: the timeout path.
void tc_set_wait_limit(long long cycles);

// Context parallelism on the tensor-core path: the local pass (chunk
// preparation, the transitions of all local segments, their fold into one
// transition (M, N) per sequence and head) and the finishing pass (incoming
// states of the local segments from S_in = a.S0, then the full chain pass).
size_t tc_cp_workspace_bytes(int N, int T, int H, int max_len);
int tc_cp_local_launches();
int tc_cp_finish_launches(int N, int H, int max_len);
cudaError_t launch_cp_local_tc(const ForwardArgs& a, float* M_out, float* N_out);
cudaError_t launch_cp_finish_tc(const ForwardArgs& a);

// S_out[i] = M[i] S_in[i] + Nt[i] for count (dk x dk, dk x dv) pairs, fp32.
cudaError_t launch_state_compose(const float* M, const float* Nt, const float* S_in, float* S_out,
                                 int count, int dk, int dv, cudaStream_t stream);

}  // namespace kda
