// kda_api.cu -- the C ABI of include/kda.h: argument validation, workspace
// sizing and kernel selection.  Every host-visible fault returns before any
// work is enqueued.
#include <nvtx3/nvToolsExt.h>
#include <cuda_runtime.h>

#include "../../include/kda.h"
#include "kda_common.cuh"
#include "kda_launch.h"

namespace {

bool dim_ok(int32_t d) { return d == 32 || d == 64 || d == 128; }

// The tensor-core path serves bf16 inputs with dk = dv = 128 and 64-token
// chunks; every other supported case runs on the fp32 CUDA-core path.
bool use_tc(kda_dtype dt, int32_t dk, int32_t dv, int32_t chunk) {
  return dt == KDA_BF16 && dk == 128 && dv == 128 && chunk == 64;
}
bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
bool opt_aligned16(const void* p) { return p == nullptr || aligned16(p); }

// Host checks common to kda_forward and kda_forward_g.  Returns KDA_OK or the
// error to report.
kda_status check_forward(const void* q, const void* k, const void* v,
                         const void* gate_src, const void* beta, const float* S0,
                         const int32_t* cu, int32_t N, int32_t T, int32_t max_len,
                         int32_t H, int32_t dk, int32_t dv, kda_dtype dt,
                         int32_t chunk, const void* o, const float* S_final,
                         const void* ws, size_t ws_bytes) {
  if (dt != KDA_F32 && dt != KDA_BF16) return KDA_ERR_UNSUPPORTED;
  if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (chunk != 16 && chunk != 64) return KDA_ERR_UNSUPPORTED;
  if (N < 0 || T < 0 || max_len < 0 || H < 1) return KDA_ERR_INVALID_ARG;
  if (!cu) {
    if ((int64_t)N * max_len != T) return KDA_ERR_INVALID_ARG;
  } else {
    if (!aligned16(cu) && ((uintptr_t)cu & 3u)) return KDA_ERR_INVALID_ARG;
  }
  if (N > 0 && (int64_t)N * ((max_len + chunk - 1) / chunk) > 0x7fffffffLL)
    return KDA_ERR_UNSUPPORTED;
  if (T > 0) {
    if (!q || !k || !v || !gate_src || !beta || !o) return KDA_ERR_INVALID_ARG;
  }
  if (!opt_aligned16(q) || !opt_aligned16(k) || !opt_aligned16(v) ||
      !opt_aligned16(gate_src) || !opt_aligned16(beta) || !opt_aligned16(o) ||
      !opt_aligned16(S0) || !opt_aligned16(S_final) || !opt_aligned16(ws))
    return KDA_ERR_INVALID_ARG;
  const size_t need = kda_forward_workspace_size(N, T, max_len, H, dk, dv, dt, chunk);
  if (need == 0 || !ws || ws_bytes < need) return KDA_ERR_INVALID_ARG;
  return KDA_OK;
}

// Output-epilogue arguments: the gate input is required when there is work,
// the gain is optional; both 16-byte aligned; eps finite and not negative.
bool epilogue_ok(bool work, const void* out_gate, const float* norm_weight, float eps) {
  if (!(eps >= 0.f && eps <= 3.0e38f)) return false;  // rejects NaN and infinities
  if (work && !out_gate) return false;
  return opt_aligned16(out_gate) && opt_aligned16(norm_weight);
}

kda_status decode_common(const void* q, const void* k, const void* v, const void* z,
                         const float* A, const void* beta, float* S_inout, int32_t B,
                         int32_t H, int32_t dk, int32_t dv, kda_dtype dt,
                         const void* out_gate, const float* norm_weight, float eps, void* o,
                         kda_stream_t stream, const kda::DecodeArgs* conv = nullptr) {
  if (dt != KDA_F32 && dt != KDA_BF16) return KDA_ERR_UNSUPPORTED;
  if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (B < 0 || H < 1) return KDA_ERR_INVALID_ARG;
  if ((int64_t)B * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
  if (B == 0) return KDA_OK;
  if (!q || !k || !v || !z || !A || !beta || !S_inout || !o) return KDA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(z) ||
      !aligned16(A) || !aligned16(beta) || !aligned16(S_inout) || !aligned16(o))
    return KDA_ERR_INVALID_ARG;
  kda::DecodeArgs a{q, k, v, z, beta, A, S_inout, o, B, H, dk, dv,
                    dt == KDA_BF16, (cudaStream_t)stream};
  a.out_gate = out_gate;
  a.norm_w = norm_weight;
  a.norm_eps = eps;
  if (conv) {
    a.conv_wq = conv->conv_wq;
    a.conv_wk = conv->conv_wk;
    a.conv_wv = conv->conv_wv;
    a.conv_state = conv->conv_state;
    a.conv_width = conv->conv_width;
  }
  return kda::launch_decode(a) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

// Byte offsets, in a kda_forward_conv workspace, of the prologue's q, k, v
// outputs and the end: after the forward's own fw bytes, 256-byte aligned.
struct Offsets4 {
  size_t v[4];
  size_t operator[](int i) const { return v[i]; }
};
Offsets4 conv_offsets(size_t fw, size_t tok, int32_t dk, int32_t dv, size_t elt) {
  auto up = [](size_t b) { return (b + 255) & ~(size_t)255; };
  Offsets4 o;
  o.v[0] = up(fw);
  o.v[1] = up(o.v[0] + tok * dk * elt);
  o.v[2] = up(o.v[1] + tok * dk * elt);
  o.v[3] = up(o.v[2] + tok * dv * elt);
  return o;
}

kda_status forward_common(kda::ForwardArgs& a) {
  // A clean error word for this call, stream-ordered before its first kernel:
  // the kernels only OR errors into it, so no report of one CTA can be wiped
  // by another CTA's reset.
  if (cudaMemsetAsync(a.ws, 0, sizeof(uint32_t), a.stream) != cudaSuccess) return KDA_ERR_CUDA;
  if (a.N == 0) return KDA_OK;  // nothing to launch
  cudaError_t err = use_tc(a.bf16 ? KDA_BF16 : KDA_F32, a.dk, a.dv, a.chunk)
                        ? kda::launch_forward_tc(a)
                        : kda::launch_forward_simt(a);
  return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace

// NVTX range around each enqueueing entry point: marks the host call that
// validates the arguments and enqueues the launches (a no-op unless a
// profiler is attached; NVTX v3 is header-only).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

extern "C" {

const char* kda_status_string(kda_status s) {
  switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
  }
  return "KDA_ERR_UNKNOWN";
}

int32_t kda_version(void) { return 100; }

size_t kda_forward_workspace_size(int32_t num_seqs, int32_t total_tokens,
                                  int32_t max_seqlen, int32_t H, int32_t dk,
                                  int32_t dv, kda_dtype dt, int32_t chunk) {
  if (dt != KDA_F32 && dt != KDA_BF16) return 0;
  if (!dim_ok(dk) || !dim_ok(dv) || (chunk != 16 && chunk != 64)) return 0;
  if (num_seqs < 0 || total_tokens < 0 || max_seqlen < 0 || H < 1) return 0;
  if (use_tc(dt, dk, dv, chunk))
    return kda::tc_workspace_bytes(num_seqs, total_tokens, H, max_seqlen);
  return kda::simt_workspace_bytes(num_seqs, total_tokens, H, dk, dv, chunk);
}

int32_t kda_forward_launches(int32_t num_seqs, int32_t total_tokens,
                             int32_t max_seqlen, int32_t H, int32_t dk,
                             int32_t dv, kda_dtype dt, int32_t chunk) {
  if (kda_forward_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv, dt, chunk) == 0)
    return 0;
  if (num_seqs == 0) return 0;  // a memset only
  if (use_tc(dt, dk, dv, chunk)) return kda::tc_launches(num_seqs, H, max_seqlen);
  return kda::simt_launches(num_seqs, max_seqlen, chunk);
}

kda_status kda_forward(const void* q, const void* k, const void* v,
                       const void* z, const float* A, const void* beta,
                       const float* S0, const int32_t* cu_seqlens,
                       int32_t num_seqs, int32_t total_tokens,
                       int32_t max_seqlen, int32_t H, int32_t dk, int32_t dv,
                       kda_dtype dt, int32_t chunk, void* o, float* S_final,
                       void* workspace, size_t workspace_bytes,
                       kda_stream_t stream) {
  const NvtxRange nvtx_range_("kda_forward");
  kda_status st = check_forward(q, k, v, z, beta, S0, cu_seqlens, num_seqs,
                                total_tokens, max_seqlen, H, dk, dv, dt, chunk,
                                o, S_final, workspace, workspace_bytes);
  if (st != KDA_OK) return st;
  if (total_tokens > 0 && (!A || !aligned16(A))) return KDA_ERR_INVALID_ARG;
  kda::ForwardArgs a{q, k, v, z, beta, A, nullptr, S0, cu_seqlens, o, S_final,
                     num_seqs, total_tokens, max_seqlen, H, dk, dv, chunk,
                     dt == KDA_BF16, workspace, workspace_bytes,
                     (cudaStream_t)stream};
  return forward_common(a);
}

kda_status kda_forward_g(const void* q, const void* k, const void* v,
                         const float* g, const void* beta, const float* S0,
                         const int32_t* cu_seqlens, int32_t num_seqs,
                         int32_t total_tokens, int32_t max_seqlen, int32_t H,
                         int32_t dk, int32_t dv, kda_dtype dt, int32_t chunk,
                         void* o, float* S_final, void* workspace,
                         size_t workspace_bytes, kda_stream_t stream) {
  const NvtxRange nvtx_range_("kda_forward_g");
  kda_status st = check_forward(q, k, v, g, beta, S0, cu_seqlens, num_seqs,
                                total_tokens, max_seqlen, H, dk, dv, dt, chunk,
                                o, S_final, workspace, workspace_bytes);
  if (st != KDA_OK) return st;
  kda::ForwardArgs a{q, k, v, nullptr, beta, nullptr, g, S0, cu_seqlens, o,
                     S_final, num_seqs, total_tokens, max_seqlen, H, dk, dv,
                     chunk, dt == KDA_BF16, workspace, workspace_bytes,
                     (cudaStream_t)stream};
  return forward_common(a);
}

kda_status kda_forward_scalar_gate(const void* q, const void* k, const void* v,
                                   const float* g_head, const void* beta, const float* S0,
                                   const int32_t* cu_seqlens, int32_t num_seqs,
                                   int32_t total_tokens, int32_t max_seqlen, int32_t H,
                                   int32_t dk, int32_t dv, kda_dtype dt, int32_t chunk,
                                   void* o, float* S_final, void* workspace,
                                   size_t workspace_bytes, kda_stream_t stream) {
  const NvtxRange nvtx_range_("kda_forward_scalar_gate");
  kda_status st = check_forward(q, k, v, g_head, beta, S0, cu_seqlens, num_seqs,
                                total_tokens, max_seqlen, H, dk, dv, dt, chunk,
                                o, S_final, workspace, workspace_bytes);
  if (st != KDA_OK) return st;
  kda::ForwardArgs a{q, k, v, nullptr, beta, nullptr, nullptr, S0, cu_seqlens, o,
                     S_final, num_seqs, total_tokens, max_seqlen, H, dk, dv,
                     chunk, dt == KDA_BF16, workspace, workspace_bytes,
                     (cudaStream_t)stream};
  a.g_head = g_head;
  return forward_common(a);
}

kda_status kda_forward_checkpoints(const void* q, const void* k, const void* v,
                                   const void* z, const float* A, const void* beta,
                                   const float* S0, const int32_t* cu_seqlens,
                                   int32_t num_seqs, int32_t total_tokens,
                                   int32_t max_seqlen, int32_t H, int32_t dk,
                                   int32_t dv, kda_dtype dt, int32_t chunk, void* o,
                                   float* S_final, float* S_ckpt, int32_t interval,
                                   void* workspace, size_t workspace_bytes,
                                   kda_stream_t stream) {
  const NvtxRange nvtx_range_("kda_forward_checkpoints");
  kda_status st = check_forward(q, k, v, z, beta, S0, cu_seqlens, num_seqs,
                                total_tokens, max_seqlen, H, dk, dv, dt, chunk,
                                o, S_final, workspace, workspace_bytes);
  if (st != KDA_OK) return st;
  if (total_tokens > 0 && (!A || !aligned16(A))) return KDA_ERR_INVALID_ARG;
  if (interval <= 0 || interval % chunk != 0) return KDA_ERR_INVALID_ARG;
  const int32_t count = max_seqlen / interval;
  if (count > 0 && (!S_ckpt || !aligned16(S_ckpt))) return KDA_ERR_INVALID_ARG;
  kda::ForwardArgs a{q, k, v, z, beta, A, nullptr, S0, cu_seqlens, o, S_final,
                     num_seqs, total_tokens, max_seqlen, H, dk, dv, chunk,
                     dt == KDA_BF16, workspace, workspace_bytes,
                     (cudaStream_t)stream};
  if (count > 0) {
    a.S_ckpt = S_ckpt;
    a.ckpt_every = interval / chunk;
    a.ckpt_count = count;
  }
  return forward_common(a);
}

kda_status kda_forward_norm_gate(const void* q, const void* k, const void* v,
                                 const void* z, const float* A, const void* beta,
                                 const float* S0, const int32_t* cu_seqlens,
                                 int32_t num_seqs, int32_t total_tokens,
                                 int32_t max_seqlen, int32_t H, int32_t dk, int32_t dv,
                                 kda_dtype dt, int32_t chunk, const void* out_gate,
                                 const float* norm_weight, float eps, void* o,
                                 float* S_final, void* workspace, size_t workspace_bytes,
                                 kda_stream_t stream) {
  const NvtxRange nvtx_range_("kda_forward_norm_gate");
  kda_status st = check_forward(q, k, v, z, beta, S0, cu_seqlens, num_seqs,
                                total_tokens, max_seqlen, H, dk, dv, dt, chunk,
                                o, S_final, workspace, workspace_bytes);
  if (st != KDA_OK) return st;
  if (total_tokens > 0 && (!A || !aligned16(A))) return KDA_ERR_INVALID_ARG;
  if (!epilogue_ok(total_tokens > 0, out_gate, norm_weight, eps)) return KDA_ERR_INVALID_ARG;
  kda::ForwardArgs a{q, k, v, z, beta, A, nullptr, S0, cu_seqlens, o, S_final,
                     num_seqs, total_tokens, max_seqlen, H, dk, dv, chunk,
                     dt == KDA_BF16, workspace, workspace_bytes,
                     (cudaStream_t)stream};
  a.out_gate = out_gate;
  a.norm_w = norm_weight;
  a.norm_eps = eps;
  return forward_common(a);
}

kda_status kda_decode_step(const void* q, const void* k, const void* v,
                           const void* z, const float* A, const void* beta,
                           float* S_inout, int32_t B, int32_t H, int32_t dk,
                           int32_t dv, kda_dtype dt, void* o,
                           kda_stream_t stream) {
  const NvtxRange nvtx_range_("kda_decode_step");
  return decode_common(q, k, v, z, A, beta, S_inout, B, H, dk, dv, dt, nullptr, nullptr, 0.f, o,
                       stream);
}

kda_status kda_decode_step_norm_gate(const void* q, const void* k, const void* v,
                                     const void* z, const float* A, const void* beta,
                                     float* S_inout, int32_t B, int32_t H, int32_t dk,
                                     int32_t dv, kda_dtype dt, const void* out_gate,
                                     const float* norm_weight, float eps, void* o,
                                     kda_stream_t stream) {
  const NvtxRange nvtx_range_("kda_decode_step_norm_gate");
  if (!epilogue_ok(B > 0, out_gate, norm_weight, eps)) return KDA_ERR_INVALID_ARG;
  return decode_common(q, k, v, z, A, beta, S_inout, B, H, dk, dv, dt, out_gate, norm_weight,
                       eps, o, stream);
}

kda_status kda_decode_step_conv(const void* x_q, const void* x_k, const void* x_v,
                                const float* w_q, const float* w_k, const float* w_v,
                                int32_t conv_width, void* conv_state, const void* z,
                                const float* A, const void* beta, float* S_inout, int32_t B,
                                int32_t H, int32_t dk, int32_t dv, kda_dtype dt, void* o,
                                kda_stream_t stream) {
  const NvtxRange nvtx_range_("kda_decode_step_conv");
  if (conv_width < 1 || conv_width > 4) return KDA_ERR_UNSUPPORTED;
  if (B > 0 && (!w_q || !w_k || !w_v || ((uintptr_t)w_q & 3u) || ((uintptr_t)w_k & 3u) ||
                ((uintptr_t)w_v & 3u)))
    return KDA_ERR_INVALID_ARG;
  if (B > 0 && conv_width > 1 &&
      (!conv_state || ((uintptr_t)conv_state & (dt == KDA_BF16 ? 1u : 3u))))
    return KDA_ERR_INVALID_ARG;
  kda::DecodeArgs c{};
  c.conv_wq = w_q;
  c.conv_wk = w_k;
  c.conv_wv = w_v;
  c.conv_state = conv_state;
  c.conv_width = conv_width;
  return decode_common(x_q, x_k, x_v, z, A, beta, S_inout, B, H, dk, dv, dt, nullptr, nullptr,
                       0.f, o, stream, &c);
}

kda_status kda_short_conv_swish(const void* x, const float* w, const int32_t* cu_seqlens,
                                int32_t num_seqs, int32_t total_tokens, int32_t max_seqlen,
                                int32_t channels, int32_t width, kda_dtype dt, void* y,
                                kda_stream_t stream) {
  const NvtxRange nvtx_range_("kda_short_conv_swish");
  if (dt != KDA_F32 && dt != KDA_BF16) return KDA_ERR_UNSUPPORTED;
  if (width < 1 || width > 4) return KDA_ERR_UNSUPPORTED;
  if (channels < 8 || channels % 8 != 0) return KDA_ERR_UNSUPPORTED;
  if (num_seqs < 0 || total_tokens < 0 || max_seqlen < 0) return KDA_ERR_INVALID_ARG;
  if (!cu_seqlens && (int64_t)num_seqs * max_seqlen != total_tokens) return KDA_ERR_INVALID_ARG;
  if (total_tokens == 0) return KDA_OK;
  if (num_seqs == 0) return KDA_ERR_INVALID_ARG;
  if (!x || !w || !y || !aligned16(x) || !aligned16(y)) return KDA_ERR_INVALID_ARG;
  if (cu_seqlens && ((uintptr_t)cu_seqlens & 3u)) return KDA_ERR_INVALID_ARG;
  if (((uintptr_t)w & 3u)) return KDA_ERR_INVALID_ARG;
  kda::ConvArgs a{};
  a.t[0] = {x, w, y, channels};
  a.ntensors = 1;
  a.cu = cu_seqlens;
  a.N = num_seqs; a.T = total_tokens; a.L = max_seqlen; a.width = width;
  a.bf16 = dt == KDA_BF16;
  a.stream = (cudaStream_t)stream;
  return kda::launch_conv_swish(a) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

size_t kda_forward_conv_workspace_size(int32_t num_seqs, int32_t total_tokens,
                                       int32_t max_seqlen, int32_t H, int32_t dk, int32_t dv,
                                       kda_dtype dt, int32_t chunk) {
  const size_t fw = kda_forward_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv,
                                               dt, chunk);
  if (fw == 0) return 0;
  // the tensor-core path runs the prologue inside its chunk preparation
  if (use_tc(dt, dk, dv, chunk)) return fw;
  const size_t elt = dt == KDA_BF16 ? 2 : 4, tok = (size_t)total_tokens * H;
  return conv_offsets(fw, tok, dk, dv, elt)[3];
}

kda_status kda_forward_conv(const void* x_q, const void* x_k, const void* x_v,
                            const float* w_q, const float* w_k, const float* w_v,
                            int32_t conv_width, const void* z, const float* A, const void* beta,
                            const float* S0, const int32_t* cu_seqlens, int32_t num_seqs,
                            int32_t total_tokens, int32_t max_seqlen, int32_t H, int32_t dk,
                            int32_t dv, kda_dtype dt, int32_t chunk, void* o, float* S_final,
                            void* workspace, size_t workspace_bytes, kda_stream_t stream) {
  const NvtxRange nvtx_range_("kda_forward_conv");
  const size_t fw = kda_forward_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv,
                                               dt, chunk);
  const size_t need = kda_forward_conv_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk,
                                                      dv, dt, chunk);
  // the forward's own checks, on its part of the workspace
  kda_status st = check_forward(x_q, x_k, x_v, z, beta, S0, cu_seqlens, num_seqs,
                                total_tokens, max_seqlen, H, dk, dv, dt, chunk, o, S_final,
                                workspace, fw);
  if (st != KDA_OK) return st;
  if (total_tokens > 0 && (!A || !aligned16(A))) return KDA_ERR_INVALID_ARG;
  if (conv_width < 1 || conv_width > 4) return KDA_ERR_UNSUPPORTED;
  if (workspace_bytes < need) return KDA_ERR_INVALID_ARG;
  if (total_tokens > 0 && (!w_q || !w_k || !w_v || ((uintptr_t)w_q & 3u) ||
                           ((uintptr_t)w_k & 3u) || ((uintptr_t)w_v & 3u)))
    return KDA_ERR_INVALID_ARG;
  if (use_tc(dt, dk, dv, chunk)) {
    // fused: the chunk preparation convolves the staged rows itself
    kda::ForwardArgs a{x_q, x_k, x_v, z, beta, A, nullptr, S0, cu_seqlens, o, S_final,
                       num_seqs, total_tokens, max_seqlen, H, dk, dv, chunk,
                       dt == KDA_BF16, workspace, fw, (cudaStream_t)stream};
    a.conv_wq = w_q;
    a.conv_wk = w_k;
    a.conv_wv = w_v;
    a.conv_width = conv_width;
    return forward_common(a);
  }
  const size_t elt = dt == KDA_BF16 ? 2 : 4, tok = (size_t)total_tokens * H;
  const auto off = conv_offsets(fw, tok, dk, dv, elt);
  char* ws = (char*)workspace;
  void *q = ws + off[0], *k = ws + off[1], *v = ws + off[2];
  if (total_tokens > 0 && num_seqs > 0) {
    kda::ConvArgs c{};
    c.t[0] = {x_q, w_q, q, H * dk};
    c.t[1] = {x_k, w_k, k, H * dk};
    c.t[2] = {x_v, w_v, v, H * dv};
    c.ntensors = 3;
    c.cu = cu_seqlens;
    c.N = num_seqs; c.T = total_tokens; c.L = max_seqlen; c.width = conv_width;
    c.bf16 = dt == KDA_BF16;
    c.stream = (cudaStream_t)stream;
    if (kda::launch_conv_swish(c) != cudaSuccess) return KDA_ERR_CUDA;
  }
  kda::ForwardArgs a{q, k, v, z, beta, A, nullptr, S0, cu_seqlens, o, S_final,
                     num_seqs, total_tokens, max_seqlen, H, dk, dv, chunk,
                     dt == KDA_BF16, workspace, fw, (cudaStream_t)stream};
  return forward_common(a);
}

size_t kda_cp_workspace_size(int32_t num_seqs, int32_t total_tokens, int32_t max_seqlen,
                             int32_t H, int32_t dk, int32_t dv, kda_dtype dt, int32_t chunk) {
  if (!use_tc(dt, dk, dv, chunk)) return 0;
  if (num_seqs < 0 || total_tokens < 0 || max_seqlen < 0 || H < 1) return 0;
  return kda::tc_cp_workspace_bytes(num_seqs, total_tokens, H, max_seqlen);
}

kda_status kda_cp_local(const void* q, const void* k, const void* v, const void* z,
                        const float* A, const void* beta, const int32_t* cu_seqlens,
                        int32_t num_seqs, int32_t total_tokens, int32_t max_seqlen, int32_t H,
                        int32_t dk, int32_t dv, kda_dtype dt, int32_t chunk, float* M_out,
                        float* N_out, void* workspace, size_t workspace_bytes,
                        kda_stream_t stream) {
  const NvtxRange nvtx_range_("kda_cp_local");
  if (!use_tc(dt, dk, dv, chunk)) return KDA_ERR_UNSUPPORTED;
  // the forward's geometry and input checks, with M_out standing in for o (its
  // workspace size is at most the one this call needs, checked next)
  kda_status st = check_forward(q, k, v, z, beta, nullptr, cu_seqlens, num_seqs, total_tokens,
                                max_seqlen, H, dk, dv, dt, chunk, M_out, nullptr, workspace,
                                workspace_bytes);
  if (st != KDA_OK) return st;
  if (workspace_bytes < kda_cp_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv, dt,
                                              chunk))
    return KDA_ERR_INVALID_ARG;
  if (num_seqs > 0 && (!M_out || !N_out || !aligned16(M_out) || !aligned16(N_out)))
    return KDA_ERR_INVALID_ARG;
  if (total_tokens > 0 && (!A || !aligned16(A))) return KDA_ERR_INVALID_ARG;
  kda::ForwardArgs a{q, k, v, z, beta, A, nullptr, nullptr, cu_seqlens, nullptr, nullptr,
                     num_seqs, total_tokens, max_seqlen, H, dk, dv, chunk,
                     true, workspace, workspace_bytes, (cudaStream_t)stream};
  if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), (cudaStream_t)stream) != cudaSuccess)
    return KDA_ERR_CUDA;
  if (num_seqs == 0) return KDA_OK;
  return kda::launch_cp_local_tc(a, M_out, N_out) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_cp_finish(const float* S_in, const int32_t* cu_seqlens, int32_t num_seqs,
                         int32_t total_tokens, int32_t max_seqlen, int32_t H, int32_t dk,
                         int32_t dv, kda_dtype dt, int32_t chunk, void* o, float* S_final,
                         void* workspace, size_t workspace_bytes, kda_stream_t stream) {
  const NvtxRange nvtx_range_("kda_cp_finish");
  if (!use_tc(dt, dk, dv, chunk)) return KDA_ERR_UNSUPPORTED;
  if (num_seqs < 0 || total_tokens < 0 || max_seqlen < 0 || H < 1) return KDA_ERR_INVALID_ARG;
  if (!cu_seqlens && (int64_t)num_seqs * max_seqlen != total_tokens) return KDA_ERR_INVALID_ARG;
  if (cu_seqlens && ((uintptr_t)cu_seqlens & 3u)) return KDA_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) ||
      workspace_bytes < kda_cp_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv, dt,
                                              chunk))
    return KDA_ERR_INVALID_ARG;
  if (total_tokens > 0 && (!o || !aligned16(o))) return KDA_ERR_INVALID_ARG;
  if (!opt_aligned16(S_in) || !opt_aligned16(S_final)) return KDA_ERR_INVALID_ARG;
  if (num_seqs == 0) return KDA_OK;
  kda::ForwardArgs a{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, S_in,
                     cu_seqlens, o, S_final, num_seqs, total_tokens, max_seqlen, H, dk, dv,
                     chunk, true, workspace, workspace_bytes, (cudaStream_t)stream};
  return kda::launch_cp_finish_tc(a) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_state_compose(const float* M, const float* N, const float* S_in, float* S_out,
                             int32_t count, int32_t dk, int32_t dv, kda_stream_t stream) {
  const NvtxRange nvtx_range_("kda_state_compose");
  if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (count < 0) return KDA_ERR_INVALID_ARG;
  if (count == 0) return KDA_OK;
  if (!M || !N || !S_out || !aligned16(M) || !aligned16(N) || !aligned16(S_out) ||
      !opt_aligned16(S_in))
    return KDA_ERR_INVALID_ARG;
  return kda::launch_state_compose(M, N, S_in, S_out, count, dk, dv, (cudaStream_t)stream) ==
                 cudaSuccess
             ? KDA_OK
             : KDA_ERR_CUDA;
}

kda_status kda_debug_set_wait_limit(int64_t cycles) {
  kda::tc_set_wait_limit((long long)cycles);
  return KDA_OK;
}

kda_status kda_check_device_error(const void* workspace, kda_stream_t stream) {
  if (!workspace || !aligned16(workspace)) return KDA_ERR_INVALID_ARG;
  uint32_t err = 0;
  if (cudaMemcpyAsync(&err, workspace, sizeof(err), cudaMemcpyDeviceToHost,
                      (cudaStream_t)stream) != cudaSuccess)
    return KDA_ERR_CUDA;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return KDA_ERR_CUDA;
  if (err == kda::kErrNone) return KDA_OK;
  if (err & kda::kErrTimeout) return KDA_ERR_TIMEOUT;
  return KDA_ERR_INVALID_ARG;
}

}  // extern "C"
