// kda_noalloc.cu -- kda_forward_noalloc: kda_forward backed by a fixed
// file-scope scratch array, for callers that cannot allocate device memory.
//
// The array below is the only scratch this entry point uses.  In host code
// its name is a host-side stand-in, not a device address, so the entry point
// looks the address up with cudaGetSymbolAddress (once per device, with that
// device current) and hands that pointer to kda_forward as its workspace.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/kda.h"

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices];  // device address of g_noalloc_scratch, per device

// Device address of the scratch array on the current device (looked up on the
// first call for that device, then cached).
kda_status scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return KDA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KDA_OK;
}

}  // namespace

extern "C" kda_status kda_forward_noalloc(const void* q, const void* k, const void* v,
                                          const void* z, const float* A, const void* beta,
                                          const float* S0, const int32_t* cu_seqlens,
                                          int32_t num_seqs, int32_t total_tokens,
                                          int32_t max_seqlen, int32_t H, int32_t dk,
                                          int32_t dv, kda_dtype dt, int32_t chunk,
                                          void* o, float* S_final, kda_stream_t stream) {
  const size_t need =
      kda_forward_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv, dt, chunk);
  if (need == 0)  // invalid or unsupported: let kda_forward report which, enqueueing nothing
    return kda_forward(q, k, v, z, A, beta, S0, cu_seqlens, num_seqs, total_tokens, max_seqlen,
                       H, dk, dv, dt, chunk, o, S_final, nullptr, 0, stream);
  if (need > KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const kda_status st = scratch_on_current_device(&scratch);
  if (st != KDA_OK) return st;
  return kda_forward(q, k, v, z, A, beta, S0, cu_seqlens, num_seqs, total_tokens, max_seqlen, H,
                     dk, dv, dt, chunk, o, S_final, scratch, KDA_NOALLOC_SCRATCH_BYTES, stream);
}
