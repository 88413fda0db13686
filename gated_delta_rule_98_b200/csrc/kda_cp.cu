// kda_cp.cu -- the state composition of KDA context parallelism.
//
// A rank that holds one shard of a long sequence summarises it by the affine
// map its tokens apply to the state, S_after = M S_before + N (M dk x dk,
// N dk x dv per head).  The incoming state of shard r is the prefix
// composition of the maps of shards 0 .. r-1 applied to the sequence's initial
// state (Kimi K3 architecture summary, KDA context parallelism: local state
// updates per rank, merged by a prefix scan over a fixed-size all-gather).
// This kernel applies one map to a batch of states:
//
//   S_out[i] = M[i] S_in[i] + N[i]   (fp32; S_in = 0 when not given)
//
// One CTA per (map, 32 state columns): the 32 columns of S_in are staged in
// shared memory (so S_out may alias S_in), each warp owns rows w, w+8, ...,
// and a lane its column; every warp reads its row of M as a broadcast.
#include "kda_common.cuh"
#include "kda_launch.h"

namespace kda {

namespace {

template <int DK, int DV>
__global__ void __launch_bounds__(256) state_compose_kernel(const float* __restrict__ M,
                                                           const float* __restrict__ Nt,
                                                           const float* S_in, float* S_out) {
  constexpr int RPW = DK / 8;  // rows per warp
  __shared__ float Ss[DK][33];
  const int i = blockIdx.x, c0 = blockIdx.y * 32;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const size_t sb = (size_t)i * DK * DV;
  for (int e = tid; e < DK * 32; e += 256) {
    const int r = e >> 5, c = e & 31;
    Ss[r][c] = S_in ? S_in[sb + (size_t)r * DV + c0 + c] : 0.f;
  }
  __syncthreads();
  const float* Mi = M + (size_t)i * DK * DK;
  float acc[RPW];
#pragma unroll
  for (int m = 0; m < RPW; ++m) acc[m] = Nt[sb + (size_t)(w + 8 * m) * DV + c0 + lane];
#pragma unroll 4
  for (int k = 0; k < DK; ++k) {
    const float s = Ss[k][lane];
#pragma unroll
    for (int m = 0; m < RPW; ++m) acc[m] = fmaf(Mi[(size_t)(w + 8 * m) * DK + k], s, acc[m]);
  }
#pragma unroll
  for (int m = 0; m < RPW; ++m) S_out[sb + (size_t)(w + 8 * m) * DV + c0 + lane] = acc[m];
}

template <int DK>
cudaError_t launch_k(const float* M, const float* Nt, const float* S_in, float* S_out, int count,
                     int dv, cudaStream_t st) {
  const dim3 grid(count, dv / 32);
  switch (dv) {
    case 32: state_compose_kernel<DK, 32><<<grid, 256, 0, st>>>(M, Nt, S_in, S_out); break;
    case 64: state_compose_kernel<DK, 64><<<grid, 256, 0, st>>>(M, Nt, S_in, S_out); break;
    case 128: state_compose_kernel<DK, 128><<<grid, 256, 0, st>>>(M, Nt, S_in, S_out); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_compose(const float* M, const float* Nt, const float* S_in, float* S_out,
                                 int count, int dk, int dv, cudaStream_t stream) {
  if (count <= 0) return cudaSuccess;
  switch (dk) {
    case 32: return launch_k<32>(M, Nt, S_in, S_out, count, dv, stream);
    case 64: return launch_k<64>(M, Nt, S_in, S_out, count, dv, stream);
    case 128: return launch_k<128>(M, Nt, S_in, S_out, count, dv, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kda
