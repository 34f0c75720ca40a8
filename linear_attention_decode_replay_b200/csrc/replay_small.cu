// Launchers of the small kernels: per-row e4m3 quantisation and rollback.
#include "replay_kernel.cuh"
#include "replay_launch.h"

namespace replay {

// Rollback / commit: keep n_keep[b] of the n_pos tentative entries of the last verify,
// i.e. move the buffer end of every sequence to base + n_keep.
__global__ void rollback_kernel(const int32_t* __restrict__ counts_in, int32_t* __restrict__ counts_out,
                                const int32_t* __restrict__ n_keep, int B, int n_pos, int32_t* status) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int32_t word = counts_in[b];
  const int32_t nk = n_keep[b];
  if (nk < 0 || nk > n_pos) {
    if (status) atomicOr(status, kErrRollback);
    counts_out[b] = word;
  } else {
    counts_out[b] = word + nk;
  }
}


cudaError_t launch_quantize_rows(const float* x, long long rows, int n, unsigned char* codes, float* scale,
                                 int grid, cudaStream_t s) {
  switch (n) {
    case 16: quantize_rows_kernel<16><<<grid, 256, 0, s>>>(x, rows, codes, scale); break;
    case 32: quantize_rows_kernel<32><<<grid, 256, 0, s>>>(x, rows, codes, scale); break;
    case 64: quantize_rows_kernel<64><<<grid, 256, 0, s>>>(x, rows, codes, scale); break;
    case 128: quantize_rows_kernel<128><<<grid, 256, 0, s>>>(x, rows, codes, scale); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_rollback(const int* counts_in, int* counts_out, const int* n_keep, int B, int n_pos,
                            int* status, cudaStream_t s) {
  const int threads = 256;
  rollback_kernel<<<(B + threads - 1) / threads, threads, 0, s>>>(counts_in, counts_out, n_keep, B, n_pos, status);
  return cudaGetLastError();
}

}  // namespace replay
