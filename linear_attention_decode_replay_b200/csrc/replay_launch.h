// Internal launch entry points, one per supported k-dim N (one translation unit each).
#pragma once

#include <cuda_runtime.h>

#include "replay_kparams.h"

namespace replay {

// mode: kModeReplay / kModeFlush / kModeEager; ckpt: kCkptF32 / kCkptFp8 / kCkptFp4 (no eager);
// io: 0 = FP32, 1 = BF16; nq: the call's query positions (1; 2..5 run the five-position
// instance, more the kMaxPos one)
cudaError_t launch_replay_n16(const KParams& p, int io, int ckpt, int mode, int nq, int grid, cudaStream_t s);
cudaError_t launch_replay_n32(const KParams& p, int io, int ckpt, int mode, int nq, int grid, cudaStream_t s);
cudaError_t launch_replay_n64(const KParams& p, int io, int ckpt, int mode, int nq, int grid, cudaStream_t s);
cudaError_t launch_replay_n128(const KParams& p, int io, int ckpt, int mode, int nq, int grid, cudaStream_t s);

cudaError_t launch_pack_entries(const PackParams& pp, int grid, cudaStream_t s);
cudaError_t launch_quantize_rows(const float* x, long long rows, int n, unsigned char* codes, float* scale,
                                 int grid, cudaStream_t s);
cudaError_t launch_quantize_rows_e2m1(const float* x, long long rows, int n, unsigned char* codes, float* scale,
                                      int grid, cudaStream_t s);
cudaError_t launch_append_slots(const int* counts_in, int* slots, int B, int L, int cap, int* status, cudaStream_t s);
cudaError_t launch_export(const SnapParams& sp, cudaStream_t s);
cudaError_t launch_import(const SnapParams& sp, cudaStream_t s);
cudaError_t launch_rollback(const int* counts_in, int* counts_out, const int* n_keep, int B, int n_pos,
                            int* status, cudaStream_t s);

}  // namespace replay
