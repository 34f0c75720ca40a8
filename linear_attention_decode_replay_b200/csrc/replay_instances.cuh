// Instantiates the replay kernel for one k-dim (REPLAY_N) and provides its launcher.
#pragma once

#include <cuda_runtime.h>

#include <mutex>

#include "replay_kernel.cuh"
#include "replay_launch.h"

#ifndef REPLAY_N
#error "define REPLAY_N before including replay_instances.cuh"
#endif

namespace replay {
namespace {

constexpr int kMaxDevices = 64;

template <typename IO, int CKPT, int MODE, int NQ>
cudaError_t launch_one(const KParams& p, int grid, cudaStream_t s) {
  auto kern = replay_kernel<REPLAY_N, IO, CKPT, MODE, NQ, kGroups>;  // NG: the host layout reserves one workspace per group
  // the dynamic shared-memory opt-in is per function and device; remember the largest set
  // (under a lock: calls may come from several threads, and a smaller concurrent setting
  // must not lower the limit below what another launch needs)
  static int configured[kMaxDevices] = {0};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= kMaxDevices || configured[dev] < p.smem_bytes) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem_bytes);
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < kMaxDevices) configured[dev] = p.smem_bytes;
    }
  }
  // Programmatic dependent launch: this grid's CTAs may be scheduled while the previous
  // kernel on the stream drains (an SM takes one as soon as its previous CTA exits); the
  // kernel waits for that kernel's completion (griddepcontrol.wait) before it reads any
  // memory, so only its set-up overlaps the previous kernel's tail.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = p.smem_bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

constexpr int kVerifyPosSmall = 5;  // positions of the smaller multi-position instance

template <typename IO, int CKPT>
cudaError_t launch_mode(const KParams& p, int mode, int nq, int grid, cudaStream_t s) {
  if (mode == kModeReplay) {
    // multi-position calls: an instance unrolled over five positions for the common
    // draft of four (n_pos <= 5), whose code fits the instruction cache better than the
    // eight-position one (measured: 327 against 372 us per verify round of five positions)
    return nq > 5 ? launch_one<IO, CKPT, kModeReplay, kMaxPos>(p, grid, s)
           : nq > 1 ? launch_one<IO, CKPT, kModeReplay, kVerifyPosSmall>(p, grid, s)
                    : launch_one<IO, CKPT, kModeReplay, 1>(p, grid, s);
  }
  if (mode == kModeFlush) return launch_one<IO, CKPT, kModeFlush, 0>(p, grid, s);
  if constexpr (CKPT == kCkptFp4) return cudaErrorInvalidValue;  // no eager baseline on an FP4 state
  else return launch_one<IO, CKPT, kModeEager, 1>(p, grid, s);
}

template <typename IO>
cudaError_t launch_ckpt(const KParams& p, int ckpt, int mode, int nq, int grid, cudaStream_t s) {
  return ckpt == kCkptFp8   ? launch_mode<IO, kCkptFp8>(p, mode, nq, grid, s)
         : ckpt == kCkptFp4 ? launch_mode<IO, kCkptFp4>(p, mode, nq, grid, s)
                            : launch_mode<IO, kCkptF32>(p, mode, nq, grid, s);
}

}  // namespace

#define REPLAY_CAT2(a, b) a##b
#define REPLAY_CAT(a, b) REPLAY_CAT2(a, b)
cudaError_t REPLAY_CAT(launch_replay_n, REPLAY_N)(const KParams& p, int io, int ckpt, int mode, int nq, int grid,
                                                   cudaStream_t s) {
  return io == 1 ? launch_ckpt<__nv_bfloat16>(p, ckpt, mode, nq, grid, s)
                 : launch_ckpt<float>(p, ckpt, mode, nq, grid, s);
}

}  // namespace replay
