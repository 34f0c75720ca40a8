// Small kernels and their launchers: the entry pre-pass, per-row e4m3 quantisation and
// rollback.
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


// Writes this call's new entries into their ring records before the main kernel runs:
// record (start + c + s) mod cap of (b, h) gets v, Delta, a of position s, and the same
// record of (b, g) its k (written by the group's first head), where (start, c) is the
// sequence's current pointer word. A flush in the main kernel reads records
// [start, start + c) and the appends land in [start + c, start + c + n_pos), so the two
// never overlap (cap = L + max_pos). Verify queries are also gathered per group into
// qpack so that a unit's queries are one contiguous piece. One warp per (b, h).
__global__ void pack_entries_kernel(const PackParams pp) {
  constexpr int kMaxChunks = 3;  // 16-byte chunks of one entry's k and v per lane: (N + P) * 4 / 16 / 32 <= 3
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x / 32;
  const int S = pp.io_bytes;
  const int kpe = pp.N * S / 16;  // 16-byte chunks of a k (or q) row
  const int vpe = pp.P * S / 16;
  const long long total = (long long)pp.B * pp.H;
  for (long long task = (long long)blockIdx.x * wpb + threadIdx.x / 32; task < total; task += (long long)gridDim.x * wpb) {
    const int b = (int)(task / pp.H);
    const int h = (int)(task - (long long)b * pp.H);
    const int g = h / pp.hpg;
    const int32_t word = pp.counts_in[b];
    for (int s = 0; s < pp.n_pos; ++s) {
      if (!pp.write_entries) {  // resident entries: only the queries are packed
        if (pp.qpack && (h % pp.hpg) == 0) {
          const size_t tok = (size_t)b * pp.n_pos + s;
          const uint8_t* qin = static_cast<const uint8_t*>(pp.q) + (tok * pp.G + g) * pp.N * S;
          uint8_t* qout = static_cast<uint8_t*>(pp.qpack) + (((size_t)b * pp.G + g) * pp.qpack_pos + s) * pp.N * S;
          for (int idx = lane; idx < kpe; idx += 32) reinterpret_cast<uint4*>(qout)[idx] = reinterpret_cast<const uint4*>(qin)[idx];
        }
        continue;
      }
      // the entry's pieces are read before the pointer word is needed, so both reads
      // are in flight together
      const size_t tok = (size_t)b * pp.n_pos + s;
      const bool k_here = (h % pp.hpg) == 0;  // the group's first head writes its k
      const uint8_t* kin = static_cast<const uint8_t*>(pp.k) + (tok * pp.G + g) * pp.N * S;
      const uint8_t* vin = static_cast<const uint8_t*>(pp.v) + (tok * pp.H + h) * pp.P * S;
      uint4 chunk[kMaxChunks];
#pragma unroll
      for (int r = 0; r < kMaxChunks; ++r) {
        const int idx = lane + 32 * r;
        chunk[r] = (idx < kpe && k_here) ? reinterpret_cast<const uint4*>(kin)[idx]
                   : (idx >= kpe && idx < kpe + vpe) ? reinterpret_cast<const uint4*>(vin)[idx - kpe]
                                                     : make_uint4(0u, 0u, 0u, 0u);
      }
      const float dts = (lane == 0) ? pp.dt[tok * pp.H + h] : 0.f;
      const float as = (lane == 0) ? pp.a[tok * pp.H + h] : 0.f;
      const int start = word >> 16;
      const int c = word & 0xFFFF;
      if (word < 0 || c > pp.L || start >= pp.cap) break;  // the main kernel reports it
      int slot = start + c + s;
      slot -= (slot >= pp.cap) ? pp.cap : 0;
      uint8_t* rec = static_cast<uint8_t*>(pp.ring) + (((size_t)b * pp.H + h) * pp.cap + slot) * pp.rec_bytes;
      uint8_t* krec = static_cast<uint8_t*>(pp.ring_k) + (((size_t)b * pp.G + g) * pp.cap + slot) * pp.rec_k_bytes;
#pragma unroll
      for (int r = 0; r < kMaxChunks; ++r) {
        const int idx = lane + 32 * r;
        if (idx < kpe) {
          if (k_here) reinterpret_cast<uint4*>(krec)[idx] = chunk[r];
        } else if (idx < kpe + vpe) {
          reinterpret_cast<uint4*>(rec)[idx - kpe] = chunk[r];
        }
      }
      if (lane == 0) {
        float* sc = reinterpret_cast<float*>(rec + pp.P * S);
        sc[0] = dts;
        sc[1] = as;
      }
      if (pp.qpack && (h % pp.hpg) == 0) {
        const uint8_t* qin = static_cast<const uint8_t*>(pp.q) + (tok * pp.G + g) * pp.N * S;
        uint8_t* qout = static_cast<uint8_t*>(pp.qpack) + (((size_t)b * pp.G + g) * pp.qpack_pos + s) * pp.N * S;
        for (int idx = lane; idx < kpe; idx += 32) reinterpret_cast<uint4*>(qout)[idx] = reinterpret_cast<const uint4*>(qin)[idx];
      }
    }
  }
}

// The ring record each sequence's next entry goes to: slots[b] = (start + count) mod cap
// from the current pointer word (-1, and the pointer error bit, for a word out of range).
// Position s of a call's entries goes to record (slots[b] + s) mod cap of every head.
__global__ void append_slots_kernel(const int32_t* __restrict__ counts_in, int32_t* __restrict__ slots, int B,
                                    int L, int cap, int32_t* status) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int32_t word = counts_in[b];
  const int start = word >> 16;
  const int c = word & 0xFFFF;
  if (word < 0 || c > L || start >= cap) {
    if (status) atomicOr(status, kErrPointer);
    slots[b] = -1;
    return;
  }
  const int slot = start + c;
  slots[b] = slot >= cap ? slot - cap : slot;
}

cudaError_t launch_append_slots(const int* counts_in, int* slots, int B, int L, int cap, int* status, cudaStream_t s) {
  const int threads = 256;
  append_slots_kernel<<<(B + threads - 1) / threads, threads, 0, s>>>(counts_in, slots, B, L, cap, status);
  return cudaGetLastError();
}

cudaError_t launch_pack_entries(const PackParams& pp, int grid, cudaStream_t s) {
  pack_entries_kernel<<<grid, 256, 0, s>>>(pp);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows_e2m1(const float* x, long long rows, int n, unsigned char* codes, float* scale,
                                      int grid, cudaStream_t s) {
  switch (n) {
    case 16: quantize_rows_e2m1_kernel<16><<<grid, 256, 0, s>>>(x, rows, codes, scale); break;
    case 32: quantize_rows_e2m1_kernel<32><<<grid, 256, 0, s>>>(x, rows, codes, scale); break;
    case 64: quantize_rows_e2m1_kernel<64><<<grid, 256, 0, s>>>(x, rows, codes, scale); break;
    case 128: quantize_rows_e2m1_kernel<128><<<grid, 256, 0, s>>>(x, rows, codes, scale); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
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
