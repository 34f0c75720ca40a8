// Snapshot export and import of single sequences: the checkpoint, the committed buffer
// entries and the count, as one self-describing block per sequence (a prefix-cache or
// migration unit). One CTA per (listed sequence, head); the state is moved with 16-byte
// loads and stores, the records one 16-byte piece per thread.
#include "replay_kernel.cuh"
#include "replay_launch.h"

namespace replay {

namespace {

// The pieces of snapshot i: header, then [H][P][N] FP32 state, then [G][L] k records of
// RK bytes, then [H][L] head records of R bytes.
__device__ __forceinline__ uint8_t* snap_state(uint8_t* snap, const SnapParams& sp, int h) {
  return snap + kSnapHeaderBytes + (size_t)h * sp.P * sp.N * 4;
}
__device__ __forceinline__ uint8_t* snap_krecords(uint8_t* snap, const SnapParams& sp, int g) {
  return snap + kSnapHeaderBytes + (size_t)sp.H * sp.P * sp.N * 4 + (size_t)g * sp.L * sp.rec_k_bytes;
}
__device__ __forceinline__ uint8_t* snap_records(uint8_t* snap, const SnapParams& sp, int h) {
  return snap + kSnapHeaderBytes + (size_t)sp.H * sp.P * sp.N * 4 + (size_t)sp.G * sp.L * sp.rec_k_bytes +
         (size_t)h * sp.L * sp.rec_bytes;
}

// Records [start, start + c) of a ring (cap records of `rb` bytes) into records 0 .. c-1.
__device__ __forceinline__ void gather_records(uint8_t* dst, const uint8_t* ring, int start, int c, int cap, int rb) {
  const int pieces = rb / 16;
  for (int t = threadIdx.x; t < c * pieces; t += blockDim.x) {
    const int j = t / pieces;
    int slot = start + j;
    slot -= (slot >= cap) ? cap : 0;
    reinterpret_cast<uint4*>(dst + (size_t)j * rb)[t - j * pieces] =
        reinterpret_cast<const uint4*>(ring + (size_t)slot * rb)[t - j * pieces];
  }
}

__device__ __forceinline__ void copy16(uint8_t* dst, const uint8_t* src, size_t bytes) {
  for (size_t o = (size_t)threadIdx.x * 16; o < bytes; o += (size_t)blockDim.x * 16)
    *reinterpret_cast<uint4*>(dst + o) = *reinterpret_cast<const uint4*>(src + o);
}

}  // namespace

// Export: snapshot i <- sequence seqs[i] (its S0, its head and k records [start, start +
// c) in order, renumbered from 0, and c). A sequence id or pointer word out of range sets the pointer
// error bit and leaves that snapshot's header marked invalid.
__global__ void export_kernel(const SnapParams sp) {
  const int i = blockIdx.x / sp.H;
  const int h = blockIdx.x - i * sp.H;
  uint8_t* snap = static_cast<uint8_t*>(sp.snap) + (size_t)i * sp.snap_bytes;
  const int b = sp.seqs[i];
  const bool seq_ok = b >= 0 && b < sp.B;
  const int32_t word = seq_ok ? sp.counts[b] : -1;
  const int start = word >> 16;
  const int c = word & 0xFFFF;
  const bool ok = seq_ok && word >= 0 && c <= sp.L && start < sp.cap;
  if (h == 0 && threadIdx.x == 0) {
    int32_t* hdr = reinterpret_cast<int32_t*>(snap);
    hdr[0] = ok ? kSnapMagic : 0;
    hdr[1] = c;
    hdr[2] = sp.H;
    hdr[3] = sp.P;
    hdr[4] = sp.N;
    hdr[5] = sp.L;
    hdr[6] = sp.rec_bytes;
    hdr[7] = sp.G;
    hdr[8] = sp.rec_k_bytes;
    for (int w = 9; w < kSnapHeaderBytes / 4; ++w) hdr[w] = 0;
    if (!ok && sp.status) atomicOr(sp.status, kErrPointer);
  }
  if (!ok) return;
  const size_t bh = (size_t)b * sp.H + h;
  copy16(snap_state(snap, sp, h), reinterpret_cast<const uint8_t*>(sp.S + bh * sp.P * sp.N), (size_t)sp.P * sp.N * 4);
  gather_records(snap_records(snap, sp, h), static_cast<const uint8_t*>(sp.ring) + bh * sp.cap * sp.rec_bytes, start,
                 c, sp.cap, sp.rec_bytes);
  const int hpg = sp.H / sp.G;
  if (h % hpg == 0) {  // the group's k records, by its first head's block
    const int g = h / hpg;
    gather_records(snap_krecords(snap, sp, g),
                   static_cast<const uint8_t*>(sp.ring_k) + ((size_t)b * sp.G + g) * sp.cap * sp.rec_k_bytes, start, c,
                   sp.cap, sp.rec_k_bytes);
  }
}

// Import: sequence seqs[i] <- snapshot i: S0, the records into ring slots 0 .. c-1 (k by
// each group's first head), the pointer word (start 0, count c) into the current half of
// the pointer words, and, with a read copy, its codes and row scales quantised from the
// imported master with the arithmetic replay_init uses. A snapshot whose header does not match this layer's sizes,
// or a sequence id out of range, sets the snapshot error bit and is skipped.
template <int N>
__global__ void import_kernel(const SnapParams sp) {
  constexpr int TPR = N / 4;
  const int i = blockIdx.x / sp.H;
  const int h = blockIdx.x - i * sp.H;
  const uint8_t* snap = static_cast<const uint8_t*>(sp.snap) + (size_t)i * sp.snap_bytes;
  const int32_t* hdr = reinterpret_cast<const int32_t*>(snap);
  const int b = sp.seqs[i];
  const int c = hdr[1];
  const bool ok = b >= 0 && b < sp.B && hdr[0] == kSnapMagic && c >= 0 && c <= sp.L && hdr[2] == sp.H &&
                  hdr[3] == sp.P && hdr[4] == N && hdr[5] == sp.L && hdr[6] == sp.rec_bytes && hdr[7] == sp.G &&
                  hdr[8] == sp.rec_k_bytes;
  if (!ok) {
    if (h == 0 && threadIdx.x == 0 && sp.status) atomicOr(sp.status, kErrSnapshot);
    return;
  }
  const size_t bh = (size_t)b * sp.H + h;
  const uint8_t* state = snap_state(const_cast<uint8_t*>(snap), sp, h);
  copy16(reinterpret_cast<uint8_t*>(sp.S + bh * sp.P * N), state, (size_t)sp.P * N * 4);
  if (sp.S8) {
    // per-row read copy (e4m3 or e2m1): TPR lanes per row, four values each (the
    // quantisers' mapping and arithmetic)
    constexpr int RPB = 256 / TPR;  // rows per block pass (blockDim.x == 256)
    const int col = (threadIdx.x % TPR) * 4;
    for (int r0 = 0; r0 < sp.P; r0 += RPB) {
      const int r = r0 + (int)threadIdx.x / TPR;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < sp.P) v = *reinterpret_cast<const float4*>(state + ((size_t)r * N + col) * 4);
      const float am = seg_allmax<TPR>(amax4(v));
      float sc, inv;
      if (sp.ckpt == kCkptFp4) {
        e2m1_row_scale(am, sc, inv);
        if (r < sp.P)
          *reinterpret_cast<unsigned short*>(sp.S8 + (bh * sp.P + r) * (N / 2) + col / 2) =
              static_cast<unsigned short>(quant4_e2m1(v, inv));
      } else {
        e4m3_row_scale(am, sc, inv);
        if (r < sp.P) *reinterpret_cast<uint32_t*>(sp.S8 + (bh * sp.P + r) * N + col) = quant4_e4m3(v, inv);
      }
      if (r < sp.P && (threadIdx.x % TPR) == 0) sp.Sscale[bh * sp.P + r] = sc;
    }
  }
  uint8_t* ring = static_cast<uint8_t*>(sp.ring) + bh * sp.cap * sp.rec_bytes;
  copy16(ring, snap_records(const_cast<uint8_t*>(snap), sp, h), (size_t)c * sp.rec_bytes);
  const int hpg = sp.H / sp.G;
  if (h % hpg == 0) {
    const int g = h / hpg;
    copy16(static_cast<uint8_t*>(sp.ring_k) + ((size_t)b * sp.G + g) * sp.cap * sp.rec_k_bytes,
           snap_krecords(const_cast<uint8_t*>(snap), sp, g), (size_t)c * sp.rec_k_bytes);
  }
  if (h == 0 && threadIdx.x == 0) sp.counts[b] = c;  // start 0, count c
}

cudaError_t launch_export(const SnapParams& sp, cudaStream_t s) {
  export_kernel<<<sp.n * sp.H, 256, 0, s>>>(sp);
  return cudaGetLastError();
}

cudaError_t launch_import(const SnapParams& sp, cudaStream_t s) {
  switch (sp.N) {
    case 16: import_kernel<16><<<sp.n * sp.H, 256, 0, s>>>(sp); break;
    case 32: import_kernel<32><<<sp.n * sp.H, 256, 0, s>>>(sp); break;
    case 64: import_kernel<64><<<sp.n * sp.H, 256, 0, s>>>(sp); break;
    case 128: import_kernel<128><<<sp.n * sp.H, 256, 0, s>>>(sp); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace replay
