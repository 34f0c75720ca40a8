// Persistent, warp-specialised kernel for the ReplaySSM decode path on sm_100a.
//
// One launch processes every (sequence b, head h) unit of a decode layer (a unit is one
// group of up to 16384/N state rows of a head). Each CTA owns chunks of heads (below)
// and streams their units through a ring of shared-memory stages:
//   * the producer warp reads each unit's buffer pointer word (prefetched 32 units at a
//     time) and fills a stage with 1-D bulk copies (TMA), one copy per lane, two units
//     per instruction: the unit's checkpoint tile (FP32 master rows, or the FP8 / FP4
//     read copy's codes + per-row scales), the live k records of the head's k/q group
//     and the head's live v, Delta, a records (each in one or two pieces of the ring),
//     the queries and, for one-position calls, the new entry's k and v straight from the
//     inputs; all complete on the stage's "full" mbarrier;
//   * NG consumer groups (kGroupGemvWarps row warps + one coefficient warp each) take
//     alternate units end to end: the coefficient warp forms the decay weights and the
//     k_j . q_s products while the row warps stream the state rows' dot products (or the
//     fused fold, its write-back and the outputs from the fresh rows); the group meets at
//     its barrier for the outputs, the coefficient warp appends a one-position call's new
//     entry to the ring meanwhile, and the group releases the stage through its "empty"
//     mbarrier.
//     Two groups keep two units in flight, so one unit's short dependent chains overlap
//     the other's, while the producer keeps the next stages' copies in flight.
// The state is streamed exactly once per call; every other byte is small.
//
// What a unit computes (blog "ReplaySSM: Cachear Inputs, No Estado": routes "estado y
// salida" and "solo salida"; arXiv 2610.13778 abstract):
//   REPLAY (step / verify over n_pos positions): if the buffer cannot take n_pos more
//     entries, fold it first, S0 <- abar S0 + sum_j s_j v_j k_j^T, writing the master
//     (and the read copy) once; then for each position s
//       y_s = alpha_s (S q_s) + sum_{j <= c+s} w_{s,j} (k_j . q_s) v_j
//     where S is the fresh fold (in registers) or the stored checkpoint.
//   FLUSH: fold the buffer of the selected sequences, no output.
//   EAGER (baseline): S <- a S + Delta v k^T, y = S q, the state read and written every
//     call (FP32, or a shared FP8 state re-quantised every call).
//
// Row layout inside a group: a state row of N floats is covered by TPR = N/4 lanes, four
// columns each; the group covers 32/TPR rows per warp per pass, and each thread takes
// kRowsPerThread rows of a row group.
#pragma once

#include "replay_device.cuh"
#include "replay_kparams.h"

namespace replay {

__device__ __forceinline__ void report_error(int32_t* status, int32_t bits) {
  if (status) atomicOr(status, bits);
}

template <int NG>
struct Groups {
  static constexpr int kWarps = kConsumerWarps / NG;  // warps per consumer group
  static constexpr int kThreads = kWarps * 32;
};

// barriers at the start of shared memory
struct Bars {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  int abort_flag;
  int last_fill[kMaxStages];  // CTA-local index of the latest unit copied into each stage
};
static_assert(sizeof(Bars) <= kHeaderBytes, "the barrier header must fit the bytes the host layout reserves");

struct Plan {
  int b, h, g, rb, r0, rows, start, c;  // rows r0 .. r0 + rows - 1 of head h of sequence b
  bool fold, corrupt, active, fp32_tile;
  uint32_t bytes;
};

// This CTA's units, in the order its producer fills them and its groups take them:
// chunks of chunk_heads consecutive heads of one k/q group (the group, or a part of it),
// chunk c on CTA c mod gridDim.x, each head with its row blocks in a row. Dealing the
// chunks round-robin keeps the CTAs on neighbouring tiles of the state at any moment,
// and a consumer group that takes several heads of one chunk forms their k . q products
// once.
__device__ __forceinline__ int cta_chunks(const KParams& p) {
  return (p.num_chunks - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
}
__device__ __forceinline__ int cta_units(const KParams& p) { return (cta_chunks(p) * p.chunk_heads) << p.rb_shift; }
// the CTA's hi-th head (chunk hi / chunk_heads, head hi mod chunk_heads within it)
__device__ __forceinline__ int cta_head(const KParams& p, int hi) {
  const int ck = hi / p.chunk_heads;
  return ((int)blockIdx.x + ck * (int)gridDim.x) * p.chunk_heads + (hi - ck * p.chunk_heads);
}
__device__ __forceinline__ int cta_unit(const KParams& p, int i) {
  return (cta_head(p, i >> p.rb_shift) << p.rb_shift) | (i & (p.row_blocks - 1));
}

// A unit's indices: sequence b, head h, its k/q group g, row block rb. The producer works
// them out once per unit (the divisions) and passes them to the consumers in the stage.
struct UnitIdx {
  int b, h, g, rb;
};
__device__ __forceinline__ UnitIdx unit_idx(const KParams& p, int u) {
  UnitIdx x;
  const int bh = u >> p.rb_shift;
  x.rb = u & (p.row_blocks - 1);
  x.b = bh / p.H;
  x.h = bh - x.b * p.H;
  x.g = x.h / p.hpg;
  return x;
}

template <int MODE, int CKPT, int S_IO>
__device__ __forceinline__ Plan make_plan(const KParams& p, const UnitIdx& x, int32_t word, int msk) {
  Plan pl;
  pl.rb = x.rb;
  pl.b = x.b;
  pl.h = x.h;
  pl.g = x.g;
  pl.r0 = pl.rb * p.rows_unit;
  pl.rows = min(p.rows_unit, p.P - pl.r0);
  const uint32_t P = pl.rows, N = p.N;  // the unit's rows
  constexpr uint32_t kCodeDiv = (CKPT == kCkptFp4) ? 2u : 1u;  // code bytes per row = N / kCodeDiv
  if (MODE == kModeEager) {
    pl.start = 0;
    pl.c = 0;
    pl.fold = true;
    pl.corrupt = false;
    pl.active = true;
    pl.fp32_tile = (CKPT == kCkptF32);
    pl.bytes = pl.fp32_tile ? P * N * 4u : P * (N / kCodeDiv) + P * 4u;  // bulk-copied (TMA) bytes
    return pl;
  }
  pl.start = word >> 16;
  pl.c = word & 0xFFFF;
  pl.corrupt = word < 0 || pl.c > p.L || pl.start >= p.cap;
  if (MODE == kModeReplay) {
    pl.fold = pl.c + p.n_pos > p.L;
    pl.active = true;
  } else {
    pl.fold = msk != 0 && pl.c > 0 && pl.c >= p.fold_min;
    pl.active = pl.fold;
  }
  pl.fp32_tile = (CKPT == kCkptF32) || pl.fold;
  if (pl.corrupt || !pl.active) {
    pl.active = false;
    pl.bytes = 0;
    return pl;
  }
  // ring records copied: the buffered ones and, unless this call's entry comes straight
  // from the inputs (one-position calls), the new ones the pre-pass appended
  const bool from_inputs = MODE == kModeReplay && p.append_here;
  const uint32_t records = pl.c + ((MODE == kModeReplay && !from_inputs) ? p.n_pos : 0);
  pl.bytes = (pl.fp32_tile ? P * N * 4u : P * (N / kCodeDiv) + P * 4u) +
             records * (uint32_t)(p.rec_bytes + p.rec_k_bytes) + ((MODE == kModeReplay) ? p.n_pos * N * S_IO : 0u) +
             (from_inputs ? (N + (uint32_t)p.P) * S_IO : 0u);
  return pl;
}

// Entry j of a unit lives in k record j and head record j of the stage: k (N io values);
// v (P io values), Delta, a. Records 0..c-1 are the buffered inputs, c.. this call's new
// tokens.
template <int N, int S_IO>
struct Records {
  const uint8_t* kbase;
  const uint8_t* base;
  int P, R, RK;
  __device__ __forceinline__ const uint8_t* k(int j) const { return kbase + (size_t)j * RK; }
  __device__ __forceinline__ const uint8_t* v(int j) const { return base + (size_t)j * R; }
  __device__ __forceinline__ float dt(int j) const {
    return *reinterpret_cast<const float*>(base + (size_t)j * R + P * S_IO);
  }
  __device__ __forceinline__ float a(int j) const {
    return *reinterpret_cast<const float*>(base + (size_t)j * R + P * S_IO + 4);
  }
};

// ---------------------------------------------------------------------------- producer
// Copies of one unit, one bulk copy (TMA) per kind: 0 the state tile (the unit's rows),
// 1 their read-copy row scales, 2-3 the head's live records and 4-5 the live k records
// of its group, [start, start + count) modulo cap in one or two pieces (whole records:
// every row block reads all of k and its rows of v), 6 the queries, and for one-position
// calls the new entry straight from the inputs, 7 its k and 8 its v, into record c of the
// stage (the producer stores its Delta and a there itself; the consumers append the
// entry to the ring later, off the stream's path). A producer lane always issues the
// same kind, so it works out what does not depend on the unit once: its source array and
// the strides that place a unit in it.
constexpr int kCopyKinds = 9;
struct LaneCopy {
  const uint8_t* base;       // source array (kind 0: the FP32 master)
  const uint8_t* base_copy;  // kind 0-1 with a read copy: the codes / scales array
  uint64_t stride, stride_copy;  // bytes per (sequence, head) [kinds 0-3] or (sequence, group) [4-6]
  uint32_t rb_stride, rb_stride_copy;  // kinds 0-1: bytes per row block
  uint32_t rec;              // kinds 2-5: record bytes
  uint32_t dst_off;          // offset in the stage
  int kind;
};
template <int MODE, int CKPT, int S_IO>
__device__ __forceinline__ LaneCopy lane_copy(const KParams& p, int kind) {
  constexpr uint32_t kCodeDiv = (CKPT == kCkptFp4) ? 2u : 1u;
  const uint32_t N = p.N, P = p.P, UR = p.rows_unit;
  LaneCopy lc;
  lc.kind = kind;
  lc.base_copy = nullptr;
  lc.stride_copy = 0;
  lc.rb_stride = lc.rb_stride_copy = 0;
  lc.rec = 0;
  if (kind == 0) {
    lc.base = reinterpret_cast<const uint8_t*>(p.S);
    lc.stride = (uint64_t)P * N * 4;
    lc.rb_stride = UR * N * 4;
    lc.base_copy = p.S8;
    lc.stride_copy = (uint64_t)P * (N / kCodeDiv);
    lc.rb_stride_copy = UR * (N / kCodeDiv);
    lc.dst_off = 0;
  } else if (kind == 1) {
    lc.base = reinterpret_cast<const uint8_t*>(p.Sscale);
    lc.stride = (uint64_t)P * 4;
    lc.rb_stride = UR * 4;
    lc.dst_off = UR * (N / kCodeDiv);  // the scales follow a full unit's codes
  } else if (kind <= 3) {
    lc.base = static_cast<const uint8_t*>(p.ring);
    lc.rec = p.rec_bytes;
    lc.stride = (uint64_t)p.cap * lc.rec;
    lc.dst_off = p.off_rec;
  } else if (kind <= 5) {
    lc.base = static_cast<const uint8_t*>(p.ring_k);
    lc.rec = p.rec_k_bytes;
    lc.stride = (uint64_t)p.cap * lc.rec;
    lc.dst_off = p.off_krec;
  } else if (kind == 6) {
    lc.base = static_cast<const uint8_t*>(p.qpack ? p.qpack : p.q);
    lc.stride = (uint64_t)(p.qpack ? p.qpack_pos : 1) * N * S_IO;
    lc.dst_off = p.off_q;
  } else if (kind == 7) {
    lc.base = static_cast<const uint8_t*>(p.k);
    lc.stride = (uint64_t)N * S_IO;
    lc.rec = p.rec_k_bytes;
    lc.dst_off = p.off_krec;
  } else {
    lc.base = static_cast<const uint8_t*>(p.v);
    lc.stride = (uint64_t)P * S_IO;
    lc.rec = p.rec_bytes;
    lc.dst_off = p.off_rec;
  }
  return lc;
}
// Source, destination and bytes of this lane's copy of the unit with plan `pl` (0 if none).
template <int MODE, int CKPT, int S_IO>
__device__ __forceinline__ uint32_t unit_copy(const KParams& p, const LaneCopy& lc, const Plan& pl, uint8_t* st,
                                              const uint8_t*& src, uint8_t*& dst) {
  constexpr uint32_t kCodeDiv = (CKPT == kCkptFp4) ? 2u : 1u;
  const uint32_t rows = pl.rows, N = p.N;
  const int bh = pl.b * p.H + pl.h;
  const int bg = pl.b * p.G + pl.g;
  const bool from_inputs = MODE == kModeReplay && p.append_here;
  const int cnt = pl.c + ((MODE == kModeReplay && !from_inputs) ? p.n_pos : 0);  // ring records
  const int first = min(cnt, p.cap - pl.start);
  const bool copy = !pl.fp32_tile;  // kinds 0-1 read the read copy
  uint32_t bytes;
  if (lc.kind <= 1) {
    const uint8_t* base = (lc.kind == 0 && copy) ? lc.base_copy : lc.base;
    const uint64_t stride = (lc.kind == 0 && copy) ? lc.stride_copy : lc.stride;
    const uint32_t rbs = (lc.kind == 0 && copy) ? lc.rb_stride_copy : lc.rb_stride;
    src = base + (uint64_t)bh * stride + (uint64_t)pl.rb * rbs;
    dst = st + lc.dst_off;
    bytes = (lc.kind == 0) ? (copy ? rows * (N / kCodeDiv) : rows * N * 4u) : (copy ? rows * 4u : 0u);
  } else if (lc.kind <= 5) {
    const bool second = (lc.kind == 3 || lc.kind == 5);  // the piece that wrapped to slot 0
    src = lc.base + (uint64_t)((lc.kind <= 3) ? bh : bg) * lc.stride + (second ? 0u : (uint32_t)pl.start * lc.rec);
    dst = st + lc.dst_off + (second ? (uint32_t)first * lc.rec : 0u);
    bytes = (uint32_t)(second ? cnt - first : first) * lc.rec;
  } else if (lc.kind == 6) {
    src = lc.base + (uint64_t)bg * lc.stride;
    dst = st + lc.dst_off;
    bytes = (MODE == kModeReplay) ? (uint32_t)p.n_pos * N * S_IO : 0u;
  } else {  // the new entry's k (7) or v (8), into record c
    src = lc.base + (uint64_t)((lc.kind == 7) ? bg : bh) * lc.stride;
    dst = st + lc.dst_off + (uint32_t)pl.c * lc.rec;
    bytes = from_inputs ? (uint32_t)lc.stride : 0u;
  }
  return pl.active ? bytes : 0u;
}

// The unit's indices, pointer word and flush mask, written into its stage for the
// consumers: int32 word, mask, b, h, g, rb.
__device__ __forceinline__ void write_meta(uint8_t* st, const KParams& p, const UnitIdx& x, int32_t word, int msk) {
  int4* m = reinterpret_cast<int4*>(st + p.off_meta);
  m[0] = make_int4(word, msk, x.b, x.h);
  m[1] = make_int4(x.g, x.rb, 0, 0);
}

// The producer warp fills the CTA's units in order, kUnitsPerIssue at a time: it waits
// until their stages are free, the lane of kind 0 arms each stage's "full" barrier
// with the unit's byte count, and then one predicated bulk-copy instruction issues every
// copy of the batch (lane = unit in batch * kCopyKinds + kind). Issuing costs the warp
// about as much for one copy as for a whole batch, so batching is what keeps the stream
// fed; the per-unit arithmetic is kept short for the same reason (the producer's loop,
// not the memory, bounds a stream of small tiles): every 32 units, lane L works out
// unit L's indices (the divisions) and reads its pointer word, once, one chunk ahead.
template <int MODE, int CKPT, int S_IO>
__device__ void producer_loop(const KParams& p, uint8_t* stages, Bars* bars) {
  constexpr int U = kUnitsPerIssue;
  static_assert(U * kCopyKinds <= 32 && (32 % U) == 0, "a batch's copies must fit one warp and tile 32 units");
  const int lane = threadIdx.x & 31;
  const int NS = p.num_stages;
  const uint64_t stream_policy = l2_evict_first_policy();
  const uint64_t keep_policy = l2_evict_normal_policy();
  const int total = cta_units(p);
  const bool from_inputs = MODE == kModeReplay && p.append_here;  // one-position call's entry
  struct Pre {
    UnitIdx x;
    int32_t word;
    int msk;
    float dt, a;  // the new entry's Delta and a (one-position calls)
  };
  auto prefetch = [&](int i0) {
    Pre q;
    q.x = UnitIdx{0, 0, 0, 0};
    q.word = 0;
    q.msk = 1;
    q.dt = q.a = 0.f;
    if (i0 + lane < total) {
      q.x = unit_idx(p, cta_unit(p, i0 + lane));
      q.word = __ldg(p.counts_in + q.x.b);
      if (MODE == kModeFlush && p.mask) q.msk = __ldg(p.mask + q.x.b);
      if (from_inputs) {
        const size_t bh = (size_t)q.x.b * p.H + q.x.h;
        q.dt = __ldg(p.dt + bh);
        q.a = __ldg(p.a + bh);
      }
    }
    return q;
  };
  auto fetch = [&](const Pre& q, int i) {  // unit i's entry of the chunk, from its lane
    Pre r;
    const int src = i & 31;
    r.x.b = __shfl_sync(0xffffffffu, q.x.b, src);
    r.x.h = __shfl_sync(0xffffffffu, q.x.h, src);
    r.x.g = __shfl_sync(0xffffffffu, q.x.g, src);
    r.x.rb = __shfl_sync(0xffffffffu, q.x.rb, src);
    r.word = __shfl_sync(0xffffffffu, q.word, src);
    r.msk = __shfl_sync(0xffffffffu, q.msk, src);
    r.dt = __shfl_sync(0xffffffffu, q.dt, src);
    r.a = __shfl_sync(0xffffffffu, q.a, src);
    return r;
  };
  Pre cur = prefetch(0), nxt = prefetch(32);
  const int j = lane / kCopyKinds;     // this lane's unit within the batch
  const int kind = lane % kCopyKinds;  // and its copy
  const LaneCopy lc = lane_copy<MODE, CKPT, S_IO>(p, kind);
  // stage and use of the batch's first unit, advanced without divisions
  int s0 = 0, k0 = 0;
  for (int i0 = 0; i0 < total; i0 += U) {
    if ((i0 & 31) == 0 && i0 > 0) {
      cur = nxt;
      nxt = prefetch(i0 + 32);
    }
    // every lane waits for the batch's stages (the releases of their previous uses; a
    // version where lane 0 alone waited and the warp followed it measured ~20% slower),
    // and the warp follows lane 0's outcome
    bool ready = true;
    {
      int s = s0, k = k0;
#pragma unroll
      for (int jj = 0; jj < U; ++jj) {
        if (i0 + jj < total && k > 0) ready = mbar_wait_bounded(&bars->empty[s], (k - 1) & 1) && ready;
        if (++s == NS) {
          s = 0;
          ++k;
        }
      }
    }
    if (lane == 0) {
      if (!ready) {
        report_error(p.status, kErrWaitTimeout);
        bars->abort_flag = 1;
      }
      ready = ready && *reinterpret_cast<volatile int*>(&bars->abort_flag) == 0;
    }
    if (!__shfl_sync(0xffffffffu, ready ? 1 : 0, 0)) break;  // the warp decides together
    const int i = i0 + j;
    const bool valid = j < U && i < total;
    int s = s0 + (j < U ? j : 0);  // this lane's unit's stage (U <= NS)
    if (s >= NS) s -= NS;
    s0 += U;
    while (s0 >= NS) {
      s0 -= NS;
      ++k0;
    }
    const Pre u = fetch(cur, i);
    uint8_t* st = stages + (size_t)s * p.stage_bytes;
    uint64_t* bar = &bars->full[s];
    const Plan pl = make_plan<MODE, CKPT, S_IO>(p, u.x, u.word, u.msk);
    if (valid && kind == 0) {
      write_meta(st, p, u.x, u.word, u.msk);
      if (pl.corrupt) report_error(p.status, kErrPointer);
      if (from_inputs && pl.active)  // the new entry's Delta, a (and zero padding) after its v
        *reinterpret_cast<float4*>(st + p.off_rec + (size_t)pl.c * p.rec_bytes + (size_t)p.P * S_IO) =
            make_float4(u.dt, u.a, 0.f, 0.f);
      mbar_arrive_expect_tx(bar, pl.bytes);
    }
    __syncwarp();
    const uint8_t* src;
    uint8_t* dst;
    uint32_t bytes = unit_copy<MODE, CKPT, S_IO>(p, lc, pl, st, src, dst);
    if (!valid) bytes = 0;
    __syncwarp();
    if (bytes) bulk_g2s_hint(dst, src, bytes, bar, kind == 0 ? stream_policy : keep_policy);
    if (valid && kind == 0) bars->last_fill[s] = i;
  }
  // Never leave with copies in flight into this CTA's shared memory: wait (bounded) for
  // the latest fill of every stage.
  __syncwarp();
  for (int st_i = 0; st_i < NS; ++st_i) {
    const int i = bars->last_fill[st_i];
    if (i >= 0 && !mbar_wait_bounded(&bars->full[st_i], (i / NS) & 1) && lane == 0)
      report_error(p.status, kErrWaitTimeout);
  }
}

// The eager baseline's producer: one unit at a time; the tile (and the shared FP8 state's
// scales) by bulk copy, the new token's k, v, Delta, a and q gathered with per-lane
// cp.async.
template <int CKPT, int S_IO>
__device__ void producer_loop_eager(const KParams& p, uint8_t* stages, Bars* bars) {
  const int lane = threadIdx.x & 31;
  const int NS = p.num_stages;
  const uint64_t stream_policy = l2_evict_first_policy();
  const size_t P = p.P, N = p.N;
  const int total = cta_units(p);
  for (int i = 0; i < total; ++i) {
    const int u = cta_unit(p, i);
    const int s = i % NS;
    const int k = i / NS;
    if (k > 0 && !__all_sync(0xffffffffu, mbar_wait_bounded(&bars->empty[s], (k - 1) & 1))) {
      if (lane == 0) {
        report_error(p.status, kErrWaitTimeout);
        bars->abort_flag = 1;
      }
      break;
    }
    const int ab = (lane == 0) ? *reinterpret_cast<volatile int*>(&bars->abort_flag) : 0;
    if (__shfl_sync(0xffffffffu, ab, 0)) break;
    const UnitIdx x = unit_idx(p, u);
    const Plan pl = make_plan<kModeEager, CKPT, S_IO>(p, x, 0, 1);
    uint8_t* st = stages + (size_t)s * p.stage_bytes;
    uint64_t* bar = &bars->full[s];
    const size_t bh = (size_t)pl.b * p.H + pl.h;
    const size_t bg = (size_t)pl.b * p.G + pl.g;
    const size_t row0 = bh * P + pl.r0;  // the unit's rows
    const uint32_t rows = (uint32_t)pl.rows;
    uint8_t* recbuf = st + p.off_rec;
    uint8_t* kbuf = st + p.off_krec;
    if (lane == 0) {
      write_meta(st, p, x, 0, 1);
      mbar_arrive_expect_tx(bar, pl.bytes);
    }
    __syncwarp();
    if (lane == 0)
      bulk_g2s_hint(st, pl.fp32_tile ? (const void*)(p.S + row0 * N) : (const void*)(p.S8 + row0 * N),
                    pl.fp32_tile ? (uint32_t)(rows * N * 4) : (uint32_t)(rows * N), bar, stream_policy);
    if (lane == 1 && !pl.fp32_tile) bulk_g2s(st + (size_t)p.rows_unit * N, p.Sscale + row0, rows * 4u, bar);
    const int kpe = (int)(N * S_IO / 16);
    const int vpe = (int)(P * S_IO / 16);
    for (int idx = lane; idx < 2 * kpe + vpe; idx += 32) {
      if (idx < kpe) {
        cp_async16(st + p.off_q + idx * 16, static_cast<const uint8_t*>(p.q) + bg * N * S_IO + idx * 16);
      } else if (idx < 2 * kpe) {
        const int ch = idx - kpe;
        cp_async16(kbuf + ch * 16, static_cast<const uint8_t*>(p.k) + bg * N * S_IO + ch * 16);
      } else {
        const int ch = idx - 2 * kpe;
        cp_async16(recbuf + ch * 16, static_cast<const uint8_t*>(p.v) + bh * P * S_IO + ch * 16);
      }
    }
    if (lane == 0) cp_async4(recbuf + P * S_IO, p.dt + bh);
    if (lane == 1) cp_async4(recbuf + P * S_IO + 4, p.a + bh);
    cp_async_arrive(bar);
    if (lane == 0) bars->last_fill[s] = i;
  }
  __syncwarp();
  for (int st_i = 0; st_i < NS; ++st_i) {
    const int i2 = bars->last_fill[st_i];
    if (i2 >= 0 && !mbar_wait_bounded(&bars->full[st_i], (i2 / NS) & 1) && lane == 0)
      report_error(p.status, kErrWaitTimeout);
  }
}

// ---------------------------------------------------------------------------- consumers
// The coefficient warp's share of a unit (all 32 lanes; ws is its group's workspace):
//  * fold weights of the c buffered entries when the unit folds (blog "Ruta 'estado y
//    salida'"): sig_j = Delta_j prod_{j<i<c} a_i and abar = prod_{i<c} a_i (the eager
//    baseline: its single entry, sig_0 = Delta, abar = a);
//  * for every position s the outputs replay the entries o0 .. c+s, o0 = c after a fold
//    and 0 otherwise (blog "Ruta 'solo salida'"):
//        alpha_s = prod_{o0<=i<=c+s} a_i,   w_{s,j} = Delta_j prod_{j<i<=c+s} a_i,
//        u_s[p]  = sum_{o0<=j<=c+s} w_{s,j} (k_j . q_s) v_j[p],
//    so that y_s = alpha_s (S q_s) + u_s. The products of decay factors are suffix
//    products over the window, one lane per entry.
template <int N, typename IO, int MODE>
__device__ __forceinline__ void fold_weights(const Records<N, IoT<IO>::bytes>& rec, int c, float* sig, int lane) {
  if (MODE == kModeEager) {
    if (lane == 0) {
      sig[0] = rec.dt(0);
      sig[kMaxWindow] = rec.a(0);
    }
    return;
  }
  float xa = 1.f, xd = 0.f;
  if (lane < c) {
    xa = rec.a(lane);
    xd = rec.dt(lane);
  }
  const float incl = warp_suffix_prod(xa, lane);  // prod_{lane <= i < c} a_i
  float excl = __shfl_down_sync(0xffffffffu, incl, 1);
  if (lane == 31) excl = 1.f;
  if (lane < c) sig[lane] = xd * excl;
  if (lane == 0) sig[kMaxWindow] = incl;
}

// The coefficients of the positions s = s0, s0 + ds, ... (< n) by one warp: alpha_s and
// cw[s][l] = w_{s,l} (k_l . q_s) with w_{s,l} = Delta_l prod_{l < i <= last_s} a_i, zero
// past the position's last entry so that the row lanes may read whole vectors. Two
// forms, chosen by measurement:
//  * output_coefs_pairs, for one-position calls on the FP32 checkpoint, where one warp
//    per group forms the coefficients while four stream the state and its chain is on
//    the unit's critical path: a lane pair per entry, sixteen entries per pass (half of k_l . q_s per lane,
//    the second half one 4-element chunk rotated so that the pair's reads fall in
//    different shared-memory banks, one shuffle to combine), and the decay weights from
//    one suffix-product scan of the window's a_i (one read per lane, five shuffles).
//    Its chain is one round of shared-memory reads, the products and a few shuffles.
//  * output_coefs_quarters, for multi-position calls, where all five warps of a group
//    form coefficients at once and the shared-memory pipe, not one warp's chain, is the
//    limit, and for the FP8 / FP4 read copies, whose row warps (decoding the codes) rather than
//    the coefficient warp set the pace: four lanes per entry, eight entries per pass,
//    and the decay weights by a suffix-product scan across the lanes, which issues fewer
//    shared-memory requests per position than the broadcast reads.
// Both keep the raw products k_l . q_s in kqraw[s][l] (the group's workspace) and, with
// `reuse`, take them from there: the heads of a chunk share their sequence's window and
// their group's k and q, so a group that takes consecutive units of one chunk forms the
// products once (blog, end of "Ruta 'solo salida'": k and q belong to the group).
template <int N, typename IO>
__device__ __forceinline__ void output_coefs_quarters(const Records<N, IoT<IO>::bytes>& rec, const uint8_t* qbuf, int c,
                                                      int n, int o0, int s0, int ds, float* alpha, float* cw,
                                                      float* kqraw, bool reuse, int lane) {
  constexpr int S_IO = IoT<IO>::bytes;
  constexpr int QN = N / 4;  // elements of a quarter row
  const int width = c + n - o0;  // window entries (at most L)
  float xa = 1.f, xd = 0.f;
  if (lane < width) {
    xa = rec.a(o0 + lane);
    xd = rec.dt(o0 + lane);
  }
  const int quarter = lane & 3;
  const int rot = (quarter >> 1) * 4;
  static_assert((QN & (QN - 1)) == 0, "a quarter row is a power of two elements");
  // raw k_l . q_s into kqraw[s][l] (kept there from the group's previous unit when that
  // unit had the same sequence and k/q group: same window, same products)
  for (int l0 = 0; l0 < (reuse ? 0 : width); l0 += 8) {
    const int l = l0 + (lane >> 2);
    const uint8_t* kq = rec.k(o0 + (l < width ? l : 0)) + (size_t)quarter * QN * S_IO;
    for (int s = s0; s < n; s += ds) {
      const uint8_t* qq = qbuf + ((size_t)s * N + quarter * QN) * S_IO;
      float d0 = 0.f, d1 = 0.f;
#pragma unroll
      for (int e = 0; e < QN; e += 8) {
        // quarters 2 and 3 start one 4-element chunk later (mod QN): with BF16 records a
        // quarter is 16 banks wide, so quarter q and q + 2 of one entry would share banks
        const int e0 = (e + rot) & (QN - 1), e1 = (e + 4 + rot) & (QN - 1);
        d0 += dot4(IoT<IO>::load4(kq + (size_t)e0 * S_IO), IoT<IO>::load4(qq + (size_t)e0 * S_IO));
        if (e + 4 < QN)
          d1 += dot4(IoT<IO>::load4(kq + (size_t)e1 * S_IO), IoT<IO>::load4(qq + (size_t)e1 * S_IO));
      }
      float d = d0 + d1;
      d += __shfl_xor_sync(0xffffffffu, d, 1);
      d += __shfl_xor_sync(0xffffffffu, d, 2);
      if (quarter == 0 && l < width) kqraw[s * kMaxWindow + l] = d;
    }
  }
  __syncwarp();
  for (int s = s0; s < n; s += ds) {
    const int last = c + s - o0;  // position s replays window entries 0 .. last
    const float incl = warp_suffix_prod(lane <= last ? xa : 1.f, lane);  // prod_{lane<=i<=last} a_i
    float excl = __shfl_down_sync(0xffffffffu, incl, 1);
    if (lane == 31) excl = 1.f;
    if (lane == 0) alpha[s] = incl;
    // w_{s,l} (k_l . q_s); zero past `last`, so that the row lanes may read whole vectors
    const float kqv = (lane <= last) ? kqraw[s * kMaxWindow + lane] : 0.f;
    cw[s * kMaxWindow + lane] = (lane <= last) ? xd * excl * kqv : 0.f;
  }
}


template <int N, typename IO>
__device__ __forceinline__ void output_coefs_pairs(const Records<N, IoT<IO>::bytes>& rec, const uint8_t* qbuf, int c,
                                                   int n, int o0, int s0, int ds, float* alpha, float* cw,
                                                   float* kqraw, bool reuse, int lane) {
  constexpr int S_IO = IoT<IO>::bytes;
  constexpr int HN = N / 2;       // elements of half a row
  constexpr int HC = HN / 4;      // 4-element chunks of half a row
  const int width = c + n - o0;   // window entries (at most kMaxWindow)
  const int half = lane & 1;
  // the window's decay factors, lane l holding a_{o0+l}: read once, then one suffix-
  // product scan per position gives every product the weights need
  const float al = (lane < width) ? rec.a(o0 + lane) : 1.f;
  for (int s = s0; s < n; s += ds) {
    const int last = c + s - o0;  // position s replays window entries 0 .. last
    const float suf = warp_suffix_prod(lane <= last ? al : 1.f, lane);  // prod_{lane <= i <= last} a_i
    if (lane == 0) alpha[s] = suf;
    for (int e0 = 0; e0 < width; e0 += 16) {
      const int e = e0 + (lane >> 1);
      const int er = (e < width) ? e : width - 1;  // lanes past the window read a valid record
      float kq;
      if (reuse) {  // the group's previous unit had the same sequence and k/q group
        kq = kqraw[s * kMaxWindow + e];
      } else {
        const uint8_t* kh = rec.k(o0 + er) + (size_t)half * HN * S_IO;
        const uint8_t* qh = qbuf + ((size_t)s * N + half * HN) * S_IO;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int t = 0; t < HC; ++t) {
          const int off = ((t + half) % HC) * 4 * S_IO;
          const float4 kk = IoT<IO>::load4(kh + off);
          const float4 qq = IoT<IO>::load4(qh + off);
          d[t & 3] = fmaf(kk.x, qq.x, fmaf(kk.y, qq.y, fmaf(kk.z, qq.z, fmaf(kk.w, qq.w, d[t & 3]))));
        }
        kq = (d[0] + d[1]) + (d[2] + d[3]);
        kq += __shfl_xor_sync(0xffffffffu, kq, 1);
        if (half == 0) kqraw[s * kMaxWindow + e] = kq;
      }
      // prod_{e < i <= last} a_i: the scan's value one lane up (empty past lane 31)
      const float up = __shfl_sync(0xffffffffu, suf, (e + 1) & 31);
      const float w = (e + 1 < 32) ? up : 1.f;
      if (half == 0 && e < kMaxWindow) cw[s * kMaxWindow + e] = (e <= last) ? rec.dt(o0 + er) * w * kq : 0.f;
    }
  }
}

// One-position calls copy their new entry from the inputs into record c of each unit's
// stage; the coefficient warp then appends it to the ring at slot (start + c) mod cap for
// the calls that follow: the head record (v, Delta, a) once per head (row block 0), the k
// record once per sequence and k/q group (its first head). Nothing else in the launch
// reads that slot: every unit copies records [start, start + c) only.
template <int S_IO>
__device__ __forceinline__ void ring_append(const KParams& p, const Plan& pl, const uint8_t* st, int lane) {
  if (pl.rb != 0) return;
  int slot = pl.start + pl.c;
  slot -= (slot >= p.cap) ? p.cap : 0;
  const int kpe = (pl.h == pl.g * p.hpg) ? p.N * S_IO / 16 : 0;  // 16-byte pieces of k (first head)
  const int rpe = p.rec_bytes / 16;                                // of the head record
  const uint4* ksrc = reinterpret_cast<const uint4*>(st + p.off_krec + (size_t)pl.c * p.rec_k_bytes);
  const uint4* rsrc = reinterpret_cast<const uint4*>(st + p.off_rec + (size_t)pl.c * p.rec_bytes);
  uint4* kdst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.ring_k) +
                                         (((size_t)pl.b * p.G + pl.g) * p.cap + slot) * p.rec_k_bytes);
  uint4* rdst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.ring) +
                                         (((size_t)pl.b * p.H + pl.h) * p.cap + slot) * p.rec_bytes);
  for (int t = lane; t < kpe + rpe; t += 32) {
    if (t < kpe)
      kdst[t] = ksrc[t];
    else
      rdst[t - kpe] = rsrc[t - kpe];
  }
}

// One unit, by one consumer group: kGroupGemvWarps warps stream the state rows (dot
// products, or the fold and its write-back) while the group's coefficient warp works out
// the decay weights and the buffer terms from the records; the two meet at the group
// barrier before the outputs are written.
template <int N, typename IO, int CKPT, int MODE, int NQ, int NG>
__device__ __forceinline__ void consume_unit(const KParams& p, const Plan& pl, uint8_t* st, uint8_t* ws, int gtid,
                                             int bar_id, int gemv_bar_id, bool reuse) {
  using Gr = Groups<NG>;
  constexpr int GT = Gr::kThreads;    // the whole group (barriers)
  constexpr int GW = kGroupGemvWarps;  // warps on the state rows
  constexpr int GTG = GW * 32;
  constexpr int TPR = N / 4;
  constexpr int RPW = 32 / TPR;  // rows per warp pass
  constexpr int RPG = GW * RPW;  // rows per group pass
  constexpr int RT = kRowsPerThread;
  constexpr int RGR = RPG * RT;  // rows per row group
  constexpr int S_IO = IoT<IO>::bytes;
  constexpr int NQR = NQ > 0 ? NQ : 1;
  using Red = SegReduce<RT, TPR>;
  const int lane = gtid & 31;
  const int gw = gtid >> 5;
  const bool coef_warp = gw == GW;
  // this thread's rows of a row group: rbase .. rbase + RT - 1 (contiguous, so that a
  // fold reads their weights as four 16-byte vectors)
  const int rbase = (gw * RPW + lane / TPR) * RT;
  const int col = (lane % TPR) * 4;
  const int P = pl.rows;  // the unit's rows: r0 .. r0 + P - 1 of the head's PH
  const int PH = p.P;
  const int r0 = pl.r0;
  const int c = pl.c;
  const int n = (MODE == kModeReplay) ? p.n_pos : (MODE == kModeEager ? 1 : 0);
  const int cf = (MODE == kModeEager) ? 1 : (pl.fold ? c : 0);  // entries folded into the state
  const int o0 = pl.fold ? c : 0;                                // first entry the outputs replay
  const int wts = p.wt_stride;  // row stride of the fold weight table, >= P, multiple of RT
  const uint8_t* tile = st;
  const uint8_t* qbuf = st + p.off_q;
  constexpr int kCodeDiv = (CKPT == kCkptFp4) ? 2 : 1;  // read copy: code bytes per row = N / kCodeDiv
  const Records<N, S_IO> rec{st + p.off_krec, st + p.off_rec, PH, p.rec_bytes, p.rec_k_bytes};  // whole records: v_j[0 .. PH)
  const float* scale_tile = reinterpret_cast<const float*>(tile + (size_t)p.rows_unit * (N / kCodeDiv));
  float* alpha = reinterpret_cast<float*>(ws + p.ws_alpha);  // [kMaxPos]
  float* sig = reinterpret_cast<float*>(ws + p.ws_sig);      // fold weights; [kMaxWindow] = abar
  float* cw = reinterpret_cast<float*>(ws + p.ws_cw);        // [kMaxPos][kMaxWindow] entry coefficients
  float* wt = reinterpret_cast<float*>(ws + p.ws_wt);        // [c][wts] fold weight times v_j[p]
  float* kqraw = reinterpret_cast<float*>(ws + p.ws_kq);     // [kMaxPos][kMaxWindow] raw k_l . q_s
  float* sinv = reinterpret_cast<float*>(ws + p.ws_inv);     // [row group] inverse row scales (fold)
  const size_t bh = (size_t)pl.b * p.H + pl.h;
  const int ngroups = (P + RGR - 1) / RGR;
  const bool fold = pl.fold;

  if (coef_warp) {
    // ---- the coefficient warp: fold weights first (the fold waits for them), then the
    // outputs' buffer terms while the fold runs
    if (fold) {
      fold_weights<N, IO, MODE>(rec, c, sig, lane);
      group_sync(bar_id, GT);
    }
    // the positions are spread over the group's warps: this warp takes 0, GW + 1, ...
    if (MODE == kModeReplay) {
      if (NQ > 1 || CKPT != kCkptF32)
        output_coefs_quarters<N, IO>(rec, qbuf, c, n, o0, 0, GW + 1, alpha, cw, kqraw, reuse, lane);
      else
        output_coefs_pairs<N, IO>(rec, qbuf, c, n, o0, 0, GW + 1, alpha, cw, kqraw, reuse, lane);
    }
    group_sync(bar_id, GT);
    // the new entry into the ring, while the row warps write the outputs
    if (MODE == kModeReplay && NQ == 1 && p.append_here) ring_append<S_IO>(p, pl, st, lane);
  } else {
    float4 qr[NQR];
#pragma unroll
    for (int s = 0; s < NQ; ++s)
      qr[s] = (s < n) ? IoT<IO>::load4(qbuf + ((size_t)s * N + col) * S_IO) : make_float4(0.f, 0.f, 0.f, 0.f);

    // state rows of one row group (the read copy keeps its row scale for the dot product)
    auto load_rows = [&](float4 (&x)[RT], int gi, bool dequant) {
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const int pr = gi * RGR + rbase + r;
        x[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (pr < P) {
          if (pl.fp32_tile) {
            x[r] = *reinterpret_cast<const float4*>(tile + ((size_t)pr * N + col) * 4);
          } else {
            const float4 e =
                (CKPT == kCkptFp4)
                    ? e2m1x4_to_float4(*reinterpret_cast<const unsigned short*>(tile + (size_t)pr * (N / 2) + col / 2))
                    : e4m3x4_to_float4(*reinterpret_cast<const uint32_t*>(tile + (size_t)pr * N + col));
            if (dequant) {  // eager on a shared FP8 state: dequantise
              const float sc = scale_tile[pr];
              x[r] = make_float4(e.x * sc, e.y * sc, e.z * sc, e.w * sc);
            } else {
              x[r] = e;
            }
          }
        }
      }
    };
    // the row dot products of one row group, reduced: lane holds rows base .. base+kHeld
    float dv[NQR][Red::kHeld];
    int dbase = 0;
    bool dwr = false;
    auto row_dots = [&](const float4 (&x)[RT]) {
#pragma unroll
      for (int s = 0; s < NQ; ++s) {
        if (s < n) {
          float part[RT];
#pragma unroll
          for (int r = 0; r < RT; ++r) part[r] = dot4(x[r], qr[s]);
          dwr = Red::run(part, lane, dbase);
#pragma unroll
          for (int i = 0; i < Red::kHeld; ++i) dv[s][i] = part[i];
        }
      }
    };
    // The read copy with BF16 inputs: the codes stay f16 (one conversion per two codes)
    // and meet the queries, as f16, in mixed-precision FMAs that accumulate in f32; the
    // products are exact, so the dot products equal those of row_dots on widened values.
    constexpr bool kHalfDots = (CKPT != kCkptF32) && (S_IO == 2) && (MODE == kModeReplay);
    uint2 qh[kHalfDots ? NQR : 1];
#pragma unroll
    for (int s = 0; s < (kHalfDots ? NQR : 1); ++s) qh[s] = float4_to_half4(qr[s]);
    auto rows_dots_half = [&](int gi) {
      uint2 xc[RT];
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const int pr = gi * RGR + rbase + r;
        xc[r] = make_uint2(0u, 0u);
        if (pr < P)
          xc[r] = (CKPT == kCkptFp4)
                      ? e2m1x4_to_half4(*reinterpret_cast<const unsigned short*>(tile + (size_t)pr * (N / 2) + col / 2))
                      : e4m3x4_to_half4(*reinterpret_cast<const uint32_t*>(tile + (size_t)pr * N + col));
      }
#pragma unroll
      for (int s = 0; s < NQ; ++s) {
        if (s < n) {
          float part[RT];
#pragma unroll
          for (int r = 0; r < RT; ++r) part[r] = dot4_h(xc[r], qh[s]);
          dwr = Red::run(part, lane, dbase);
#pragma unroll
          for (int i = 0; i < Red::kHeld; ++i) dv[s][i] = part[i];
        }
      }
    };
    // Multi-position calls, where a lane ends with one row (N >= 64): the v_l[p] of the
    // first kPre window entries and the row's scale are read into registers before the
    // group barrier, while the group forms the coefficients; after the barrier only the
    // coefficients are read. (One-position calls measured no gain from it.)
    constexpr int kPre = (MODE == kModeReplay && NQ > 1 && Red::kHeld == 1) ? 16 : 0;  // 0 or 16
    float vpre[16];  // the first kPre used
    float scpre = 1.f;
    auto preload = [&](int gi, bool from_copy) {
      if constexpr (kPre > 0) {
        const int pr = gi * RGR + rbase + dbase;
        const bool own = dwr && pr < P;
        const int width = c + n - o0;
#pragma unroll
        for (int r = 0; r < kPre; ++r)
          vpre[r] = (own && r < width) ? IoT<IO>::load1(rec.v(o0 + r) + (size_t)(r0 + pr) * S_IO) : 0.f;
        scpre = (own && from_copy) ? scale_tile[pr] : 1.f;
      }
    };
    // y_s[p] = alpha_s d + sum_l cw[s][l] v_l[p] (replay) or y[p] = d (eager), by the
    // lanes that hold row p's dot products; each v_l[p] is read once for all positions,
    // eight entries in flight at a time (cw is zero past each position's window, v is
    // zero past the unit's). `pre`: the preload above ran for this row group.
    auto emit = [&](int gi, bool from_copy, bool pre) {
      if (MODE == kModeFlush) return;
#pragma unroll
      for (int i = 0; i < Red::kHeld; ++i) {
        const int pr = gi * RGR + rbase + dbase + i;
        if (dwr && pr < P) {
          const float sc = (kPre > 0 && pre) ? scpre : (from_copy ? scale_tile[pr] : 1.f);
          if (MODE == kModeReplay && NQR == 1) {
            const int last = c - o0;  // the one position replays window entries 0 .. last
            float b0 = 0.f, b1 = 0.f;
            int l0 = 0;
            if (kPre > 0 && pre) {
              const float4* c4 = reinterpret_cast<const float4*>(cw);
              const float4 c0 = c4[0], c1 = c4[1], c2 = c4[2], c3 = c4[3];
              b0 = fmaf(c0.x, vpre[0], fmaf(c0.y, vpre[1], fmaf(c0.z, vpre[2], fmaf(c0.w, vpre[3],
                   fmaf(c1.x, vpre[4], fmaf(c1.y, vpre[5], fmaf(c1.z, vpre[6], c1.w * vpre[7])))))));
              b1 = fmaf(c2.x, vpre[8], fmaf(c2.y, vpre[9], fmaf(c2.z, vpre[10], fmaf(c2.w, vpre[11],
                   fmaf(c3.x, vpre[12], fmaf(c3.y, vpre[13], fmaf(c3.z, vpre[14], c3.w * vpre[15])))))));
              l0 = kPre;
            }
            for (; l0 <= last; l0 += 8) {
              float vv[8];
#pragma unroll
              for (int r = 0; r < 8; ++r)
                vv[r] = (l0 + r <= last) ? IoT<IO>::load1(rec.v(o0 + l0 + r) + (size_t)(r0 + pr) * S_IO) : 0.f;
#pragma unroll
              for (int r = 0; r < 8; r += 2) {
                if (l0 + r <= last) b0 = fmaf(cw[l0 + r], vv[r], b0);
                if (l0 + r + 1 <= last) b1 = fmaf(cw[l0 + r + 1], vv[r + 1], b1);
              }
            }
            p.y[(((size_t)pl.b * n) * p.H + pl.h) * PH + r0 + pr] = fmaf(alpha[0], dv[0][i] * sc, b0 + b1);
          } else if (MODE == kModeReplay) {
            const int width = c + n - o0;
            float b[NQR];
#pragma unroll
            for (int s = 0; s < NQR; ++s) b[s] = 0.f;
            int l0 = 0;
            if (kPre > 0 && pre) {
#pragma unroll
              for (int h = 0; h < kPre; h += 8) {
                if (h < width) {
#pragma unroll
                  for (int s = 0; s < NQR; ++s) {
                    if (s < n) {
                      const float4 c0 = *reinterpret_cast<const float4*>(cw + s * kMaxWindow + h);
                      const float4 c1 = *reinterpret_cast<const float4*>(cw + s * kMaxWindow + h + 4);
                      const float* vv = vpre + h;
                      b[s] = fmaf(c0.x, vv[0], fmaf(c0.y, vv[1], fmaf(c0.z, vv[2], fmaf(c0.w, vv[3],
                             fmaf(c1.x, vv[4], fmaf(c1.y, vv[5], fmaf(c1.z, vv[6], fmaf(c1.w, vv[7], b[s]))))))));
                    }
                  }
                }
              }
              l0 = kPre;
            }
            for (; l0 < width; l0 += 8) {
              float vv[8];
#pragma unroll
              for (int r = 0; r < 8; ++r)
                vv[r] = (l0 + r < width) ? IoT<IO>::load1(rec.v(o0 + l0 + r) + (size_t)(r0 + pr) * S_IO) : 0.f;
#pragma unroll
              for (int s = 0; s < NQR; ++s) {
                if (s < n) {
                  const float4 c0 = *reinterpret_cast<const float4*>(cw + s * kMaxWindow + l0);
                  const float4 c1 = *reinterpret_cast<const float4*>(cw + s * kMaxWindow + l0 + 4);
                  b[s] = fmaf(c0.x, vv[0], fmaf(c0.y, vv[1], fmaf(c0.z, vv[2], fmaf(c0.w, vv[3],
                         fmaf(c1.x, vv[4], fmaf(c1.y, vv[5], fmaf(c1.z, vv[6], fmaf(c1.w, vv[7], b[s]))))))));
                }
              }
            }
#pragma unroll
            for (int s = 0; s < NQR; ++s)
              if (s < n) p.y[(((size_t)pl.b * n + s) * p.H + pl.h) * PH + r0 + pr] = fmaf(alpha[s], dv[s][i] * sc, b[s]);
          } else {
            p.y[bh * PH + r0 + pr] = dv[0][i] * sc;
          }
        }
      }
    };

    float4 x[RT];
    if (!fold) {
      // ---- output-only route: row group 0's dot products, then wait for the buffer
      // terms; further row groups (P > one row group) follow with the terms in hand
      if (kHalfDots && !pl.fp32_tile) {
        rows_dots_half(0);
      } else {
        load_rows(x, 0, false);
        row_dots(x);
      }
      preload(0, !pl.fp32_tile);
      if (NQ > 1) output_coefs_quarters<N, IO>(rec, qbuf, c, n, o0, gw + 1, GW + 1, alpha, cw, kqraw, reuse, lane);  // positions gw+1, ...
      group_sync(bar_id, GT);
      emit(0, !pl.fp32_tile, true);
      for (int gi = 1; gi < ngroups; ++gi) {
        if (kHalfDots && !pl.fp32_tile) {
          rows_dots_half(gi);
        } else {
          load_rows(x, gi, false);
          row_dots(x);
        }
        preload(gi, !pl.fp32_tile);
        emit(gi, !pl.fp32_tile, true);
      }
    } else {
      // ---- fold (state route), write the state back, outputs from the fresh rows
      load_rows(x, 0, MODE == kModeEager);
      group_sync(bar_id, GT);  // the fold weights are in
      // wt[j][p] = sig_j v_j[p] (zero for p >= P), a thread per (8 entries, row): every
      // load independent, consecutive threads on consecutive rows
      for (int job = gtid; job < wts * ((cf + 7) / 8); job += GTG) {
        const int j8 = job / wts;
        const int pp = job - j8 * wts;
        const int pv = pp < P ? pp : 0;
        float wv[8];  // all eight reads first: the table writes could alias them
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const int jj = min(j8 * 8 + r, cf - 1);
          wv[r] = sig[jj] * IoT<IO>::load1(rec.v(jj) + (size_t)(r0 + pv) * S_IO);
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const int jj = j8 * 8 + r;
          if (jj < cf) wt[(size_t)jj * wts + pp] = pp < P ? wv[r] : 0.f;
        }
      }
      group_sync(gemv_bar_id, GTG);
      const float abar = sig[kMaxWindow];
      for (int gi = 0; gi < ngroups; ++gi) {
        if (gi > 0) load_rows(x, gi, MODE == kModeEager);
#pragma unroll
        for (int r = 0; r < RT; ++r) x[r] = make_float4(abar * x[r].x, abar * x[r].y, abar * x[r].z, abar * x[r].w);
        // rank-cf update: per entry, k_j's four columns of this lane and the weights of
        // the thread's RT rows (four 16-byte broadcasts), then 4 * RT FMAs
        const int wbase = (gi * RGR + rbase < P) ? gi * RGR + rbase : 0;  // all-invalid threads read row 0
        // the next entry's k and weights are read while this entry's FMAs run
        float4 kt = IoT<IO>::load4(rec.k(0) + col * S_IO);
        float4 wcur[RT / 4];
#pragma unroll
        for (int r4 = 0; r4 < RT / 4; ++r4) wcur[r4] = reinterpret_cast<const float4*>(wt + wbase)[r4];
        for (int jj = 0; jj < cf; ++jj) {
          const int jn = min(jj + 1, cf - 1);
          const float4 kn = IoT<IO>::load4(rec.k(jn) + col * S_IO);
          float4 wn[RT / 4];
#pragma unroll
          for (int r4 = 0; r4 < RT / 4; ++r4) wn[r4] = reinterpret_cast<const float4*>(wt + (size_t)jn * wts + wbase)[r4];
#pragma unroll
          for (int r4 = 0; r4 < RT / 4; ++r4) {
            const float ws4[4] = {wcur[r4].x, wcur[r4].y, wcur[r4].z, wcur[r4].w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              float4& xr = x[r4 * 4 + t];
              xr.x = fmaf(ws4[t], kt.x, xr.x);
              xr.y = fmaf(ws4[t], kt.y, xr.y);
              xr.z = fmaf(ws4[t], kt.z, xr.z);
              xr.w = fmaf(ws4[t], kt.w, xr.w);
            }
          }
          kt = kn;
#pragma unroll
          for (int r4 = 0; r4 < RT / 4; ++r4) wcur[r4] = wn[r4];
        }
        // write the state: FP32 master, and/or the read copy's (or the shared FP8 state's)
        // codes with per-row scales, re-quantised from the fresh row
        const bool store_f32 = (MODE != kModeEager) || (CKPT == kCkptF32);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          const int pr = gi * RGR + rbase + r;
          if (store_f32 && pr < P) __stcs(reinterpret_cast<float4*>(p.S + (bh * PH + r0 + pr) * N + col), x[r]);
        }
        if constexpr (CKPT != kCkptF32) {
          // the rows' scales: their largest magnitudes by the transposing reduction (a lane
          // ends with kHeld whole rows), each row's scale and inverse worked out once, by
          // the lane that holds the row, and the inverses read back from the workspace by
          // the row's lanes (a warp's rows are its own)
          using RedMax = SegReduce<RT, TPR, true>;
          float m[RT];
#pragma unroll
          for (int r = 0; r < RT; ++r) m[r] = amax4(x[r]);
          int mbase = 0;
          const bool mwr = RedMax::run(m, lane, mbase);
          if (mwr) {
#pragma unroll
            for (int i = 0; i < RedMax::kHeld; ++i) {
              const int rr = rbase + mbase + i;
              const int pr = gi * RGR + rr;
              float sc, inv;
              if (CKPT == kCkptFp4)
                e2m1_row_scale(m[i], sc, inv);
              else
                e4m3_row_scale(m[i], sc, inv);
              sinv[rr] = inv;
              if (pr < P) p.Sscale[bh * PH + r0 + pr] = sc;
            }
          }
          __syncwarp();
#pragma unroll
          for (int r = 0; r < RT; ++r) {
            const int pr = gi * RGR + rbase + r;
            const float inv = sinv[rbase + r];
            const size_t row = bh * PH + r0 + pr;
            if (pr < P) {
              if (CKPT == kCkptFp4)
                __stcs(reinterpret_cast<unsigned short*>(p.S8 + row * (N / 2) + col / 2),
                       static_cast<unsigned short>(quant4_e2m1(x[r], inv)));
              else
                __stcs(reinterpret_cast<unsigned int*>(p.S8 + row * N + col), quant4_e4m3(x[r], inv));
            }
          }
        }
        if (MODE != kModeFlush) row_dots(x);
        if (MODE == kModeReplay && NQ > 1 && gi == 0)
          output_coefs_quarters<N, IO>(rec, qbuf, c, n, o0, gw + 1, GW + 1, alpha, cw, kqraw, reuse, lane);
        if (gi == 0) group_sync(bar_id, GT);  // the outputs' buffer terms are in
        emit(gi, false, false);
      }
    }
  }

  // ---- publish the pointer word (the pre-pass already wrote this call's entries)
  const int start = pl.start;
  const int cap = p.cap;
  if (MODE == kModeReplay) {
    if (pl.h == 0 && pl.rb == 0 && gtid == 0) {
      int start2 = fold ? start + c : start;
      start2 -= (start2 >= cap) ? cap : 0;
      const int base = fold ? 0 : c;
      const int cnt2 = base + (p.commit ? n : 0);
      p.counts_out[pl.b] = (start2 << 16) | cnt2;
      if (p.flushed && (!p.flushed_or || fold)) p.flushed[pl.b] = fold ? 1 : 0;
    }
  } else if (MODE == kModeFlush) {
    if (pl.h == 0 && pl.rb == 0 && gtid == 0) {
      int start2 = start + c;
      start2 -= (start2 >= cap) ? cap : 0;
      p.counts_out[pl.b] = start2 << 16;
      if (p.flushed) p.flushed[pl.b] = 1;
    }
  }
}

template <int N, typename IO, int CKPT, int MODE, int NQ, int NG>
__global__ void __launch_bounds__(kThreads, 1) replay_kernel(const __grid_constant__ KParams p) {
  static_assert(NG == 1 || NG == 2, "the stage protocol relies on a stage's uses two apart being one group's");
  static_assert(kProducerWarps == 1, "stages must be filled in unit order");
  using Gr = Groups<NG>;
  extern __shared__ __align__(128) uint8_t smem[];
  Bars* bars = reinterpret_cast<Bars*>(smem);
  uint8_t* stages = smem + p.stages_off;
  constexpr int S_IO = IoT<IO>::bytes;

  // this CTA lets the next kernel on the stream be scheduled (see the launch), and sets
  // up its barriers before waiting for the previous kernel to complete
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.num_stages; ++s) {
      // the producer's expect_tx (the eager gather adds its 32 lanes' cp.async arrivals)
      mbar_init(&bars->full[s], MODE == kModeEager ? 1 + 32 : 1);
      mbar_init(&bars->empty[s], Gr::kThreads);
    }
    bars->abort_flag = 0;
    for (int s = 0; s < kMaxStages; ++s) bars->last_fill[s] = -1;
    fence_mbar_init();
  }
  __syncthreads();
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the previous kernel's writes are visible

  const int warp = threadIdx.x / 32;
  if (warp >= kConsumerWarps) {
    if constexpr (MODE == kModeEager)
      producer_loop_eager<CKPT, S_IO>(p, stages, bars);
    else
      producer_loop<MODE, CKPT, S_IO>(p, stages, bars);
    return;
  }
  const int g = warp / Gr::kWarps;  // consumer group
  const int gtid = threadIdx.x - g * Gr::kThreads;
  const int bar_id = 1 + g;                 // the whole group
  const int gemv_bar_id = 1 + NG + g;       // the group's row warps only
  uint8_t* ws = smem + p.ws_off + (size_t)g * p.ws_group_bytes;
  const int NS = p.num_stages;
  const int total = cta_units(p);
  int prev_bg = -1;  // (sequence, k/q group) of the group's previous unit, -1 if none
  int s = g, k = 0;  // stage and use of unit i, advanced without divisions
  while (s >= NS) {
    s -= NS;
    ++k;
  }
  for (int i = g; i < total; i += NG) {
    // Parity waits only tell apart a phase and the one just before it, so before waiting
    // for its own fill (phase k of "full"), a group waits for the stage's previous use to
    // be released (phase k-1 of "empty"). That release may come from the other group;
    // the use before it (k-2) was this group's own, already released, so both waits are
    // exact even when the two groups drift apart.
    bool ready = true;
    if (k > 0) ready = mbar_wait_bounded(&bars->empty[s], (k - 1) & 1);
    if (ready) ready = mbar_wait_bounded(&bars->full[s], k & 1);
    const bool ok = group_all(ready, bar_id, Gr::kThreads);
    if (!ok) {
      if (gtid == 0) {
        report_error(p.status, kErrWaitTimeout);
        bars->abort_flag = 1;
      }
      break;
    }
    uint8_t* st = stages + (size_t)s * p.stage_bytes;
    const int4 m0 = reinterpret_cast<const int4*>(st + p.off_meta)[0];  // word, mask, b, h
    const int4 m1 = reinterpret_cast<const int4*>(st + p.off_meta)[1];  // g, rb
    const int32_t word = m0.x;
    const int msk = m0.y;
    const Plan pl = make_plan<MODE, CKPT, S_IO>(p, UnitIdx{m0.z, m0.w, m1.x, m1.y}, word, msk);
    // the group's previous unit had the same sequence and k/q group: its k . q products hold
    const int bg = pl.b * p.G + pl.g;
    const bool reuse = bg == prev_bg;
    prev_bg = pl.active ? bg : -1;
    if (pl.active) {
      consume_unit<N, IO, CKPT, MODE, NQ, NG>(p, pl, st, ws, gtid, bar_id, gemv_bar_id, reuse);
    } else if (pl.h == 0 && pl.rb == 0 && gtid == 0) {
      p.counts_out[pl.b] = word;  // nothing to fold: the pointer word carries over
      if (MODE == kModeFlush && p.flushed && !pl.corrupt) p.flushed[pl.b] = 0;
    }
    group_sync(bar_id, Gr::kThreads);
    mbar_arrive(&bars->empty[s]);
    s += NG;
    while (s >= NS) {
      s -= NS;
      ++k;
    }
  }
}

// ---------------------------------------------------------------------------- small kernels
// Per-row FP8 e4m3 quantisation of rows x [rows][N] (same row mapping and arithmetic as
// the fold epilogue above): scale = amax/448, codes = e4m3(x * (448/amax)).
template <int N>
__global__ void quantize_rows_kernel(const float* __restrict__ x, int64_t rows, uint8_t* __restrict__ codes,
                                     float* __restrict__ scale) {
  constexpr int TPR = N / 4;
  constexpr int RPB = 256 / TPR;  // rows per block pass
  const int t = threadIdx.x;
  const int r0 = t / TPR;
  const int col = (t % TPR) * 4;
  const int64_t passes = (rows + RPB - 1) / RPB;
  for (int64_t pass = blockIdx.x; pass < passes; pass += gridDim.x) {
    const int64_t r = pass * RPB + r0;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < rows) v = *reinterpret_cast<const float4*>(x + r * N + col);
    const float am = seg_allmax<TPR>(amax4(v));
    float sc, inv;
    e4m3_row_scale(am, sc, inv);
    if (r < rows) {
      *reinterpret_cast<uint32_t*>(codes + r * N + col) = quant4_e4m3(v, inv);
      if ((t % TPR) == 0) scale[r] = sc;
    }
  }
}

// Per-row FP4 e2m1 quantisation of rows x [rows][N] (the fold epilogue's mapping and
// arithmetic): scale = amax/6, codes = e2m1(x * (6/amax)), two codes per byte.
template <int N>
__global__ void quantize_rows_e2m1_kernel(const float* __restrict__ x, int64_t rows, uint8_t* __restrict__ codes,
                                          float* __restrict__ scale) {
  constexpr int TPR = N / 4;
  constexpr int RPB = 256 / TPR;  // rows per block pass
  const int t = threadIdx.x;
  const int r0 = t / TPR;
  const int col = (t % TPR) * 4;
  const int64_t passes = (rows + RPB - 1) / RPB;
  for (int64_t pass = blockIdx.x; pass < passes; pass += gridDim.x) {
    const int64_t r = pass * RPB + r0;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < rows) v = *reinterpret_cast<const float4*>(x + r * N + col);
    const float am = seg_allmax<TPR>(amax4(v));
    float sc, inv;
    e2m1_row_scale(am, sc, inv);
    if (r < rows) {
      *reinterpret_cast<unsigned short*>(codes + r * (N / 2) + col / 2) = static_cast<unsigned short>(quant4_e2m1(v, inv));
      if ((t % TPR) == 0) scale[r] = sc;
    }
  }
}

}  // namespace replay
