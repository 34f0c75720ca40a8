// Persistent, warp-specialised kernel for the ReplaySSM decode path on sm_100a.
//
// One launch processes every (sequence b, head h) unit of a decode layer (a unit is one
// group of up to 8192/N state rows of a head). Each CTA owns the heads blockIdx.x,
// blockIdx.x + gridDim.x, ... and streams their units through a ring of shared-memory
// stages, with three kinds of warps that hand a stage on through mbarriers:
//   * the producer warp reads each unit's buffer pointer word (prefetched 32 units at a
//     time) and fills a stage with 1-D bulk copies (TMA), one copy per lane and two
//     units per instruction: the unit's live ring records (k, v, Delta, a of every
//     buffered input and of this call's new tokens) and its queries, completing on the
//     stage's "rfull" barrier, and the unit's checkpoint tile (FP32 master rows, or FP8
//     codes + per-row scales), completing on "tfull";
//   * kCoefWarps coefficient warps take alternate units as soon as their records land
//     (long before the tile): the decay weights and k_j . q_s products, and from them
//     the whole buffer term u_s[p] = sum_j w_{s,j} (k_j . q_s) v_j[p] of every row and
//     position, the output decays alpha_s and, for a fold, the fold weights and the
//     table sig_j v_j[p]; they write these into the stage and arrive on "cready";
//   * kRowWarps row warps take every unit, each its own rows, independently of one
//     another: the state rows' dot products with the queries and y = alpha (S q) + u,
//     or the fold (rank-c update in registers), its write-back and the outputs from the
//     fresh rows; they release the stage through "empty".
// The row warps' work per unit is only what the state tile itself needs, and no barrier
// other than the stage's own ties them to the coefficient work, so the state streams at
// the memory's pace while the coefficient chains of later units run meanwhile.
// The state is streamed exactly once per call; every other byte is small.
//
// What a unit computes (blog "ReplaySSM: Cachear Inputs, No Estado": routes "estado y
// salida" and "solo salida"; arXiv 2610.13778 abstract):
//   REPLAY (step / verify over n_pos positions): if the buffer cannot take n_pos more
//     entries, fold it first, S0 <- abar S0 + sum_j s_j v_j k_j^T, writing the master
//     (and the FP8 copy) once; then for each position s
//       y_s = alpha_s (S q_s) + sum_{j <= c+s} w_{s,j} (k_j . q_s) v_j
//     where S is the fresh fold (in registers) or the stored checkpoint.
//   FLUSH: fold the buffer of the selected sequences, no output.
//   EAGER (baseline): S <- a S + Delta v k^T, y = S q, the state read and written every
//     call (FP32, or a shared FP8 state re-quantised every call).
//
// Row layout of a unit: a state row of N floats is covered by TPR = N/4 lanes, four
// columns each; a warp covers 32/TPR rows per pass and kRowsPerThread contiguous rows
// per lane.
#pragma once

#include "replay_device.cuh"
#include "replay_kparams.h"

namespace replay {

__device__ __forceinline__ void report_error(int32_t* status, int32_t bits) {
  if (status) atomicOr(status, bits);
}

// A row warp's release of a stage, counted (after the warp's reads of the stage, which
// __syncwarp orders before lane 0's fence).
__device__ __forceinline__ void count_release(int* released, int lane) {
  __syncwarp();
  if (lane == 0) {
    __threadfence_block();
    atomicAdd(released, 1);
  }
}
// Waits (bounded, about two seconds) until at least `target` row-warp releases of a stage
// have been counted; the whole warp returns the outcome.
__device__ __forceinline__ bool wait_released(const int* released, int target, int lane) {
  bool ok = true;
  if (lane == 0) {
    const volatile int* r = released;
    if (*r < target) {
      const long long t0 = clock64();
      while (*r < target) {
        if (clock64() - t0 > kWaitLimitCycles) {
          ok = false;
          break;
        }
        __nanosleep(64);
      }
    }
    __threadfence_block();
  }
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// barriers at the start of shared memory
struct Bars {
  uint64_t tfull[kMaxTileStages];   // the unit's state tile (and read-copy scales) landed
  uint64_t tempty[kMaxTileStages];  // every row warp is done with the tile stage
  uint64_t rfull[kMaxRecStages];    // the unit's records and queries landed, pointer word written
  uint64_t cready[kMaxRecStages];   // its coefficients and buffer terms are in the record stage
  uint64_t rempty[kMaxRecStages];   // every row warp is done with the record stage
  int abort_flag;
  int last_tfill[kMaxTileStages];   // CTA-local index of the latest unit copied into each stage
  int last_rfill[kMaxRecStages];
  int released[kMaxRecStages];      // row-warp releases of each record stage so far (kRowWarps per use)
};
static_assert(sizeof(Bars) <= kHeaderBytes, "the barrier header must fit the bytes the host layout reserves");

struct Plan {
  int b, h, g, rb, r0, rows, start, c;  // rows r0 .. r0 + rows - 1 of head h of sequence b
  bool fold, corrupt, active, fp32_tile;
  uint32_t tile_bytes, rec_bytes;       // bulk-copied bytes completing on tfull / rfull
};

// This CTA's units, in the order every role takes them: chunks of chunk_heads consecutive
// heads of one k/q group (the group, or a part of it, so that its heads share one
// coefficient warp and its k . q products), chunk c on CTA c mod gridDim.x, each head
// with its row blocks in a row. Dealing the chunks round-robin keeps the 148 CTAs on
// neighbouring tiles of the state at any moment, and one CTA holds every unit of a head
// (the in-kernel append writes a head's new record once, before any copy of it).
__device__ __forceinline__ int cta_chunks(const KParams& p) {
  return (p.num_chunks - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
}
__device__ __forceinline__ int cta_units(const KParams& p) { return (cta_chunks(p) * p.chunk_heads) << p.rb_shift; }
// the CTA's i-th head (chunk i / chunk_heads, head i mod chunk_heads within it)
__device__ __forceinline__ int cta_head(const KParams& p, int hi) {
  const int ck = hi / p.chunk_heads;
  return ((int)blockIdx.x + ck * (int)gridDim.x) * p.chunk_heads + (hi - ck * p.chunk_heads);
}
__device__ __forceinline__ int cta_unit(const KParams& p, int i) {
  return (cta_head(p, i >> p.rb_shift) << p.rb_shift) | (i & (p.row_blocks - 1));
}
// the CTA-local chunk of unit i
__device__ __forceinline__ int unit_chunk(const KParams& p, int i) { return (i >> p.rb_shift) / p.chunk_heads; }

template <int MODE, int CKPT, int S_IO>
__device__ __forceinline__ Plan make_plan(const KParams& p, int u, int32_t word, int msk) {
  Plan pl;
  const int bh = u >> p.rb_shift;
  pl.rb = u & (p.row_blocks - 1);
  pl.b = bh / p.H;
  pl.h = bh - pl.b * p.H;
  pl.g = pl.h / p.hpg;
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
    pl.tile_bytes = pl.fp32_tile ? P * N * 4u : P * (N / kCodeDiv) + P * 4u;
    pl.rec_bytes = 0;  // gathered with cp.async, counted as arrivals
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
    pl.tile_bytes = 0;
    pl.rec_bytes = 0;
    return pl;
  }
  const uint32_t records = pl.c + ((MODE == kModeReplay) ? p.n_pos : 0);
  pl.tile_bytes = pl.fp32_tile ? P * N * 4u : P * (N / kCodeDiv) + P * 4u;
  pl.rec_bytes = records * (uint32_t)(p.rec_bytes + p.rec_k_bytes) + ((MODE == kModeReplay) ? p.n_pos * N * S_IO : 0u);
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

// ---------------------------------------------------------------------------- append
// This CTA's units' new entries (one position) into their ring records, slot
// (start + c) mod cap, by the worker threads before any bulk copy is issued: each head's
// v, then Delta and a in one 16-byte piece, and the group's k once per chunk (a group of
// more than kMaxChunkHeads heads spans chunks, possibly on several CTAs, each writing the
// same bytes before it reads them). The input pieces do not depend on the pointer word,
// so both reads are in flight together.
template <int S_IO>
__device__ __forceinline__ void append_entries(const KParams& p) {
  constexpr int kPool = kWorkerWarps * 32;
  constexpr int kBatch = 8;  // pieces per thread in flight
  const int kpe = p.N * S_IO / 16;  // 16-byte pieces of k
  const int vpe = p.P * S_IO / 16;  // of v
  const int per_unit = kpe + vpe + 1;
  const int total = cta_chunks(p) * p.chunk_heads * per_unit;
  for (int t0 = threadIdx.x; t0 < total; t0 += kBatch * kPool) {
    uint4 val[kBatch];
    uint8_t* dst[kBatch];
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      const int t = t0 + r * kPool;
      dst[r] = nullptr;
      val[r] = make_uint4(0u, 0u, 0u, 0u);
      if (t < total) {
        const int iu = t / per_unit;
        const int ch = t - iu * per_unit;
        const int bh = cta_head(p, iu);
        const int b = bh / p.H;
        const int h = bh - b * p.H;
        const int g = h / p.hpg;
        const bool k_here = (iu % p.chunk_heads) == 0;  // the chunk's first head writes the group's k
        const int32_t word = __ldg(p.counts_in + b);
        if (ch < kpe) {
          if (k_here)
            val[r] = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.k) + ((size_t)b * p.G + g) * p.N * S_IO)[ch];
        } else if (ch < kpe + vpe) {
          val[r] = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.v) + ((size_t)b * p.H + h) * p.P * S_IO)[ch - kpe];
        } else {
          val[r].x = __float_as_uint(__ldg(p.dt + (size_t)b * p.H + h));
          val[r].y = __float_as_uint(__ldg(p.a + (size_t)b * p.H + h));
        }
        const int start = word >> 16;
        const int c = word & 0xFFFF;
        if (!(word < 0 || c > p.L || start >= p.cap) && (ch >= kpe || k_here)) {  // a bad word is reported by the consumers
          int slot = start + c;
          slot -= (slot >= p.cap) ? p.cap : 0;
          dst[r] = ch < kpe ? static_cast<uint8_t*>(p.ring_k) + (((size_t)b * p.G + g) * p.cap + slot) * p.rec_k_bytes + (size_t)ch * 16
                            : static_cast<uint8_t*>(p.ring) + (((size_t)b * p.H + h) * p.cap + slot) * p.rec_bytes + (size_t)(ch - kpe) * 16;
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kBatch; ++r)
      if (dst[r]) *reinterpret_cast<uint4*>(dst[r]) = val[r];
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// ---------------------------------------------------------------------------- producer
// Copies of one unit, one bulk copy (TMA) per kind: 0 the state tile (the unit's rows)
// and 1 their read-copy row scales, into its tile stage `tst`, completing on tfull; into
// its record stage `rst`: 2-3 the live head records and
// 4-5 the live k records of the head's group, [start, start + count) modulo cap in one
// or two pieces (whole records: every row block reads all of k and its rows of v), and
// 6 the queries, completing on rfull. Returns the bytes of copy `kind` (0 if none) and
// its addresses.
constexpr int kCopyKinds = 7;
template <int MODE, int CKPT, int S_IO>
__device__ __forceinline__ uint32_t unit_copy(const KParams& p, const Plan& pl, uint8_t* tst, uint8_t* rst, int kind,
                                              const uint8_t*& src, uint8_t*& dst) {
  constexpr size_t kCodeDiv = (CKPT == kCkptFp4) ? 2 : 1;
  const size_t P = pl.rows, N = p.N;
  const size_t bh = (size_t)pl.b * p.H + pl.h;
  const size_t bg = (size_t)pl.b * p.G + pl.g;
  const size_t row0 = bh * p.P + pl.r0;  // the unit's first state row
  const int R = p.rec_bytes;
  const int RK = p.rec_k_bytes;
  const int cnt = pl.c + ((MODE == kModeReplay) ? p.n_pos : 0);
  const int first = min(cnt, p.cap - pl.start);
  const uint8_t* ring = static_cast<const uint8_t*>(p.ring) + bh * p.cap * R;
  const uint8_t* ring_k = static_cast<const uint8_t*>(p.ring_k) + bg * p.cap * RK;
  const uint8_t* qsrc = p.qpack ? static_cast<const uint8_t*>(p.qpack) + bg * p.qpack_pos * N * S_IO
                                : static_cast<const uint8_t*>(p.q) + bg * N * S_IO;
  const uint8_t* tsrc = pl.fp32_tile ? reinterpret_cast<const uint8_t*>(p.S + row0 * N) : p.S8 + row0 * (N / kCodeDiv);
  src = (kind == 0)   ? tsrc
        : (kind == 1) ? reinterpret_cast<const uint8_t*>(p.Sscale + row0)
        : (kind == 2) ? ring + (size_t)pl.start * R
        : (kind == 3) ? ring
        : (kind == 4) ? ring_k + (size_t)pl.start * RK
        : (kind == 5) ? ring_k
                      : qsrc;
  dst = (kind == 0)   ? tst
        : (kind == 1) ? tst + (size_t)p.rows_unit * (N / kCodeDiv)  // the scales follow a full unit's codes
        : (kind == 2) ? rst + p.off_rec
        : (kind == 3) ? rst + p.off_rec + (size_t)first * R
        : (kind == 4) ? rst + p.off_krec
        : (kind == 5) ? rst + p.off_krec + (size_t)first * RK
                      : rst + p.off_q;
  uint32_t bytes = 0;
  bytes = (kind == 0) ? (pl.fp32_tile ? (uint32_t)(P * N * 4) : (uint32_t)(P * (N / kCodeDiv))) : bytes;
  bytes = (kind == 1 && !pl.fp32_tile) ? (uint32_t)(P * 4) : bytes;
  bytes = (kind == 2) ? (uint32_t)(first * R) : bytes;
  bytes = (kind == 3) ? (uint32_t)((cnt - first) * R) : bytes;
  bytes = (kind == 4) ? (uint32_t)(first * RK) : bytes;
  bytes = (kind == 5) ? (uint32_t)((cnt - first) * RK) : bytes;
  bytes = (kind == 6 && MODE == kModeReplay) ? (uint32_t)(p.n_pos * N * S_IO) : bytes;
  return pl.active ? bytes : 0u;
}

// The producer warp. Step t copies the records (and queries) of unit t into its record
// stage and the tile of unit t - D into its tile stage, D = p.lookahead: a unit's records
// land D units before its tile, so the coefficient warps finish with them before the row
// warps reach the unit. The tiles of the first num_tstages units go out at once (when the
// kernel appends this call's entries itself, before the append is complete; their records
// after it). Steps go kUnitsPerIssue at a time: the producer waits until their stages are
// free, writes each unit's pointer word into its record stage, arms the stages' barriers
// with the byte counts and issues every copy of the batch with one predicated bulk-copy
// instruction (lane = step in batch * kCopyKinds + kind), which costs the warp about as
// much as one copy. A tile's plan takes the pointer word its record stage holds (written
// D steps before; the stage stays until the row warps are done with the unit). Waits are
// exact: the producer visits every use of every stage in order.
template <int MODE, int CKPT, int S_IO, bool APPEND>
__device__ void producer_loop(const KParams& p, uint8_t* tstages, uint8_t* rstages, Bars* bars) {
  constexpr int U = kUnitsPerIssue;
  static_assert(U * kCopyKinds <= 32 && (32 % U) == 0, "a batch's copies must fit one warp and tile 32 units");
  const int lane = threadIdx.x & 31;
  const int NT = p.num_tstages, NR = p.num_rstages, D = p.lookahead;
  const uint64_t stream_policy = l2_evict_first_policy();
  const uint64_t keep_policy = l2_evict_normal_policy();
  const int total = cta_units(p);
  auto unit_of = [&](int i) { return cta_unit(p, i); };
  auto tst_of = [&](int i) { return tstages + (size_t)(i % NT) * p.tstage_bytes; };
  auto rst_of = [&](int i) { return rstages + (size_t)(i % NR) * p.rstage_bytes; };
  // pointer words (and flush masks) of the record units, 32 at a time, one chunk ahead:
  // lane j of a chunk holds the word of the chunk's j-th unit
  auto load_words = [&](int i0, int32_t& w, int& msk) {
    w = 0;
    msk = 1;
    if (i0 + lane < total) {
      const int b = (unit_of(i0 + lane) >> p.rb_shift) / p.H;
      w = __ldg(p.counts_in + b);
      if (MODE == kModeFlush && p.mask) msk = __ldg(p.mask + b);
    }
  };
  int32_t w_cur, w_nxt;
  int m_cur, m_nxt;
  load_words(0, w_cur, m_cur);
  load_words(32, w_nxt, m_nxt);
  const int j = lane / kCopyKinds;     // this lane's step within the batch
  const int kind = lane % kCopyKinds;  // and its copy
  const int pre = min(NT, total);      // tiles issued up front
  for (int i = 0; i < pre; ++i) {
    const Plan pl = make_plan<MODE, CKPT, S_IO>(p, unit_of(i), __shfl_sync(0xffffffffu, w_cur, i),
                                               __shfl_sync(0xffffffffu, m_cur, i));
    if (lane == 0) mbar_arrive_expect_tx(&bars->tfull[i], pl.tile_bytes);
    __syncwarp();
    const uint8_t* src;
    uint8_t* dst;
    uint32_t bytes = unit_copy<MODE, CKPT, S_IO>(p, pl, tst_of(i), rst_of(i), lane, src, dst);
    if (lane > 1) bytes = 0;
    __syncwarp();
    if (bytes) bulk_g2s_hint(dst, src, bytes, &bars->tfull[i], lane == 0 ? stream_policy : keep_policy);
    if (lane == 0) bars->last_tfill[i] = i;
  }
  if (APPEND && p.append_here) group_sync(kAppendBar, kThreads);  // the entries are in the ring
  for (int t0 = 0; t0 < total + D; t0 += U) {
    if ((t0 & 31) == 0 && t0 > 0) {
      w_cur = w_nxt;
      m_cur = m_nxt;
      load_words(t0 + 32, w_nxt, m_nxt);
    }
    // every lane waits for the batch's stages, the warp agrees
    bool ready = true;
#pragma unroll
    for (int jj = 0; jj < U; ++jj) {
      const int r = t0 + jj;      // record unit
      const int u = t0 + jj - D;  // tile unit
      if (r < total && r >= NR) ready = ready && mbar_wait_bounded(&bars->rempty[r % NR], ((r / NR) - 1) & 1);
      if (u >= pre && u < total && u >= NT) ready = ready && mbar_wait_bounded(&bars->tempty[u % NT], ((u / NT) - 1) & 1);
    }
    if (!__all_sync(0xffffffffu, ready)) {
      if (lane == 0) {
        report_error(p.status, kErrWaitTimeout);
        bars->abort_flag = 1;
      }
      break;
    }
    const int ab = (lane == 0) ? *reinterpret_cast<volatile int*>(&bars->abort_flag) : 0;
    if (__shfl_sync(0xffffffffu, ab, 0)) break;  // the warp decides together
    const int r = t0 + j;
    const int u = t0 + j - D;
    const bool rec_step = j < U && r < total;
    const bool tile_step = j < U && u >= pre && u < total;
    // record side: the unit's pointer word and flush mask from the prefetched chunk
    const int32_t word_r = __shfl_sync(0xffffffffu, w_cur, r & 31);
    const int msk_r = __shfl_sync(0xffffffffu, m_cur, r & 31);
    uint8_t* rst = rst_of(r);
    const Plan plr = make_plan<MODE, CKPT, S_IO>(p, unit_of(r), word_r, msk_r);
    if (rec_step && kind == 2) {
      reinterpret_cast<int32_t*>(rst + p.off_meta)[0] = word_r;
      reinterpret_cast<int32_t*>(rst + p.off_meta)[1] = msk_r;
      if (plr.corrupt) report_error(p.status, kErrPointer);
      mbar_arrive_expect_tx(&bars->rfull[r % NR], plr.rec_bytes);
    }
    __syncwarp();  // a record stage armed in this step may hold a tile unit's word (lookahead < batch)
    // tile side: the pointer word from the unit's record stage
    int32_t word_u = 0;
    int msk_u = 1;
    if (tile_step && kind <= 1) {
      const uint8_t* rsu = rst_of(u);
      word_u = reinterpret_cast<const int32_t*>(rsu + p.off_meta)[0];
      msk_u = reinterpret_cast<const int32_t*>(rsu + p.off_meta)[1];
    }
    uint8_t* tst = tst_of(u < 0 ? 0 : u);
    const Plan plt = make_plan<MODE, CKPT, S_IO>(p, unit_of(u < 0 ? 0 : u), word_u, msk_u);
    if (tile_step && kind == 0) mbar_arrive_expect_tx(&bars->tfull[u % NT], plt.tile_bytes);
    __syncwarp();
    const uint8_t* src;
    uint8_t* dst;
    uint32_t bytes = 0;
    if (kind <= 1) {
      bytes = unit_copy<MODE, CKPT, S_IO>(p, plt, tst, rst, kind, src, dst);
      if (!tile_step) bytes = 0;
    } else {
      bytes = unit_copy<MODE, CKPT, S_IO>(p, plr, tst, rst, kind, src, dst);
      if (!rec_step) bytes = 0;
    }
    __syncwarp();
    if (bytes)
      bulk_g2s_hint(dst, src, bytes, kind <= 1 ? &bars->tfull[u % NT] : &bars->rfull[r % NR],
                    kind == 0 ? stream_policy : keep_policy);
    if (tile_step && kind == 0) bars->last_tfill[u % NT] = u;
    if (rec_step && kind == 2) bars->last_rfill[r % NR] = r;
  }
  // Never leave with copies in flight into this CTA's shared memory: wait (bounded) for
  // the latest fill of every stage.
  __syncwarp();
  bool ok = true;
  for (int st_i = 0; st_i < NT; ++st_i) {
    const int i = bars->last_tfill[st_i];
    if (i >= 0) ok = mbar_wait_bounded(&bars->tfull[st_i], (i / NT) & 1) && ok;
  }
  for (int st_i = 0; st_i < NR; ++st_i) {
    const int i = bars->last_rfill[st_i];
    if (i >= 0) ok = mbar_wait_bounded(&bars->rfull[st_i], (i / NR) & 1) && ok;
  }
  if (!ok && lane == 0) report_error(p.status, kErrWaitTimeout);
}

// The eager baseline's producer: one unit at a time, no lookahead (its coefficients are
// two numbers); the tile (and FP8 scales) by bulk copy on tfull, the new token's k, v,
// Delta, a and q gathered with per-lane cp.async into the record stage, each lane arriving
// on rfull once its copies have landed.
template <int CKPT, int S_IO>
__device__ void producer_loop_eager(const KParams& p, uint8_t* tstages, uint8_t* rstages, Bars* bars) {
  const int lane = threadIdx.x & 31;
  const int NT = p.num_tstages, NR = p.num_rstages;
  const uint64_t stream_policy = l2_evict_first_policy();
  const size_t P = p.P, N = p.N;
  const int total = cta_units(p);
  for (int i = 0; i < total; ++i) {
    const int u = cta_unit(p, i);
    bool ready = true;
    if (i >= NT) ready = mbar_wait_bounded(&bars->tempty[i % NT], ((i / NT) - 1) & 1);
    if (ready && i >= NR) ready = mbar_wait_bounded(&bars->rempty[i % NR], ((i / NR) - 1) & 1);
    if (!__all_sync(0xffffffffu, ready)) {
      if (lane == 0) {
        report_error(p.status, kErrWaitTimeout);
        bars->abort_flag = 1;
      }
      break;
    }
    const int ab = (lane == 0) ? *reinterpret_cast<volatile int*>(&bars->abort_flag) : 0;
    if (__shfl_sync(0xffffffffu, ab, 0)) break;
    const Plan pl = make_plan<kModeEager, CKPT, S_IO>(p, u, 0, 1);
    uint8_t* tst = tstages + (size_t)(i % NT) * p.tstage_bytes;
    uint8_t* rst = rstages + (size_t)(i % NR) * p.rstage_bytes;
    const size_t bh = (size_t)pl.b * p.H + pl.h;
    const size_t bg = (size_t)pl.b * p.G + pl.g;
    const size_t row0 = bh * P + pl.r0;  // the unit's rows
    const uint32_t rows = (uint32_t)pl.rows;
    constexpr size_t kCodeDiv = (CKPT == kCkptFp4) ? 2 : 1;
    uint8_t* recbuf = rst + p.off_rec;
    uint8_t* kbuf = rst + p.off_krec;
    if (lane == 0) mbar_arrive_expect_tx(&bars->tfull[i % NT], pl.tile_bytes);
    __syncwarp();
    if (lane == 0)
      bulk_g2s_hint(tst, pl.fp32_tile ? (const void*)(p.S + row0 * N) : (const void*)(p.S8 + row0 * (N / kCodeDiv)),
                    pl.fp32_tile ? (uint32_t)(rows * N * 4) : (uint32_t)(rows * (N / kCodeDiv)), &bars->tfull[i % NT],
                    stream_policy);
    if (lane == 1 && !pl.fp32_tile)
      bulk_g2s(tst + (size_t)p.rows_unit * (N / kCodeDiv), p.Sscale + row0, rows * 4u, &bars->tfull[i % NT]);
    const int kpe = (int)(N * S_IO / 16);
    const int vpe = (int)(P * S_IO / 16);
    for (int idx = lane; idx < 2 * kpe + vpe; idx += 32) {
      if (idx < kpe) {
        cp_async16(rst + p.off_q + idx * 16, static_cast<const uint8_t*>(p.q) + bg * N * S_IO + idx * 16);
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
    cp_async_arrive(&bars->rfull[i % NR]);
    if (lane == 0) {
      bars->last_tfill[i % NT] = i;
      bars->last_rfill[i % NR] = i;
    }
  }
  __syncwarp();
  bool ok = true;
  for (int st_i = 0; st_i < NT; ++st_i) {
    const int i2 = bars->last_tfill[st_i];
    if (i2 >= 0) ok = mbar_wait_bounded(&bars->tfull[st_i], (i2 / NT) & 1) && ok;
  }
  for (int st_i = 0; st_i < NR; ++st_i) {
    const int i2 = bars->last_rfill[st_i];
    if (i2 >= 0) ok = mbar_wait_bounded(&bars->rfull[st_i], (i2 / NR) & 1) && ok;
  }
  if (!ok && lane == 0) report_error(p.status, kErrWaitTimeout);
}

// ---------------------------------------------------------------------------- coefficients
// What a coefficient warp forms for a unit, from its records in shared memory (all 32
// lanes; the results go into the stage's coefficient area for the row warps):
//  * fold weights when the unit folds (blog "Ruta 'estado y salida'"): sig_j = Delta_j
//    prod_{j<i<c} a_i and abar = prod_{i<c} a_i (the eager baseline: its single entry,
//    sig_0 = Delta, abar = a), and the table wt[j][p] = sig_j v_j[p] of the unit's rows;
//  * for every position s the outputs replay the entries o0 .. c+s, o0 = c after a fold
//    and 0 otherwise (blog "Ruta 'solo salida'"):
//        alpha_s = prod_{o0<=i<=c+s} a_i,   w_{s,j} = Delta_j prod_{j<i<=c+s} a_i,
//        u_s[p]  = sum_{o0<=j<=c+s} w_{s,j} (k_j . q_s) v_j[p],
//    so that the row warps only add y_s = alpha_s (S q_s) + u_s. The products of decay
//    factors are suffix products over the window.
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

// k_l . q_s of the window entries l < width (entry o0 + l) for the positions s < n, into
// kq[s][l]: four lanes per entry (a quarter row each, one shuffle pair to combine), eight
// entries per pass. The products belong to the k/q group, so a coefficient warp forms
// them once for all the group's heads and row blocks.
template <int N, typename IO>
__device__ __forceinline__ void window_kq(const Records<N, IoT<IO>::bytes>& rec, const uint8_t* qbuf, int o0,
                                          int width, int n, float* kq, int lane) {
  constexpr int S_IO = IoT<IO>::bytes;
  constexpr int QN = N / 4;  // elements of a quarter row
  const int quarter = lane & 3;
  for (int l0 = 0; l0 < width; l0 += 8) {
    const int l = l0 + (lane >> 2);
    const uint8_t* kp = rec.k(o0 + (l < width ? l : 0)) + (size_t)quarter * QN * S_IO;
    float4 kr[QN / 4];  // the lane's quarter of k_l, read once for every position
#pragma unroll
    for (int e = 0; e < QN / 4; ++e) kr[e] = IoT<IO>::load4(kp + (size_t)e * 4 * S_IO);
    for (int s = 0; s < n; ++s) {
      const uint8_t* qq = qbuf + ((size_t)s * N + quarter * QN) * S_IO;
      float d0 = 0.f, d1 = 0.f;
#pragma unroll
      for (int e = 0; e < QN / 4; e += 2) {
        d0 += dot4(kr[e], IoT<IO>::load4(qq + (size_t)e * 4 * S_IO));
        if (e + 1 < QN / 4) d1 += dot4(kr[e + 1], IoT<IO>::load4(qq + (size_t)(e + 1) * 4 * S_IO));
      }
      float d = d0 + d1;
      d += __shfl_xor_sync(0xffffffffu, d, 1);
      d += __shfl_xor_sync(0xffffffffu, d, 2);
      if (quarter == 0 && l < width) kq[s * kMaxWindow + l] = d;
    }
  }
}

// The output coefficients of one head from its decay factors and the group's k . q: for
// every position s, alpha_s = prod_{l<=last_s} a_{o0+l} and cw[s][l] = w_{s,l} kq[s][l]
// with w_{s,l} = Delta_{o0+l} prod_{l<i<=last_s} a_{o0+i}, zero past last_s (all 32 lanes
// written, so that the buffer terms may read whole vectors); a lane per entry and a
// suffix-product scan across the lanes per position.
template <int N, typename IO>
__device__ __forceinline__ void output_weights(const Records<N, IoT<IO>::bytes>& rec, int c, int n, int o0,
                                               const float* kq, float* alpha, float* cw, int lane) {
  const int width = c + n - o0;  // window entries (at most kMaxWindow)
  float xa = 1.f, xd = 0.f;
  if (lane < width) {
    xa = rec.a(o0 + lane);
    xd = rec.dt(o0 + lane);
  }
  for (int s = 0; s < n; ++s) {
    const int last = c + s - o0;  // position s replays window entries 0 .. last
    const float incl = warp_suffix_prod(lane <= last ? xa : 1.f, lane);  // prod_{lane<=i<=last} a_i
    float excl = __shfl_down_sync(0xffffffffu, incl, 1);
    if (lane == 31) excl = 1.f;
    if (lane == 0) alpha[s] = incl;
    cw[s * kMaxWindow + lane] = (lane <= last) ? xd * excl * kq[s * kMaxWindow + lane] : 0.f;
  }
}


template <int N, typename IO, int CKPT, int MODE, int NQ>
__device__ __forceinline__ void coef_unit(const KParams& p, const Plan& pl, uint8_t* st, float* kq, float* cw,
                                          bool kq_ready, int lane) {
  constexpr int S_IO = IoT<IO>::bytes;
  constexpr int NQR = NQ > 0 ? NQ : 1;
  const Records<N, S_IO> rec{st + p.off_krec, st + p.off_rec, p.P, p.rec_bytes, p.rec_k_bytes};
  uint8_t* co = st + p.off_coef;
  float* alpha = reinterpret_cast<float*>(co + p.co_alpha);  // [kMaxPos]
  float* sig = reinterpret_cast<float*>(co + p.co_sig);      // fold weights; [kMaxWindow] = abar
  float* u = reinterpret_cast<float*>(co + p.co_u);          // [n][u_stride] buffer terms
  float* wt = reinterpret_cast<float*>(co + p.co_wt);        // [cf][wt_stride] fold weights times v
  const int c = pl.c;
  const int n = (MODE == kModeReplay) ? p.n_pos : 0;
  const int cf = (MODE == kModeEager) ? 1 : (pl.fold ? c : 0);  // entries folded into the state
  const int o0 = pl.fold ? c : 0;                                // first entry the outputs replay
  const int rows = pl.rows;
  const int r0 = pl.r0;
  const int wts = p.wt_stride;
  if (cf > 0) {
    fold_weights<N, IO, MODE>(rec, c, sig, lane);
    __syncwarp();
    // wt[j][p] = sig_j v_j[r0 + p], zero for the rows past the unit's (the row warps read
    // whole vectors)
    for (int j = 0; j < cf; ++j) {
      const float sj = sig[j];
      const uint8_t* vj = rec.v(j) + (size_t)r0 * S_IO;
      for (int pp = lane; pp < wts; pp += 32)
        wt[(size_t)j * wts + pp] = pp < rows ? sj * IoT<IO>::load1(vj + (size_t)pp * S_IO) : 0.f;
    }
  }
  if (MODE == kModeReplay) {
    const int width = c + n - o0;
    if (!kq_ready) {
      window_kq<N, IO>(rec, st + p.off_q, o0, width, n, kq, lane);
      __syncwarp();
    }
    output_weights<N, IO>(rec, c, n, o0, kq, alpha, cw, lane);
    __syncwarp();
    // u_s[p] = sum_l cw[s][l] v_{o0+l}[r0 + p]: two rows per lane at a time (p and p + 32),
    // each v read once for every position, eight entries in flight per row (cw is zero
    // past each position's window)
    for (int pr0 = lane; pr0 < rows; pr0 += 64) {
      const int pr1 = pr0 + 32 < rows ? pr0 + 32 : pr0;  // the second row, or the first again
      const uint8_t* vrow0 = rec.base + (size_t)(r0 + pr0) * S_IO;
      const uint8_t* vrow1 = rec.base + (size_t)(r0 + pr1) * S_IO;
      float acc0[NQR], acc1[NQR];
#pragma unroll
      for (int s = 0; s < NQR; ++s) acc0[s] = acc1[s] = 0.f;
      for (int l0 = 0; l0 < width; l0 += 8) {
        float v0[8], v1[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const size_t off = (size_t)(o0 + (l0 + r < width ? l0 + r : 0)) * rec.R;
          v0[r] = (l0 + r < width) ? IoT<IO>::load1(vrow0 + off) : 0.f;
          v1[r] = (l0 + r < width) ? IoT<IO>::load1(vrow1 + off) : 0.f;
        }
#pragma unroll
        for (int s = 0; s < NQR; ++s) {
          if (s < n) {
            const float4 ca = *reinterpret_cast<const float4*>(cw + s * kMaxWindow + l0);
            const float4 cb = *reinterpret_cast<const float4*>(cw + s * kMaxWindow + l0 + 4);
            acc0[s] = fmaf(ca.x, v0[0], fmaf(ca.y, v0[1], fmaf(ca.z, v0[2], fmaf(ca.w, v0[3],
                      fmaf(cb.x, v0[4], fmaf(cb.y, v0[5], fmaf(cb.z, v0[6], fmaf(cb.w, v0[7], acc0[s]))))))));
            acc1[s] = fmaf(ca.x, v1[0], fmaf(ca.y, v1[1], fmaf(ca.z, v1[2], fmaf(ca.w, v1[3],
                      fmaf(cb.x, v1[4], fmaf(cb.y, v1[5], fmaf(cb.z, v1[6], fmaf(cb.w, v1[7], acc1[s]))))))));
          }
        }
      }
#pragma unroll
      for (int s = 0; s < NQR; ++s) {
        if (s < n) {
          u[s * p.u_stride + pr0] = acc0[s];
          if (pr0 + 32 < rows) u[s * p.u_stride + pr0 + 32] = acc1[s];
        }
      }
    }
  }
}

// The coefficient warps' loop, on the record ring: the units of a chunk (heads of one k/q
// group, each with its row blocks) all go to one warp, chunks in turn, so that the warp
// forms the group's k . q once per chunk. A warp's consecutive units may lie any distance
// apart, so its parity waits are made exact by counting: before it waits for the k-th use
// of a record stage it waits until the row warps' releases of that stage's use k-2 have
// all been counted (the row warps take the units in order and cannot be two uses further
// on, since they need this warp's coefficients for use k). Then it waits for the stage's
// previous release (rempty, phase k-1), after which no one else touches the stage, and
// for its records (rfull, phase k), whose phase k-1 completed before the row warps could
// release use k-1. Each warp takes its units in order, so no wait can close a cycle.
template <int N, typename IO, int CKPT, int MODE, int NQ>
__device__ void coef_loop(const KParams& p, uint8_t* rstages, Bars* bars, float* kq, float* cw, int cwarp, int lane) {
  constexpr int S_IO = IoT<IO>::bytes;
  const int NR = p.num_rstages;
  const int total = cta_units(p);
  int cached = -1;  // the CTA-local chunk whose k . q products the warp holds in kq
  for (int i = 0; i < total; ++i) {
    const int key = unit_chunk(p, i);
    if (key % kCoefWarps != cwarp) continue;
    const int s = i % NR;
    const int k = i / NR;
    bool ready = *reinterpret_cast<volatile int*>(&bars->abort_flag) == 0;
    if (ready && k > 1) ready = wait_released(&bars->released[s], (k - 1) * kRowWarps, lane);
    if (ready && k > 0) ready = mbar_wait_bounded(&bars->rempty[s], (k - 1) & 1);
    if (ready) ready = mbar_wait_bounded(&bars->rfull[s], k & 1);
    if (!__all_sync(0xffffffffu, ready)) {
      if (lane == 0) {
        report_error(p.status, kErrWaitTimeout);
        bars->abort_flag = 1;
      }
      break;
    }
    uint8_t* st = rstages + (size_t)s * p.rstage_bytes;
    const int32_t word = reinterpret_cast<const int32_t*>(st + p.off_meta)[0];
    const int msk = reinterpret_cast<const int32_t*>(st + p.off_meta)[1];
    const Plan pl = make_plan<MODE, CKPT, S_IO>(p, cta_unit(p, i), word, msk);
    if (pl.active) {
      coef_unit<N, IO, CKPT, MODE, NQ>(p, pl, st, kq, cw, cached == key, lane);
      if (MODE == kModeReplay) cached = key;
    }
    // publish the sequence's pointer word (the entries are already in the ring) and flag
    if (MODE != kModeEager && lane == 0 && pl.h == 0 && pl.rb == 0) {
      const int start = pl.start;
      const int cap = p.cap;
      if (!pl.active) {
        p.counts_out[pl.b] = word;  // nothing folded: the pointer word carries over
        if (MODE == kModeFlush && p.flushed && !pl.corrupt) p.flushed[pl.b] = 0;
      } else if (MODE == kModeReplay) {
        int start2 = pl.fold ? start + pl.c : start;
        start2 -= (start2 >= cap) ? cap : 0;
        const int cnt2 = (pl.fold ? 0 : pl.c) + (p.commit ? p.n_pos : 0);
        p.counts_out[pl.b] = (start2 << 16) | cnt2;
        if (p.flushed && (!p.flushed_or || pl.fold)) p.flushed[pl.b] = pl.fold ? 1 : 0;
      } else {
        int start2 = start + pl.c;
        start2 -= (start2 >= cap) ? cap : 0;
        p.counts_out[pl.b] = start2 << 16;
        if (p.flushed) p.flushed[pl.b] = 1;
      }
    }
    __syncwarp();
    mbar_arrive(&bars->cready[s]);
  }
}

// ---------------------------------------------------------------------------- rows
// One unit's rows by one row warp (rows rbase .. rbase + kRowsPerThread - 1 of the unit
// per lane, four columns each). Output-only: y_s = alpha_s (S q_s) + u_s. Fold: x <- abar
// x + sum_j wt[j][rows] k_j[cols] in registers, the write-back (FP32 master and/or FP8
// codes with per-row scales), then the outputs from the fresh rows.
template <int N, typename IO, int CKPT, int MODE, int NQ>
__device__ __forceinline__ void row_unit(const KParams& p, const Plan& pl, const uint8_t* tst, const uint8_t* st, int warp,
                                         int lane) {
  constexpr int S_IO = IoT<IO>::bytes;
  constexpr int TPR = N / 4;
  constexpr int RPW = 32 / TPR;  // rows per warp pass
  constexpr int RT = kRowsPerThread;
  constexpr int NQR = NQ > 0 ? NQ : 1;
  using Red = SegReduce<RT, TPR>;
  const int rbase = (warp * RPW + lane / TPR) * RT;
  const int col = (lane % TPR) * 4;
  const int P = pl.rows;  // the unit's rows: r0 .. r0 + P - 1 of the head's PH
  const int PH = p.P;
  const int r0 = pl.r0;
  const int n = (MODE == kModeReplay) ? p.n_pos : (MODE == kModeEager ? 1 : 0);
  const int cf = (MODE == kModeEager) ? 1 : (pl.fold ? pl.c : 0);
  const uint8_t* tile = tst;  // the tile stage; records, queries and coefficients in the record stage `st`
  const uint8_t* qbuf = st + p.off_q;
  constexpr int kCodeDiv = (CKPT == kCkptFp4) ? 2 : 1;  // read copy: code bytes per row = N / kCodeDiv
  const Records<N, S_IO> rec{st + p.off_krec, st + p.off_rec, PH, p.rec_bytes, p.rec_k_bytes};
  const float* scale_tile = reinterpret_cast<const float*>(tile + (size_t)p.rows_unit * (N / kCodeDiv));
  const uint8_t* co = st + p.off_coef;
  const float* alpha = reinterpret_cast<const float*>(co + p.co_alpha);
  const float* sig = reinterpret_cast<const float*>(co + p.co_sig);
  const float* u = reinterpret_cast<const float*>(co + p.co_u);
  const float* wt = reinterpret_cast<const float*>(co + p.co_wt);
  const size_t bh = (size_t)pl.b * p.H + pl.h;
  const bool fold = pl.fold;

  float4 x[RT];
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    const int pr = rbase + r;
    x[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (pr < P) {
      if (pl.fp32_tile) {
        x[r] = *reinterpret_cast<const float4*>(tile + ((size_t)pr * N + col) * 4);
      } else {
        const float4 e =
            (CKPT == kCkptFp4)
                ? e2m1x4_to_float4(*reinterpret_cast<const unsigned short*>(tile + (size_t)pr * (N / 2) + col / 2))
                : e4m3x4_to_float4(*reinterpret_cast<const uint32_t*>(tile + (size_t)pr * N + col));
        if (MODE == kModeEager) {  // a shared FP8 state: dequantise
          const float sc = scale_tile[pr];
          x[r] = make_float4(e.x * sc, e.y * sc, e.z * sc, e.w * sc);
        } else {  // the read copy: the row scale multiplies the dot product
          x[r] = e;
        }
      }
    }
  }

  if (fold) {
    // ---- fold (state route) and write-back
    const float abar = sig[kMaxWindow];
#pragma unroll
    for (int r = 0; r < RT; ++r) x[r] = make_float4(abar * x[r].x, abar * x[r].y, abar * x[r].z, abar * x[r].w);
    // rank-cf update: per entry, k_j's four columns and the weights of the thread's RT
    // rows (two 16-byte reads), then 4 RT FMAs; the next entry is read ahead
    const int wb = rbase < p.wt_stride ? rbase : 0;
    float4 kt = IoT<IO>::load4(rec.k(0) + col * S_IO);
    float4 w0 = *reinterpret_cast<const float4*>(wt + wb);
    float4 w1 = *reinterpret_cast<const float4*>(wt + wb + 4);
    for (int jj = 0; jj < cf; ++jj) {
      const int jn = min(jj + 1, cf - 1);
      const float4 kn = IoT<IO>::load4(rec.k(jn) + col * S_IO);
      const float4 n0 = *reinterpret_cast<const float4*>(wt + (size_t)jn * p.wt_stride + wb);
      const float4 n1 = *reinterpret_cast<const float4*>(wt + (size_t)jn * p.wt_stride + wb + 4);
      const float ws8[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        x[r].x = fmaf(ws8[r], kt.x, x[r].x);
        x[r].y = fmaf(ws8[r], kt.y, x[r].y);
        x[r].z = fmaf(ws8[r], kt.z, x[r].z);
        x[r].w = fmaf(ws8[r], kt.w, x[r].w);
      }
      kt = kn;
      w0 = n0;
      w1 = n1;
    }
    const bool store_f32 = (MODE != kModeEager) || (CKPT == kCkptF32);
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const int pr = rbase + r;
      const size_t row = bh * PH + r0 + pr;
      if (store_f32 && pr < P) __stcs(reinterpret_cast<float4*>(p.S + row * N + col), x[r]);
      if (CKPT != kCkptF32) {  // re-quantise the read copy (or the shared FP8 state) from the fresh row
        const float am = seg_allmax<TPR>(amax4(x[r]));
        float sc, inv;
        if (CKPT == kCkptFp4) {
          e2m1_row_scale(am, sc, inv);
          if (pr < P)
            __stcs(reinterpret_cast<unsigned short*>(p.S8 + row * (N / 2) + col / 2),
                   static_cast<unsigned short>(quant4_e2m1(x[r], inv)));
        } else {
          e4m3_row_scale(am, sc, inv);
          if (pr < P) __stcs(reinterpret_cast<unsigned int*>(p.S8 + row * N + col), quant4_e4m3(x[r], inv));
        }
        if (pr < P && (lane % TPR) == 0) p.Sscale[row] = sc;
      }
    }
  }
  if (MODE == kModeFlush) return;

  // ---- outputs: the rows' dot products with the queries, reduced over the row's lanes
  static_assert(RT == kRowsPerThread, "one reduction per row group");
  float dv[NQR][Red::kHeld];
  int dbase = 0;
  bool dwr = false;
#pragma unroll
  for (int s = 0; s < NQR; ++s) {
    if (s < n) {
      const float4 qs = IoT<IO>::load4(qbuf + ((size_t)s * N + col) * S_IO);
      float part[RT];
#pragma unroll
      for (int r = 0; r < RT; ++r) part[r] = dot4(x[r], qs);
      dwr = Red::run(part, lane, dbase);
#pragma unroll
      for (int i = 0; i < Red::kHeld; ++i) dv[s][i] = part[i];
    }
  }
#pragma unroll
  for (int i = 0; i < Red::kHeld; ++i) {
    const int pr = rbase + dbase + i;
    if (dwr && pr < P) {
      if (MODE == kModeEager) {
        p.y[bh * PH + r0 + pr] = dv[0][i];
      } else {
        const float sc = pl.fp32_tile ? 1.f : scale_tile[pr];
#pragma unroll
        for (int s = 0; s < NQR; ++s)
          if (s < n)
            p.y[(((size_t)pl.b * n + s) * p.H + pl.h) * PH + r0 + pr] =
                fmaf(alpha[s], dv[s][i] * sc, u[s * p.u_stride + pr]);
      }
    }
  }
}

// The row warps' loop: every row warp takes every unit of the CTA in order, waiting for
// the unit's tile (tfull) and its coefficients (cready); the warp's own waits for the
// uses before came first, so both parity waits are exact. Releasing a unit frees its
// tile stage and its record stage, and counts the release for the coefficient warps.
template <int N, typename IO, int CKPT, int MODE, int NQ>
__device__ void row_loop(const KParams& p, uint8_t* tstages, uint8_t* rstages, Bars* bars, int warp, int lane) {
  constexpr int S_IO = IoT<IO>::bytes;
  const int NT = p.num_tstages, NR = p.num_rstages;
  const int total = cta_units(p);
  for (int i = 0; i < total; ++i) {
    const int st_t = i % NT, st_r = i % NR;
    bool ready = *reinterpret_cast<volatile int*>(&bars->abort_flag) == 0;
    if (ready) ready = mbar_wait_bounded(&bars->tfull[st_t], (i / NT) & 1);
    if (ready) ready = mbar_wait_bounded(&bars->cready[st_r], (i / NR) & 1);
    if (!__all_sync(0xffffffffu, ready)) {
      if (lane == 0) {
        report_error(p.status, kErrWaitTimeout);
        bars->abort_flag = 1;
      }
      break;
    }
    const uint8_t* tst = tstages + (size_t)st_t * p.tstage_bytes;
    const uint8_t* rst = rstages + (size_t)st_r * p.rstage_bytes;
    const int32_t word = reinterpret_cast<const int32_t*>(rst + p.off_meta)[0];
    const int msk = reinterpret_cast<const int32_t*>(rst + p.off_meta)[1];
    const Plan pl = make_plan<MODE, CKPT, S_IO>(p, cta_unit(p, i), word, msk);
    if (pl.active) row_unit<N, IO, CKPT, MODE, NQ>(p, pl, tst, rst, warp, lane);
    count_release(&bars->released[st_r], lane);
    mbar_arrive(&bars->rempty[st_r]);
    mbar_arrive(&bars->tempty[st_t]);
  }
}

template <int N, typename IO, int CKPT, int MODE, int NQ>
__global__ void __launch_bounds__(kThreads, 1) replay_kernel(const __grid_constant__ KParams p) {
  static_assert(kProducerWarps == 1, "stages must be filled in unit order");
  extern __shared__ __align__(128) uint8_t smem[];
  Bars* bars = reinterpret_cast<Bars*>(smem);
  uint8_t* tstages = smem + p.tstages_off;
  uint8_t* rstages = smem + p.rstages_off;
  constexpr int S_IO = IoT<IO>::bytes;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.num_tstages; ++s) {
      mbar_init(&bars->tfull[s], 1);                  // the producer's expect_tx
      mbar_init(&bars->tempty[s], kRowWarps * 32);    // every row warp's lanes
    }
    for (int s = 0; s < p.num_rstages; ++s) {
      mbar_init(&bars->rfull[s], MODE == kModeEager ? 32 : 1);  // the eager gather: 32 lanes' cp.async
      mbar_init(&bars->cready[s], 32);                // a coefficient warp's lanes
      mbar_init(&bars->rempty[s], kRowWarps * 32);    // every row warp's lanes
    }
    bars->abort_flag = 0;
    for (int s = 0; s < kMaxTileStages; ++s) bars->last_tfill[s] = -1;
    for (int s = 0; s < kMaxRecStages; ++s) {
      bars->last_rfill[s] = -1;
      bars->released[s] = 0;
    }
    fence_mbar_init();
  }
  __syncthreads();
  if constexpr (MODE == kModeReplay && NQ == 1) {
    // One-position calls append their entries here rather than in a pre-pass: the row and
    // coefficient warps write the new ring records of the CTA's heads (v, then Delta and a
    // in one 16-byte piece; k once per chunk), make the writes visible to the bulk copies
    // that read them, and tell the producer, which meanwhile streams the first tiles.
    if (p.append_here && threadIdx.x < kWorkerWarps * 32) {
      append_entries<S_IO>(p);
      named_arrive(kAppendBar, kThreads);
    }
  }

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (warp >= kWorkerWarps) {
    if constexpr (MODE == kModeEager)
      producer_loop_eager<CKPT, S_IO>(p, tstages, rstages, bars);
    else
      producer_loop<MODE, CKPT, S_IO, MODE == kModeReplay && NQ == 1>(p, tstages, rstages, bars);
  } else if (warp >= kRowWarps) {
    const int cwarp = warp - kRowWarps;
    float* kq = reinterpret_cast<float*>(smem + p.ws_off + (size_t)cwarp * p.ws_bytes);
    coef_loop<N, IO, CKPT, MODE, NQ>(p, rstages, bars, kq, kq + p.ws_bytes / 8, cwarp, lane);
  } else {
    row_loop<N, IO, CKPT, MODE, NQ>(p, tstages, rstages, bars, warp, lane);
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
