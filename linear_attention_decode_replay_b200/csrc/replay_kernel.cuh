// Persistent, warp-specialised kernel for the ReplaySSM decode path on sm_100a.
//
// One launch processes every (sequence b, head h) unit of a decode layer. Each CTA owns
// the units blockIdx.x, blockIdx.x + gridDim.x, ... and streams them through a ring of
// shared-memory stages:
//   * the producer warp reads the unit's buffer pointer word (prefetched 32 units at a
//     time) and fills a stage with 1-D bulk copies (TMA), one copy per lane: the unit's
//     checkpoint tile S0[b,h] (P x N, FP32 master or FP8 read copy + per-row scales),
//     the unit's live ring records (k, v, Delta, a of every buffered input and of this
//     call's new tokens, which a pre-pass has already written into the ring) in one or
//     two pieces, and the queries; all complete on the stage's "full" mbarrier;
//   * NG consumer groups (8/NG warps each) take alternate units end to end: the state
//     row dot products together with the decay scans and k_j . q_s products, spread
//     over the group's warps, then the outputs (or the fused fold, its write-back and
//     the outputs from the fresh rows); each group releases the stage through its
//     "empty" mbarrier. Two groups keep two units in flight, so one unit's short
//     dependent chains overlap the other's.
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
static_assert(sizeof(Bars) <= 256, "the barrier header must fit the 256 bytes the host layout reserves");

struct Plan {
  int b, h, g, start, c;
  bool fold, corrupt, active, fp32_tile;
  uint32_t bytes;
};

template <int MODE, int CKPT, int S_IO>
__device__ __forceinline__ Plan make_plan(const KParams& p, int u, int32_t word, int msk) {
  Plan pl;
  pl.b = u / p.H;
  pl.h = u - pl.b * p.H;
  pl.g = pl.h / p.hpg;
  const uint32_t P = p.P, N = p.N;
  if (MODE == kModeEager) {
    pl.start = 0;
    pl.c = 0;
    pl.fold = true;
    pl.corrupt = false;
    pl.active = true;
    pl.fp32_tile = (CKPT == kCkptF32);
    pl.bytes = pl.fp32_tile ? P * N * 4u : P * N + P * 4u;  // bulk-copied (TMA) bytes
    return pl;
  }
  pl.start = word >> 16;
  pl.c = word & 0xFFFF;
  pl.corrupt = word < 0 || pl.c > p.L || pl.start >= p.cap;
  if (MODE == kModeReplay) {
    pl.fold = pl.c + p.n_pos > p.L;
    pl.active = true;
  } else {
    pl.fold = msk != 0 && pl.c > 0;
    pl.active = pl.fold;
  }
  pl.fp32_tile = (CKPT == kCkptF32) || pl.fold;
  if (pl.corrupt || !pl.active) {
    pl.active = false;
    pl.bytes = 0;
    return pl;
  }
  const uint32_t records = pl.c + ((MODE == kModeReplay) ? p.n_pos : 0);
  pl.bytes = (pl.fp32_tile ? P * N * 4u : P * N + P * 4u) + records * (uint32_t)p.rec_bytes +
             ((MODE == kModeReplay) ? p.n_pos * N * S_IO : 0u);
  return pl;
}

// Entry j of a unit lives in record j of the stage: k (N io values), v (P io values),
// Delta, a. Records 0..c-1 are the buffered inputs, c.. this call's new tokens.
template <int N, int S_IO>
struct Records {
  const uint8_t* base;
  int P, R;
  __device__ __forceinline__ const uint8_t* k(int j) const { return base + (size_t)j * R; }
  __device__ __forceinline__ const uint8_t* v(int j) const { return base + (size_t)j * R + N * S_IO; }
  __device__ __forceinline__ float dt(int j) const {
    return *reinterpret_cast<const float*>(base + (size_t)j * R + (N + P) * S_IO);
  }
  __device__ __forceinline__ float a(int j) const {
    return *reinterpret_cast<const float*>(base + (size_t)j * R + (N + P) * S_IO + 4);
  }
};

// ---------------------------------------------------------------------------- producer
// One unit's copies into stage `st`, one bulk copy (TMA) per lane, counted in bytes on
// `bar`: lane 0 the state tile, lane 1 the FP8 row scales, lanes 2-3 the live ring
// records [start, start + count) modulo cap, lane 4 the queries. The eager baseline has
// no ring: its new token's k, v, Delta, a (and q) are gathered with per-lane cp.async.
template <int MODE, int CKPT, int S_IO>
__device__ __forceinline__ void issue_unit_copies(const KParams& p, const Plan& pl, uint8_t* st, uint64_t* bar,
                                                  int lane, uint64_t stream_policy, uint64_t keep_policy) {
  const size_t P = p.P, N = p.N;
  const size_t bh = (size_t)pl.b * p.H + pl.h;
  if (!pl.active) return;
  uint8_t* recbuf = st + p.off_rec;
  if (MODE == kModeEager) {
    if (lane == 0)
      bulk_g2s_hint(st, pl.fp32_tile ? (const void*)(p.S + bh * P * N) : (const void*)(p.S8 + bh * P * N),
                    pl.fp32_tile ? (uint32_t)(P * N * 4) : (uint32_t)(P * N), bar, stream_policy);
    if (lane == 1 && !pl.fp32_tile) bulk_g2s(st + P * N, p.Sscale + bh * P, (uint32_t)(P * 4), bar);
    const int kpe = (int)(N * S_IO / 16);
    const int vpe = (int)(P * S_IO / 16);
    const size_t bg = (size_t)pl.b * p.G + pl.g;
    for (int idx = lane; idx < 2 * kpe + vpe; idx += 32) {
      if (idx < kpe) {
        cp_async16(st + p.off_q + idx * 16, static_cast<const uint8_t*>(p.q) + bg * N * S_IO + idx * 16);
      } else if (idx < 2 * kpe) {
        const int ch = idx - kpe;
        cp_async16(recbuf + ch * 16, static_cast<const uint8_t*>(p.k) + bg * N * S_IO + ch * 16);
      } else {
        const int ch = idx - 2 * kpe;
        cp_async16(recbuf + N * S_IO + ch * 16, static_cast<const uint8_t*>(p.v) + bh * P * S_IO + ch * 16);
      }
    }
    if (lane == 0) cp_async4(recbuf + (N + P) * S_IO, p.dt + bh);
    if (lane == 1) cp_async4(recbuf + (N + P) * S_IO + 4, p.a + bh);
    return;
  }
  // every lane works out its copy without branching, then one predicated instruction
  // issues all of them
  const int R = p.rec_bytes;
  const int cnt = pl.c + ((MODE == kModeReplay) ? p.n_pos : 0);
  const int first = min(cnt, p.cap - pl.start);
  const uint8_t* ring = static_cast<const uint8_t*>(p.ring) + bh * p.cap * R;
  const size_t bg = (size_t)pl.b * p.G + pl.g;
  const uint8_t* qsrc = p.qpack ? static_cast<const uint8_t*>(p.qpack) + bg * p.qpack_pos * N * S_IO
                                : static_cast<const uint8_t*>(p.q) + bg * N * S_IO;
  const uint8_t* tsrc = pl.fp32_tile ? reinterpret_cast<const uint8_t*>(p.S + bh * P * N) : p.S8 + bh * P * N;
  const uint8_t* src = (lane == 0)   ? tsrc
                       : (lane == 1) ? reinterpret_cast<const uint8_t*>(p.Sscale + bh * P)
                       : (lane == 2) ? ring + (size_t)pl.start * R
                       : (lane == 3) ? ring
                                     : qsrc;
  uint8_t* dst = (lane == 0)   ? st
                 : (lane == 1) ? st + P * N
                 : (lane == 2) ? recbuf
                 : (lane == 3) ? recbuf + (size_t)first * R
                               : st + p.off_q;
  uint32_t bytes = 0;
  bytes = (lane == 0) ? (pl.fp32_tile ? (uint32_t)(P * N * 4) : (uint32_t)(P * N)) : bytes;
  bytes = (lane == 1 && !pl.fp32_tile) ? (uint32_t)(P * 4) : bytes;
  bytes = (lane == 2) ? (uint32_t)(first * R) : bytes;
  bytes = (lane == 3) ? (uint32_t)((cnt - first) * R) : bytes;
  bytes = (lane == 4 && MODE == kModeReplay) ? (uint32_t)(p.n_pos * N * S_IO) : bytes;
  __syncwarp();
  if (bytes) bulk_g2s_hint(dst, src, bytes, bar, lane == 0 ? stream_policy : keep_policy);
}

template <int MODE, int CKPT, int S_IO>
__device__ void producer_loop(const KParams& p, uint8_t* stages, Bars* bars, int pw) {
  const int lane = threadIdx.x & 31;
  const int NS = p.num_stages;
  const uint64_t stream_policy = l2_evict_first_policy();
  const uint64_t keep_policy = l2_evict_normal_policy();
  // Producer warp pw fills the CTA's units i = pw, pw + kProducerWarps, ... Their pointer
  // words (and flush masks) are prefetched 32 units at a time, one chunk ahead: lane j
  // of a chunk holds the word of the chunk's j-th unit.
  auto unit_of = [&](int m) { return blockIdx.x + (pw + kProducerWarps * m) * gridDim.x; };
  auto load_words = [&](int m0, int32_t& w, int& msk) {
    w = 0;
    msk = 1;
    const int uu = unit_of(m0 + lane);
    if (MODE != kModeEager && uu < p.num_units) {
      const int b = uu / p.H;
      w = __ldg(p.counts_in + b);
      if (MODE == kModeFlush && p.mask) msk = __ldg(p.mask + b);
    }
  };
  int32_t w_cur, w_nxt;
  int m_cur, m_nxt;
  load_words(0, w_cur, m_cur);
  load_words(32, w_nxt, m_nxt);
  int m = 0;
  for (int u = unit_of(0); u < p.num_units; ++m, u = unit_of(m)) {
    const int i = pw + kProducerWarps * m;  // the CTA-local unit index
    const int s = i % NS;
    const int k = i / NS;
    if ((m & 31) == 0 && m > 0) {
      w_cur = w_nxt;
      m_cur = m_nxt;
      load_words(m + 32, w_nxt, m_nxt);
    }
    if (k > 0) {
      // every lane waits (each lane then writes into the stage), the warp agrees
      const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->empty[s], (k - 1) & 1));
      if (!ok) {
        if (lane == 0) {
          report_error(p.status, kErrWaitTimeout);
          bars->abort_flag = 1;
        }
        break;
      }
    }
    int ab = (lane == 0) ? *reinterpret_cast<volatile int*>(&bars->abort_flag) : 0;
    if (__shfl_sync(0xffffffffu, ab, 0)) break;  // the warp decides together
    const int32_t word = __shfl_sync(0xffffffffu, w_cur, m & 31);
    const int msk = __shfl_sync(0xffffffffu, m_cur, m & 31);
    const Plan pl = make_plan<MODE, CKPT, S_IO>(p, u, word, msk);
    uint8_t* st = stages + (size_t)s * p.stage_bytes;
    if (lane == 0) {
      reinterpret_cast<int32_t*>(st + p.off_meta)[0] = word;
      reinterpret_cast<int32_t*>(st + p.off_meta)[1] = msk;
      if (pl.corrupt) report_error(p.status, kErrPointer);
      mbar_arrive_expect_tx(&bars->full[s], pl.bytes);
    }
    __syncwarp();
    issue_unit_copies<MODE, CKPT, S_IO>(p, pl, st, &bars->full[s], lane, stream_policy, keep_policy);
    cp_async_arrive(&bars->full[s]);
    if (lane == 0) bars->last_fill[s] = i;
  }
  // Never leave with copies in flight into this CTA's shared memory. A fill that was
  // followed by a later fill of the same stage has been consumed; so once both producer
  // warps are done, each waits (bounded) for the latest fill of every stage that it made.
  asm volatile("bar.sync %0, %1;" ::"r"(kProducerBarrier), "r"(kProducerWarps * 32) : "memory");
  for (int st_i = 0; st_i < NS; ++st_i) {
    const int i = bars->last_fill[st_i];
    if (i >= 0 && i % kProducerWarps == pw) {
      if (!mbar_wait_bounded(&bars->full[st_i], (i / NS) & 1) && lane == 0) report_error(p.status, kErrWaitTimeout);
    }
  }
}

// ---------------------------------------------------------------------------- consumers
// kq[s][jj] = k_{o0+jj} . q_s for every query s < n and entry jj < width (<= 32).
template <int N, typename IO, int GW>
__device__ __forceinline__ void entry_dots(const Records<N, IoT<IO>::bytes>& rec, const uint8_t* qbuf, int o0,
                                           int width, int n, float* kq, int gw, int lane) {
  constexpr int S_IO = IoT<IO>::bytes;
  if constexpr (N == 128) {
    // a warp per (query, 8 entries): the lanes split N, a transposing reduction sums them
    const int chunks = (width + 7) / 8;
    for (int t = gw; t < n * chunks; t += GW) {
      const int s = t / chunks;
      const int ch = t - s * chunks;
      const float4 qv = IoT<IO>::load4(qbuf + ((size_t)s * N + lane * 4) * S_IO);
      float part[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int jj = ch * 8 + r;
        part[r] = (jj < width) ? dot4(IoT<IO>::load4(rec.k(o0 + jj) + lane * 4 * S_IO), qv) : 0.f;
      }
      int base;
      const bool wr = SegReduce<8, 32>::run(part, lane, base);
      const int jj = ch * 8 + base;
      if (wr && jj < width) kq[s * kMaxWindow + jj] = part[0];
    }
  } else {
    // short rows: a lane per (query, entry)
    for (int t = gw * 32 + lane; t < n * width; t += GW * 32) {
      const int s = t / width;
      const int jj = t - s * width;
      const uint8_t* kr = rec.k(o0 + jj);
      const uint8_t* qr = qbuf + (size_t)s * N * S_IO;
      float d = 0.f;
#pragma unroll
      for (int c4 = 0; c4 < N; c4 += 4) d += dot4(IoT<IO>::load4(kr + (size_t)c4 * S_IO), IoT<IO>::load4(qr + (size_t)c4 * S_IO));
      kq[s * kMaxWindow + jj] = d;
    }
  }
}

template <int N, typename IO, int CKPT, int MODE, int NQ, int NG>
__device__ __forceinline__ void consume_unit(const KParams& p, const Plan& pl, uint8_t* st, uint8_t* ws, int gtid,
                                             int bar_id) {
  using Gr = Groups<NG>;
  constexpr int GT = Gr::kThreads;
  constexpr int GW = Gr::kWarps;
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
  const int row0 = gw * RPW + lane / TPR;
  const int col = (lane % TPR) * 4;
  const int P = p.P;
  const int c = pl.c;
  const int n = (MODE == kModeReplay) ? p.n_pos : (MODE == kModeEager ? 1 : 0);
  const int cf = (MODE == kModeEager) ? 1 : (pl.fold ? c : 0);  // entries folded into the state
  const int o0 = pl.fold ? c : 0;                                // first entry the outputs read
  const int width = c + n - o0;                                  // entries the outputs read
  const int fp = p.fp;
  const uint8_t* tile = st;
  const uint8_t* qbuf = st + p.off_q;
  const Records<N, S_IO> rec{st + p.off_rec, P, p.rec_bytes};
  const float* scale_tile = reinterpret_cast<const float*>(tile + (size_t)P * N);
  float* wout = reinterpret_cast<float*>(ws + p.ws_w);     // [kMaxPos][kMaxWindow] decay weight of entry o0+jj
  float* kq = reinterpret_cast<float*>(ws + p.ws_kq);      // [kMaxPos][kMaxWindow] k_{o0+jj} . q_s
  float* alpha = reinterpret_cast<float*>(ws + p.ws_alpha);
  float* sig = reinterpret_cast<float*>(ws + p.ws_sig);    // fold weights; [kMaxWindow] = abar
  float* wt = reinterpret_cast<float*>(ws + p.ws_wt);      // [P][fp] fold weight times v_j[p]
  const size_t bh = (size_t)pl.b * p.H + pl.h;
  const int ngroups = (P + RGR - 1) / RGR;

  float4 qr[NQR];
#pragma unroll
  for (int s = 0; s < NQ; ++s)
    qr[s] = (s < n) ? IoT<IO>::load4(qbuf + ((size_t)s * N + col) * S_IO) : make_float4(0.f, 0.f, 0.f, 0.f);

  // state rows of one row group (the read copy keeps its row scale for the dot product)
  auto load_rows = [&](float4 (&x)[RT], int gi, bool dequant) {
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const int pr = gi * RGR + row0 + RPG * r;
      x[r] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (pr < P) {
        if (pl.fp32_tile) {
          x[r] = *reinterpret_cast<const float4*>(tile + ((size_t)pr * N + col) * 4);
        } else {
          const float4 e = e4m3x4_to_float4(*reinterpret_cast<const uint32_t*>(tile + (size_t)pr * N + col));
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
  float4 x[RT];
  load_rows(x, 0, MODE == kModeEager);

  // output-only units with a single row group: the row dot products and their reduction
  // need nothing from the scans, so they run first; the sums wait in registers
  const bool early = !pl.fold && ngroups == 1;
  float dv[NQR][Red::kHeld];
  int dbase = 0;
  bool dwr = false;
  if (early) {
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
  }

  // ---- phase A: decay scans (a warp per task, on the group's last warps) and k_j . q_s
  {
    const int tasks = ((MODE == kModeReplay) ? n : 0) + (cf > 0 ? 1 : 0);
    for (int t = GW - 1 - gw; t < tasks; t += GW) {
      const bool fold_task = !(MODE == kModeReplay && t < n);
      const int last = fold_task ? cf - 1 : c + t - o0;  // last lane of the scanned window
      const int e0 = fold_task ? 0 : o0;
      float xa = 1.f, xd = 0.f;
      if (lane <= last) {
        xa = rec.a(e0 + lane);
        xd = rec.dt(e0 + lane);
      }
      const float incl = warp_suffix_prod(xa, lane);  // prod_{lane <= i <= last} a_i
      float excl = __shfl_down_sync(0xffffffffu, incl, 1);
      if (lane == 31) excl = 1.f;
      if (fold_task) {
        if (lane <= last) sig[lane] = xd * excl;
        if (lane == 0) sig[kMaxWindow] = incl;
      } else {
        if (lane <= last) wout[t * kMaxWindow + lane] = xd * excl;
        if (lane == 0) alpha[t] = incl;
      }
    }
    if (MODE == kModeReplay) entry_dots<N, IO, GW>(rec, qbuf, o0, width, n, kq, gw, lane);
  }
  group_sync(bar_id, GT);

  // y = alpha_s d + sum_{jj} w_{s,jj} kq_{s,jj} v_{o0+jj}[p], by the lanes that hold row p's d
  auto emit = [&](float d, int s, int pr) {
    if (MODE == kModeReplay) {
      const int last = c + s - o0;
      float b0 = 0.f, b1 = 0.f;
      int jj = 0;
      for (; jj + 1 <= last; jj += 2) {
        b0 = fmaf(wout[s * kMaxWindow + jj] * kq[s * kMaxWindow + jj], IoT<IO>::load1(rec.v(o0 + jj) + pr * S_IO), b0);
        b1 = fmaf(wout[s * kMaxWindow + jj + 1] * kq[s * kMaxWindow + jj + 1],
                  IoT<IO>::load1(rec.v(o0 + jj + 1) + pr * S_IO), b1);
      }
      if (jj <= last)
        b0 = fmaf(wout[s * kMaxWindow + jj] * kq[s * kMaxWindow + jj], IoT<IO>::load1(rec.v(o0 + jj) + pr * S_IO), b0);
      p.y[(((size_t)pl.b * n + s) * p.H + pl.h) * P + pr] = fmaf(alpha[s], d, b0 + b1);
    } else {
      p.y[bh * P + pr] = d;
    }
  };
  auto write_outputs = [&](float (&part)[RT], int s, int gi, bool from_tile_fp8) {
    int base;
    const bool wr = Red::run(part, lane, base);
#pragma unroll
    for (int i = 0; i < Red::kHeld; ++i) {
      const int pr = gi * RGR + row0 + RPG * (base + i);
      if (wr && pr < P) emit(from_tile_fp8 ? part[i] * scale_tile[pr] : part[i], s, pr);
    }
  };

  if (early) {
    // ---- phase B: combine the early row sums with the buffer term
#pragma unroll
    for (int s = 0; s < NQ; ++s) {
      if (s < n) {
#pragma unroll
        for (int i = 0; i < Red::kHeld; ++i) {
          const int pr = row0 + RPG * (dbase + i);
          if (dwr && pr < P) emit(pl.fp32_tile ? dv[s][i] : dv[s][i] * scale_tile[pr], s, pr);
        }
      }
    }
  } else if (!pl.fold) {
    // ---- phase B: output-only route, several row groups
    for (int gi = 0; gi < ngroups; ++gi) {
      if (gi > 0) load_rows(x, gi, false);
#pragma unroll
      for (int s = 0; s < NQ; ++s) {
        if (s < n) {
          float part[RT];
#pragma unroll
          for (int r = 0; r < RT; ++r) part[r] = dot4(x[r], qr[s]);
          write_outputs(part, s, gi, !pl.fp32_tile);
        }
      }
    }
  } else {
    // ---- phase B: fold (state route), write the state back, outputs from the fresh rows
    const int cf_pad = (cf + kFoldChunk - 1) / kFoldChunk * kFoldChunk;
    for (int idx = gtid; idx < P * cf_pad; idx += GT) {
      const int pp = idx / cf_pad;
      const int j = idx - pp * cf_pad;
      wt[pp * fp + j] = j < cf ? sig[j] * IoT<IO>::load1(rec.v(j) + pp * S_IO) : 0.f;
    }
    group_sync(bar_id, GT);
    const float abar = sig[kMaxWindow];
    for (int gi = 0; gi < ngroups; ++gi) {
      if (gi > 0) load_rows(x, gi, MODE == kModeEager);
#pragma unroll
      for (int r = 0; r < RT; ++r) x[r] = make_float4(abar * x[r].x, abar * x[r].y, abar * x[r].z, abar * x[r].w);
      for (int ch = 0; ch < cf_pad; ch += kFoldChunk) {
        float4 kr[kFoldChunk];
#pragma unroll
        for (int jj = 0; jj < kFoldChunk; ++jj) {
          const int j = ch + jj;
          kr[jj] = (j < cf) ? IoT<IO>::load4(rec.k(j) + col * S_IO) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          const int pr = gi * RGR + row0 + RPG * r;
          if (pr < P) {
            const float* wrow = wt + (size_t)pr * fp + ch;
#pragma unroll
            for (int jj = 0; jj < kFoldChunk; jj += 4) {
              const float4 w4 = *reinterpret_cast<const float4*>(wrow + jj);
              const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                x[r].x = fmaf(wv[t], kr[jj + t].x, x[r].x);
                x[r].y = fmaf(wv[t], kr[jj + t].y, x[r].y);
                x[r].z = fmaf(wv[t], kr[jj + t].z, x[r].z);
                x[r].w = fmaf(wv[t], kr[jj + t].w, x[r].w);
              }
            }
          }
        }
      }
      // write the state: FP32 master, and/or the FP8 codes with per-row scales
      const bool store_f32 = (MODE != kModeEager) || (CKPT == kCkptF32);
      const bool store_fp8 = (CKPT == kCkptFp8);
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const int pr = gi * RGR + row0 + RPG * r;
        if (store_f32 && pr < P) __stcs(reinterpret_cast<float4*>(p.S + (bh * P + pr) * N + col), x[r]);
        if (store_fp8) {
          const float am = seg_allmax<TPR>(amax4(x[r]));
          float sc, inv;
          e4m3_row_scale(am, sc, inv);
          if (pr < P) {
            __stcs(reinterpret_cast<unsigned int*>(p.S8 + (bh * P + pr) * N + col), quant4_e4m3(x[r], inv));
            if ((lane % TPR) == 0) p.Sscale[bh * P + pr] = sc;
          }
        }
      }
      if (MODE != kModeFlush) {
#pragma unroll
        for (int s = 0; s < NQ; ++s) {
          if (s < n) {
            float part[RT];
#pragma unroll
            for (int r = 0; r < RT; ++r) part[r] = dot4(x[r], qr[s]);
            write_outputs(part, s, gi, false);
          }
        }
      }
    }
  }

  // ---- publish the pointer word (the pre-pass already wrote this call's entries)
  const int start = pl.start;
  const int cap = p.cap;
  if (MODE == kModeReplay) {
    if (pl.h == 0 && gtid == 0) {
      int start2 = pl.fold ? start + c : start;
      start2 -= (start2 >= cap) ? cap : 0;
      const int base = pl.fold ? 0 : c;
      const int cnt2 = base + (p.commit ? n : 0);
      p.counts_out[pl.b] = (start2 << 16) | cnt2;
      if (p.flushed) p.flushed[pl.b] = pl.fold ? 1 : 0;
    }
  } else if (MODE == kModeFlush) {
    if (pl.h == 0 && gtid == 0) {
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

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.num_stages; ++s) {
      mbar_init(&bars->full[s], 1 + 32);  // the filling warp: lane 0's expect_tx + 32 lanes' cp.async
      mbar_init(&bars->empty[s], Gr::kThreads);
    }
    bars->abort_flag = 0;
    for (int s = 0; s < kMaxStages; ++s) bars->last_fill[s] = -1;
    fence_mbar_init();
  }
  __syncthreads();

  const int warp = threadIdx.x / 32;
  if (warp >= kConsumerWarps) {
    producer_loop<MODE, CKPT, S_IO>(p, stages, bars, warp - kConsumerWarps);
    return;
  }
  const int g = warp / Gr::kWarps;  // consumer group
  const int gtid = threadIdx.x - g * Gr::kThreads;
  const int bar_id = 1 + g;
  uint8_t* ws = smem + p.ws_off + (size_t)g * p.ws_group_bytes;
  const int NS = p.num_stages;
  int i = g;
  for (int u = blockIdx.x + g * gridDim.x; u < p.num_units; u += NG * gridDim.x, i += NG) {
    const int s = i % NS;
    const int k = i / NS;  // this is the k-th use of stage s
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
    const int32_t word = reinterpret_cast<const int32_t*>(st + p.off_meta)[0];
    const int msk = reinterpret_cast<const int32_t*>(st + p.off_meta)[1];
    const Plan pl = make_plan<MODE, CKPT, S_IO>(p, u, word, msk);
    if (pl.active) {
      consume_unit<N, IO, CKPT, MODE, NQ, NG>(p, pl, st, ws, gtid, bar_id);
    } else if (pl.h == 0 && gtid == 0) {
      p.counts_out[pl.b] = word;  // nothing to fold: the pointer word carries over
      if (MODE == kModeFlush && p.flushed && !pl.corrupt) p.flushed[pl.b] = 0;
    }
    group_sync(bar_id, Gr::kThreads);
    mbar_arrive(&bars->empty[s]);
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

}  // namespace replay
