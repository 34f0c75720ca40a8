// Launch parameters shared by the host launcher and the replay kernels.
#pragma once

#include <stdint.h>

namespace replay {

enum { kModeReplay = 0, kModeFlush = 1, kModeEager = 2 };
enum { kCkptF32 = 0, kCkptFp8 = 1, kCkptFp4 = 2 };

struct KParams {
  // sizes
  int32_t B, H, G, P, N, L, cap, n_pos, hpg;
  // units: a unit is rows [rb * rows_unit, min(P, (rb + 1) * rows_unit)) of one head of one
  // sequence, u = (b * H + h) * row_blocks + rb with row_blocks = 1 << rb_shift (1 or 2);
  // all row blocks of a head go to one CTA. Heads are dealt to CTAs in chunks of
  // chunk_heads consecutive heads of one k/q group (chunk c to CTA c mod grid).
  int32_t rows_unit, row_blocks, rb_shift, num_bh, num_units;
  int32_t chunk_heads, num_chunks;
  int32_t commit;  // replay: 1 = step (new entries committed), 0 = verify (tentative)
  int32_t fold_min;     // flush: fold only buffers holding at least this many entries (>= 1)
  int32_t flushed_or;   // replay: OR this call's fold flags into `flushed` (a flush before it wrote them)
  int32_t append_here;  // replay, one position: the entry comes from the inputs; the kernel appends it (no pre-pass)
  // this call's inputs and outputs
  const void* q;
  const void* k;
  const void* v;
  const float* dt;
  const float* a;
  float* y;
  uint8_t* flushed;
  const uint8_t* mask;
  // state (checkpoint or eager state)
  float* S;
  uint8_t* S8;
  float* Sscale;
  void* ring_k;        // [B][G][cap] k records of rec_k_bytes: k (N io)
  void* ring;          // [B][H][cap] head records of rec_bytes: v (P io), Delta, a
  const void* qpack;   // [B][G][qpack_pos][N] io verify queries packed per group, or null
  const int32_t* counts_in;
  int32_t* counts_out;
  int32_t* status;
  // shared-memory layout, bytes: a ring of stages, each holding one unit's tile, records,
  // queries and pointer word; one workspace per consumer group
  int32_t num_stages, stage_bytes, stages_off;
  int32_t rec_bytes, rec_k_bytes, qpack_pos;   // head / k record sizes; positions per qpack group
  int32_t off_krec, off_rec, off_q, off_meta;  // within a stage
  int32_t ws_off, ws_group_bytes;              // one workspace per consumer group
  int32_t ws_alpha, ws_sig, ws_cw, ws_kq, ws_wt, ws_inv;  // within a group's workspace
  int32_t wt_stride;                           // row stride of the fold weight table [L][wt_stride]
  int32_t smem_bytes;
};

// The pre-pass that writes this call's new entries into their ring records.
struct PackParams {
  int32_t B, H, G, P, N, L, cap, n_pos, hpg, rec_bytes, rec_k_bytes, io_bytes, qpack_pos;
  int32_t write_entries;  // 0: the entries are already in the ring (resident calls): pack queries only
  const void* q;
  const void* k;
  const void* v;
  const float* dt;
  const float* a;
  void* ring_k;
  void* ring;
  void* qpack;  // null: no packing of the queries
  const int32_t* counts_in;
};

// Snapshot export / import of n listed sequences.
struct SnapParams {
  int32_t B, H, G, P, N, L, cap, rec_bytes, rec_k_bytes, n;
  int64_t snap_bytes;      // bytes of one sequence's snapshot
  const int32_t* seqs;     // [n] sequence ids (device)
  void* snap;              // [n][snap_bytes] snapshots (device)
  float* S;
  uint8_t* S8;             // the read copy's codes and its scales (import re-quantises), or null
  float* Sscale;
  int32_t ckpt;            // kCkptFp8 / kCkptFp4: the read copy's format (import re-quantises)
  void* ring_k;
  void* ring;
  int32_t* counts;         // the current half of the pointer words
  int32_t* status;
};

}  // namespace replay
