// Launch parameters shared by the host launcher and the replay kernels.
#pragma once

#include <stdint.h>

namespace replay {

enum { kModeReplay = 0, kModeFlush = 1, kModeEager = 2 };
enum { kCkptF32 = 0, kCkptFp8 = 1 };

struct KParams {
  // sizes
  int32_t B, H, G, P, N, L, cap, n_pos, hpg;
  // units: a unit is rows [rb * rows_unit, min(P, (rb + 1) * rows_unit)) of one head of one
  // sequence, u = (b * H + h) * row_blocks + rb with row_blocks = 1 << rb_shift (1 or 2);
  // all row blocks of a head go to one CTA
  int32_t rows_unit, row_blocks, rb_shift, num_bh, num_units;
  int32_t commit;  // replay: 1 = step (new entries committed), 0 = verify (tentative)
  int32_t fold_min;     // flush: fold only buffers holding at least this many entries (>= 1)
  int32_t flushed_or;   // replay: OR this call's fold flags into `flushed` (a flush before it wrote them)
  int32_t append_here;  // replay, one position: the kernel appends the entries (no pre-pass)
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
  void* ring;          // [B][H][cap] records of rec_bytes: k (N io), v (P io), Delta, a
  const void* qpack;   // [B][G][qpack_pos][N] io verify queries packed per group, or null
  const int32_t* counts_in;
  int32_t* counts_out;
  int32_t* status;
  // shared-memory layout, bytes
  int32_t num_stages, stage_bytes, stages_off;
  int32_t rec_bytes, qpack_pos;                // ring record size; positions per qpack group
  int32_t off_rec, off_q, off_meta;            // within a stage
  int32_t ws_off, ws_group_bytes;          // one workspace per consumer group
  int32_t ws_alpha, ws_sig, ws_cw, ws_wt;  // within a group's workspace
  int32_t wt_stride;                           // row stride of the fold weight table [L][wt_stride]
  int32_t smem_bytes;
};

// The pre-pass that writes this call's new entries into their ring records.
struct PackParams {
  int32_t B, H, G, P, N, L, cap, n_pos, hpg, rec_bytes, io_bytes, qpack_pos;
  const void* q;
  const void* k;
  const void* v;
  const float* dt;
  const float* a;
  void* ring;
  void* qpack;  // null: no packing of the queries
  const int32_t* counts_in;
};

}  // namespace replay
