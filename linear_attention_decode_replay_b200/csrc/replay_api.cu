// Host side of the C ABI declared in include/replay.h: argument validation, the shared-
// memory layout of the replay kernel, the double-buffered pointer words, the pending-
// verify protocol, and launches on the caller's stream. No device memory is allocated.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>

#include "../../include/replay.h"
#include "replay_device.cuh"
#include "replay_launch.h"

using replay::KParams;
using replay::SnapParams;

struct replay_ctx {
  replay_config cfg;
  replay_buffers bufs;
  int cap;
  int parity;   // which half of counts holds the current pointer words
  int pending;  // n_pos of an unresolved verify, 0 if none
  int device;
  int num_sms;
  KParams kp_step, kp_verify, kp_flush;  // prebuilt launch layouts (pointers filled per call)
  int verify_ok;                          // kp_verify was built (max_pos > 1)
  int smem_optin;                         // the device's per-block shared-memory limit
  KParams kp_static[replay::kMaxPos + 1]; // replay_verify_static_scratch layouts, by n_pos
  int kp_static_ok[replay::kMaxPos + 1];  // ... built on first use
};

namespace {

constexpr int kHeaderBytes = replay::kHeaderBytes;  // the kernel's mbarriers and flags

inline int round_up(int x, int m) { return (x + m - 1) / m * m; }
inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int validate_config(const replay_config* c, bool needs_window) {
  if (!c) return REPLAY_EINVAL;
  if (c->batch < 1 || c->heads < 1 || c->groups < 1 || c->heads % c->groups) return REPLAY_EINVAL;
  if (c->P < 8 || c->P > 256 || c->P % 8) return REPLAY_EINVAL;
  if (c->N != 16 && c->N != 32 && c->N != 64 && c->N != 128) return REPLAY_EINVAL;
  if ((int64_t)c->P * c->N * 4 > 65536) return REPLAY_EINVAL;
  if (c->io != REPLAY_F32 && c->io != REPLAY_BF16) return REPLAY_EINVAL;
  if ((int64_t)c->batch * c->heads > INT32_MAX / 2) return REPLAY_EINVAL;
  if (needs_window) {
    if (c->L < 1 || c->L > replay::kMaxWindow) return REPLAY_EINVAL;
    if (c->max_pos < 1 || c->max_pos > replay::kMaxPos || c->max_pos > c->L) return REPLAY_EINVAL;
    if (c->ckpt != REPLAY_CKPT_F32 && c->ckpt != REPLAY_CKPT_F32_FP8READ && c->ckpt != REPLAY_CKPT_F32_FP4READ)
      return REPLAY_EINVAL;
  }
  return REPLAY_OK;
}

int ring_capacity(const replay_config& c) { return c.L + c.max_pos; }
// head record: v (P io values), Delta, a; k record: k (N io values)
int record_bytes(const replay_config& c) {
  const int s_io = c.io == REPLAY_BF16 ? 2 : 4;
  return round_up(c.P * s_io + 8, 16);
}
// k record: k (N io values), then 16 bytes of padding. The padding staggers consecutive
// records by four shared-memory banks once a unit's records sit in a stage, so that the
// lanes that read several entries' k at once (one entry per lane pair or quarter) spread
// over all 32 banks; without it every record starts on the same bank.
int record_k_bytes(const replay_config& c) { return c.N * (c.io == REPLAY_BF16 ? 2 : 4) + 16; }
int ckpt_kind(int ckpt) {
  return ckpt == REPLAY_CKPT_F32_FP8READ ? replay::kCkptFp8 : ckpt == REPLAY_CKPT_F32_FP4READ ? replay::kCkptFp4
                                                                                              : replay::kCkptF32;
}

struct DeviceInfo {
  int device, num_sms, smem_optin;
};

int device_info(DeviceInfo* d) {
  if (cudaGetDevice(&d->device) != cudaSuccess) return REPLAY_ECUDA;
  if (cudaDeviceGetAttribute(&d->num_sms, cudaDevAttrMultiProcessorCount, d->device) != cudaSuccess)
    return REPLAY_ECUDA;
  if (cudaDeviceGetAttribute(&d->smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, d->device) != cudaSuccess)
    return REPLAY_ECUDA;
  return REPLAY_OK;
}

// Shared-memory layout of one launch mode. nq_alloc = query slots per stage, jmax =
// entries a stage holds (buffer + new), lfold = most entries one unit folds; fp8_eager:
// the eager launch on a shared FP8 state (its tile is the codes and scales).
int build_layout(KParams* p, const replay_config& c, int mode, int fp8_eager, int cap, int smem_optin) {
  std::memset(p, 0, sizeof(*p));
  const int s_io = c.io == REPLAY_BF16 ? 2 : 4;
  const int P = c.P, N = c.N;
  int jmax, nq_alloc, lfold;  // records a stage holds, query slots, most entries one unit folds
  if (mode == replay::kModeReplay) {
    jmax = c.L + c.max_pos;
    nq_alloc = c.max_pos;
    lfold = c.L;
  } else if (mode == replay::kModeFlush) {
    jmax = c.L;
    nq_alloc = 0;
    lfold = c.L;
  } else {
    jmax = 1;
    nq_alloc = 1;
    lfold = 1;
  }
  p->rec_bytes = record_bytes(c);
  p->rec_k_bytes = record_k_bytes(c);
  // a unit is one row group of a head (all of it when P is smaller): its tile is at most
  // 64 rows x 128 floats, whatever P
  const int UR = P < replay::row_group_rows(N) ? P : replay::row_group_rows(N);
  // stage: the unit's FP32 rows (a read copy's codes and scales fit in the same space),
  // then its k records, head records, queries and pointer word
  const int tile = fp8_eager ? round_up(UR * N + UR * 4, 16) : UR * N * 4;
  p->off_krec = round_up(tile, 16);
  p->off_rec = p->off_krec + jmax * p->rec_k_bytes;
  p->off_q = p->off_rec + jmax * p->rec_bytes;
  p->off_meta = p->off_q + round_up(nq_alloc * N * s_io, 16);
  p->stage_bytes = round_up(p->off_meta + 32, 128);  // meta: word, mask, b, h, g, rb

  // one workspace per consumer group: alpha[kMaxPos], the fold weights [kMaxWindow] +
  // abar, the outputs' entry coefficients [kMaxPos][kMaxWindow], the raw k . q products
  // [kMaxPos][kMaxWindow] (kept for the group's next unit of the same chunk), and the
  // fold weights times v, [lfold][wt_stride] (a unit's rows, padded to a multiple of
  // kRowsPerThread)
  p->wt_stride = round_up(UR, replay::kRowsPerThread);
  p->ws_alpha = 0;
  p->ws_sig = p->ws_alpha + replay::kMaxPos * 4;
  p->ws_cw = round_up(p->ws_sig + (replay::kMaxWindow + 4) * 4, 16);
  p->ws_kq = p->ws_cw + replay::kMaxPos * replay::kMaxWindow * 4;
  p->ws_wt = round_up(p->ws_kq + replay::kMaxPos * replay::kMaxWindow * 4, 16);
  // ... and the inverse scales of a row group's rows, for the fold's re-quantisation
  p->ws_inv = round_up(p->ws_wt + lfold * p->wt_stride * 4, 16);
  p->ws_group_bytes = round_up(p->ws_inv + replay::row_group_rows(N) * 4, 128);
  p->ws_off = kHeaderBytes;
  p->stages_off = round_up(p->ws_off + replay::kGroups * p->ws_group_bytes, 128);
  const int avail = smem_optin - p->stages_off;
  int ns = avail / p->stage_bytes;
  if (ns > replay::kMaxStages) ns = replay::kMaxStages;
  if (ns < 2) return REPLAY_EINVAL;
  p->num_stages = ns;
  p->smem_bytes = p->stages_off + ns * p->stage_bytes;

  p->B = c.batch;
  p->H = c.heads;
  p->G = c.groups;
  p->P = P;
  p->N = N;
  p->L = c.L;
  p->cap = cap;
  p->hpg = c.heads / c.groups;
  p->rows_unit = UR;
  p->row_blocks = (P + UR - 1) / UR;  // 1 or 2: P <= 65536 / (4 N) <= 2 row groups
  p->rb_shift = p->row_blocks == 1 ? 0 : 1;
  if (p->row_blocks > 2) return REPLAY_EINVAL;
  p->num_bh = c.batch * c.heads;
  p->num_units = p->num_bh * p->row_blocks;
  // heads dealt to CTAs in chunks: the largest divisor of the heads per k/q group that is
  // at most kMaxChunkHeads, so that a chunk never spans two groups
  int ch = p->hpg < replay::kMaxChunkHeads ? p->hpg : replay::kMaxChunkHeads;
  while (p->hpg % ch) --ch;
  p->chunk_heads = ch;
  p->num_chunks = p->num_bh / ch;
  return REPLAY_OK;
}

cudaError_t launch_main(const KParams& p, const replay_config& c, int ckpt, int mode, int nq, int num_sms,
                        cudaStream_t s) {
  const int grid = p.num_chunks < num_sms ? p.num_chunks : num_sms;  // every CTA holds whole chunks of heads
  switch (c.N) {
    case 16: return replay::launch_replay_n16(p, c.io, ckpt, mode, nq, grid, s);
    case 32: return replay::launch_replay_n32(p, c.io, ckpt, mode, nq, grid, s);
    case 64: return replay::launch_replay_n64(p, c.io, ckpt, mode, nq, grid, s);
    case 128: return replay::launch_replay_n128(p, c.io, ckpt, mode, nq, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

void set_state(KParams* p, const replay_ctx* ctx) {
  p->S = ctx->bufs.S0;
  p->S8 = ctx->bufs.S0_codes;
  p->Sscale = ctx->bufs.S0_scale;
  p->ring = ctx->bufs.ring;
  p->ring_k = ctx->bufs.ring_k;
  p->qpack = nullptr;
  p->qpack_pos = ctx->cfg.max_pos;
  p->counts_in = ctx->bufs.counts + (size_t)ctx->parity * ctx->cfg.batch;
  p->counts_out = ctx->bufs.counts + (size_t)(1 - ctx->parity) * ctx->cfg.batch;
  p->status = ctx->bufs.status;
}

int check_inputs(const void* q, const void* k, const void* v, const float* dt, const float* a, const float* y) {
  if (!q || !k || !v || !dt || !a || !y) return REPLAY_EINVAL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16)) return REPLAY_EALIGN;
  if (!aligned(dt, 4) || !aligned(a, 4) || !aligned(y, 4)) return REPLAY_EALIGN;
  return REPLAY_OK;
}

// One step or verify call. resident: the call's entries are already in the ring (the
// caller wrote them at replay_append_slots' records), so nothing is appended.
int replay_call(replay_ctx* ctx, int n_pos, int commit, const void* q, const void* k, const void* v,
                const float* dt, const float* a, float* y, uint8_t* flushed, cudaStream_t s,
                bool resident = false) {
  KParams p = (n_pos > 1) ? ctx->kp_verify : ctx->kp_step;
  set_state(&p, ctx);
  p.n_pos = n_pos;
  p.commit = commit;
  p.q = q;
  p.k = k;
  p.v = v;
  p.dt = dt;
  p.a = a;
  p.y = y;
  p.flushed = flushed;
  // pre-pass: this call's entries into their ring records (and verify queries into qpack)
  replay::PackParams pp;
  pp.B = p.B;
  pp.H = p.H;
  pp.G = p.G;
  pp.P = p.P;
  pp.N = p.N;
  pp.L = p.L;
  pp.cap = p.cap;
  pp.n_pos = n_pos;
  pp.hpg = p.hpg;
  pp.rec_bytes = p.rec_bytes;
  pp.rec_k_bytes = p.rec_k_bytes;
  pp.io_bytes = ctx->cfg.io == REPLAY_BF16 ? 2 : 4;
  pp.qpack_pos = ctx->cfg.max_pos;
  pp.q = q;
  pp.k = k;
  pp.v = v;
  pp.dt = dt;
  pp.a = a;
  pp.ring = ctx->bufs.ring;
  pp.ring_k = ctx->bufs.ring_k;
  pp.qpack = n_pos > 1 ? ctx->bufs.qpack : nullptr;
  pp.counts_in = p.counts_in;
  pp.write_entries = resident ? 0 : 1;
  p.qpack = pp.qpack;
  if (n_pos == 1) {
    p.append_here = resident ? 0 : 1;  // the main kernel appends the one new entry itself
  } else {
    const long long tasks = (long long)p.B * p.H;
    const long long blocks = (tasks + 7) / 8;
    const int grid = (int)(blocks < (long long)ctx->num_sms * 16 ? blocks : (long long)ctx->num_sms * 16);
    if (replay::launch_pack_entries(pp, grid, s) != cudaSuccess) return REPLAY_ECUDA;
  }
  if (launch_main(p, ctx->cfg, ckpt_kind(ctx->cfg.ckpt), replay::kModeReplay, n_pos, ctx->num_sms, s) !=
      cudaSuccess)
    return REPLAY_ECUDA;
  ctx->parity ^= 1;
  return REPLAY_OK;
}

int eager_call(const replay_config* cfg, float* S, uint8_t* S8, float* scale, const void* q, const void* k,
               const void* v, const float* dt, const float* a, float* y, cudaStream_t s) {
  replay_config c = *cfg;
  c.L = 1;
  c.max_pos = 1;
  c.ckpt = REPLAY_CKPT_F32;
  int rc = validate_config(&c, true);
  if (rc) return rc;
  if ((rc = check_inputs(q, k, v, dt, a, y))) return rc;
  const bool fp8 = S8 != nullptr;
  if (fp8) {
    if (!scale) return REPLAY_EINVAL;
    if (!aligned(S8, 16) || !aligned(scale, 16)) return REPLAY_EALIGN;
  } else {
    if (!S) return REPLAY_EINVAL;
    if (!aligned(S, 16)) return REPLAY_EALIGN;
  }
  DeviceInfo d;
  if ((rc = device_info(&d))) return rc;
  KParams p;
  if ((rc = build_layout(&p, c, replay::kModeEager, fp8 ? 1 : 0, 0, d.smem_optin))) return rc;
  p.S = S;
  p.S8 = S8;
  p.Sscale = scale;
  p.n_pos = 1;
  p.q = q;
  p.k = k;
  p.v = v;
  p.dt = dt;
  p.a = a;
  p.y = y;
  p.status = nullptr;
  if (launch_main(p, c, fp8 ? replay::kCkptFp8 : replay::kCkptF32, replay::kModeEager, 1, d.num_sms, s) !=
      cudaSuccess)
    return REPLAY_ECUDA;
  return REPLAY_OK;
}

int64_t snapshot_bytes(const replay_config& c) {
  return replay::kSnapHeaderBytes + (int64_t)c.heads * c.P * c.N * 4 + (int64_t)c.groups * c.L * record_k_bytes(c) +
         (int64_t)c.heads * c.L * record_bytes(c);
}

int snapshot_params(replay_ctx* ctx, const int32_t* seqs, int32_t n, void* snap, SnapParams* sp) {
  if (!ctx || n < 0 || (n > 0 && (!seqs || !snap))) return REPLAY_EINVAL;
  if (ctx->pending) return REPLAY_EPENDING;
  if (n > 0 && (!aligned(seqs, 4) || !aligned(snap, 16))) return REPLAY_EALIGN;
  const replay_config& c = ctx->cfg;
  if ((int64_t)n * c.heads > INT32_MAX) return REPLAY_EINVAL;
  sp->B = c.batch;
  sp->H = c.heads;
  sp->P = c.P;
  sp->N = c.N;
  sp->L = c.L;
  sp->cap = ctx->cap;
  sp->rec_bytes = record_bytes(c);
  sp->rec_k_bytes = record_k_bytes(c);
  sp->G = c.groups;
  sp->ckpt = ckpt_kind(c.ckpt);
  sp->n = n;
  sp->snap_bytes = snapshot_bytes(c);
  sp->seqs = seqs;
  sp->snap = snap;
  sp->S = ctx->bufs.S0;
  sp->S8 = ctx->bufs.S0_codes;
  sp->Sscale = ctx->bufs.S0_scale;
  sp->ring = ctx->bufs.ring;
  sp->ring_k = ctx->bufs.ring_k;
  sp->counts = ctx->bufs.counts + (size_t)ctx->parity * c.batch;
  sp->status = ctx->bufs.status;
  return REPLAY_OK;
}

}  // namespace

extern "C" {

int32_t replay_ring_capacity(const replay_config* cfg) {
  const int rc = validate_config(cfg, true);
  if (rc) return rc;
  return ring_capacity(*cfg);
}

int32_t replay_ring_record_bytes(const replay_config* cfg) {
  const int rc = validate_config(cfg, true);
  if (rc) return rc;
  return record_bytes(*cfg);
}

int32_t replay_ring_k_record_bytes(const replay_config* cfg) {
  const int rc = validate_config(cfg, true);
  if (rc) return rc;
  return record_k_bytes(*cfg);
}

int replay_init(const replay_config* cfg, const replay_buffers* bufs, replay_stream_t stream, replay_ctx** out) {
  if (!out) return REPLAY_EINVAL;
  *out = nullptr;
  int rc = validate_config(cfg, true);
  if (rc) return rc;
  if (!bufs || !bufs->S0 || !bufs->ring || !bufs->ring_k || !bufs->counts || !bufs->status) return REPLAY_EINVAL;
  const bool copy = cfg->ckpt != REPLAY_CKPT_F32;  // a low-precision read copy
  if (copy && (!bufs->S0_codes || !bufs->S0_scale)) return REPLAY_EINVAL;
  if (cfg->max_pos > 1 && !bufs->qpack) return REPLAY_EINVAL;
  if (!aligned(bufs->S0, 16) || !aligned(bufs->ring, 16) || !aligned(bufs->ring_k, 16) ||
      !aligned(bufs->counts, 4) || !aligned(bufs->status, 4))
    return REPLAY_EALIGN;
  if (copy && (!aligned(bufs->S0_codes, 16) || !aligned(bufs->S0_scale, 16))) return REPLAY_EALIGN;
  if (cfg->max_pos > 1 && !aligned(bufs->qpack, 16)) return REPLAY_EALIGN;

  DeviceInfo d;
  if ((rc = device_info(&d))) return rc;
  replay_ctx* ctx = new (std::nothrow) replay_ctx;
  if (!ctx) return REPLAY_ENOMEM;
  std::memset(ctx, 0, sizeof(*ctx));
  ctx->cfg = *cfg;
  ctx->bufs = *bufs;
  if (!copy) {
    ctx->bufs.S0_codes = nullptr;
    ctx->bufs.S0_scale = nullptr;
  }
  ctx->cap = ring_capacity(*cfg);
  ctx->device = d.device;
  ctx->num_sms = d.num_sms;
  ctx->smem_optin = d.smem_optin;
  replay_config one = *cfg;
  one.max_pos = 1;
  if ((rc = build_layout(&ctx->kp_step, one, replay::kModeReplay, 0, ctx->cap, d.smem_optin)) ||
      (rc = build_layout(&ctx->kp_flush, *cfg, replay::kModeFlush, 0, ctx->cap, d.smem_optin))) {
    delete ctx;
    return rc;
  }
  ctx->kp_flush.fold_min = 1;  // a flush folds every selected buffer that holds an entry
  if (cfg->max_pos > 1) {
    if ((rc = build_layout(&ctx->kp_verify, *cfg, replay::kModeReplay, 0, ctx->cap, d.smem_optin))) {
      delete ctx;
      return rc;
    }
    ctx->verify_ok = 1;
  }
  // the step layout was built with max_pos = 1 but indexes the same ring (capacity cap)
  ctx->kp_step.cap = ctx->cap;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(bufs->counts, 0, sizeof(int32_t) * 2 * (size_t)cfg->batch, s) != cudaSuccess ||
      cudaMemsetAsync(bufs->status, 0, sizeof(int32_t), s) != cudaSuccess) {
    delete ctx;
    return REPLAY_ECUDA;
  }
  if (copy) {
    const long long rows = (long long)cfg->batch * cfg->heads * cfg->P;
    const long long passes = (rows + (256 / (cfg->N / 4)) - 1) / (256 / (cfg->N / 4));
    const int grid = (int)(passes < (long long)d.num_sms * 8 ? passes : (long long)d.num_sms * 8);
    const cudaError_t e =
        cfg->ckpt == REPLAY_CKPT_F32_FP4READ
            ? replay::launch_quantize_rows_e2m1(bufs->S0, rows, cfg->N, bufs->S0_codes, bufs->S0_scale, grid, s)
            : replay::launch_quantize_rows(bufs->S0, rows, cfg->N, bufs->S0_codes, bufs->S0_scale, grid, s);
    if (e != cudaSuccess) {
      delete ctx;
      return REPLAY_ECUDA;
    }
  }
  *out = ctx;
  return REPLAY_OK;
}

int replay_step(replay_ctx* ctx, const void* q, const void* k, const void* v, const float* dt, const float* a,
                float* y, uint8_t* flushed, replay_stream_t stream) {
  if (!ctx) return REPLAY_EINVAL;
  if (ctx->pending) return REPLAY_EPENDING;
  int rc = check_inputs(q, k, v, dt, a, y);
  if (rc) return rc;
  return replay_call(ctx, 1, 1, q, k, v, dt, a, y, flushed, reinterpret_cast<cudaStream_t>(stream));
}

int replay_verify(replay_ctx* ctx, int32_t n_pos, const void* q, const void* k, const void* v, const float* dt,
                  const float* a, float* y, uint8_t* flushed, replay_stream_t stream) {
  if (!ctx) return REPLAY_EINVAL;
  if (ctx->pending) return REPLAY_EPENDING;
  if (n_pos < 1 || n_pos > ctx->cfg.max_pos || n_pos > ctx->cfg.L) return REPLAY_EINVAL;
  int rc = check_inputs(q, k, v, dt, a, y);
  if (rc) return rc;
  if (n_pos > 1 && !ctx->verify_ok) return REPLAY_EINVAL;
  rc = replay_call(ctx, n_pos, 0, q, k, v, dt, a, y, flushed, reinterpret_cast<cudaStream_t>(stream));
  if (rc == REPLAY_OK) ctx->pending = n_pos;
  return rc;
}

int replay_append_slots(replay_ctx* ctx, int32_t* slots, replay_stream_t stream) {
  if (!ctx || !slots) return REPLAY_EINVAL;
  if (ctx->pending) return REPLAY_EPENDING;
  if (!aligned(slots, 4)) return REPLAY_EALIGN;
  const int B = ctx->cfg.batch;
  if (replay::launch_append_slots(ctx->bufs.counts + (size_t)ctx->parity * B, slots, B, ctx->cfg.L, ctx->cap,
                                  ctx->bufs.status, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return REPLAY_ECUDA;
  return REPLAY_OK;
}

int replay_step_resident(replay_ctx* ctx, const void* q, float* y, uint8_t* flushed, replay_stream_t stream) {
  if (!ctx) return REPLAY_EINVAL;
  if (ctx->pending) return REPLAY_EPENDING;
  if (!q || !y) return REPLAY_EINVAL;
  if (!aligned(q, 16) || !aligned(y, 4)) return REPLAY_EALIGN;
  return replay_call(ctx, 1, 1, q, nullptr, nullptr, nullptr, nullptr, y, flushed,
                     reinterpret_cast<cudaStream_t>(stream), true);
}

int replay_verify_resident(replay_ctx* ctx, int32_t n_pos, const void* q, float* y, uint8_t* flushed,
                           replay_stream_t stream) {
  if (!ctx) return REPLAY_EINVAL;
  if (ctx->pending) return REPLAY_EPENDING;
  if (n_pos < 1 || n_pos > ctx->cfg.max_pos || n_pos > ctx->cfg.L) return REPLAY_EINVAL;
  if (!q || !y) return REPLAY_EINVAL;
  if (!aligned(q, 16) || !aligned(y, 4)) return REPLAY_EALIGN;
  if (n_pos > 1 && !ctx->verify_ok) return REPLAY_EINVAL;
  const int rc = replay_call(ctx, n_pos, 0, q, nullptr, nullptr, nullptr, nullptr, y, flushed,
                             reinterpret_cast<cudaStream_t>(stream), true);
  if (rc == REPLAY_OK) ctx->pending = n_pos;
  return rc;
}

int64_t replay_snapshot_bytes(const replay_config* cfg) {
  const int rc = validate_config(cfg, true);
  if (rc) return rc;
  return snapshot_bytes(*cfg);
}

int replay_export(replay_ctx* ctx, const int32_t* seqs, int32_t n, void* dst, replay_stream_t stream) {
  SnapParams sp;
  const int rc = snapshot_params(ctx, seqs, n, dst, &sp);
  if (rc || n == 0) return rc;
  return replay::launch_export(sp, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? REPLAY_OK : REPLAY_ECUDA;
}

int replay_import(replay_ctx* ctx, const int32_t* seqs, int32_t n, const void* src, replay_stream_t stream) {
  SnapParams sp;
  const int rc = snapshot_params(ctx, seqs, n, const_cast<void*>(src), &sp);
  if (rc || n == 0) return rc;
  return replay::launch_import(sp, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? REPLAY_OK : REPLAY_ECUDA;
}

int replay_rollback(replay_ctx* ctx, const int32_t* n_keep, replay_stream_t stream) {
  if (!ctx || !n_keep) return REPLAY_EINVAL;
  if (!ctx->pending) return REPLAY_ENOPENDING;
  if (!aligned(n_keep, 4)) return REPLAY_EALIGN;
  const int B = ctx->cfg.batch;
  const int32_t* cin = ctx->bufs.counts + (size_t)ctx->parity * B;
  int32_t* cout = ctx->bufs.counts + (size_t)(1 - ctx->parity) * B;
  if (replay::launch_rollback(cin, cout, n_keep, B, ctx->pending, ctx->bufs.status,
                              reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return REPLAY_ECUDA;
  ctx->parity ^= 1;
  ctx->pending = 0;
  return REPLAY_OK;
}

int replay_flush(replay_ctx* ctx, const uint8_t* mask, replay_stream_t stream) {
  if (!ctx) return REPLAY_EINVAL;
  if (ctx->pending) return REPLAY_EPENDING;
  KParams p = ctx->kp_flush;
  set_state(&p, ctx);
  p.mask = mask;
  if (launch_main(p, ctx->cfg, ckpt_kind(ctx->cfg.ckpt), replay::kModeFlush, 0, ctx->num_sms,
                  reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return REPLAY_ECUDA;
  ctx->parity ^= 1;
  return REPLAY_OK;
}

int replay_read_counts(replay_ctx* ctx, int32_t* host_counts, replay_stream_t stream) {
  if (!ctx || !host_counts) return REPLAY_EINVAL;
  const int B = ctx->cfg.batch;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(host_counts, ctx->bufs.counts + (size_t)ctx->parity * B, sizeof(int32_t) * B,
                      cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return REPLAY_ECUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return REPLAY_ECUDA;
  for (int b = 0; b < B; ++b) host_counts[b] &= 0xFFFF;
  return REPLAY_OK;
}

int replay_check_status(replay_ctx* ctx, int32_t* host_bits, replay_stream_t stream) {
  if (!ctx) return REPLAY_EINVAL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t bits = 0;
  if (cudaMemcpyAsync(&bits, ctx->bufs.status, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return REPLAY_ECUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return REPLAY_ECUDA;
  if (host_bits) *host_bits = bits;
  return bits ? REPLAY_EDEVICE : REPLAY_OK;
}

void replay_destroy(replay_ctx* ctx) { delete ctx; }

int eager_step(const replay_config* cfg, float* S, const void* q, const void* k, const void* v, const float* dt,
               const float* a, float* y, replay_stream_t stream) {
  if (!cfg) return REPLAY_EINVAL;
  return eager_call(cfg, S, nullptr, nullptr, q, k, v, dt, a, y, reinterpret_cast<cudaStream_t>(stream));
}

int eager_step_fp8(const replay_config* cfg, uint8_t* S8, float* scale, const void* q, const void* k, const void* v,
                   const float* dt, const float* a, float* y, replay_stream_t stream) {
  if (!cfg || !S8) return REPLAY_EINVAL;
  return eager_call(cfg, nullptr, S8, scale, q, k, v, dt, a, y, reinterpret_cast<cudaStream_t>(stream));
}

int replay_quantize_rows_e4m3(const float* x, int64_t rows, int32_t n, uint8_t* codes, float* scale,
                              replay_stream_t stream) {
  if (!x || !codes || !scale || rows < 0) return REPLAY_EINVAL;
  if (n != 16 && n != 32 && n != 64 && n != 128) return REPLAY_EINVAL;
  if (!aligned(x, 16) || !aligned(codes, 4) || !aligned(scale, 4)) return REPLAY_EALIGN;
  if (rows == 0) return REPLAY_OK;
  DeviceInfo d;
  int rc = device_info(&d);
  if (rc) return rc;
  const long long rpb = 256 / (n / 4);
  const long long passes = (rows + rpb - 1) / rpb;
  const int grid = (int)(passes < (long long)d.num_sms * 8 ? passes : (long long)d.num_sms * 8);
  if (replay::launch_quantize_rows(x, rows, n, codes, scale, grid, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return REPLAY_ECUDA;
  return REPLAY_OK;
}

int replay_quantize_rows_e2m1(const float* x, int64_t rows, int32_t n, uint8_t* codes, float* scale,
                              replay_stream_t stream) {
  if (!x || !codes || !scale || rows < 0) return REPLAY_EINVAL;
  if (n != 16 && n != 32 && n != 64 && n != 128) return REPLAY_EINVAL;
  if (!aligned(x, 16) || !aligned(codes, 2) || !aligned(scale, 4)) return REPLAY_EALIGN;
  if (rows == 0) return REPLAY_OK;
  DeviceInfo d;
  int rc = device_info(&d);
  if (rc) return rc;
  const long long rpb = 256 / (n / 4);
  const long long passes = (rows + rpb - 1) / rpb;
  const int grid = (int)(passes < (long long)d.num_sms * 8 ? passes : (long long)d.num_sms * 8);
  if (replay::launch_quantize_rows_e2m1(x, rows, n, codes, scale, grid, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return REPLAY_ECUDA;
  return REPLAY_OK;
}

const char* replay_strerror(int code) {
  switch (code) {
    case REPLAY_OK: return "ok";
    case REPLAY_EINVAL: return "invalid argument";
    case REPLAY_EALIGN: return "misaligned pointer";
    case REPLAY_ECUDA: return "CUDA runtime error";
    case REPLAY_EPENDING: return "a verify is pending: call replay_rollback first";
    case REPLAY_ENOPENDING: return "no verify is pending";
    case REPLAY_EDEVICE: return "device reported an error (see the status bits)";
    case REPLAY_ENOMEM: return "host allocation failed";
    case REPLAY_ESCRATCH: return "the call needs more query scratch than REPLAY_STATIC_SCRATCH_BYTES";
    default: return "unknown status";
  }
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Verify with the query scratch in a fixed device array (replay_verify_static_scratch).
// A library extension without a counterpart in the method: for callers that cannot
// allocate device memory, so cannot give replay_init a qpack buffer.
// ---------------------------------------------------------------------------------------

// The scratch itself. Every GPU that loads this library holds it until the process exits.
// In host code this name is only a handle for the runtime, not a device address.
static __device__ __align__(256) unsigned char replay_static_qpack[REPLAY_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kScratchDevices = 64;
std::mutex g_scratch_mu;
struct ScratchSlot {
  unsigned long long ctx_id;  // the CUDA context the address belongs to (0: none yet)
  void* addr;                 // that context's copy of replay_static_qpack
};
ScratchSlot g_scratch[kScratchDevices];

// The unique id of the calling thread's current CUDA context, 0 if it cannot be had.
// The driver calls are looked up through the runtime, so the library needs no link to
// the driver library.
unsigned long long current_context_id() {
  typedef int (*GetCurrentFn)(void**);
  typedef int (*GetIdFn)(void*, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {  // under g_scratch_mu
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
        q1 == cudaDriverEntryPointSuccess && q2 == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<GetCurrentFn>(f1);
      get_id = reinterpret_cast<GetIdFn>(f2);
    }
    looked_up = true;
  }
  if (!get_current || !get_id) return 0;
  void* cu_ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&cu_ctx) != 0 || !cu_ctx || get_id(cu_ctx, &id) != 0) return 0;
  return id;
}

// Set-up, once per device and CUDA context, with that device current: the context's
// address of the scratch array. A device reset ends the context that held the array; the
// next call sees a new context id and looks the address up again. Where the id cannot be
// had, the address is looked up on every call.
int static_scratch_address(int device, void** out) {
  if (device < 0 || device >= kScratchDevices) return REPLAY_EINVAL;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& slot = g_scratch[device];
  const unsigned long long id = current_context_id();
  if (id != 0 && slot.addr && slot.ctx_id == id) {
    *out = slot.addr;
    return REPLAY_OK;
  }
  void* ptr = nullptr;
  if (cudaGetSymbolAddress((void**)&ptr, replay_static_qpack) != cudaSuccess || !ptr) return REPLAY_ECUDA;
  slot.ctx_id = current_context_id();  // the lookup above made the context current if it was not
  slot.addr = ptr;
  *out = ptr;
  return REPLAY_OK;
}

}  // namespace

extern "C" int replay_verify_static_scratch(replay_ctx* ctx, int32_t n_pos, const void* q, const void* k,
                                            const void* v, const float* dt, const float* a, float* y,
                                            uint8_t* flushed, replay_stream_t stream) {
  if (!ctx) return REPLAY_EINVAL;
  if (ctx->pending) return REPLAY_EPENDING;
  const replay_config& cfg = ctx->cfg;
  if (n_pos < 1 || n_pos > replay::kMaxPos || n_pos > cfg.L) return REPLAY_EINVAL;
  const int64_t s_io = cfg.io == REPLAY_BF16 ? 2 : 4;
  const int64_t need = n_pos > 1 ? (int64_t)cfg.batch * cfg.groups * n_pos * cfg.N * s_io : 0;
  if (need > (int64_t)REPLAY_STATIC_SCRATCH_BYTES) return REPLAY_ESCRATCH;
  int rc = check_inputs(q, k, v, dt, a, y);
  if (rc) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (n_pos == 1) {
    // a single position packs no queries: the plain tentative step, no scratch
    rc = replay_call(ctx, 1, 0, q, k, v, dt, a, y, flushed, s);
    if (rc == REPLAY_OK) ctx->pending = 1;
    return rc;
  }
  int device = -1;
  if (cudaGetDevice(&device) != cudaSuccess) return REPLAY_ECUDA;
  if (device != ctx->device) return REPLAY_EINVAL;
  void* scratch = nullptr;
  if ((rc = static_scratch_address(device, &scratch))) return rc;
  if (!ctx->kp_static_ok[n_pos]) {
    replay_config c = cfg;
    c.max_pos = n_pos;
    if ((rc = build_layout(&ctx->kp_static[n_pos], c, replay::kModeReplay, 0, ctx->cap, ctx->smem_optin))) return rc;
    ctx->kp_static_ok[n_pos] = 1;
  }
  KParams p = ctx->kp_static[n_pos];
  const int ckpt = ckpt_kind(cfg.ckpt);
  const bool prefold = cfg.max_pos < n_pos;
  if (prefold) {
    // The ring holds cap = L + max_pos records per head, so a buffer of c entries has room
    // for the n_pos new ones only while c <= cap - n_pos: fold just the fuller buffers
    // first (the verify folds the others itself when c + n_pos > L). The flush writes
    // `flushed` for every sequence; the verify then ORs its own folds into it.
    KParams f = ctx->kp_flush;
    set_state(&f, ctx);
    f.flushed = flushed;
    f.fold_min = ctx->cap - n_pos + 1;
    if (launch_main(f, cfg, ckpt, replay::kModeFlush, 0, ctx->num_sms, s) != cudaSuccess) return REPLAY_ECUDA;
    ctx->parity ^= 1;
  }
  set_state(&p, ctx);
  p.qpack = scratch;
  p.qpack_pos = n_pos;
  p.n_pos = n_pos;
  p.commit = 0;
  p.flushed_or = prefold ? 1 : 0;
  p.q = q;
  p.k = k;
  p.v = v;
  p.dt = dt;
  p.a = a;
  p.y = y;
  p.flushed = flushed;
  replay::PackParams pp;
  pp.B = p.B;
  pp.H = p.H;
  pp.G = p.G;
  pp.P = p.P;
  pp.N = p.N;
  pp.L = p.L;
  pp.cap = p.cap;
  pp.n_pos = n_pos;
  pp.hpg = p.hpg;
  pp.rec_bytes = p.rec_bytes;
  pp.rec_k_bytes = p.rec_k_bytes;
  pp.io_bytes = (int)s_io;
  pp.qpack_pos = n_pos;
  pp.q = q;
  pp.k = k;
  pp.v = v;
  pp.dt = dt;
  pp.a = a;
  pp.ring = ctx->bufs.ring;
  pp.ring_k = ctx->bufs.ring_k;
  pp.qpack = scratch;
  pp.counts_in = p.counts_in;
  pp.write_entries = 1;
  const long long tasks = (long long)p.B * p.H;
  const long long blocks = (tasks + 7) / 8;
  const int grid = (int)(blocks < (long long)ctx->num_sms * 16 ? blocks : (long long)ctx->num_sms * 16);
  if (replay::launch_pack_entries(pp, grid, s) != cudaSuccess) return REPLAY_ECUDA;
  if (launch_main(p, cfg, ckpt, replay::kModeReplay, n_pos, ctx->num_sms, s) != cudaSuccess)
    return REPLAY_ECUDA;
  ctx->parity ^= 1;
  ctx->pending = n_pos;
  return REPLAY_OK;
}
