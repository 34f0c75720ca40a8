/*
 * replay.h -- C ABI of the ReplaySSM decode path for scalar-decay (Mamba-2-style) SSM
 * layers on NVIDIA B200 (sm_100a).
 *
 * The method (blog "ReplaySSM: Cachear Inputs, No Estado", sections "Forma resumen",
 * "Forma historia", the two routes, "Decodificacion estandar", "Rollback",
 * "Paralelismo"; abstract of arXiv 2610.13778 "ReplaySSM: Cache SSM Inputs, Not State";
 * video page "The SSM Layer Nobody Made Fast (Until Now): ReplaySSM Explained", key
 * takeaways): instead of reading and writing the recurrent state
 *     S_t = a_t S_{t-1} + Delta_t v_t k_t^T,   y_t = S_t q_t
 * at every decode step, each sequence keeps a checkpoint S0 and a buffer of its inputs
 * (k_j, v_j, Delta_j, a_j) since S0. Most steps take the output-only route
 *     y_t = abar_t (S0 q_t) + sum_j s_{j,t} v_j (k_j^T q_t),
 *     abar_t = prod_{i<=t} a_i,   s_{j,t} = Delta_j prod_{j<i<=t} a_i,
 * and once per window of L tokens a flush folds the buffer into the checkpoint,
 *     S0 <- abar S0 + sum_j s_j v_j k_j^T.
 * Speculative verification scores several positions output-only with a causal mask,
 * rollback only moves the buffer pointer, and an optional FP8 e4m3 copy of S0 (one FP32
 * scale per row) serves the outputs while the flush updates an FP32 master.
 *
 * Conventions for every call below:
 *  - All pointers named "device" point to device memory owned by the caller; the
 *    library never allocates device memory. A replay_ctx holds host metadata only.
 *  - Work is queued asynchronously on the given stream. Only replay_read_counts and
 *    replay_check_status synchronise (that stream only).
 *  - The decode kernel is launched with programmatic stream serialization: its blocks may
 *    be scheduled while the previous kernel on the stream drains, but they read and write
 *    no global memory before that kernel has completed (griddepcontrol.wait), so stream
 *    order holds as for any launch; work queued after it waits for it as usual.
 *  - Invalid arguments return a negative replay_status at once and queue nothing.
 *    Errors found on the device are OR-ed into the caller's status word; read them
 *    with replay_check_status. No kernel traps.
 *  - Layouts are dense, row-major, batch-major. Shapes use B = batch, H = heads,
 *    G = k/q groups (H % G == 0; head h uses group h / (H/G)), P = v-dim, N = k-dim,
 *    L = window, cap = replay_ring_capacity(cfg), R = replay_ring_record_bytes(cfg).
 *    "io" is the replay_config.io dtype.
 *  - A replay_ctx is not thread-safe; calls on one context must be serialised.
 *  - replay_step and replay_flush queue kernels only, so a run of them can be captured
 *    into a CUDA graph and replayed (a graph launch per window instead of a host call
 *    per step), under three conditions: one call of the same kind has run outside the
 *    capture (the first launch of a kernel sets its shared-memory limit); the inputs
 *    and outputs are the buffers named at capture; and the run holds an even number of
 *    calls, because each call flips which half of `counts` holds the pointer words and
 *    the graph keeps the halves it was captured with.
 */
#ifndef REPLAY_H
#define REPLAY_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (cudaStream_t / CUstream); NULL is the legacy default stream. */
typedef struct CUstream_st* replay_stream_t;

typedef enum {
  REPLAY_OK = 0,
  REPLAY_EINVAL = -1,      /* bad size, null pointer, unsupported combination */
  REPLAY_EALIGN = -2,      /* a pointer misses its required alignment */
  REPLAY_ECUDA = -3,       /* a CUDA runtime call failed (launch, copy, attribute) */
  REPLAY_EPENDING = -4,    /* a verify is pending: call replay_rollback first */
  REPLAY_ENOPENDING = -5,  /* replay_rollback without a pending verify */
  REPLAY_EDEVICE = -6,     /* the device status word is non-zero (see replay_check_status) */
  REPLAY_ENOMEM = -7,      /* host allocation of the context failed */
  REPLAY_ESCRATCH = -8     /* replay_verify_static_scratch: the call's queries exceed
                              REPLAY_STATIC_SCRATCH_BYTES */
} replay_status;

typedef enum { REPLAY_F32 = 0, REPLAY_BF16 = 1 } replay_dtype;

typedef enum {
  REPLAY_CKPT_F32 = 0,          /* outputs and flushes use the FP32 checkpoint */
  REPLAY_CKPT_F32_FP8READ = 1,  /* outputs read an FP8 e4m3 copy; flushes update the FP32
                                   master and re-quantise the copy (abstract: separate
                                   state precisions; video takeaways: dual precision) */
  REPLAY_CKPT_F32_FP4READ = 2   /* the same with an FP4 e2m1 copy (video takeaways: FP8/FP4):
                                   one FP32 scale per row, scale = amax/6 */
} replay_ckpt;

/* Device-detected error bits OR-ed into the status word. */
#define REPLAY_DEV_WAIT_TIMEOUT 1 /* a pipeline wait gave up after ~2 s (results invalid) */
#define REPLAY_DEV_POINTER 2      /* a buffer pointer word was out of range */
#define REPLAY_DEV_ROLLBACK 4     /* n_keep outside [0, n_pos]; that sequence kept none */
#define REPLAY_DEV_SNAPSHOT 8     /* replay_import: a snapshot or sequence id did not match
                                     the layer; that snapshot was skipped */

typedef struct {
  int32_t batch;   /* B >= 1 */
  int32_t heads;   /* H >= 1 */
  int32_t groups;  /* G >= 1, H % G == 0 (k and q are shared by the H/G heads of a group) */
  int32_t P;       /* v-dim: multiple of 8, 8..256 */
  int32_t N;       /* k-dim: 16, 32, 64 or 128 */
  int32_t L;       /* window: buffer entries between checkpoint flushes, 1..32 */
  int32_t max_pos; /* largest n_pos of replay_verify, 1..8 and <= L (1 = plain decode) */
  int32_t io;      /* replay_dtype of q, k, v and of the ring of k, v */
  int32_t ckpt;    /* replay_ckpt */
} replay_config;

/* Caller-owned device buffers of one decode layer. All 16-byte aligned except counts and
 * status (4-byte). P*N*4 bytes per head must not exceed 65536.
 *
 * The buffer of recent inputs is a ring of `cap` records per sequence: one k record per
 * k/q group and one record per head. A group's heads share its k (blog, end of "Ruta
 * 'solo salida'": k and q belong to the group), so k is stored once per group. k record
 * j of (b, g): RK bytes, k (N io values) then padding. Head record j of (b, h): R bytes, v (P io values),
 * Delta (FP32), a (FP32), zero padding to a multiple of 16 bytes. Keeping an entry's pieces
 * together lets a unit's whole buffer arrive in one or two bulk copies per ring. */
typedef struct {
  float* S0;         /* [B][H][P][N] FP32 checkpoint (master); row p of N floats contiguous */
  uint8_t* S0_codes; /* the read copy's codes: FP8 [B][H][P][N] bytes; FP4 [B][H][P][N/2] bytes,
                        element 2i of a row in the low nibble of byte i, 2i+1 in the high
                        nibble; NULL for REPLAY_CKPT_F32 */
  float* S0_scale;   /* [B][H][P] FP32 per-row scale of the copy (same condition) */
  void* ring_k;      /* [B][G][cap] k records of RK bytes */
  void* ring;        /* [B][H][cap] head records of R bytes (v, Delta, a) */
  void* qpack;       /* [B][G][max_pos][N] io scratch for verify queries (max_pos > 1, else NULL) */
  int32_t* counts;   /* [2][B] buffer pointer words, double-buffered (the library alternates
                        halves each call so that no launch reads what it writes) */
  int32_t* status;   /* [1] device error word (REPLAY_DEV_* bits) */
} replay_buffers;

typedef struct replay_ctx replay_ctx;

/* Records the ring holds per (sequence, group) and per (sequence, head): L + max_pos. A
 * flush and the appends of the same call touch disjoint records. Returns a negative
 * replay_status on a bad config. */
int32_t replay_ring_capacity(const replay_config* cfg);

/* Bytes of one head record: P*s + 8 rounded up to a multiple of 16, s = 2 (BF16) or 4
 * (FP32). Returns a negative replay_status on a bad config. */
int32_t replay_ring_record_bytes(const replay_config* cfg);

/* Bytes of one k record: N*s + 16 (k, then 16 bytes of padding that keep consecutive
 * records on different shared-memory banks inside the kernel). Returns a negative
 * replay_status on a bad config. */
int32_t replay_ring_k_record_bytes(const replay_config* cfg);

/* Validates cfg and bufs, zeroes both halves of counts (every buffer empty) and the
 * status word, and with a read copy fills S0_codes / S0_scale from S0 (per-row e4m3 with
 * scale = amax/448, or e2m1 with scale = amax/6). S0 must already hold the initial
 * checkpoint. On success *out receives a context owned by the caller (free with
 * replay_destroy). REPLAY_EINVAL also when two pipeline stages of one unit do not fit in
 * shared memory (only the largest P, L and max_pos together with FP32 inputs). */
int replay_init(const replay_config* cfg, const replay_buffers* bufs, replay_stream_t stream,
                replay_ctx** out);

/* One decode token per sequence (blog "Decodificacion estandar"). Per sequence: if its
 * buffer already holds L entries, fold them into the checkpoint first, in the same launch
 * (the state is read once and written once); append (k, v, Delta, a); write
 *   y = abar (S q) + sum_j s_j v_j (k_j^T q)
 * over the buffer, S being the stored checkpoint (or its FP8 copy times the row scales)
 * or the fresh fold.
 *   q, k:  device [B][G][N] io        v: device [B][H][P] io
 *   dt, a: device [B][H] FP32         y: device [B][H][P] FP32 (written)
 *   flushed: device [B] uint8 (written: 1 where this call folded) or NULL.
 * Returns REPLAY_EPENDING while a verify awaits its rollback. */
int replay_step(replay_ctx* ctx, const void* q, const void* k, const void* v, const float* dt,
                const float* a, float* y, uint8_t* flushed, replay_stream_t stream);

/* Output-only verification of n_pos speculative positions (blog "Paralelismo";
 * abstract: output-only verification without intermediate states). Per sequence with c
 * committed entries: if c + n_pos > L, fold the c entries first (same launch); then the
 * n_pos entries are written to the ring tentatively and position s gets
 *   y_s = abar_{c+s} (S q_s) + sum_{j <= c+s} s_{j,c+s} v_j (k_j^T q_s)
 * (causal: position s sees the buffer up to its own entry). 1 <= n_pos <= min(L, max_pos).
 *   q, k:  device [B][n_pos][G][N] io     v: device [B][n_pos][H][P] io
 *   dt, a: device [B][n_pos][H] FP32      y: device [B][n_pos][H][P] FP32 (written)
 *   flushed: device [B] uint8 or NULL.
 * Must be followed by replay_rollback before the next step, verify or flush. */
int replay_verify(replay_ctx* ctx, int32_t n_pos, const void* q, const void* k, const void* v,
                  const float* dt, const float* a, float* y, uint8_t* flushed,
                  replay_stream_t stream);

/* ---- Zero-copy appends: the caller writes the entries straight into the ring ----
 * The buffer holds the raw inputs of the recent tokens (blog "Decodificacion estandar";
 * video takeaways: a ring buffer of the last L inputs). A caller whose projection kernel
 * produces k, v, Delta and a can write them directly into their ring records instead of
 * into separate input tensors that replay_step then copies: ask for the slots, write
 * the records, then call the resident variant, which reads the entries from the ring.
 *
 * replay_append_slots writes, for every sequence b, the ring record of its next entry:
 *   slots[b] = (start + count) mod cap   (device int32 [B], written on the stream),
 * from the current buffer pointer word. The entry of position s (0 for a step, 0..n_pos-1
 * for a verify) of sequence b goes to record (slots[b] + s) mod cap: its k into
 * ring_k[b][g] for every group g, its v, Delta and a into ring[b][h] for every head h
 * (layouts: see replay_buffers). slots[b] is -1 (and REPLAY_DEV_POINTER is set) for a
 * pointer word out of
 * range. The slots stay valid until the next step, verify, rollback or flush; a call
 * that folds reads records [start, start + count) and appends after them, so writing the
 * new records before that call never overwrites a buffered entry. Returns
 * REPLAY_EPENDING while a verify awaits its rollback. */
int replay_append_slots(replay_ctx* ctx, int32_t* slots, replay_stream_t stream);

/* replay_step whose entry is already in the ring (written at replay_append_slots' record
 * on this stream, or ordered before this call): only the query is passed.
 *   q: device [B][G][N] io   y: device [B][H][P] FP32   flushed: device [B] uint8 or NULL */
int replay_step_resident(replay_ctx* ctx, const void* q, float* y, uint8_t* flushed,
                         replay_stream_t stream);

/* replay_verify whose n_pos entries are already in the ring (records slots[b] + s mod
 * cap); only the queries are passed. Must be followed by replay_rollback.
 *   q: device [B][n_pos][G][N] io   y: device [B][n_pos][H][P] FP32   flushed: [B] or NULL */
int replay_verify_resident(replay_ctx* ctx, int32_t n_pos, const void* q, float* y, uint8_t* flushed,
                           replay_stream_t stream);

/* Resolves the pending verify (blog "Rollback (deshacer)"; video takeaways: rollback is a
 * pointer move): sequence b keeps the first n_keep[b] of the n_pos tentative entries
 * (device int32 [B], values in [0, n_pos]); the rest are dropped by moving the buffer end
 * back, O(1) per sequence, no state traffic. A value outside the range sets
 * REPLAY_DEV_ROLLBACK and keeps none for that sequence. */
int replay_rollback(replay_ctx* ctx, const int32_t* n_keep, replay_stream_t stream);

/* Folds the buffer of every sequence with mask[b] != 0 (device uint8 [B]; NULL = all)
 * into the checkpoint (state route) and empties it; also refreshes the FP8 copy. */
int replay_flush(replay_ctx* ctx, const uint8_t* mask, replay_stream_t stream);

/* ---- Snapshots of single sequences (export / import) ----
 * A sequence's decode state is its checkpoint, its committed buffer entries and their
 * count, nothing else (blog "Decodificacion estandar"; abstract: the buffer keeps the
 * raw inputs since the checkpoint). A snapshot holds exactly that, as one self-describing
 * block per sequence: a prefix-cache or migration unit (the hamidun.com page and the video
 * takeaways on snapshots and prefix caching). Layout of one block, replay_snapshot_bytes
 * long, all little-endian:
 *   int32[16] header: magic 0x4E535052, count c, H, P, N, L, R, G, RK, then zeros;
 *   FP32 [H][P][N]: the checkpoint S0 (the FP32 master);
 *   [G][L] k records of RK bytes, then [H][L] head records of R bytes: the committed
 *   entries, oldest first, in records 0 .. c-1 (the ring layouts; records c .. L-1 are
 *   unspecified).
 * The read copy is not stored: it is a function of the master (replay_init's per-row
 * quantiser), and import recomputes it. */

/* Bytes of one sequence's snapshot: 64 + H*P*N*4 + G*L*RK + H*L*R (a multiple of 16).
 * Returns a negative replay_status on a bad config. */
int64_t replay_snapshot_bytes(const replay_config* cfg);

/* Writes the snapshots of the n sequences seqs[0 .. n) (device int32 [n]) into dst
 * (device, [n][replay_snapshot_bytes], 16-byte aligned), on the stream. The state is
 * read, not changed. A sequence id out of range (or a corrupt pointer word) writes a
 * header with magic 0 and sets REPLAY_DEV_POINTER. Returns REPLAY_EPENDING while a verify
 * awaits its rollback (tentative entries are not part of a snapshot). */
int replay_export(replay_ctx* ctx, const int32_t* seqs, int32_t n, void* dst, replay_stream_t stream);

/* Restores snapshot i of src (device, [n][replay_snapshot_bytes], as replay_export wrote
 * it, from a context of the same H, G, P, N, L and io; batch and max_pos may differ) into
 * sequence seqs[i] of this context: its S0, its rings (entries in records 0 .. c-1) and
 * its pointer word; with a read copy also its codes and row scales, quantised from the
 * restored master. Decoding then continues exactly as it would have in the exporting
 * context (with the same checkpoint kind). A snapshot whose header does not match this
 * layer, or a
 * sequence id out of range, is skipped and sets REPLAY_DEV_SNAPSHOT. The seqs must be
 * distinct. Returns REPLAY_EPENDING while a verify awaits its rollback. */
int replay_import(replay_ctx* ctx, const int32_t* seqs, int32_t n, const void* src,
                  replay_stream_t stream);

/* Copies the committed entry count of every sequence to host_counts (host int32 [B]);
 * synchronises the stream. */
int replay_read_counts(replay_ctx* ctx, int32_t* host_counts, replay_stream_t stream);

/* Reads the device status word (synchronises the stream). Returns REPLAY_OK if it is
 * zero, else REPLAY_EDEVICE; *host_bits (may be NULL) receives the REPLAY_DEV_* bits. */
int replay_check_status(replay_ctx* ctx, int32_t* host_bits, replay_stream_t stream);

/* Frees the host context (the caller's device buffers are untouched). NULL is a no-op. */
void replay_destroy(replay_ctx* ctx);

/* Baseline: one eager decode step (blog "Forma resumen"), S <- a S + Delta v k^T and
 * y = S q, the FP32 state read and written in place. cfg supplies B, H, G, P, N, io
 * (L, max_pos and ckpt are ignored).
 *   S: device [B][H][P][N] FP32 (updated)   q, k: device [B][G][N] io   v: [B][H][P] io
 *   dt, a: device [B][H] FP32               y: device [B][H][P] FP32 (written) */
int eager_step(const replay_config* cfg, float* S, const void* q, const void* k, const void* v,
               const float* dt, const float* a, float* y, replay_stream_t stream);

/* Baseline: eager step on a state kept only in FP8 e4m3 with a per-row FP32 scale (a
 * shared low-precision checkpoint, whose rounding enters every later update; abstract
 * and video takeaways): dequantise, update, y from the updated FP32 values, re-quantise.
 *   S8: device [B][H][P][N] e4m3 (updated)   scale: device [B][H][P] FP32 (updated)
 *   other arguments as eager_step. */
int eager_step_fp8(const replay_config* cfg, uint8_t* S8, float* scale, const void* q,
                   const void* k, const void* v, const float* dt, const float* a, float* y,
                   replay_stream_t stream);

/* Per-row e2m1 quantisation used for the FP4 read copy: for each row of n FP32 values,
 * scale = amax/6 (1 for an all-zero row) and code = e2m1(x * (6/amax)) with the product
 * rounded to FP32, round-to-nearest-even, saturating to +-6; codes packed two per byte
 * (element 2i in the low nibble).
 *   x: device [rows][n] FP32   codes: device [rows][n/2] uint8   scale: device [rows] FP32
 *   n: 16, 32, 64 or 128. */
int replay_quantize_rows_e2m1(const float* x, int64_t rows, int32_t n, uint8_t* codes,
                              float* scale, replay_stream_t stream);

/* Per-row e4m3 quantisation used for the FP8 read copy: for each row of n FP32 values,
 * scale = amax/448 (1 for an all-zero row) and code = e4m3(x * (448/amax)) with the
 * product rounded to FP32, round-to-nearest-even, saturating to +-448.
 *   x: device [rows][n] FP32   codes: device [rows][n] uint8   scale: device [rows] FP32
 *   n: 16, 32, 64 or 128. */
int replay_quantize_rows_e4m3(const float* x, int64_t rows, int32_t n, uint8_t* codes,
                              float* scale, replay_stream_t stream);

/* ---- Verify without a query buffer from the caller (library extension) ----
 * The paper has no counterpart to this call. It serves callers that cannot allocate
 * device memory: a layer hosted by a program that owns all of the GPU's memory (a serving
 * engine that gives the free HBM to its own cache pool at start-up and hands each layer
 * only its state and per-call tensors), or a plug-in interface that passes inputs and
 * outputs but offers no way to ask for extra buffers. Such a caller cannot cudaMalloc the
 * qpack buffer that replay_verify needs when max_pos > 1.
 *
 * Size of the fixed device array that holds the packed queries: 32 MiB, enough for
 * B * G * n_pos * N io values up to B = 256, G = 64, n_pos = 8, N = 128 in BF16. */
#define REPLAY_STATIC_SCRATCH_BYTES (32u << 20)

/* replay_verify with the queries packed into the library's own fixed device array instead
 * of bufs.qpack, which this call never touches (it may be NULL: a context made with
 * max_pos = 1 needs none). Arguments, outputs and the pending-verify protocol are those of
 * replay_verify, with these differences:
 *  - Limit: B * G * n_pos * N * s bytes (s = 2 for BF16, 4 for FP32) must not exceed
 *    REPLAY_STATIC_SCRATCH_BYTES, else REPLAY_ESCRATCH is returned and nothing is queued.
 *  - 1 <= n_pos <= min(L, 8), even above the context's max_pos. When n_pos > max_pos the
 *    ring (cap = L + max_pos records per head) has room for the n_pos new entries only
 *    where the buffer holds c <= cap - n_pos entries, so the call first folds the
 *    buffers of the sequences with more (one more launch, which reads and writes only
 *    their states); the verify then folds the others itself where c + n_pos > L, as
 *    replay_verify does. `flushed` (if not NULL) reports both folds: 1 where either ran.
 *    With the FP8 read copy, a pre-folded sequence's outputs are read from its freshly
 *    re-quantised copy rather than from the fresh master (replay_verify, folding inside
 *    the verify, reads the master), so they differ from replay_verify's within the FP8
 *    error; with the FP32 checkpoint the two give the same outputs.
 *  - Allocation: none, on the device or the host. The array is part of the library's
 *    device code, so every GPU that loads libreplay.so holds its 32 MiB until the process
 *    exits.
 *  - Set-up: the first call with n_pos > 1 in a CUDA context (the device's primary
 *    context, as the runtime uses it) looks up that context's copy of the array
 *    (cudaGetSymbolAddress) and keeps it for later calls in the same context; after a
 *    device reset the next call looks it up again. The call must run with the context's
 *    device current (else REPLAY_EINVAL), and its first call should come before any
 *    stream capture.
 *  - Sharing: every call on a device, from any context, stream or thread, uses the same
 *    array. Calls whose work overlaps on the GPU race and corrupt each other's queries;
 *    order them (one stream, or events). The array keeps the last call's contents, but
 *    nothing in it needs to start at zero: a call writes each query before reading it. */
int replay_verify_static_scratch(replay_ctx* ctx, int32_t n_pos, const void* q, const void* k,
                                 const void* v, const float* dt, const float* a, float* y,
                                 uint8_t* flushed, replay_stream_t stream);

/* Static text for a replay_status code. */
const char* replay_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* REPLAY_H */
