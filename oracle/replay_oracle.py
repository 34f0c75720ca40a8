"""CPU oracle for the scalar-decay SSM decode path of ReplaySSM -- TEST INFRASTRUCTURE.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import this
module. The product path (the CUDA library and its Python binding) never does, and
this module imports nothing from it.

Everything is plain float64 numpy, written for a reader to check against the pages
by eye. Sources, cited by page title and section:

* blog "ReplaySSM: Cachear Inputs, No Estado" (carlosgant.es), sections
  "Forma resumen" (summary / eager recurrence), "Forma historia" (unrolled form),
  "Ruta 'estado y salida' (outer product)", "Ruta 'solo salida' (inner product)",
  "Decodificacion estandar" (checkpoint + buffer, flush when full),
  "Rollback (deshacer)", "Paralelismo" (causal mask over the speculative window);
* abstract of arXiv 2610.13778 "ReplaySSM: Cache SSM Inputs, Not State"
  (periodic checkpoint update, output-only verification, buffer-pointer rollback,
  low-precision read copy with a high-precision master for the updates);
* video page "The SSM Layer Nobody Made Fast (Until Now): ReplaySSM Explained",
  key takeaways (ring buffer of L recent inputs, one flush write per window,
  rollback by moving the buffer pointer, FP8 dual precision).

Readings taken where the pages are garbled or silent (the blog's subscripts in the
state and output routes lost their braces):

* the decay product of the routes, written "a-bar t", is the product of a_i over every
  buffer entry i up to and including position t since the checkpoint, and the sum runs
  over every buffer entry j <= t; this is the only reading under which the routes equal
  the history form started from S0;
* y_t = S_t q_t uses the state after token t's own update;
* the flush is lazy: a call that cannot append its entries to a full buffer first folds
  the committed entries into the checkpoint (state route), then appends;
* FP8 is OCP e4m3 (1-4-3, bias 7, largest finite 448, no infinities), one FP32 scale
  per state row (amax / 448; 1 for an all-zero row), round to nearest even, saturate;
  the quantisation decision is taken in FP32 arithmetic, like the kernels';
* at a step that flushed, the output is read from the fresh master state, not from
  the FP8 copy.

Array conventions (head-batched; h = head, g = k/q group, h -> g = h // (H // G)):
S [H, P, N] (row p of length N), q, k [G, N], v [H, P], dt, a [H].
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


# --------------------------------------------------------------------------------------
# The recurrence and its two forms (blog, "Forma resumen" and "Forma historia")
# --------------------------------------------------------------------------------------

def eager_step(S, a, dt, v, k, q):
    """Summary (eager) form: S_t = a_t S_{t-1} + Delta_t v_t k_t^T, then y_t = S_t q_t.

    S [H,P,N]; a, dt [H]; v [H,P]; k, q [H,N] (already expanded to heads).
    Returns (S_t, y_t [H,P])."""
    S_t = a[:, None, None] * S + dt[:, None, None] * v[:, :, None] * k[:, None, :]
    y_t = np.einsum("hpn,hn->hp", S_t, q)
    return S_t, y_t


def history_state(S_init, a, dt, v, k):
    """History (unrolled) form, started from S_init instead of zero:

        S_t = (prod_{i<=t} a_i) S_init + sum_{j<=t} Delta_j (prod_{j<i<=t} a_i) v_j k_j^T

    over the T given tokens (a, dt [T,H]; v [T,H,P]; k [T,H,N]). Each product is
    taken directly from its definition."""
    T = a.shape[0]
    S = np.prod(a, axis=0)[:, None, None] * S_init
    for j in range(T):
        w = dt[j] * np.prod(a[j + 1:T], axis=0)  # [H]
        S = S + w[:, None, None] * v[j][:, :, None] * k[j][:, None, :]
    return S


# --------------------------------------------------------------------------------------
# Checkpoint + buffer routes (blog, "Ruta estado y salida" and "Ruta solo salida")
# --------------------------------------------------------------------------------------

def decay_weights(a_buf, dt_buf):
    """Decay factors of the routes at the newest buffer position t = T - 1:

        abar_t  = prod_{i<=t} a_i                  (weight of the checkpoint S0)
        s_{j,t} = Delta_j prod_{j<i<=t} a_i        (weight of buffer entry j <= t)

    a_buf, dt_buf [T,H]. Returns (abar [H], s [T,H])."""
    T = a_buf.shape[0]
    abar = np.prod(a_buf, axis=0)
    s = np.stack([dt_buf[j] * np.prod(a_buf[j + 1:T], axis=0) for j in range(T)]) \
        if T else np.zeros((0,) + a_buf.shape[1:])
    return abar, s


def state_route(S0, abar, s, v_buf, k_buf):
    """Outer-product route: S_t = abar_t S0 + sum_j s_{j,t} v_j k_j^T.

    S0 [H,P,N]; abar [H]; s [T,H]; v_buf [T,H,P]; k_buf [T,H,N]."""
    return abar[:, None, None] * S0 + np.einsum("th,thp,thn->hpn", s, v_buf, k_buf)


def output_only(S0, abar, s, v_buf, k_buf, q):
    """Inner-product route: y_t = abar_t (S0 q) + sum_j s_{j,t} v_j (k_j^T q).

    No state is formed; q [H,N]. Returns y [H,P]."""
    kq = np.einsum("thn,hn->th", k_buf, q)
    return abar[:, None] * np.einsum("hpn,hn->hp", S0, q) + \
        np.einsum("th,th,thp->hp", s, kq, v_buf)


def route_flops(P, N, entries):
    """Multiply-adds spent on the buffer entries by each route (blog, end of "Ruta solo
    salida"): the outer product forms P*N terms per entry, the inner product one N-dot
    plus one P-vector scale per entry."""
    return {"outer": entries * P * N, "inner": entries * (N + P)}


# --------------------------------------------------------------------------------------
# FP8 e4m3 (OCP 8-bit floating point, E4M3 variant) -- dual-precision read copy
# --------------------------------------------------------------------------------------

def e4m3_decode(codes):
    """Value of each e4m3 code: sign bit, 4 exponent bits (bias 7), 3 mantissa bits.
    Exponent field 0 is subnormal (M * 2^-9); S.1111.111 is NaN; no infinities."""
    c = np.asarray(codes).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    E = (c >> 3) & 0xF
    M = c & 0x7
    mag = np.where(E == 0, M * 2.0 ** -9, (1.0 + M / 8.0) * np.exp2(E - 7.0))
    mag = np.where((E == 15) & (M == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(x):
    """Round each value to the nearest e4m3 value (ties to even mantissa), saturating
    finite values beyond +-448 to +-448; NaN maps to 0x7F / 0xFF. Returns uint8 codes."""
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x).astype(np.int64) << 7
    nan = np.isnan(x)
    mag = np.minimum(np.abs(np.where(nan, 0.0, x)), E4M3_MAX)
    # spacing of representable values in the binade of mag: 2^(e-3), where e is the
    # binade exponent, held at -6 below the smallest normal (subnormal spacing 2^-9)
    _, e = np.frexp(mag)  # mag = f * 2^e with f in [0.5, 1)
    e = np.maximum(e - 1, -6)
    quantum = np.exp2(e - 3.0)
    val = np.rint(mag / quantum) * quantum  # exact scaling; rint = half to even
    # bit pattern of val (val may have rounded up into the next binade: still exact)
    f2, e2 = np.frexp(val)
    normal = val >= 2.0 ** -6
    E = np.where(normal, e2 + 6, 0)
    M = np.where(normal, (2.0 * f2 - 1.0) * 8.0, val / 2.0 ** -9)
    code = sign | (E.astype(np.int64) << 3) | M.astype(np.int64)
    code = np.where(nan, 0x7F | sign, code)
    return code.astype(np.uint8)


def quantize_rows_e4m3(S):
    """Per-row FP8 read copy of a state: the row (over N) is taken at its FP32 value,
    scale = amax / 448 in FP32 (1 when the row is all zero), codes = e4m3(x * (448 /
    amax)) with the product rounded to FP32 first. Returns (codes uint8 [...,N],
    scale float32 [...])."""
    x = np.asarray(S).astype(np.float32)
    amax = np.max(np.abs(x), axis=-1)
    zero = amax == 0
    safe = np.where(zero, np.float32(1), amax).astype(np.float32)
    scale = np.where(zero, np.float32(1), safe / np.float32(E4M3_MAX)).astype(np.float32)
    inv = np.where(zero, np.float32(1), np.float32(E4M3_MAX) / safe).astype(np.float32)
    codes = e4m3_encode((x * inv[..., None]).astype(np.float32))
    return codes, scale


def dequantize_rows_e4m3(codes, scale):
    """Read copy back to values: e4m3 value times its row's scale."""
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[..., None]


# --------------------------------------------------------------------------------------
# FP4 e2m1 (OCP Microscaling formats, FP4 E2M1 element) -- the 4-bit read copy
# --------------------------------------------------------------------------------------

E2M1_MAX = 6.0


def e2m1_decode(codes):
    """Value of each 4-bit e2m1 code: sign bit, 2 exponent bits (bias 1), 1 mantissa bit.
    Exponent field 0 is subnormal (M * 0.5); every code is finite (largest 6)."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    E = (c >> 1) & 0x3
    M = c & 0x1
    mag = np.where(E == 0, M * 0.5, (1.0 + M / 2.0) * np.exp2(E - 1.0))
    return sign * mag


def e2m1_encode(x):
    """Round each value to the nearest e2m1 value (ties to the even mantissa), saturating
    beyond +-6. Returns 4-bit codes (uint8, one per value)."""
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x).astype(np.int64) << 3
    mag = np.minimum(np.abs(x), E2M1_MAX)
    # spacing of representable values in the binade of mag: 2^(e-1) for mag in [2^e, 2^(e+1)),
    # held at 0.5 below 1 (subnormal spacing)
    _, e = np.frexp(mag)
    e = np.maximum(e - 1, 0)
    quantum = np.exp2(e - 1.0)
    val = np.rint(mag / quantum) * quantum  # half to even on the mantissa bit
    f2, e2 = np.frexp(val)
    normal = val >= 1.0
    E = np.where(normal, e2, 0)  # val = 2^(E-1) * (1 + M/2): E = e2 for val in [2^(e2-1), 2^e2)
    M = np.where(normal, (2.0 * f2 - 1.0) * 2.0, val / 0.5)
    return (sign | (E.astype(np.int64) << 1) | M.astype(np.int64)).astype(np.uint8)


def quantize_rows_e2m1(S):
    """Per-row FP4 read copy, the FP8 copy's recipe with the e2m1 range: scale = amax / 6
    in FP32 (1 for an all-zero row), codes = e2m1(x * (6 / amax)) with the product rounded
    to FP32 first. Returns (codes uint8 [..., N], one 4-bit code per value; scale float32
    [...])."""
    x = np.asarray(S).astype(np.float32)
    amax = np.max(np.abs(x), axis=-1)
    zero = amax == 0
    safe = np.where(zero, np.float32(1), amax).astype(np.float32)
    scale = np.where(zero, np.float32(1), safe / np.float32(E2M1_MAX)).astype(np.float32)
    inv = np.where(zero, np.float32(1), np.float32(E2M1_MAX) / safe).astype(np.float32)
    codes = e2m1_encode((x * inv[..., None]).astype(np.float32))
    return codes, scale


def dequantize_rows_e2m1(codes, scale):
    """FP4 read copy back to values: e2m1 value times its row's scale."""
    return e2m1_decode(codes) * np.asarray(scale, dtype=np.float64)[..., None]


# --------------------------------------------------------------------------------------
# One sequence with a checkpoint and a buffer (blog, "Decodificacion estandar",
# "Rollback", "Paralelismo"; arXiv abstract)
# --------------------------------------------------------------------------------------

class ReplaySeq:
    """Checkpoint S0 plus a buffer of the inputs (k, v, Delta, a) since S0.

    ckpt="f32":          every output reads the master S0.
    ckpt="f32_fp8read":  outputs read an e4m3 copy of S0 (per-row scale); the flush
                         updates the master and re-quantises the copy.
    ckpt="f32_fp4read":  the same with an e2m1 copy (video takeaways: FP8/FP4).
    Counters: state_reads / state_writes count full passes over the per-head state."""

    def __init__(self, S0, G, L, ckpt="f32"):
        S0 = np.array(S0, dtype=np.float64)
        self.H, self.P, self.N = S0.shape
        if self.H % G:
            raise ValueError("groups must divide heads")
        self.G, self.L, self.ckpt = G, L, ckpt
        self.group_of_head = np.arange(self.H) // (self.H // G)
        self.S0 = S0
        self.k, self.v, self.dt, self.a = [], [], [], []
        self.pending = None  # (base, n_pos) of an unresolved verify
        self.state_reads = 0
        self.state_writes = 0
        self._read_copy = None  # dequantised FP8 copy, kept until the next flush
        if ckpt not in ("f32", "f32_fp8read", "f32_fp4read"):
            raise ValueError(f"unknown checkpoint kind {ckpt}")
        self._quantize, self._dequantize = {
            "f32_fp8read": (quantize_rows_e4m3, dequantize_rows_e4m3),
            "f32_fp4read": (quantize_rows_e2m1, dequantize_rows_e2m1),
        }.get(ckpt, (None, None))
        if self._quantize is not None:
            self.codes, self.scale = self._quantize(self.S0)

    @property
    def count(self):
        return len(self.k)

    def _append(self, k, v, dt, a):
        self.k.append(np.asarray(k, np.float64))
        self.v.append(np.asarray(v, np.float64))
        self.dt.append(np.asarray(dt, np.float64))
        self.a.append(np.asarray(a, np.float64))

    def _buffer(self, upto):
        """Entries 0..upto-1, k expanded from groups to heads."""
        kb = np.array(self.k[:upto]).reshape(upto, self.G, self.N)[:, self.group_of_head]
        vb = np.array(self.v[:upto]).reshape(upto, self.H, self.P)
        ab = np.array(self.a[:upto]).reshape(upto, self.H)
        db = np.array(self.dt[:upto]).reshape(upto, self.H)
        return ab, db, vb, kb

    def fold(self):
        """Flush: fold every buffer entry into the checkpoint with the state route and
        empty the buffer (one state read and one state write)."""
        c = self.count
        if c:
            ab, db, vb, kb = self._buffer(c)
            abar, s = decay_weights(ab, db)
            self.S0 = state_route(self.S0, abar, s, vb, kb)
            if self._quantize is not None:
                self.codes, self.scale = self._quantize(self.S0)
                self._read_copy = None
            self.state_reads += 1
            self.state_writes += 1
        self.k, self.v, self.dt, self.a = [], [], [], []

    def _output(self, q, t, from_master):
        """Output-only route at buffer position t for query q [G,N]."""
        ab, db, vb, kb = self._buffer(t + 1)
        abar, s = decay_weights(ab, db)
        if self.ckpt == "f32" or from_master:
            S_read = self.S0
        else:
            if self._read_copy is None:
                self._read_copy = self._dequantize(self.codes, self.scale)
            S_read = self._read_copy
        return output_only(S_read, abar, s, vb, kb, np.asarray(q, np.float64)[self.group_of_head])

    def step(self, q, k, v, dt, a):
        """One decode token. Returns (y [H,P], flushed)."""
        if self.pending is not None:
            raise RuntimeError("a verify is pending: roll back first")
        flushed = self.count == self.L
        if flushed:
            self.fold()  # fused into this step: S0 is read once and written once
            self.state_reads -= 1
        self._append(k, v, dt, a)
        self.state_reads += 1
        return self._output(q, self.count - 1, from_master=flushed), flushed

    def verify(self, q, k, v, dt, a):
        """Score n_pos speculative positions output-only against the same S0 and buffer
        (position s sees entries up to its own, the causal mask). The entries stay
        tentative until rollback(). q, k [n,G,N]; v [n,H,P]; dt, a [n,H].
        Returns (y [n,H,P], flushed)."""
        if self.pending is not None:
            raise RuntimeError("a verify is pending: roll back first")
        n = len(q)
        if n > self.L:
            raise ValueError("n_pos exceeds the window")
        flushed = self.count + n > self.L
        if flushed:
            self.fold()
            self.state_reads -= 1
        base = self.count
        for s in range(n):
            self._append(k[s], v[s], dt[s], a[s])
        self.state_reads += 1
        ys = np.stack([self._output(q[s], base + s, from_master=flushed) for s in range(n)])
        self.pending = (base, n)
        return ys, flushed

    def rollback(self, n_keep):
        """Keep the first n_keep tentative entries of the pending verify; drop the rest
        by moving the buffer end back."""
        if self.pending is None:
            raise RuntimeError("no verify is pending")
        base, n = self.pending
        if not 0 <= n_keep <= n:
            raise ValueError("n_keep out of range")
        keep = base + n_keep
        self.k, self.v, self.dt, self.a = self.k[:keep], self.v[:keep], self.dt[:keep], self.a[:keep]
        self.pending = None


class ReplayBatch:
    """B independent sequences (the batch of a decode layer). Inputs are float64
    arrays with the batch as leading dim, laid out as the workloads module draws them."""

    def __init__(self, S0, G, L, ckpt="f32"):
        self.seqs = [ReplaySeq(S0[b], G, L, ckpt) for b in range(len(S0))]

    @property
    def counts(self):
        return np.array([s.count for s in self.seqs], dtype=np.int32)

    def step(self, q, k, v, dt, a):
        out = [s.step(q[b], k[b], v[b], dt[b], a[b]) for b, s in enumerate(self.seqs)]
        return np.stack([o[0] for o in out]), np.array([o[1] for o in out], dtype=np.uint8)

    def verify(self, q, k, v, dt, a):
        out = [s.verify(q[b], k[b], v[b], dt[b], a[b]) for b, s in enumerate(self.seqs)]
        return np.stack([o[0] for o in out]), np.array([o[1] for o in out], dtype=np.uint8)

    def rollback(self, n_keep):
        for b, s in enumerate(self.seqs):
            s.rollback(int(n_keep[b]))

    def flush(self, mask=None):
        for b, s in enumerate(self.seqs):
            if mask is None or mask[b]:
                s.fold()

    def checkpoints(self):
        return np.stack([s.S0 for s in self.seqs])


def eager_batch_step(S, q, k, v, dt, a, G):
    """Eager step over a batch: S [B,H,P,N]; q, k [B,G,N]; v [B,H,P]; dt, a [B,H].
    Returns (S_t, y [B,H,P])."""
    B, H = S.shape[:2]
    gh = np.arange(H) // (H // G)
    outs = [eager_step(S[b], a[b], dt[b], v[b], k[b][gh], q[b][gh]) for b in range(B)]
    return np.stack([o[0] for o in outs]), np.stack([o[1] for o in outs])


def eager_fp8_batch_step(codes, scale, q, k, v, dt, a, G):
    """Eager step on a state kept only in FP8 (shared low-precision checkpoint): the
    state is dequantised, updated and re-quantised every step, so each step's rounding
    enters every later update. The output is read from the updated state before it is
    re-quantised. Returns (codes, scale, y)."""
    S = dequantize_rows_e4m3(codes, scale)
    S_t, y = eager_batch_step(S, q, k, v, dt, a, G)
    codes, scale = quantize_rows_e4m3(S_t)
    return codes, scale, y


def relative_error(y, y_ref):
    """Max over all leading indices of ||y - y_ref||_2 / max(||y_ref||_2, 1e-30), the
    norm taken over the last axis (one output vector of one head)."""
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    num = np.linalg.norm(y - y_ref, axis=-1)
    den = np.maximum(np.linalg.norm(y_ref, axis=-1), 1e-30)
    return float(np.max(num / den)) if num.size else 0.0
