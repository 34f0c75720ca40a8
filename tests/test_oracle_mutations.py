"""Planted mistakes in the CPU oracle must each make at least one pin fail.

Every mutation below replaces one oracle function (on the CPU, inside this test only)
with a plausibly wrong version: a dropped term, an off-by-one in a decay product, a
wrong sign, a transposed operand, a wrong flush or rollback boundary, a wrong rounding
or scale in the FP8 encoder, an FP8 state read at the wrong moment or never
re-quantised. If no pin noticed one of them, the pins would not be pinning that part
of the oracle.
"""

import numpy as np
import pytest

import pins
from oracle import replay_oracle as ro

_orig = {name: getattr(ro, name) for name in dir(ro)}
_orig_seq = {name: getattr(ro.ReplaySeq, name) for name in ("step", "verify", "rollback", "fold", "_output")}


def m_decay_includes_own_a(a_buf, dt_buf):
    T = a_buf.shape[0]
    abar = np.prod(a_buf, axis=0)
    s = np.stack([dt_buf[j] * np.prod(a_buf[j:T], axis=0) for j in range(T)])
    return abar, s


def m_decay_abar_drops_newest(a_buf, dt_buf):
    abar, s = _orig["decay_weights"](a_buf, dt_buf)
    return np.prod(a_buf[:-1], axis=0), s


def m_decay_prefix_products(a_buf, dt_buf):
    T = a_buf.shape[0]
    abar = np.prod(a_buf, axis=0)
    s = np.stack([dt_buf[j] * np.prod(a_buf[:j], axis=0) for j in range(T)])
    return abar, s


def m_decay_drops_delta(a_buf, dt_buf):
    return _orig["decay_weights"](a_buf, np.ones_like(dt_buf))


def m_state_route_drops_abar(S0, abar, s, v_buf, k_buf):
    return _orig["state_route"](S0, np.ones_like(abar), s, v_buf, k_buf)


def m_state_route_transposed(S0, abar, s, v_buf, k_buf):
    # the rank-1 terms laid out as k v^T instead of v k^T
    return abar[:, None, None] * S0 + np.einsum("th,thp,thn->hnp", s, v_buf, k_buf)


def m_output_only_drops_buffer(S0, abar, s, v_buf, k_buf, q):
    return abar[:, None] * np.einsum("hpn,hn->hp", S0, q)


def m_output_only_transposed_s0(S0, abar, s, v_buf, k_buf, q):
    return _orig["output_only"](np.swapaxes(S0, 1, 2), abar, s, v_buf, k_buf, q)


def m_eager_decays_update(S, a, dt, v, k, q):
    S_t = a[:, None, None] * (S + dt[:, None, None] * v[:, :, None] * k[:, None, :])
    return S_t, np.einsum("hpn,hn->hp", S_t, q)


def m_eager_sign(S, a, dt, v, k, q):
    S_t = a[:, None, None] * S - dt[:, None, None] * v[:, :, None] * k[:, None, :]
    return S_t, np.einsum("hpn,hn->hp", S_t, q)


def m_eager_output_before_update(S, a, dt, v, k, q):
    S_t = a[:, None, None] * S + dt[:, None, None] * v[:, :, None] * k[:, None, :]
    return S_t, np.einsum("hpn,hn->hp", S, q)


def m_history_skips_first(S_init, a, dt, v, k):
    return _orig["history_state"](S_init, a, dt * (np.arange(len(a)) > 0)[:, None], v, k)


def m_step_flushes_early(self, q, k, v, dt, a):
    if self.count == self.L - 1 and self.L > 1:
        self.fold()
        self.state_reads -= 1
        self._append(k, v, dt, a)
        self.state_reads += 1
        return self._output(q, self.count - 1, from_master=True), True
    return _orig_seq["step"](self, q, k, v, dt, a)


def m_rollback_keeps_one_less(self, n_keep):
    return _orig_seq["rollback"](self, max(n_keep - 1, 0))


def m_verify_no_causal_mask(self, q, k, v, dt, a):
    ys, flushed = _orig_seq["verify"](self, q, k, v, dt, a)
    base, n = self.pending
    last = np.stack([self._output(q[s], base + n - 1, from_master=flushed) for s in range(n)])
    return last, flushed


def m_fold_keeps_buffer(self):
    k, v, dt, a = list(self.k), list(self.v), list(self.dt), list(self.a)
    _orig_seq["fold"](self)
    if k:
        self.k, self.v, self.dt, self.a = k[-1:], v[-1:], dt[-1:], a[-1:]


def m_output_reads_copy_at_flush(self, q, t, from_master):
    return _orig_seq["_output"](self, q, t, False)


def m_e4m3_round_half_up(x):
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x).astype(np.int64) << 7
    mag = np.minimum(np.abs(np.nan_to_num(x)), 448.0)
    _, e = np.frexp(mag)
    e = np.maximum(e - 1, -6)
    quantum = np.exp2(e - 3.0)
    val = np.floor(mag / quantum + 0.5) * quantum
    f2, e2 = np.frexp(val)
    normal = val >= 2.0 ** -6
    E = np.where(normal, e2 + 6, 0)
    M = np.where(normal, (2.0 * f2 - 1.0) * 8.0, val / 2.0 ** -9)
    return (sign | (E.astype(np.int64) << 3) | M.astype(np.int64)).astype(np.uint8)


def m_e4m3_no_saturation(x):
    x = np.asarray(x, dtype=np.float64)
    codes = _orig["e4m3_encode"](x)
    return np.where(np.abs(x) > 448.0, (np.signbit(x).astype(np.uint8) << 7) | 0x7F, codes).astype(np.uint8)


def m_e4m3_decode_bias8(codes):
    return _orig["e4m3_decode"](codes) / 2.0


def m_quantize_scale_256(S):
    x = np.asarray(S).astype(np.float32)
    amax = np.max(np.abs(x), axis=-1)
    safe = np.where(amax == 0, np.float32(1), amax).astype(np.float32)
    scale = np.where(amax == 0, np.float32(1), safe / np.float32(256)).astype(np.float32)
    inv = np.where(amax == 0, np.float32(1), np.float32(256) / safe).astype(np.float32)
    return _orig["e4m3_encode"]((x * inv[..., None]).astype(np.float32)), scale


def m_eager_fp8_output_after_requantise(codes, scale, q, k, v, dt, a, G):
    codes2, scale2, _ = _orig["eager_fp8_batch_step"](codes, scale, q, k, v, dt, a, G)
    S = ro.dequantize_rows_e4m3(codes2, scale2)
    B, H = S.shape[:2]
    gh = np.arange(H) // (H // G)
    y = np.stack([np.einsum("hpn,hn->hp", S[b], q[b][gh]) for b in range(B)])
    return codes2, scale2, y


def m_eager_fp8_never_requantises(codes, scale, q, k, v, dt, a, G):
    _, _, y = _orig["eager_fp8_batch_step"](codes, scale, q, k, v, dt, a, G)
    return codes, scale, y


def m_e2m1_round_half_up(x):
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x).astype(np.int64) << 3
    mag = np.minimum(np.abs(x), 6.0)
    _, e = np.frexp(mag)
    quantum = np.exp2(np.maximum(e - 1, 0) - 1.0)
    val = np.floor(mag / quantum + 0.5) * quantum
    f2, e2 = np.frexp(val)
    normal = val >= 1.0
    E = np.where(normal, e2, 0)
    M = np.where(normal, (2.0 * f2 - 1.0) * 2.0, val / 0.5)
    return (sign | (E.astype(np.int64) << 1) | np.minimum(M, 1).astype(np.int64)).astype(np.uint8)


def m_e2m1_decode_bias2(codes):
    return _orig["e2m1_decode"](codes) / 2.0


def m_quantize_e2m1_scale_4(S):
    x = np.asarray(S).astype(np.float32)
    amax = np.max(np.abs(x), axis=-1)
    safe = np.where(amax == 0, np.float32(1), amax).astype(np.float32)
    scale = np.where(amax == 0, np.float32(1), safe / np.float32(4)).astype(np.float32)
    inv = np.where(amax == 0, np.float32(1), np.float32(4) / safe).astype(np.float32)
    return _orig["e2m1_encode"]((x * inv[..., None]).astype(np.float32)), scale


def m_e2m1_no_saturation(x):
    x = np.asarray(x, dtype=np.float64)
    return np.where(np.abs(x) > 6.0, 0, _orig["e2m1_encode"](x)).astype(np.uint8)


def m_route_flops_counts_outer_twice(P, N, entries):
    f = _orig["route_flops"](P, N, entries)
    return {"outer": 2 * f["outer"], "inner": f["inner"]}


MODULE_MUTATIONS = [
    ("decay_weights", m_decay_includes_own_a),
    ("decay_weights", m_decay_abar_drops_newest),
    ("decay_weights", m_decay_prefix_products),
    ("decay_weights", m_decay_drops_delta),
    ("state_route", m_state_route_drops_abar),
    ("state_route", m_state_route_transposed),
    ("output_only", m_output_only_drops_buffer),
    ("output_only", m_output_only_transposed_s0),
    ("eager_step", m_eager_decays_update),
    ("eager_step", m_eager_sign),
    ("eager_step", m_eager_output_before_update),
    ("history_state", m_history_skips_first),
    ("e4m3_encode", m_e4m3_round_half_up),
    ("e4m3_encode", m_e4m3_no_saturation),
    ("e4m3_decode", m_e4m3_decode_bias8),
    ("quantize_rows_e4m3", m_quantize_scale_256),
    ("route_flops", m_route_flops_counts_outer_twice),
    ("eager_fp8_batch_step", m_eager_fp8_output_after_requantise),
    ("eager_fp8_batch_step", m_eager_fp8_never_requantises),
    ("e2m1_encode", m_e2m1_round_half_up),
    ("e2m1_encode", m_e2m1_no_saturation),
    ("e2m1_decode", m_e2m1_decode_bias2),
    ("quantize_rows_e2m1", m_quantize_e2m1_scale_4),
]
SEQ_MUTATIONS = [
    ("step", m_step_flushes_early),
    ("rollback", m_rollback_keeps_one_less),
    ("verify", m_verify_no_causal_mask),
    ("fold", m_fold_keeps_buffer),
    ("_output", m_output_reads_copy_at_flush),
]


def _failing_pins():
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin()
        except Exception:  # noqa: BLE001 - any error means the pin caught the mistake
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name,fn", MODULE_MUTATIONS, ids=[f.__name__ for _, f in MODULE_MUTATIONS])
def test_module_mutation_is_caught(monkeypatch, name, fn):
    monkeypatch.setattr(ro, name, fn)
    assert _failing_pins(), f"no pin catches {fn.__name__}"


@pytest.mark.parametrize("name,fn", SEQ_MUTATIONS, ids=[f.__name__ for _, f in SEQ_MUTATIONS])
def test_sequence_mutation_is_caught(monkeypatch, name, fn):
    monkeypatch.setattr(ro.ReplaySeq, name, fn)
    assert _failing_pins(), f"no pin catches {fn.__name__}"


def test_unmutated_oracle_passes_every_pin():
    assert _failing_pins() == []
