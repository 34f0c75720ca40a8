"""Pins of the CPU oracle: checks against what the ReplaySSM pages and the mathematics
fix, never against the oracle's own formulas retyped.

Each ``pin_*`` function raises AssertionError (or any exception) when the oracle is
wrong. ``test_oracle_pins.py`` runs them one by one; ``test_oracle_mutations.py``
plants mistakes into the oracle and requires that some pin fails for each.
All oracle calls go through the module object so that planted mistakes take effect.
"""

from __future__ import annotations

import math
import os

import numpy as np
import torch

from oracle import replay_oracle as ro
from workloads import gen

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read_fixture(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                key, *vals = line.split()
                rows[key] = vals
    return rows


def _rng(seed):
    return np.random.default_rng(seed)


def _rand_tokens(rng, T, H, G, P, N):
    q = rng.standard_normal((T, G, N))
    k = rng.standard_normal((T, G, N))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, P))
    dt = np.log1p(np.exp(rng.standard_normal((T, H))))
    a = np.exp(-dt * rng.uniform(0.5, 2.0, H))
    return q, k, v, dt, a


def _eager_outputs(S0, q, k, v, dt, a, G):
    """Outputs of the summary recurrence for one sequence over T tokens."""
    H = S0.shape[0]
    gh = np.arange(H) // (H // G)
    S, ys = S0.copy(), []
    for t in range(len(q)):
        S, y = ro.eager_step(S, a[t], dt[t], v[t], k[t][gh], q[t][gh])
        ys.append(y)
    return S, np.stack(ys)


# ---------------------------------------------------------------- worked example

def pin_hand_example():
    """The hand-worked example (tests/golden/hand_example.txt) holds exactly."""
    fx = {k: np.array([float(x) for x in v]) for k, v in _read_fixture("hand_example.txt").items()}
    S0 = fx["S0"].reshape(1, 2, 2)
    S = S0.copy()
    seq = ro.ReplaySeq(S0, G=1, L=2)
    for t in range(3):
        a = fx["a"][t:t + 1]
        dt = fx["dt"][t:t + 1]
        v = fx[f"v{t + 1}"].reshape(1, 2)
        k = fx[f"k{t + 1}"].reshape(1, 2)
        q = fx[f"q{t + 1}"].reshape(1, 2)
        S, y = ro.eager_step(S, a, dt, v, k, q)
        assert np.array_equal(y[0], fx[f"y{t + 1}"]), ("eager", t, y, fx[f"y{t + 1}"])
        yr, flushed = seq.step(q, k, v, dt, a)
        assert np.array_equal(yr[0], fx[f"y{t + 1}"]), ("replay", t, yr, fx[f"y{t + 1}"])
        assert flushed == (t == 2)
    assert np.array_equal(S[0].ravel(), fx["S3"])
    assert np.array_equal(seq.S0[0].ravel(), fx["S2"]) and seq.count == 1


# ---------------------------------------------------------------- two forms, two routes

def pin_eager_equals_history():
    """Summary form iterated T times equals the history form (blog: both forms give
    the same result), from a non-zero initial state, P != N."""
    rng = _rng(1)
    H, G, P, N, T = 3, 3, 5, 7, 9
    S0 = rng.standard_normal((H, P, N))
    q, k, v, dt, a = _rand_tokens(rng, T, H, G, P, N)
    S_eager, _ = _eager_outputs(S0, q, k, v, dt, a, G)
    S_hist = ro.history_state(S0, a, dt, v, k)
    assert np.max(np.abs(S_eager - S_hist)) < 1e-12 * max(1.0, np.max(np.abs(S_hist)))


def pin_history_from_zero():
    """History form from a zero state, checked term by term on a 2-token case:
    S_2 = Delta_1 a_2 v_1 k_1^T + Delta_2 v_2 k_2^T."""
    rng = _rng(2)
    H, P, N = 2, 3, 4
    _, k, v, dt, a = _rand_tokens(rng, 2, H, H, P, N)
    S = ro.history_state(np.zeros((H, P, N)), a, dt, v, k)
    for h in range(H):
        want = dt[0, h] * a[1, h] * np.outer(v[0, h], k[0, h]) + dt[1, h] * np.outer(v[1, h], k[1, h])
        assert np.allclose(S[h], want, rtol=0, atol=1e-14)


def pin_routes_agree():
    """Output-only route y = abar (S0 q) + sum_j s_j v_j (k_j^T q) equals the state
    route's S_t applied to q (matrix-vector product distributes over the sum)."""
    rng = _rng(3)
    H, P, N, T = 4, 6, 5, 7
    S0 = rng.standard_normal((H, P, N))
    q, k, v, dt, a = _rand_tokens(rng, T, H, H, P, N)
    abar, s = ro.decay_weights(a, dt)
    S_t = ro.state_route(S0, abar, s, v, k)
    y_state = np.stack([S_t[h] @ q[-1, h] for h in range(H)])
    y_out = ro.output_only(S0, abar, s, v, k, q[-1])
    assert np.max(np.abs(y_state - y_out)) < 1e-12


def pin_state_route_is_history():
    """The state route over the buffer equals the history form started from S0."""
    rng = _rng(4)
    H, P, N, T = 2, 4, 3, 6
    S0 = rng.standard_normal((H, P, N))
    _, k, v, dt, a = _rand_tokens(rng, T, H, H, P, N)
    abar, s = ro.decay_weights(a, dt)
    assert np.max(np.abs(ro.state_route(S0, abar, s, v, k) - ro.history_state(S0, a, dt, v, k))) < 1e-12


# ---------------------------------------------------------------- replay == eager

def _replay_vs_eager(shape, steps):
    """Replay decode of the seeded workload compared with eager decode every step."""
    S0 = gen.to_numpy64(gen.initial_state(shape))
    batch = ro.ReplayBatch(S0, shape.G, shape.L)
    S = S0.copy()
    worst = 0.0
    flush_steps = []
    for t in range(steps):
        x = {k: gen.to_numpy64(v) for k, v in gen.step_inputs(shape, t).items()}
        y_r, fl = batch.step(x["q"], x["k"], x["v"], x["dt"], x["a"])
        S, y_e = ro.eager_batch_step(S, x["q"], x["k"], x["v"], x["dt"], x["a"], shape.G)
        worst = max(worst, float(np.max(np.abs(y_r - y_e))) / max(1.0, float(np.max(np.abs(y_e)))))
        flush_steps.append(fl.copy())
    return worst, np.array(flush_steps), batch, S


def pin_replay_equals_eager_tiny():
    """Tiny workload (B=2, H=2, P=N=16, L=4, FP32, 32 steps): replay output equals the
    eager output at every step (blog conclusion: the results do not change), and the
    flush comes exactly when a step meets a full buffer (steps 4, 8, ... 0-based)."""
    shape = gen.SHAPES["tiny"]
    worst, fl, batch, S = _replay_vs_eager(shape, shape.steps)
    assert worst < 1e-12, worst
    expect = np.array([[t >= shape.L and t % shape.L == 0] * shape.B for t in range(shape.steps)])
    assert np.array_equal(fl.astype(bool), expect)
    batch.flush()
    assert np.max(np.abs(batch.checkpoints() - S)) < 1e-12


def pin_replay_equals_eager_groups():
    """Same with k/q shared by head groups (G=2 < H=4) and P != N."""
    shape = gen.Shape("grp", B=2, H=4, G=2, P=8, N=12, L=3, io="f32", steps=14, seed=7)
    worst, _, batch, S = _replay_vs_eager(shape, shape.steps)
    assert worst < 1e-12, worst
    batch.flush()
    assert np.max(np.abs(batch.checkpoints() - S)) < 1e-12


def pin_window_one_is_eager():
    """L = 1: every step folds the previous token, so replay is eager step by step and
    the checkpoint always holds the state before the newest token."""
    shape = gen.Shape("l1", B=1, H=2, G=1, P=4, N=4, L=1, io="f32", steps=6, seed=8)
    worst, fl, batch, S = _replay_vs_eager(shape, shape.steps)
    assert worst < 1e-12
    assert fl[1:].all() and not fl[0].any()


# ---------------------------------------------------------------- special cases

def pin_unit_decay_is_linear_attention():
    """a = 1, Delta = 1: the recurrence is plain unnormalised linear attention,
    y_t = (S0 + V_{1..t}^T K_{1..t}) q_t, evaluated here with one matrix product of the
    stacked token matrices."""
    rng = _rng(5)
    H, P, N, T, L = 1, 3, 5, 9, 4
    S0 = rng.standard_normal((H, P, N))
    q, k, v, _, _ = _rand_tokens(rng, T, H, H, P, N)
    ones = np.ones((1,))
    seq = ro.ReplaySeq(S0, G=1, L=L)
    for t in range(T):
        y, _ = seq.step(q[t], k[t], v[t], ones, ones)
        Vt = v[:t + 1, 0, :]  # [t+1, P]
        Kt = k[:t + 1, 0, :]  # [t+1, N]
        want = (S0[0] + Vt.T @ Kt) @ q[t, 0]
        assert np.max(np.abs(y[0] - want)) < 1e-12


def pin_zero_decay_forgets():
    """a = 0: S_t = Delta_t v_t k_t^T, so y_t = Delta_t v_t (k_t . q_t) whatever came before."""
    rng = _rng(6)
    H, P, N, T, L = 2, 4, 3, 7, 3
    S0 = rng.standard_normal((H, P, N))
    q, k, v, dt, _ = _rand_tokens(rng, T, H, H, P, N)
    seq = ro.ReplaySeq(S0, G=H, L=L)
    for t in range(T):
        y, _ = seq.step(q[t], k[t], v[t], dt[t], np.zeros(H))
        for h in range(H):
            assert np.max(np.abs(y[h] - dt[t, h] * v[t, h] * np.dot(k[t, h], q[t, h]))) < 1e-14


def pin_geometric_closed_form():
    """a = rho, Delta = 1, v = k = q = e_0, S0 = c e_0 e_0^T: the state's corner is the
    geometric series S_t = rho^t c + (1 - rho^t) / (1 - rho); checked through several
    flushes (L = 3) on both the replay and the eager path."""
    rho, c, T, L = 0.75, 2.0, 11, 3
    e0 = np.zeros((1, 2))
    e0[0, 0] = 1.0
    S0 = c * np.einsum("hp,hn->hpn", e0, e0)
    seq = ro.ReplaySeq(S0, G=1, L=L)
    S = S0.copy()
    for t in range(1, T + 1):
        want = rho ** t * c + (1 - rho ** t) / (1 - rho)
        y, _ = seq.step(e0, e0, e0, np.ones(1), np.full(1, rho))
        S, ye = ro.eager_step(S, np.full(1, rho), np.ones(1), e0, e0, e0)
        assert abs(y[0, 0] - want) < 1e-13 and abs(ye[0, 0] - want) < 1e-13, (t, y, want)


# ---------------------------------------------------------------- verify / rollback

def pin_verify_positions_are_eager_prefixes():
    """Verify at position s equals the eager state after the committed tokens and the
    drafts 0..s, applied to q_s (blog "Paralelismo": causal mask over the window)."""
    rng = _rng(9)
    H, G, P, N, L = 2, 1, 4, 5, 6
    S0 = rng.standard_normal((H, P, N))
    seq = ro.ReplaySeq(S0, G=G, L=L)
    S = S0.copy()
    gh = np.zeros(H, dtype=int)
    q, k, v, dt, a = _rand_tokens(rng, 3, H, G, P, N)
    for t in range(3):
        seq.step(q[t], k[t], v[t], dt[t], a[t])
        S, _ = ro.eager_step(S, a[t], dt[t], v[t], k[t][gh], q[t][gh])
    n = 4  # 3 committed + 4 > 6: the verify also folds first
    qd, kd, vd, dd, ad = _rand_tokens(rng, n, H, G, P, N)
    ys, flushed = seq.verify(qd, kd, vd, dd, ad)
    assert flushed
    Sd = S.copy()
    for s in range(n):
        Sd, ye = ro.eager_step(Sd, ad[s], dd[s], vd[s], kd[s][gh], qd[s][gh])
        assert np.max(np.abs(ys[s] - ye)) < 1e-12


def pin_rollback_equals_never_seen():
    """Rolling back to n_keep drafts equals never having seen the rejected ones
    (blog "Rollback (deshacer)"; abstract: rollback is a buffer-pointer operation)."""
    rng = _rng(10)
    H, G, P, N, L, n = 2, 2, 3, 4, 8, 5
    S0 = rng.standard_normal((H, P, N))
    for n_keep in range(n + 1):
        spec = ro.ReplaySeq(S0, G=G, L=L)
        plain = ro.ReplaySeq(S0, G=G, L=L)
        r = _rng(100 + n_keep)
        q0, k0, v0, d0, a0 = _rand_tokens(r, 2, H, G, P, N)
        for t in range(2):
            spec.step(q0[t], k0[t], v0[t], d0[t], a0[t])
            plain.step(q0[t], k0[t], v0[t], d0[t], a0[t])
        qd, kd, vd, dd, ad = _rand_tokens(r, n, H, G, P, N)
        spec.verify(qd, kd, vd, dd, ad)
        spec.rollback(n_keep)
        for s in range(n_keep):
            plain.step(qd[s], kd[s], vd[s], dd[s], ad[s])
        assert spec.count == plain.count
        q1, k1, v1, d1, a1 = _rand_tokens(r, 9, H, G, P, N)
        for t in range(9):
            ys, fs = spec.step(q1[t], k1[t], v1[t], d1[t], a1[t])
            yp, fp = plain.step(q1[t], k1[t], v1[t], d1[t], a1[t])
            assert fs == fp and np.max(np.abs(ys - yp)) < 1e-12
        spec.fold()
        plain.fold()
        assert np.max(np.abs(spec.S0 - plain.S0)) < 1e-12


# ---------------------------------------------------------------- page ratios

def pin_route_flop_ratio():
    """Inner vs outer product route at d = n = 128: about 64x (blog, "Ruta solo salida")."""
    P, N, ratio = (int(x) for x in _read_fixture("page_ratios.txt")["route_flops"])
    f = ro.route_flops(P, N, 16)
    assert f["outer"] / f["inner"] == ratio


def pin_one_flush_write_per_window():
    """One state write per window of L tokens instead of L (video page takeaways), and
    eager/replay state traffic in the 'roughly halves' band (abstract) at L = 16."""
    fx = _read_fixture("page_ratios.txt")
    L, eager_w, replay_w = (int(x) for x in fx["flush_writes"])
    Lt, lo, hi = int(fx["state_traffic"][0]), float(fx["state_traffic"][1]), float(fx["state_traffic"][2])
    assert L == Lt
    windows = 4
    rng = _rng(11)
    H, P, N = 1, 2, 3
    seq = ro.ReplaySeq(rng.standard_normal((H, P, N)), G=1, L=L)
    q, k, v, dt, a = _rand_tokens(rng, (windows + 1) * L, H, 1, P, N)
    # steady state: count over the windows after the first one
    for t in range(L):
        seq.step(q[t], k[t], v[t], dt[t], a[t])
    r0, w0 = seq.state_reads, seq.state_writes
    for t in range(L, (windows + 1) * L):
        seq.step(q[t], k[t], v[t], dt[t], a[t])
    reads, writes = seq.state_reads - r0, seq.state_writes - w0
    assert writes == windows * replay_w
    eager_traffic = 2 * windows * L  # eager reads and writes the state every token
    assert eager_w == L
    ratio = eager_traffic / (reads + writes)
    assert lo <= ratio <= hi, ratio
    assert abs(ratio - 2 * L / (L + 1)) < 1e-12


# ---------------------------------------------------------------- FP8 e4m3

def pin_e4m3_table():
    """Decoded values of selected codes match the OCP E4M3 table (golden fixture)."""
    for code, val in _read_fixture("e4m3_table.txt").items():
        got = ro.e4m3_decode(np.array([int(code, 16)], dtype=np.uint8))[0]
        if val[0] == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val[0]) and math.copysign(1, got) == math.copysign(1, float(val[0]))


def pin_e4m3_all_codes():
    """All 256 codes: 254 finite, strictly increasing over the positive codes 0..126,
    symmetric in sign, largest 448; each finite code encodes back to itself."""
    codes = np.arange(256, dtype=np.uint8)
    vals = ro.e4m3_decode(codes)
    assert np.isnan(vals).sum() == 2
    pos = vals[:127]
    assert np.all(np.diff(pos) > 0) and pos[-1] == 448.0
    assert np.array_equal(np.abs(vals[128:255]), pos)
    back = ro.e4m3_encode(vals[:127])
    assert np.array_equal(back, codes[:127])
    back_neg = ro.e4m3_encode(vals[129:255])
    assert np.array_equal(back_neg, codes[129:255])


def pin_e4m3_matches_torch():
    """Round-to-nearest-even encoding agrees bit for bit with torch's float8_e4m3fn
    conversion (a library routine) on every in-range FP32 value of a dense sweep:
    all exact midpoints between neighbouring codes, subnormals, and random values."""
    codes = np.arange(127, dtype=np.uint8)
    vals = ro.e4m3_decode(codes)
    mids = (vals[:-1] + vals[1:]) / 2
    rng = _rng(12)
    rand = np.concatenate([rng.uniform(0, 448, 20000), np.exp2(rng.uniform(-12, 8.8, 20000))])
    x = np.concatenate([vals, mids, rand, np.nextafter(mids, 0), np.nextafter(mids, 1000)])
    x = x[np.abs(x) <= 448].astype(np.float32)
    x = np.concatenate([x, -x])
    ours = ro.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref), np.flatnonzero(ours != ref)[:5]


def pin_e4m3_saturates_and_ties():
    """Saturation to +-448 beyond the largest finite value; ties go to the even code."""
    sat = ro.e4m3_encode(np.array([449.0, 464.0, 500.0, 1e9, -1e9, -470.0]))
    assert list(sat) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    ties = ro.e4m3_encode(np.array([1.0625, 1.1875, 2 ** -10, 3 * 2 ** -10]))
    assert list(ties) == [0x38, 0x3A, 0x00, 0x02]


def pin_row_quantiser():
    """Per-row scale: the row's largest magnitude maps to 448 (code 0x7E); an all-zero
    row has scale 1 and zero codes; dequantised values lie within half a code spacing."""
    rng = _rng(13)
    S = rng.standard_normal((5, 64)) * np.array([[1e-3], [1.0], [30.0], [0.0], [2.5]])
    codes, scale = ro.quantize_rows_e4m3(S)
    assert scale.dtype == np.float32 and codes.dtype == np.uint8
    assert np.all((codes[3] & 0x7F) == 0) and scale[3] == 1.0
    for r in (0, 1, 2, 4):
        amax = np.max(np.abs(S[r].astype(np.float32)))
        assert scale[r] == np.float32(amax) / np.float32(448)
        assert (codes[r] & 0x7F).max() == 0x7E
    deq = ro.dequantize_rows_e4m3(codes, scale)
    x = S.astype(np.float32).astype(np.float64)
    # normal range: relative error <= 2^-4; subnormal range: absolute <= 2^-10 * scale
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * scale[:, None]) * (1 + 1e-6)
    assert np.all(np.abs(deq - x) <= bound)


def pin_dual_precision_master_is_exact():
    """Dual precision: the FP8 copy serves outputs but its rounding never enters the
    updates (abstract), so the master after flushes is identical to the FP32-only run,
    while the shared-FP8 eager state drifts away from the exact state."""
    shape = gen.Shape("dp", B=1, H=2, G=2, P=8, N=16, L=4, io="f32", steps=13, seed=14)
    S0 = gen.to_numpy64(gen.initial_state(shape))
    exact = ro.ReplayBatch(S0, shape.G, shape.L, ckpt="f32")
    dual = ro.ReplayBatch(S0, shape.G, shape.L, ckpt="f32_fp8read")
    codes, scale = ro.quantize_rows_e4m3(S0)
    S = S0.copy()
    err_dual, err_shared = 0.0, 0.0
    for t in range(shape.steps):
        x = {k: gen.to_numpy64(v) for k, v in gen.step_inputs(shape, t).items()}
        y_e, _ = exact.step(x["q"], x["k"], x["v"], x["dt"], x["a"])
        y_d, _ = dual.step(x["q"], x["k"], x["v"], x["dt"], x["a"])
        codes, scale, y_s = ro.eager_fp8_batch_step(codes, scale, x["q"], x["k"], x["v"], x["dt"], x["a"], shape.G)
        S, _ = ro.eager_batch_step(S, x["q"], x["k"], x["v"], x["dt"], x["a"], shape.G)
        err_dual = max(err_dual, ro.relative_error(y_d, y_e))
        err_shared = max(err_shared, ro.relative_error(y_s, y_e))
    exact.flush()
    dual.flush()
    assert np.array_equal(exact.checkpoints(), dual.checkpoints())
    assert 0 < err_dual < 0.1 and err_shared > 0
    deq = ro.dequantize_rows_e4m3(codes, scale)
    assert np.max(np.abs(deq - S)) > 0


def _fp8_fixture():
    rows = _read_fixture("fp8_hand_example.txt")
    codes = {k: np.array([int(x, 16) for x in v], dtype=np.uint8) for k, v in rows.items() if "codes" in k}
    vals = {k: np.array([float(x) for x in v]) for k, v in rows.items() if "codes" not in k}
    return codes, vals


def pin_shared_fp8_hand_example():
    """Shared-FP8 eager step worked by hand from the OCP table (fixture, example A): the
    initial codes, the output taken from the updated values before re-quantising, and
    the re-quantised codes and scale."""
    codes, fx = _fp8_fixture()
    S = fx["A_S"].reshape(1, 1, 1, 4)
    c0, s0 = ro.quantize_rows_e4m3(S)
    assert np.array_equal(c0.ravel(), codes["A_codes0"]) and s0.ravel()[0] == fx["A_scale"][0]
    one = lambda x: np.asarray(x, np.float64).reshape(1, 1, -1)  # noqa: E731 - [B=1][H or G=1][...]
    c1, s1, y = ro.eager_fp8_batch_step(c0, s0, one(fx["A_q"]), one(fx["A_k"]), one(fx["A_v"]),
                                        fx["A_dt"].reshape(1, 1), fx["A_a"].reshape(1, 1), 1)
    assert abs(y.ravel()[0] - fx["A_y"][0]) < 1e-12, y
    assert np.array_equal(c1.ravel(), codes["A_codes1"]), [hex(x) for x in c1.ravel()]
    assert s1.ravel()[0] == fx["A_scale"][0]


def pin_dual_precision_hand_example():
    """Dual precision with L = 1 (fixture, example B): a step that does not flush reads
    the FP8 copy, the step that flushes reads the fresh master."""
    codes, fx = _fp8_fixture()
    seq = ro.ReplaySeq(fx["B_S0"].reshape(1, 1, 4), G=1, L=1, ckpt="f32_fp8read")
    assert np.array_equal(seq.codes.ravel(), codes["B_codes"])
    q = fx["B_q"].reshape(1, 4)
    zero_k, zero_v, one, zero = np.zeros((1, 4)), np.zeros((1, 1)), np.ones(1), np.zeros(1)
    y0, f0 = seq.step(q, zero_k, zero_v, zero, one)
    y1, f1 = seq.step(q, zero_k, zero_v, zero, one)
    assert not f0 and f1
    assert y0.ravel()[0] == fx["B_y0"][0], y0
    assert abs(y1.ravel()[0] - fx["B_y1"][0]) < 1e-12, y1


def pin_dual_precision_fp4_hand_example():
    """The same split with the FP4 e2m1 copy (fixture, example C): codes worked by hand,
    the copy read by a step without a flush, the master by the flushing step."""
    codes, fx = _fp8_fixture()
    seq = ro.ReplaySeq(fx["C_S0"].reshape(1, 1, 4), G=1, L=1, ckpt="f32_fp4read")
    assert np.array_equal(seq.codes.ravel(), codes["C_codes"]) and seq.scale.ravel()[0] == 1.0
    q = fx["C_q"].reshape(1, 4)
    zero_k, zero_v, one, zero = np.zeros((1, 4)), np.zeros((1, 1)), np.ones(1), np.zeros(1)
    y0, f0 = seq.step(q, zero_k, zero_v, zero, one)
    y1, f1 = seq.step(q, zero_k, zero_v, zero, one)
    assert not f0 and f1
    assert y0.ravel()[0] == fx["C_y0"][0], y0
    assert abs(y1.ravel()[0] - fx["C_y1"][0]) < 1e-12, y1


def pin_e2m1_table():
    """Every e2m1 code decodes to the OCP MX table value (golden fixture) and encodes
    back to itself (the two zeros to themselves)."""
    rows = _read_fixture("e2m1_table.txt")
    assert len(rows) == 16
    for code, val in rows.items():
        c = int(code, 16)
        got = ro.e2m1_decode(np.array([c], dtype=np.uint8))[0]
        assert got == float(val[0]) and math.copysign(1, got) == math.copysign(1, float(val[0])), code
        assert ro.e2m1_encode(np.array([float(val[0])]))[0] == c, code


def pin_e2m1_nearest_by_brute_force():
    """Encoding = the nearest of the 16 table values by exhaustive search (ties to the
    code with the even mantissa bit, beyond +-6 to +-6), over a dense sweep with every
    midpoint and its neighbours."""
    table = {int(k, 16): float(v[0]) for k, v in _read_fixture("e2m1_table.txt").items()}
    pos = sorted((v, c) for c, v in table.items() if c < 8)
    mids = [(pos[i][0] + pos[i + 1][0]) / 2 for i in range(7)]
    rng = _rng(15)
    x = np.concatenate([rng.uniform(-8, 8, 4000), np.array(mids), -np.array(mids), np.nextafter(mids, 0),
                        np.nextafter(mids, 10), [6.0, 6.5, 7.9, 100.0, -7.0, 0.0]])

    def brute(xi):
        m = min(abs(xi), 6.0)
        best = min(pos, key=lambda vc: (abs(vc[0] - m), vc[1] & 1))  # nearest, then even mantissa
        return best[1] | (8 if math.copysign(1, xi) < 0 else 0)

    want = np.array([brute(xi) for xi in x], dtype=np.uint8)
    assert np.array_equal(ro.e2m1_encode(x), want), np.flatnonzero(ro.e2m1_encode(x) != want)[:5]


def pin_row_quantiser_e2m1():
    """Per-row FP4 scale: the row's largest magnitude maps to 6 (code 0x7); an all-zero
    row has scale 1 and zero codes; dequantised values lie within half a code spacing."""
    rng = _rng(16)
    S = rng.standard_normal((5, 32)) * np.array([[1e-3], [1.0], [30.0], [0.0], [2.5]])
    codes, scale = ro.quantize_rows_e2m1(S)
    assert scale.dtype == np.float32 and codes.dtype == np.uint8 and codes.max() <= 0xF
    assert np.all((codes[3] & 0x7) == 0) and scale[3] == 1.0
    for r in (0, 1, 2, 4):
        amax = np.max(np.abs(S[r].astype(np.float32)))
        assert scale[r] == np.float32(amax) / np.float32(6)
        assert (codes[r] & 0x7).max() == 0x7
    deq = ro.dequantize_rows_e2m1(codes, scale)
    x = S.astype(np.float32).astype(np.float64)
    # normal range (|x| >= scale): relative error <= 2^-2; below it: absolute <= 0.25 * scale
    bound = np.maximum(np.abs(x) * 0.25, 0.25 * scale[:, None]) * (1 + 1e-6)
    assert np.all(np.abs(deq - x) <= bound)


def pin_relative_error_metric():
    """The error metric is the max over vectors of the relative L2 error."""
    y_ref = np.array([[3.0, 4.0], [0.0, 1.0]])
    y = np.array([[3.0, 4.5], [0.0, 1.0]])
    assert abs(ro.relative_error(y, y_ref) - 0.1) < 1e-15
    assert ro.relative_error(y_ref, y_ref) == 0.0


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
