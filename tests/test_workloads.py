"""The seeded input recipe (workloads/gen.py) against what it promises: determinism per
(seed, stream, index), the stated distributions, and the prefill checkpoint equal to the
history form (from a zero state) over the very tokens it draws. CPU only."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import replay_oracle as ro
from workloads import gen

TINY = gen.Shape("w1", B=3, H=4, G=2, P=6, N=8, L=4, io="f32", seed=71)


def test_draws_repeat_per_index_and_differ_across_indices():
    a = gen.step_inputs(TINY, 5)
    b = gen.step_inputs(TINY, 5)
    c = gen.step_inputs(TINY, 6)
    for k in a:
        assert torch.equal(a[k], b[k]), k
        assert not torch.equal(a[k], c[k]), k
    v1 = gen.verify_inputs(TINY, 2, 3)
    assert torch.equal(v1["q"], gen.verify_inputs(TINY, 2, 3)["q"])
    assert not torch.equal(v1["q"], gen.verify_inputs(TINY, 3, 3)["q"])


def test_step_input_shapes_and_dtypes():
    for io, dt in (("f32", torch.float32), ("bf16", torch.bfloat16)):
        s = TINY.replace(io=io)
        x = gen.step_inputs(s, 0)
        assert x["q"].shape == (3, 2, 8) and x["k"].shape == (3, 2, 8) and x["v"].shape == (3, 4, 6)
        assert x["dt"].shape == (3, 4) and x["a"].shape == (3, 4)
        assert x["q"].dtype == dt and x["k"].dtype == dt and x["v"].dtype == dt
        assert x["dt"].dtype == torch.float32 and x["a"].dtype == torch.float32
        y = gen.verify_inputs(s, 0, 5)
        assert y["q"].shape == (3, 5, 2, 8) and y["v"].shape == (3, 5, 4, 6) and y["a"].shape == (3, 5, 4)


def test_queries_and_keys_are_unit_vectors():
    big = TINY.replace(B=64, N=128)
    x = gen.step_inputs(big, 1)
    for k in ("q", "k"):
        n = x[k].double().norm(dim=-1)
        assert torch.allclose(n, torch.ones_like(n), atol=1e-6), k
    xb = gen.step_inputs(big.replace(io="bf16"), 1)
    n = xb["q"].double().norm(dim=-1)
    assert torch.allclose(n, torch.ones_like(n), atol=1e-2)  # BF16 rounding of each element


def test_decay_is_one_rate_per_head_shared_by_the_batch():
    s = TINY.replace(B=32)
    rates = []
    for t in range(4):
        x = gen.step_inputs(s, t)
        dt, a = x["dt"].double(), x["a"].double()
        assert (dt > 0).all() and (a > 0).all() and (a < 1).all()
        rates.append(-torch.log(a) / dt)  # the head's A, one value per head
    r = torch.stack(rates)  # [steps, B, H]
    ref = r[0, 0]
    assert torch.allclose(r, ref.expand_as(r), rtol=1e-5)
    assert ((ref >= 0.5) & (ref <= 2.0)).all()
    assert torch.allclose(ref.float(), gen.head_decay_rates(s), rtol=1e-5)


def test_delta_is_softplus_of_a_standard_normal():
    s = TINY.replace(B=4096, H=8, G=8)
    dt = gen.step_inputs(s, 0)["dt"].double()
    z = torch.log(torch.expm1(dt))  # inverse softplus
    assert abs(float(z.mean())) < 0.03 and abs(float(z.std()) - 1.0) < 0.03


def test_accepted_lengths_cover_zero_to_draft():
    s = TINY.replace(B=4096)
    acc = gen.accepted_lengths(s, 0, 5)
    assert acc.dtype == torch.int32 and int(acc.min()) == 0 and int(acc.max()) == 4
    counts = torch.bincount(acc.long(), minlength=5).double() / acc.numel()
    assert torch.allclose(counts, torch.full_like(counts, 0.2), atol=0.03)


def test_gauss_checkpoint_spread():
    s = TINY.replace(B=64, P=32, N=32, s0="gauss")
    S0 = gen.initial_state(s)
    assert S0.shape == (64, 4, 32, 32) and S0.dtype == torch.float32
    assert abs(float(S0.std()) - 0.1) < 0.005 and abs(float(S0.mean())) < 0.005


@pytest.mark.parametrize("G", [4, 2], ids=["G=H", "G<H"])
def test_prefill_checkpoint_is_the_history_form_of_its_tokens(G):
    """The prefill state equals the history form from a zero state over the tail tokens
    it draws (Delta_j prod_{i>j} a_i weights), per sequence and head."""
    s = TINY.replace(G=G, s0="prefill")
    S0 = gen.initial_state(s).double().numpy()
    rates = gen.head_decay_rates(s)
    T = gen.PREFILL_TAIL
    g = gen._gen("cpu", s.seed, gen._STREAM_PREFILL, 0)  # one batch chunk covers B = 3
    q, k, v, dt, a = gen._draw_tokens(s, g, (s.B, T), "cpu", rates)
    hpg = s.H // s.G
    for b in range(s.B):
        kh = k[b].repeat_interleave(hpg, dim=1).double().numpy()  # [T, H, N]
        want = ro.history_state(np.zeros((s.H, s.P, s.N)), a[b].double().numpy(), dt[b].double().numpy(),
                                v[b].double().numpy(), kh)
        err = np.abs(S0[b] - want).max() / np.abs(want).max()
        assert err < 1e-5, (b, err)
