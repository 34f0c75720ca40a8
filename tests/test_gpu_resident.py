"""Zero-copy appends: the caller writes each token's k, v, Delta and a straight into its ring
record, at the slots replay_append_slots gives, and calls the resident step or verify,
which reads the entries from the ring. Outputs, flush flags and counts must equal those of
the copying calls bit for bit (the kernels read the same record bytes either way) and the
oracle's within the FP32 tolerance."""

import numpy as np
import pytest
import torch

import gpu_harness as hx
import linear_attention_decode_replay_b200 as lar
from linear_attention_decode_replay_b200 import _abi
from oracle import replay_oracle as ro
from workloads import gen

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


def _write_records(layer, slots, x, n_pos):
    """What a caller's projection epilogue would do: each entry's k into
    ring_k[b][g][(slots[b] + s) % cap] and its v, Delta, a (zero padding) into
    ring[b][h][(slots[b] + s) % cap]."""
    cfg = layer.cfg
    ring, ring_k = layer.buffers["ring"], layer.buffers["ring_k"]
    B, H, G, P, N = cfg.batch, cfg.heads, cfg.groups, cfg.P, cfg.N
    cap, R = ring.shape[2], ring.shape[3]
    s_io = 2 if cfg.io == "bf16" else 4
    bi = torch.arange(B, device=ring.device)[:, None]
    hi = torch.arange(H, device=ring.device)[None, :]
    gi = torch.arange(G, device=ring.device)[None, :]
    for s in range(n_pos):
        pick = (lambda t: t[:, s]) if x["k"].dim() == 4 else (lambda t: t)  # verify inputs carry n_pos
        k, v, dt, a = pick(x["k"]), pick(x["v"]), pick(x["dt"]), pick(x["a"])
        slot = ((slots.long() + s) % cap)[:, None]
        krec = torch.zeros(B, G, ring_k.shape[3], dtype=torch.uint8, device=ring.device)  # k, then padding
        krec[:, :, :N * s_io] = k.contiguous().view(torch.uint8).reshape(B, G, N * s_io)
        ring_k[bi, gi, slot] = krec
        rec = torch.zeros(B, H, R, dtype=torch.uint8, device=ring.device)
        rec[:, :, :P * s_io] = v.contiguous().view(torch.uint8).reshape(B, H, P * s_io)
        rec[:, :, P * s_io:P * s_io + 8] = torch.stack([dt, a], -1).contiguous().view(torch.uint8).reshape(B, H, 8)
        ring[bi, hi, slot] = rec


SHAPES = [
    gen.Shape("z1", B=3, H=4, G=2, P=24, N=32, L=5, io="f32", max_pos=3, seed=61),
    gen.Shape("z2", B=2, H=2, G=1, P=64, N=128, L=4, io="bf16", max_pos=4, seed=62),
    gen.Shape("z3", B=2, H=2, G=2, P=32, N=64, L=6, io="bf16", ckpt="f32_fp8read", max_pos=2, seed=63),
    gen.Shape("z4", B=2, H=8, G=2, P=16, N=32, L=4, io="bf16", ckpt="f32_fp4read", max_pos=2, seed=64),
]


@pytest.mark.parametrize("shape", SHAPES, ids=[s.name for s in SHAPES])
def test_resident_decode_equals_copying_decode(shape):
    _, _, copy, S0 = hx.setup(shape)
    _, _, res, _ = hx.setup(shape)
    oracle = ro.ReplayBatch(gen.to_numpy64(S0), shape.G, shape.L, ckpt=shape.ckpt)
    fl_c = torch.zeros(shape.B, dtype=torch.uint8, device="cuda")
    fl_r = torch.zeros_like(fl_c)
    for t in range(3 * shape.L + 2):
        x = gen.step_inputs(shape, t, device="cuda")
        y_c = copy.step(x["q"], x["k"], x["v"], x["dt"], x["a"], flushed=fl_c)
        slots = res.append_slots()
        _write_records(res, slots, x, 1)
        y_r = res.step_resident(x["q"], flushed=fl_r)
        xs = {k: gen.to_numpy64(v) for k, v in x.items()}
        y_o, f_o = oracle.step(xs["q"], xs["k"], xs["v"], xs["dt"], xs["a"])
        assert torch.equal(y_r, y_c), t
        assert torch.equal(fl_r, fl_c) and np.array_equal(fl_r.cpu().numpy(), f_o), t
        tol = hx.TOL_F32 if shape.ckpt == "f32" else 1e-3  # a read copy: against the oracle's emulation
        assert ro.relative_error(gen.to_numpy64(y_r), y_o) <= tol, t
    assert res.read_counts() == copy.read_counts() == list(oracle.counts)
    assert res.check_status() == 0 and copy.check_status() == 0
    res.close()
    copy.close()


@pytest.mark.parametrize("shape", SHAPES[:2], ids=[s.name for s in SHAPES[:2]])
def test_resident_verify_equals_copying_verify(shape):
    _, _, copy, S0 = hx.setup(shape)
    _, _, res, _ = hx.setup(shape)
    oracle = ro.ReplayBatch(gen.to_numpy64(S0), shape.G, shape.L)
    n_pos = shape.max_pos
    for rnd in range(2 * shape.L):
        x = gen.verify_inputs(shape, rnd, n_pos, device="cuda")
        y_c = copy.verify(x["q"], x["k"], x["v"], x["dt"], x["a"])
        slots = res.append_slots()
        _write_records(res, slots, x, n_pos)
        y_r = res.verify_resident(x["q"])
        with pytest.raises(lar.ReplayError) as e:  # slots are asked for between calls only
            res.append_slots()
        assert e.value.code == _abi.REPLAY_EPENDING
        assert torch.equal(y_r, y_c), rnd
        xs = {k: gen.to_numpy64(v) for k, v in x.items()}
        y_o, _ = oracle.verify(xs["q"], xs["k"], xs["v"], xs["dt"], xs["a"])
        assert ro.relative_error(gen.to_numpy64(y_r), y_o) <= hx.TOL_F32, rnd
        n_keep = (gen.accepted_lengths(shape, rnd, n_pos, device="cuda") + 1).to(torch.int32)
        copy.rollback(n_keep)
        res.rollback(n_keep)
        oracle.rollback(n_keep.cpu().numpy())
        assert res.read_counts() == copy.read_counts() == list(oracle.counts), rnd
    assert res.check_status() == 0 and copy.check_status() == 0
    res.close()
    copy.close()
