"""Snapshot export and import of single sequences: a layer that decoded to the middle of a
window exports two sequences, a fresh layer (another batch size and state) imports them
at other positions, and both continue on the same inputs for those sequences: outputs,
flush flags and counts bit-identical to the uninterrupted run, and equal to the oracle's
continuation. Snapshots that do not match a layer are refused with a status bit."""

import numpy as np
import pytest
import torch

import gpu_harness as hx
import linear_attention_decode_replay_b200 as lar
from oracle import replay_oracle as ro
from workloads import gen

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

SHAPES = [
    gen.Shape("sn1", B=4, H=4, G=2, P=24, N=32, L=5, io="f32", seed=71),
    gen.Shape("sn2", B=3, H=2, G=2, P=64, N=128, L=6, io="bf16", ckpt="f32_fp8read", seed=72),
    gen.Shape("sn3", B=3, H=2, G=1, P=256, N=64, L=4, io="bf16", seed=73),  # two row blocks per head
    gen.Shape("sn4", B=3, H=8, G=2, P=32, N=64, L=5, io="bf16", ckpt="f32_fp4read", seed=74),
]


@pytest.mark.parametrize("shape", SHAPES, ids=[s.name for s in SHAPES])
def test_export_import_continues_bit_identically(shape):
    _, bufs_a, A, S0 = hx.setup(shape)
    seqs_a = torch.tensor([shape.B - 1, 0], dtype=torch.int32, device="cuda")
    rows = seqs_a.cpu().numpy()
    oracle = ro.ReplayBatch(gen.to_numpy64(S0)[rows], shape.G, shape.L, ckpt=shape.ckpt)
    before = 2 * shape.L + 2  # two flushes, then two buffered entries
    for t in range(before):
        x = gen.step_inputs(shape, t, device="cuda")
        A.step(x["q"], x["k"], x["v"], x["dt"], x["a"])
        xs = {k: gen.to_numpy64(v)[rows] for k, v in x.items()}
        oracle.step(xs["q"], xs["k"], xs["v"], xs["dt"], xs["a"])
    snap = A.export(seqs_a)
    hdr = snap[:, :64].view(torch.int32).cpu().numpy()
    assert (hdr[:, 0] == 0x4E535052).all() and list(hdr[:, 1]) == [2, 2]
    cfg = hx.lar_config(shape)
    assert list(hdr[0, 2:9]) == [shape.H, shape.P, shape.N, shape.L, lar.ring_record_bytes(cfg), shape.G,
                                 lar.ring_k_record_bytes(cfg)]

    shape_b = shape.replace(B=shape.B + 1, seed=shape.seed + 100)  # other batch size, other state
    _, bufs_b, Bl, _ = hx.setup(shape_b)
    for t in range(3):  # some history of its own first
        x = gen.step_inputs(shape_b, 50 + t, device="cuda")
        Bl.step(x["q"], x["k"], x["v"], x["dt"], x["a"])
    seqs_b = torch.tensor([1, shape_b.B - 1], dtype=torch.int32, device="cuda")
    Bl.import_(seqs_b, snap)
    counts_b = Bl.read_counts()
    assert [counts_b[i] for i in seqs_b.tolist()] == [2, 2]

    fl_a = torch.zeros(shape.B, dtype=torch.uint8, device="cuda")
    fl_b = torch.zeros(shape_b.B, dtype=torch.uint8, device="cuda")
    ia, ib = seqs_a.long(), seqs_b.long()
    for t in range(before, before + shape.L + 3):
        xa = gen.step_inputs(shape, t, device="cuda")
        xb = gen.step_inputs(shape_b, t, device="cuda")
        for key in xb:
            xb[key][ib] = xa[key][ia]
        ya = A.step(xa["q"], xa["k"], xa["v"], xa["dt"], xa["a"], flushed=fl_a)
        yb = Bl.step(xb["q"], xb["k"], xb["v"], xb["dt"], xb["a"], flushed=fl_b)
        assert torch.equal(yb[ib], ya[ia]), t
        assert torch.equal(fl_b[ib], fl_a[ia]), t
        xs = {k: gen.to_numpy64(v)[rows] for k, v in xa.items()}
        y_o, f_o = oracle.step(xs["q"], xs["k"], xs["v"], xs["dt"], xs["a"])
        tol = hx.TOL_F32 if shape.ckpt == "f32" else 1e-3  # a read copy: against the oracle's emulation
        assert ro.relative_error(gen.to_numpy64(yb[ib]), y_o) <= tol, t
        assert np.array_equal(fl_b[ib].cpu().numpy(), f_o), t
    counts_a, counts_b = A.read_counts(), Bl.read_counts()
    assert [counts_b[i] for i in seqs_b.tolist()] == [counts_a[i] for i in seqs_a.tolist()] == list(oracle.counts)
    A.flush()
    Bl.flush()
    oracle.flush()
    assert torch.equal(bufs_b["S0"][ib], bufs_a["S0"][ia])
    assert ro.relative_error(gen.to_numpy64(bufs_b["S0"][ib]), oracle.checkpoints()) <= hx.TOL_F32
    assert A.check_status() == 0 and Bl.check_status() == 0
    A.close()
    Bl.close()


def test_snapshot_mismatch_and_bad_ids_are_refused():
    shape = SHAPES[0]
    _, _, A, _ = hx.setup(shape)
    for t in range(3):
        x = gen.step_inputs(shape, t, device="cuda")
        A.step(x["q"], x["k"], x["v"], x["dt"], x["a"])
    snap = A.export(torch.tensor([0], dtype=torch.int32, device="cuda"))
    # a layer with another window has another snapshot size; a header naming other sizes is refused
    other = shape.replace(L=shape.L + 1)
    _, bufs_c, C, _ = hx.setup(other)
    nb = lar.snapshot_bytes(hx.lar_config(other))
    forged = torch.zeros(1, nb, dtype=torch.uint8, device="cuda")
    forged[:, :snap.shape[1]] = snap[:, :min(nb, snap.shape[1])]
    S0_before = bufs_c["S0"].clone()
    C.import_(torch.tensor([0], dtype=torch.int32, device="cuda"), forged)
    assert C.check_status() == lar.DEV_SNAPSHOT
    assert C.read_counts() == [0] * other.B and torch.equal(bufs_c["S0"], S0_before)
    # a sequence id out of range: export marks the header invalid and reports it
    bad = A.export(torch.tensor([shape.B], dtype=torch.int32, device="cuda"))
    assert bad[0, :4].view(torch.int32).item() == 0
    assert A.check_status() == lar.DEV_POINTER
    A.close()
    C.close()
