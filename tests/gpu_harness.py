"""Runs the CUDA path (through the C ABI) and the CPU oracle side by side on the same
seeded inputs, and reports their differences. Used by the GPU parity tests."""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

import linear_attention_decode_replay_b200 as lar
from oracle import replay_oracle as ro
from workloads import gen

# Tolerances on the max over (sequence, head, step) of ||y - y_ref||_2 / ||y_ref||_2.
TOL_F32 = 1e-4   # FP32 arithmetic on exactly represented inputs (FP32 or BF16 I/O)
TOL_BF16 = 2e-2  # contract bar for BF16 inputs (the FP32 bar above is tighter and also met)
TOL_FP8 = 6e-2   # FP8 read copy against the unquantised oracle


def lar_config(shape: gen.Shape) -> lar.Config:
    return lar.Config(batch=shape.B, heads=shape.H, groups=shape.G, P=shape.P, N=shape.N, L=shape.L,
                      max_pos=shape.max_pos, io=shape.io, ckpt=shape.ckpt)


def sample_rows(B: int, n: int, seed: int = 0) -> np.ndarray:
    """n sequences spread over the batch, always including the first and last."""
    if n >= B:
        return np.arange(B)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, B - 1), size=n - 2, replace=False)
    return np.sort(np.concatenate([[0, B - 1], mid]))


def _np(t, rows):
    return gen.to_numpy64(t[torch.as_tensor(rows, device=t.device)])


@dataclass
class Report:
    max_err: float = 0.0
    max_err_fp8_emul: float = 0.0
    max_err_shared_fp8: float = 0.0
    steps: int = 0
    flags_equal: bool = True
    counts_equal: bool = True
    ckpt_err: float = 0.0
    per_step: list = field(default_factory=list)
    fro_err: float = 0.0          # max over steps of ||Y - Y_ref||_F / ||Y_ref||_F (sampled batch)
    shared_fro_err: float = 0.0   # same for the shared-FP8 eager kernel
    per_vector: list = field(default_factory=list)  # every per-(sequence, head) error
    shared_per_vector: list = field(default_factory=list)  # the same for the shared-FP8 eager kernel
    per_step_fro: list = field(default_factory=list)
    shared_per_step_fro: list = field(default_factory=list)


def frobenius_error(y, y_ref) -> float:
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    return float(np.linalg.norm(y - y_ref) / max(np.linalg.norm(y_ref), 1e-30))


def vector_errors(y, y_ref) -> np.ndarray:
    num = np.linalg.norm(np.asarray(y, np.float64) - y_ref, axis=-1)
    return (num / np.maximum(np.linalg.norm(y_ref, axis=-1), 1e-30)).ravel()


def setup(shape: gen.Shape, device="cuda"):
    cfg = lar_config(shape)
    bufs = lar.alloc_buffers(cfg, device)
    S0 = gen.initial_state(shape, device=device)
    bufs["S0"].copy_(S0)
    r = lar.Replay(cfg, bufs)
    return cfg, bufs, r, S0


def run_decode(shape: gen.Shape, steps: int, rows, flush_at_end=True, fp8_emulation=False,
               shared_fp8=False) -> Report:
    """Plain decode for `steps` steps; sampled sequences `rows` checked against the oracle
    every step (y, flush flags); all sequences' counts checked at the end."""
    cfg, bufs, r, S0 = setup(shape)
    ref = ro.ReplayBatch(_np(S0, rows), shape.G, shape.L, ckpt="f32")
    # the oracle's emulation of the same read-copy method (FP8 or FP4), beside the FP32 oracle
    emu = ro.ReplayBatch(_np(S0, rows), shape.G, shape.L, ckpt=shape.ckpt) if fp8_emulation else None
    if shared_fp8:  # the in-house shared-FP8 eager kernel on the same inputs, for comparison
        codes_d, scale_d = lar.quantize_rows_e4m3(S0)
    rep = Report()
    fl = torch.zeros(shape.B, dtype=torch.uint8, device="cuda")
    all_flags = []
    for t in range(steps):
        x = gen.step_inputs(shape, t, device="cuda")
        y = r.step(x["q"], x["k"], x["v"], x["dt"], x["a"], flushed=fl)
        xs = {k: _np(v, rows) for k, v in x.items()}
        y_ref, f_ref = ref.step(xs["q"], xs["k"], xs["v"], xs["dt"], xs["a"])
        y_gpu = _np(y, rows)
        e = ro.relative_error(y_gpu, y_ref)
        rep.per_step.append(e)
        rep.max_err = max(rep.max_err, e)
        fro = frobenius_error(y_gpu, y_ref)
        rep.fro_err = max(rep.fro_err, fro)
        if shared_fp8:
            rep.per_vector.append(vector_errors(y_gpu, y_ref))
            rep.per_step_fro.append(fro)
        if emu is not None:
            y_emu, _ = emu.step(xs["q"], xs["k"], xs["v"], xs["dt"], xs["a"])
            rep.max_err_fp8_emul = max(rep.max_err_fp8_emul, ro.relative_error(y_gpu, y_emu))
        if shared_fp8:
            y_sh = lar.eager_step_fp8(cfg, codes_d, scale_d, x["q"], x["k"], x["v"], x["dt"], x["a"])
            y_sh_np = _np(y_sh, rows)
            rep.max_err_shared_fp8 = max(rep.max_err_shared_fp8, ro.relative_error(y_sh_np, y_ref))
            sh_fro = frobenius_error(y_sh_np, y_ref)
            rep.shared_fro_err = max(rep.shared_fro_err, sh_fro)
            rep.shared_per_step_fro.append(sh_fro)
            rep.shared_per_vector.append(vector_errors(y_sh_np, y_ref))
        f_gpu = fl.cpu().numpy()
        all_flags.append(f_gpu.copy())
        if not np.array_equal(f_gpu[rows], f_ref):
            rep.flags_equal = False
    rep.steps = steps
    counts = np.array(r.read_counts())
    want = np.array([s.count for s in ref.seqs])
    # every sequence follows the same schedule in plain decode: all counts equal the oracle's
    rep.counts_equal = bool(np.all(counts[rows] == want) and np.all(counts == counts[0]))
    # flags must also agree across the whole batch (lockstep schedule)
    flags = np.array(all_flags)
    rep.flags_equal = rep.flags_equal and bool(np.all(flags == flags[:, :1]))
    if flush_at_end:
        r.flush()
        ref.flush()
        S_gpu = _np(bufs["S0"], rows)
        S_ref = ref.checkpoints()
        rep.ckpt_err = ro.relative_error(S_gpu, S_ref)
        assert r.read_counts() == [0] * shape.B
    assert r.check_status() == 0
    r.close()
    return rep


def run_spec(shape: gen.Shape, rounds: int, rows, n_pos=None, steps_after=0) -> Report:
    """Speculative rounds: verify n_pos positions, roll back to 1 + accepted; sampled
    sequences checked every round, counts of all sequences checked every round."""
    n_pos = n_pos or shape.max_pos
    cfg, bufs, r, S0 = setup(shape)
    ref_all = None
    ref = ro.ReplayBatch(_np(S0, rows), shape.G, shape.L)
    rep = Report()
    fl = torch.zeros(shape.B, dtype=torch.uint8, device="cuda")
    # a full-batch count model: counts follow from accepted lengths alone
    count_model = np.zeros(shape.B, dtype=np.int64)
    for rnd in range(rounds):
        x = gen.verify_inputs(shape, rnd, n_pos, device="cuda")
        y = r.verify(x["q"], x["k"], x["v"], x["dt"], x["a"], flushed=fl)
        acc = gen.accepted_lengths(shape, rnd, n_pos, device="cuda")
        n_keep = (acc + 1).to(torch.int32)
        r.rollback(n_keep)
        xs = {k: _np(v, rows) for k, v in x.items()}
        y_ref, f_ref = ref.verify(xs["q"], xs["k"], xs["v"], xs["dt"], xs["a"])
        nk = n_keep.cpu().numpy()
        ref.rollback(nk[rows])
        e = ro.relative_error(_np(y, rows), y_ref)
        rep.max_err = max(rep.max_err, e)
        rep.per_step.append(e)
        f_gpu = fl.cpu().numpy()
        flush_model = count_model + n_pos > shape.L
        if not (np.array_equal(f_gpu[rows], f_ref) and np.array_equal(f_gpu.astype(bool), flush_model)):
            rep.flags_equal = False
        count_model = np.where(flush_model, 0, count_model) + nk
        counts = np.array(r.read_counts())
        if not (np.array_equal(counts, count_model) and np.array_equal(counts[rows], ref.counts)):
            rep.counts_equal = False
    for t in range(steps_after):
        xx = gen.step_inputs(shape, 10_000 + t, device="cuda")
        y = r.step(xx["q"], xx["k"], xx["v"], xx["dt"], xx["a"])
        xs = {k: _np(v, rows) for k, v in xx.items()}
        y_ref, _ = ref.step(xs["q"], xs["k"], xs["v"], xs["dt"], xs["a"])
        rep.max_err = max(rep.max_err, ro.relative_error(_np(y, rows), y_ref))
    r.flush()
    ref.flush()
    rep.ckpt_err = ro.relative_error(_np(bufs["S0"], rows), ref.checkpoints())
    assert r.check_status() == 0
    r.close()
    rep.steps = rounds
    del ref_all
    return rep


def run_eager(shape: gen.Shape, steps: int, rows, fp8=False) -> Report:
    """The in-house eager kernel (FP32 state, or shared FP8 state) against the oracle."""
    cfg = lar_config(shape)
    S0 = gen.initial_state(shape, device="cuda")
    rep = Report()
    if fp8:
        codes_d, scale_d = lar.quantize_rows_e4m3(S0)
        codes, scale = ro.quantize_rows_e4m3(_np(S0, rows))
    else:
        S = S0.clone()
        S_ref = _np(S0, rows)
    for t in range(steps):
        x = gen.step_inputs(shape, t, device="cuda")
        xs = {k: _np(v, rows) for k, v in x.items()}
        if fp8:
            y = lar.eager_step_fp8(cfg, codes_d, scale_d, x["q"], x["k"], x["v"], x["dt"], x["a"])
            codes, scale, y_ref = ro.eager_fp8_batch_step(codes, scale, xs["q"], xs["k"], xs["v"], xs["dt"],
                                                          xs["a"], shape.G)
        else:
            y = lar.eager_step(cfg, S, x["q"], x["k"], x["v"], x["dt"], x["a"])
            S_ref, y_ref = ro.eager_batch_step(S_ref, xs["q"], xs["k"], xs["v"], xs["dt"], xs["a"], shape.G)
        e = ro.relative_error(_np(y, rows), y_ref)
        rep.per_step.append(e)
        rep.max_err = max(rep.max_err, e)
    if not fp8:
        rep.ckpt_err = ro.relative_error(_np(S, rows), S_ref)
    rep.steps = steps
    return rep
