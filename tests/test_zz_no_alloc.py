"""replay_verify_static_scratch: verify whose packed queries live in a fixed device array
inside libreplay.so, for callers that cannot allocate device memory (a layer hosted by a
program that owns all of the GPU's memory and hands it only its state and per-call
tensors, so it has no way to get the qpack buffer that replay_verify needs).

Each test calls the entry point through the C ABI and compares it with replay_verify on
the same seeded inputs, and with the CPU oracle, over verify calls in a row, within the
FP32 tolerance of the other parity tests; flush flags and buffer counts must match
exactly. The file is named to be collected last.
"""

from __future__ import annotations

import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import linear_attention_decode_replay_b200 as lar
from linear_attention_decode_replay_b200 import _abi
from oracle import replay_oracle as ro
from workloads import gen

from gpu_harness import TOL_F32, lar_config, vector_errors

SHAPE_F32 = gen.Shape("no_alloc_small", B=5, H=4, G=2, P=24, N=32, L=6, io="f32", max_pos=4, steps=0, seed=77)
SHAPE_FP8 = gen.Shape("no_alloc_fp8", B=3, H=2, G=1, P=32, N=64, L=6, io="bf16", ckpt="f32_fp8read", max_pos=4,
                      steps=0, seed=79)


def _layer(shape: gen.Shape, S0: torch.Tensor) -> lar.Replay:
    cfg = lar_config(shape)
    bufs = lar.alloc_buffers(cfg, "cuda")
    bufs["S0"].copy_(S0)
    return lar.Replay(cfg, bufs)


def _verify_static(layer: lar.Replay, x: dict, y: torch.Tensor, flushed=None) -> int:
    """The entry point called directly through ctypes; returns its status code."""
    vp = ctypes.c_void_p
    return _abi.load().replay_verify_static_scratch(
        layer._ctx, x["q"].shape[1], vp(x["q"].data_ptr()), vp(x["k"].data_ptr()), vp(x["v"].data_ptr()),
        vp(x["dt"].data_ptr()), vp(x["a"].data_ptr()), vp(y.data_ptr()),
        None if flushed is None else vp(flushed.data_ptr()), vp(torch.cuda.current_stream().cuda_stream))


def _np(t):
    return gen.to_numpy64(t)


CASES = [(SHAPE_F32, 1), (SHAPE_F32, 4), (SHAPE_FP8, 4)]


@pytest.mark.gpu
@pytest.mark.parametrize("shape,variant_max_pos", CASES,
                         ids=["f32_no_qpack_max_pos1", "f32_same_ring_max_pos4", "bf16_fp8read_max_pos4"])
def test_static_scratch_verify_matches_replay_verify(shape, variant_max_pos):
    S0 = gen.initial_state(shape, device="cuda")
    ref = _layer(shape, S0)                                     # replay_verify with its qpack
    var = _layer(dataclasses.replace(shape, max_pos=variant_max_pos), S0)
    assert (var.buffers.get("qpack") is None) == (variant_max_pos == 1)
    fp8 = shape.ckpt == "f32_fp8read"
    oracle = ro.ReplayBatch(_np(S0), shape.G, shape.L, ckpt=shape.ckpt)
    # five buffered entries: with max_pos = 1 (ring of 7 records) the first verify of four
    # positions must fold those buffers first; with max_pos = 4 the verify folds them itself
    for t in range(5):
        x = gen.step_inputs(shape, t, device="cuda")
        y_ref = ref.step(x["q"], x["k"], x["v"], x["dt"], x["a"])
        y_var = var.step(x["q"], x["k"], x["v"], x["dt"], x["a"])
        xs = {k: _np(v) for k, v in x.items()}
        oracle.step(xs["q"], xs["k"], xs["v"], xs["dt"], xs["a"])
        assert vector_errors(_np(y_var), _np(y_ref)).max() <= TOL_F32
    counts = np.full(shape.B, 5)
    # calls in a row; later ones pack fewer positions than the first, so queries an earlier
    # call left in the array would show if a later one read them
    fl_ref = torch.zeros(shape.B, dtype=torch.uint8, device="cuda")
    fl_var = torch.full((shape.B,), 7, dtype=torch.uint8, device="cuda")
    for rnd, n_pos in enumerate((4, 2, 3)):
        x = gen.verify_inputs(shape, rnd, n_pos, device="cuda")
        y_ref = ref.verify(x["q"], x["k"], x["v"], x["dt"], x["a"], flushed=fl_ref)
        y_var = torch.full_like(y_ref, float("nan"))
        assert _verify_static(var, x, y_var, fl_var) == _abi.REPLAY_OK
        torch.cuda.synchronize()
        xs = {k: _np(v) for k, v in x.items()}
        y_orc, f_orc = oracle.verify(xs["q"], xs["k"], xs["v"], xs["dt"], xs["a"])
        y_ref_h = _np(y_ref)
        assert np.linalg.norm(y_ref_h) > 0
        err = vector_errors(_np(y_var), y_ref_h)
        assert np.isfinite(err).all() and err.max() <= TOL_F32, (rnd, n_pos, err.max())
        if not fp8:  # the FP8 read path is checked against the unquantised oracle elsewhere
            assert vector_errors(_np(y_var), y_orc).max() <= TOL_F32, (rnd, n_pos)
        else:
            assert vector_errors(_np(y_var), y_orc).max() <= 1e-3, (rnd, n_pos)
        folds = counts + n_pos > shape.L
        assert np.array_equal(fl_var.cpu().numpy(), folds.astype(np.uint8)), (rnd, fl_var)
        assert np.array_equal(fl_ref.cpu().numpy(), f_orc)
        n_keep = (gen.accepted_lengths(shape, rnd, n_pos, device="cuda") + 1).to(torch.int32)
        ref.rollback(n_keep)
        var.rollback(n_keep)
        oracle.rollback(n_keep.cpu().numpy())
        counts = np.where(folds, 0, counts) + n_keep.cpu().numpy()
        assert var.read_counts() == ref.read_counts() == list(counts) == list(oracle.counts)
    # the layer keeps decoding from the rolled-back buffer
    x = gen.step_inputs(shape, 100, device="cuda")
    y_ref = ref.step(x["q"], x["k"], x["v"], x["dt"], x["a"])
    y_var = var.step(x["q"], x["k"], x["v"], x["dt"], x["a"])
    assert vector_errors(_np(y_var), _np(y_ref)).max() <= TOL_F32
    assert ref.check_status() == 0 and var.check_status() == 0
    ref.close()
    var.close()


@pytest.mark.gpu
def test_static_scratch_rejects_calls_beyond_its_size():
    # B * G * n_pos * N * 4 = 1025 * 8 * n_pos * 128 * 4: 29.4 MB for n_pos = 7, 33.6 MB for 8
    shape = gen.Shape("no_alloc_limit", B=1025, H=8, G=8, P=16, N=128, L=8, io="f32", max_pos=1, steps=0,
                      seed=78)
    assert 1025 * 8 * 7 * 128 * 4 <= _abi.STATIC_SCRATCH_BYTES < 1025 * 8 * 8 * 128 * 4
    layer = _layer(shape, torch.zeros(1025, 8, 16, 128, device="cuda"))
    x = gen.verify_inputs(shape, 0, 8, device="cuda")
    y = torch.empty(1025, 8, 8, 16, device="cuda")
    assert _verify_static(layer, x, y) == _abi.REPLAY_ESCRATCH
    assert "REPLAY_STATIC_SCRATCH_BYTES" in _abi.strerror(_abi.REPLAY_ESCRATCH)
    # nothing was queued and no verify is pending: the largest call that fits still runs
    x7 = {k: v[:, :7].contiguous() for k, v in x.items()}
    y7 = torch.empty(1025, 7, 8, 16, device="cuda")
    assert _verify_static(layer, x7, y7) == _abi.REPLAY_OK
    layer.rollback(torch.zeros(1025, dtype=torch.int32, device="cuda"))
    assert layer.check_status() == 0
    assert torch.isfinite(y7).all()
    layer.close()


def test_static_scratch_size_matches_header():
    import os
    import re
    here = os.path.dirname(os.path.abspath(__file__))
    with open(os.path.join(here, "..", "include", "replay.h")) as f:
        m = re.search(r"#define REPLAY_STATIC_SCRATCH_BYTES \((\d+)u << (\d+)\)", f.read())
    assert m and int(m.group(1)) << int(m.group(2)) == _abi.STATIC_SCRATCH_BYTES
