"""Decode steps captured in a CUDA graph (the small-batch path: one graph launch per
window instead of one host call per step) give the same results as the direct calls.

A window of L replay_step calls is captured once and replayed on fresh inputs copied into
the captured input buffers; a twin layer runs the same steps as direct calls. Outputs,
buffer counts and flush flags must agree bit for bit (same kernels, same inputs), and the
layer must keep stepping directly after the replays.
"""

from __future__ import annotations

import pytest
import torch

import gpu_harness as hx
from workloads import gen

pytestmark = pytest.mark.gpu


def _copy_into(dst: dict, src: dict):
    for k in dst:
        dst[k].copy_(src[k])


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_captured_window_matches_direct_steps(io):
    shape = gen.Shape("g1", B=3, H=4, G=2, P=24, N=32, L=4, io=io, seed=51)
    _, _, direct, S0 = hx.setup(shape)
    _, bufs_g, graphed, _ = hx.setup(shape)
    L = shape.L
    y_direct = torch.empty(shape.B, shape.H, shape.P, device="cuda")
    # one call outside the capture (the first launch sets the kernel's shared-memory limit)
    x = gen.step_inputs(shape, 0, device="cuda")
    graphed.step(x["q"], x["k"], x["v"], x["dt"], x["a"])
    direct.step(x["q"], x["k"], x["v"], x["dt"], x["a"])
    torch.cuda.synchronize()
    # the captured window: fixed input and output buffers per step (an even number of
    # calls, so the host-side pointer parity is the same before and after the window)
    xs = [{k: torch.empty_like(v) for k, v in gen.step_inputs(shape, 0, device="cuda").items()} for _ in range(L)]
    ys = [torch.empty(shape.B, shape.H, shape.P, device="cuda") for _ in range(L)]
    fl = [torch.empty(shape.B, dtype=torch.uint8, device="cuda") for _ in range(L)]
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for t in range(L):
                graphed.step(xs[t]["q"], xs[t]["k"], xs[t]["v"], xs[t]["dt"], xs[t]["a"], y=ys[t], flushed=fl[t])
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert graphed.read_counts() == direct.read_counts()  # capturing queued no work
    fl_direct = torch.empty(shape.B, dtype=torch.uint8, device="cuda")
    step = 1
    for _ in range(3):  # three windows through the graph, fresh inputs each time
        for t in range(L):
            _copy_into(xs[t], gen.step_inputs(shape, step + t, device="cuda"))
        g.replay()
        for t in range(L):
            x = gen.step_inputs(shape, step + t, device="cuda")
            direct.step(x["q"], x["k"], x["v"], x["dt"], x["a"], y=y_direct, flushed=fl_direct)
            torch.cuda.synchronize()
            assert torch.equal(ys[t], y_direct), (step + t)
            assert torch.equal(fl[t], fl_direct), (step + t)
        step += L
        assert graphed.read_counts() == direct.read_counts()
    # direct calls continue from where the replays left the buffers
    for t in range(3):
        x = gen.step_inputs(shape, step + t, device="cuda")
        a = graphed.step(x["q"], x["k"], x["v"], x["dt"], x["a"])
        b = direct.step(x["q"], x["k"], x["v"], x["dt"], x["a"])
        assert torch.equal(a, b)
    assert torch.equal(bufs_g["S0"], direct.buffers["S0"])
    assert graphed.check_status() == 0 and direct.check_status() == 0
    del g
    graphed.close()
    direct.close()
