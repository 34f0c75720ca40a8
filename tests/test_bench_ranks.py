"""Host-side multi-rank logic of bench.py on CPU (gloo, world size 2): the timing that
bench reports is the maximum over ranks, every rank takes the same collective steps,
and the reference arm runs on rank 0 only."""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 10.0 + 5.0 * rank
        got = bench.max_over_ranks(mine, world, torch.device("cpu"))
        bench.barrier(world)
        ref = bench.run_reference(type("A", (), {"workload": "mamba2_b256", "warmup": 0, "steps": 0})(),
                                  rank, world) if rank else None
        out[rank] = (got, ref)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_gloo():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn")
        res = dict(out)
    assert res[0][0] == 15.0 and res[1][0] == 15.0
    assert res[1][1] is None  # non-zero ranks do no reference work


def test_single_rank_max_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5


def test_algorithmic_bytes_per_token_of_the_b256_layer():
    """Per-token bytes of the B=256, L=16 layer: 2,228,224 state bytes for replay vs
    4,194,304 for eager (a 32/17 cut), 2,524,416 in total."""
    sys.path.insert(0, ROOT)
    import bench
    from workloads import gen

    b = bench.algorithmic_bytes_per_token(gen.SHAPES["mamba2_b256"])
    assert b["replay_state"] == 2_228_224 and b["eager_state"] == 4_194_304
    assert b["replay"] == 2_524_416
    assert b["eager_state"] / b["replay_state"] == pytest.approx(32 / 17)
    f = bench.algorithmic_bytes_per_token(gen.SHAPES["mamba2_b256_fp8"])
    assert f["replay_state"] == 802_816


def test_verify_round_bytes_by_hand():
    """Bytes of one verify round, counted by hand for two sequences of the B=256 layer's
    head shape: one that folds (12 committed + 5 positions > L = 16) and one that does
    not (3 + 5)."""
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    from workloads import gen

    s = gen.SHAPES["mamba2_b256_spec"]
    assert (s.H, s.G, s.P, s.N, s.L, s.io_bytes) == (64, 64, 64, 128, 16, 2)
    entry = 64 * 128 * 2 + 64 * 64 * 2 + 8 * 64        # k, v, Delta and a of all heads
    state = 64 * 64 * 128 * 4
    q5 = 5 * 64 * 128 * 2
    y5 = 5 * 4 * 64 * 64
    fold = 2 * state + (12 + 5) * entry + 5 * entry + q5 + y5
    no_fold = state + (3 + 5) * entry + 5 * entry + q5 + y5
    assert bench.verify_round_bytes(s, np.array([12, 3]), 5) == float(fold + no_fold)
