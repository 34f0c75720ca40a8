#!/usr/bin/env python
"""Decode throughput of the ReplaySSM path on one SSM layer (B200).

One bench step is one window of L decode tokens for the whole batch: L calls of
replay_step, one of which folds the buffer into the checkpoint (every row of the hot
path: append, decay scan, k.q products, output-only reads of S0, the fused flush).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

`--workload sweep` times replay_step against eager_step over the batch x window x
head-layout sweep and prints one line with every point.

Under torchrun every rank runs its own replica of the batch on its own GPU (sequences
are independent; there is no collective on the data path) and the timing is the max
over ranks. Rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import gen  # noqa: E402

METRIC = "decode tokens/s per SSM layer at batch 256, L=16 (1 B200); achieved HBM GB/s vs peak"
UNIT = "tokens/s"
SPEC_METRIC = "speculative decode tokens/s per SSM layer at batch 256, L=16, draft 4 (1 B200); achieved HBM GB/s vs peak"
FALLBACK_HBM_GBS = 6650.0

# DRAM traffic of one replay_step launch (flush and output-only launches averaged over a
# window) of the workload it was captured on, from an ncu capture, and the hash of the
# kernel sources it applies to. For another workload, or once the sources change, the
# figure does not apply and is reported as null. "captured_on" is the hash of the sources
# of the capture itself (they differ from the current ones only in the kernel's header
# comment and in two unused device helpers since removed). Measured on the fold launch
# and an 8-entry output-only launch: (fold + 15 x output-only) / 16.
NCU_TRAFFIC = {"workload": "mamba2_b256",
               "sources_sha256": "ca5c0a8c8f3c97581a3b95deec93766a80041e023cd01d3a2fcda67ef3bd8f8a",
               "captured_on": "e21d8dddf37eccd0f0edeb00f8e98d6b152826fcde7bec1dd8fcedccd8204fe7",
               "bytes_per_launch": 646.1e6}


def kernel_sources_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_attention_decode_replay_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode())
            h.update(fh.read())
    return h.hexdigest()


def algorithmic_bytes_per_token(s: gen.Shape) -> dict:
    """Bytes a decoded token must move, per sequence (steady state, lazy flush once per
    window of L tokens):
      replay: state (L+1)/L * H*P*N*4 (L-1 output-only reads + one fused read+write; with
              a read copy, L-1 reads of the codes and scales, and the fold reads and writes
              the master and writes the copy),
              buffer re-reads (L+1)/2 * E, new inputs q + E, entry write E, output 4*H*P,
              with E = G*N*s + H*P*s + 8*H (one entry: k, v, Delta, a);
      eager:  state 2 * H*P*N*4 (read + write), inputs q + E, output 4*H*P."""
    sio = s.io_bytes
    E = s.G * s.N * sio + s.H * s.P * sio + 8 * s.H
    q = s.G * s.N * sio
    y = 4 * s.H * s.P
    state = s.H * s.P * s.N * 4
    if s.ckpt in ("f32_fp8read", "f32_fp4read"):
        code_bytes = s.N if s.ckpt == "f32_fp8read" else s.N // 2
        copy = s.H * s.P * (code_bytes + 4)  # e4m3 or e2m1 codes + per-row scales
        replay_state = ((s.L - 1) * copy + 2 * state + copy) / s.L
    else:
        replay_state = (s.L + 1) / s.L * state
    replay = replay_state + (s.L + 1) / 2 * E + (q + E) + E + y
    eager = 2 * state + q + E + y
    return {"replay": replay, "eager": eager, "replay_state": replay_state, "eager_state": 2 * state}


# ------------------------------------------------------------------ distributed plumbing

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def max_over_ranks(value: float, world: int, device) -> float:
    """Max of a per-rank float over all ranks (the slowest rank sets the time)."""
    if world <= 1:
        return value
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clocks and throttle reasons of one GPU with nvidia-smi while running."""

    FIELDS = ["uuid", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device: int):
        self.uuid = None
        try:
            self.uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:  # noqa: BLE001
            pass
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(", ") for r in out.strip().splitlines() if r.strip()]
        rows = [r for r in rows if len(r) == len(self.FIELDS) and (self.uuid is None or r[0] == self.uuid)]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ CPU oracle baseline

def _oracle_sample_inputs(shape: gen.Shape):
    """One sequence of the workload (all heads) and the inputs of one oracle sample: one
    window of L decode steps plus the step that folds it, or, for verify workloads, L
    verify rounds with their n_keep. Returns (S0 [H,P,N], inputs, keeps or None, tokens)."""
    one = shape.replace(B=1)
    S0 = gen.to_numpy64(gen.initial_state(one, device="cpu"))[0]
    if shape.max_pos > 1:
        xs = [{k: gen.to_numpy64(v) for k, v in gen.verify_inputs(one, t, shape.max_pos, device="cpu").items()}
              for t in range(shape.L)]
        keeps = [gen.accepted_lengths(one, t, shape.max_pos, device="cpu").numpy().astype(np.int64) + 1
                 for t in range(shape.L)]
        return S0, xs, keeps, int(sum(k.sum() for k in keeps))
    xs = [{k: gen.to_numpy64(v) for k, v in gen.step_inputs(one, t, device="cpu").items()}
          for t in range(shape.L)]
    return S0, xs + xs[:1], None, shape.L + 1


def _sample_text(shape: gen.Shape, tokens: int) -> str:
    if shape.max_pos > 1:
        return (f"1 sequence x {shape.H} heads x {shape.L} verify rounds of {shape.max_pos} positions "
                f"({tokens} accepted tokens) of {shape.name}")
    return f"1 sequence x {shape.H} heads x {shape.L + 1} decode steps (one window and its fold) of {shape.name}"


def cpu_oracle_rate(shape: gen.Shape, budget_s: float):
    """Tokens/s of the CPU oracle (float64 numpy) on sequences of the workload's shape,
    on all host cores (one process per core, each replaying whole sequences with one
    BLAS thread; sequences are independent) and on one core, each for about budget_s
    seconds of wall time. Returns the cpu_baseline record."""
    from oracle.pool import OraclePool, cpu_model, host_cores

    S0, xs, keeps, tokens = _oracle_sample_inputs(shape)
    cores = host_cores()
    with OraclePool(1, S0, xs, keeps, shape.G, shape.L) as pool:
        s1, t1 = pool.run_for(budget_s / 2)
    with OraclePool(cores, S0, xs, keeps, shape.G, shape.L) as pool:
        sn, tn = pool.run_for(budget_s / 2)
    return {"value": sn * tokens / tn, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": (f"{sn} samples on {cores} processes in {tn:.1f} s, each {_sample_text(shape, tokens)}, "
                       f"float64 numpy, one BLAS thread per process"),
            "one_core": {"value": s1 * tokens / t1, "cores": 1, "sample": f"{s1} samples in {t1:.1f} s"},
            "cpu_model": cpu_model()}


# ------------------------------------------------------------------ our arm

def e2e_overlapped(lar, cfg, shape, r, host_in, S0, device, nwin):
    """Decode windows end to end with the copies on their own streams: inputs copied from
    pinned host memory into one of two device slots, y copied back from one of two
    output slots, so that the input copy of step j+1 and the output copy of step j-1
    overlap the kernel of step j. Events order every slot's reuse. Returns the time of
    one window (ms) on layer `r` and whether a self-check passed: one window through
    this path and one through plain calls on the same stream, each on a fresh layer from
    the same checkpoint, must give the same outputs bit for bit (a missing dependency
    shows up there as stale inputs or outputs)."""
    B, H, P, L = shape.B, shape.H, shape.P, shape.L
    stream = torch.cuda.current_stream(device)
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    dev_in = [{k: torch.empty(v.shape, dtype=v.dtype, device=device) for k, v in host_in[0].items()}
              for _ in range(2)]
    dev_y = [torch.empty(B, H, P, device=device) for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def windows(layer, count, host_out):
        j = 0
        for _ in range(count):
            for hx in host_in:
                s_ = j % 2
                if j >= 2:
                    up.wait_event(ev_done[s_])     # the kernel that read this slot is done
                with torch.cuda.stream(up):
                    for k, t in dev_in[s_].items():
                        t.copy_(hx[k], non_blocking=True)
                    ev_in[s_].record(up)
                stream.wait_event(ev_in[s_])
                if j >= 2:
                    stream.wait_event(ev_out[s_])  # this slot's previous y has been copied out
                d = dev_in[s_]
                layer.step(d["q"], d["k"], d["v"], d["dt"], d["a"], y=dev_y[s_])
                ev_done[s_].record(stream)
                down.wait_event(ev_done[s_])
                with torch.cuda.stream(down):
                    host_out[j % len(host_out)].copy_(dev_y[s_], non_blocking=True)
                    ev_out[s_].record(down)
                j += 1
        stream.wait_stream(up)
        stream.wait_stream(down)

    # self-check on two fresh layers
    twins = []
    for _ in range(2):
        b = lar.alloc_buffers(cfg, device)
        b["S0"].copy_(S0)
        twins.append((b, lar.Replay(cfg, b)))
    out_a = [torch.empty(B, H, P).pin_memory() for _ in range(L)]
    windows(twins[0][1], 1, out_a)
    torch.cuda.synchronize()
    ok = True
    yb = torch.empty(B, H, P, device=device)
    for t, hx in enumerate(host_in):
        d = {k: v.to(device) for k, v in hx.items()}
        twins[1][1].step(d["q"], d["k"], d["v"], d["dt"], d["a"], y=yb)
        ok = ok and torch.equal(yb.cpu(), out_a[t])
    for b, layer in twins:
        layer.close()
    del twins, out_a
    torch.cuda.empty_cache()

    host_y = [torch.empty(B, H, P).pin_memory() for _ in range(2)]
    windows(r, 1, host_y)
    torch.cuda.synchronize()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    up.wait_event(x0)
    down.wait_event(x0)
    windows(r, nwin, host_y)
    x1.record(stream)
    torch.cuda.synchronize()
    return x0.elapsed_time(x1) / nwin, ok


def run_ours(args, rank, world, local):
    import linear_attention_decode_replay_b200 as lar

    shape = gen.SHAPES[args.workload]
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    cfg = lar.Config(batch=shape.B, heads=shape.H, groups=shape.G, P=shape.P, N=shape.N, L=shape.L,
                     max_pos=1, io=shape.io, ckpt=shape.ckpt)
    L, B = shape.L, shape.B
    bufs = lar.alloc_buffers(cfg, device)
    S0 = gen.initial_state(shape, device=device)
    bufs["S0"].copy_(S0)
    r = lar.Replay(cfg, bufs)
    window = [gen.step_inputs(shape, t, device=device) for t in range(L)]
    y = torch.empty(B, shape.H, shape.P, device=device)

    def one_window():
        for x in window:
            r.step(x["q"], x["k"], x["v"], x["dt"], x["a"], y=y)

    for _ in range(args.warmup):
        one_window()
    torch.cuda.synchronize()
    barrier(world)

    K = args.steps
    stream = torch.cuda.current_stream()
    t_start, t_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    t_start.record(stream)
    for _ in range(K):
        one_window()
    t_stop.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_stop), world, device)
    # one replay_kernel launch per step, back to back: the average launch over the timed
    # region (gaps between launches included)
    avg_launch_ms = elapsed_ms / (K * L)
    status = r.check_status()
    if status:
        raise RuntimeError(f"device status bits {status} after the timed region")

    # ---- fold and output-only launches apart: an instrumented pass with an event pair
    # around every launch (the events add gaps, so this pass is not the timed one); in
    # lockstep decode the first launch of every window folds the buffers
    Ki = max(3, min(K, 100))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(Ki * L)]
    i = 0
    for _ in range(Ki):
        for x in window:
            ev[i][0].record(stream)
            r.step(x["q"], x["k"], x["v"], x["dt"], x["a"], y=y)
            ev[i][1].record(stream)
            i += 1
    torch.cuda.synchronize()
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    fold_ms = statistics.mean(launch_ms[0::L])
    out_ms = statistics.mean([t for j, t in enumerate(launch_ms) if j % L]) if L > 1 else fold_ms

    bpt = algorithmic_bytes_per_token(shape)
    bytes_per_launch = bpt["replay"] * B  # one launch decodes one token of every sequence
    achieved_gbs = bytes_per_launch / (avg_launch_ms * 1e-3) / 1e9
    peak, peak_kind = measured_hbm_peak()
    traffic = None
    if NCU_TRAFFIC["sources_sha256"] == kernel_sources_hash() and NCU_TRAFFIC["workload"] == shape.name:
        traffic = NCU_TRAFFIC["bytes_per_launch"]

    tokens = world * B * L * K
    value = tokens / (elapsed_ms * 1e-3)

    # ---- phased flush: the sequences' windows staggered so that each step folds 1/L of
    # the batch (replay_flush with a mask sets the phases once); same inputs, same bytes
    phase_of = torch.arange(B, device=device) % L
    for t in range(L - 1):
        r.step(window[t]["q"], window[t]["k"], window[t]["v"], window[t]["dt"], window[t]["a"], y=y)
        r.flush((phase_of == t).to(torch.uint8))
    for _ in range(2):
        one_window()
    torch.cuda.synchronize()
    counts = np.array(r.read_counts())
    ph0, ph1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    Kp = max(3, min(K, 300))
    ph0.record(stream)
    for _ in range(Kp):
        one_window()
    ph1.record(stream)
    torch.cuda.synchronize()
    phased_ms = max_over_ranks(ph0.elapsed_time(ph1) / Kp, world, device)
    if r.check_status():
        raise RuntimeError("device status bits set in the phased run")
    phased = {"value": world * B * L / (phased_ms * 1e-3), "unit": UNIT, "ms_per_step": phased_ms,
              "windows": Kp, "distinct_buffer_counts": int(len(np.unique(counts)))}

    # ---- the in-house eager kernel on the same inputs (state read + written every token)
    S = S0.clone()
    Ke = max(3, K // 4)
    for _ in range(2):
        for x in window:
            lar.eager_step(cfg, S, x["q"], x["k"], x["v"], x["dt"], x["a"], y=y)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(Ke):
        for x in window:
            lar.eager_step(cfg, S, x["q"], x["k"], x["v"], x["dt"], x["a"], y=y)
    e1.record(stream)
    torch.cuda.synchronize()
    eager_ms = max_over_ranks(e0.elapsed_time(e1) / Ke, world, device)
    del S

    # ---- end to end through the public API: pinned host inputs in, y back to the host
    host_in = [{k: v.cpu().pin_memory() for k, v in x.items()} for x in window]
    dev_in = {k: torch.empty_like(v) for k, v in window[0].items()}
    host_y = torch.empty(B, shape.H, shape.P).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host_in[0].values()) * L
    d2h = host_y.numel() * host_y.element_size() * L
    Kx = max(3, min(K, 100))
    torch.cuda.synchronize()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for _ in range(Kx):
        for hx in host_in:
            for k in dev_in:
                dev_in[k].copy_(hx[k], non_blocking=True)
            r.step(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["dt"], dev_in["a"], y=y)
            host_y.copy_(y, non_blocking=True)
    x1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(x0.elapsed_time(x1) / Kx, world, device)
    # the same with the copies overlapping the kernels (self-checked; the plain figure
    # above stands if the check fails or the path raises on any rank)
    ovl_ms, ovl_note = -1.0, "overlapped copies: self-check passed"
    try:
        ovl_ms, ok = e2e_overlapped(lar, cfg, shape, r, host_in, S0, device, Kx)
        if not ok:
            ovl_ms, ovl_note = -1.0, "overlapped copies not used: their outputs differed from plain calls"
    except Exception as exc:  # noqa: BLE001 - a failed optional measurement must not end the bench
        ovl_ms, ovl_note = -1.0, f"overlapped copies not used: {type(exc).__name__}: {exc}"[:200]
    ovl_failed = max_over_ranks(1.0 if ovl_ms <= 0 else 0.0, world, device)
    ovl_ms = max_over_ranks(ovl_ms, world, device)
    if ovl_failed and not ovl_note.startswith("overlapped copies not used"):
        ovl_note = "overlapped copies not used: not every rank passed its self-check"
    r.close()

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": elapsed_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": shape.name, "batch": B, "heads": shape.H, "groups": shape.G, "P": shape.P,
                   "N": shape.N, "L": L, "io": shape.io, "ckpt": shape.ckpt,
                   "step": f"one window = {L} replay_step launches x {B} sequences",
                   "global_batch": B * world, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (checkpoint %d MiB per GPU)" % (B * shape.H * shape.P * shape.N * 4 >> 20)},
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peak, "unit": "GB/s",
                     "frac": achieved_gbs / peak, "traffic": traffic, "peak_source": peak_kind,
                     "kernel": "replay_kernel (replay_step: appends the entries, then streams the state)",
                     "avg_launch_us": avg_launch_ms * 1e3,
                     "fold_launch_us": fold_ms * 1e3, "output_launch_us": out_ms * 1e3,
                     "launch_split": f"fold / output-only launch times from {Ki} instrumented windows",
                     "algorithmic_bytes_per_launch": bytes_per_launch},
        "e2e": {"value": world * B * L / ((e2e_ms if ovl_failed else min(e2e_ms, ovl_ms)) * 1e-3), "unit": UNIT,
                "plain_calls_value": world * B * L / (e2e_ms * 1e-3),
                "overlapped_value": None if ovl_failed else world * B * L / (ovl_ms * 1e-3),
                "copies": ovl_note, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": K * L,  # one replay_kernel launch per replay_step (it appends the entries itself)
        "clocks": clk,
        "eager": {"value": world * B * L / (eager_ms * 1e-3), "unit": UNIT, "ms_per_step": eager_ms,
                  "kernel": "replay_kernel (eager_step)",
                  "achieved_gbs": bpt["eager"] * B * L / (eager_ms * 1e-3) / 1e9},
        "speedup_vs_eager": value / (world * B * L / (eager_ms * 1e-3)),
        "phased_flush": phased,
        "state_bytes_per_token": {"replay": bpt["replay_state"], "eager": bpt["eager_state"],
                                  "cut": bpt["eager_state"] / bpt["replay_state"]},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_oracle_rate(shape, args.cpu_seconds)
    return result


# ------------------------------------------------------------------ our arm, speculative verify

def verify_round_bytes(s: gen.Shape, counts: np.ndarray, n_pos: int) -> float:
    """Algorithmic bytes of one verify round over the batch, given every sequence's
    committed count before it: the state read (and written when the round folds), the
    buffered and new entries read, the new entries written, the queries, the outputs."""
    sio = s.io_bytes
    E = s.G * s.N * sio + s.H * s.P * sio + 8 * s.H
    state = s.H * s.P * s.N * 4
    fold = counts + n_pos > s.L
    per_seq = (state * (1 + fold) + (counts + n_pos) * E + n_pos * E + n_pos * s.G * s.N * sio
               + n_pos * 4 * s.H * s.P)
    return float(per_seq.sum())


def run_spec_ours(args, rank, world, local):
    """One bench step = R verify rounds of n_pos = max_pos positions over the batch, each
    followed by the rollback that keeps 1 + accepted entries (accepted drawn per sequence
    and round); tokens = sum of (1 + accepted)."""
    import linear_attention_decode_replay_b200 as lar

    shape = gen.SHAPES[args.workload]
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    n_pos = shape.max_pos
    cfg = lar.Config(batch=shape.B, heads=shape.H, groups=shape.G, P=shape.P, N=shape.N, L=shape.L,
                     max_pos=n_pos, io=shape.io, ckpt=shape.ckpt)
    B, R = shape.B, shape.L
    bufs = lar.alloc_buffers(cfg, device)
    bufs["S0"].copy_(gen.initial_state(shape, device=device))
    r = lar.Replay(cfg, bufs)
    rounds = [gen.verify_inputs(shape, t, n_pos, device=device) for t in range(R)]
    keeps = [(gen.accepted_lengths(shape, t, n_pos, device=device) + 1).to(torch.int32) for t in range(R)]
    keeps_h = [k.cpu().numpy().astype(np.int64) for k in keeps]
    y = torch.empty(B, n_pos, shape.H, shape.P, device=device)

    def one_step():
        for x, nk in zip(rounds, keeps):
            r.verify(x["q"], x["k"], x["v"], x["dt"], x["a"], y=y)
            r.rollback(nk)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    counts0 = np.array(r.read_counts(), dtype=np.int64)
    barrier(world)

    K = args.steps
    stream = torch.cuda.current_stream()
    t_start, t_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    t_start.record(stream)
    for _ in range(K):
        one_step()
    t_stop.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_stop), world, device)
    status = r.check_status()
    if status:
        raise RuntimeError(f"device status bits {status} after the timed region")

    # algorithmic bytes of the timed rounds, following the counts
    counts = counts0.copy()
    total_bytes = 0.0
    for _ in range(K):
        for nk in keeps_h:
            total_bytes += verify_round_bytes(shape, counts, n_pos)
            counts = np.where(counts + n_pos > shape.L, 0, counts) + nk
    tokens_per_step = float(sum(k.sum() for k in keeps_h))
    tokens = world * tokens_per_step * K
    value = tokens / (elapsed_ms * 1e-3)
    round_ms = elapsed_ms / (K * R)
    achieved_gbs = total_bytes / (K * R) / (round_ms * 1e-3) / 1e9
    peak, peak_kind = measured_hbm_peak()

    # end to end: pinned host inputs of every round in, y back
    host_rounds = [{k: v.cpu().pin_memory() for k, v in x.items()} for x in rounds]
    host_keeps = [k.cpu().pin_memory() for k in keeps]
    dev_in = {k: torch.empty_like(v) for k, v in rounds[0].items()}
    dev_keep = torch.empty_like(keeps[0])
    host_y = torch.empty(B, n_pos, shape.H, shape.P).pin_memory()
    h2d = (sum(v.numel() * v.element_size() for v in host_rounds[0].values()) + B * 4) * R
    d2h = host_y.numel() * host_y.element_size() * R
    Kx = max(3, min(K, 50))
    torch.cuda.synchronize()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for _ in range(Kx):
        for hx, hk in zip(host_rounds, host_keeps):
            for k in dev_in:
                dev_in[k].copy_(hx[k], non_blocking=True)
            dev_keep.copy_(hk, non_blocking=True)
            r.verify(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["dt"], dev_in["a"], y=y)
            r.rollback(dev_keep)
            host_y.copy_(y, non_blocking=True)
    x1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(x0.elapsed_time(x1) / Kx, world, device)
    r.close()

    cpu = cpu_oracle_rate(shape, args.cpu_seconds) if rank == 0 and world == 1 and not args.no_cpu_baseline else None
    return {
        "cpu_baseline": cpu,
        "metric": SPEC_METRIC,
        "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": elapsed_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": shape.name, "batch": B, "heads": shape.H, "groups": shape.G, "P": shape.P,
                   "N": shape.N, "L": shape.L, "n_pos": n_pos, "io": shape.io, "ckpt": shape.ckpt,
                   "step": f"{R} verify rounds of {n_pos} positions x {B} sequences, each rolled back to 1 + accepted",
                   "global_batch": B * world, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (checkpoint %d MiB per GPU)" % (B * shape.H * shape.P * shape.N * 4 >> 20)},
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peak, "unit": "GB/s",
                     "frac": achieved_gbs / peak, "traffic": None, "peak_source": peak_kind,
                     "kernel": "verify round = pack_entries_kernel + replay_kernel + rollback_kernel (events bracket the rounds)",
                     "round_us": round_ms * 1e3, "algorithmic_bytes_per_round": total_bytes / (K * R)},
        "e2e": {"value": world * tokens_per_step / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": 3 * K * R,
        "clocks": clk,
        "tokens_per_round": tokens_per_step / R,
    }


# ------------------------------------------------------------------ reference arm (the oracle)

def run_reference(args, rank, world):
    """The reference arm: the CPU oracle (there is no reference implementation to
    install: the reference holds only web pages). Each step, every one of the host's
    cores (one spawned process each) replays one sample of the workload."""
    if rank != 0:
        return None
    shape = gen.SHAPES[args.workload]
    from oracle.pool import OraclePool, cpu_model, host_cores

    S0, xs, keeps, tokens = _oracle_sample_inputs(shape)
    cores = host_cores()
    with OraclePool(cores, S0, xs, keeps, shape.G, shape.L) as pool:
        # a step gives every process about half a second of samples (sized in warm-up),
        # so that handing out the work is a small part of it
        per = 1
        for _ in range(args.warmup):
            t0 = time.perf_counter()
            pool.run_each(per)
            per = max(1, min(1000, round(per * 0.5 / max(time.perf_counter() - t0, 1e-3))))
        t0 = time.perf_counter()
        samples = 0
        for _ in range(args.steps):
            samples += pool.run_each(per)
        secs = time.perf_counter() - t0
    value = samples * tokens / secs
    sample = f"each step: {cores} processes x {per} x ({_sample_text(shape, tokens)})"
    spec = shape.max_pos > 1
    return {
        "impl": "reference", "metric": SPEC_METRIC if spec else METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3 / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": shape.name, "batch": shape.B, "heads": shape.H, "groups": shape.G, "P": shape.P,
                   "N": shape.N, "L": shape.L, "io": shape.io, "ckpt": shape.ckpt},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                         "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------ our arm, batch x window sweep

SWEEP_METRIC = "decode tokens/s per SSM layer, replay vs the in-house eager kernel, over batch x window x head layout (1 B200)"


def run_sweep_ours(args, rank, world, local):
    """Every point of gen.sweep_shapes(): replay_step in lockstep windows (host calls, and
    replays of one window captured in a CUDA graph) and eager_step, each over the same 256
    decode steps (256 / L windows), the median of three timed repetitions after one
    warm-up window. Per point: tokens/s of each, the replay/eager ratios and the fraction
    of the measured HBM bandwidth by the algorithmic bytes. Points whose checkpoint fits
    in L2 (126 MB) are marked: their steps re-read it from L2."""
    import linear_attention_decode_replay_b200 as lar

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream()
    peak, peak_kind = measured_hbm_peak()
    steps = 256

    def timed(fn, reps=3):
        out = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            out.append(e0.elapsed_time(e1))
        return statistics.median(out)

    points = []
    clocks = ClockSampler(local)
    clocks.start()
    for shape in gen.sweep_shapes(steps):
        L, B = shape.L, shape.B
        cfg = lar.Config(batch=B, heads=shape.H, groups=shape.G, P=shape.P, N=shape.N, L=L, max_pos=1,
                         io=shape.io, ckpt=shape.ckpt)
        bufs = lar.alloc_buffers(cfg, device)
        S0 = gen.initial_state(shape, device=device)
        bufs["S0"].copy_(S0)
        r = lar.Replay(cfg, bufs)
        window = [gen.step_inputs(shape, t, device=device) for t in range(L)]
        y = torch.empty(B, shape.H, shape.P, device=device)

        def replay_steps():
            for _ in range(steps // L):
                for x in window:
                    r.step(x["q"], x["k"], x["v"], x["dt"], x["a"], y=y)

        for x in window:
            r.step(x["q"], x["k"], x["v"], x["dt"], x["a"], y=y)
        replay_ms = max_over_ranks(timed(replay_steps), world, device)
        # the same steps as replays of one captured window (one graph launch per window
        # instead of one host call per step: the small-batch path)
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        with torch.cuda.graph(g, stream=side):
            for x in window:
                r.step(x["q"], x["k"], x["v"], x["dt"], x["a"], y=y)
        stream.wait_stream(side)
        torch.cuda.synchronize()

        def graph_steps():
            for _ in range(steps // L):
                g.replay()

        g.replay()
        graph_ms = max_over_ranks(timed(graph_steps), world, device)
        status_bits = r.check_status()
        del g
        r.close()
        del bufs
        S = S0

        def eager_steps():
            for j in range(steps):
                x = window[j % L]
                lar.eager_step(cfg, S, x["q"], x["k"], x["v"], x["dt"], x["a"], y=y)

        for x in window:
            lar.eager_step(cfg, S, x["q"], x["k"], x["v"], x["dt"], x["a"], y=y)
        eager_ms = max_over_ranks(timed(eager_steps), world, device)
        bpt = algorithmic_bytes_per_token(shape)
        tok = world * B * steps
        state_bytes = B * shape.H * shape.P * shape.N * 4
        points.append({
            "batch": B, "L": L, "heads": shape.H, "P": shape.P, "N": shape.N,
            "replay_tokens_s": tok / (replay_ms * 1e-3), "eager_tokens_s": tok / (eager_ms * 1e-3),
            "replay_graph_tokens_s": tok / (graph_ms * 1e-3),
            "speedup": eager_ms / replay_ms, "graph_speedup": eager_ms / graph_ms,
            "replay_frac": bpt["replay"] * B * steps / (replay_ms * 1e-3) / 1e9 / peak,
            "eager_frac": bpt["eager"] * B * steps / (eager_ms * 1e-3) / 1e9 / peak,
            "l2_resident": state_bytes <= 126 * 2**20,
            "status_bits": status_bits,  # device error bits after the replay runs (0 = none)
        })
        del S, S0, window, y
        torch.cuda.empty_cache()
    clk = clocks.stop()
    hbm = [p["speedup"] for p in points if not p["l2_resident"] and not p["status_bits"]]
    geo = float(np.exp(np.mean(np.log(hbm))))
    return {
        "metric": SWEEP_METRIC, "value": geo, "unit": "x (replay / eager tokens/s, geometric mean over the points whose state exceeds L2)",
        "n_gpus": world, "steps": steps, "warmup": 1, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "sweep", "batch": [1, 16, 64, 256, 1024], "L": [4, 8, 16, 32],
                   "heads_P": [[64, 64], [32, 128]], "N": 128, "io": "bf16", "ckpt": "f32",
                   "step": f"{steps} decode steps per point, median of 3",
                   "l2": "points with a checkpoint under 126 MB are L2-resident and marked"},
        "peak_gbs": peak, "peak_source": peak_kind, "clocks": clk, "points": points,
        "gpu_launches": 3 * 3 * steps * len(points),
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1500, help="timed windows of L decode steps")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="mamba2_b256",
                    choices=sorted(k for k in gen.SHAPES if k != "tiny") + ["sweep"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference" and args.workload == "sweep":
        ap.error("the sweep has no reference arm: --impl reference times the oracle on one workload")
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            out = run_reference(args, rank, world)
        elif args.workload == "sweep":
            out = run_sweep_ours(args, rank, world, local)
        elif gen.SHAPES[args.workload].max_pos > 1:
            out = run_spec_ours(args, rank, world, local)
        else:
            out = run_ours(args, rank, world, local)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
