"""Seeded input generators for the scalar-decay SSM decode workloads.

Every tensor here is drawn from a ``torch.Generator`` seeded from (workload seed,
stream, index), on whatever device the caller names. The CUDA path receives the
tensors directly; the oracle receives exact float64 copies of the very same values
(``to_numpy64``), so both sides always see identical inputs.

Distributions follow the workloads on the ReplaySSM pages ("ReplaySSM: Cache SSM
Inputs, Not State"; the blog's history form and the arXiv abstract's batch-256
serving setting):

* q, k ~ N(0, 1), L2-normalised over the k-dim N, then rounded to the I/O dtype;
* v ~ N(0, 1), rounded to the I/O dtype;
* Delta = softplus(N(0, 1)) in FP32;
* a = exp(-Delta * A) in FP32 with one rate A ~ U(0.5, 2) per head, shared by the batch;
* the initial checkpoint S0 is either N(0, 0.1^2) per element, or a state shaped like the
  end of a 4096-token random prefill (``initial_state(kind="prefill")``).

Nothing in this module evaluates the replay method itself.
"""

from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np
import torch
import torch.nn.functional as F

# stream ids keep the draws for different purposes independent
_STREAM_RATES = 1
_STREAM_STEP = 2
_STREAM_VERIFY = 3
_STREAM_S0 = 4
_STREAM_PREFILL = 5
_STREAM_ACCEPT = 6

PREFILL_TOKENS = 4096
# Tokens of the prefill that are actually summed. A token m positions before the end
# of the prefill is scaled by exp(-A * sum of the m later Deltas); with A >= 0.5 and
# E[Delta] = E[softplus(N(0,1))] ~= 0.81, the weight of every token more than 128
# positions back is below exp(-25) ~= 1e-11 of the newest one even 6 standard
# deviations into the tail of the sum, i.e. below FP32 resolution of the result.
PREFILL_TAIL = 128


@dataclass(frozen=True)
class Shape:
    """One decode workload: sizes, dtypes and seeds."""

    name: str
    B: int  # sequences
    H: int  # heads
    G: int  # k/q groups (G divides H)
    P: int  # v-dim (rows of the per-head state)
    N: int  # k-dim (columns of the per-head state)
    L: int  # window: buffer entries between two checkpoint flushes
    io: str = "bf16"  # dtype of q, k, v: "bf16" or "f32"
    ckpt: str = "f32"  # "f32", "f32_fp8read" or "f32_fp4read" (FP32 master + FP8 / FP4 read copy)
    max_pos: int = 1  # query positions per verify call (1 = plain decode)
    s0: str = "gauss"  # "gauss" or "prefill"
    steps: int = 32
    seed: int = 0

    def replace(self, **kw) -> "Shape":
        return dataclasses.replace(self, **kw)

    @property
    def io_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.io == "bf16" else torch.float32

    @property
    def io_bytes(self) -> int:
        return 2 if self.io == "bf16" else 4


# The workloads the method is evaluated on (sizes from the decode serving setting).
SHAPES = {
    # tiny case the oracle runs in full: replay vs eager every step
    "tiny": Shape("tiny", B=2, H=2, G=2, P=16, N=16, L=4, io="f32", steps=32, seed=0),
    # Mamba-2-like decode layer at serving batch 256
    "mamba2_b256": Shape("mamba2_b256", B=256, H=64, G=64, P=64, N=128, L=16,
                         io="bf16", s0="prefill", steps=512, seed=1000),
    # same layer, FP32 master checkpoint + FP8 e4m3 read copy
    "mamba2_b256_fp8": Shape("mamba2_b256_fp8", B=256, H=64, G=64, P=64, N=128, L=16,
                             io="bf16", ckpt="f32_fp8read", s0="prefill", steps=2048,
                             seed=2000),
    # same layer, FP32 master checkpoint + FP4 e2m1 read copy
    "mamba2_b256_fp4": Shape("mamba2_b256_fp4", B=256, H=64, G=64, P=64, N=128, L=16,
                             io="bf16", ckpt="f32_fp4read", s0="prefill", steps=2048,
                             seed=2500),
    # same layer with k and q shared by groups of 8 heads (8 groups)
    "mamba2_b256_g8": Shape("mamba2_b256_g8", B=256, H=64, G=8, P=64, N=128, L=16,
                            io="bf16", s0="prefill", steps=512, seed=1500),
    # speculative verify + rollback, draft length 4 (5 query positions)
    "mamba2_b256_spec": Shape("mamba2_b256_spec", B=256, H=64, G=64, P=64, N=128, L=16,
                              io="bf16", max_pos=5, s0="prefill", steps=256, seed=3000),
}


def sweep_shapes(steps: int = 256):
    """Batch x window x head-layout sweep (BF16 inputs, FP32 checkpoint)."""
    out = []
    for heads, P in ((64, 64), (32, 128)):
        for B in (1, 16, 64, 256, 1024):
            for L in (4, 8, 16, 32):
                out.append(Shape(f"sweep_b{B}_l{L}_h{heads}p{P}", B=B, H=heads, G=heads,
                                 P=P, N=128, L=L, io="bf16", s0="prefill", steps=steps,
                                 seed=4000 + B * 10 + L))
    return out


def _seed(base: int, stream: int, index: int) -> int:
    return (base * 1_000_003 + stream * 1_000_000_007 + index * 7_919 + 17) & 0x7FFF_FFFF_FFFF


def _gen(device, base: int, stream: int, index: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(base, stream, index))
    return g


def head_decay_rates(shape: Shape, device="cpu") -> torch.Tensor:
    """A ~ U(0.5, 2), one per head, FP32 [H]."""
    g = _gen(device, shape.seed, _STREAM_RATES, 0)
    return 0.5 + 1.5 * torch.rand(shape.H, generator=g, device=device, dtype=torch.float32)


def _draw_tokens(shape: Shape, g: torch.Generator, lead: tuple, device, rates):
    """One batch of decode inputs with leading dims ``lead`` (FP32, before I/O rounding)."""
    q = torch.randn(*lead, shape.G, shape.N, generator=g, device=device)
    k = torch.randn(*lead, shape.G, shape.N, generator=g, device=device)
    q = q / q.norm(dim=-1, keepdim=True)
    k = k / k.norm(dim=-1, keepdim=True)
    v = torch.randn(*lead, shape.H, shape.P, generator=g, device=device)
    dt = F.softplus(torch.randn(*lead, shape.H, generator=g, device=device))
    a = torch.exp(-dt * rates)
    return q, k, v, dt.contiguous(), a.contiguous()


def step_inputs(shape: Shape, step: int, device="cpu") -> dict:
    """Inputs of one decode step: q, k [B][G][N], v [B][H][P] (I/O dtype); dt, a [B][H] FP32."""
    g = _gen(device, shape.seed, _STREAM_STEP, step)
    rates = head_decay_rates(shape, device)
    q, k, v, dt, a = _draw_tokens(shape, g, (shape.B,), device, rates)
    t = shape.io_dtype
    return {"q": q.to(t).contiguous(), "k": k.to(t).contiguous(), "v": v.to(t).contiguous(),
            "dt": dt, "a": a}


def verify_inputs(shape: Shape, rnd: int, n_pos: int, device="cpu") -> dict:
    """Inputs of one verify call over n_pos positions: q, k [B][n_pos][G][N],
    v [B][n_pos][H][P] (I/O dtype); dt, a [B][n_pos][H] FP32."""
    g = _gen(device, shape.seed, _STREAM_VERIFY, rnd)
    rates = head_decay_rates(shape, device)
    q, k, v, dt, a = _draw_tokens(shape, g, (shape.B, n_pos), device, rates)
    t = shape.io_dtype
    return {"q": q.to(t).contiguous(), "k": k.to(t).contiguous(), "v": v.to(t).contiguous(),
            "dt": dt, "a": a}


def accepted_lengths(shape: Shape, rnd: int, n_pos: int, device="cpu") -> torch.Tensor:
    """Accepted draft length per sequence, uniform in {0, ..., n_pos - 1}; int32 [B]."""
    g = _gen(device, shape.seed, _STREAM_ACCEPT, rnd)
    return torch.randint(0, n_pos, (shape.B,), generator=g, device=device, dtype=torch.int32)


def initial_state(shape: Shape, device="cpu", kind: str | None = None,
                  batch_chunk: int = 16) -> torch.Tensor:
    """Initial checkpoint S0, FP32 [B][H][P][N] (row p of length N contiguous).

    kind="gauss":   every element ~ N(0, 0.1^2).
    kind="prefill": the state a sequence holds after a random 4096-token prefill drawn
                    from the decode distributions, i.e. a weighted sum of the prefill
                    tokens' outer products v k^T, the weight of a token being its Delta
                    times exp(-A * (sum of the Deltas of the later tokens)). Only the last
                    PREFILL_TAIL tokens carry weight above FP32 resolution and only they
                    are drawn. This is input synthesis done once, outside any timed
                    region; both the CUDA path and the oracle receive the result as input.
    """
    kind = kind or shape.s0
    B, H, G, P, N = shape.B, shape.H, shape.G, shape.P, shape.N
    if kind == "gauss":
        g = _gen(device, shape.seed, _STREAM_S0, 0)
        return 0.1 * torch.randn(B, H, P, N, generator=g, device=device)
    if kind != "prefill":
        raise ValueError(f"unknown initial state kind {kind!r}")
    rates = head_decay_rates(shape, device)
    out = torch.empty(B, H, P, N, device=device, dtype=torch.float32)
    T = PREFILL_TAIL
    hpg = H // G
    for b0 in range(0, B, batch_chunk):
        nb = min(batch_chunk, B - b0)
        g = _gen(device, shape.seed, _STREAM_PREFILL, b0)
        q, k, v, dt, a = _draw_tokens(shape, g, (nb, T), device, rates)
        del q, a
        # log-weight of token i = log(dt_i) - A * sum_{j > i} dt_j
        later = torch.flip(torch.cumsum(torch.flip(dt, [1]), 1), [1]) - dt  # [nb,T,H]
        w = dt * torch.exp(-later * rates)
        kh = k.repeat_interleave(hpg, dim=2)  # [nb,T,H,N]
        out[b0:b0 + nb] = torch.einsum("bthp,bthn->bhpn", v * w[..., None], kh)
    return out


def to_numpy64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy on the host (BF16 and FP32 widen exactly)."""
    if t.dtype in (torch.int32, torch.int64, torch.uint8, torch.bool):
        return t.detach().cpu().numpy()
    return t.detach().to("cpu", torch.float64).numpy()
