"""ReplaySSM decode path for scalar-decay (Mamba-2-style) SSM layers on B200.

A thin Python binding over the C ABI of ``include/replay.h`` (``libreplay.so``): every
step of the path runs in the library's CUDA kernels; this module only checks tensor
shapes and dtypes and passes device pointers and the current CUDA stream. PyTorch
provides device memory and streams.

    cfg = Config(batch=256, heads=64, groups=64, P=64, N=128, L=16)
    bufs = alloc_buffers(cfg, "cuda")          # caller-owned device buffers
    bufs["S0"].copy_(initial_checkpoint)
    r = Replay(cfg, bufs)
    y = r.step(q, k, v, dt, a)                 # one decode token per sequence
    y = r.verify(q5, k5, v5, dt5, a5)          # 5 speculative positions, output-only
    r.rollback(n_keep)                         # keep n_keep[b] of them (pointer move)
    r.flush()                                  # fold every buffer into the checkpoint

Small batches are bound by the host's launch rate; an even number of ``step`` calls on
fixed input and output tensors can be captured in a CUDA graph once one call has run
outside the capture (the conditions are in ``include/replay.h``). Each call flips which
half of the pointer words is current, so capture two windows when L is odd:

    r.step(q[0], k[0], v[0], dt[0], a[0], y=y[0])   # one call outside the capture
    n = cfg.L if cfg.L % 2 == 0 else 2 * cfg.L      # an even number of calls
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for t in range(n):
            r.step(q[t % cfg.L], k[t % cfg.L], v[t % cfg.L], dt[t % cfg.L], a[t % cfg.L], y=y[t % cfg.L])
    g.replay()                                       # n decode steps, one graph launch
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _abi
from ._abi import (  # noqa: F401
    DEV_POINTER,
    DEV_ROLLBACK,
    DEV_SNAPSHOT,
    DEV_WAIT_TIMEOUT,
    ReplayError,
    check,
    load,
    strerror,
)

__all__ = ["Config", "Replay", "alloc_buffers", "ring_capacity", "ring_record_bytes", "ring_k_record_bytes",
           "code_shape", "snapshot_bytes", "eager_step", "eager_step_fp8", "quantize_rows_e4m3", "quantize_rows_e2m1",
           "ReplayError", "load", "strerror"]


_CKPT = {"f32": _abi.REPLAY_CKPT_F32, "f32_fp8read": _abi.REPLAY_CKPT_F32_FP8READ,
         "f32_fp4read": _abi.REPLAY_CKPT_F32_FP4READ}


@dataclass(frozen=True)
class Config:
    """Sizes of one decode layer (see replay_config in include/replay.h)."""

    batch: int
    heads: int
    groups: int
    P: int
    N: int
    L: int
    max_pos: int = 1
    io: str = "bf16"  # "bf16" or "f32": dtype of q, k, v
    ckpt: str = "f32"  # "f32", "f32_fp8read" or "f32_fp4read"

    def c(self) -> _abi.CConfig:
        return _abi.CConfig(self.batch, self.heads, self.groups, self.P, self.N, self.L, self.max_pos,
                            _abi.REPLAY_BF16 if self.io == "bf16" else _abi.REPLAY_F32,
                            _CKPT[self.ckpt])

    @property
    def io_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.io == "bf16" else torch.float32


def ring_capacity(cfg: Config) -> int:
    cap = load().replay_ring_capacity(ctypes.byref(cfg.c()))
    if cap < 0:
        raise ReplayError(cap, "replay_ring_capacity")
    return cap


def ring_record_bytes(cfg: Config) -> int:
    """Bytes of one head record of the ring (v, Delta, a)."""
    r = load().replay_ring_record_bytes(ctypes.byref(cfg.c()))
    if r < 0:
        raise ReplayError(r, "replay_ring_record_bytes")
    return r


def ring_k_record_bytes(cfg: Config) -> int:
    """Bytes of one k record of the ring (one per k/q group)."""
    r = load().replay_ring_k_record_bytes(ctypes.byref(cfg.c()))
    if r < 0:
        raise ReplayError(r, "replay_ring_k_record_bytes")
    return r


def code_shape(cfg: Config):
    """Shape of the read copy's codes (uint8): FP8 one byte per value, FP4 two values per byte."""
    n = cfg.N // 2 if cfg.ckpt == "f32_fp4read" else cfg.N
    return (cfg.batch, cfg.heads, cfg.P, n)


def snapshot_bytes(cfg: Config) -> int:
    """Bytes of one sequence's snapshot (replay_export / replay_import)."""
    r = load().replay_snapshot_bytes(ctypes.byref(cfg.c()))
    if r < 0:
        raise ReplayError(r, "replay_snapshot_bytes")
    return r


def alloc_buffers(cfg: Config, device="cuda") -> dict:
    """Allocates the caller-owned device buffers of one layer (S0 left uninitialised)."""
    cap = ring_capacity(cfg)
    rec = ring_record_bytes(cfg)
    rk = ring_k_record_bytes(cfg)
    B, H, G, P, N = cfg.batch, cfg.heads, cfg.groups, cfg.P, cfg.N
    bufs = {
        "S0": torch.empty(B, H, P, N, device=device, dtype=torch.float32),
        "ring_k": torch.zeros(B, G, cap, rk, device=device, dtype=torch.uint8),
        "ring": torch.zeros(B, H, cap, rec, device=device, dtype=torch.uint8),
        "counts": torch.zeros(2, B, device=device, dtype=torch.int32),
        "status": torch.zeros(1, device=device, dtype=torch.int32),
    }
    if cfg.max_pos > 1:
        bufs["qpack"] = torch.empty(B, G, cfg.max_pos, N, device=device, dtype=cfg.io_dtype)
    if cfg.ckpt != "f32":
        bufs["S0_codes"] = torch.empty(code_shape(cfg), device=device, dtype=torch.uint8)
        bufs["S0_scale"] = torch.empty(B, H, P, device=device, dtype=torch.float32)
    return bufs


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t, shape=None, dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


class Replay:
    """One decode layer's checkpoint + buffer state, over caller-owned device buffers."""

    def __init__(self, cfg: Config, buffers: dict, stream=None):
        self.cfg = cfg
        self.buffers = buffers
        lib = load()
        B, H, G, P, N = cfg.batch, cfg.heads, cfg.groups, cfg.P, cfg.N
        cap = ring_capacity(cfg)
        copy = cfg.ckpt != "f32"
        rec = ring_record_bytes(cfg)
        rk = ring_k_record_bytes(cfg)
        cb = _abi.CBuffers(
            _ptr(buffers["S0"], (B, H, P, N), torch.float32, "S0"),
            _ptr(buffers.get("S0_codes"), code_shape(cfg), torch.uint8, "S0_codes") if copy else None,
            _ptr(buffers.get("S0_scale"), (B, H, P), torch.float32, "S0_scale") if copy else None,
            _ptr(buffers["ring_k"], (B, G, cap, rk), torch.uint8, "ring_k"),
            _ptr(buffers["ring"], (B, H, cap, rec), torch.uint8, "ring"),
            _ptr(buffers.get("qpack"), (B, G, cfg.max_pos, N), cfg.io_dtype, "qpack") if cfg.max_pos > 1 else None,
            _ptr(buffers["counts"], (2, B), torch.int32, "counts"),
            _ptr(buffers["status"], (1,), torch.int32, "status"),
        )
        self._ctx = ctypes.c_void_p()
        check(lib.replay_init(ctypes.byref(cfg.c()), ctypes.byref(cb), _stream(stream),
                              ctypes.byref(self._ctx)), "replay_init")
        self._lib = lib

    def _token_shapes(self, n_pos):
        B, H, G, P, N = self.cfg.batch, self.cfg.heads, self.cfg.groups, self.cfg.P, self.cfg.N
        lead = (B,) if n_pos is None else (B, n_pos)
        return (*lead, G, N), (*lead, H, P), (*lead, H)

    def step(self, q, k, v, dt, a, y=None, flushed=None, stream=None):
        """One decode token per sequence; returns y [B][H][P] FP32."""
        qs, vs, ds = self._token_shapes(None)
        t = self.cfg.io_dtype
        if y is None:
            y = torch.empty(vs, device=q.device, dtype=torch.float32)
        check(self._lib.replay_step(self._ctx, _ptr(q, qs, t, "q"), _ptr(k, qs, t, "k"), _ptr(v, vs, t, "v"),
                                    _ptr(dt, ds, torch.float32, "dt"), _ptr(a, ds, torch.float32, "a"),
                                    _ptr(y, vs, torch.float32, "y"),
                                    _ptr(flushed, (self.cfg.batch,), torch.uint8, "flushed"), _stream(stream)),
              "replay_step")
        return y

    def verify(self, q, k, v, dt, a, y=None, flushed=None, stream=None):
        """Output-only scoring of n_pos = q.shape[1] positions; returns y [B][n_pos][H][P]."""
        n_pos = q.shape[1]
        qs, vs, ds = self._token_shapes(n_pos)
        t = self.cfg.io_dtype
        if y is None:
            y = torch.empty(vs, device=q.device, dtype=torch.float32)
        check(self._lib.replay_verify(self._ctx, n_pos, _ptr(q, qs, t, "q"), _ptr(k, qs, t, "k"),
                                      _ptr(v, vs, t, "v"), _ptr(dt, ds, torch.float32, "dt"),
                                      _ptr(a, ds, torch.float32, "a"), _ptr(y, vs, torch.float32, "y"),
                                      _ptr(flushed, (self.cfg.batch,), torch.uint8, "flushed"), _stream(stream)),
              "replay_verify")
        return y

    def verify_static_scratch(self, q, k, v, dt, a, y=None, flushed=None, stream=None):
        """verify() for callers that cannot allocate device memory: the queries are packed
        into the library's fixed 32 MiB device array instead of the qpack buffer, so the
        layer needs no qpack (max_pos = 1 works; n_pos above max_pos first folds the
        buffers too full to take the new entries). Calls that overlap on the GPU share
        that array and race. Pass `y` to keep this binding from allocating the output."""
        n_pos = q.shape[1]
        qs, vs, ds = self._token_shapes(n_pos)
        t = self.cfg.io_dtype
        if y is None:
            y = torch.empty(vs, device=q.device, dtype=torch.float32)
        check(self._lib.replay_verify_static_scratch(
            self._ctx, n_pos, _ptr(q, qs, t, "q"), _ptr(k, qs, t, "k"), _ptr(v, vs, t, "v"),
            _ptr(dt, ds, torch.float32, "dt"), _ptr(a, ds, torch.float32, "a"), _ptr(y, vs, torch.float32, "y"),
            _ptr(flushed, (self.cfg.batch,), torch.uint8, "flushed"), _stream(stream)),
            "replay_verify_static_scratch")
        return y

    def append_slots(self, slots=None, stream=None):
        """Ring record of every sequence's next entry (int32 [B] on the device, written on
        the stream): position s of head h of sequence b goes to record (slots[b] + s) % cap
        of ring[b][h]. For callers that write the entries there themselves and then call
        step_resident / verify_resident."""
        if slots is None:
            slots = torch.empty(self.cfg.batch, device=self.buffers["counts"].device, dtype=torch.int32)
        check(self._lib.replay_append_slots(self._ctx, _ptr(slots, (self.cfg.batch,), torch.int32, "slots"),
                                            _stream(stream)), "replay_append_slots")
        return slots

    def step_resident(self, q, y=None, flushed=None, stream=None):
        """step() whose entry the caller already wrote into the ring at append_slots()."""
        qs, vs, _ = self._token_shapes(None)
        if y is None:
            y = torch.empty(vs, device=q.device, dtype=torch.float32)
        check(self._lib.replay_step_resident(self._ctx, _ptr(q, qs, self.cfg.io_dtype, "q"),
                                             _ptr(y, vs, torch.float32, "y"),
                                             _ptr(flushed, (self.cfg.batch,), torch.uint8, "flushed"),
                                             _stream(stream)), "replay_step_resident")
        return y

    def verify_resident(self, q, y=None, flushed=None, stream=None):
        """verify() whose n_pos = q.shape[1] entries the caller already wrote into the ring."""
        n_pos = q.shape[1]
        qs, vs, _ = self._token_shapes(n_pos)
        if y is None:
            y = torch.empty(vs, device=q.device, dtype=torch.float32)
        check(self._lib.replay_verify_resident(self._ctx, n_pos, _ptr(q, qs, self.cfg.io_dtype, "q"),
                                               _ptr(y, vs, torch.float32, "y"),
                                               _ptr(flushed, (self.cfg.batch,), torch.uint8, "flushed"),
                                               _stream(stream)), "replay_verify_resident")
        return y

    def export(self, seqs, dst=None, stream=None):
        """Snapshots of the sequences seqs (int32 [n] on the device) into dst (uint8 [n,
        snapshot_bytes] on the device, allocated here if None); returns dst."""
        n = seqs.shape[0]
        nb = snapshot_bytes(self.cfg)
        if dst is None:
            dst = torch.empty(n, nb, device=seqs.device, dtype=torch.uint8)
        check(self._lib.replay_export(self._ctx, _ptr(seqs, (n,), torch.int32, "seqs"), n,
                                      _ptr(dst, (n, nb), torch.uint8, "dst"), _stream(stream)), "replay_export")
        return dst

    def import_(self, seqs, src, stream=None):
        """Restores snapshot i of src (uint8 [n, snapshot_bytes]) into sequence seqs[i]."""
        n = seqs.shape[0]
        check(self._lib.replay_import(self._ctx, _ptr(seqs, (n,), torch.int32, "seqs"), n,
                                      _ptr(src, (n, snapshot_bytes(self.cfg)), torch.uint8, "src"), _stream(stream)),
              "replay_import")

    def rollback(self, n_keep, stream=None):
        """Keep n_keep[b] (int32 [B] on the device) of the pending verify's positions."""
        check(self._lib.replay_rollback(self._ctx, _ptr(n_keep, (self.cfg.batch,), torch.int32, "n_keep"),
                                        _stream(stream)), "replay_rollback")

    def flush(self, mask=None, stream=None):
        """Fold the buffers of the sequences with mask[b] != 0 (uint8 [B]; None = all)."""
        check(self._lib.replay_flush(self._ctx, _ptr(mask, (self.cfg.batch,), torch.uint8, "mask"),
                                     _stream(stream)), "replay_flush")

    def read_counts(self, stream=None):
        """Committed entries per sequence (synchronises the stream)."""
        out = (ctypes.c_int32 * self.cfg.batch)()
        check(self._lib.replay_read_counts(self._ctx, ctypes.cast(out, ctypes.c_void_p), _stream(stream)),
              "replay_read_counts")
        return list(out)

    def check_status(self, stream=None) -> int:
        """Device error bits (0 = none); synchronises the stream."""
        bits = ctypes.c_int32(0)
        rc = self._lib.replay_check_status(self._ctx, ctypes.byref(bits), _stream(stream))
        if rc not in (_abi.REPLAY_OK, _abi.REPLAY_EDEVICE):
            raise ReplayError(rc, "replay_check_status")
        return bits.value

    def close(self):
        if getattr(self, "_ctx", None) and self._ctx.value:
            self._lib.replay_destroy(self._ctx)
            self._ctx = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001 - interpreter shutdown
            pass


def eager_step(cfg: Config, S, q, k, v, dt, a, y=None, stream=None):
    """Baseline eager step: S <- a S + dt v k^T (in place), y = S q."""
    B, H, G, P, N = cfg.batch, cfg.heads, cfg.groups, cfg.P, cfg.N
    t = cfg.io_dtype
    if y is None:
        y = torch.empty(B, H, P, device=S.device, dtype=torch.float32)
    check(load().eager_step(ctypes.byref(cfg.c()), _ptr(S, (B, H, P, N), torch.float32, "S"),
                            _ptr(q, (B, G, N), t, "q"), _ptr(k, (B, G, N), t, "k"), _ptr(v, (B, H, P), t, "v"),
                            _ptr(dt, (B, H), torch.float32, "dt"), _ptr(a, (B, H), torch.float32, "a"),
                            _ptr(y, (B, H, P), torch.float32, "y"), _stream(stream)), "eager_step")
    return y


def eager_step_fp8(cfg: Config, S8, scale, q, k, v, dt, a, y=None, stream=None):
    """Baseline eager step on a shared FP8 e4m3 state with per-row scales (in place)."""
    B, H, G, P, N = cfg.batch, cfg.heads, cfg.groups, cfg.P, cfg.N
    t = cfg.io_dtype
    if y is None:
        y = torch.empty(B, H, P, device=S8.device, dtype=torch.float32)
    check(load().eager_step_fp8(ctypes.byref(cfg.c()), _ptr(S8, (B, H, P, N), torch.uint8, "S8"),
                                _ptr(scale, (B, H, P), torch.float32, "scale"), _ptr(q, (B, G, N), t, "q"),
                                _ptr(k, (B, G, N), t, "k"), _ptr(v, (B, H, P), t, "v"),
                                _ptr(dt, (B, H), torch.float32, "dt"), _ptr(a, (B, H), torch.float32, "a"),
                                _ptr(y, (B, H, P), torch.float32, "y"), _stream(stream)), "eager_step_fp8")
    return y


def quantize_rows_e2m1(x, codes=None, scale=None, stream=None):
    """Per-row e2m1 codes (two per byte, element 2i in the low nibble) and FP32 scales of
    x [..., n] (FP32, n in 16/32/64/128)."""
    n = x.shape[-1]
    rows = x.numel() // n
    cshape = (*x.shape[:-1], n // 2)
    if codes is None:
        codes = torch.empty(cshape, device=x.device, dtype=torch.uint8)
    if scale is None:
        scale = torch.empty(x.shape[:-1], device=x.device, dtype=torch.float32)
    check(load().replay_quantize_rows_e2m1(_ptr(x, None, torch.float32, "x"), rows, n,
                                           _ptr(codes, cshape, torch.uint8, "codes"),
                                           _ptr(scale, x.shape[:-1], torch.float32, "scale"), _stream(stream)),
          "replay_quantize_rows_e2m1")
    return codes, scale


def quantize_rows_e4m3(x, codes=None, scale=None, stream=None):
    """Per-row e4m3 codes and FP32 scales of x [..., n] (FP32, n in 16/32/64/128)."""
    n = x.shape[-1]
    rows = x.numel() // n
    if codes is None:
        codes = torch.empty(x.shape, device=x.device, dtype=torch.uint8)
    if scale is None:
        scale = torch.empty(x.shape[:-1], device=x.device, dtype=torch.float32)
    check(load().replay_quantize_rows_e4m3(_ptr(x, None, torch.float32, "x"), rows, n,
                                           _ptr(codes, x.shape, torch.uint8, "codes"),
                                           _ptr(scale, x.shape[:-1], torch.float32, "scale"), _stream(stream)),
          "replay_quantize_rows_e4m3")
    return codes, scale
