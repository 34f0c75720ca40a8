"""The C-ABI library loads and exports every function that include/replay.h declares,
and its host-side argument checks answer without touching a GPU (no compute calls)."""

import ctypes
import os
import re

import pytest

import linear_attention_decode_replay_b200 as lar
from linear_attention_decode_replay_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "replay.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?(?:int|int32_t|int64_t|void|char)\s*\*?\s*(\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("replay_init", "replay_step", "replay_verify", "replay_rollback", "replay_flush",
                 "replay_read_counts", "replay_check_status", "replay_destroy", "eager_step",
                 "eager_step_fp8", "replay_quantize_rows_e4m3", "replay_ring_capacity", "replay_ring_record_bytes",
                 "replay_strerror", "replay_append_slots", "replay_step_resident", "replay_verify_resident",
                 "replay_verify_static_scratch", "replay_snapshot_bytes", "replay_export", "replay_import",
                 "replay_ring_k_record_bytes", "replay_quantize_rows_e2m1"):
        assert want in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(_abi.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def _cfg(**kw):
    base = dict(batch=2, heads=4, groups=2, P=16, N=16, L=4, max_pos=2, io=_abi.REPLAY_F32,
                ckpt=_abi.REPLAY_CKPT_F32)
    base.update(kw)
    return _abi.CConfig(**base)


def test_ring_capacity_and_config_checks():
    lib = _abi.load()
    assert lib.replay_ring_capacity(ctypes.byref(_cfg())) == 6  # L + max_pos
    assert lib.replay_ring_capacity(ctypes.byref(_cfg(L=16, max_pos=1))) == 17
    assert lib.replay_ring_capacity(ctypes.byref(_cfg(L=16, max_pos=5))) == 21
    # head record: v (P io) + Delta + a, padded to 16 bytes; k record: k (N io), once per group
    assert lib.replay_ring_record_bytes(ctypes.byref(_cfg())) == 80  # 16 * 4 + 8 -> 80
    assert lib.replay_ring_record_bytes(ctypes.byref(_cfg(P=64, N=128, io=_abi.REPLAY_BF16))) == 144  # 136 -> 144
    assert lib.replay_ring_k_record_bytes(ctypes.byref(_cfg())) == 64 + 16  # k, then 16 bytes of padding
    assert lib.replay_ring_k_record_bytes(ctypes.byref(_cfg(P=64, N=128, io=_abi.REPLAY_BF16))) == 256 + 16
    for bad in (dict(groups=3), dict(P=12), dict(P=0), dict(N=48), dict(N=256), dict(L=0),
                dict(max_pos=9), dict(max_pos=5, L=4), dict(io=7), dict(ckpt=3), dict(ckpt=-1), dict(batch=0),
                dict(P=256, N=128)):
        assert lib.replay_ring_capacity(ctypes.byref(_cfg(**bad))) == _abi.REPLAY_EINVAL, bad
        assert lib.replay_ring_record_bytes(ctypes.byref(_cfg(**bad))) == _abi.REPLAY_EINVAL, bad
        assert lib.replay_ring_k_record_bytes(ctypes.byref(_cfg(**bad))) == _abi.REPLAY_EINVAL, bad


def test_snapshot_bytes():
    lib = _abi.load()
    # header 64 + H*P*N*4 + G*L*RK + H*L*R
    assert lib.replay_snapshot_bytes(ctypes.byref(_cfg())) == 64 + 4 * 16 * 16 * 4 + 2 * 4 * 80 + 4 * 4 * 80
    big = _cfg(batch=256, heads=64, groups=64, P=64, N=128, L=16, max_pos=1, io=_abi.REPLAY_BF16)
    assert lib.replay_snapshot_bytes(ctypes.byref(big)) == 64 + 64 * 64 * 128 * 4 + 64 * 16 * 272 + 64 * 16 * 144
    shared = _cfg(batch=256, heads=64, groups=8, P=64, N=128, L=16, max_pos=1, io=_abi.REPLAY_BF16)
    assert lib.replay_snapshot_bytes(ctypes.byref(shared)) == 64 + 64 * 64 * 128 * 4 + 8 * 16 * 272 + 64 * 16 * 144
    assert lib.replay_snapshot_bytes(ctypes.byref(_cfg(groups=3))) == _abi.REPLAY_EINVAL


def test_init_rejects_bad_arguments_before_any_cuda_call():
    lib = _abi.load()
    ctx = ctypes.c_void_p()
    good = ctypes.c_void_p(0x10000)
    bufs = _abi.CBuffers(good, None, None, good, good, good, good, good)
    assert lib.replay_init(ctypes.byref(_cfg(groups=3)), ctypes.byref(bufs), None, ctypes.byref(ctx)) == \
        _abi.REPLAY_EINVAL
    nulls = _abi.CBuffers(None, None, None, good, good, good, good, good)
    assert lib.replay_init(ctypes.byref(_cfg()), ctypes.byref(nulls), None, ctypes.byref(ctx)) == _abi.REPLAY_EINVAL
    no_ring_k = _abi.CBuffers(good, None, None, None, good, good, good, good)
    assert lib.replay_init(ctypes.byref(_cfg()), ctypes.byref(no_ring_k), None, ctypes.byref(ctx)) == \
        _abi.REPLAY_EINVAL
    assert lib.replay_init(ctypes.byref(_cfg()), ctypes.byref(nulls), None, ctypes.byref(ctx)) == _abi.REPLAY_EINVAL
    odd = _abi.CBuffers(ctypes.c_void_p(0x10008), None, None, good, good, good, good, good)
    assert lib.replay_init(ctypes.byref(_cfg()), ctypes.byref(odd), None, ctypes.byref(ctx)) == _abi.REPLAY_EALIGN
    codes_missing = _abi.CBuffers(good, None, None, good, good, good, good, good)
    for ckpt in (_abi.REPLAY_CKPT_F32_FP8READ, _abi.REPLAY_CKPT_F32_FP4READ):
        assert lib.replay_init(ctypes.byref(_cfg(ckpt=ckpt)), ctypes.byref(codes_missing), None,
                               ctypes.byref(ctx)) == _abi.REPLAY_EINVAL
    no_qpack = _abi.CBuffers(good, None, None, good, good, None, good, good)
    assert lib.replay_init(ctypes.byref(_cfg(max_pos=2)), ctypes.byref(no_qpack), None, ctypes.byref(ctx)) == \
        _abi.REPLAY_EINVAL
    assert not ctx.value


def test_calls_on_a_null_context_are_rejected():
    lib = _abi.load()
    p = ctypes.c_void_p(0x10000)
    assert lib.replay_step(None, p, p, p, p, p, p, None, None) == _abi.REPLAY_EINVAL
    assert lib.replay_verify(None, 2, p, p, p, p, p, p, None, None) == _abi.REPLAY_EINVAL
    assert lib.replay_rollback(None, p, None) == _abi.REPLAY_EINVAL
    assert lib.replay_flush(None, None, None) == _abi.REPLAY_EINVAL
    assert lib.replay_read_counts(None, p, None) == _abi.REPLAY_EINVAL
    assert lib.replay_check_status(None, None, None) == _abi.REPLAY_EINVAL
    assert lib.replay_append_slots(None, p, None) == _abi.REPLAY_EINVAL
    assert lib.replay_step_resident(None, p, p, None, None) == _abi.REPLAY_EINVAL
    assert lib.replay_verify_resident(None, 2, p, p, None, None) == _abi.REPLAY_EINVAL
    assert lib.replay_export(None, p, 1, p, None) == _abi.REPLAY_EINVAL
    assert lib.replay_import(None, p, 1, p, None) == _abi.REPLAY_EINVAL
    lib.replay_destroy(None)


def test_eager_and_quantize_argument_checks():
    lib = _abi.load()
    p = ctypes.c_void_p(0x10000)
    assert lib.eager_step(ctypes.byref(_cfg(N=20)), p, p, p, p, p, p, p, None) == _abi.REPLAY_EINVAL
    assert lib.eager_step(ctypes.byref(_cfg()), None, p, p, p, p, p, p, None) == _abi.REPLAY_EINVAL
    assert lib.eager_step(ctypes.byref(_cfg()), ctypes.c_void_p(0x10004), p, p, p, p, p, p, None) == \
        _abi.REPLAY_EALIGN
    assert lib.eager_step_fp8(ctypes.byref(_cfg()), p, None, p, p, p, p, p, p, None) == _abi.REPLAY_EINVAL
    assert lib.replay_quantize_rows_e4m3(p, 4, 24, p, p, None) == _abi.REPLAY_EINVAL
    assert lib.replay_quantize_rows_e4m3(p, 0, 16, p, p, None) == _abi.REPLAY_OK  # nothing to do
    assert lib.replay_quantize_rows_e2m1(p, 4, 24, p, p, None) == _abi.REPLAY_EINVAL
    assert lib.replay_quantize_rows_e2m1(p, 0, 16, p, p, None) == _abi.REPLAY_OK


def test_strerror_covers_every_code():
    for code in range(0, -9, -1):
        assert lar.strerror(code) != "unknown status"
    assert lar.strerror(-99) == "unknown status"


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_abi, "_lib", None)
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        _abi.load()
