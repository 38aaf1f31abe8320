"""Host-side checks of the C ABI (no GPU needed): the library builds for
sm_100a, loads, exports every function include/bitnet.h declares, and rejects
bad arguments synchronously before touching any device."""
import ctypes as C

import pytest

import ternary_weight_i2_b200 as tw2
from ternary_weight_i2_b200 import _abi, build


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.load()


def test_exports_every_declared_function(lib):
    names = _abi.header_functions()
    assert len(names) >= 15
    for name in names:
        assert hasattr(lib, name), name
    # every bound signature is declared in the header too
    for name in _abi._SIGNATURES:
        assert name in names, name


def test_size_helpers(lib):
    assert tw2.packed_bytes(1536, 1536) == 1536 * 384
    assert tw2.packed_bytes(8960, 1536) == 3440640
    assert tw2.packed_bytes(1, 9024) == 32 * 71 == 2272
    assert tw2.packed_bytes(0, 5) == 0 and tw2.packed_bytes(3, 0) == 0
    assert tw2.packed_bytes(1, 65537) == 0
    assert tw2.kpad(1) == 128 and tw2.kpad(128) == 128 and tw2.kpad(129) == 256
    assert tw2.kpad(9024) == 9088
    assert tw2.linear_workspace_bytes(8, 1536) == 0
    assert tw2.linear_workspace_bytes(2048, 8960) >= 2048 * 8960 + 4 * 2048


def test_status_from_flags(lib):
    assert tw2.status_from_flags(0) == _abi.OK
    assert tw2.status_from_flags(tw2.FLAG_NOT_TERNARY) == _abi.ERR_NOT_TERNARY
    assert tw2.status_from_flags(tw2.FLAG_NONFINITE | tw2.FLAG_NOT_TERNARY) == _abi.ERR_NONFINITE
    assert tw2.status_from_flags(7) == _abi.ERR_TIMEOUT
    for s in range(8):
        assert lib.bitnet_status_str(s)


def _tw(ptr=0x1000, n=4, k=128, s=0.1):
    return _abi.TW(ptr, n, k, s)


def test_rejects_bad_arguments_before_any_device_call(lib):
    P = C.c_void_p
    good = P(0x10000)
    # pack: null, bad sizes, misaligned
    assert lib.bitnet_pack_ternary(None, 4, 4, good, None, None) == _abi.ERR_INVALID_ARG
    assert lib.bitnet_pack_ternary(good, 0, 4, good, None, None) == _abi.ERR_INVALID_ARG
    assert lib.bitnet_pack_ternary(good, 4, 65537, good, None, None) == _abi.ERR_INVALID_ARG
    assert lib.bitnet_pack_ternary(good, 4, 4, P(0x10001), None, None) == _abi.ERR_INVALID_ARG
    # quant
    assert lib.bitnet_quant_act(None, 1, 4, good, good, None, None) == _abi.ERR_INVALID_ARG
    assert lib.bitnet_quant_act(P(0x10004), 1, 4, good, good, None, None) == _abi.ERR_INVALID_ARG
    assert lib.bitnet_quant_act(good, 0, 4, good, good, None, None) == _abi.ERR_INVALID_ARG
    # linear: null weight pointer, misaligned, bad k, missing workspace
    w = _tw(ptr=0)
    assert lib.bitnet_linear(good, 1, C.byref(w), good, None, None, 0, None, None) == _abi.ERR_INVALID_ARG
    w = _tw(ptr=0x10008)
    assert lib.bitnet_linear(good, 1, C.byref(w), good, None, None, 0, None, None) == _abi.ERR_INVALID_ARG
    w = _tw(k=0)
    assert lib.bitnet_linear(good, 1, C.byref(w), good, None, None, 0, None, None) == _abi.ERR_INVALID_ARG
    w = _tw(k=1536)
    assert lib.bitnet_linear(good, 64, C.byref(w), good, None, None, 0, None, None) == _abi.ERR_WORKSPACE
    assert b"workspace" in lib.bitnet_last_error()
    # stack: count bounds and null entries
    xs = (C.c_void_p * 2)(0x10000, 0x10000)
    ys = (C.c_void_p * 2)(0x20000, None)
    ws = (_abi.TW * 2)(_tw(), _tw())
    assert lib.bitnet_linear_stack(xs, 1, ws, 0, ys, None, None, None) == _abi.ERR_INVALID_ARG
    assert lib.bitnet_linear_stack(xs, 1, ws, 257, ys, None, None, None) == _abi.ERR_INVALID_ARG
    assert lib.bitnet_linear_stack(xs, 1, ws, 2, ys, None, None, None) == _abi.ERR_INVALID_ARG
    assert b"NULL" in lib.bitnet_last_error()


def _has_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.mark.skipif(_has_gpu(), reason="checks the no-device path")
def test_no_device_is_an_error_not_a_silent_success(lib):
    """A well-formed call on a machine without a usable CUDA device must
    return an error: the library never reports success without running."""
    P = C.c_void_p
    st = lib.bitnet_pack_ternary(P(0x10000), 4, 4, P(0x20000), None, None)
    assert st in (_abi.ERR_CUDA, _abi.ERR_UNSUPPORTED_DEVICE)


def test_library_refuses_missing_build(tmp_path, monkeypatch):
    monkeypatch.setattr(_abi, "_lib", None)
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        _abi.load(str(tmp_path / "missing.so"))


def test_quantize_pack_rejects_bad_arguments_before_any_device_call(lib):
    P = C.c_void_p
    good = P(0x10000)
    ws_bytes = lib.bitnet_quantize_pack_workspace_bytes()
    assert ws_bytes == tw2.quantize_pack_workspace_bytes() >= 1024 * 12

    def call(w=good, n=4, k=4, packed=good, scale=good, ws=good, wsb=ws_bytes):
        return lib.bitnet_quantize_pack(w, n, k, packed, scale, ws, wsb, None, None)

    assert call(w=None) == _abi.ERR_INVALID_ARG
    assert call(scale=None) == _abi.ERR_INVALID_ARG
    assert call(ws=None) == _abi.ERR_INVALID_ARG
    assert call(n=0) == _abi.ERR_INVALID_ARG
    assert call(k=65537) == _abi.ERR_INVALID_ARG
    assert call(w=P(0x10002)) == _abi.ERR_INVALID_ARG          # fp32 input not 4-byte aligned
    assert call(packed=P(0x10004)) == _abi.ERR_INVALID_ARG     # packed rows need 16 bytes
    assert call(ws=P(0x10004)) == _abi.ERR_INVALID_ARG         # fp64 partials need 8 bytes
    assert call(wsb=ws_bytes - 1) == _abi.ERR_WORKSPACE
    assert b"workspace" in lib.bitnet_last_error()


def test_epilogue_descriptor_checked_before_any_device_call(lib):
    """A reserved field other than 0 or a misaligned operand is refused on
    every entry point that takes an epilogue, before the device is touched."""
    P = C.c_void_p
    good = P(0x10000)
    w = _tw()
    bad_reserved = _abi.Epilogue(None, None, None, 0, 1)
    bad_align = _abi.Epilogue(0x10002, None, None, 0, 0)
    for epi in (bad_reserved, bad_align):
        assert lib.bitnet_linear_ex(good, 1, C.byref(w), C.byref(epi), good, None, None, 0, None, None) \
            == _abi.ERR_INVALID_ARG
        assert lib.bitnet_linear_q_ex(good, good, 1, C.byref(w), C.byref(epi), good, None, None, None) \
            == _abi.ERR_INVALID_ARG
        xs = (C.c_void_p * 2)(0x10000, 0x10000)
        ys = (C.c_void_p * 2)(0x20000, 0x30000)
        ws = (_abi.TW * 2)(_tw(), _tw())
        epis = (_abi.Epilogue * 2)(_abi.Epilogue(), epi)   # the second layer's is bad
        assert lib.bitnet_linear_stack_ex(xs, 1, ws, epis, 2, ys, None, None, None) == _abi.ERR_INVALID_ARG
        assert b"layer 1" in lib.bitnet_last_error()
        assert lib.bitnet_linear_q_grouped_ex(xs, xs, 16, ws, epis, 2, ys, None, None, None) \
            == _abi.ERR_INVALID_ARG
    assert C.sizeof(_abi.Epilogue) == 32   # three pointers and two int32 (bitnet_epilogue)


@pytest.mark.skipif(_has_gpu(), reason="checks the no-device path")
def test_epilogue_forms_report_no_device(lib):
    """Well-formed epilogue calls on a machine without a usable CUDA device
    fail with a device error rather than succeeding silently."""
    P = C.c_void_p
    w = _tw()
    epi = _abi.Epilogue(0x40000, 0x50000, 0x60000, 1, 0)
    st = lib.bitnet_linear_ex(P(0x10000), 1, C.byref(w), C.byref(epi), P(0x20000), None, None, 0, None, None)
    assert st in (_abi.ERR_CUDA, _abi.ERR_UNSUPPORTED_DEVICE)
    st = lib.bitnet_quantize_pack(P(0x10000), 4, 4, P(0x20000), P(0x30000), P(0x40000),
                                  lib.bitnet_quantize_pack_workspace_bytes(), None, None)
    assert st in (_abi.ERR_CUDA, _abi.ERR_UNSUPPORTED_DEVICE)


def test_i8_sizes_and_grouped_workspace_layout(lib):
    assert tw2.i8_row_bytes(1) == 32 and tw2.i8_row_bytes(1536) == 1536 and tw2.i8_row_bytes(8961) == 8992
    assert tw2.i8_row_bytes(0) == 0 and tw2.i8_row_bytes(65537) == 0
    assert tw2.linear_i8_workspace_bytes(1, 1536) == 1536 + 4
    # inputs are shared when both the pointer and k match: A(1536), A(1536),
    # B(8960) and A(8960) are three distinct inputs
    xs = (C.c_void_p * 4)(0x10000, 0x10000, 0x20000, 0x10000)
    ws = (_abi.I8W * 4)(_abi.I8W(0x1000, 8, 1536, 1.0), _abi.I8W(0x1000, 8, 1536, 1.0),
                        _abi.I8W(0x1000, 8, 8960, 1.0), _abi.I8W(0x1000, 8, 8960, 1.0))
    per = {1536: 1536 + 256, 8960: 8960 + 256}   # int8 rows [1, kpad] then scales, each rounded to 256 bytes
    assert lib.bitnet_linear_i8_grouped_workspace_bytes(xs, 1, ws, 4) == per[1536] + 2 * per[8960]
    assert lib.bitnet_linear_i8_grouped_workspace_bytes(xs, 1, ws, 2) == per[1536]
    assert lib.bitnet_linear_i8_grouped_workspace_bytes(xs, 1, ws, 65) == 0
    # argument checks before any device call
    ys = (C.c_void_p * 4)(0x30000, 0x40000, 0x50000, 0x60000)
    big = lib.bitnet_linear_i8_grouped_workspace_bytes(xs, 1, ws, 4)
    assert lib.bitnet_linear_i8_grouped(xs, 1, ws, None, 4, ys, None, C.c_void_p(0x100000), big - 1, None,
                                        None) == _abi.ERR_WORKSPACE
    bad = (_abi.I8W * 1)(_abi.I8W(0x1008, 8, 1536, 1.0))
    assert lib.bitnet_linear_i8_grouped(xs, 1, bad, None, 1, ys, None, C.c_void_p(0x100000), big, None,
                                        None) == _abi.ERR_INVALID_ARG
