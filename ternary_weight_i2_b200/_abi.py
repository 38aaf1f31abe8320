"""ctypes binding of the C ABI in ``include/bitnet.h`` (libbitnet.so).

Argument marshalling only: every step of the layer runs in the CUDA kernels
behind the ABI.  Tensors are passed as raw device pointers (``data_ptr()``)
and the stream as the handle of ``torch.cuda.current_stream()`` unless one is
given.  If the library is missing the first call raises: there is no CPU path.
"""
from __future__ import annotations

import ctypes as C
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbitnet.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "bitnet.h")

OK, ERR_INVALID_ARG, ERR_NOT_TERNARY, ERR_UNSUPPORTED_DEVICE = 0, 1, 2, 3
ERR_CUDA, ERR_NONFINITE, ERR_TIMEOUT, ERR_WORKSPACE = 4, 5, 6, 7
FLAG_NOT_TERNARY, FLAG_NONFINITE, FLAG_TIMEOUT = 0x1, 0x2, 0x4
GEMV_MAX_M = 8
STACK_MAX = 256
MAX_K = 65536


class TW(C.Structure):
    """bitnet_tw: one packed ternary weight tensor (device pointer + shape + scale)."""
    _fields_ = [("packed", C.c_void_p), ("n", C.c_int64), ("k", C.c_int64), ("scale", C.c_float)]


class I8W(C.Structure):
    """bitnet_i8w: one I8_S int8 weight tensor (device pointer + shape + scale)."""
    _fields_ = [("w", C.c_void_p), ("n", C.c_int64), ("k", C.c_int64), ("scale", C.c_float)]


class Epilogue(C.Structure):
    """bitnet_epilogue: fused bias / ReLU / layer-scaled residual add (device
    pointers, NULL = step skipped)."""
    _fields_ = [("bias", C.c_void_p), ("gamma", C.c_void_p), ("residual", C.c_void_p),
                ("relu", C.c_int32), ("reserved", C.c_int32)]


class BitnetError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(what)


_P, _I64, _I32 = C.c_void_p, C.c_int64, C.c_int32
_SIGNATURES = {
    "bitnet_version": ([], C.c_int),
    "bitnet_status_str": ([C.c_int], C.c_char_p),
    "bitnet_last_error": ([], C.c_char_p),
    "bitnet_status_from_flags": ([_I32], C.c_int),
    "bitnet_packed_bytes": ([_I64, _I64], C.c_size_t),
    "bitnet_kpad": ([_I64], _I64),
    "bitnet_pack_ternary": ([_P, _I64, _I64, _P, _P, _P], C.c_int),
    "bitnet_unpack_ternary": ([_P, _I64, _I64, _P, _P], C.c_int),
    "bitnet_quantize_pack_workspace_bytes": ([], C.c_size_t),
    "bitnet_quantize_pack": ([_P, _I64, _I64, _P, _P, _P, C.c_size_t, _P, _P], C.c_int),
    "bitnet_quant_act": ([_P, _I64, _I64, _P, _P, _P, _P], C.c_int),
    "bitnet_linear_workspace_bytes": ([_I64, _I64], C.c_size_t),
    "bitnet_linear": ([_P, _I64, C.POINTER(TW), _P, _P, _P, C.c_size_t, _P, _P], C.c_int),
    "bitnet_linear_q": ([_P, _P, _I64, C.POINTER(TW), _P, _P, _P, _P], C.c_int),
    "bitnet_linear_stack": ([_P, _I64, C.POINTER(TW), _I64, _P, _P, _P, _P], C.c_int),
    "bitnet_linear_q_grouped": ([_P, _P, _I64, C.POINTER(TW), _I64, _P, _P, _P, _P], C.c_int),
    "bitnet_linear_stack_noalloc": ([_P, _I64, C.POINTER(TW), _I64, _P, _P, _P, _P], C.c_int),
    "bitnet_linear_ex": ([_P, _I64, C.POINTER(TW), C.POINTER(Epilogue), _P, _P, _P, C.c_size_t, _P, _P], C.c_int),
    "bitnet_linear_q_ex": ([_P, _P, _I64, C.POINTER(TW), C.POINTER(Epilogue), _P, _P, _P, _P], C.c_int),
    "bitnet_linear_q_grouped_ex": ([_P, _P, _I64, C.POINTER(TW), C.POINTER(Epilogue), _I64, _P, _P, _P, _P],
                                   C.c_int),
    "bitnet_linear_stack_ex": ([_P, _I64, C.POINTER(TW), C.POINTER(Epilogue), _I64, _P, _P, _P, _P], C.c_int),
    "bitnet_i8_row_bytes": ([_I64], C.c_size_t),
    "bitnet_linear_i8_workspace_bytes": ([_I64, _I64], C.c_size_t),
    "bitnet_linear_i8": ([_P, _I64, C.POINTER(I8W), C.POINTER(Epilogue), _P, _P, _P, C.c_size_t, _P, _P], C.c_int),
    "bitnet_linear_i8_grouped_workspace_bytes": ([_P, _I64, C.POINTER(I8W), _I64], C.c_size_t),
    "bitnet_linear_i8_grouped": ([_P, _I64, C.POINTER(I8W), C.POINTER(Epilogue), _I64, _P, _P, _P, C.c_size_t,
                                  _P, _P], C.c_int),
    "bitnet_debug_set_wait_limit": ([C.c_uint64], C.c_int),
    "bitnet_debug_force_stall": ([C.c_int], C.c_int),
    "bitnet_debug_set_trace": ([_P], C.c_int),
    "bitnet_release_device_cache": ([], C.c_int),
}

_lib = None


def header_functions() -> list[str]:
    """Names of every function ``include/bitnet.h`` declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bitnet_[a-z0-9_]+)\s*\(", text)))


def load(path: str | None = None) -> C.CDLL:
    """Load libbitnet.so (and bind every signature).  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libbitnet.so not built ({p}); run __graft_entry__.build() "
                           "or python ternary_weight_i2_b200/build.py -- there is no CPU fallback")
    lib = C.CDLL(p)
    for name, (args, ret) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes, fn.restype = args, ret
    _lib = lib
    return lib


def _check(status: int, what: str):
    if status != OK:
        lib = load()
        detail = lib.bitnet_last_error().decode(errors="replace")
        name = lib.bitnet_status_str(status).decode()
        raise BitnetError(status, f"{what}: {name} ({detail})")


def _stream(stream):
    if stream is None:
        import torch
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return C.c_void_p(stream)
    return C.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


# ------------------------------------------------------------------ helpers

def version() -> int:
    return load().bitnet_version()


def packed_bytes(n: int, k: int) -> int:
    return int(load().bitnet_packed_bytes(n, k))


def kpad(k: int) -> int:
    return int(load().bitnet_kpad(k))


def status_from_flags(flags: int) -> int:
    return int(load().bitnet_status_from_flags(int(flags)))


def linear_workspace_bytes(m: int, k: int) -> int:
    return int(load().bitnet_linear_workspace_bytes(m, k))


def release_device_cache() -> None:
    _check(load().bitnet_release_device_cache(), "bitnet_release_device_cache")


def set_wait_limit(cycles: int) -> None:
    _check(load().bitnet_debug_set_wait_limit(int(cycles)), "set_wait_limit")


def set_trace(buf) -> None:
    """Profiling aid: per-warp phase timestamps of later GEMV launches go to
    ``buf`` (a uint64/int64 device tensor of 8*16*160 entries), None to stop."""
    _check(load().bitnet_debug_set_trace(_ptr(buf)), "set_trace")


def force_stall(on: bool) -> None:
    _check(load().bitnet_debug_force_stall(1 if on else 0), "force_stall")


# ------------------------------------------------------------ the entry points

def pack_ternary(w, packed, flags=None, stream=None) -> None:
    """w: int8 [n,k] device tensor -> packed uint8 [n, 32*ceil(k/128)]."""
    n, k = w.shape
    _check(load().bitnet_pack_ternary(_ptr(w), n, k, _ptr(packed), _ptr(flags), _stream(stream)),
           "bitnet_pack_ternary")


def quantize_pack_workspace_bytes() -> int:
    return int(load().bitnet_quantize_pack_workspace_bytes())


def quantize_pack(w, packed, scale, workspace, flags=None, stream=None) -> None:
    """w: fp32 [n,k] device tensor -> packed uint8 [n, 32*ceil(k/128)] and the
    absmean scale in the one-element fp32 device tensor ``scale``."""
    n, k = w.shape
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().bitnet_quantize_pack(_ptr(w), n, k, _ptr(packed), _ptr(scale), _ptr(workspace), ws_bytes,
                                       _ptr(flags), _stream(stream)), "bitnet_quantize_pack")


def unpack_ternary(packed, n, k, w, stream=None) -> None:
    _check(load().bitnet_unpack_ternary(_ptr(packed), n, k, _ptr(w), _stream(stream)),
           "bitnet_unpack_ternary")


def quant_act(x, xq, act_scale, flags=None, stream=None) -> None:
    m, k = x.shape
    _check(load().bitnet_quant_act(_ptr(x), m, k, _ptr(xq), _ptr(act_scale), _ptr(flags),
                                   _stream(stream)), "bitnet_quant_act")


def make_tw(packed, n: int, k: int, scale: float) -> TW:
    return TW(packed.data_ptr(), n, k, float(scale))


def make_epilogue(bias=None, gamma=None, residual=None, relu=False) -> Epilogue:
    """Epilogue descriptor from optional device tensors: bias [n], gamma [n],
    residual [m, n] (may be the output tensor itself)."""
    return Epilogue(_ptr(bias), _ptr(gamma), _ptr(residual), 1 if relu else 0, 0)


def linear(x, tw: TW, y, acc=None, workspace=None, flags=None, stream=None, epi: Epilogue | None = None) -> None:
    m = x.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if epi is None:
        _check(load().bitnet_linear(_ptr(x), m, C.byref(tw), _ptr(y), _ptr(acc), _ptr(workspace),
                                    ws_bytes, _ptr(flags), _stream(stream)), "bitnet_linear")
    else:
        _check(load().bitnet_linear_ex(_ptr(x), m, C.byref(tw), C.byref(epi), _ptr(y), _ptr(acc), _ptr(workspace),
                                       ws_bytes, _ptr(flags), _stream(stream)), "bitnet_linear_ex")


def i8_row_bytes(k: int) -> int:
    return int(load().bitnet_i8_row_bytes(k))


def linear_i8_workspace_bytes(m: int, k: int) -> int:
    return int(load().bitnet_linear_i8_workspace_bytes(m, k))


def make_i8w(w_rows, n: int, k: int, scale: float) -> I8W:
    """I8_S weight descriptor over a device int8 tensor [n, i8_row_bytes(k)]."""
    return I8W(w_rows.data_ptr(), n, k, float(scale))


def linear_i8(x, w8: I8W, y, workspace, acc=None, flags=None, stream=None, epi: Epilogue | None = None) -> None:
    """I8_S layer: int8 weights x per-token int8 activations (bitnet_linear_i8)."""
    m = x.shape[0]
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().bitnet_linear_i8(_ptr(x), m, C.byref(w8), None if epi is None else C.byref(epi), _ptr(y),
                                   _ptr(acc), _ptr(workspace), ws_bytes, _ptr(flags), _stream(stream)),
           "bitnet_linear_i8")


class I8GroupCall:
    """Marshalled arguments of one bitnet_linear_i8_grouped call (reusable);
    ``workspace_bytes`` is what the call needs."""

    def __init__(self, xs, w8s, ys, accs=None, epis=None):
        count = len(w8s)
        self.count = count
        self.m = xs[0].shape[0]
        self.x_arr = (C.c_void_p * count)(*[x.data_ptr() for x in xs])
        self.y_arr = (C.c_void_p * count)(*[y.data_ptr() for y in ys])
        self.w_arr = (I8W * count)(*w8s)
        self.acc_arr = None
        if accs is not None:
            self.acc_arr = (C.c_void_p * count)(*[(a.data_ptr() if a is not None else None) for a in accs])
        self.epi_arr = None if epis is None else (Epilogue * count)(*[e if e is not None else Epilogue()
                                                                      for e in epis])
        self.workspace_bytes = int(load().bitnet_linear_i8_grouped_workspace_bytes(self.x_arr, self.m, self.w_arr,
                                                                                   count))
        self._keep = (xs, ys, accs)

    def __call__(self, workspace, flags=None, stream=None) -> None:
        ws_bytes = workspace.numel() * workspace.element_size()
        _check(load().bitnet_linear_i8_grouped(self.x_arr, self.m, self.w_arr, self.epi_arr, self.count, self.y_arr,
                                               self.acc_arr, _ptr(workspace), ws_bytes, _ptr(flags),
                                               _stream(stream)), "bitnet_linear_i8_grouped")


def linear_q(xq, act_scale, tw: TW, y, acc=None, flags=None, stream=None, epi: Epilogue | None = None) -> None:
    m = xq.shape[0]
    if epi is None:
        _check(load().bitnet_linear_q(_ptr(xq), _ptr(act_scale), m, C.byref(tw), _ptr(y), _ptr(acc),
                                      _ptr(flags), _stream(stream)), "bitnet_linear_q")
    else:
        _check(load().bitnet_linear_q_ex(_ptr(xq), _ptr(act_scale), m, C.byref(tw), C.byref(epi), _ptr(y),
                                         _ptr(acc), _ptr(flags), _stream(stream)), "bitnet_linear_q_ex")


class GroupedCall:
    """Marshalled arguments of one bitnet_linear_q_grouped call (reusable)."""

    def __init__(self, xqs, scales, tws, ys, accs=None, epis=None):
        count = len(tws)
        self.count = count
        self.m = xqs[0].shape[0]
        self.xq_arr = (C.c_void_p * count)(*[x.data_ptr() for x in xqs])
        self.s_arr = (C.c_void_p * count)(*[s.data_ptr() for s in scales])
        self.y_arr = (C.c_void_p * count)(*[y.data_ptr() for y in ys])
        self.tw_arr = (TW * count)(*tws)
        self.acc_arr = None
        if accs is not None:
            self.acc_arr = (C.c_void_p * count)(*[(a.data_ptr() if a is not None else None) for a in accs])
        self.epi_arr = None if epis is None else (Epilogue * count)(*[e if e is not None else Epilogue()
                                                                      for e in epis])
        self._keep = (xqs, scales, ys, accs)

    def __call__(self, flags=None, stream=None) -> None:
        if self.epi_arr is None:
            _check(load().bitnet_linear_q_grouped(self.xq_arr, self.s_arr, self.m, self.tw_arr, self.count,
                                                  self.y_arr, self.acc_arr, _ptr(flags), _stream(stream)),
                   "bitnet_linear_q_grouped")
        else:
            _check(load().bitnet_linear_q_grouped_ex(self.xq_arr, self.s_arr, self.m, self.tw_arr, self.epi_arr,
                                                     self.count, self.y_arr, self.acc_arr, _ptr(flags),
                                                     _stream(stream)), "bitnet_linear_q_grouped_ex")


def linear_q_grouped(xqs, scales, tws, ys, accs=None, flags=None, stream=None, epis=None) -> None:
    GroupedCall(xqs, scales, tws, ys, accs, epis)(flags=flags, stream=stream)


class StackCall:
    """Marshalled arguments of one bitnet_linear_stack call, built once and
    reusable (the pointer arrays are kept alive by this object)."""

    def __init__(self, xs, tws, ys, accs=None, epis=None):
        count = len(tws)
        self.count = count
        self.m = xs[0].shape[0]
        self.x_arr = (C.c_void_p * count)(*[x.data_ptr() for x in xs])
        self.y_arr = (C.c_void_p * count)(*[y.data_ptr() for y in ys])
        self.tw_arr = (TW * count)(*tws)
        self.acc_arr = None
        if accs is not None:
            self.acc_arr = (C.c_void_p * count)(*[(a.data_ptr() if a is not None else None) for a in accs])
        self.epi_arr = None if epis is None else (Epilogue * count)(*[e if e is not None else Epilogue()
                                                                      for e in epis])
        self._keep = (xs, ys, accs)

    def __call__(self, flags=None, stream=None) -> None:
        if self.epi_arr is None:
            _check(load().bitnet_linear_stack(self.x_arr, self.m, self.tw_arr, self.count, self.y_arr,
                                              self.acc_arr, _ptr(flags), _stream(stream)),
                   "bitnet_linear_stack")
        else:
            _check(load().bitnet_linear_stack_ex(self.x_arr, self.m, self.tw_arr, self.epi_arr, self.count,
                                                 self.y_arr, self.acc_arr, _ptr(flags), _stream(stream)),
                   "bitnet_linear_stack_ex")


def linear_stack(xs, tws, ys, accs=None, flags=None, stream=None, epis=None) -> None:
    StackCall(xs, tws, ys, accs, epis)(flags=flags, stream=stream)


def linear_stack_noalloc(xs, tws, ys, accs=None, flags=None, stream=None) -> None:
    """bitnet_linear_stack_noalloc: the stack call that allocates no device
    memory (tensor maps in the library's fixed device array)."""
    c = StackCall(xs, tws, ys, accs)
    _check(load().bitnet_linear_stack_noalloc(c.x_arr, c.m, c.tw_arr, c.count, c.y_arr, c.acc_arr,
                                              _ptr(flags), _stream(stream)), "bitnet_linear_stack_noalloc")
