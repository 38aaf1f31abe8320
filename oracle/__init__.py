"""CPU oracle for the I2_S ternary linear layer -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps the plain C oracle
(``bitnet_oracle.c``; readings R1-R4 are stated in ``bitnet_oracle.h``) with
numpy-friendly functions.  It shares no code with the CUDA library.
"""
import ctypes as _C

import numpy as _np

from .build import build as _build

OK, NONFINITE, NOT_TERNARY, OVERFLOW = 0, 1, 2, 4

_lib = _C.CDLL(_build())
_i64, _f32 = _C.c_int64, _C.c_float
_P = _C.c_void_p
for _name, _args, _ret in [
    ("oracle_blocks", [_i64], _i64),
    ("oracle_kpad", [_i64], _i64),
    ("oracle_quant_act", [_P, _i64, _i64, _P, _P], _C.c_int),
    ("oracle_pack", [_P, _i64, _i64, _P], _C.c_int),
    ("oracle_absmean_ternary", [_P, _i64, _i64, _P, _P], _C.c_int),
    ("oracle_ternary_round", [_P, _i64, _f32, _P], None),
    ("oracle_epilogue", [_P, _P, _P, _C.c_int, _i64, _i64, _P, _P], None),
    ("oracle_i8_row_bytes", [_i64], _i64),
    ("oracle_i8_matmul", [_P, _i64, _P, _i64, _i64, _P], _C.c_int),
    ("oracle_linear_i8", [_P, _i64, _i64, _P, _i64, _f32, _P, _P, _P], _C.c_int),
    ("oracle_unpack", [_P, _i64, _i64, _P], None),
    ("oracle_unpack_misread64", [_P, _i64, _i64, _P], None),
    ("oracle_ternary_matmul", [_P, _i64, _P, _i64, _i64, _P], _C.c_int),
    ("oracle_dequant", [_P, _P, _f32, _i64, _i64, _P, _P], None),
    ("oracle_linear", [_P, _i64, _i64, _P, _i64, _f32, _P, _P, _P], _C.c_int),
    ("oracle_linear_rows", [_P, _i64, _i64, _P, _i64, _f32, _P, _i64, _P, _P], _C.c_int),
]:
    _fn = getattr(_lib, _name)
    _fn.argtypes, _fn.restype = _args, _ret


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_P)


def _c(a, dtype):
    return _np.ascontiguousarray(a, dtype=dtype)


def blocks(k: int) -> int:
    return int(_lib.oracle_blocks(k))


def kpad(k: int) -> int:
    return int(_lib.oracle_kpad(k))


def packed_row_bytes(k: int) -> int:
    return 32 * blocks(k)


def quant_act(x):
    """x fp32 [m,k] -> (q int8 [m,kpad], s_act fp32 [m], status)."""
    x = _c(x, _np.float32)
    m, k = x.shape
    q = _np.empty((m, kpad(k)), _np.int8)
    s = _np.empty((m,), _np.float32)
    st = _lib.oracle_quant_act(_ptr(x), m, k, _ptr(q), _ptr(s))
    return q, s, st


def absmean_ternary(W):
    """W fp32 [n,k] -> (w int8 [n,k] in {-1,0,1}, scale fp32, status) (reading R5)."""
    W = _c(W, _np.float32)
    n, k = W.shape
    w = _np.empty((n, k), _np.int8)
    sc = _np.zeros((1,), _np.float32)
    st = _lib.oracle_absmean_ternary(_ptr(W), n, k, _ptr(w), _ptr(sc))
    return w, _np.float32(sc[0]), st


def ternary_round(W, scale):
    """Codes of W fp32 [n,k] at a given fp32 scale (second pass of reading R5)."""
    W = _c(W, _np.float32)
    w = _np.empty(W.shape, _np.int8)
    _lib.oracle_ternary_round(_ptr(W), W.size, _np.float32(scale), _ptr(w))
    return w


def pack(w):
    """w int8 [n,k] in {-1,0,1} -> (packed uint8 [n, 32*blocks], status)."""
    w = _c(w, _np.int8)
    n, k = w.shape
    p = _np.empty((n, packed_row_bytes(k)), _np.uint8)
    st = _lib.oracle_pack(_ptr(w), n, k, _ptr(p))
    return p, st


def unpack(packed, k):
    packed = _c(packed, _np.uint8)
    n = packed.shape[0]
    w = _np.empty((n, k), _np.int8)
    _lib.oracle_unpack(_ptr(packed), n, k, _ptr(w))
    return w


def unpack_misread64(packed, k):
    """The planted 64-element misreading (mutation test only)."""
    packed = _c(packed, _np.uint8)
    n = packed.shape[0]
    w = _np.empty((n, k), _np.int8)
    _lib.oracle_unpack_misread64(_ptr(packed), n, k, _ptr(w))
    return w


def ternary_matmul(q, packed, k):
    """q int8 [m,kpad] x packed [n,...] -> (acc int32 [m,n], status)."""
    q = _c(q, _np.int8)
    packed = _c(packed, _np.uint8)
    m, n = q.shape[0], packed.shape[0]
    acc = _np.empty((m, n), _np.int32)
    st = _lib.oracle_ternary_matmul(_ptr(q), m, _ptr(packed), n, k, _ptr(acc))
    return acc, st


def dequant(acc, s_act, s_w):
    """-> (y64 fp64 [m,n], y32 fp32 [m,n])."""
    acc = _c(acc, _np.int32)
    s_act = _c(s_act, _np.float32)
    m, n = acc.shape
    y64 = _np.empty((m, n), _np.float64)
    y32 = _np.empty((m, n), _np.float32)
    _lib.oracle_dequant(_ptr(acc), _ptr(s_act), float(s_w), m, n, _ptr(y64), _ptr(y32))
    return y64, y32


def linear(x, packed, n, k, s_w):
    """Whole layer -> (acc int32, y64 fp64, y32 fp32, status)."""
    x = _c(x, _np.float32)
    packed = _c(packed, _np.uint8)
    m = x.shape[0]
    acc = _np.empty((m, n), _np.int32)
    y64 = _np.empty((m, n), _np.float64)
    y32 = _np.empty((m, n), _np.float32)
    st = _lib.oracle_linear(_ptr(x), m, k, _ptr(packed), n, float(s_w),
                            _ptr(acc), _ptr(y64), _ptr(y32))
    return acc, y64, y32, st


def epilogue(y32=None, y64=None, bias=None, gamma=None, residual=None, relu=False):
    """Fused epilogue (reading R6) on copies of y32 fp32 [m,n] and/or y64 fp64
    [m,n]: h = relu(y + bias); out = residual + gamma * h.  Returns (y32, y64)."""
    ref = y32 if y32 is not None else y64
    m, n = ref.shape
    y32 = None if y32 is None else _np.array(y32, _np.float32, copy=True, order="C")
    y64 = None if y64 is None else _np.array(y64, _np.float64, copy=True, order="C")
    b = None if bias is None else _c(bias, _np.float32)
    g = None if gamma is None else _c(gamma, _np.float32)
    r = None if residual is None else _c(residual, _np.float32)
    assert b is None or b.shape == (n,)
    assert g is None or g.shape == (n,)
    assert r is None or r.shape == (m, n)
    _lib.oracle_epilogue(_ptr(b), _ptr(g), _ptr(r), 1 if relu else 0, m, n, _ptr(y32), _ptr(y64))
    return y32, y64


def i8_row_bytes(k: int) -> int:
    return int(_lib.oracle_i8_row_bytes(k))


def i8_layout(w):
    """int8 weights [n,k] -> the I8_S row layout [n, 32*ceil(k/32)], pads 0
    (reading R7)."""
    w = _c(w, _np.int8)
    n, k = w.shape
    out = _np.zeros((n, i8_row_bytes(k)), _np.int8)
    out[:, :k] = w
    return out


def i8_matmul(q, w_rows, k):
    """q int8 [m, kpad] x I8_S rows [n, 32*ceil(k/32)] -> (acc int32 [m,n], status)."""
    q = _c(q, _np.int8)
    w_rows = _c(w_rows, _np.int8)
    m, n = q.shape[0], w_rows.shape[0]
    acc = _np.empty((m, n), _np.int32)
    st = _lib.oracle_i8_matmul(_ptr(q), m, _ptr(w_rows), n, k, _ptr(acc))
    return acc, st


def linear_i8(x, w_rows, k, s_w):
    """I8_S layer (reading R7) -> (acc int32, y64 fp64, y32 fp32, status)."""
    x = _c(x, _np.float32)
    w_rows = _c(w_rows, _np.int8)
    m, n = x.shape[0], w_rows.shape[0]
    acc = _np.empty((m, n), _np.int32)
    y64 = _np.empty((m, n), _np.float64)
    y32 = _np.empty((m, n), _np.float32)
    st = _lib.oracle_linear_i8(_ptr(x), m, k, _ptr(w_rows), n, float(s_w), _ptr(acc), _ptr(y64), _ptr(y32))
    return acc, y64, y32, st


# Reading R8: the decoder layer's linears as a dependence chain.  The path
# holds no attention, normalisation or activation op, so each is replaced by
# the plainest stand-in of matching width: the attention output by q's
# output, the gated activation by up's output.  Input of each linear, by
# position in (q, k, v, o, gate, up, down): the layer input for q, k, v; q's
# output for o; o's output for gate and up; up's output for down.  down's
# output is the next layer's input.
CHAIN_INPUT_OF = (-1, -1, -1, 0, 3, 3, 5)   # -1: the layer input


def linear_chain(x0, layers):
    """Decode chain (reading R8): ``layers`` is a list of decoder layers, each
    a list of seven (packed, n, k, s_w) in (q, k, v, o, gate, up, down) order.
    Every linear quantises its fp32 input (R1) and feeds its fp32 output (the
    R4 fp32 form) forward.  Returns (outputs per layer as lists of y32 [m, n],
    status)."""
    x = _np.ascontiguousarray(x0, _np.float32)
    outs, st = [], 0
    for layer in layers:
        ys = []
        for i, (packed, n, k, s_w) in enumerate(layer):
            src = x if CHAIN_INPUT_OF[i] < 0 else ys[CHAIN_INPUT_OF[i]]
            assert src.shape[1] == k, "chain width mismatch"
            _, _, y32, s1 = linear(src, packed, n, k, s_w)
            ys.append(y32)
            st |= s1
        outs.append(ys)
        x = ys[6]
    return outs, st


def linear_rows(x, packed, n, k, s_w, rows):
    """Only the output columns ``rows`` -> (acc int32 [m,cnt], y64 [m,cnt], status)."""
    x = _c(x, _np.float32)
    packed = _c(packed, _np.uint8)
    idx = _c(rows, _np.int64)
    m, cnt = x.shape[0], idx.shape[0]
    acc = _np.empty((m, cnt), _np.int32)
    y64 = _np.empty((m, cnt), _np.float64)
    st = _lib.oracle_linear_rows(_ptr(x), m, k, _ptr(packed), n, float(s_w),
                                 _ptr(idx), cnt, _ptr(acc), _ptr(y64))
    return acc, y64, st


def linear_stack(xs, packed_list, shapes, scales):
    """Loops the layers in order: xs[i] is the fp32 input of layer i (aliasing
    allowed), shapes[i] = (n, k).  Returns lists (acc, y64, status)."""
    accs, ys, st = [], [], 0
    for x, p, (n, k), s in zip(xs, packed_list, shapes, scales):
        a, y64, _, s1 = linear(x, p, n, k, s)
        accs.append(a)
        ys.append(y64)
        st |= s1
    return accs, ys, st
