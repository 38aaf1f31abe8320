"""Parity of the fused absmean quantiser + pack (through the C ABI) with the
CPU oracle's absmean quantiser followed by its pack.

Both sides sum |W| in fp64 and round the mean once to fp32, but in different
orders (the oracle row-major, the kernel over a fixed grid of partial sums).
Two fp64 sums of the same n*k fp32 terms differ by far less than half an fp32
ulp, so the scales are expected to be equal, and they are checked to within
one ulp.  The codes are an integer decision taken in fp32 on both sides: they
must equal the oracle's codes at the kernel's own scale bit for bit, and the
oracle's absmean codes whenever the scales are equal.
"""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_i2_b200 as tw2
from ternary_weight_i2_b200 import synth

from gpu_helpers import DEV, Guarded, flags_tensor, upload

pytestmark = pytest.mark.gpu


def _run(W, ws_bytes=None):
    n, k = W.shape
    pk = Guarded((n, 32 * oracle.blocks(k)), torch.uint8)
    sc = Guarded((1,), torch.float32)
    ws = torch.empty(ws_bytes if ws_bytes is not None else tw2.quantize_pack_workspace_bytes(),
                     dtype=torch.uint8, device=DEV)
    fl = flags_tensor()
    tw2.quantize_pack(upload(W), pk.t, sc.t, ws, flags=fl)
    torch.cuda.synchronize()
    assert pk.guard_intact() and sc.guard_intact()
    return pk.t.cpu().numpy(), np.float32(sc.t.item()), int(fl.item())


def _ulps(a, b):
    ia = np.array([a], np.float32).view(np.int32)[0]
    ib = np.array([b], np.float32).view(np.int32)[0]
    return abs(int(ia) - int(ib))


def _check_against_oracle(W):
    packed, s, flags = _run(W)
    w_or, s_or, st = oracle.absmean_ternary(W)
    assert st == oracle.OK and flags == 0
    assert _ulps(s, s_or) <= 1, (s, s_or)
    at_own_scale, _ = oracle.pack(oracle.ternary_round(W, s))
    np.testing.assert_array_equal(packed, at_own_scale)
    if s == s_or:
        want, _ = oracle.pack(w_or)
        np.testing.assert_array_equal(packed, want)
    return s == s_or


@pytest.mark.parametrize("n,k", [(1, 1), (3, 5), (2, 31), (33, 127), (7, 128), (256, 129), (5, 300),
                                 (1536, 1536), (8960, 1536), (1536, 8960)])
def test_quantize_pack_matches_oracle(n, k):
    rng = np.random.default_rng(31 * n + k)
    W = (synth.normal(rng, n, k) * np.float32(0.02)).astype(np.float32)
    assert _check_against_oracle(W)


def test_quantize_pack_exact_halves_round_to_even():
    """A tensor whose scale is exactly 1 and whose entries sit at +-1/2 and
    +-3/2: every quotient is an exact half."""
    rng = np.random.default_rng(5)
    n, k = 64, 520
    sign = rng.choice(np.array([1.0, -1.0], np.float32), size=(n, k))
    # magnitudes alternate 0.5, 1.5: the mean is exactly 1
    mag = np.where(np.arange(n * k).reshape(n, k) % 2 == 0, np.float32(0.5), np.float32(1.5))
    W = (sign * mag).astype(np.float32)
    packed, s, flags = _run(W)
    assert s == np.float32(1.0) and flags == 0
    w_or, s_or, _ = oracle.absmean_ternary(W)
    assert s_or == s
    want, _ = oracle.pack(w_or)
    np.testing.assert_array_equal(packed, want)
    # 0.5 -> 0 and 1.5 -> 2 -> clamp 1: every even position is weight 0
    back = oracle.unpack(packed, k)
    assert not back[:, 0::2].any() and (np.abs(back[:, 1::2]) == 1).all()


def test_quantize_pack_decisions_next_to_one_half():
    """Scale exactly 1 (a bulk of +-1/2 and +-3/2 entries; a handful of probes
    moves the fp64 mean by far less than half an ulp of 1), probes at 1/2 and
    its neighbouring floats: 1/2 and below give 0, the next float above gives
    +-1."""
    n, k = 64, 520
    mag = np.where(np.arange(n * k).reshape(n, k) % 2 == 0, np.float32(0.5), np.float32(1.5))
    W = mag.copy()
    up = np.nextafter(np.float32(0.5), np.float32(1))
    down = np.nextafter(np.float32(0.5), np.float32(0))
    probes = [up, -up, down, -down, np.float32(0.5), np.float32(-0.5), np.nextafter(up, np.float32(1))]
    for i, v in enumerate(probes):
        W[3, 2 * i] = v
    packed, s, flags = _run(W)
    w_or, s_or, _ = oracle.absmean_ternary(W)
    assert s == np.float32(1.0) == s_or and flags == 0
    want, _ = oracle.pack(w_or)
    np.testing.assert_array_equal(packed, want)
    back = oracle.unpack(packed, k)
    assert list(back[3, 0:14:2]) == [1, -1, 0, 0, 0, 0, 1]


@pytest.mark.parametrize("magnitude", [1e-40, 1e-30, 1e30, 3e37])
def test_quantize_pack_extreme_magnitudes(magnitude):
    """Subnormal and very large weights: the scale and every code still match
    the oracle's fp32 divide (denormals are not flushed on either side)."""
    rng = np.random.default_rng(int(np.log10(magnitude)) + 100)
    W = (synth.normal(rng, 37, 333).astype(np.float64) * magnitude).astype(np.float32)
    assert np.isfinite(W).all()
    assert _check_against_oracle(W)


def test_quantize_pack_all_zero_tensor():
    W = np.zeros((17, 333), np.float32)
    packed, s, flags = _run(W)
    assert s == 0.0 and flags == 0
    want, _ = oracle.pack(np.zeros((17, 333), np.int8))
    np.testing.assert_array_equal(packed, want)


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf])
def test_quantize_pack_nonfinite_tensor(bad):
    rng = np.random.default_rng(9)
    W = synth.normal(rng, 40, 700).astype(np.float32)
    W[37, 611] = bad
    packed, s, flags = _run(W)
    assert s == 0.0 and flags & tw2.FLAG_NONFINITE
    w_or, s_or, st = oracle.absmean_ternary(W)
    assert st == oracle.NONFINITE and s_or == 0.0
    want, _ = oracle.pack(w_or)
    np.testing.assert_array_equal(packed, want)


def test_quantize_pack_is_deterministic_and_unaligned_input_ok():
    rng = np.random.default_rng(12)
    W = (synth.normal(rng, 300, 1000) * np.float32(0.05)).astype(np.float32)
    a = _run(W)
    b = _run(W)
    np.testing.assert_array_equal(a[0], b[0])
    assert a[1] == b[1]
    # a 4-byte-aligned (not 16) input pointer
    big = torch.zeros(W.size + 1, dtype=torch.float32, device=DEV)
    big[1:] = upload(W.ravel())
    pk = torch.empty((300, 32 * oracle.blocks(1000)), dtype=torch.uint8, device=DEV)
    sc = torch.empty(1, dtype=torch.float32, device=DEV)
    ws = torch.empty(tw2.quantize_pack_workspace_bytes(), dtype=torch.uint8, device=DEV)
    tw2.quantize_pack(big[1:].view(300, 1000), pk, sc, ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(pk.cpu().numpy(), a[0])
    assert np.float32(sc.item()) == a[1]


def test_quantize_pack_rejects_small_workspace():
    W = torch.ones((4, 64), dtype=torch.float32, device=DEV)
    pk = torch.empty((4, 32), dtype=torch.uint8, device=DEV)
    sc = torch.empty(1, dtype=torch.float32, device=DEV)
    ws = torch.empty(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(tw2.BitnetError) as e:
        tw2.quantize_pack(W, pk, sc, ws)
    assert e.value.status == 7   # BITNET_ERR_WORKSPACE


def test_quantize_pack_feeds_the_linear_layer():
    """Weights quantised and packed on the device drive the GEMV to the
    oracle's result on the oracle's codes and scale."""
    rng = np.random.default_rng(21)
    n, k, m = 256, 1536, 1
    W = (synth.normal(rng, n, k) * np.float32(0.02)).astype(np.float32)
    x = synth.normal(rng, m, k)
    packed, s, _ = _run(W)
    w_or, s_or, _ = oracle.absmean_ternary(W)
    assert s == s_or
    pk = upload(packed)
    y = torch.empty((m, n), dtype=torch.float32, device=DEV)
    acc = torch.empty((m, n), dtype=torch.int32, device=DEV)
    tw2.linear(upload(x), tw2.make_tw(pk, n, k, float(s)), y, acc=acc)
    torch.cuda.synchronize()
    q, xs, _ = oracle.quant_act(x)
    want_pk, _ = oracle.pack(w_or)
    want_acc, _ = oracle.ternary_matmul(q, want_pk, k)
    np.testing.assert_array_equal(acc.cpu().numpy(), want_acc)
