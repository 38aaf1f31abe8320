"""Parity of the I8_S layer (int8 weights x per-token int8 activations, the
technical report's §2.2.1 and §2.4.2) with the oracle, through the C ABI.

int32 sums must match bit for bit; the fp32 outputs must equal the oracle's
fp32 form bit for bit (the int-to-float conversion of sums above 2^24
rounds to nearest even on both sides) and lie within 1e-5 relative of its
fp64 form.  Weight-row pads are filled with garbage: they meet zero
activation pads and must not change any result."""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_i2_b200 as tw2
from ternary_weight_i2_b200 import synth

from gpu_helpers import DEV, Guarded, flags_tensor, rel_err, upload

pytestmark = pytest.mark.gpu
RTOL = 1e-5


def _weights(rng, n, k):
    w = rng.integers(-127, 128, size=(n, k), dtype=np.int64).astype(np.int8)
    rows = oracle.i8_layout(w)
    rows[:, k:] = rng.integers(-128, 128, size=(n, rows.shape[1] - k), dtype=np.int64).astype(np.int8)
    return rows


def _run(x, rows, k, s_w, epi=None):
    m = x.shape[0]
    n = rows.shape[0]
    assert rows.shape[1] == tw2.i8_row_bytes(k)
    wd = upload(rows)
    y = Guarded((m, n), torch.float32)
    acc = Guarded((m, n), torch.int32)
    ws = torch.empty(tw2.linear_i8_workspace_bytes(m, k), dtype=torch.uint8, device=DEV)
    fl = flags_tensor()
    tw2.linear_i8(upload(x), tw2.make_i8w(wd, n, k, s_w), y.t, ws, acc=acc.t, flags=fl, epi=epi)
    torch.cuda.synchronize()
    assert y.guard_intact() and acc.guard_intact()
    return y.t.cpu().numpy(), acc.t.cpu().numpy(), int(fl.item())


@pytest.mark.parametrize("m,n,k", [(1, 256, 1536), (1, 300, 33), (2, 1536, 1536), (3, 257, 9024), (5, 64, 32),
                                   (8, 100, 1000), (13, 100, 1000), (1, 8960, 1536), (1, 1536, 8960)])
def test_linear_i8_matches_oracle(m, n, k):
    rng = np.random.default_rng(1000 * m + n + k)
    rows = _weights(rng, n, k)
    x = synth.normal_outliers(rng, m, k)
    s_w = synth.weight_scale(rng)
    yg, ag, fl = _run(x, rows, k, s_w)
    assert fl == 0
    acc, y64, y32, st = oracle.linear_i8(x, rows, k, s_w)
    assert st == oracle.OK
    np.testing.assert_array_equal(ag, acc)
    np.testing.assert_array_equal(yg.view(np.uint32), y32.view(np.uint32))
    assert rel_err(yg, y64) <= RTOL


def test_linear_i8_saturated_sums_round_like_the_oracle():
    """w = +-127, x constant: |acc| = 127^2 K = 145,560,576 at K = 9024, far
    above 2^24, so the fp32 form depends on the conversion's rounding."""
    m, n, k = 3, 64, 9024
    rows = oracle.i8_layout(np.where(np.arange(n)[:, None] % 2 == 0, 127, -127).astype(np.int8) *
                            np.ones((1, k), np.int8))
    x = np.full((m, k), 0.5, np.float32)
    x[1] = -3.0
    x[2, ::2] = -1.0
    yg, ag, fl = _run(x, rows, k, 0.03125)
    acc, y64, y32, _ = oracle.linear_i8(x, rows, k, 0.03125)
    assert abs(int(acc[0, 0])) == 127 * 127 * k
    np.testing.assert_array_equal(ag, acc)
    np.testing.assert_array_equal(yg.view(np.uint32), y32.view(np.uint32))


def test_linear_i8_special_rows():
    """A non-finite row raises the flag and gives 0; a zero row gives 0."""
    m, n, k = 4, 96, 520
    rng = np.random.default_rng(4)
    rows = _weights(rng, n, k)
    x = synth.normal(rng, m, k)
    x[1, 17] = np.nan
    x[2] = 0.0
    yg, ag, fl = _run(x, rows, k, 0.05)
    assert fl & tw2.FLAG_NONFINITE
    acc, _, y32, st = oracle.linear_i8(x, rows, k, 0.05)
    assert st & oracle.NONFINITE
    np.testing.assert_array_equal(ag, acc)
    np.testing.assert_array_equal(yg.view(np.uint32), y32.view(np.uint32))
    assert not yg[1].any() and not yg[2].any()


@pytest.mark.parametrize("m", [1, 13])
def test_linear_i8_fused_epilogue(m):
    n, k = 300, 1536
    rng = np.random.default_rng(90 + m)
    rows = _weights(rng, n, k)
    x = synth.normal_outliers(rng, m, k)
    s_w = synth.weight_scale(rng)
    b = rng.standard_normal(n).astype(np.float32)
    g = rng.uniform(0.25, 2.0, n).astype(np.float32)
    r = rng.standard_normal((m, n)).astype(np.float32)
    bd, gd, rd = upload(b), upload(g), upload(r)
    epi = tw2.make_epilogue(bias=bd, gamma=gd, residual=rd, relu=True)
    yg, ag, _ = _run(x, rows, k, s_w, epi=epi)
    acc, y64, y32, _ = oracle.linear_i8(x, rows, k, s_w)
    o32, _ = oracle.epilogue(y32, bias=b, gamma=g, residual=r, relu=True)
    np.testing.assert_array_equal(ag, acc)
    np.testing.assert_array_equal(yg.view(np.uint32), o32.view(np.uint32))


@pytest.mark.parametrize("m", [1, 13])
def test_linear_i8_grouped_decoder_layer(m):
    """One decoder layer's seven linears in one grouped call (the four
    distinct inputs quantised once each, one GEMV launch per 8-token slice),
    epilogues on some layers: every layer against the oracle."""
    rng = np.random.default_rng(500 + m)
    xs_host = synth.layer_inputs(0, m, 2)
    xdev = [upload(a) for a in xs_host]
    w8s, keep, ys, accs, epis, ref = [], [], [], [], [], []
    for i, ((name, n, k), j) in enumerate(zip(synth.LAYER_SHAPES, synth.LAYER_INPUT_OF)):
        rows = _weights(rng, n, k)
        s_w = synth.weight_scale(rng)
        wd = upload(rows)
        keep.append(wd)
        w8s.append(tw2.make_i8w(wd, n, k, s_w))
        ys.append(Guarded((m, n), torch.float32))
        accs.append(Guarded((m, n), torch.int32))
        if i % 2 == 0:
            b = rng.standard_normal(n).astype(np.float32)
            r = rng.standard_normal((m, n)).astype(np.float32)
            bd, rd = upload(b), upload(r)
            keep.append((bd, rd))
            epis.append(tw2.make_epilogue(bias=bd, residual=rd, relu=(i == 4)))
            ref.append((xs_host[j], rows, k, s_w, b, r, i == 4))
        else:
            epis.append(None)
            ref.append((xs_host[j], rows, k, s_w, None, None, False))
    call = tw2.I8GroupCall([xdev[j] for j in synth.LAYER_INPUT_OF], w8s, [y.t for y in ys], [a.t for a in accs],
                           epis=epis)
    ws = torch.empty(call.workspace_bytes, dtype=torch.uint8, device=DEV)
    fl = flags_tensor()
    call(ws, flags=fl)
    torch.cuda.synchronize()
    assert int(fl.item()) == 0
    for y, a, (x, rows, k, s_w, b, r, relu) in zip(ys, accs, ref):
        assert y.guard_intact() and a.guard_intact()
        acc, y64, y32, _ = oracle.linear_i8(x, rows, k, s_w)
        o32, _ = oracle.epilogue(y32, bias=b, residual=r, relu=relu)
        np.testing.assert_array_equal(a.t.cpu().numpy(), acc)
        np.testing.assert_array_equal(y.t.cpu().numpy().view(np.uint32), o32.view(np.uint32))
