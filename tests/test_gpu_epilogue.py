"""Parity of the fused epilogue (bias, ReLU, layer-scaled residual add: the
operator fusion of the technical report's §2.4.1) with the oracle, through
the C ABI, on the decode GEMV (m <= 8), the stack, and the tensor-core GEMM.

Every epilogue step is one rounded fp32 operation on both sides, so outputs
must equal the oracle's fp32 form bit for bit.  Against the fp64 form the
residual add can cancel, so the tolerance is 1e-5 of the operands'
magnitude |r| + |gamma| (|y| + |b|) rather than of the output."""
import itertools

import numpy as np
import pytest
import torch

import oracle
import ternary_weight_i2_b200 as tw2
from ternary_weight_i2_b200 import synth

from gpu_helpers import DEV, Guarded, flags_tensor, pack_on_gpu, upload

pytestmark = pytest.mark.gpu
TOL = 1e-5

COMBOS = [dict(bias=True), dict(relu=True), dict(bias=True, relu=True), dict(gamma=True, res=True),
          dict(bias=True, relu=True, gamma=True, res=True), dict(res=True)]


def _operands(rng, m, n, combo):
    b = rng.standard_normal(n).astype(np.float32) if combo.get("bias") else None
    g = rng.uniform(0.25, 2.0, n).astype(np.float32) if combo.get("gamma") else None
    r = (rng.standard_normal((m, n)) * 2).astype(np.float32) if combo.get("res") else None
    return b, g, r, bool(combo.get("relu"))


def _expected(x, w, s_w, b, g, r, relu, cols=None):
    """Oracle: acc, the epilogue's fp32 form and fp64 form (optionally only
    the output columns ``cols``)."""
    n, k = w.shape
    if cols is not None:
        w = w[cols]
        b = None if b is None else b[cols]
        g = None if g is None else g[cols]
        r = None if r is None else r[:, cols]
    pk_np, _ = oracle.pack(w)
    acc, y64, y32, st = oracle.linear(x, pk_np, w.shape[0], k, s_w)
    o32, o64 = oracle.epilogue(y32, y64, bias=b, gamma=g, residual=r, relu=relu)
    scale = np.abs(y64) + (0 if b is None else np.abs(b.astype(np.float64)))
    scale = scale * (1 if g is None else np.abs(g.astype(np.float64)))
    scale = scale + (0 if r is None else np.abs(r.astype(np.float64)))
    return acc, o32, o64, scale


def _check(yg, ag, acc, o32, o64, scale):
    np.testing.assert_array_equal(ag, acc)
    np.testing.assert_array_equal(yg.view(np.uint32), o32.view(np.uint32))
    assert (np.abs(yg.astype(np.float64) - o64) <= TOL * scale + 1e-30).all()


def _epi_dev(b, g, r, relu, y_dev=None):
    """Device operands and the descriptor; with y_dev the residual is written
    into the output buffer first (in-place residual add)."""
    bd = None if b is None else upload(b)
    gd = None if g is None else upload(g)
    rd = None
    if r is not None:
        if y_dev is not None:
            y_dev.copy_(upload(r))
            rd = y_dev
        else:
            rd = upload(r)
    return tw2.make_epilogue(bias=bd, gamma=gd, residual=rd, relu=relu), (bd, gd, rd)


@pytest.mark.parametrize("m", [1, 5, 8, 130, 300])
@pytest.mark.parametrize("ci", range(len(COMBOS)))
def test_linear_epilogue_parity(m, ci):
    """bitnet_linear_ex: GEMV for m <= 8, per-token quantiser + tcgen05 GEMM
    above; n = 300 leaves ragged 32-row and 128-feature tiles."""
    n, k = 300, 1536
    rng = np.random.default_rng(100 * m + ci)
    w = synth.ternary(rng, n, k)
    x = synth.normal_row_spread(rng, m, k) if m > 8 else synth.normal_outliers(rng, m, k)
    s_w = synth.weight_scale(rng)
    b, g, r, relu = _operands(rng, m, n, COMBOS[ci])
    pk = pack_on_gpu(w)
    tw = tw2.make_tw(pk, n, k, s_w)
    y = Guarded((m, n), torch.float32)
    acc = Guarded((m, n), torch.int32)
    epi, keep = _epi_dev(b, g, r, relu)
    ws = torch.empty(max(tw2.linear_workspace_bytes(m, k), 1), dtype=torch.uint8, device=DEV)
    fl = flags_tensor()
    tw2.linear(upload(x), tw, y.t, acc=acc.t, workspace=ws, flags=fl, epi=epi)
    torch.cuda.synchronize()
    assert int(fl.item()) == 0 and y.guard_intact() and acc.guard_intact()
    _check(y.t.cpu().numpy(), acc.t.cpu().numpy(), *_expected(x, w, s_w, b, g, r, relu))


@pytest.mark.parametrize("m", [1, 7, 200])
def test_linear_epilogue_in_place_residual(m):
    """residual == y: each element is read before it is overwritten."""
    n, k = 264, 9024
    rng = np.random.default_rng(7 + m)
    w = synth.ternary(rng, n, k)
    x = synth.normal_row_spread(rng, m, k)
    s_w = synth.weight_scale(rng)
    b, g, r, relu = _operands(rng, m, n, dict(bias=True, relu=True, gamma=True, res=True))
    pk = pack_on_gpu(w)
    tw = tw2.make_tw(pk, n, k, s_w)
    y = Guarded((m, n), torch.float32)
    epi, keep = _epi_dev(b, g, r, relu, y_dev=y.t)
    ws = torch.empty(max(tw2.linear_workspace_bytes(m, k), 1), dtype=torch.uint8, device=DEV)
    acc = Guarded((m, n), torch.int32)
    tw2.linear(upload(x), tw, y.t, acc=acc.t, workspace=ws, epi=epi)
    torch.cuda.synchronize()
    assert y.guard_intact()
    _check(y.t.cpu().numpy(), acc.t.cpu().numpy(), *_expected(x, w, s_w, b, g, r, relu))


def test_linear_q_epilogue_prequantised():
    m, n, k = 130, 520, 1536
    rng = np.random.default_rng(77)
    w = synth.ternary(rng, n, k)
    x = synth.normal_row_spread(rng, m, k)
    s_w = synth.weight_scale(rng)
    b, g, r, relu = _operands(rng, m, n, dict(bias=True, gamma=True, res=True))
    q, s_act, _ = oracle.quant_act(x)
    pk = pack_on_gpu(w)
    y = Guarded((m, n), torch.float32)
    acc = Guarded((m, n), torch.int32)
    epi, keep = _epi_dev(b, g, r, relu)
    tw2.linear_q(upload(q), upload(s_act), tw2.make_tw(pk, n, k, s_w), y.t, acc=acc.t, epi=epi)
    torch.cuda.synchronize()
    _check(y.t.cpu().numpy(), acc.t.cpu().numpy(), *_expected(x, w, s_w, b, g, r, relu))


@pytest.mark.parametrize("m", [1, 13])
def test_stack_epilogue_per_layer(m):
    """One decoder layer's seven linears in one stack call, each with its own
    epilogue (one without); m = 13 runs in slices of 8 and 5 tokens, the
    residual sliced like the outputs."""
    rng = np.random.default_rng(300 + m)
    xs_host = synth.layer_inputs(0, m, 2)
    combos = [COMBOS[i % len(COMBOS)] for i in range(6)] + [None]
    tws, xd, ys, accs, epis, keep, ref = [], [], [], [], [], [], []
    xdev = [upload(a) for a in xs_host]
    for (name, n, k), j, combo in zip(synth.LAYER_SHAPES, synth.LAYER_INPUT_OF, combos):
        w = synth.ternary(rng, n, k)
        s_w = synth.weight_scale(rng)
        pk = pack_on_gpu(w)
        keep.append(pk)
        tws.append(tw2.make_tw(pk, n, k, s_w))
        xd.append(xdev[j])
        ys.append(Guarded((m, n), torch.float32))
        accs.append(Guarded((m, n), torch.int32))
        if combo is None:
            epis.append(None)
            ref.append((xs_host[j], w, s_w, None, None, None, False))
        else:
            b, g, r, relu = _operands(rng, m, n, combo)
            e, k_ = _epi_dev(b, g, r, relu)
            epis.append(e)
            keep.append(k_)
            ref.append((xs_host[j], w, s_w, b, g, r, relu))
    fl = flags_tensor()
    tw2.linear_stack(xd, tws, [y.t for y in ys], [a.t for a in accs], flags=fl, epis=epis)
    torch.cuda.synchronize()
    assert int(fl.item()) == 0
    for y, a, args in zip(ys, accs, ref):
        assert y.guard_intact() and a.guard_intact()
        _check(y.t.cpu().numpy(), a.t.cpu().numpy(), *_expected(*args))


def test_grouped_epilogue_prefill_2048_sampled():
    """The prefill launch (seven decoder shapes at M = 2048, one grouped call)
    with a different epilogue per layer: sampled columns against the oracle,
    every output against the epilogue applied to its own exact int32 sum."""
    m = 2048
    xs_by_k = synth.prefill_inputs(m)
    rng = np.random.default_rng(2048)
    xq, xsc, tws, ys, accs, epis, keep, ref = {}, {}, [], [], [], [], [], []
    for i, ((name, n, k), combo) in enumerate(zip(synth.LAYER_SHAPES, itertools.cycle(COMBOS))):
        r_ = np.random.default_rng(synth.seed_for(4, i))
        w = synth.ternary(r_, n, k)
        s_w = synth.weight_scale(r_)
        if k not in xq:
            q, s_act, _ = oracle.quant_act(xs_by_k[k])
            xq[k], xsc[k] = upload(q), (upload(s_act), s_act)
        pk = pack_on_gpu(w)
        keep.append(pk)
        tws.append(tw2.make_tw(pk, n, k, s_w))
        ys.append(Guarded((m, n), torch.float32))
        accs.append(Guarded((m, n), torch.int32))
        b, g, r, relu = _operands(rng, m, n, combo)
        e, k_ = _epi_dev(b, g, r, relu)
        epis.append(e)
        keep.append(k_)
        ref.append((xs_by_k[k], w, s_w, b, g, r, relu))
    fl = flags_tensor()
    tw2.linear_q_grouped([xq[t.k] for t in tws], [xsc[t.k][0] for t in tws], tws, [y.t for y in ys],
                         [a.t for a in accs], flags=fl, epis=epis)
    torch.cuda.synchronize()
    assert int(fl.item()) == 0
    for y, a, (x, w, s_w, b, g, r, relu) in zip(ys, accs, ref):
        assert y.guard_intact() and a.guard_intact()
        yg, ag = y.t.cpu().numpy(), a.t.cpu().numpy()
        n, k = w.shape
        cols = np.unique(np.concatenate([[0, n - 1], rng.choice(n, 6, replace=False)]))
        acc, o32, o64, scale = _expected(x, w, s_w, b, g, r, relu, cols=cols)
        _check(yg[:, cols], ag[:, cols], acc, o32, o64, scale)
        # every output: the oracle's epilogue on the dequantised exact sums
        s_act = xsc[k][1]
        y32 = (ag.astype(np.float32) * s_act[:, None]).astype(np.float32) * np.float32(s_w)
        full, _ = oracle.epilogue(y32, bias=b, gamma=g, residual=r, relu=relu)
        np.testing.assert_array_equal(yg.view(np.uint32), full.view(np.uint32))


def test_epilogue_reserved_field_rejected():
    pk = torch.zeros((4, 32), dtype=torch.uint8, device=DEV)
    tw = tw2.make_tw(pk, 4, 100, 1.0)
    x = torch.zeros((1, 100), dtype=torch.float32, device=DEV)
    y = torch.zeros((1, 4), dtype=torch.float32, device=DEV)
    epi = tw2.Epilogue(None, None, None, 0, 1)
    with pytest.raises(tw2.BitnetError) as e:
        tw2.linear(x, tw, y, epi=epi)
    assert e.value.status == 1   # BITNET_ERR_INVALID_ARG
