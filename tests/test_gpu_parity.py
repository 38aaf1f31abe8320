"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

int32 accumulators and int8 codes must match bit for bit; fp32 outputs must be
within 1e-5 relative of the oracle's fp64 value (they are in fact expected to
equal the oracle's fp32 form bit for bit, which is checked too).  Outputs are
poisoned with NaN and followed by guard canaries before every call.
"""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_i2_b200 as tw2
from ternary_weight_i2_b200 import synth

from gpu_helpers import DEV, Guarded, flags_tensor, pack_on_gpu, rel_err, upload

pytestmark = pytest.mark.gpu
RTOL = 1e-5


# ------------------------------------------------------------------ pack

@pytest.mark.parametrize("k", [1, 5, 31, 127, 128, 129, 300, 1536, 8960, 9024])
@pytest.mark.parametrize("n", [1, 3, 33, 256])
def test_pack_matches_oracle(n, k):
    rng = np.random.default_rng(1000 * n + k)
    w = synth.ternary(rng, n, k)
    want, _ = oracle.pack(w)
    wt = upload(w)
    pk = Guarded((n, 32 * oracle.blocks(k)), torch.uint8)
    fl = flags_tensor()
    tw2.pack_ternary(wt, pk.t, flags=fl)
    torch.cuda.synchronize()
    assert int(fl.item()) == 0
    np.testing.assert_array_equal(pk.t.cpu().numpy(), want)
    assert pk.guard_intact()
    back = Guarded((n, k), torch.int8)
    tw2.unpack_ternary(pk.t, n, k, back.t)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(back.t.cpu().numpy(), w)
    assert back.guard_intact()


def test_pack_flags_non_ternary():
    w = np.zeros((4, 200), np.int8)
    w[2, 150] = 3
    want, st = oracle.pack(w)
    assert st == oracle.NOT_TERNARY
    pk = torch.empty((4, 64), dtype=torch.uint8, device=DEV)
    fl = flags_tensor()
    tw2.pack_ternary(upload(w), pk, flags=fl)
    torch.cuda.synchronize()
    assert int(fl.item()) & tw2.FLAG_NOT_TERNARY
    np.testing.assert_array_equal(pk.cpu().numpy(), want)


# ----------------------------------------------------------------- quant

def _special_x(k):
    x = synth.normal_outliers(np.random.default_rng(k), 9, k)
    x[1] = 2.5
    x[2] = 0
    x[3, :] = np.float32(1.0)
    x[3, k // 3] = np.nan
    x[4] *= np.float32(1e-30)
    x[5, :min(k, 4)] = np.array([1e-38, -5e-39, 0.0, 2e-39], np.float32)[:min(k, 4)]
    x[5, 4:] = 0
    halves = (np.arange(k, dtype=np.float32) % 255) - np.float32(126.5)
    x[6] = halves
    x[6, 0] = 127.0                       # inv == 1: every half is a tie
    x[7] = -np.abs(x[7])
    x[8, -1] = np.inf
    return x


@pytest.mark.parametrize("k", [1, 3, 128, 130, 1536, 8960, 9024])
def test_quant_matches_oracle(k):
    x = _special_x(k)
    q_want, s_want, st = oracle.quant_act(x)
    m = x.shape[0]
    kp = oracle.kpad(k)
    xq = Guarded((m, kp), torch.int8)
    sc = Guarded((m,), torch.float32)
    fl = flags_tensor()
    tw2.quant_act(upload(x), xq.t, sc.t, flags=fl)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(xq.t.cpu().numpy(), q_want)
    np.testing.assert_array_equal(sc.t.cpu().numpy().view(np.uint32), s_want.view(np.uint32))
    assert xq.guard_intact() and sc.guard_intact()
    assert bool(int(fl.item()) & tw2.FLAG_NONFINITE) == bool(st & oracle.NONFINITE)


# ---------------------------------------------------------------- linear

def _check_linear(x, w, s_w, rows=None, m_limit_full=None):
    """Run bitnet_linear and compare with the oracle (all outputs, or the
    sampled output rows `rows`)."""
    m, k = x.shape
    n = w.shape[0]
    pk_np, _ = oracle.pack(w)
    pk = pack_on_gpu(w)
    tw = tw2.make_tw(pk, n, k, s_w)
    y = Guarded((m, n), torch.float32)
    acc = Guarded((m, n), torch.int32)
    ws_bytes = tw2.linear_workspace_bytes(m, k)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=DEV) if ws_bytes else None
    fl = flags_tensor()
    tw2.linear(upload(x), tw, y.t, acc=acc.t, workspace=ws, flags=fl)
    torch.cuda.synchronize()
    assert y.guard_intact() and acc.guard_intact()
    yg = y.t.cpu().numpy()
    ag = acc.t.cpu().numpy()
    assert not np.isnan(yg).any()
    if rows is None:
        a_want, y64, y32, st = oracle.linear(x, pk_np, n, k, s_w)
        np.testing.assert_array_equal(ag, a_want)
        assert rel_err(yg, y64) <= RTOL
        np.testing.assert_array_equal(yg.view(np.uint32), y32.view(np.uint32))
    else:
        a_want, y64, st = oracle.linear_rows(x, pk_np, n, k, s_w, rows)
        np.testing.assert_array_equal(ag[:, rows], a_want)
        assert rel_err(yg[:, rows], y64) <= RTOL
    # dequantisation of every output is consistent with its accumulator
    _, s_act, _ = oracle.quant_act(x)
    y32_all = (ag.astype(np.float32) * s_act[:, None]).astype(np.float32) * np.float32(s_w)
    np.testing.assert_array_equal(yg.view(np.uint32), y32_all.astype(np.float32).view(np.uint32))
    assert (int(fl.item()) != 0) == (st != 0)
    return ag, yg


def test_single_layer_1536():
    w, s_w, x = synth.single_layer()
    _check_linear(x, w, s_w)


def _edge_rows(n):
    r = np.unique(np.concatenate([np.arange(min(n, 40)), np.linspace(0, n - 1, 24).astype(np.int64),
                                  [n - 33, n - 32, n - 31, n - 2, n - 1]]))
    return r[(r >= 0) & (r < n)]


@pytest.mark.parametrize("n", synth.EDGE_N)
@pytest.mark.parametrize("k", synth.EDGE_K)
@pytest.mark.parametrize("m", synth.EDGE_M)
def test_edge_sweep(m, k, n):
    w, s_w, x = synth.edge_case(m, k, n, seed=synth.seed_for(5, 100 * m + n % 97, k))
    full = m * n * k <= 40_000_000
    _check_linear(x, w, s_w, rows=None if full else _edge_rows(n))


@pytest.mark.parametrize("m", [1, 2, 3, 4, 5, 6, 7, 8])
def test_saturation_max_k(m):
    k, n = 9024, 64
    x = np.full((m, k), 0.5, np.float32)
    if m > 1:
        x[m - 1] = -0.5
    w = np.ones((n, k), np.int8)
    w[1::2] = -1
    ag, _ = _check_linear(x, w, 0.05)
    assert ag[0, 0] == 127 * 9024 and ag[0, 1] == -127 * 9024
    if m > 1:
        assert ag[m - 1, 0] == -127 * 9024


@pytest.mark.parametrize("m", [1, 4, 8])
def test_linear_q_prequantised(m):
    rng = np.random.default_rng(77 + m)
    k, n = 1536, 1536
    w = synth.ternary(rng, n, k)
    x = synth.normal_outliers(rng, m, k)
    s_w = synth.weight_scale(rng)
    q, s_act, _ = oracle.quant_act(x)
    pk_np, _ = oracle.pack(w)
    a_want, y64, y32, _ = oracle.linear(x, pk_np, n, k, s_w)
    pk = pack_on_gpu(w)
    y = Guarded((m, n), torch.float32)
    acc = Guarded((m, n), torch.int32)
    tw2.linear_q(upload(q), upload(s_act), tw2.make_tw(pk, n, k, s_w), y.t, acc=acc.t)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(acc.t.cpu().numpy(), a_want)
    np.testing.assert_array_equal(y.t.cpu().numpy().view(np.uint32), y32.view(np.uint32))
    assert y.guard_intact() and acc.guard_intact()


# ---------------------------------------------------------------- stack

_WEIGHT_CACHE = {}


def _stack_weights(layers, config):
    """Packed device weights + host int8 copies of `layers` (cached per config)."""
    key = (tuple(layers), config)
    if key not in _WEIGHT_CACHE:
        _WEIGHT_CACHE.clear()
        out = []
        for L in layers:
            for (name, n, k), (w, s) in zip(synth.LAYER_SHAPES, synth.layer_weights(L, config)):
                out.append((w, s, n, k, pack_on_gpu(w)))
        _WEIGHT_CACHE[key] = out
    return _WEIGHT_CACHE[key]


def _layer_stack(layers, m, config=3):
    """GPU descriptors, inputs and poisoned outputs of a stack of decoder layers."""
    host = _stack_weights(list(layers), config)
    tws, xs_dev, xs_host, ys, accs = [], [], [], [], []
    for li, L in enumerate(layers):
        xl = synth.layer_inputs(L, m, config)
        xd = [upload(a) for a in xl]
        for j, (w, s, n, k, pk) in zip(synth.LAYER_INPUT_OF, host[7 * li: 7 * li + 7]):
            tws.append(tw2.make_tw(pk, n, k, s))
            xs_dev.append(xd[j])
            xs_host.append(xl[j])
            ys.append(Guarded((m, n), torch.float32))
            accs.append(Guarded((m, n), torch.int32))
    return tws, host, xs_dev, xs_host, ys, accs


@pytest.mark.parametrize("m", [1, 3, 8])
def test_stack_one_layer_full(m):
    tws, host, xd, xh, ys, accs = _layer_stack([0], m, config=2)
    fl = flags_tensor()
    tw2.linear_stack(xd, tws, [y.t for y in ys], [a.t for a in accs], flags=fl)
    torch.cuda.synchronize()
    assert int(fl.item()) == 0
    for (w, s, n, k, _), x, y, a in zip(host, xh, ys, accs):
        pk_np, _ = oracle.pack(w)
        a_want, y64, y32, _ = oracle.linear(x, pk_np, n, k, s)
        np.testing.assert_array_equal(a.t.cpu().numpy(), a_want)
        np.testing.assert_array_equal(y.t.cpu().numpy().view(np.uint32), y32.view(np.uint32))
        assert rel_err(y.t.cpu().numpy(), y64) <= RTOL
        assert y.guard_intact() and a.guard_intact()


@pytest.mark.parametrize("m", [1, 2, 4, 8])
def test_stack_28_layers_sampled(m):
    """The full 28-layer stack in the benchmark's launch configuration: sampled
    output rows of every layer against the oracle, every output checked
    against the same layer run alone."""
    tws, host, xd, xh, ys, accs = _layer_stack(range(synth.NUM_LAYERS), m)
    fl = flags_tensor()
    tw2.linear_stack(xd, tws, [y.t for y in ys], [a.t for a in accs], flags=fl)
    torch.cuda.synchronize()
    assert int(fl.item()) == 0
    rng = np.random.default_rng(m)
    for i, ((w, s, n, k, pk), x, y, a) in enumerate(zip(host, xh, ys, accs)):
        assert y.guard_intact() and a.guard_intact()
        rows = np.unique(np.concatenate([[0, 31, 32, n - 1], rng.choice(n, 6, replace=False)]))
        pk_np, _ = oracle.pack(w[rows])
        a_want, y64, y32, _ = oracle.linear(x, pk_np, len(rows), k, s)
        ag = a.t.cpu().numpy()
        np.testing.assert_array_equal(ag[:, rows], a_want)
        np.testing.assert_array_equal(y.t.cpu().numpy()[:, rows].view(np.uint32), y32.view(np.uint32))
        if i % 7 in (0, 6):   # one K=1536 and the K=8960 layer of each decoder layer
            y1 = Guarded((m, n), torch.float32)
            a1 = Guarded((m, n), torch.int32)
            tw2.linear(xd[i], tws[i], y1.t, acc=a1.t)
            torch.cuda.synchronize()
            assert torch.equal(a1.t, a.t) and torch.equal(y1.t, y.t)


# -------------------------------------------------------- failure paths

def test_forced_timeout_returns_status_and_context_survives():
    rng = np.random.default_rng(3)
    w = synth.ternary(rng, 256, 1536)
    x = synth.normal(rng, 1, 1536)
    pk = pack_on_gpu(w)
    tw = tw2.make_tw(pk, 256, 1536, 0.05)
    y = torch.zeros((1, 256), dtype=torch.float32, device=DEV)
    fl = flags_tensor()
    try:
        tw2._abi.set_wait_limit(20000)
        tw2._abi.force_stall(True)
        tw2.linear(upload(x), tw, y, flags=fl)
        torch.cuda.synchronize()
    finally:
        tw2._abi.force_stall(False)
        tw2._abi.set_wait_limit(0)
    assert int(fl.item()) & tw2.FLAG_TIMEOUT
    assert tw2.status_from_flags(int(fl.item())) == tw2._abi.ERR_TIMEOUT
    # the context is still usable and the next call is correct
    fl.zero_()
    tw2.linear(upload(x), tw, y, flags=fl)
    torch.cuda.synchronize()
    assert int(fl.item()) == 0
    pk_np, _ = oracle.pack(w)
    _, _, y32, _ = oracle.linear(x, pk_np, 256, 1536, 0.05)
    np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), y32.view(np.uint32))


def test_unsupported_device_is_refused(monkeypatch):
    x = torch.zeros((1, 128), dtype=torch.float32, device=DEV)
    pk = torch.zeros((4, 32), dtype=torch.uint8, device=DEV)
    y = torch.full((1, 4), float("nan"), device=DEV)
    monkeypatch.setenv("BITNET_TEST_FORCE_SM", "90")
    with pytest.raises(tw2.BitnetError) as e:
        tw2.linear(x, tw2.make_tw(pk, 4, 128, 1.0), y)
    assert e.value.status == tw2._abi.ERR_UNSUPPORTED_DEVICE
    torch.cuda.synchronize()
    assert torch.isnan(y).all()        # nothing was launched
