"""Parity of the prefill path (M > 8: per-token quantiser + tcgen05 int8 GEMM)
with the CPU oracle, through the C ABI.  Full comparisons on shapes the oracle
finishes in seconds (several 128 x 192 tiles and ragged tails); at the prefill
size (M = 2048 over the seven decoder-layer shapes, the launch bench.py times)
every output is checked against its exact int32 sum by the dequantisation
identity and sampled output columns against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_i2_b200 as tw2
from ternary_weight_i2_b200 import synth

from gpu_helpers import DEV, Guarded, flags_tensor, pack_on_gpu, rel_err, upload

pytestmark = pytest.mark.gpu
RTOL = 1e-5


def _run(x, w, s_w, quantised=False):
    m, k = x.shape
    n = w.shape[0]
    pk = pack_on_gpu(w)
    tw = tw2.make_tw(pk, n, k, s_w)
    y = Guarded((m, n), torch.float32)
    acc = Guarded((m, n), torch.int32)
    fl = flags_tensor()
    if quantised:
        q, s_act, _ = oracle.quant_act(x)
        tw2.linear_q(upload(q), upload(s_act), tw, y.t, acc=acc.t, flags=fl)
    else:
        ws = torch.empty(tw2.linear_workspace_bytes(m, k), dtype=torch.uint8, device=DEV)
        tw2.linear(upload(x), tw, y.t, acc=acc.t, workspace=ws, flags=fl)
    torch.cuda.synchronize()
    assert int(fl.item()) == 0
    assert y.guard_intact() and acc.guard_intact()
    return y.t.cpu().numpy(), acc.t.cpu().numpy()


@pytest.mark.parametrize("m,k,n", [(9, 128, 256), (128, 128, 256), (128, 1536, 256), (130, 1536, 300),
                                   (257, 1536, 512), (300, 9024, 264), (2048, 1536, 256)])
@pytest.mark.parametrize("quantised", [False, True])
def test_gemm_full_parity(m, k, n, quantised):
    rng = np.random.default_rng(m * 7 + k + n)
    w = synth.ternary(rng, n, k)
    x = synth.normal_row_spread(rng, m, k)
    s_w = synth.weight_scale(rng)
    yg, ag = _run(x, w, s_w, quantised)
    pk_np, _ = oracle.pack(w)
    a_want, y64, y32, st = oracle.linear(x, pk_np, n, k, s_w)
    assert st == 0
    np.testing.assert_array_equal(ag, a_want)
    assert rel_err(yg, y64) <= RTOL
    np.testing.assert_array_equal(yg.view(np.uint32), y32.view(np.uint32))


def test_gemm_special_rows_and_saturation():
    m, k, n = 200, 9024, 256
    x = np.full((m, k), 0.25, np.float32)
    x[1] = -0.25
    x[2] = 0.0
    x[3, 5] = np.float32(3e4)
    w = np.ones((n, k), np.int8)
    w[1] = -1
    w[2] = 0
    w[3::2] = synth.ternary(np.random.default_rng(1), (n - 3 + 1) // 2, k)
    yg, ag = _run(x, w, 0.03)
    pk_np, _ = oracle.pack(w)
    a_want, _, y32, _ = oracle.linear(x, pk_np, n, k, 0.03)
    np.testing.assert_array_equal(ag, a_want)
    np.testing.assert_array_equal(yg.view(np.uint32), y32.view(np.uint32))
    assert ag[0, 0] == 127 * 9024 and ag[1, 0] == -127 * 9024 and ag[0, 1] == -127 * 9024


@pytest.mark.parametrize("shape", range(len(synth.LAYER_SHAPES)))
def test_prefill_2048_sampled(shape):
    name, n, k = synth.LAYER_SHAPES[shape]
    rng = np.random.default_rng(synth.seed_for(4, shape))
    w = synth.ternary(rng, n, k)
    s_w = synth.weight_scale(rng)
    x = synth.prefill_inputs(2048)[k]
    yg, ag = _run(x, w, s_w)
    cols = np.unique(np.concatenate([[0, 1, 255, min(256, n - 1), n - 1], rng.choice(n, 11, replace=False)]))
    pk_np, _ = oracle.pack(w[cols])
    a_want, y64, y32, _ = oracle.linear(x, pk_np, len(cols), k, s_w)
    np.testing.assert_array_equal(ag[:, cols], a_want)
    np.testing.assert_array_equal(yg[:, cols].view(np.uint32), y32.view(np.uint32))
    # every output is the dequantisation of its own accumulator
    _, s_act, _ = oracle.quant_act(x)
    y_all = (ag.astype(np.float32) * s_act[:, None]).astype(np.float32) * np.float32(s_w)
    np.testing.assert_array_equal(yg.view(np.uint32), y_all.view(np.uint32))
    # |acc| is bounded by sum_k |q| for ternary weights
    q, _, _ = oracle.quant_act(x)
    assert (np.abs(ag.astype(np.int64)) <= np.abs(q.astype(np.int64)).sum(axis=1)[:, None]).all()


def _grouped(xs, ws, scales, shared_index=None):
    """Run bitnet_linear_q_grouped over layers (x_i, w_i); returns y, acc lists."""
    xq_dev, s_dev = {}, {}
    keys = shared_index or list(range(len(ws)))
    for key, x in zip(keys, xs):
        if key not in xq_dev:
            q, s, _ = oracle.quant_act(x)
            xq_dev[key], s_dev[key] = upload(q), upload(s)
    tws, ys, accs = [], [], []
    for w, sw in zip(ws, scales):
        n, k = w.shape
        pk = pack_on_gpu(w)
        tws.append(tw2.make_tw(pk, n, k, sw))
        ys.append(Guarded((xs[0].shape[0], n), torch.float32))
        accs.append(Guarded((xs[0].shape[0], n), torch.int32))
        tws[-1]._keep = pk
    fl = flags_tensor()
    tw2.linear_q_grouped([xq_dev[k] for k in keys], [s_dev[k] for k in keys], tws, [y.t for y in ys],
                         [a.t for a in accs], flags=fl)
    torch.cuda.synchronize()
    assert int(fl.item()) == 0
    for y, a in zip(ys, accs):
        assert y.guard_intact() and a.guard_intact()
    return [y.t.cpu().numpy() for y in ys], [a.t.cpu().numpy() for a in accs]


def test_grouped_full_parity_mixed_shapes():
    rng = np.random.default_rng(31)
    m = 200
    shapes = [(300, 1536), (256, 9024), (512, 1536), (100, 128)]
    xa = synth.normal_row_spread(rng, m, 1536)
    xb = synth.normal_row_spread(rng, m, 9024)
    xc = synth.normal_row_spread(rng, m, 128)
    xs = [xa, xb, xa, xc]
    ws = [synth.ternary(rng, n, k) for n, k in shapes]
    sc = [synth.weight_scale(rng) for _ in shapes]
    ys, accs = _grouped(xs, ws, sc, shared_index=[0, 1, 0, 2])
    for x, w, s, y, a in zip(xs, ws, sc, ys, accs):
        pk_np, _ = oracle.pack(w)
        a_want, y64, y32, _ = oracle.linear(x, pk_np, w.shape[0], w.shape[1], s)
        np.testing.assert_array_equal(a, a_want)
        np.testing.assert_array_equal(y.view(np.uint32), y32.view(np.uint32))
        assert rel_err(y, y64) <= RTOL


def test_grouped_prefill_2048_seven_shapes_sampled():
    """The launch bench.py times: all seven decoder shapes at M = 2048 in one call."""
    xs_by_k = synth.prefill_inputs(2048)
    xs, ws, sc, keys = [], [], [], []
    for i, (name, n, k) in enumerate(synth.LAYER_SHAPES):
        rng = np.random.default_rng(synth.seed_for(4, i))
        ws.append(synth.ternary(rng, n, k))
        sc.append(synth.weight_scale(rng))
        xs.append(xs_by_k[k])
        keys.append(k)
    ys, accs = _grouped(xs, ws, sc, shared_index=keys)
    rng = np.random.default_rng(5)
    for x, w, s, y, a in zip(xs, ws, sc, ys, accs):
        n, k = w.shape
        cols = np.unique(np.concatenate([[0, n - 1], rng.choice(n, 6, replace=False)]))
        pk_np, _ = oracle.pack(w[cols])
        a_want, _, y32, _ = oracle.linear(x, pk_np, len(cols), k, s)
        np.testing.assert_array_equal(a[:, cols], a_want)
        np.testing.assert_array_equal(y[:, cols].view(np.uint32), y32.view(np.uint32))
        _, s_act, _ = oracle.quant_act(x)
        y_all = (a.astype(np.float32) * s_act[:, None]).astype(np.float32) * np.float32(s)
        np.testing.assert_array_equal(y.view(np.uint32), y_all.view(np.uint32))


def test_gemm_forced_timeout_returns_status_and_context_survives():
    """The prefill kernel's bounded waits: with the test aid on, one K block's
    copies are never issued; the expanders' wait for them runs out, the launch
    ends with the timeout flag (every role still passes its barriers), and the
    next call is correct."""
    rng = np.random.default_rng(17)
    m, k, n = 200, 1536, 1536
    w = synth.ternary(rng, n, k)
    x = synth.normal_row_spread(rng, m, k)
    s_w = synth.weight_scale(rng)
    pk = pack_on_gpu(w)
    tw = tw2.make_tw(pk, n, k, s_w)
    y = torch.zeros((m, n), dtype=torch.float32, device=DEV)
    ws = torch.empty(tw2.linear_workspace_bytes(m, k), dtype=torch.uint8, device=DEV)
    fl = flags_tensor()
    try:
        tw2._abi.set_wait_limit(20000)
        tw2._abi.force_stall(True)
        tw2.linear(upload(x), tw, y, workspace=ws, flags=fl)
        torch.cuda.synchronize()
    finally:
        tw2._abi.force_stall(False)
        tw2._abi.set_wait_limit(0)
    assert int(fl.item()) & tw2.FLAG_TIMEOUT
    assert tw2.status_from_flags(int(fl.item())) == tw2._abi.ERR_TIMEOUT
    fl.zero_()
    tw2.linear(upload(x), tw, y, workspace=ws, flags=fl)
    torch.cuda.synchronize()
    assert int(fl.item()) == 0
    pk_np, _ = oracle.pack(w)
    _, _, y32, _ = oracle.linear(x, pk_np, n, k, s_w)
    np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), y32.view(np.uint32))
