"""bitnet_linear_stack_noalloc: the decode stack for callers that cannot call
cudaMalloc (an application whose device memory belongs to its own pooling
allocator, or a loop that must not allocate after start-up).  It keeps the
per-layer TMA tensor maps in the library's fixed device array instead of the
allocated per-device cache, so its results must be exactly those of
bitnet_linear_stack.  The calls below compare the two on consecutive calls,
including calls that switch to different weights (the array is rewritten) and
back.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import ternary_weight_i2_b200 as tw2
from ternary_weight_i2_b200 import synth

from gpu_helpers import DEV, Guarded, flags_tensor, pack_on_gpu, rel_err, upload

pytestmark = pytest.mark.gpu
RTOL = 1e-5


def _stack(layers, m, config):
    tws, xs, keep = [], [], []
    for L in layers:
        xl = [upload(a) for a in synth.layer_inputs(L, m, config)]
        keep.append(xl)
        for (_, n, k), (w, s), j in zip(synth.LAYER_SHAPES, synth.layer_weights(L, config),
                                        synth.LAYER_INPUT_OF):
            pk = pack_on_gpu(w)
            keep.append(pk)
            tws.append(tw2.make_tw(pk, n, k, s))
            xs.append(xl[j])
    return tws, xs, keep


def _outputs(tws, m):
    ys = [Guarded((m, tw.n), torch.float32) for tw in tws]
    accs = [Guarded((m, tw.n), torch.int32) for tw in tws]
    return ys, accs


def _run(fn, tws, xs, m):
    ys, accs = _outputs(tws, m)
    fl = flags_tensor()
    fn(xs, tws, [y.t for y in ys], [a.t for a in accs], flags=fl)
    torch.cuda.synchronize()
    assert int(fl.item()) == 0
    for y, a in zip(ys, accs):
        assert y.guard_intact() and a.guard_intact()
        assert not torch.isnan(y.t).any()
    return ys, accs


def test_noalloc_stack_equals_stack_on_consecutive_calls():
    stacks = {
        "a": (_stack([0, 1], 1, 3), 1),
        "b": (_stack([5, 9, 20], 3, 3), 3),
    }
    for name in ("a", "a", "b", "a"):        # two calls in a row, then switch and back
        (tws, xs, _), m = stacks[name]
        ys_ref, accs_ref = _run(tw2.linear_stack, tws, xs, m)
        ys, accs = _run(tw2.linear_stack_noalloc, tws, xs, m)
        for y, yr, a, ar in zip(ys, ys_ref, accs, accs_ref):
            assert torch.equal(a.t, ar.t)
            assert rel_err(y.t.cpu().numpy(), yr.t.cpu().numpy()) <= RTOL
            assert torch.equal(y.t, yr.t)


def test_noalloc_stack_rejects_more_layers_than_its_array_holds():
    rng = np.random.default_rng(0)
    w = synth.ternary(rng, 32, 128)
    pk = pack_on_gpu(w)
    x = upload(synth.normal(rng, 1, 128))
    tws = [tw2.make_tw(pk, 32, 128, 0.1)] * 257
    ys = [torch.empty((1, 32), device=DEV) for _ in range(257)]
    with pytest.raises(tw2.BitnetError) as e:
        tw2._abi.linear_stack_noalloc([x] * 257, tws, ys)
    assert e.value.status == tw2._abi.ERR_INVALID_ARG
    assert "256" in str(e.value)
