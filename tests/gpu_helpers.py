"""Shared helpers of the GPU tests: guarded device buffers (NaN / canary
poisoned, with a 256-byte guard after the live region) and upload helpers."""
import numpy as np
import torch

import oracle
import ternary_weight_i2_b200 as tw2

DEV = "cuda"
GUARD_BYTES = 256
CANARY = {torch.int8: 0x5A, torch.uint8: 0xA5, torch.int32: -123456789}


class Guarded:
    """A device tensor with a poisoned guard region after it."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) if len(shape) else 1
        esz = torch.empty((), dtype=dtype).element_size()
        self.n = n
        self.g = GUARD_BYTES // esz
        self.buf = torch.empty(n + self.g, dtype=dtype, device=DEV)
        if dtype.is_floating_point:
            self.fill = float("nan")
        else:
            self.fill = CANARY[dtype]
        self.buf.fill_(self.fill)
        self.t = self.buf[:n].view(*shape)

    def guard_intact(self) -> bool:
        tail = self.buf[self.n:]
        if self.buf.dtype.is_floating_point:
            return bool(torch.isnan(tail).all())
        return bool((tail == self.fill).all())


def upload(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def flags_tensor():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def pack_on_gpu(w: np.ndarray):
    """Pack int8 weights with the CUDA kernel; returns the device buffer."""
    n, k = w.shape
    wt = upload(w)
    pk = torch.empty((n, 32 * oracle.blocks(k)), dtype=torch.uint8, device=DEV)
    fl = flags_tensor()
    tw2.pack_ternary(wt, pk, flags=fl)
    torch.cuda.synchronize()
    assert int(fl.item()) == 0
    return pk


def rel_err(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.maximum(np.abs(b), 1e-30)
    return float(np.max(np.abs(a - b) / den)) if a.size else 0.0
