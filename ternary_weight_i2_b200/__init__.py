"""I2_S ternary linear layer for NVIDIA B200 (sm_100a).

The compute lives in ``libbitnet.so`` (CUDA kernels behind the C ABI of
``include/bitnet.h``); this package binds it with ctypes.  PyTorch is only
used by callers for device memory and streams.
"""
from ._abi import (  # noqa: F401
    BitnetError, Epilogue, I8GroupCall, I8W, StackCall, TW, make_epilogue, make_i8w, linear_i8, i8_row_bytes,
    linear_i8_workspace_bytes, header_functions, kpad, linear, linear_q, linear_stack,
    linear_stack_noalloc, linear_q_grouped, GroupedCall,
    linear_workspace_bytes, load, make_tw, pack_ternary, packed_bytes, quant_act,
    quantize_pack, quantize_pack_workspace_bytes,
    status_from_flags, unpack_ternary, version,
    FLAG_NONFINITE, FLAG_NOT_TERNARY, FLAG_TIMEOUT, GEMV_MAX_M, MAX_K, STACK_MAX,
)
