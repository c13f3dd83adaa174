"""ctypes binding of libbitlinear.so (include/bitlinear.h).

Argument marshalling only: every step of the BitLinear path runs in the CUDA
kernels behind the C ABI. The library must be built (build.build_library()); a
missing library raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbitlinear.so")

BL_OK = 0
STATUS_NAMES = {
    0: "BL_OK",
    1: "BL_ERR_NULL",
    2: "BL_ERR_SHAPE",
    3: "BL_ERR_ALIGN",
    4: "BL_ERR_WORKSPACE",
    5: "BL_ERR_NONFINITE",
    6: "BL_ERR_DEVICE",
    7: "BL_ERR_CUDA",
    8: "BL_ERR_UNSUPPORTED",
    9: "BL_ERR_FORMAT",
}

# name -> (restype, argtypes), mirroring include/bitlinear.h
_VP = ctypes.c_void_p
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
SIGNATURES = {
    "bitlinear_abi_version": (ctypes.c_int, []),
    "bitlinear_build_id": (ctypes.c_char_p, []),
    "bitlinear_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "bitlinear_device_check": (ctypes.c_int, []),
    "bitlinear_pack_workspace_size": (_SZ, [_I64, _I64]),
    "bitlinear_pack_weights": (ctypes.c_int, [_VP, _I64, _I64, _VP, _VP, _VP, _SZ, _VP]),
    "bitlinear_pack_weights_async": (ctypes.c_int, [_VP, _I64, _I64, _VP, _VP, _VP, _SZ, _VP]),
    "bitlinear_pack_status": (ctypes.c_int, [_VP, _SZ, _VP]),
    "bitlinear_quant_act": (ctypes.c_int, [_VP, _I64, _I64, _VP, _VP, _VP, _VP]),
    "bitlinear_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "bitlinear_forward": (ctypes.c_int, [_VP, _I64, _I64, _I64, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "bitlinear_forward_acc": (ctypes.c_int, [_VP, _I64, _I64, _I64, _VP, _VP, _VP, _SZ, _VP]),
    "bitlinear_prepare_act": (ctypes.c_int, [_VP, _I64, _I64, _VP, _SZ, _VP]),
    "bitlinear_forward_prepared": (ctypes.c_int, [_I64, _I64, _I64, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "bitlinear_batch_workspace_size": (_SZ, [_VP, ctypes.c_int]),
    "bitlinear_forward_batch": (ctypes.c_int, [_VP, ctypes.c_int, ctypes.c_uint32, _VP, _SZ, _VP]),
    "bitlinear_host_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "bitlinear_forward_host": (ctypes.c_int, [_VP, _I64, _I64, _I64, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "bitlinear_forward_host_async": (ctypes.c_int, [_VP, _I64, _I64, _I64, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "bitlinear_forward_q": (ctypes.c_int, [_VP, _VP, _I64, _I64, _I64, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "bitlinear_pack_weights_bf16": (ctypes.c_int, [_VP, _I64, _I64, _VP, _VP, _VP, _SZ, _VP]),
    "bitlinear_quant_act_bf16": (ctypes.c_int, [_VP, _I64, _I64, _VP, _VP, _VP, _VP]),
    "bitlinear_forward_bf16": (ctypes.c_int, [_VP, _I64, _I64, _I64, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "bitlinear_batch_host_workspace_size": (ctypes.c_size_t, [_VP, ctypes.c_int]),
    "bitlinear_forward_batch_host": (ctypes.c_int, [_VP, ctypes.c_int, ctypes.c_uint32, _VP, _SZ, _VP]),
    "bitlinear_i2s_bytes": (_SZ, [ctypes.c_int64, ctypes.c_int64]),
    "bitlinear_i2s_workspace_size": (_SZ, []),
    "bitlinear_i2s_export": (ctypes.c_int, [_VP, _VP, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, _VP, _VP, _SZ,
                                            _VP]),
    "bitlinear_i2s_import": (ctypes.c_int, [_VP, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, _VP, _VP, _VP, _SZ,
                                            _VP]),
    "bitlinear_i2s_export_async": (ctypes.c_int, [_VP, _VP, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, _VP, _VP,
                                                  _SZ, _VP]),
    "bitlinear_i2s_import_async": (ctypes.c_int, [_VP, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, _VP, _VP, _VP,
                                                  _SZ, _VP]),
    "bitlinear_i2s_status": (ctypes.c_int, [_VP, _SZ, _VP]),
    "bitlinear_rmsnorm_quant_act": (ctypes.c_int, [_VP, _VP, ctypes.c_float, _I64, _I64, _VP, _VP, _VP, _VP]),
    "bitlinear_forward_rmsnorm": (ctypes.c_int, [_VP, _VP, ctypes.c_float, _I64, _I64, _I64, _VP, _VP, _VP,
                                                 _VP, _SZ, _VP]),
    "bitlinear_block_scales": (_I64, [_I64]),
    "bitlinear_blocks_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "bitlinear_pack_weights_blocks": (ctypes.c_int, [_VP, _I64, _I64, _VP, _VP, _VP, _SZ, _VP]),
    "bitlinear_forward_blocks": (ctypes.c_int, [_VP, _I64, _I64, _I64, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "bitlinear_pack_weights_blocks_bf16": (ctypes.c_int, [_VP, _I64, _I64, _VP, _VP, _VP, _SZ, _VP]),
    "bitlinear_forward_blocks_bf16": (ctypes.c_int, [_VP, _I64, _I64, _I64, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "bitlinear_workspace_error": (ctypes.c_int, [_VP, _SZ, _VP]),
    "bitlinear_selftest_wait_timeout": (ctypes.c_int, [_VP, _SZ, ctypes.c_uint64, _VP]),
    "bitlinear_forward_noalloc": (ctypes.c_int, [_VP, _I64, _I64, _I64, _VP, _VP, _VP, _VP]),
    "bitlinear_noalloc_error": (ctypes.c_int, [_VP]),
    "bitlinear_noalloc_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_uint64, _VP]),
}

_lock = threading.Lock()
_lib = None


class LinearCall(ctypes.Structure):
    """Mirror of bl_linear_call (include/bitlinear.h)."""

    _fields_ = [
        ("x", ctypes.c_void_p),
        ("M", ctypes.c_int64),
        ("N", ctypes.c_int64),
        ("K", ctypes.c_int64),
        ("packed", ctypes.c_void_p),
        ("D", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
    ]


BL_FLAG_STREAM_WEIGHTS_EARLY = 1
BL_FLAG_ONE_LAUNCH_PER_CALL = 2
BL_I2S_CONSECUTIVE = 0
BL_I2S_QUARTERS = 1


class BitLinearError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)} ({status})")


def lib() -> ctypes.CDLL:
    """Load libbitlinear.so once. Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m bit_ternary_b200.build` "
                    "(there is no fallback implementation)")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            from . import build

            built = L.bitlinear_build_id().decode()
            if built != build.sources_sha():
                raise RuntimeError(
                    f"{LIB_PATH} was built from other sources (build id {built}, sources "
                    f"{build.sources_sha()}): rebuild it with `python -m bit_ternary_b200.build --force`")
            _lib = L
    return _lib


def check(fn: str, status: int) -> None:
    if status != BL_OK:
        raise BitLinearError(fn, status)


def call(fn: str, *args) -> int:
    """Call an int-returning entry point and raise on a non-OK status."""
    st = getattr(lib(), fn)(*args)
    check(fn, st)
    return st
