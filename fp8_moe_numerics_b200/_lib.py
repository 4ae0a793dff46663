"""ctypes loader for libmxmoe.so, the C-ABI CUDA library (include/mxmoe.h).

The library is built in-tree by ``python -m fp8_moe_numerics_b200.build``.  A
missing library raises immediately: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# MX_DEBUG=1 loads the bounds-checked build (python -m fp8_moe_numerics_b200.build --debug-bounds)
LIB_PATH = os.path.join(_HERE, "libmxmoe_debug.so" if os.environ.get("MX_DEBUG") == "1" else "libmxmoe.so")

MX_OK, MX_EINVAL, MX_ECUDA, MX_ETIMEOUT, MX_EUNSUPPORTED, MX_EDATA = 0, 1, 2, 3, 4, 5
MX_SF_ROWMAJOR, MX_SF_MMA = 0, 1
MX_OUT_F32, MX_OUT_BF16 = 0, 1
MX_ROUND_RNE, MX_ROUND_SR = 0, 1
MX_GEMM_DGRAD, MX_GEMM_WGRAD = 0, 1

STATUS_NAMES = {0: "MX_OK", 1: "MX_EINVAL", 2: "MX_ECUDA", 3: "MX_ETIMEOUT", 4: "MX_EUNSUPPORTED", 5: "MX_EDATA"}

P = ctypes.c_void_p
I64 = ctypes.c_int64
U64 = ctypes.c_uint64
I32 = ctypes.c_int
SZ = ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/mxmoe.h
SIGNATURES = {
    "mx_version": (I32, []),
    "mx_last_cuda_error": (I32, []),
    "mx_kernel_launches": (ctypes.c_ulonglong, []),
    "mx_sync_status": (I32, [P]),
    "mx_wait_selftest": (I32, [I64, P]),
    "mx_sf_bytes": (SZ, [I64, I64, I32, I32]),
    "mx_debug_bounds_build": (I32, []),
    "mx_debug_bounds_violations": (ctypes.c_ulonglong, [I32]),
    "nvfp4_quantize": (I32, [P, I64, I64, I64, P, P, P, I32, P]),
    "mxfp8_requant_transpose_sr": (I32, [P, P, P, I64, I64, I64, I32, P, U64, U64, I32, P, P, I32, P]),
    "mxfp8_quantize": (I32, [P, I64, I64, I32, U64, U64, I32, P, P, P, P, P, I32, P]),
    "grouped_gemm_nvfp4": (I32, [P, P, P, P, P, P, P, I64, I64, I64, I64, P, I32, P]),
    "grouped_gemm_mxfp8": (I32, [I32, P, P, P, P, P, I64, I64, I64, I64, P, I32, P]),
    "mx_route_workspace_bytes": (SZ, [I64, I64]),
    "moe_route": (I32, [P, I64, I64, I64, I64, P, P, P, P, SZ, P]),
    "moe_route_static": (I32, [P, I64, I64, I64, I64, P, P, P, P]),
    "moe_route_aligned": (I32, [P, I64, I64, I64, I64, I64, P, P, P, P, SZ, P]),
    "nvfp4_gather_rows": (I32, [P, P, P, P, I64, I64, I64, P, P, P, P]),
    "moe_permute_row_groups": (I32, [P, I64, P, I64, I64, P, P]),
    "swiglu_fwd": (I32, [P, I64, I64, I32, P, P, P]),
    "swiglu_bwd": (I32, [P, P, I64, I64, I32, P, P, P]),
    "swiglu_nvfp4_quantize": (I32, [P, I64, I64, I32, P, P, P, P, I32, P]),
    "moe_combine": (I32, [P, P, P, I64, I64, I64, P, P]),
    "moe_dispatch_grad": (I32, [P, P, P, P, I64, I64, I64, I64, P, P]),
    "moe_dispatch_grad_mxfp8_quantize": (I32, [P, P, P, I64, I64, I64, I64, P, P, P, P, P, I32, P]),
    "hadamard_s2f6_quantize": (I32, [P, I64, I64, U64, U64, P, P, P]),
    "grouped_gemm_nvfp4_s2f6": (I32, [P, P, P, P, P, P, P, I64, I64, I64, I64, U64, U64, P, P, P]),
    "moe_combine_s2f6": (I32, [P, P, P, P, I64, I64, I64, U64, U64, P, P]),
    "nvfp4_quantize_sr": (I32, [P, I64, I64, I64, I32, U64, U64, I32, P, P, P, I32, P]),
    "nvfp4_requant_transpose_sr": (I32, [P, P, P, I64, I64, I64, I32, I64, I32, I32, U64, U64, I32, P, P, P, I32,
                                         P]),
    "nvfp4_quantize_tile16": (I32, [P, I64, I64, I64, P, P, P, P]),
    "nvfp4_quantize_transpose_segments": (I32, [P, I64, I64, P, I64, I32, I32, U64, U64, I32, P, P, P, I32, P]),
    "nvfp4_requant_transpose_segments": (I32, [P, P, P, I32, I64, I64, I64, P, I64, I32, I32, U64, U64, I32, P, P,
                                               P, I32, P]),
    "grouped_gemm_nvfp4_wgrad": (I32, [P, P, P, P, P, P, P, I64, I64, I64, I64, P, I32, P]),
}

_lib = None


class MxError(RuntimeError):
    def __init__(self, fn: str, status: int, cuda_err: int = 0):
        msg = f"{fn} returned {STATUS_NAMES.get(status, status)}"
        if status == MX_ECUDA:
            msg += f" (cudaError {cuda_err})"
        super().__init__(msg)
        self.status = status


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m fp8_moe_numerics_b200.build`"
                               f"{' --debug-bounds' if LIB_PATH.endswith('_debug.so') else ''} "
                               "(there is no non-CUDA implementation of this library)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def call(name: str, *args) -> None:
    st = getattr(lib(), name)(*args)
    if st != MX_OK:
        raise MxError(name, st, lib().mx_last_cuda_error() if st == MX_ECUDA else 0)
