"""CPU oracle for the NVFP4-forward / MXFP8-backward expert-layer numerics.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  It shares no code with ``fp8_moe_numerics_b200`` and imports nothing
from it; the CUDA path never imports this package.

The element-level arithmetic lives in ``oracle.c`` (plain scalar C, built with
``-ffp-contract=off`` and no fast-math, OpenMP over rows only) and is loaded
here with ctypes.  The fp64 GEMM references and the glue steps (routing
permutation, SwiGLU, combine) are plain numpy.

Sources are the web pages on Thinking Machines' "End-to-End 4-Bit Training":
"Inkling 2 Small uses four-bit training, Thinking Machines reports 8% and 20%
savings" (ai-primer.com; sections "NVFP4 forward, MXFP8 backward", "Block scales
and per-token activations", "Stochastic rounding across transposes", "Quantized
NVLink and BBBK") and the Hermes page "Thinking Machines' Inkling 2 Small Trains
a 594B Model in 68 Hours" (section "594B weights, 17B at work": 8 of 384
experts per token).

Parity pins (tests/test_oracle_*.py):
  codecs ............ exhaustive decode tables; encode vs ml_dtypes; toy grid
  philox ............ vs Triton's independent Philox4x32-10 (CPU interpreter)
  stochastic round .. worked example 4.5 -> 4 (p=.75) / 6 (p=.25) by
                      enumeration; exact mean; bias bound
  nvfp4_quantize .... closed forms, 4.5 bits/value, element rounding vs
                      ml_dtypes, row independence, error bound
  e8m0 exponent ..... brute-force definition
  requant / mxfp8 ... 8.25 bits/value, on-grid identity, unbiasedness over
                      streams, transpose/regroup effect
  GEMMs ............. brute-force loops on tiny inputs; plain matmul special
                      cases; empty experts
  glue .............. brute-force permutation; SiLU vs torch; combine loops
  nvfp4 backward .... equal to the forward quantiser without SR; grid
                      neighbours and the 4.5 example with SR; the regrouping
                      example across the transpose; unbiasedness over
                      streams; brute-force dgrad/wgrad; the 16x16 tile's
                      outlier statement and orientation invariance
  hadamard / s2f6 ... butterflies vs the Kronecker-built Sylvester matrix on
                      integer vectors; H32 H32 = 32 I; exponent by search
                      over all exponents; ties to even; one-hot outlier
                      closed form; reconstruction error bound; combine loops
No oracle function is "parity unpinned".  tests/test_oracle_mutants.py plants
plausible mistakes in a copy of this package and checks that a pin fails on
each.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile oracle.c into oracle/liboracle.so (gcc)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


P = ctypes.c_void_p
I64 = ctypes.c_int64
U64 = ctypes.c_uint64
I32 = ctypes.c_int


def _declare(L: ctypes.CDLL) -> None:
    sig = {
        "orc_f32_to_bf16": (ctypes.c_uint16, [ctypes.c_float]),
        "orc_e2m1_decode": (ctypes.c_float, [ctypes.c_uint8]),
        "orc_e4m3_decode": (ctypes.c_float, [ctypes.c_uint8]),
        "orc_e8m0_decode": (ctypes.c_double, [ctypes.c_uint8]),
        "orc_e2m1_encode": (ctypes.c_uint8, [ctypes.c_float]),
        "orc_e4m3_encode": (ctypes.c_uint8, [ctypes.c_float]),
        "orc_e2m1_encode_array": (None, [P, I64, P]),
        "orc_e4m3_encode_array": (None, [P, I64, P]),
        "orc_round_nearest_on_grid": (ctypes.c_double, [ctypes.c_double, P, I32]),
        "orc_philox4x32_10": (None, [P, P, P]),
        "orc_sr_bits": (ctypes.c_uint32, [U64, U64, I32, U64]),
        "orc_sr_value": (ctypes.c_double, [ctypes.c_double, ctypes.c_uint32, I32, I32, I32]),
        "orc_e4m3_sr": (ctypes.c_uint8, [ctypes.c_double, ctypes.c_uint32, I32]),
        "orc_e2m1_sr": (ctypes.c_uint8, [ctypes.c_double, ctypes.c_uint32, I32]),
        "orc_nvfp4_quantize": (None, [P, I64, I64, I64, P, P, P]),
        "orc_nvfp4_dequantize": (None, [P, P, P, I64, I64, I64, P]),
        "orc_nvfp4_block_values": (None, [P, P, I64, I64, P]),
        "orc_e8m0_exponent": (I32, [ctypes.c_double]),
        "orc_mxfp8_requant_transpose_sr": (None, [P, P, P, I64, I64, I64, U64, U64, I32, P, P]),
        "orc_mxfp8_quantize_rows": (None, [P, I64, I64, I32, U64, U64, I32, P, P]),
        "orc_mxfp8_quantize_cols": (None, [P, I64, I64, I32, U64, U64, I32, P, P]),
        "orc_mxfp8_dequantize": (None, [P, P, I64, I64, P]),
        "orc_nvfp4_quantize_f32": (None, [P, I64, I64, I64, I32, U64, U64, I32, P, P, P]),
        "orc_nvfp4_quantize_tile16": (None, [P, I64, I64, I64, P, P, P]),
        "orc_nvfp4_quantize_f32_block_outer": (None, [P, I64, I64, P, I32, U64, U64, I32, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


# --------------------------------------------------------------------------
# bf16 helpers (numpy has no bf16: bf16 tensors are uint16 bit patterns)
# --------------------------------------------------------------------------

def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 bit patterns (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 with a single rounding: round to 8 significant bits, RNE."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                          # x = m * 2^e, |m| in [0.5,1)
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)  # np.rint is round-half-even
    return f32_to_bf16(r.astype(np.float32))    # r has <= 8 significant bits: exact


# --------------------------------------------------------------------------
# Codecs
# --------------------------------------------------------------------------

def e2m1_decode_table() -> np.ndarray:
    return np.array([lib().orc_e2m1_decode(c) for c in range(16)], dtype=np.float32)


def e4m3_decode_table() -> np.ndarray:
    return np.array([lib().orc_e4m3_decode(c) for c in range(256)], dtype=np.float32)


def e8m0_decode_table() -> np.ndarray:
    return np.array([lib().orc_e8m0_decode(c) for c in range(256)], dtype=np.float64)


def e2m1_encode(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().orc_e2m1_encode_array(_p(x), x.size, _p(out))
    return out


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().orc_e4m3_encode_array(_p(x), x.size, _p(out))
    return out


def round_nearest_on_grid(x: float, grid) -> float:
    g = np.ascontiguousarray(grid, dtype=np.float64)
    return lib().orc_round_nearest_on_grid(float(x), _p(g), len(g))


# --------------------------------------------------------------------------
# Random bits and stochastic rounding
# --------------------------------------------------------------------------

def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().orc_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def sr_bits(seed: int, stream: int, R: int, L: int) -> int:
    return int(lib().orc_sr_bits(seed, stream, R, L))


def sr_value(y: float, u: int, R: int, mbits: int, qmin: int) -> float:
    return lib().orc_sr_value(float(y), u, R, mbits, qmin)


def e4m3_sr(y: float, u: int, R: int) -> int:
    return int(lib().orc_e4m3_sr(float(y), u, R))


def e2m1_sr(y: float, u: int, R: int) -> int:
    return int(lib().orc_e2m1_sr(float(y), u, R))


def e8m0_exponent(amax: float) -> int:
    return int(lib().orc_e8m0_exponent(float(amax)))


# --------------------------------------------------------------------------
# NVFP4
# --------------------------------------------------------------------------

def nvfp4_quantize(x_bf16: np.ndarray, group_rows: int = 1):
    """x_bf16 [rows, cols] uint16 -> (codes [rows, cols/2] u8, sf [rows, cols/16]
    u8 row-major E4M3, outer [rows/group_rows] f32)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    assert cols % 16 == 0 and rows % group_rows == 0
    codes = np.empty((rows, cols // 2), dtype=np.uint8)
    sf = np.empty((rows, cols // 16), dtype=np.uint8)
    outer = np.empty(rows // group_rows, dtype=np.float32)
    lib().orc_nvfp4_quantize(_p(x), rows, cols, group_rows, _p(codes), _p(sf), _p(outer))
    return codes, sf, outer


def nvfp4_dequantize(codes, sf, outer, group_rows: int = 1) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    outer = np.ascontiguousarray(outer, dtype=np.float32)
    rows, cols = codes.shape[0], codes.shape[1] * 2
    out = np.empty((rows, cols), dtype=np.float32)
    lib().orc_nvfp4_dequantize(_p(codes), _p(sf), _p(outer), rows, cols, group_rows, _p(out))
    return out


def nvfp4_block_values(codes, sf) -> np.ndarray:
    """q * sf in fp64 (exact), without the outer scale."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows, cols = codes.shape[0], codes.shape[1] * 2
    out = np.empty((rows, cols), dtype=np.float64)
    lib().orc_nvfp4_block_values(_p(codes), _p(sf), rows, cols, _p(out))
    return out


# --------------------------------------------------------------------------
# MXFP8
# --------------------------------------------------------------------------

def mxfp8_requant_transpose_sr(codes, sf, outer, group_rows: int, seed: int, stream: int, R: int = 8):
    """Saved NVFP4 [rows, cols] -> MXFP8 transpose: codes [cols, rows] u8 (E4M3),
    E8M0 scales [cols, rows/32] u8."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    outer = np.ascontiguousarray(outer, dtype=np.float32)
    rows, cols = codes.shape[0], codes.shape[1] * 2
    assert rows % 32 == 0 and R in (8, 16, 32)
    oc = np.empty((cols, rows), dtype=np.uint8)
    oe = np.empty((cols, rows // 32), dtype=np.uint8)
    lib().orc_mxfp8_requant_transpose_sr(_p(codes), _p(sf), _p(outer), rows, cols, group_rows,
                                         seed, stream, R, _p(oc), _p(oe))
    return oc, oe


def mxfp8_requant_entry(codes32, sf32, outer32, col: int, t: int, rows: int, row0: int, seed: int, stream: int,
                        R: int):
    """One entry of mxfp8_requant_transpose_sr, computed alone: output [col, row0 + t]
    of a call on a tensor with `rows` rows, from the 32 input rows row0..row0+31
    (codes32 [32, cols/2], row-major sf32 [32, cols/16], per-row outer32 [32]).
    Returns (E4M3 code, E8M0 byte) following the same steps as the full call:
    dequantise, block amax, E8M0 exponent, exact scaling, SR with the bits of
    linear index col * rows + row0 + t."""
    xh = nvfp4_dequantize(codes32, sf32, outer32, 1)[:, col].astype(np.float64)
    e = e8m0_exponent(float(np.max(np.abs(xh))))
    y = float(np.ldexp(xh[t], -e))
    L = col * rows + row0 + t
    return e4m3_sr(y, sr_bits(seed, stream, R, L), R), e + 127


def mxfp8_quantize_rows(x_bf16, sr: bool = False, seed: int = 0, stream: int = 0, R: int = 8):
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    assert cols % 32 == 0
    codes = np.empty((rows, cols), dtype=np.uint8)
    e8 = np.empty((rows, cols // 32), dtype=np.uint8)
    lib().orc_mxfp8_quantize_rows(_p(x), rows, cols, int(sr), seed, stream, R, _p(codes), _p(e8))
    return codes, e8


def mxfp8_quantize_cols(x_bf16, sr: bool = False, seed: int = 0, stream: int = 0, R: int = 8):
    """Column-wise MXFP8 stored transposed: codes [cols, rows], E8M0 [cols, rows/32]."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    assert rows % 32 == 0
    codes = np.empty((cols, rows), dtype=np.uint8)
    e8 = np.empty((cols, rows // 32), dtype=np.uint8)
    lib().orc_mxfp8_quantize_cols(_p(x), rows, cols, int(sr), seed, stream, R, _p(codes), _p(e8))
    return codes, e8


def mxfp8_dequantize(codes, e8m0) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    e8m0 = np.ascontiguousarray(e8m0, dtype=np.uint8)
    rows, cols = codes.shape
    out = np.empty((rows, cols), dtype=np.float64)
    lib().orc_mxfp8_dequantize(_p(codes), _p(e8m0), rows, cols, _p(out))
    return out


# --------------------------------------------------------------------------
# Grouped GEMMs, fp64 over the dequantised operands
# [ai-primer §NVFP4 forward, MXFP8 backward]: forward expert matmuls in NVFP4,
# gradients with MXFP8 matmuls.  The reference sums the exact block products
# q*sf in fp64 and applies the fp32 outer scales after the sum.
# --------------------------------------------------------------------------

def grouped_gemm_nvfp4(a_codes, a_sf, a_outer, b_codes, b_sf, b_outer, seg, N: int) -> np.ndarray:
    """A [M, K] NVFP4 (per-row outer), B [E*N, K] NVFP4 (per-expert outer),
    seg [E+1] row offsets of A.  Returns C [M, N] fp64, rows of expert e =
    A_e @ B_e^T * a_outer[row] * b_outer[e]; rows outside all segments are 0."""
    M = a_codes.shape[0]
    E = len(seg) - 1
    C = np.zeros((M, N), dtype=np.float64)
    for e in range(E):
        r0, r1 = int(seg[e]), int(seg[e + 1])
        if r1 <= r0:
            continue
        Av = nvfp4_block_values(a_codes[r0:r1], a_sf[r0:r1])
        Bv = nvfp4_block_values(b_codes[e * N:(e + 1) * N], b_sf[e * N:(e + 1) * N])
        C[r0:r1] = (Av @ Bv.T) * a_outer[r0:r1, None].astype(np.float64) * float(b_outer[e])
    return C


def grouped_gemm_nvfp4_sampled(a_codes, a_sf, a_outer, b_codes, b_sf, b_outer, seg, N: int,
                               rows, cols) -> np.ndarray:
    """Entries C[rows[i], cols[i]] of grouped_gemm_nvfp4, computed one by one."""
    seg = np.asarray(seg)
    out = np.empty(len(rows), dtype=np.float64)
    for i, (r, n) in enumerate(zip(rows, cols)):
        e = int(np.searchsorted(seg, r, side="right") - 1)
        if e < 0 or e >= len(seg) - 1 or r >= seg[e + 1]:
            out[i] = 0.0
            continue
        a = nvfp4_block_values(a_codes[r:r + 1], a_sf[r:r + 1])[0]
        b = nvfp4_block_values(b_codes[e * N + n:e * N + n + 1], b_sf[e * N + n:e * N + n + 1])[0]
        out[i] = float(np.dot(a, b)) * float(a_outer[r]) * float(b_outer[e])
    return out


def grouped_gemm_mxfp8_dgrad(a_codes, a_e8, b_codes, b_e8, seg) -> np.ndarray:
    """DGRAD: A [M, Kc] MXFP8 (blocks along Kc), B [Nout, E*Kc] MXFP8 (blocks
    along its rows' length; expert e = columns [e*Kc, (e+1)*Kc)).
    C [M, Nout]: rows of expert e = A_e @ B_e^T."""
    M, Kc = a_codes.shape
    Nout = b_codes.shape[0]
    E = len(seg) - 1
    C = np.zeros((M, Nout), dtype=np.float64)
    for e in range(E):
        r0, r1 = int(seg[e]), int(seg[e + 1])
        if r1 <= r0:
            continue
        Av = mxfp8_dequantize(a_codes[r0:r1], a_e8[r0:r1])
        Bv = mxfp8_dequantize(np.ascontiguousarray(b_codes[:, e * Kc:(e + 1) * Kc]),
                              np.ascontiguousarray(b_e8[:, e * Kc // 32:(e + 1) * Kc // 32]))
        C[r0:r1] = Av @ Bv.T
    return C


def grouped_gemm_mxfp8_wgrad(a_codes, a_e8, b_codes, b_e8, seg) -> np.ndarray:
    """WGRAD: A [Nw, M] and B [Kw, M] MXFP8 (blocks along M, the tokens);
    C [E, Nw, Kw], C[e] = A[:, seg e] @ B[:, seg e]^T; empty experts give 0."""
    Nw = a_codes.shape[0]
    Kw = b_codes.shape[0]
    E = len(seg) - 1
    C = np.zeros((E, Nw, Kw), dtype=np.float64)
    for e in range(E):
        t0, t1 = int(seg[e]), int(seg[e + 1])
        if t1 <= t0:
            continue
        Av = mxfp8_dequantize(np.ascontiguousarray(a_codes[:, t0:t1]), np.ascontiguousarray(a_e8[:, t0 // 32:t1 // 32]))
        Bv = mxfp8_dequantize(np.ascontiguousarray(b_codes[:, t0:t1]), np.ascontiguousarray(b_e8[:, t0 // 32:t1 // 32]))
        C[e] = Av @ Bv.T
    return C


# --------------------------------------------------------------------------
# NVFP4 in the backward pass (the pages' stated future work) and the rejected
# 16x16 shared-scale alternative.  [ai-primer §NVFP4 forward, MXFP8 backward]:
# the lab is exploring four-bit arithmetic in the backward pass; [ai-primer
# §Stochastic rounding across transposes]: a scale shared by each 16x16 tile
# proved too sensitive to outliers.  Readings taken (pages silent):
#   quantiser   the NVFP4 scale rules of the forward quantiser on fp32 input,
#               element codes rounded stochastically (E2M1, random integer of
#               the linear output index), see orc_nvfp4_quantize_f32;
#   requant     dequantise ((q sf) s in fp32), transpose, re-quantise to NVFP4
#               with SR; the transposed tensor takes one outer scale per row
#               (per feature) for activations and gradients, one per expert
#               for an expert weight stack, so that in every backward GEMM
#               both outer scales factor out of the contraction;
#   dgrad       dX = dY W_e per expert is the forward grouped GEMM with B the
#               stack of W_e^T [E*K, N] (grouped_gemm_nvfp4);
#   wgrad       dW_e = dY_e^T X_e with both operands NVFP4 along the tokens,
#               outer scales per expert segment of the tokens: per (segment,
#               row) for dY^T, per segment for X^T, so that the GEMM applies a
#               per-row times a per-expert factor as in the forward
#               (nvfp4_quantize_transpose_segments, grouped_gemm_nvfp4_wgrad);
#   tile16      one E4M3 scale per 16x16 tile, one outer scale per group of
#               rows (a multiple of 16), codes to nearest even.
# --------------------------------------------------------------------------

def nvfp4_quantize_f32(x_f32: np.ndarray, group_rows: int = 1, sr: bool = False, seed: int = 0, stream: int = 0,
                       R: int = 8):
    """fp32 [rows, cols] -> NVFP4 (codes [rows, cols/2], sf [rows, cols/16] row-major, outer
    [rows/group_rows]); element codes stochastically rounded when sr."""
    x = np.ascontiguousarray(x_f32, dtype=np.float32)
    rows, cols = x.shape
    assert cols % 16 == 0 and rows % group_rows == 0 and R in (8, 16, 32)
    codes = np.empty((rows, cols // 2), dtype=np.uint8)
    sf = np.empty((rows, cols // 16), dtype=np.uint8)
    outer = np.empty(rows // group_rows, dtype=np.float32)
    lib().orc_nvfp4_quantize_f32(_p(x), rows, cols, group_rows, int(sr), seed, stream, R, _p(codes), _p(sf),
                                 _p(outer))
    return codes, sf, outer


def nvfp4_requant_transpose_sr(codes, sf, outer, group_rows: int, seed: int, stream: int, R: int = 8,
                               sr: bool = True):
    """Saved NVFP4 [rows, cols] (outer per group_rows rows) -> NVFP4 of its transpose
    [cols, rows], one outer scale per output row, blocks of 16 along the old rows."""
    xh = nvfp4_dequantize(codes, sf, outer, group_rows)
    return nvfp4_quantize_f32(np.ascontiguousarray(xh.T), 1, sr, seed, stream, R)


def nvfp4_requant_transpose_experts_sr(codes, sf, outer, E: int, seed: int, stream: int, R: int = 8,
                                       sr: bool = True):
    """Saved expert weight stack [E*N, K] (outer per expert) -> NVFP4 stack of the
    per-expert transposes W_e^T, [E*K, N], outer per expert; the B operand of
    the NVFP4 dgrad (grouped_gemm_nvfp4 with output width K)."""
    rows, K = codes.shape[0], codes.shape[1] * 2
    N = rows // E
    xh = nvfp4_dequantize(codes, sf, outer, N).reshape(E, N, K)
    return nvfp4_quantize_f32(np.ascontiguousarray(xh.transpose(0, 2, 1).reshape(E * K, N)), K, sr, seed, stream, R)


def nvfp4_quantize_transpose_segments(x_f32: np.ndarray, seg, per_row: bool, sr: bool = True, seed: int = 0,
                                      stream: int = 0, R: int = 8):
    """x fp32 [M, C] -> NVFP4 of its transpose [C, M] (blocks of 16 along M, the
    tokens) with outer scales per expert segment of M (seg [E+1], starts at
    multiples of 16): one per (segment, row), outer [E, C], when per_row; one
    per segment, outer [E], otherwise.  Each scale is the segment's amax / 2688
    (fp32); columns past seg[E] (padding rows of the expert-major layout)
    quantise to zero.  The wgrad operands: dY^T per (segment, row), X^T per
    segment, so that the GEMM's outer factors are a per-row and a per-expert
    value, as in the forward GEMM."""
    x = np.ascontiguousarray(x_f32, dtype=np.float32)
    M, C = x.shape
    seg = np.asarray(seg, dtype=np.int64)
    E = len(seg) - 1
    assert M % 16 == 0 and np.all(seg % 16 == 0) and seg[-1] <= M and R in (8, 16, 32)
    xt = np.ascontiguousarray(x.T)
    s_blk = np.zeros((C, M // 16), dtype=np.float32)
    outer = np.zeros((E, C) if per_row else E, dtype=np.float32)
    for e in range(E):
        t0, t1 = int(seg[e]), int(seg[e + 1])
        if t1 <= t0:
            continue
        amax = np.abs(xt[:, t0:t1]).max(axis=1) if per_row else np.abs(xt[:, t0:t1]).max()
        s = np.asarray(amax, dtype=np.float32) / np.float32(2688.0)              # one fp32 division
        outer[e] = s
        s_blk[:, t0 // 16:t1 // 16] = s[:, None] if per_row else s
    codes = np.empty((C, M // 2), dtype=np.uint8)
    sf = np.empty((C, M // 16), dtype=np.uint8)
    lib().orc_nvfp4_quantize_f32_block_outer(_p(xt), C, M, _p(s_blk), int(sr), seed, stream, R, _p(codes), _p(sf))
    return codes, sf, outer


def grouped_gemm_nvfp4_wgrad(a_codes, a_sf, a_outer, b_codes, b_sf, b_outer, seg) -> np.ndarray:
    """WGRAD in NVFP4: A [Nw, M] and B [Kw, M] (blocks of 16 along M, the tokens)
    with outer scales per expert segment: a_outer [E, Nw], b_outer [E] (or
    [E, Kw]).  C [E, Nw, Kw] fp64:
    C[e, n, k] = a_outer[e, n] b_outer[e(, k)] sum_{t in segment e} (qa sfa)[n, t] (qb sfb)[k, t];
    empty experts give 0."""
    Nw, Kw = a_codes.shape[0], b_codes.shape[0]
    E = len(seg) - 1
    Av = nvfp4_block_values(a_codes, a_sf)
    Bv = nvfp4_block_values(b_codes, b_sf)
    ao = np.asarray(a_outer, np.float64).reshape(E, Nw)
    bo = np.asarray(b_outer, np.float64)
    bo = bo.reshape(E, 1) if bo.ndim == 1 else bo.reshape(E, Kw)
    C = np.zeros((E, Nw, Kw), dtype=np.float64)
    for e in range(E):
        t0, t1 = int(seg[e]), int(seg[e + 1])
        if t1 > t0:
            C[e] = (Av[:, t0:t1] @ Bv[:, t0:t1].T) * ao[e][:, None] * bo[e][None, :]
    return C


def nvfp4_quantize_tile16(x_f32: np.ndarray, group_rows: int = 16):
    """fp32 [rows, cols] -> (codes [rows, cols/2], sf_tile [rows/16, cols/16], outer
    [rows/group_rows]) with one E4M3 scale per 16x16 tile."""
    x = np.ascontiguousarray(x_f32, dtype=np.float32)
    rows, cols = x.shape
    assert rows % 16 == 0 and cols % 16 == 0 and group_rows % 16 == 0 and rows % group_rows == 0
    codes = np.empty((rows, cols // 2), dtype=np.uint8)
    sf = np.empty((rows // 16, cols // 16), dtype=np.uint8)
    outer = np.empty(rows // group_rows, dtype=np.float32)
    lib().orc_nvfp4_quantize_tile16(_p(x), rows, cols, group_rows, _p(codes), _p(sf), _p(outer))
    return codes, sf, outer


def nvfp4_tile16_dequantize(codes, sf_tile, outer, group_rows: int = 16) -> np.ndarray:
    """fp32 (q sf_tile) s of each element (one rounding, as nvfp4_dequantize)."""
    sf_rows = np.repeat(np.asarray(sf_tile, np.uint8), 16, axis=0)           # each 1x16 block's tile scale
    outer_rows = np.repeat(np.asarray(outer, np.float32), group_rows)         # each row's outer scale
    return nvfp4_dequantize(codes, np.ascontiguousarray(sf_rows), outer_rows, 1)


def nvfp4_tile16_transpose(codes, sf_tile):
    """The same tile-scaled tensor in the other orientation: element codes moved
    to [cols, rows] (two per byte, element 2j in the low nibble), tile scales
    transposed.  No value changes."""
    q = np.stack([codes & 15, codes >> 4], axis=-1).reshape(codes.shape[0], -1).T
    q = np.ascontiguousarray(q)
    return (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8), np.ascontiguousarray(np.asarray(sf_tile).T)


# --------------------------------------------------------------------------
# Glue: routing permutation, SiLU / SwiGLU, combine
# Readings taken (pages silent): tokens are dispatched once in NVFP4 and
# gathered into expert-major order ([ai-primer §Quantized NVLink and BBBK]:
# tokens travel to their experts in NVFP4); each expert's rows are a segment
# padded with zero rows to a multiple of 128; inside a segment rows are in
# token order; SwiGLU gate = first F columns of W1's output, up = last F.
# --------------------------------------------------------------------------

def route(topk_ids: np.ndarray, E: int, align: int = 128):
    """topk_ids [T, k] (distinct per token) -> (seg [E+1] int64, src_token [M]
    int32 with -1 on padding rows, pos [T, k] int32 row of each (t, j))."""
    T, k = topk_ids.shape
    counts = np.bincount(topk_ids.reshape(-1), minlength=E)[:E]
    padded = (counts + align - 1) // align * align
    seg = np.zeros(E + 1, dtype=np.int64)
    seg[1:] = np.cumsum(padded)
    src = np.full(int(seg[-1]), -1, dtype=np.int32)
    pos = np.empty((T, k), dtype=np.int32)
    fill = seg[:-1].copy()
    for t in range(T):                          # token order inside each expert
        for j in range(k):
            e = int(topk_ids[t, j])
            pos[t, j] = fill[e]
            src[fill[e]] = t
            fill[e] += 1
    return seg, src, pos


def gather_nvfp4_rows(codes, sf, outer, src):
    """Rows of a per-row NVFP4 tensor in src order; src == -1 gives a zero row
    (codes 0, scales 0, outer 0)."""
    M = len(src)
    oc = np.zeros((M, codes.shape[1]), dtype=np.uint8)
    osf = np.zeros((M, sf.shape[1]), dtype=np.uint8)
    oo = np.zeros(M, dtype=np.float32)
    ok = src >= 0
    oc[ok] = codes[src[ok]]
    osf[ok] = sf[src[ok]]
    oo[ok] = outer[src[ok]]
    return oc, osf, oo


def _silu(g):
    return g / (1.0 + np.exp(-g))


def _dsilu(g):
    s = 1.0 / (1.0 + np.exp(-g))
    return s * (1.0 + g * (1.0 - s))


def swiglu_fwd(h_bf16: np.ndarray, gated: bool = True) -> np.ndarray:
    """gated: a = silu(g) * u with g, u the two halves of h; else a = silu(h).
    fp64, one rounding to bf16."""
    h = bf16_to_f32(h_bf16).astype(np.float64)
    if gated:
        F = h.shape[1] // 2
        a = _silu(h[:, :F]) * h[:, F:]
    else:
        a = _silu(h)
    return f64_to_bf16(a)


def swiglu_bwd(h_bf16: np.ndarray, da_bf16: np.ndarray, gated: bool = True) -> np.ndarray:
    h = bf16_to_f32(h_bf16).astype(np.float64)
    da = bf16_to_f32(da_bf16).astype(np.float64)
    if gated:
        F = h.shape[1] // 2
        g, u = h[:, :F], h[:, F:]
        dh = np.concatenate([da * u * _dsilu(g), da * _silu(g)], axis=1)
    else:
        dh = da * _dsilu(h)
    return f64_to_bf16(dh)


def combine(y_bf16: np.ndarray, pos: np.ndarray, w: np.ndarray) -> np.ndarray:
    """out[t] = sum_j w[t, j] * y[pos[t, j]]  (fp64, one rounding to bf16)."""
    y = bf16_to_f32(y_bf16).astype(np.float64)
    out = np.einsum("tj,tjd->td", w.astype(np.float64), y[pos])
    return f64_to_bf16(out)


def dispatch_grad(dout_bf16: np.ndarray, pos: np.ndarray, w: np.ndarray, M: int) -> np.ndarray:
    """Gradient of combine w.r.t. y: dy[pos[t, j]] = w[t, j] * dout[t]; padding 0."""
    d = bf16_to_f32(dout_bf16).astype(np.float64)
    T, k = pos.shape
    dy = np.zeros((M, d.shape[1]), dtype=np.float64)
    for j in range(k):
        dy[pos[:, j]] = w[:, j, None].astype(np.float64) * d
    return f64_to_bf16(dy)


# --------------------------------------------------------------------------
# Combine path: 32-d random Hadamard rotation + block-scaled S2F6
# [ai-primer §Quantized NVLink and BBBK]: expert outputs are rotated by a
# 32-dimensional random Hadamard transform and quantised to S2F6 (eight-bit
# fixed point: two signed integer bits, six fractional bits) with a block
# scale before the combine.  Readings taken where the pages are silent:
#   rotation  z = H32 (sigma_j * x) per 32-column block j of a row, H32 the
#             unnormalised Sylvester matrix, H[a][b] = (-1)^popcount(a & b);
#             sigma_j in {+1,-1}^32: coordinate i flipped iff bit i of word 0
#             of Philox4x32-10(counter (j, stream), key seed) is set.  Inverse
#             x = sigma_j * (H32 z) / 32 (H32 H32 = 32 I), so both directions
#             scale by powers of two only.
#   order     z is the fp32 result of the five butterfly stages h = 1, 2, 4,
#             8, 16: (a, b) -> (a + b, a - b) for every pair (i, i + h) with
#             i & h == 0, each an fp32 round-to-nearest add.
#   scale     one E8M0 exponent per 32-value block: e = smallest integer with
#             amax|z| <= (127/64) 2^e, clamped to [-127, 127] (-127 for a zero
#             block); code c = RNE(z 2^(6-e)) clamped to [-127, 127] (int8);
#             value c 2^(e-6).  -128 is never produced (symmetric range).
# --------------------------------------------------------------------------
S2F6_MAX = 127.0 / 64.0


def hadamard_sign_words(seed: int, stream: int, nblocks: int) -> np.ndarray:
    """Sign mask of each 32-column block j < nblocks (bit i set: coordinate i
    is negated before the transform)."""
    key = [seed & 0xFFFFFFFF, seed >> 32]
    out = np.empty(nblocks, dtype=np.uint32)
    for j in range(nblocks):
        out[j] = philox4x32_10([j & 0xFFFFFFFF, j >> 32, stream & 0xFFFFFFFF, stream >> 32], key)[0]
    return out


def hadamard_signs(seed: int, stream: int, cols: int) -> np.ndarray:
    """+1/-1 per column (float64), from hadamard_sign_words."""
    words = hadamard_sign_words(seed, stream, cols // 32)
    bits = (words[:, None] >> np.arange(32, dtype=np.uint32)[None, :]) & 1
    return np.where(bits.reshape(-1) == 1, -1.0, 1.0)


def fwht32_f32(y: np.ndarray) -> np.ndarray:
    """Unnormalised Walsh-Hadamard transform of the last axis (length 32) in
    fp32, stage by stage as stated above."""
    z = np.array(y, dtype=np.float32, copy=True)
    lead = z.shape[:-1]
    h = 1
    while h < 32:
        z = z.reshape(lead + (32 // (2 * h), 2, h))
        a, b = z[..., 0, :], z[..., 1, :]
        z = np.stack([a + b, a - b], axis=-2).reshape(lead + (32,))
        h *= 2
    return z


def s2f6_exponent(amax: float) -> int:
    """Smallest integer e with amax <= (127/64) 2^e, clamped to [-127, 127]."""
    if amax == 0.0:
        return -127
    m, E = math.frexp(float(amax))              # amax = m 2^E, m in [0.5, 1)
    m2, E1 = 2.0 * m, E - 1                     # amax = m2 2^E1, m2 in [1, 2)
    e = E1 if m2 <= S2F6_MAX else E1 + 1
    return max(-127, min(127, e))


def s2f6_quantize_hadamard(x_f32: np.ndarray, seed: int, stream: int):
    """x fp32 [rows, cols] (cols % 32 == 0) -> (codes int8 [rows, cols],
    e8m0 uint8 [rows, cols/32], biased by 127)."""
    x = np.ascontiguousarray(x_f32, dtype=np.float32)
    rows, cols = x.shape
    sig = hadamard_signs(seed, stream, cols).astype(np.float32)
    z = fwht32_f32((x * sig[None, :]).reshape(rows, cols // 32, 32))       # sign flips are exact
    amax = np.abs(z).max(axis=-1).astype(np.float64)
    e = np.array([s2f6_exponent(a) for a in amax.reshape(-1)], dtype=np.int64).reshape(amax.shape)
    y = z.astype(np.float64) * np.ldexp(1.0, 6 - e)[..., None]             # exact: power-of-two scaling
    c = np.clip(np.rint(y), -127, 127).astype(np.int8)                     # np.rint: round half to even
    return c.reshape(rows, cols), (e + 127).astype(np.uint8)


def s2f6_dequantize_hadamard(codes: np.ndarray, e8m0: np.ndarray, seed: int, stream: int) -> np.ndarray:
    """Inverse of s2f6_quantize_hadamard up to the quantisation: fp64 [rows, cols]."""
    rows, cols = codes.shape
    zhat = codes.astype(np.float64).reshape(rows, cols // 32, 32) * np.ldexp(1.0, e8m0.astype(np.int64) - 127 - 6)[..., None]
    H = sylvester_hadamard(32)
    x = (zhat @ H.T).reshape(rows, cols) / 32.0
    return x * hadamard_signs(seed, stream, cols)[None, :]


def sylvester_hadamard(n: int) -> np.ndarray:
    """H_n by Kronecker products of [[1, 1], [1, -1]] (fp64)."""
    H = np.ones((1, 1))
    while H.shape[0] < n:
        H = np.kron(H, np.array([[1.0, 1.0], [1.0, -1.0]]))
    return H


def combine_s2f6(codes: np.ndarray, e8m0: np.ndarray, pos: np.ndarray, w: np.ndarray, seed: int,
                 stream: int) -> np.ndarray:
    """out[t] = sum_j w[t, j] * xhat[pos[t, j]], xhat the dequantised, rotated-
    back rows (fp64, one rounding to bf16)."""
    xhat = s2f6_dequantize_hadamard(codes, e8m0, seed, stream)
    out = np.einsum("tj,tjd->td", w.astype(np.float64), xhat[pos])
    return f64_to_bf16(out)
