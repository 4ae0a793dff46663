"""Python binding of the mxmoe C ABI (include/mxmoe.h).

Argument marshalling only: each function allocates its outputs with torch on
the inputs' CUDA device, passes raw device pointers and the current CUDA
stream to the library, and raises MxError on a non-MX_OK status.  Every
computation happens in the library's sm_100a kernels.

Since the library sees bare pointers, the binding checks what only it can:
every tensor is contiguous, on the current CUDA device, and holds at least
the bytes include/mxmoe.h gives for its role (ValueError otherwise, before
anything is launched).  Index contents (routing rows, segment offsets) are
not read on the host.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib as L
from ._lib import (MX_GEMM_DGRAD, MX_GEMM_WGRAD, MX_OUT_BF16, MX_OUT_F32, MX_ROUND_RNE, MX_ROUND_SR,
                   MX_SF_MMA, MX_SF_ROWMAJOR, MxError)

__all__ = [
    "MX_SF_ROWMAJOR", "MX_SF_MMA", "MX_ROUND_RNE", "MX_ROUND_SR", "MX_GEMM_DGRAD", "MX_GEMM_WGRAD", "MxError",
    "sf_bytes", "sync_status", "wait_selftest", "nvfp4_quantize", "mxfp8_requant_transpose_sr", "mxfp8_quantize",
    "grouped_gemm_nvfp4", "grouped_gemm_mxfp8", "moe_route", "nvfp4_gather_rows", "swiglu_fwd", "swiglu_bwd",
    "moe_combine", "moe_dispatch_grad", "swiglu_nvfp4_quantize", "hadamard_s2f6_quantize", "grouped_gemm_nvfp4_s2f6",
    "moe_combine_s2f6", "nvfp4_quantize_sr", "nvfp4_requant_transpose_sr", "nvfp4_quantize_tile16",
    "nvfp4_quantize_transpose_segments", "nvfp4_requant_transpose_segments", "grouped_gemm_nvfp4_wgrad",
    "max_routed_rows", "moe_permute_row_groups",
]


def _p(t) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if not t.is_cuda:
        raise ValueError("mxmoe operates on CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("mxmoe expects contiguous tensors")
    if t.get_device() != torch.cuda.current_device():
        raise ValueError(f"mxmoe launches on the current device (cuda:{torch.cuda.current_device()}); "
                         f"a tensor is on cuda:{t.get_device()}")
    return ctypes.c_void_p(t.data_ptr())


def _fits(what: str, t, need: int) -> None:
    """The library receives bare pointers and cannot see a buffer's extent:
    raise unless tensor `t` (when given) holds the `need` bytes the call
    reads or writes through it, as include/mxmoe.h sizes them."""
    if t is not None and t.numel() * t.element_size() < need:
        raise ValueError(f"{what}: {t.numel() * t.element_size()} bytes, the call needs {need}")


def _bf16_2d(what: str, t) -> None:
    if t.dtype != torch.bfloat16 or t.dim() != 2:
        raise ValueError(f"{what} must be a 2-D bf16 tensor, got {t.dtype} of {t.dim()} dims")


def _s() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _u8(n: int, dev) -> torch.Tensor:
    return torch.empty(int(n), dtype=torch.uint8, device=dev)


def sf_bytes(rows: int, cols: int, block: int, layout: int) -> int:
    n = L.lib().mx_sf_bytes(rows, cols, block, layout)
    if n == 0 and rows * cols > 0:
        raise ValueError(f"scale shape {rows}x{cols}/{block} not allowed for layout {layout}")
    return n


def sync_status(stream=None) -> None:
    s = ctypes.c_void_p((stream or torch.cuda.current_stream()).cuda_stream)
    st = L.lib().mx_sync_status(s)
    if st != L.MX_OK:
        raise MxError("mx_sync_status", st, L.lib().mx_last_cuda_error())


def wait_selftest(limit_us: int) -> None:
    """Run the bounded-wait expiry path once; the next sync_status() raises
    MxError with status MX_ETIMEOUT."""
    L.call("mx_wait_selftest", int(limit_us), _s())


def nvfp4_quantize(x: torch.Tensor, group_rows: int = 1, sf_layout: int = MX_SF_MMA, out=None):
    """bf16 [rows, cols] -> (codes u8 [rows, cols/2], sf u8, outer f32 [rows/group_rows])."""
    _bf16_2d("x", x)
    rows, cols = x.shape
    dev = x.device
    if out is None:
        out = (torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev),
               _u8(sf_bytes(rows, cols, 16, sf_layout), dev),
               torch.empty(rows // group_rows, dtype=torch.float32, device=dev))
    codes, sf, outer = out
    _fits("codes", codes, rows * cols // 2)
    _fits("sf", sf, rows * (cols // 16))
    _fits("outer", outer, 4 * (rows // max(group_rows, 1)))
    L.call("nvfp4_quantize", _p(x), rows, cols, group_rows, _p(codes), _p(sf), _p(outer), sf_layout, _s())
    return codes, sf, outer


def mxfp8_requant_transpose_sr(codes, sf, outer, rows: int, cols: int, group_rows: int = 1,
                               in_sf_layout: int = MX_SF_MMA, rows_valid=None, seed: int = 0, stream_id: int = 0,
                               rbits: int = 16, out_sf_layout: int = MX_SF_MMA, out=None):
    """Saved NVFP4 [rows, cols] -> MXFP8 [cols, rows] codes and E8M0 scales."""
    dev = codes.device
    if out is None:
        out = (torch.empty(cols, rows, dtype=torch.uint8, device=dev), _u8(sf_bytes(cols, rows, 32, out_sf_layout), dev))
    oc, oe = out
    _fits("codes", codes, rows * cols // 2)
    _fits("sf", sf, rows * (cols // 16))
    _fits("outer", outer, 4 * (rows // max(group_rows, 1)))
    _fits("rows_valid", rows_valid, 8)
    _fits("out codes", oc, rows * cols)
    _fits("out e8m0", oe, cols * (rows // 32))
    L.call("mxfp8_requant_transpose_sr", _p(codes), _p(sf), _p(outer), rows, cols, group_rows, in_sf_layout,
           _p(rows_valid), ctypes.c_uint64(seed), ctypes.c_uint64(stream_id), rbits, _p(oc), _p(oe),
           out_sf_layout, _s())
    return oc, oe


def mxfp8_quantize(x: torch.Tensor, row: bool = True, col: bool = True, rounding: int = MX_ROUND_RNE,
                   seed: int = 0, stream_id: int = 0, rbits: int = 16, rows_valid=None,
                   sf_layout: int = MX_SF_MMA, out=None):
    """bf16 [rows, cols] -> (row codes [rows, cols], row E8M0, col codes [cols, rows], col E8M0);
    the forms not requested are None."""
    _bf16_2d("x", x)
    rows, cols = x.shape
    dev = x.device
    if out is None:
        out = (torch.empty(rows, cols, dtype=torch.uint8, device=dev) if row else None,
               _u8(sf_bytes(rows, cols, 32, sf_layout), dev) if row else None,
               torch.empty(cols, rows, dtype=torch.uint8, device=dev) if col else None,
               _u8(sf_bytes(cols, rows, 32, sf_layout), dev) if col else None)
    rc, re, cc, ce = out
    _fits("row codes", rc, rows * cols)
    _fits("row e8m0", re, rows * (cols // 32))
    _fits("col codes", cc, rows * cols)
    _fits("col e8m0", ce, cols * (rows // 32))
    _fits("rows_valid", rows_valid, 8)
    L.call("mxfp8_quantize", _p(x), rows, cols, rounding, ctypes.c_uint64(seed), ctypes.c_uint64(stream_id), rbits,
           _p(rows_valid), _p(rc), _p(re), _p(cc), _p(ce), sf_layout, _s())
    return rc, re, cc, ce


def _out_code(dtype) -> int:
    if dtype == torch.float32:
        return MX_OUT_F32
    if dtype == torch.bfloat16:
        return MX_OUT_BF16
    raise ValueError(dtype)


def _nvfp4_operands_fit(a, b, seg, E: int, M_cap: int, N: int, K: int) -> None:
    _fits("a codes", a[0], M_cap * K // 2)
    _fits("a sf", a[1], M_cap * (K // 16))
    _fits("a outer", a[2], 4 * M_cap)
    _fits("b codes", b[0], E * N * K // 2)
    _fits("b sf", b[1], E * N * (K // 16))
    _fits("b outer", b[2], 4 * E)
    _fits("seg", seg, 8 * (E + 1))


def grouped_gemm_nvfp4(a, b, seg: torch.Tensor, E: int, N: int, K: int, out_dtype=torch.bfloat16, out=None):
    """a = (codes [M_cap, K/2], sf, outer [M_cap]); b = (codes [E*N, K/2], sf, outer [E]).
    Returns out [M_cap, N]; rows >= seg[E] are not written."""
    M_cap = a[0].shape[0]
    if out is None:
        out = torch.empty(M_cap, N, dtype=out_dtype, device=a[0].device)
    _nvfp4_operands_fit(a, b, seg, E, M_cap, N, K)
    _fits("out", out, M_cap * N * out.element_size())
    L.call("grouped_gemm_nvfp4", _p(a[0]), _p(a[1]), _p(a[2]), _p(b[0]), _p(b[1]), _p(b[2]), _p(seg), E, M_cap, N,
           K, _p(out), _out_code(out.dtype), _s())
    return out


def grouped_gemm_mxfp8(mode: int, a_codes, a_e8m0, b_codes, b_e8m0, seg: torch.Tensor, E: int, M_cap: int, N: int,
                       K: int, out_dtype=torch.bfloat16, out=None):
    """DGRAD: A [M_cap, K], B [N, E*K] -> out [M_cap, N].
    WGRAD: A [N, M_cap], B [K, M_cap] -> out [E, N, K]."""
    if out is None:
        shape = (M_cap, N) if mode == MX_GEMM_DGRAD else (E, N, K)
        out = torch.empty(*shape, dtype=out_dtype, device=a_codes.device)
    if mode == MX_GEMM_DGRAD:
        _fits("a codes", a_codes, M_cap * K)
        _fits("a e8m0", a_e8m0, M_cap * (K // 32))
        _fits("b codes", b_codes, N * E * K)
        _fits("b e8m0", b_e8m0, N * (E * K // 32))
        _fits("out", out, M_cap * N * out.element_size())
    else:
        _fits("a codes", a_codes, N * M_cap)
        _fits("a e8m0", a_e8m0, N * (M_cap // 32))
        _fits("b codes", b_codes, K * M_cap)
        _fits("b e8m0", b_e8m0, K * (M_cap // 32))
        _fits("out", out, E * N * K * out.element_size())
    _fits("seg", seg, 8 * (E + 1))
    L.call("grouped_gemm_mxfp8", mode, _p(a_codes), _p(a_e8m0), _p(b_codes), _p(b_e8m0), _p(seg), E, M_cap, N, K,
           _p(out), _out_code(out.dtype), _s())
    return out


def max_routed_rows(T: int, k: int, E: int, align: int = 128) -> int:
    cap = T * k + (align - 1) * E
    return (cap + align - 1) // align * align


def moe_route(topk: torch.Tensor, E: int, M_cap: int | None = None, out=None, align: int = 128):
    """topk int32 [T, k] -> (seg int64 [E+1], src int32 [M_cap], pos int32 [T, k]); segments
    padded to a multiple of `align` rows (128, or 256 for the NVFP4 wgrad)."""
    T, k = topk.shape
    dev = topk.device
    if M_cap is None:
        M_cap = max_routed_rows(T, k, E, align)
    ws_bytes = L.lib().mx_route_workspace_bytes(T, E)
    if out is None:
        out = (torch.empty(E + 1, dtype=torch.int64, device=dev), torch.empty(M_cap, dtype=torch.int32, device=dev),
               torch.empty(T, k, dtype=torch.int32, device=dev), _u8(max(ws_bytes, 16), dev))
    seg, src, pos, ws = out
    _fits("seg", seg, 8 * (E + 1))
    _fits("src", src, 4 * M_cap)
    _fits("pos", pos, 4 * T * k)
    if align == 128:
        L.call("moe_route", _p(topk), T, k, E, M_cap, _p(seg), _p(src), _p(pos), _p(ws),
               ws.numel() * ws.element_size(), _s())
    else:
        L.call("moe_route_aligned", _p(topk), T, k, E, align, M_cap, _p(seg), _p(src), _p(pos), _p(ws),
               ws.numel() * ws.element_size(), _s())
    return seg, src, pos


def nvfp4_gather_rows(codes, sf_rowmajor, outer, src: torch.Tensor, k: int, cols: int, out=None):
    M_cap = src.shape[0]
    dev = codes.device
    if out is None:
        out = (torch.empty(M_cap, cols // 2, dtype=torch.uint8, device=dev), _u8(sf_bytes(M_cap, cols, 16, MX_SF_MMA), dev),
               torch.empty(M_cap, dtype=torch.float32, device=dev))
    oc, osf, oo = out
    _fits("out codes", oc, M_cap * cols // 2)
    _fits("out sf", osf, M_cap * (cols // 16))
    _fits("out outer", oo, 4 * M_cap)
    L.call("nvfp4_gather_rows", _p(codes), _p(sf_rowmajor), _p(outer), _p(src), k, M_cap, cols, _p(oc), _p(osf),
           _p(oo), _s())
    return oc, osf, oo


def moe_permute_row_groups(x: torch.Tensor, group_src: torch.Tensor, group_bytes: int, out=None):
    """Regroup a row buffer array by whole groups of `group_bytes` bytes (128
    rows' worth): out group g = x group group_src[g] (int32 on the device), or
    zeros where group_src[g] < 0."""
    nin = x.numel() * x.element_size() // group_bytes
    nout = group_src.numel()
    if out is None:
        out = torch.empty(nout * group_bytes // x.element_size(), dtype=x.dtype, device=x.device)
    if group_src.dtype != torch.int32:
        raise ValueError("group_src must be int32")
    _fits("out", out, nout * group_bytes)
    if out.data_ptr() < x.data_ptr() + x.numel() * x.element_size() and \
            x.data_ptr() < out.data_ptr() + out.numel() * out.element_size():
        raise ValueError("moe_permute_row_groups: in and out overlap")
    L.call("moe_permute_row_groups", _p(x), nin, _p(out), nout, group_bytes, _p(group_src), _s())
    return out


def swiglu_fwd(h: torch.Tensor, F: int, gated: bool = True, rows_valid=None, out=None):
    rows = h.shape[0]
    if out is None:
        out = torch.empty(rows, F, dtype=torch.bfloat16, device=h.device)
    _fits("h", h, rows * (2 * F if gated else F) * 2)
    _fits("a", out, rows * F * 2)
    _fits("rows_valid", rows_valid, 8)
    L.call("swiglu_fwd", _p(h), rows, F, int(gated), _p(rows_valid), _p(out), _s())
    return out


def swiglu_bwd(h: torch.Tensor, da: torch.Tensor, F: int, gated: bool = True, rows_valid=None, out=None):
    rows = h.shape[0]
    if out is None:
        out = torch.empty_like(h)
    _fits("h", h, rows * (2 * F if gated else F) * 2)
    _fits("da", da, rows * F * 2)
    _fits("dh", out, rows * (2 * F if gated else F) * 2)
    _fits("rows_valid", rows_valid, 8)
    L.call("swiglu_bwd", _p(h), _p(da), rows, F, int(gated), _p(rows_valid), _p(out), _s())
    return out


def moe_combine(y: torch.Tensor, pos: torch.Tensor, w, D: int, out=None):
    T, k = pos.shape
    if out is None:
        out = torch.empty(T, D, dtype=torch.bfloat16, device=y.device)
    _fits("w", w, 4 * T * k)
    _fits("out", out, T * D * 2)
    L.call("moe_combine", _p(y), _p(pos), _p(w), T, k, D, _p(out), _s())
    return out


def moe_dispatch_grad(dout: torch.Tensor, src: torch.Tensor, pos: torch.Tensor, w, out=None):
    """dout bf16 [T, D], src [M_cap], pos [T, k] from moe_route -> dy bf16 [M_cap, D]."""
    M_cap = src.shape[0]
    T, k = pos.shape
    D = dout.shape[1]
    if out is None:
        out = torch.empty(M_cap, D, dtype=torch.bfloat16, device=dout.device)
    _fits("dout", dout, T * D * 2)
    _fits("w", w, 4 * T * k)
    _fits("dy", out, M_cap * D * 2)
    L.call("moe_dispatch_grad", _p(dout), _p(src), _p(pos), _p(w), T, k, M_cap, D, _p(out), _s())
    return out


def _mxfp8_pair_out(rows: int, cols: int, sf_layout: int, dev, out):
    """The four outputs of an MXFP8 quantisation of [rows, cols] (both forms)."""
    if out is None:
        out = (torch.empty(rows, cols, dtype=torch.uint8, device=dev), _u8(sf_bytes(rows, cols, 32, sf_layout), dev),
               torch.empty(cols, rows, dtype=torch.uint8, device=dev), _u8(sf_bytes(cols, rows, 32, sf_layout), dev))
    rc, re, cc, ce = out
    _fits("row codes", rc, rows * cols)
    _fits("row e8m0", re, rows * (cols // 32))
    _fits("col codes", cc, rows * cols)
    _fits("col e8m0", ce, cols * (rows // 32))
    return out


def moe_dispatch_grad_mxfp8_quantize(dout: torch.Tensor, src: torch.Tensor, w, k: int, rows_valid=None,
                                     sf_layout: int = MX_SF_MMA, out=None):
    """mxfp8_quantize(moe_dispatch_grad(dout, src, pos, w), RNE, both forms, rows_valid) without the bf16 dy:
    (row codes, row E8M0, col codes, col E8M0) of dy [M_cap, D]."""
    M_cap = src.shape[0]
    T, D = dout.shape
    _fits("w", w, 4 * T * k)
    _fits("rows_valid", rows_valid, 8)
    rc, re, cc, ce = _mxfp8_pair_out(M_cap, D, sf_layout, dout.device, out)
    L.call("moe_dispatch_grad_mxfp8_quantize", _p(dout), _p(src), _p(w), T, k, M_cap, D, _p(rows_valid), _p(rc),
           _p(re), _p(cc), _p(ce), sf_layout, _s())
    return rc, re, cc, ce


def hadamard_s2f6_quantize(x: torch.Tensor, seed: int, stream_id: int, out=None):
    """bf16 [rows, cols] -> (codes int8 [rows, cols], e8m0 u8 [rows, cols/32]):
    32-d random Hadamard rotation per column block, block-scaled S2F6."""
    _bf16_2d("x", x)
    rows, cols = x.shape
    if out is None:
        out = (torch.empty(rows, cols, dtype=torch.int8, device=x.device),
               torch.empty(rows, cols // 32, dtype=torch.uint8, device=x.device))
    codes, e8m0 = out
    _fits("codes", codes, rows * cols)
    _fits("e8m0", e8m0, rows * (cols // 32))
    L.call("hadamard_s2f6_quantize", _p(x), rows, cols, seed, stream_id, _p(codes), _p(e8m0), _s())
    return codes, e8m0


def grouped_gemm_nvfp4_s2f6(a, b, seg: torch.Tensor, E: int, N: int, K: int, seed: int, stream_id: int, out=None):
    """grouped_gemm_nvfp4 whose epilogue writes S2F6: (codes int8 [M_cap, N], e8m0 u8 [M_cap, N/32])."""
    M_cap = a[0].shape[0]
    if out is None:
        out = (torch.empty(M_cap, N, dtype=torch.int8, device=a[0].device),
               torch.empty(M_cap, N // 32, dtype=torch.uint8, device=a[0].device))
    codes, e8m0 = out
    _nvfp4_operands_fit(a, b, seg, E, M_cap, N, K)
    _fits("codes", codes, M_cap * N)
    _fits("e8m0", e8m0, M_cap * (N // 32))
    L.call("grouped_gemm_nvfp4_s2f6", _p(a[0]), _p(a[1]), _p(a[2]), _p(b[0]), _p(b[1]), _p(b[2]), _p(seg), E, M_cap,
           N, K, seed, stream_id, _p(codes), _p(e8m0), _s())
    return codes, e8m0


def moe_combine_s2f6(codes: torch.Tensor, e8m0: torch.Tensor, pos: torch.Tensor, w, seed: int, stream_id: int,
                     out=None):
    """out[t] = sum_j w[t, j] * rotated-back S2F6 row pos[t, j]; bf16 [T, D]."""
    T, k = pos.shape
    D = codes.shape[1]
    if out is None:
        out = torch.empty(T, D, dtype=torch.bfloat16, device=codes.device)
    _fits("e8m0", e8m0, codes.shape[0] * (D // 32))
    _fits("w", w, 4 * T * k)
    _fits("out", out, T * D * 2)
    L.call("moe_combine_s2f6", _p(codes), _p(e8m0), _p(pos), _p(w), T, k, D, seed, stream_id, _p(out), _s())
    return out


def swiglu_nvfp4_quantize(h: torch.Tensor, F: int, gated: bool = True, rows_valid=None, sf_layout: int = MX_SF_MMA,
                          out=None):
    """SwiGLU of h (bf16 [rows, 2F] or [rows, F]) quantised to NVFP4 per token:
    (codes u8 [rows, F/2], sf u8, outer f32 [rows])."""
    _bf16_2d("h", h)
    rows = h.shape[0]
    if out is None:
        out = (torch.empty(rows, F // 2, dtype=torch.uint8, device=h.device),
               _u8(sf_bytes(rows, F, 16, sf_layout), h.device),
               torch.empty(rows, dtype=torch.float32, device=h.device))
    codes, sf, outer = out
    _fits("h", h, rows * (2 * F if gated else F) * 2)
    _fits("codes", codes, rows * F // 2)
    _fits("sf", sf, rows * (F // 16))
    _fits("outer", outer, 4 * rows)
    _fits("rows_valid", rows_valid, 8)
    L.call("swiglu_nvfp4_quantize", _p(h), rows, F, int(gated), _p(rows_valid), _p(codes), _p(sf), _p(outer),
           sf_layout, _s())
    return codes, sf, outer


# NVFP4 in the backward pass and the 16x16 shared-scale format
# (include/mxmoe.h gives the readings).

def nvfp4_quantize_sr(x: torch.Tensor, group_rows: int = 1, rounding: int = MX_ROUND_SR, seed: int = 0,
                      stream_id: int = 0, rbits: int = 16, sf_layout: int = MX_SF_MMA, out=None):
    """bf16 [rows, cols] -> NVFP4 (codes u8 [rows, cols/2], sf u8, outer f32 [rows/group_rows]) with
    stochastically rounded E2M1 codes (MX_ROUND_SR) or to nearest (MX_ROUND_RNE)."""
    _bf16_2d("x", x)
    rows, cols = x.shape
    dev = x.device
    if out is None:
        out = (torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev),
               _u8(sf_bytes(rows, cols, 16, sf_layout), dev),
               torch.empty(rows // group_rows, dtype=torch.float32, device=dev))
    codes, sf, outer = out
    _fits("codes", codes, rows * cols // 2)
    _fits("sf", sf, rows * (cols // 16))
    _fits("outer", outer, 4 * (rows // max(group_rows, 1)))
    L.call("nvfp4_quantize_sr", _p(x), rows, cols, group_rows, rounding, ctypes.c_uint64(seed),
           ctypes.c_uint64(stream_id), rbits, _p(codes), _p(sf), _p(outer), sf_layout, _s())
    return codes, sf, outer


def nvfp4_requant_transpose_sr(codes, sf, outer, rows: int, cols: int, group_rows: int = 1,
                               in_sf_layout: int = MX_SF_MMA, experts: int = 1, out_outer_per_expert: bool = False,
                               rounding: int = MX_ROUND_SR, seed: int = 0, stream_id: int = 0, rbits: int = 16,
                               out_sf_layout: int = MX_SF_MMA, out=None):
    """Saved NVFP4 [rows, cols] (`experts` stacked row blocks) -> NVFP4 of each block's transpose,
    stacked: (codes u8 [experts*cols, rows/experts/2], sf u8, outer f32 [experts*cols or experts])."""
    dev = codes.device
    orows, ocols = experts * cols, rows // max(experts, 1)
    n_outer = experts if out_outer_per_expert else orows
    if out is None:
        out = (torch.empty(orows, ocols // 2, dtype=torch.uint8, device=dev),
               _u8(sf_bytes(orows, ocols, 16, out_sf_layout), dev),
               torch.empty(n_outer, dtype=torch.float32, device=dev))
    oc, osf, oo = out
    _fits("codes", codes, rows * cols // 2)
    _fits("sf", sf, rows * (cols // 16))
    _fits("outer", outer, 4 * (rows // max(group_rows, 1)))
    _fits("out codes", oc, orows * ocols // 2)
    _fits("out sf", osf, orows * (ocols // 16))
    _fits("out outer", oo, 4 * n_outer)
    L.call("nvfp4_requant_transpose_sr", _p(codes), _p(sf), _p(outer), rows, cols, group_rows, in_sf_layout, experts,
           int(out_outer_per_expert), rounding, ctypes.c_uint64(seed), ctypes.c_uint64(stream_id), rbits, _p(oc),
           _p(osf), _p(oo), out_sf_layout, _s())
    return oc, osf, oo


def nvfp4_quantize_tile16(x: torch.Tensor, group_rows: int = 16, out=None):
    """bf16 [rows, cols] -> NVFP4 with one E4M3 scale per 16x16 tile: (codes u8 [rows, cols/2],
    sf_tile u8 [rows/16, cols/16], outer f32 [rows/group_rows])."""
    _bf16_2d("x", x)
    rows, cols = x.shape
    dev = x.device
    if out is None:
        out = (torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev),
               torch.empty(rows // 16, cols // 16, dtype=torch.uint8, device=dev),
               torch.empty(rows // max(group_rows, 1), dtype=torch.float32, device=dev))
    codes, sf_tile, outer = out
    _fits("codes", codes, rows * cols // 2)
    _fits("sf_tile", sf_tile, (rows // 16) * (cols // 16))
    _fits("outer", outer, 4 * (rows // max(group_rows, 1)))
    L.call("nvfp4_quantize_tile16", _p(x), rows, cols, group_rows, _p(codes), _p(sf_tile), _p(outer), _s())
    return codes, sf_tile, outer


def _segment_outputs(M: int, C: int, E: int, per_row: bool, out_sf_layout: int, dev, out):
    n_outer = E * C if per_row else E
    if out is None:
        out = (torch.empty(C, M // 2, dtype=torch.uint8, device=dev), _u8(sf_bytes(C, M, 16, out_sf_layout), dev),
               torch.empty(n_outer, dtype=torch.float32, device=dev))
    oc, osf, oo = out
    _fits("out codes", oc, C * M // 2)
    _fits("out sf", osf, C * (M // 16))
    _fits("out outer", oo, 4 * n_outer)
    return oc, osf, oo


def nvfp4_quantize_transpose_segments(x: torch.Tensor, seg: torch.Tensor, E: int, per_row: bool = True,
                                      rounding: int = MX_ROUND_SR, seed: int = 0, stream_id: int = 0, rbits: int = 16,
                                      out_sf_layout: int = MX_SF_MMA, out=None):
    """bf16 [M, C] token-major -> NVFP4 of its transpose [C, M] with outer scales per expert
    segment (per (segment, row) when per_row): (codes u8 [C, M/2], sf u8, outer f32)."""
    _bf16_2d("x", x)
    M, C = x.shape
    _fits("seg", seg, 8 * (E + 1))
    oc, osf, oo = _segment_outputs(M, C, E, per_row, out_sf_layout, x.device, out)
    L.call("nvfp4_quantize_transpose_segments", _p(x), M, C, _p(seg), E, int(per_row), rounding, ctypes.c_uint64(seed),
           ctypes.c_uint64(stream_id), rbits, _p(oc), _p(osf), _p(oo), out_sf_layout, _s())
    return oc, osf, oo


def nvfp4_requant_transpose_segments(codes, sf, outer, M: int, C: int, seg: torch.Tensor, E: int,
                                     per_row: bool = False, group_rows: int = 1, in_sf_layout: int = MX_SF_MMA,
                                     rounding: int = MX_ROUND_SR, seed: int = 0, stream_id: int = 0, rbits: int = 16,
                                     out_sf_layout: int = MX_SF_MMA, out=None):
    """Saved NVFP4 [M, C] -> NVFP4 of its transpose [C, M] with outer scales per expert segment."""
    _fits("codes", codes, M * C // 2)
    _fits("sf", sf, M * (C // 16))
    _fits("outer", outer, 4 * (M // max(group_rows, 1)))
    _fits("seg", seg, 8 * (E + 1))
    oc, osf, oo = _segment_outputs(M, C, E, per_row, out_sf_layout, codes.device, out)
    L.call("nvfp4_requant_transpose_segments", _p(codes), _p(sf), _p(outer), in_sf_layout, group_rows, M, C, _p(seg),
           E, int(per_row), rounding, ctypes.c_uint64(seed), ctypes.c_uint64(stream_id), rbits, _p(oc), _p(osf),
           _p(oo), out_sf_layout, _s())
    return oc, osf, oo


def grouped_gemm_nvfp4_wgrad(a, b, seg: torch.Tensor, E: int, N: int, K: int, out_dtype=torch.float32, out=None):
    """a = (codes [N, M_cap/2], sf, outer [E*N]); b = (codes [K, M_cap/2], sf, outer [E]).
    Returns out [E, N, K] = per-expert sums over the segment's tokens (segments at multiples of 256)."""
    M_cap = a[0].shape[1] * 2
    if out is None:
        out = torch.empty(E, N, K, dtype=out_dtype, device=a[0].device)
    _fits("a codes", a[0], N * M_cap // 2)
    _fits("a sf", a[1], N * (M_cap // 16))
    _fits("a outer", a[2], 4 * E * N)
    _fits("b codes", b[0], K * M_cap // 2)
    _fits("b sf", b[1], K * (M_cap // 16))
    _fits("b outer", b[2], 4 * E)
    _fits("seg", seg, 8 * (E + 1))
    _fits("out", out, E * N * K * out.element_size())
    L.call("grouped_gemm_nvfp4_wgrad", _p(a[0]), _p(a[1]), _p(a[2]), _p(b[0]), _p(b[1]), _p(b[2]), _p(seg), E, M_cap,
           N, K, _p(out), _out_code(out.dtype), _s())
    return out
