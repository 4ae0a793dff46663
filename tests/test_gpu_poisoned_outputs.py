"""Every output byte an entry point promises to write is written.

include/mxmoe.h fixes each output's extent from the arguments ("every output
byte, including padding, is written"; the grouped GEMMs leave rows >= seg[E]
alone).  Each entry runs twice on the same inputs, once into outputs filled
with 0x00 and once into outputs filled with 0xFF: the kernels are
deterministic, so a byte that is written comes out the same both times and a
byte that is not keeps its two fills.  The check compares the promised region
of each output, whole.
"""
import numpy as np
import pytest
import torch

from fp8_moe_numerics_b200 import api, workloads

pytestmark = pytest.mark.gpu


def _twice(run, make_outs, regions=None):
    """run(outs) on outputs prefilled 0x00 and 0xFF; regions[i] slices output i
    (whole when None).  Asserts the two results agree byte for byte."""
    res = []
    for fill in (0x00, 0xFF):
        outs = make_outs()
        for o in outs:
            if o is not None:
                o.view(torch.uint8).fill_(fill)
        run(outs)
        api.sync_status()
        res.append([None if o is None else o.view(torch.uint8).clone() for o in outs])
    for i, (a, b) in enumerate(zip(*res)):
        if a is None:
            continue
        sl = regions[i] if regions and regions[i] is not None else slice(None)
        assert torch.equal(a.reshape(a.shape[0], -1)[sl] if a.dim() > 1 else a[sl],
                           b.reshape(b.shape[0], -1)[sl] if b.dim() > 1 else b[sl]), f"output {i} has unwritten bytes"


def _u8(n):
    return torch.empty(int(n), dtype=torch.uint8, device="cuda")


@pytest.fixture(scope="module")
def layer_bits():
    """A small routed problem: 6 experts (one empty), top-2 of 300 tokens, D 256, F 128."""
    E, T, k, D, F = 6, 300, 2, 256, 128
    ids = workloads.routing(T, k, E, "zipf", 1.2, 1, seed=3)
    x = workloads.activations(T, D, "normal", 4, "cuda")
    seg, src, pos = api.moe_route(ids.cuda(), E)
    xq = api.nvfp4_quantize(x, 1, api.MX_SF_ROWMAJOR)
    xp = api.nvfp4_gather_rows(*xq, src, k, D)
    w1 = workloads.weights(E, 2 * F, D, 0.02, 5, "cuda").view(E * 2 * F, D)
    w1q = api.nvfp4_quantize(w1, 2 * F, api.MX_SF_MMA)
    api.sync_status()
    return dict(E=E, T=T, k=k, D=D, F=F, ids=ids.cuda(), x=x, seg=seg, src=src, pos=pos, xq=xq, xp=xp, w1q=w1q,
                M=src.shape[0], Mp=int(seg[-1]))


@pytest.mark.parametrize("layout,group", [(api.MX_SF_ROWMAJOR, 1), (api.MX_SF_MMA, 1), (api.MX_SF_MMA, 128)])
def test_nvfp4_quantize_writes_every_byte(cuda, layout, group):
    x = workloads.activations(256, 192, "t4_rowscale", 9, "cuda")
    _twice(lambda o: api.nvfp4_quantize(x, group, layout, out=tuple(o)),
           lambda: [_u8(256 * 96), _u8(api.sf_bytes(256, 192, 16, layout)),
                    torch.empty(256 // group, dtype=torch.float32, device="cuda")])


@pytest.mark.parametrize("R", [8, 16, 32])
@pytest.mark.parametrize("lout", [api.MX_SF_ROWMAJOR, api.MX_SF_MMA])
def test_requant_writes_every_byte(cuda, R, lout):
    x = workloads.activations(256, 256, "t4_rowscale", 10, "cuda")
    q = api.nvfp4_quantize(x, 1, api.MX_SF_MMA)
    _twice(lambda o: api.mxfp8_requant_transpose_sr(*q, 256, 256, 1, api.MX_SF_MMA, None, 1, 2, R, lout, out=tuple(o)),
           lambda: [_u8(256 * 256), _u8(api.sf_bytes(256, 256, 32, lout))])


@pytest.mark.parametrize("rounding", [api.MX_ROUND_RNE, api.MX_ROUND_SR])
def test_mxfp8_quantize_writes_every_byte(cuda, rounding):
    x = workloads.gradient(384, 256, 1.0, 11, "cuda")
    _twice(lambda o: api.mxfp8_quantize(x, rounding=rounding, seed=3, out=tuple(o)),
           lambda: [_u8(384 * 256), _u8(api.sf_bytes(384, 256, 32, api.MX_SF_MMA)), _u8(384 * 256),
                    _u8(api.sf_bytes(256, 384, 32, api.MX_SF_MMA))])


def test_routing_and_dispatch_write_every_byte(cuda, layer_bits):
    L = layer_bits
    E, T, k, D, M = L["E"], L["T"], L["k"], L["D"], L["M"]
    ws = _u8(max(16, api.L.lib().mx_route_workspace_bytes(T, E)))
    _twice(lambda o: api.moe_route(L["ids"], E, M, out=(o[0], o[1], o[2], ws)),
           lambda: [torch.empty(E + 1, dtype=torch.int64, device="cuda"), torch.empty(M, dtype=torch.int32, device="cuda"),
                    torch.empty(T, k, dtype=torch.int32, device="cuda")])
    _twice(lambda o: api.nvfp4_gather_rows(*L["xq"], L["src"], k, D, out=tuple(o)),
           lambda: [_u8(M * D // 2), _u8(api.sf_bytes(M, D, 16, api.MX_SF_MMA)),
                    torch.empty(M, dtype=torch.float32, device="cuda")])
    dout = workloads.gradient(T, D, 1.0, 12, "cuda")
    w = torch.rand(T, k, device="cuda")
    _twice(lambda o: api.moe_dispatch_grad(dout, L["src"], L["pos"], w, out=o[0]),
           lambda: [torch.empty(M, D, dtype=torch.bfloat16, device="cuda")])
    y = workloads.gradient(M, D, 1.0, 13, "cuda")
    _twice(lambda o: api.moe_combine(y, L["pos"], w, D, out=o[0]),
           lambda: [torch.empty(T, D, dtype=torch.bfloat16, device="cuda")])


def test_swiglu_kernels_write_every_byte(cuda, layer_bits):
    L = layer_bits
    M, F = L["M"], L["F"]
    h = workloads.gradient(M, 2 * F, 1.0, 14, "cuda")
    da = workloads.gradient(M, F, 1.0, 15, "cuda")
    rv = L["seg"][L["E"]:L["E"] + 1]
    _twice(lambda o: api.swiglu_fwd(h, F, True, rv, out=o[0]),
           lambda: [torch.empty(M, F, dtype=torch.bfloat16, device="cuda")])
    _twice(lambda o: api.swiglu_bwd(h, da, F, True, rv, out=o[0]),
           lambda: [torch.empty(M, 2 * F, dtype=torch.bfloat16, device="cuda")])
    _twice(lambda o: api.swiglu_nvfp4_quantize(h, F, True, rv, api.MX_SF_MMA, out=tuple(o)),
           lambda: [_u8(M * F // 2), _u8(api.sf_bytes(M, F, 16, api.MX_SF_MMA)),
                    torch.empty(M, dtype=torch.float32, device="cuda")])


def test_gemms_write_every_promised_byte(cuda, layer_bits):
    L = layer_bits
    E, D, F, M, Mp, seg = L["E"], L["D"], L["F"], L["M"], L["Mp"], L["seg"]
    for dt in (torch.float32, torch.bfloat16):
        _twice(lambda o: api.grouped_gemm_nvfp4(L["xp"], L["w1q"], seg, E, 2 * F, D, out=o[0]),
               lambda: [torch.empty(M, 2 * F, dtype=dt, device="cuda")], regions=[slice(0, Mp)])
    dh = workloads.gradient(M, 2 * F, 1e-3, 16, "cuda")
    q = api.mxfp8_quantize(dh, rows_valid=seg[E:E + 1])
    w1t = api.mxfp8_requant_transpose_sr(*L["w1q"], E * 2 * F, D, 2 * F, seed=1, stream_id=1)
    xt = api.mxfp8_requant_transpose_sr(*L["xp"], M, D, 1, rows_valid=seg[E:E + 1], seed=1, stream_id=2)
    _twice(lambda o: api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, q[0], q[1], *w1t, seg, E, M, D, 2 * F, out=o[0]),
           lambda: [torch.empty(M, D, dtype=torch.bfloat16, device="cuda")], regions=[slice(0, Mp)])
    _twice(lambda o: api.grouped_gemm_mxfp8(api.MX_GEMM_WGRAD, q[2], q[3], *xt, seg, E, M, 2 * F, D, out=o[0]),
           lambda: [torch.empty(E, 2 * F, D, dtype=torch.float32, device="cuda")])


def test_s2f6_path_writes_every_promised_byte(cuda, layer_bits):
    L = layer_bits
    E, D, F, M, Mp, T, seg = L["E"], L["D"], L["F"], L["M"], L["Mp"], L["T"], L["seg"]
    x = workloads.activations(256, 256, "normal", 17, "cuda")
    _twice(lambda o: api.hadamard_s2f6_quantize(x, 3, 4, out=(o[0].view(torch.int8), o[1])),
           lambda: [_u8(256 * 256).view(256, 256), _u8(256 * 8).view(256, 8)])
    w2 = workloads.weights(E, D, 2 * F, 0.02, 18, "cuda").view(E * D, 2 * F)
    w2q = api.nvfp4_quantize(w2, D, api.MX_SF_MMA)
    aq = api.nvfp4_quantize(workloads.activations(M, 2 * F, "normal", 19, "cuda"), 1, api.MX_SF_MMA)
    _twice(lambda o: api.grouped_gemm_nvfp4_s2f6(aq, w2q, seg, E, D, 2 * F, 5, 6,
                                                 out=(o[0].view(torch.int8), o[1])),
           lambda: [_u8(M * D).view(M, D), _u8(M * D // 32).view(M, D // 32)], regions=[slice(0, Mp), slice(0, Mp)])
    codes = torch.randint(-127, 128, (M, D), dtype=torch.int8, device="cuda")
    e8 = torch.randint(100, 140, (M, D // 32), dtype=torch.uint8, device="cuda")
    w = torch.rand(T, L["k"], device="cuda")
    _twice(lambda o: api.moe_combine_s2f6(codes, e8, L["pos"], w, 5, 6, out=o[0]),
           lambda: [torch.empty(T, D, dtype=torch.bfloat16, device="cuda")])


def test_nvfp4_backward_entries_write_every_byte(cuda, layer_bits):
    L = layer_bits
    x = workloads.activations(256, 128, "t4_rowscale", 20, "cuda")
    _twice(lambda o: api.nvfp4_quantize_sr(x, 1, api.MX_ROUND_SR, 3, 4, 16, api.MX_SF_MMA, out=tuple(o)),
           lambda: [_u8(256 * 64), _u8(api.sf_bytes(256, 128, 16, api.MX_SF_MMA)),
                    torch.empty(256, dtype=torch.float32, device="cuda")])
    q = api.nvfp4_quantize(x, 1, api.MX_SF_MMA)
    _twice(lambda o: api.nvfp4_requant_transpose_sr(*q, 256, 128, 1, api.MX_SF_MMA, 1, False, api.MX_ROUND_SR, 3, 4,
                                                    16, api.MX_SF_MMA, out=tuple(o)),
           lambda: [_u8(128 * 128), _u8(api.sf_bytes(128, 256, 16, api.MX_SF_MMA)),
                    torch.empty(128, dtype=torch.float32, device="cuda")])
    _twice(lambda o: api.nvfp4_quantize_tile16(x, 64, out=tuple(o)),
           lambda: [_u8(256 * 64), _u8(256 // 16 * 128 // 16), torch.empty(4, dtype=torch.float32, device="cuda")])
