"""The dispatch gradient fused into the MXFP8 gradient quantiser, on the GPU.

moe_dispatch_grad_mxfp8_quantize promises the bytes of moe_dispatch_grad
followed by mxfp8_quantize (RNE, both forms, the same rows_valid), without
the bf16 intermediate.  Each case runs both ways on the
same inputs and compares the four outputs over the row tiles below
rows_valid; the chain's own parity against the oracle is covered by the glue
and quantiser tests and by the layer's stage-wise test.  Outputs are filled
with 0x00 and 0xFF beforehand so that an unwritten byte shows.
"""
import pytest
import torch

from fp8_moe_numerics_b200 import api, workloads

pytestmark = pytest.mark.gpu


def _filled(outs, fill):
    for o in outs:
        o.view(torch.uint8).fill_(fill)
    return outs


def _mx_out(rows, cols, layout):
    return (torch.empty(rows, cols, dtype=torch.uint8, device="cuda"),
            torch.empty(api.sf_bytes(rows, cols, 32, layout), dtype=torch.uint8, device="cuda"),
            torch.empty(cols, rows, dtype=torch.uint8, device="cuda"),
            torch.empty(api.sf_bytes(cols, rows, 32, layout), dtype=torch.uint8, device="cuda"))


def _same(fused, chain, rows_ok, rows, cols, layout):
    """Outputs agree on row tiles [0, rows_ok): row codes and column codes
    whole over those rows; the scale arrays compared through their row-major
    views of the same rows."""
    from tests.layouts import mma_to_rowmajor
    g = lambda t: t.cpu().numpy()
    assert torch.equal(fused[0][:rows_ok], chain[0][:rows_ok])
    assert torch.equal(fused[2][:, :rows_ok], chain[2][:, :rows_ok])
    rm = (lambda a, r, c: mma_to_rowmajor(a, r, c)) if layout == api.MX_SF_MMA else (lambda a, r, c: a.reshape(r, c))
    assert (rm(g(fused[1]), rows, cols // 32)[:rows_ok] == rm(g(chain[1]), rows, cols // 32)[:rows_ok]).all()
    assert (rm(g(fused[3]), cols, rows // 32)[:, :rows_ok // 32] ==
            rm(g(chain[3]), cols, rows // 32)[:, :rows_ok // 32]).all()


@pytest.mark.parametrize("E,T,k,D,weighted,layout", [
    (6, 300, 2, 256, True, api.MX_SF_MMA),       # one empty expert, padding rows, rows past seg[E]
    (6, 300, 2, 256, False, api.MX_SF_ROWMAJOR),
    (64, 4096, 8, 1024, True, api.MX_SF_MMA),    # many tiles per block: the producer's look-ahead
])
def test_dispatch_grad_fused_equals_chain(cuda, E, T, k, D, weighted, layout):
    ids = workloads.routing(T, k, E, "zipf", 1.2, 1, seed=3).cuda()
    seg, src, pos = api.moe_route(ids, E)
    M = src.shape[0]
    dout = workloads.gradient(T, D, 1.0, 12, "cuda")
    w = torch.rand(T, k, device="cuda") if weighted else None
    rv = seg[E:E + 1]
    dy = api.moe_dispatch_grad(dout, src, pos, w)
    chain = api.mxfp8_quantize(dy, rows_valid=rv, sf_layout=layout)
    valid = int(seg[E])
    for fill in (0x00, 0xFF):
        fused = api.moe_dispatch_grad_mxfp8_quantize(dout, src, w, k, rv, layout,
                                                     out=_filled(_mx_out(M, D, layout), fill))
        api.sync_status()
        _same(fused, chain, valid, M, D, layout)


def test_fused_backward_layer_equals_unfused(cuda):
    # the tiny layer stepped both ways: the same gradients, and the same dY2
    # codes on the rows the backward GEMMs read (row tiles below seg[E])
    from fp8_moe_numerics_b200.layer import ExpertLayer
    inp = workloads.layer_inputs("tiny_layer", device="cpu")
    outs = []
    for fuse in (True, False):
        L = ExpertLayer(inp["x"].cuda(), inp["topk"].cuda(), inp["w_comb"].cuda(), inp["w1"].cuda(),
                        inp["w2"].cuda(), inp["dout"].cuda(), gated=False, seed=4, fuse_backward=fuse)
        L.step()
        api.sync_status()
        valid = int(L.seg[L.E])
        outs.append([t.cpu() for t in (L.dx, L.dw1, L.dw2, L.dy2q[0][:valid], L.dy2q[2][:, :valid])])
    for a, b in zip(*outs):
        assert torch.equal(a, b)
