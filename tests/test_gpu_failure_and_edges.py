"""Failure detection without a fault, and degenerate inputs, on the GPU.

- A bounded device wait that runs out (a barrier nothing completes) is
  reported as MX_ETIMEOUT by the next status query, which also clears it; the
  context stays usable (a quantisation afterwards is still bit-exact).
- Empty problems: zero rows, zero tokens, a grouped GEMM with no routed rows,
  and a weight-gradient GEMM whose experts are all empty.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_moe_numerics_b200 import api
from fp8_moe_numerics_b200._lib import MX_ETIMEOUT, MxError

pytestmark = pytest.mark.gpu


def test_bounded_wait_expiry_is_reported_and_cleared(cuda):
    api.sync_status()                                   # nothing pending
    api.wait_selftest(20_000)                           # 20 ms
    with pytest.raises(MxError) as err:
        api.sync_status()
    assert err.value.status == MX_ETIMEOUT
    api.sync_status()                                   # cleared by the previous query
    rng = np.random.default_rng(0)
    x = oracle.f32_to_bf16(rng.standard_normal((128, 256)).astype(np.float32))
    codes, sf, outer = oracle.nvfp4_quantize(x)
    g = api.nvfp4_quantize(torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16), sf_layout=api.MX_SF_ROWMAJOR)
    api.sync_status()
    assert np.array_equal(g[0].cpu().numpy(), codes)


def test_empty_quantisations(cuda):
    x = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    c, s, o = api.nvfp4_quantize(x)
    assert c.shape == (0, 128) and o.numel() == 0
    rc, re, cc, ce = api.mxfp8_quantize(torch.empty(0, 128, dtype=torch.bfloat16, device="cuda"))
    assert rc.shape == (0, 128) and cc.shape == (128, 0)
    oc, oe = api.mxfp8_requant_transpose_sr(c, s, o, 0, 256)
    assert oc.shape == (256, 0)
    api.sync_status()


def test_routing_with_no_tokens(cuda):
    E, k = 8, 2
    seg, src, pos = api.moe_route(torch.empty(0, k, dtype=torch.int32, device="cuda"), E)
    api.sync_status()
    assert np.all(seg.cpu().numpy() == 0)
    assert np.all(src.cpu().numpy() == -1) and pos.numel() == 0


def test_gemms_with_no_routed_rows(cuda):
    E, N, K = 3, 256, 256
    seg = torch.zeros(E + 1, dtype=torch.int64, device="cuda")
    # forward GEMM over an empty row buffer: nothing to compute
    a = (torch.empty(0, K // 2, dtype=torch.uint8, device="cuda"), torch.empty(0, dtype=torch.uint8, device="cuda"),
         torch.empty(0, dtype=torch.float32, device="cuda"))
    b = (torch.ones(E * N, K // 2, dtype=torch.uint8, device="cuda"),
         torch.full((E * N * K // 16,), 0x38, dtype=torch.uint8, device="cuda"), torch.ones(E, device="cuda"))
    out = api.grouped_gemm_nvfp4(a, b, seg, E, N, K)
    assert out.shape == (0, N)
    # weight gradient with every expert empty: zeros
    M_cap = 128
    ac = torch.full((N, M_cap), 0x38, dtype=torch.uint8, device="cuda")
    ae = torch.full((N * M_cap // 32,), 127, dtype=torch.uint8, device="cuda")
    bc = torch.full((K, M_cap), 0x38, dtype=torch.uint8, device="cuda")
    be = torch.full((K * M_cap // 32,), 127, dtype=torch.uint8, device="cuda")
    dw = torch.full((E, N, K), float("nan"), dtype=torch.float32, device="cuda")
    api.grouped_gemm_mxfp8(api.MX_GEMM_WGRAD, ac, ae, bc, be, seg, E, M_cap, N, K, out=dw)
    api.sync_status()
    assert torch.all(dw == 0)


def test_routing_leaves_out_bad_ids_and_reports_them(cuda):
    """Expert ids outside [0, E) and an id repeated within a token are left
    out of the routing (pos = -1, no row), flagged as MX_EDATA by the next
    status query, and skipped by the combine; nothing is written outside the
    buffers and the context stays usable."""
    from fp8_moe_numerics_b200._lib import MX_EDATA
    rng = np.random.default_rng(3)
    T, k, E, D = 300, 4, 8, 64
    topk = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    topk[5, 1] = -3
    topk[17, 0] = E
    topk[40, 3] = 1 << 30
    topk[41, 2] = topk[41, 0]                            # repeat within one token
    topk[299, 1] = -(1 << 31)
    valid = np.ones((T, k), bool)
    valid[5, 1] = valid[17, 0] = valid[40, 3] = valid[41, 2] = valid[299, 1] = False
    api.sync_status()
    seg, src, pos = api.moe_route(torch.from_numpy(topk).cuda(), E)
    with pytest.raises(MxError) as err:
        api.sync_status()
    assert err.value.status == MX_EDATA
    api.sync_status()                                   # cleared by the previous query
    # expected routing of the valid entries: per expert in token order, segments padded to 128
    counts = np.bincount(topk[valid], minlength=E)
    seg_ref = np.concatenate([[0], np.cumsum((counts + 127) // 128 * 128)])
    assert np.array_equal(seg.cpu().numpy(), seg_ref)
    pos_ref = np.full((T, k), -1, np.int64)
    fill = seg_ref[:-1].copy()
    for t in range(T):
        for j in range(k):
            if valid[t, j]:
                pos_ref[t, j] = fill[topk[t, j]]
                fill[topk[t, j]] += 1
    assert np.array_equal(pos.cpu().numpy(), pos_ref)
    src_np = src.cpu().numpy()
    src_ref = np.full(src_np.shape, -1, np.int64)
    src_ref[pos_ref[valid]] = np.flatnonzero(valid.ravel())
    assert np.array_equal(src_np, src_ref)
    # the combine skips the left-out entries
    y = torch.randn(src.shape[0], D, device="cuda").to(torch.bfloat16)
    w = torch.rand(T, k, device="cuda")
    out = api.moe_combine(y, pos, w, D).float().cpu()
    yh, wh = y.float().cpu(), w.cpu()
    ref = torch.zeros(T, D)
    for j in range(k):
        p = torch.from_numpy(pos_ref[:, j])
        ok = p >= 0
        ref[ok] += wh[ok, j:j + 1] * yh[p[ok]]
    assert torch.allclose(out, ref, rtol=2 ** -7, atol=1e-6)
    # a valid routing afterwards matches the oracle
    good = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    seg, src, pos = api.moe_route(torch.from_numpy(good).cuda(), E)
    api.sync_status()
    seg_o, src_o, pos_o = oracle.route(good, E)
    assert np.array_equal(seg.cpu().numpy(), seg_o) and np.array_equal(pos.cpu().numpy(), pos_o)
