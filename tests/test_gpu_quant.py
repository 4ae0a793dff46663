"""GPU parity of the quantisers, the stochastic requantisation and the glue
kernels against the CPU oracle, through the C ABI.

Bar: bit-exact codes, scales, outer scales, permutations; SwiGLU / combine
within one bf16 rounding (the oracle computes them in fp64).  All inputs are
seeded and synthetic; every expected value comes from the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_moe_numerics_b200 import api, workloads
from tests.layouts import mma_to_rowmajor, rowmajor_to_mma

pytestmark = pytest.mark.gpu


def to_dev_bf16(u16: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).cuda()


def to_np_u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def np_(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def heavy_rows(rows, cols, seed, nu=4, spread=3.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(nu, (rows, cols)) * 10.0 ** rng.uniform(-spread, spread, (rows, 1))
    return oracle.f32_to_bf16(x.astype(np.float32))


def crafted_rows():
    """Rows whose blocks land exactly on E2M1 and E4M3 rounding ties, zero
    blocks, zero rows, negative zeros and saturating values."""
    rows = []
    ties_e2m1 = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float64)
    # outer scale 1 (row max 2688); a block with max 1536 gets sf = 256 exactly,
    # so x/(sf*s) = x/256 is exact and elements 256*tie are exact ties
    r = np.zeros(256, np.float64)
    r[0] = 2688.0
    blk = np.concatenate([ties_e2m1, -ties_e2m1]) * 256.0
    blk[7] = 1536.0
    r[16:32] = blk
    r[32:48] = -blk
    # E4M3 ties on the block scale: block max 6 * midpoint, s = 1
    e4 = np.abs(np.arange(0x7F, dtype=np.uint8).view(__import__("ml_dtypes").float8_e4m3fn).astype(np.float64))
    mids = (e4[1:] + e4[:-1]) / 2
    for i, m in enumerate(mids[[0, 5, 20, 60, 100, 120]]):
        r[64 + 16 * i] = 6.0 * m
    r[200:216] = -0.0
    rows.append(r)
    rows.append(np.zeros(256))
    rr = np.zeros(256); rr[5] = -1e-30; rr[6] = 3e-39; rows.append(rr)   # tiny / subnormal-range values
    return oracle.f32_to_bf16(np.array(rows, np.float32))


# ---------------------------------------------------------------------------
# NVFP4 quantiser
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("rows,cols", [(256, 4096), (128, 1024), (384, 256), (7, 48), (130, 3072),
                                       (16, 8192), (3, 12304), (5, 16400), (4, 40960)])
def test_nvfp4_quantize_per_token_bit_exact(cuda, rows, cols):
    x = heavy_rows(rows, cols, seed=rows + cols)
    codes, sf, outer = oracle.nvfp4_quantize(x)
    xd = to_dev_bf16(x)
    gc, gsf, go = api.nvfp4_quantize(xd, sf_layout=api.MX_SF_ROWMAJOR)
    torch.cuda.synchronize()
    assert np.array_equal(np_(gc), codes)
    assert np.array_equal(np_(gsf).reshape(rows, cols // 16), sf)
    assert np.array_equal(np_(go).view(np.uint32), outer.view(np.uint32))
    if rows % 128 == 0 and cols % 64 == 0:
        gc2, gsf2, go2 = api.nvfp4_quantize(xd, sf_layout=api.MX_SF_MMA)
        assert np.array_equal(np_(gc2), codes)
        assert np.array_equal(mma_to_rowmajor(np_(gsf2), rows, cols // 16), sf)


def test_nvfp4_quantize_crafted_ties_and_zeros(cuda):
    x = crafted_rows()
    codes, sf, outer = oracle.nvfp4_quantize(x)
    gc, gsf, go = api.nvfp4_quantize(to_dev_bf16(x), sf_layout=api.MX_SF_ROWMAJOR)
    assert np.array_equal(np_(gc), codes)
    assert np.array_equal(np_(gsf).reshape(sf.shape), sf)
    assert np.array_equal(np_(go).view(np.uint32), outer.view(np.uint32))


@pytest.mark.parametrize("E,N,K", [(4, 128, 256), (3, 256, 512), (2, 128, 4096)])
def test_nvfp4_quantize_per_expert_bit_exact(cuda, E, N, K):
    w = workloads.weights(E, N, K, 0.02, seed=E * N + K)
    wn = w.reshape(E * N, K).view(torch.int16).numpy().view(np.uint16)
    codes, sf, outer = oracle.nvfp4_quantize(wn, group_rows=N)
    gc, gsf, go = api.nvfp4_quantize(w.reshape(E * N, K).cuda(), group_rows=N, sf_layout=api.MX_SF_MMA)
    assert np.array_equal(np_(gc), codes)
    assert np.array_equal(mma_to_rowmajor(np_(gsf), E * N, K // 16), sf)
    assert np.array_equal(np_(go).view(np.uint32), outer.view(np.uint32))


@pytest.mark.parametrize("E,N,K", [(2, 16, 64), (64, 128, 256), (5, 2048, 4096)])
def test_nvfp4_quantize_per_expert_group_sizes(cuda, E, N, K):
    # two tiny groups, 64 small groups, five 16.8 MB groups; experts decades
    # apart so that a scale from another group changes codes
    w = workloads.weights(E, N, K, 0.02, seed=E * 7 + N + K).float()
    w *= (10.0 ** torch.linspace(-2, 2, E)).view(E, 1, 1)
    w = w.to(torch.bfloat16)
    wn = w.reshape(E * N, K).view(torch.int16).numpy().view(np.uint16)
    codes, sf, outer = oracle.nvfp4_quantize(wn, group_rows=N)
    gc, gsf, go = api.nvfp4_quantize(w.reshape(E * N, K).cuda(), group_rows=N, sf_layout=api.MX_SF_ROWMAJOR)
    api.sync_status()
    assert np.array_equal(np_(go).view(np.uint32), outer.view(np.uint32))
    assert np.array_equal(np_(gsf).reshape(sf.shape), sf)
    assert np.array_equal(np_(gc), codes)


def test_nvfp4_quantize_per_expert_unaligned_groups(cuda):
    # 3 experts of 2046 x 4096 (16.8 MB each): expert boundaries fall inside a
    # block of rows of the quantiser, with row-major scales
    E, N, K = 3, 2046, 4096
    w = workloads.weights(E, N, K, 0.02, seed=77)
    wn = w.reshape(E * N, K).view(torch.int16).numpy().view(np.uint16)
    codes, sf, outer = oracle.nvfp4_quantize(wn, group_rows=N)
    gc, gsf, go = api.nvfp4_quantize(w.reshape(E * N, K).cuda(), group_rows=N, sf_layout=api.MX_SF_ROWMAJOR)
    assert np.array_equal(np_(gc), codes)
    assert np.array_equal(np_(gsf).reshape(sf.shape), sf)
    assert np.array_equal(np_(go).view(np.uint32), outer.view(np.uint32))


@pytest.mark.parametrize("E,N,K,layout", [
    (8, 512, 4096, api.MX_SF_MMA),        # 4 rows per quantiser block
    (24, 2048, 1024, api.MX_SF_MMA),      # 16 rows per quantiser block
    (6, 4096, 1024, api.MX_SF_ROWMAJOR),  # the W2 shape of the 384-expert layer, 6 experts
    (4, 256, 16384, api.MX_SF_MMA),       # one row per quantiser block
    (3, 128, 20480, api.MX_SF_ROWMAJOR),  # rows of 1280 blocks: each row read twice by its threads
])
def test_nvfp4_quantize_per_expert_spread_and_zero_experts(cuda, E, N, K, layout):
    # experts six decades apart, one all-zero expert and one expert whose amax
    # is a single element: a per-expert scale taken from the wrong expert, or
    # an amax missing some of the expert's rows, changes codes
    w = workloads.weights(E, N, K, 0.02, seed=E + N + K).float()
    w *= (10.0 ** torch.linspace(-3, 3, E)).view(E, 1, 1)
    w[1] = 0
    w[E - 1, N // 2, K // 3] = 1e4
    w = w.to(torch.bfloat16)
    wn = w.reshape(E * N, K).view(torch.int16).numpy().view(np.uint16)
    codes, sf, outer = oracle.nvfp4_quantize(wn, group_rows=N)
    gc, gsf, go = api.nvfp4_quantize(w.reshape(E * N, K).cuda(), group_rows=N, sf_layout=layout)
    api.sync_status()
    assert np.array_equal(np_(gc), codes)
    got_sf = mma_to_rowmajor(np_(gsf), E * N, K // 16) if layout == api.MX_SF_MMA else np_(gsf).reshape(sf.shape)
    assert np.array_equal(got_sf, sf)
    assert np.array_equal(np_(go).view(np.uint32), outer.view(np.uint32))
    assert outer[1] == 0 and np.all(codes[N:2 * N] == 0)


@pytest.mark.parametrize("rows,F,gated,valid,layout", [(384, 1024, True, 300, api.MX_SF_MMA),
                                                        (256, 512, False, None, api.MX_SF_MMA),
                                                        (128, 4096, True, None, api.MX_SF_MMA),
                                                        (130, 96, False, 77, api.MX_SF_ROWMAJOR)])
def test_swiglu_nvfp4_quantize_fuses_the_two_kernels(cuda, rows, F, gated, valid, layout):
    rng = np.random.default_rng(rows + F)
    h = oracle.f32_to_bf16((rng.standard_normal((rows, 2 * F if gated else F)) * 3).astype(np.float32))
    hd = to_dev_bf16(h)
    rv = torch.tensor([valid], dtype=torch.int64, device="cuda") if valid is not None else None
    fused = api.swiglu_nvfp4_quantize(hd, F, gated, rv, layout)
    a = api.swiglu_fwd(hd, F, gated, rv)
    two = api.nvfp4_quantize(a, 1, layout)
    api.sync_status()
    for got, want in zip(fused, two):                          # the same bytes as the two kernels in sequence
        assert torch.equal(got, want)
    # against the oracle's SwiGLU (fp64, one bf16 rounding) and quantiser: the
    # GPU's fast sigmoid can move a value by one bf16 unit, so rare codes differ
    n = rows if valid is None else valid
    ref_a = oracle.swiglu_fwd(h[:n], gated=gated)
    rc, rs, ro = oracle.nvfp4_quantize(ref_a)
    gc = np_(fused[0])
    assert np.mean(gc[:n] == rc) >= 0.99
    go = np_(fused[2])
    assert np.all(np.abs(go[:n] - ro) <= 2.0 ** -7 * np.abs(ro))
    assert np.all(gc[n:] == 0) and np.all(go[n:] == 0)


# ---------------------------------------------------------------------------
# MXFP8 quantiser
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("rounding,R", [(api.MX_ROUND_RNE, 8), (api.MX_ROUND_SR, 8), (api.MX_ROUND_SR, 16),
                                        (api.MX_ROUND_SR, 32)])
@pytest.mark.parametrize("rows,cols", [(128, 128), (256, 384), (512, 1024)])
def test_mxfp8_quantize_rows_and_cols_bit_exact(cuda, rows, cols, rounding, R):
    x = heavy_rows(rows, cols, seed=3 * rows + cols, spread=6.0)
    sr = rounding == api.MX_ROUND_SR
    seed, stream = 0xDEADBEEF12345, 7
    rc, re = oracle.mxfp8_quantize_rows(x, sr=sr, seed=seed, stream=stream, R=R)
    cc, ce = oracle.mxfp8_quantize_cols(x, sr=sr, seed=seed, stream=stream + 1, R=R)
    for layout in (api.MX_SF_ROWMAJOR, api.MX_SF_MMA):
        g = api.mxfp8_quantize(to_dev_bf16(x), rounding=rounding, seed=seed, stream_id=stream, rbits=R,
                               sf_layout=layout)
        assert np.array_equal(np_(g[0]), rc)
        assert np.array_equal(np_(g[2]), cc)
        if layout == api.MX_SF_ROWMAJOR:
            assert np.array_equal(np_(g[1]).reshape(re.shape), re)
            assert np.array_equal(np_(g[3]).reshape(ce.shape), ce)
        else:
            assert np.array_equal(mma_to_rowmajor(np_(g[1]), rows, cols // 32), re)
            assert np.array_equal(mma_to_rowmajor(np_(g[3]), cols, rows // 32), ce)


def test_mxfp8_quantize_column_only_and_rows_valid(cuda):
    rows, cols = 384, 256
    x = heavy_rows(rows, cols, seed=11)
    cc, ce = oracle.mxfp8_quantize_cols(x[:256])
    valid = torch.tensor([256], dtype=torch.int64, device="cuda")
    out = (None, None, torch.full((cols, rows), 0xAB, dtype=torch.uint8, device="cuda"),
           torch.full((cols * rows // 32,), 0xAB, dtype=torch.uint8, device="cuda"))
    g = api.mxfp8_quantize(to_dev_bf16(x), row=False, col=True, rows_valid=valid, sf_layout=api.MX_SF_ROWMAJOR,
                           out=out)
    gc = np_(g[2])
    assert np.array_equal(gc[:, :256], cc)
    assert np.all(gc[:, 256:] == 0xAB)              # rows beyond rows_valid untouched


# ---------------------------------------------------------------------------
# Requantisation across the transpose
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("R", [8, 16, 32])
@pytest.mark.parametrize("rows,cols", [(128, 64), (256, 512), (512, 4096)])
def test_requant_transpose_sr_bit_exact(cuda, rows, cols, R):
    x = heavy_rows(rows, cols, seed=rows * 7 + cols + R)
    codes, sf, outer = oracle.nvfp4_quantize(x)
    seed, stream = 0x0123456789ABCDEF, 0xFEDCBA98
    oc, oe = oracle.mxfp8_requant_transpose_sr(codes, sf, outer, 1, seed, stream, R)
    dc = torch.from_numpy(codes).cuda()
    do = torch.from_numpy(outer).cuda()
    for lin in (api.MX_SF_ROWMAJOR, api.MX_SF_MMA):
        if lin == api.MX_SF_MMA and (rows % 128 or cols % 64):
            continue
        dsf = torch.from_numpy(sf.reshape(-1).copy() if lin == api.MX_SF_ROWMAJOR else rowmajor_to_mma(sf)).cuda()
        for lout in (api.MX_SF_ROWMAJOR, api.MX_SF_MMA):
            if lout == api.MX_SF_MMA and cols % 128:
                continue
            gc, ge = api.mxfp8_requant_transpose_sr(dc, dsf, do, rows, cols, 1, lin, None, seed, stream, R, lout)
            assert np.array_equal(np_(gc), oc)
            ge = np_(ge)
            got_e = ge.reshape(oe.shape) if lout == api.MX_SF_ROWMAJOR else mma_to_rowmajor(ge, cols, rows // 32)
            assert np.array_equal(got_e, oe)


@pytest.mark.parametrize("R", [8, 16, 32])
def test_requant_extreme_dynamic_range(cuda, R):
    # per-row scales over 24 decades: inside one 32-row block most values sit
    # far below E4M3's normal range (and many below its smallest subnormal),
    # exercising every branch of the stochastic rounding down to fp32 subnormals
    x = heavy_rows(256, 128, seed=77 + R, spread=12.0)
    codes, sf, outer = oracle.nvfp4_quantize(x)
    oc, oe = oracle.mxfp8_requant_transpose_sr(codes, sf, outer, 1, 11, 12, R)
    gc, ge = api.mxfp8_requant_transpose_sr(torch.from_numpy(codes).cuda(), torch.from_numpy(sf.reshape(-1).copy()).cuda(),
                                            torch.from_numpy(outer).cuda(), 256, 128, 1, api.MX_SF_ROWMAJOR, None, 11, 12,
                                            R, api.MX_SF_ROWMAJOR)
    assert np.array_equal(np_(gc), oc)
    assert np.array_equal(np_(ge).reshape(oe.shape), oe)


@pytest.mark.parametrize("E,N,K,R", [(3, 128, 256, 8), (3, 384, 256, 16), (2, 1024, 128, 16)])
def test_requant_weights_per_expert_outer(cuda, E, N, K, R):
    # expert sizes a power of two (outer scale found by a shift) and not (by a division);
    # experts six decades apart, so a scale taken from the wrong expert changes codes
    w = workloads.weights(E, N, K, 0.02, seed=5 + N).float()
    w *= (10.0 ** torch.linspace(-3, 3, E)).view(E, 1, 1)
    w = w.to(torch.bfloat16).reshape(E * N, K).view(torch.int16).numpy().view(np.uint16)
    codes, sf, outer = oracle.nvfp4_quantize(w, group_rows=N)
    oc, oe = oracle.mxfp8_requant_transpose_sr(codes, sf, outer, N, 3, 4, R)
    gc, ge = api.mxfp8_requant_transpose_sr(torch.from_numpy(codes).cuda(), torch.from_numpy(rowmajor_to_mma(sf)).cuda(),
                                            torch.from_numpy(outer).cuda(), E * N, K, N, api.MX_SF_MMA, None, 3, 4, R,
                                            api.MX_SF_MMA)
    assert np.array_equal(np_(gc), oc)
    assert np.array_equal(mma_to_rowmajor(np_(ge), K, E * N // 32), oe)


@pytest.mark.parametrize("R", [8, 16, 32])
@pytest.mark.parametrize("scale_exp", [-40, -36, -30, 0, 30])
def test_requant_weights_fold_boundary(cuda, scale_exp, R):
    """One outer scale per expert: the kernel folds the outer scale
    and 2^-e into one product while p*s stays in fp32's normal range (outer
    scale >= 2^-100) and takes the two products below it.  Experts scaled by
    10^scale_exp (outer scales around the 2^-100 switch, fp32 subnormal
    dequantised values, and large values), a zero expert, and the scales read
    both from aligned words and (when misaligned) by the byte-wise kernel."""
    E, N, K = 4, 256, 256
    w = workloads.weights(E, N, K, 1.0, seed=41).double()
    w *= torch.tensor([10.0 ** scale_exp, 10.0 ** (scale_exp + 2), 0.0, 10.0 ** (scale_exp - 1)]).view(E, 1, 1)
    wf = w.reshape(E * N, K).to(torch.float32).numpy()
    w16 = oracle.f32_to_bf16(wf)
    codes, sf, outer = oracle.nvfp4_quantize(w16, group_rows=N)
    oc, oe = oracle.mxfp8_requant_transpose_sr(codes, sf, outer, N, 21, 22, R)
    sf_mma = rowmajor_to_mma(sf)
    for off in (0, 1):                                   # scales at an aligned and a misaligned address
        buf = torch.zeros(sf_mma.size + 16, dtype=torch.uint8, device="cuda")
        buf[off:off + sf_mma.size] = torch.from_numpy(sf_mma).cuda()
        gc, ge = api.mxfp8_requant_transpose_sr(torch.from_numpy(codes).cuda(), buf[off:off + sf_mma.size],
                                                torch.from_numpy(outer).cuda(), E * N, K, N, api.MX_SF_MMA, None, 21,
                                                22, R, api.MX_SF_MMA)
        assert np.array_equal(np_(gc), oc), off
        assert np.array_equal(mma_to_rowmajor(np_(ge), K, E * N // 32), oe), off


def test_requant_crafted_values(cuda):
    # the crafted row (ties, zeros, -0) repeated with power-of-two row scales
    base = oracle.bf16_to_f32(crafted_rows()[0:1, :128]).astype(np.float64)
    x = oracle.f32_to_bf16((np.repeat(base, 128, 0) * 2.0 ** (np.arange(128) % 7 - 3)[:, None]).astype(np.float32))
    codes, sf, outer = oracle.nvfp4_quantize(x)
    oc, oe = oracle.mxfp8_requant_transpose_sr(codes, sf, outer, 1, 9, 9, 8)
    gc, ge = api.mxfp8_requant_transpose_sr(torch.from_numpy(codes).cuda(), torch.from_numpy(sf.reshape(-1).copy()).cuda(),
                                            torch.from_numpy(outer).cuda(), 128, 128, 1, api.MX_SF_ROWMAJOR, None, 9, 9, 8,
                                            api.MX_SF_ROWMAJOR)
    assert np.array_equal(np_(gc), oc)
    assert np.array_equal(np_(ge).reshape(oe.shape), oe)


# ---------------------------------------------------------------------------
# Glue
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,k,E,kind,n_empty", [(256, 2, 4, "uniform", 0), (1000, 8, 64, "zipf", 3),
                                                (3000, 8, 384, "zipf", 8), (5, 3, 7, "uniform", 0)])
def test_route_gather_bit_exact(cuda, T, k, E, kind, n_empty):
    ids = workloads.routing(T, k, E, kind, 1.2, n_empty, seed=T + E)
    seg, src, pos = oracle.route(ids.numpy(), E)
    M_cap = api.max_routed_rows(T, k, E)
    gseg, gsrc, gpos = api.moe_route(ids.cuda(), E, M_cap)
    gseg, gsrc, gpos = np_(gseg), np_(gsrc), np_(gpos)
    assert np.array_equal(gseg, seg)
    assert np.array_equal(gpos, pos)
    Mp = int(seg[-1])
    # the ABI stores the assignment index t*k + j; the oracle stores the token
    flat = np.full(Mp, -1, np.int64)
    flat[pos.reshape(-1)] = np.arange(T * k)
    assert np.array_equal(gsrc[:Mp], flat)
    assert np.all(gsrc[Mp:] == -1)
    assert np.array_equal(np.where(flat >= 0, flat // k, -1), src)
    # NVFP4 dispatch: gather the per-token rows
    D = 256
    x = heavy_rows(T, D, seed=T)
    codes, sf, outer = oracle.nvfp4_quantize(x)
    oc, osf, oo = oracle.gather_nvfp4_rows(codes, sf, outer, src)
    gc, gsf, go = api.nvfp4_gather_rows(torch.from_numpy(codes).cuda(), torch.from_numpy(sf.reshape(-1).copy()).cuda(),
                                        torch.from_numpy(outer).cuda(), torch.from_numpy(gsrc).cuda(), k, D)
    gc, gsf, go = np_(gc), np_(gsf), np_(go)
    assert np.array_equal(gc[:Mp], oc)
    assert np.array_equal(mma_to_rowmajor(gsf, M_cap, D // 16)[:Mp], osf)
    assert np.array_equal(go[:Mp].view(np.uint32), oo.view(np.uint32))
    assert np.all(gc[Mp:] == 0) and np.all(go[Mp:] == 0)


def _ulp_close(got_u16, ref_u16):
    g = oracle.bf16_to_f32(got_u16).astype(np.float64)
    r = oracle.bf16_to_f32(ref_u16).astype(np.float64)
    tol = np.maximum(np.abs(r), 1e-30) * 2.0 ** -7
    return np.all(np.abs(g - r) <= tol)


@pytest.mark.parametrize("gated", [True, False])
def test_swiglu_fwd_bwd_within_one_rounding(cuda, gated):
    rows, F = 256, 512
    rng = np.random.default_rng(3)
    h = oracle.f32_to_bf16((rng.standard_normal((rows, 2 * F if gated else F)) * 3).astype(np.float32))
    da = oracle.f32_to_bf16(rng.standard_normal((rows, F)).astype(np.float32))
    a = oracle.swiglu_fwd(h, gated)
    dh = oracle.swiglu_bwd(h, da, gated)
    valid = torch.tensor([128], dtype=torch.int64, device="cuda")
    ga = to_np_u16(api.swiglu_fwd(to_dev_bf16(h), F, gated, rows_valid=valid))
    gdh = to_np_u16(api.swiglu_bwd(to_dev_bf16(h), to_dev_bf16(da), F, gated, rows_valid=valid))
    assert _ulp_close(ga[:128], a[:128]) and np.all(ga[128:] == 0)
    assert _ulp_close(gdh[:128], dh[:128]) and np.all(gdh[128:] == 0)


def test_combine_and_dispatch_grad(cuda):
    T, k, E, D = 300, 4, 16, 256
    ids = workloads.routing(T, k, E, "zipf", 1.1, 0, seed=2)
    seg, src, pos = oracle.route(ids.numpy(), E)
    M = int(seg[-1])
    rng = np.random.default_rng(4)
    y = oracle.f32_to_bf16(rng.standard_normal((M, D)).astype(np.float32))
    w = np.full((T, k), 1.0 / k, np.float32)
    ref = oracle.combine(y, pos, w)
    got = to_np_u16(api.moe_combine(to_dev_bf16(y), torch.from_numpy(pos).cuda(), torch.from_numpy(w).cuda(), D))
    assert _ulp_close(got, ref)
    dout = oracle.f32_to_bf16(rng.standard_normal((T, D)).astype(np.float32))
    M_cap = api.max_routed_rows(T, k, E)
    _, gsrc, gpos = api.moe_route(ids.cuda(), E, M_cap)
    # non-uniform weights and the all-ones (NULL) form; padding rows and the tail are zero
    wr = rng.uniform(0.1, 1.0, (T, k)).astype(np.float32)
    for wv, wd in ((wr, torch.from_numpy(wr).cuda()), (np.ones((T, k), np.float32), None)):
        ref_dy = oracle.dispatch_grad(dout, pos, wv, M)
        gdy = to_np_u16(api.moe_dispatch_grad(to_dev_bf16(dout), gsrc, gpos, wd))
        assert np.array_equal(gdy[:M], ref_dy)
        assert np.all(gdy[M:] == 0)


def test_permute_row_groups_against_indexing(cuda):
    """moe_permute_row_groups moves whole 128-row groups (the expert-parallel
    regrouping): equal to indexing by the table, zeros for -1; an index past
    the input gives zeros and MX_EDATA, not a fault."""
    from fp8_moe_numerics_b200._lib import MX_EDATA, MxError
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    for group_bytes, n_in in ((128 * 2048, 9), (128 * 128, 5), (512, 40)):
        x = torch.randint(0, 256, (n_in * group_bytes,), dtype=torch.uint8, device="cuda", generator=g)
        table = torch.tensor([3, -1, 0, n_in - 1, 1, 1, 2, -1], dtype=torch.int32, device="cuda")
        out = api.moe_permute_row_groups(x, table, group_bytes)
        api.sync_status()
        xg = x.view(-1, group_bytes)
        want = torch.zeros(table.numel(), group_bytes, dtype=torch.uint8, device="cuda")
        ok = (table >= 0) & (table < n_in)
        want[ok] = xg[table[ok].long()]
        assert torch.equal(out.view(-1, group_bytes), want)
    bad = torch.tensor([0, 7], dtype=torch.int32, device="cuda")
    out = api.moe_permute_row_groups(torch.ones(2 * 512, dtype=torch.uint8, device="cuda"), bad, 512)
    with pytest.raises(MxError) as err:
        api.sync_status()
    assert err.value.status == MX_EDATA
    assert torch.all(out[:512] == 1) and torch.all(out[512:] == 0)
    api.sync_status()
