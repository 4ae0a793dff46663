"""Parity at the benchmark's full sizes, in the launch configurations bench.py
times.

- Quantiser stream (bf16 16384 x 4096): NVFP4 quantisation and the R = 16
  requantisation compared with the oracle element for element.
- The 384-expert layer's four grouped GEMM shapes (bf16 output, CTA pairs)
  on seeded random operands: sampled outputs against fp64 dot products of the
  oracle-decoded operand rows.
- One full step of the 384-expert layer: routing and the token quantisation
  compared whole; dispatch gather, expert weights, the weight requantisation,
  the combine gradient and its MXFP8 rows on sampled rows and entries, each
  recomputed by the oracle from the seeded inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_moe_numerics_b200 import api, workloads
from fp8_moe_numerics_b200.layer import ExpertLayer
from tests.layouts import mma_to_rowmajor

pytestmark = pytest.mark.gpu

MOE = workloads.CONFIGS["moe_layer"]


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def np_(t):
    return t.detach().cpu().numpy()


def mma_rows(buf_cpu: np.ndarray, rows, S: int) -> np.ndarray:
    """Row-major scales [len(rows), S] read out of an MMA-layout buffer."""
    r = np.asarray(rows, dtype=np.int64)[:, None]
    s = np.arange(S, dtype=np.int64)[None, :]
    off = ((r // 128) * (S // 4) + s // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + s % 4
    return buf_cpu.reshape(-1)[off]


def test_quant_stream_full_size_bit_exact(cuda):
    c = workloads.CONFIGS["quant_stream"]
    rows, cols = c["rows"], c["cols"]
    x = workloads.activations(rows, cols, c["x_dist"], c["seed"], "cpu")
    codes, sf, outer = oracle.nvfp4_quantize(x.view(torch.int16).numpy().view(np.uint16))
    g = api.nvfp4_quantize(x.cuda())                                   # MMA scale layout, as benchmarked
    assert np.array_equal(np_(g[0]), codes)
    assert np.array_equal(mma_to_rowmajor(np_(g[1]), rows, cols // 16), sf)
    assert np.array_equal(np_(g[2]).view(np.uint32), outer.view(np.uint32))
    rc, re = oracle.mxfp8_requant_transpose_sr(codes, sf, outer, 1, seed=c["sr_seed"], stream=0, R=16)
    gc, ge = api.mxfp8_requant_transpose_sr(*g, rows, cols, seed=c["sr_seed"], stream_id=0, rbits=16)
    assert np.array_equal(np_(gc), rc)
    assert np.array_equal(mma_to_rowmajor(np_(ge), cols, rows // 32), re)


# ---------------------------------------------------------------------------
# grouped GEMMs at the 384-expert layer's shapes
# ---------------------------------------------------------------------------
def _moe_routing():
    T, k, E = MOE["T"], MOE["k"], MOE["E"]
    ids = workloads.routing(T, k, E, MOE["routing"], MOE["zipf"], MOE["n_empty"], MOE["seed"])
    seg, src, pos = oracle.route(ids.numpy(), E)
    return seg, api.max_routed_rows(T, k, E)


def _rand_u8(shape, lo, hi, g):
    return torch.randint(lo, hi, shape, dtype=torch.uint8, device="cuda", generator=g)


def _sample_rows_cols(seg, E, N, n, seed):
    """n (row, col, expert) samples over the routed rows (padding rows included), a quarter of
    them in the last row tile of experts with an odd tile count (at this layer those tiles run in
    the grouped GEMMs' tail kernel, the rest in the CTA-pair kernel)."""
    rng = np.random.default_rng(seed)
    tiles = np.diff(seg[:E + 1]) // 128
    odd = np.flatnonzero(tiles % 2 == 1)
    n_tail = n // 4
    tail_rows = seg[odd[rng.integers(0, len(odd), n_tail)] + 1] - 128 + rng.integers(0, 128, n_tail)
    rows = np.concatenate([rng.integers(0, int(seg[E]), n - n_tail), tail_rows])
    cols = rng.integers(0, N, n)
    experts = np.searchsorted(seg, rows, side="right") - 1
    return rows, cols, experts


def _close_bf16(got, ref):
    tol = 2.0 ** -8 * np.abs(ref) + 1e-3 * np.sqrt(np.mean(ref ** 2))
    return np.all(np.abs(got - ref) <= tol)


@pytest.mark.parametrize("N,K", [(2 * MOE["F"], MOE["D"]), (MOE["D"], MOE["F"])])   # GEMM1, GEMM2
def test_grouped_gemm_nvfp4_full_layer_shape(cuda, N, K):
    seg, M_cap = _moe_routing()
    E = MOE["E"]
    g = torch.Generator(device="cuda")
    g.manual_seed(N + K)
    a = (_rand_u8((M_cap, K // 2), 0, 256, g), _rand_u8((M_cap * K // 16,), 0x28, 0x49, g),
         torch.rand(M_cap, device="cuda", generator=g) + 0.5)
    b = (_rand_u8((E * N, K // 2), 0, 256, g), _rand_u8((E * N * K // 16,), 0x28, 0x49, g),
         torch.rand(E, device="cuda", generator=g) + 0.5)
    out = api.grouped_gemm_nvfp4(a, b, torch.from_numpy(seg).cuda(), E, N, K, out_dtype=torch.bfloat16)
    api.sync_status()
    rows, cols, ex = _sample_rows_cols(seg, E, N, 384, seed=N)
    a_sf, b_sf = np_(a[1]), np_(b[1])
    a_val = oracle.nvfp4_block_values(np_(a[0][torch.from_numpy(rows).cuda()]), mma_rows(a_sf, rows, K // 16))
    brow = ex * N + cols
    b_val = oracle.nvfp4_block_values(np_(b[0][torch.from_numpy(brow).cuda()]), mma_rows(b_sf, brow, K // 16))
    ref = np.sum(a_val * b_val, axis=1) * np_(a[2])[rows].astype(np.float64) * np_(b[2])[ex].astype(np.float64)
    got = oracle.bf16_to_f32(u16(out[torch.from_numpy(rows).cuda(), torch.from_numpy(cols).cuda()])).astype(np.float64)
    assert _close_bf16(got, ref)


def test_grouped_gemm_nvfp4_s2f6_epilogue_full_layer_shape(cuda):
    # GEMM2 of the 384-expert layer with the rotate + S2F6 epilogue: sampled
    # 32-column blocks against the oracle's rotation and quantisation of the
    # fp64 product (rounded to fp32); codes within one, exponents equal away
    # from a boundary
    seg, M_cap = _moe_routing()
    E, N, K = MOE["E"], MOE["D"], MOE["F"]
    seed, stream = 5, 101
    g = torch.Generator(device="cuda")
    g.manual_seed(77)
    a = (_rand_u8((M_cap, K // 2), 0, 256, g), _rand_u8((M_cap * K // 16,), 0x28, 0x49, g),
         torch.rand(M_cap, device="cuda", generator=g) + 0.5)
    b = (_rand_u8((E * N, K // 2), 0, 256, g), _rand_u8((E * N * K // 16,), 0x28, 0x49, g),
         torch.rand(E, device="cuda", generator=g) + 0.5)
    codes, e8 = api.grouped_gemm_nvfp4_s2f6(a, b, torch.from_numpy(seg).cuda(), E, N, K, seed, stream)
    api.sync_status()
    rows, _, ex = _sample_rows_cols(seg, E, N, 48, seed=3)
    blocks = np.random.default_rng(4).integers(0, N // 32, 48)
    a_sf, b_sf = np_(a[1]), np_(b[1])
    a_val = oracle.nvfp4_block_values(np_(a[0][torch.from_numpy(rows).cuda()]), mma_rows(a_sf, rows, K // 16))
    flips = 0
    for i, (r, jb, e) in enumerate(zip(rows, blocks, ex)):
        brow = e * N + 32 * jb + np.arange(32)
        b_val = oracle.nvfp4_block_values(np_(b[0][torch.from_numpy(brow).cuda()]), mma_rows(b_sf, brow, K // 16))
        ref = (b_val @ a_val[i]) * float(np_(a[2])[r]) * float(np_(b[2])[e])
        xrow = np.zeros((1, 32 * (jb + 1)), np.float32)
        xrow[0, 32 * jb:] = ref.astype(np.float32)
        rc, re = oracle.s2f6_quantize_hadamard(xrow, seed, stream)
        gc = np_(codes[int(r), 32 * jb:32 * (jb + 1)]).astype(np.int64)
        ge = int(np_(e8[int(r), jb]))
        if ge != int(re[0, jb]):                      # only where the block amax sits on a boundary
            z = oracle.fwht32_f32(xrow[:, 32 * jb:] * oracle.hadamard_signs(seed, stream, 32 * (jb + 1))[32 * jb:]
                                  .astype(np.float32))
            ratio = np.abs(z).max() / np.ldexp(127 / 64, int(re[0, jb]) - 127)
            assert min(abs(ratio - 1.0), abs(2 * ratio - 1.0)) < 1e-5
            continue
        d = np.abs(gc - rc[0, 32 * jb:].astype(np.int64))
        assert d.max() <= 1
        flips += int(np.count_nonzero(d))
    assert flips <= 0.01 * 48 * 32


def _rand_e4m3(shape, g):
    """Random E4M3 code bytes without the two NaN codes."""
    c = torch.randint(0, 254, shape, dtype=torch.int32, device="cuda", generator=g)
    return (c + (c >= 0x7F).to(torch.int32)).to(torch.uint8)          # skip 0x7F; 0xFF is never drawn


def test_grouped_gemm_mxfp8_dgrad_full_layer_shape(cuda):
    # dgrad1: dX = dH1 . W1 -> A [M_cap, 2F] row-wise, B [D, E*2F], out [M_cap, D]
    seg, M_cap = _moe_routing()
    E, D, Kc = MOE["E"], MOE["D"], 2 * MOE["F"]
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    a, ae = _rand_e4m3((M_cap, Kc), g), _rand_u8((M_cap * Kc // 32,), 120, 135, g)
    b, be = _rand_e4m3((D, E * Kc), g), _rand_u8((D * E * Kc // 32,), 120, 135, g)
    out = api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, a, ae, b, be, torch.from_numpy(seg).cuda(), E, M_cap, D, Kc,
                                 out_dtype=torch.bfloat16)
    api.sync_status()
    rows, cols, ex = _sample_rows_cols(seg, E, D, 256, seed=4)
    ae_c, be_c = np_(ae), np_(be)
    a_val = oracle.mxfp8_dequantize(np_(a[torch.from_numpy(rows).cuda()]), mma_rows(ae_c, rows, Kc // 32))
    b_rows, b_sf = np_(b[torch.from_numpy(cols).cuda()]), mma_rows(be_c, cols, E * Kc // 32)
    ref = np.empty(len(rows))
    for i, e in enumerate(ex):                          # decode only expert e's K range of B's row
        bv = oracle.mxfp8_dequantize(b_rows[i:i + 1, e * Kc:(e + 1) * Kc], b_sf[i:i + 1, e * Kc // 32:(e + 1) * Kc // 32])
        ref[i] = np.dot(a_val[i], bv[0])
    got = oracle.bf16_to_f32(u16(out[torch.from_numpy(rows).cuda(), torch.from_numpy(cols).cuda()])).astype(np.float64)
    assert _close_bf16(got, ref)


def test_grouped_gemm_mxfp8_wgrad_full_layer_shape(cuda):
    # wgrad1: dW1_e = dH1_e^T . X_e -> A [2F, M_cap], B [D, M_cap] (blocks along tokens), out [E, 2F, D]
    seg, M_cap = _moe_routing()
    E, Nw, Kw = MOE["E"], 2 * MOE["F"], MOE["D"]
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    a, ae = _rand_e4m3((Nw, M_cap), g), _rand_u8((Nw * M_cap // 32,), 120, 135, g)
    b, be = _rand_e4m3((Kw, M_cap), g), _rand_u8((Kw * M_cap // 32,), 120, 135, g)
    out = api.grouped_gemm_mxfp8(api.MX_GEMM_WGRAD, a, ae, b, be, torch.from_numpy(seg).cuda(), E, M_cap, Nw, Kw,
                                 out_dtype=torch.bfloat16)
    api.sync_status()
    rng = np.random.default_rng(6)
    ex, n, kk = rng.integers(0, E, 192), rng.integers(0, Nw, 192), rng.integers(0, Kw, 192)
    a_rows, a_sf = np_(a[torch.from_numpy(n).cuda()]), mma_rows(np_(ae), n, M_cap // 32)
    b_rows, b_sf = np_(b[torch.from_numpy(kk).cuda()]), mma_rows(np_(be), kk, M_cap // 32)
    ref = np.zeros(len(ex))
    for i, e in enumerate(ex):                          # decode only expert e's token range
        s0, s1 = int(seg[e]), int(seg[e + 1])
        if s1 > s0:
            av = oracle.mxfp8_dequantize(a_rows[i:i + 1, s0:s1], a_sf[i:i + 1, s0 // 32:s1 // 32])
            bv = oracle.mxfp8_dequantize(b_rows[i:i + 1, s0:s1], b_sf[i:i + 1, s0 // 32:s1 // 32])
            ref[i] = np.dot(av[0], bv[0])
    idx = [torch.from_numpy(v).cuda() for v in (ex, n, kk)]
    got = oracle.bf16_to_f32(u16(out[idx[0], idx[1], idx[2]])).astype(np.float64)
    empty = seg[ex + 1] == seg[ex]
    assert np.all(got[empty] == 0)
    assert _close_bf16(got[~empty], ref[~empty])


# ---------------------------------------------------------------------------
# one step of the 384-expert layer, as bench.py runs it
# ---------------------------------------------------------------------------
def test_moe_layer_step_full_size(cuda):
    T, k, E, D, F = MOE["T"], MOE["k"], MOE["E"], MOE["D"], MOE["F"]
    N1 = 2 * F
    inp = workloads.layer_inputs("moe_layer", device="cuda")
    seed = 1234
    L = ExpertLayer(inp["x"], inp["topk"].cuda(), inp["w_comb"].cuda(), inp["w1"], inp["w2"], inp["dout"], gated=True,
                    seed=seed)
    L.step()
    api.sync_status()
    rng = np.random.default_rng(8)

    # routing, whole (the library's src holds t*k + j where the oracle's holds the token t)
    seg, src, pos = oracle.route(np_(inp["topk"]), E)
    Mp = int(seg[-1])
    assert np.array_equal(np_(L.seg), seg) and np.array_equal(np_(L.pos), pos)
    copy_of = np.full(Mp, -1, np.int64)
    copy_of[pos.reshape(-1)] = np.arange(T * k)
    assert np.array_equal(np_(L.src)[:Mp], copy_of)

    # token quantisation (per-token outer scale, row-major scales), whole
    xc, xs, xo = oracle.nvfp4_quantize(u16(inp["x"]))
    assert np.array_equal(np_(L.xq[0]), xc) and np.array_equal(np_(L.xq[1]).reshape(xs.shape), xs)
    assert np.array_equal(np_(L.xq[2]).view(np.uint32), xo.view(np.uint32))

    # dispatch gather into expert order, sampled rows (padding rows included)
    p = rng.integers(0, Mp, 256)
    gc, gs, go = oracle.gather_nvfp4_rows(xc, xs, xo, src[p])
    assert np.array_equal(np_(L.xp[0])[p], gc)
    assert np.array_equal(mma_rows(np_(L.xp[1]), p, D // 16), gs)
    assert np.array_equal(np_(L.xp[2])[p].view(np.uint32), go.view(np.uint32))

    # expert weights (per-expert outer scale) and the W1 requantisation, sampled experts
    w1q_sf, w1t_c, w1t_e = np_(L.w1q[1]), np_(L.w1t[0]), np_(L.w1t[1])
    for e in rng.choice(E, 2, replace=False):
        w = u16(inp["w1"][e])                                          # [N1, D]
        qc, qs, qo = oracle.nvfp4_quantize(w, group_rows=N1)
        rows = np.arange(e * N1, (e + 1) * N1)
        assert np.array_equal(np_(L.w1q[0][e * N1:(e + 1) * N1]), qc)
        assert np.array_equal(mma_rows(w1q_sf, rows, D // 16), qs)
        assert np_(L.w1q[2])[e].view(np.uint32) == qo.view(np.uint32)[0]
        per_row = np.full(N1, qo[0], np.float32)
        for _ in range(24):                                            # W1^T entries [c, e*N1 + r]
            c, r = int(rng.integers(D)), int(rng.integers(N1))
            r0 = r - r % 32
            code, e8 = oracle.mxfp8_requant_entry(qc[r0:r0 + 32], qs[r0:r0 + 32], per_row[r0:r0 + 32], c, r % 32,
                                                  E * N1, e * N1 + r0, seed, 3, 16)
            assert w1t_c[c, e * N1 + r] == code
            assert mma_rows(w1t_e, [c], E * N1 // 32)[0, (e * N1 + r) // 32] == e8
        w2 = u16(inp["w2"][e])                                         # [D, F]
        qc2, qs2, qo2 = oracle.nvfp4_quantize(w2, group_rows=D)
        assert np.array_equal(np_(L.w2q[0][e * D:(e + 1) * D]), qc2)
        assert np_(L.w2q[2])[e].view(np.uint32) == qo2.view(np.uint32)[0]

    # combine gradient and its row-wise MXFP8 form, sampled rows of true tokens and padding
    dout, w = u16(inp["dout"]), np_(inp["w_comb"])
    dy2c, dy2e = np_(L.dy2q[0]), mma_rows(np_(L.dy2q[1]), p, D // 32)
    for i, row in enumerate(p):
        s = int(copy_of[row])                                          # t*k + j, or -1 on padding
        if s >= 0:
            ref = oracle.dispatch_grad(dout[s // k][None], np.zeros((1, 1), np.int32), w[s // k, s % k].reshape(1, 1), 1)
        else:
            ref = np.zeros((1, D), np.uint16)
        rc, re = oracle.mxfp8_quantize_rows(ref)
        assert np.array_equal(dy2c[row], rc[0]) and np.array_equal(dy2e[i], re[0])
