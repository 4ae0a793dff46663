"""Pins for the oracle's NVFP4 quantiser, MXFP8 quantiser and the
dequantise -> transpose -> MXFP8 stochastic requantisation.

Checks use closed forms, ml_dtypes' independent rounding, invariants the
pages state (per-token outer scales make quantisation independent of other
batch members; SR preserves values in expectation; 4.5 / 8.25 bits per value)
and exhaustive enumeration.
"""
import ml_dtypes
import numpy as np
import pytest


def _bf16(orc, x):
    return orc.f32_to_bf16(np.asarray(x, dtype=np.float32))


def _rand_rows(orc, rows, cols, seed=0, heavy=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(4, (rows, cols)) if heavy else rng.standard_normal((rows, cols))
    x *= 10.0 ** rng.uniform(-3, 3, (rows, 1))
    return _bf16(orc, x)


def test_nvfp4_constant_row_closed_form(orc):
    for c in (1.0, -3.5, 1e-20, 7.0e30):
        x = _bf16(orc, np.full((1, 64), c))
        cf = float(orc.bf16_to_f32(x)[0, 0])
        codes, sf, outer = orc.nvfp4_quantize(x)
        s = np.float32(abs(cf)) / np.float32(2688.0)
        assert outer[0] == s
        assert np.all(sf == 0x7E)                                  # 448
        want = 0x7 | (0x8 if cf < 0 else 0)                        # +-6
        assert np.all(codes == (want | (want << 4)))
        xh = orc.nvfp4_dequantize(codes, sf, outer)
        assert np.allclose(xh, cf, rtol=2 ** -20)


def test_nvfp4_zero_row_and_zero_block(orc):
    x = np.zeros((2, 32), np.float32)
    x[1, 16:] = 1.0                              # row 1: first block zero
    codes, sf, outer = orc.nvfp4_quantize(_bf16(orc, x))
    assert outer[0] == 0 and np.all(sf[0] == 0) and np.all(codes[0] == 0)
    assert sf[1, 0] == 0 and np.all(codes[1, :8] == 0) and sf[1, 1] == 0x7E


def test_nvfp4_element_rounding_matches_ml_dtypes(orc):
    # Given the reading's scales, every code is the RNE-saturating E2M1 of
    # x * (1/(sf*s)) and every block scale the RNE E4M3 of amax_b/(6 s):
    # both roundings are re-done here by ml_dtypes.
    x = _rand_rows(orc, 64, 256, seed=4)
    codes, sf, outer = orc.nvfp4_quantize(x)
    xf = orc.bf16_to_f32(x)
    for r in range(x.shape[0]):
        s = np.float32(outer[r])
        for b in range(16):
            blk = xf[r, b * 16:(b + 1) * 16]
            d = np.float32(np.max(np.abs(blk))) / (np.float32(6.0) * s)
            sc = np.array([d], np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)[0]
            assert sf[r, b] == sc
            if sc == 0:
                continue
            scv = np.float32(np.array([sc], np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float32)[0])
            inv = np.float32(1.0) / (scv * s)
            q = (blk * inv).astype(np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
            packed = codes[r, b * 8:(b + 1) * 8]
            assert np.array_equal(packed & 15, q[0::2]) and np.array_equal(packed >> 4, q[1::2])


def test_nvfp4_row_max_maps_to_top_of_grid(orc):
    x = _rand_rows(orc, 32, 128, seed=5)
    codes, sf, outer = orc.nvfp4_quantize(x)
    xf = orc.bf16_to_f32(x)
    for r in range(32):
        i = int(np.argmax(np.abs(xf[r])))
        assert sf[r, i // 16] == 0x7E                              # block scale 448
        nib = (codes[r, i // 2] >> (4 * (i & 1))) & 7
        assert nib == 7                                            # |code| = 6


def test_nvfp4_error_bound(orc):
    # |x - xhat| <= sf*s (half the widest E2M1 gap, 2) unless x/(sf s) > 6
    x = _rand_rows(orc, 128, 256, seed=6)
    codes, sf, outer = orc.nvfp4_quantize(x)
    xf = orc.bf16_to_f32(x).astype(np.float64)
    xh = orc.nvfp4_dequantize(codes, sf, outer).astype(np.float64)
    unit = orc.e4m3_decode_table()[sf].astype(np.float64).repeat(16, axis=1) * outer[:, None]
    ratio = np.abs(xf) / np.where(unit > 0, unit, 1)
    bound = np.maximum(1.0, ratio - 6.0) * unit * (1 + 2 ** -20) + 1e-45
    assert np.all(np.abs(xf - xh) <= bound)


def test_nvfp4_per_token_outer_scale_is_row_independent(orc):
    # ai-primer "Block scales and per-token activations": one outer scale per
    # token keeps quantisation independent of other batch members.
    x = _rand_rows(orc, 48, 128, seed=7)
    full = orc.nvfp4_quantize(x)
    for r in (0, 17, 47):
        one = orc.nvfp4_quantize(x[r:r + 1])
        for a, b in zip(one, full):
            assert np.array_equal(a[0], b[r])
    # quantise-then-gather == gather-then-quantise
    perm = np.random.default_rng(0).permutation(48)
    g = orc.nvfp4_quantize(x[perm])
    for a, b in zip(g, full):
        assert np.array_equal(a, b[perm])


def test_nvfp4_per_expert_outer_scale(orc):
    E, N, K = 3, 16, 64
    w = _rand_rows(orc, E * N, K, seed=8, heavy=False)
    codes, sf, outer = orc.nvfp4_quantize(w, group_rows=N)
    wf = orc.bf16_to_f32(w).reshape(E, N, K)
    assert outer.shape == (E,)
    for e in range(E):
        assert outer[e] == np.float32(np.abs(wf[e]).max()) / np.float32(2688.0)
        sub = orc.nvfp4_quantize(w[e * N:(e + 1) * N], group_rows=N)
        assert np.array_equal(sub[0], codes[e * N:(e + 1) * N])


# --------------------------------------------------------------------------
# MXFP8
# --------------------------------------------------------------------------

def test_mxfp8_rows_rne_matches_ml_dtypes(orc):
    x = _rand_rows(orc, 16, 256, seed=9)
    codes, e8 = orc.mxfp8_quantize_rows(x)
    xf = orc.bf16_to_f32(x).astype(np.float64)
    for r in range(16):
        for b in range(8):
            blk = xf[r, b * 32:(b + 1) * 32]
            e = int(e8[r, b]) - 127
            assert e == orc.e8m0_exponent(np.abs(blk).max())
            y = np.ldexp(blk, -e).astype(np.float32)
            ref = y.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
            assert np.array_equal(codes[r, b * 32:(b + 1) * 32], ref)


def test_mxfp8_cols_is_transpose_of_rows(orc):
    x = _rand_rows(orc, 64, 96, seed=10)
    ct, et = orc.mxfp8_quantize_cols(x)
    cr, er = orc.mxfp8_quantize_rows(np.ascontiguousarray(x.T))
    assert np.array_equal(ct, cr) and np.array_equal(et, er)


def test_mxfp8_block_max_lands_in_top_binade(orc):
    # e minimal => the block max scaled by 2^-e lies in (224, 448]
    x = _rand_rows(orc, 8, 512, seed=11)
    codes, e8 = orc.mxfp8_quantize_rows(x)
    xf = orc.bf16_to_f32(x).astype(np.float64)
    for r in range(8):
        for b in range(16):
            m = np.abs(xf[r, b * 32:(b + 1) * 32]).max()
            if m == 0:
                continue
            y = m * 2.0 ** -(int(e8[r, b]) - 127)
            assert 224 < y <= 448


# --------------------------------------------------------------------------
# Requantisation across the transpose
# --------------------------------------------------------------------------

def test_requant_bits_per_value_and_shapes(orc):
    x = _rand_rows(orc, 64, 128, seed=12)
    nv = orc.nvfp4_quantize(x)
    oc, oe = orc.mxfp8_requant_transpose_sr(*nv, group_rows=1, seed=0, stream=0)
    assert oc.shape == (128, 64) and oe.shape == (128, 2)
    assert 8 * (oc.nbytes + oe.nbytes) / oc.size == 8.25


def test_requant_identity_when_values_sit_on_the_new_grid(orc):
    # Power-of-two outer and block scales: every dequantised value is an E2M1
    # value times 2^k, which E4M3 holds exactly after the block's 2^-e, so the
    # stochastic rounding has nothing to round, for every seed.
    rng = np.random.default_rng(13)
    rows, cols = 64, 64
    codes = rng.integers(0, 256, (rows, cols // 2), dtype=np.uint8)
    sf = np.full((rows, cols // 16), 0x38, np.uint8)               # E4M3 1.0
    sf[::3] = 0x40                                                  # E4M3 2.0
    outer = np.full(rows, 0.25, np.float32)
    xh = orc.nvfp4_dequantize(codes, sf, outer).astype(np.float64)
    for seed in (0, 1, 99):
        oc, oe = orc.mxfp8_requant_transpose_sr(codes, sf, outer, 1, seed, 0)
        back = orc.mxfp8_dequantize(oc, oe)
        assert np.array_equal(back, xh.T)


def test_requant_rne_regrouping_changes_values_but_sr_keeps_them_in_expectation(orc):
    # ai-primer "Stochastic rounding across transposes": transposing changes
    # which values share a scale, so independent re-quantisation changes the
    # represented values; stochastic re-quantisation keeps them in expectation.
    x = _rand_rows(orc, 64, 64, seed=14)
    codes, sf, outer = orc.nvfp4_quantize(x)
    xh = orc.nvfp4_dequantize(codes, sf, outer).astype(np.float64).T      # [cols, rows]
    # deterministic RNE of the regrouped values
    rne_codes, rne_e8 = orc.mxfp8_quantize_rows(orc.f32_to_bf16(xh.astype(np.float32)))
    xh_bf = orc.bf16_to_f32(orc.f32_to_bf16(xh.astype(np.float32))).astype(np.float64)
    assert np.count_nonzero(orc.mxfp8_dequantize(rne_codes, rne_e8) != xh_bf) > 0
    n = 128
    acc = np.zeros_like(xh)
    acc2 = np.zeros_like(xh)
    for stream in range(n):
        oc, oe = orc.mxfp8_requant_transpose_sr(codes, sf, outer, 1, seed=5, stream=stream, R=16)
        v = orc.mxfp8_dequantize(oc, oe)
        acc += v
        acc2 += v * v
    mean = acc / n
    # Each draw is lo or lo+q, so its standard deviation is at most q/2 with q
    # the element's own quantum 2^(max(floor(log2|y|)-3, -9) + e), y = xh*2^-e.
    e = np.array([[orc.e8m0_exponent(np.abs(xh[c, b * 32:(b + 1) * 32]).max()) for b in range(2)]
                  for c in range(64)]).repeat(32, axis=1)
    y = np.abs(xh) * 2.0 ** -e
    fl = np.floor(np.log2(np.where(y > 0, y, 1.0)))
    q = 2.0 ** (np.maximum(fl - 3, -9) + e)
    tol = 6 * (q / 2) / np.sqrt(n) + q * 2.0 ** -16
    assert np.all(np.abs(mean - xh) <= tol)
    # and the average error is far below one quantum (no systematic drift)
    assert abs(np.sum(mean - xh)) <= 6 * np.sqrt(np.sum((q / 2) ** 2) / n) + np.sum(q) * 2.0 ** -16


def test_requant_exact_expectation_by_enumerating_u(orc):
    # For one element the result over all 2^R values of u has the exact mean
    # lo + q*floor(frac*2^R)/2^R (checked on the E4M3 grid with R = 8).
    x = _rand_rows(orc, 32, 16, seed=15)
    codes, sf, outer = orc.nvfp4_quantize(x)
    xh = orc.nvfp4_dequantize(codes, sf, outer).astype(np.float64)
    col = xh[:, 3]
    e = orc.e8m0_exponent(np.abs(col).max())
    e4 = np.abs(np.arange(0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64))
    for t in range(32):
        y = col[t] * 2.0 ** -e
        vals = np.array([orc.sr_value(y, u, 8, 3, -9) for u in range(256)])
        lo = e4[e4 <= abs(y)].max()
        hi = e4[e4 >= abs(y)].min()
        if lo == hi:
            assert np.all(np.abs(vals) == abs(y))
        else:
            q = hi - lo
            assert np.abs(vals).mean() == lo + q * np.floor((abs(y) - lo) / q * 256) / 256


def test_requant_per_expert_outer_for_weights(orc):
    E, N, K = 2, 32, 64
    w = _rand_rows(orc, E * N, K, seed=16, heavy=False)
    codes, sf, outer = orc.nvfp4_quantize(w, group_rows=N)
    oc, oe = orc.mxfp8_requant_transpose_sr(codes, sf, outer, N, seed=1, stream=2)
    xh = orc.nvfp4_dequantize(codes, sf, outer, group_rows=N).astype(np.float64)
    back = orc.mxfp8_dequantize(oc, oe)
    # each dequantised value lies between its two neighbouring grid points:
    # |back - xh| is below one quantum of the element's block
    q = 2.0 ** (oe.astype(np.int64) - 127 + 5).repeat(32, axis=1)
    assert np.all(np.abs(back - xh.T) <= q)


def test_requant_entry_matches_the_full_call(orc):
    # the single-entry form used for sampled checks at full size equals the
    # full requantisation, per-token and per-expert outer scales, R = 8 and 16
    for group_rows, R in ((1, 16), (128, 8)):
        rows, cols = 256, 96
        x = _rand_rows(orc, rows, cols, seed=11 + R)
        codes, sf, outer = orc.nvfp4_quantize(x, group_rows=group_rows)
        full_c, full_e = orc.mxfp8_requant_transpose_sr(codes, sf, outer, group_rows, seed=5, stream=9, R=R)
        per_row = np.repeat(outer, group_rows).astype(np.float32)
        rng = np.random.default_rng(R)
        for _ in range(200):
            col, r = int(rng.integers(cols)), int(rng.integers(rows))
            row0, t = r - r % 32, r % 32
            code, e8 = orc.mxfp8_requant_entry(codes[row0:row0 + 32], sf[row0:row0 + 32], per_row[row0:row0 + 32],
                                               col, t, rows, row0, 5, 9, R)
            assert code == full_c[col, r] and e8 == full_e[col, r // 32]
