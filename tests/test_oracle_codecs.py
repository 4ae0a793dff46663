"""Pins for the oracle's element codecs, rounding rules and random stream.

Each check compares the oracle with something other than itself: closed
forms, the ml_dtypes package's independent float4/float8 conversions, Triton's
independent Philox4x32-10 (run on the CPU by its interpreter), exhaustive
enumeration, and the numbers the pages print (tests/golden/pages_worked_examples.json,
each with its page and section).
"""
import json
import os
import subprocess
import sys
import textwrap

import ml_dtypes
import numpy as np
import pytest


def test_f32_to_bf16_matches_ml_dtypes_on_ties(orc):
    # exact ties (dropped half 0x8000) above even and odd kept bits, their
    # neighbours, values that overflow to infinity, and random finite patterns;
    # ml_dtypes' bfloat16 conversion rounds to nearest even independently
    rng = np.random.default_rng(31)
    hi = rng.integers(0, 0x7F7F, 4000, dtype=np.uint32)
    sign = rng.integers(0, 2, 4000, dtype=np.uint32) << 31
    pats = [(hi << 16) | d | sign for d in (0x8000, 0x7FFF, 0x8001, 0x0000, 0xFFFF)]
    pats.append(np.array([0x7F7FFFFF, 0x7F7F8000, 0x7F7F7FFF, 0xFF7FFFFF, 0x00008000, 0x00018000,
                          0x80008000], dtype=np.uint32))
    finite = rng.integers(0, 0xFFFFFFFF, 20000, dtype=np.uint64, endpoint=True).astype(np.uint32)
    pats.append(finite[(finite & 0x7F800000) != 0x7F800000])
    x = np.concatenate(pats).view(np.float32)
    want = x.astype(ml_dtypes.bfloat16).view(np.uint16)
    assert np.array_equal(orc.f32_to_bf16(x), want)
    lib = orc.lib()
    got_c = np.array([lib.orc_f32_to_bf16(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(got_c, want)


def test_e2m1_decode_table_closed_form_and_ml_dtypes(orc):
    t = orc.e2m1_decode_table()
    expect = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=np.float32)
    assert np.array_equal(t[:8], expect)
    assert np.array_equal(t[8:], -expect)
    assert np.signbit(t[8])                      # code 0x8 is -0
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float32)
    assert np.array_equal(t, lib)


def test_e4m3_decode_table_closed_form_and_ml_dtypes(orc):
    t = orc.e4m3_decode_table()
    codes = np.arange(256, dtype=np.uint8)
    lib = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float32)
    nan = (codes & 0x7F) == 0x7F
    assert np.all(np.isnan(t[nan])) and np.all(np.isnan(lib[nan]))
    assert np.array_equal(t[~nan], lib[~nan])
    assert t[0x7E] == 448.0 and t[0x01] == 2.0 ** -9 and t[0x08] == 2.0 ** -6
    # closed form: e=0 -> m/8 * 2^-6, else (1+m/8) * 2^(e-7)
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        v = m / 8 * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        assert t[c] == v and t[c | 0x80] == -v


def test_e8m0_decode_table(orc):
    t = orc.e8m0_decode_table()
    assert np.isnan(t[255])
    assert np.array_equal(t[:255], 2.0 ** (np.arange(255) - 127.0))
    lib = np.arange(255, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    assert np.array_equal(t[:255], lib)


def _probe_values():
    """Every finite bf16 value, plus fp32 values with random low mantissa bits
    and all exact midpoints of the E2M1/E4M3 grids."""
    allbf = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    allbf = allbf[np.isfinite(allbf)]
    rng = np.random.default_rng(7)
    noisy = (allbf.view(np.uint32) | rng.integers(0, 1 << 16, allbf.size, dtype=np.uint32)).view(np.float32)
    e2 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    e4 = np.unique(np.abs(np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)))
    e4 = e4[np.isfinite(e4)]
    mids = np.concatenate([(e2[1:] + e2[:-1]) / 2, (e4[1:] + e4[:-1]) / 2]).astype(np.float32)
    v = np.concatenate([allbf, noisy, mids, -mids])
    return v[np.isfinite(v)]


def test_e2m1_encode_matches_ml_dtypes_rne(orc):
    v = _probe_values()
    got = orc.e2m1_encode(v)
    ref = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8)   # RNE, saturating
    assert np.array_equal(got, ref)


def test_e4m3_encode_matches_ml_dtypes_rne_and_saturates(orc):
    v = _probe_values()
    inrange = np.abs(v) <= 464.0                 # ml_dtypes turns larger values into NaN
    got = orc.e4m3_encode(v)
    ref = v[inrange].astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(got[inrange], ref)
    big = v[~inrange]
    assert np.all((got[~inrange] & 0x7F) == 0x7E)                 # satfinite: +-448
    assert np.array_equal(got[~inrange] >> 7, np.signbit(big).astype(np.uint8))


def test_negative_values_that_round_to_zero_keep_sign(orc):
    assert orc.e2m1_encode(np.array([-0.2], np.float32))[0] == 0x8
    assert orc.e4m3_encode(np.array([-1e-6], np.float32))[0] == 0x80
    assert orc.e4m3_encode(np.array([0.0], np.float32))[0] == 0x00


def _pages(name):
    """A worked example as the pages print it (tests/golden, with its citation)."""
    with open(os.path.join(os.path.dirname(__file__), "golden", "pages_worked_examples.json")) as f:
        return json.load(f)[name]


def test_toy_round_to_nearest_example(orc):
    # aibuzzwire "Why Fewer Bits Means Faster Training": a format holding only
    # 3 and 4 stores 3.2 as 3, an error of 0.2.
    ex = _pages("round_to_nearest_toy")
    r = orc.round_nearest_on_grid(ex["value"], ex["grid"])
    assert r == ex["stored"]
    assert abs((ex["value"] - r) - ex["error"]) < 1e-12


def test_bits_per_value_of_the_formats(orc):
    # ai-primer "Block scales and per-token activations" table:
    # BF16 16, MXFP8 8.25, NVFP4 4.5 bits per value including block scales;
    # aibuzzwire "Three Formats": NVFP4 stores 3.6x fewer bits than BF16.
    bits = _pages("bits_per_value")
    rows, cols = 8, 256
    x = orc.f32_to_bf16(np.random.default_rng(0).standard_normal((rows, cols)).astype(np.float32))
    codes, sf, outer = orc.nvfp4_quantize(x)
    assert sf.shape[1] * _pages("nvfp4_block")["values_per_scale"] == cols
    nvfp4_bits = 8 * (codes.nbytes + sf.nbytes) / x.size
    assert nvfp4_bits == bits["nvfp4"]
    c8, e8 = orc.mxfp8_quantize_rows(x)
    assert 8 * (c8.nbytes + e8.nbytes) / x.size == bits["mxfp8"]
    assert 8 * x.nbytes / x.size == bits["bf16"]
    assert round(bits["bf16"] / nvfp4_bits, 1) == bits["bf16_over_nvfp4"]


# --------------------------------------------------------------------------
# Stochastic rounding
# --------------------------------------------------------------------------

@pytest.mark.parametrize("R", [8, 16])
def test_worked_example_4_5_on_fp4_grid(orc, R):
    # ai-primer "Stochastic rounding across transposes": a represented 4.5
    # becomes 4 with probability 0.75 and 6 with probability 0.25, so its
    # expectation stays 4.5.  Enumerate every R-bit random value.
    ex = _pages("stochastic_rounding_example")
    vals = np.array([orc.sr_value(ex["value"], u, R, 1, -1) for u in range(1 << R)])
    assert set(np.unique(vals)) == {v for v, _ in ex["outcomes"]}
    for v, p in ex["outcomes"]:
        assert np.count_nonzero(vals == v) == p * (1 << R)
    assert vals.mean() == ex["expectation"]
    codes = {orc.e2m1_sr(4.5, u, R) for u in range(1 << R)}
    assert codes == {0x6, 0x7}                   # E2M1 codes of 4 and 6
    neg = np.array([orc.sr_value(-4.5, u, R, 1, -1) for u in range(0, 1 << R, 7)])
    assert set(np.unique(neg)) <= {-4.0, -6.0}


def test_worked_example_fraction_with_32_bit_draws(orc):
    # R = 32 cannot be enumerated; the decision is u < floor(frac * 2^32)
    # with frac = 0.25 for 4.5 between 4 and 6.
    t = 1 << 30
    assert orc.sr_value(4.5, t - 1, 32, 1, -1) == 6.0
    assert orc.sr_value(4.5, t, 32, 1, -1) == 4.0


@pytest.mark.parametrize("R", [8, 16])
def test_sr_exact_mean_and_bias_bound_on_e4m3_grid(orc, R):
    rng = np.random.default_rng(1)
    e4 = np.abs(np.arange(0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64))
    ys = np.concatenate([rng.uniform(0, 448, 12), rng.uniform(0, 2.0 ** -6, 6), [2.0 ** -10, 447.9, 3.3e-3]])
    for y in ys:
        y = float(np.float32(y))
        lo = e4[e4 <= y].max()
        hi = e4[e4 >= y].min()
        us = range(0, 1 << R) if R == 8 else range(0, 1 << R, 1)
        vals = np.array([orc.sr_value(y, u, R, 3, -9) for u in us])
        assert set(np.unique(vals)) <= {lo, hi}
        if hi == lo:
            assert np.all(vals == y)
            continue
        q = hi - lo
        frac = (y - lo) / q
        assert vals.mean() == lo + q * np.floor(frac * 2 ** R) / 2 ** R
        assert 0 <= y - vals.mean() < q * 2.0 ** -R
        for u in (0, (1 << R) - 1):
            code = orc.e4m3_sr(y, u, R)
            assert orc.e4m3_decode_table()[code] == orc.sr_value(y, u, R, 3, -9)


def test_e8m0_exponent_brute_force_definition(orc):
    # Reading: e is the smallest integer with amax <= 448 * 2^e, in [-127, 127].
    rng = np.random.default_rng(2)
    mags = np.concatenate([
        np.float32(rng.uniform(1, 2, 200)) * np.float32(2.0) ** rng.integers(-140, 120, 200).astype(np.float32),
        np.array([448.0, 448.0 * 1.0000001, 447.99997, 1.75, 1.7500001, 3.5, 2.0 ** -149, 2.0 ** -130], np.float32),
    ]).astype(np.float64)
    mags = mags[(mags > 0) & np.isfinite(mags)]
    for a in mags:
        e = -127
        while e < 127 and not (a <= 448.0 * 2.0 ** e):
            e += 1
        assert orc.e8m0_exponent(a) == e, a
    assert orc.e8m0_exponent(0.0) == -127


# --------------------------------------------------------------------------
# Philox4x32-10 against Triton's implementation (independent code, run on the
# CPU by the Triton interpreter in a subprocess).
# --------------------------------------------------------------------------

_TRITON_SCRIPT = textwrap.dedent(
    """
    import os, sys, json
    os.environ["TRITON_INTERPRET"] = "1"
    import torch, triton, triton.language as tl
    from triton.language.random import philox_impl

    @triton.jit
    def k(ctr_ptr, key_ptr, out_ptr, N: tl.constexpr):
        i = tl.arange(0, N)
        c0 = tl.load(ctr_ptr + i * 4 + 0).to(tl.uint32, bitcast=True)
        c1 = tl.load(ctr_ptr + i * 4 + 1).to(tl.uint32, bitcast=True)
        c2 = tl.load(ctr_ptr + i * 4 + 2).to(tl.uint32, bitcast=True)
        c3 = tl.load(ctr_ptr + i * 4 + 3).to(tl.uint32, bitcast=True)
        k0 = tl.load(key_ptr + i * 2 + 0).to(tl.uint32, bitcast=True)
        k1 = tl.load(key_ptr + i * 2 + 1).to(tl.uint32, bitcast=True)
        a, b, c, d = philox_impl(c0, c1, c2, c3, k0, k1, 10)
        tl.store(out_ptr + i * 4 + 0, a.to(tl.int32, bitcast=True))
        tl.store(out_ptr + i * 4 + 1, b.to(tl.int32, bitcast=True))
        tl.store(out_ptr + i * 4 + 2, c.to(tl.int32, bitcast=True))
        tl.store(out_ptr + i * 4 + 3, d.to(tl.int32, bitcast=True))

    data = json.loads(sys.stdin.read())
    n = len(data["ctr"])
    ctr = torch.tensor(data["ctr"], dtype=torch.int64).to(torch.int32)
    key = torch.tensor(data["key"], dtype=torch.int64).to(torch.int32)
    out = torch.zeros(n * 4, dtype=torch.int32)
    k[(1,)](ctr, key, out, n)
    print(json.dumps([x & 0xffffffff for x in out.tolist()]))
    """
)


def test_philox_matches_triton_reference_implementation(orc):
    import json
    rng = np.random.default_rng(3)
    n = 16
    ctr = rng.integers(0, 2 ** 32, (n, 4), dtype=np.uint64)
    key = rng.integers(0, 2 ** 32, (n, 2), dtype=np.uint64)
    ctr[0] = 0
    key[0] = 0
    ctr[1] = 0xFFFFFFFF
    key[1] = 0xFFFFFFFF
    payload = json.dumps({"ctr": [[int(v) - (1 << 32) if v >= 1 << 31 else int(v) for v in r] for r in ctr],
                          "key": [[int(v) - (1 << 32) if v >= 1 << 31 else int(v) for v in r] for r in key]})
    env = dict(os.environ, TRITON_INTERPRET="1", CUDA_VISIBLE_DEVICES="")
    res = subprocess.run([sys.executable, "-c", _TRITON_SCRIPT], input=payload, capture_output=True,
                         text=True, env=env, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    ref = np.array(json.loads(res.stdout.strip().splitlines()[-1]), dtype=np.uint64).reshape(n, 4)
    for i in range(n):
        got = orc.philox4x32_10(ctr[i].astype(np.uint32), key[i].astype(np.uint32))
        assert np.array_equal(got.astype(np.uint64), ref[i]), i


def test_sr_bits_stream_layout(orc):
    # Element L takes R bits of Philox block L // (128/R); counter (g, stream),
    # key = seed.  Checked against direct generator calls.
    seed, stream = 0x1234_5678_9ABC_DEF0, 0xAB
    for R in (8, 16, 32):
        per = 128 // R
        for L in (0, 1, per - 1, per, 5 * per + 3, (1 << 33) + 7):
            g, j = divmod(L, per)
            w = orc.philox4x32_10([g & 0xFFFFFFFF, g >> 32, stream & 0xFFFFFFFF, stream >> 32],
                                  [seed & 0xFFFFFFFF, seed >> 32])
            bit = j * R
            expect = (int(w[bit // 32]) >> (bit % 32)) & ((1 << R) - 1)
            assert orc.sr_bits(seed, stream, R, L) == expect


def test_sr_bits_are_uniform(orc):
    # byte histogram of the R=8 stream: chi-square with 255 dof
    vals = np.array([orc.sr_bits(0, 0, 8, L) for L in range(1 << 16)])
    hist = np.bincount(vals, minlength=256)
    exp = vals.size / 256
    chi2 = ((hist - exp) ** 2 / exp).sum()
    assert chi2 < 255 + 6 * np.sqrt(2 * 255)
