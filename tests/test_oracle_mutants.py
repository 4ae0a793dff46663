"""The oracle's pins catch planted mistakes.

Each mutant below is one plausible slip in the oracle: a dropped factor, a
wrong sign, a comparison off by one at a boundary, a wrong index or slice, a
swapped operand.  The test copies oracle/ into a temporary directory, plants
one mutant there, and runs the pin tests (tests/test_oracle_*.py) against the
copy in a subprocess; at least one pin must fail.  An unmutated copy must pass
the same pins, so a failure is caused by the planted mistake.  The committed
oracle is never modified.
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.join(ROOT, "tests")
CODECS, QUANT, GEMM, HAD, BWD = ("test_oracle_codecs.py", "test_oracle_quant.py", "test_oracle_gemm_glue.py",
                                 "test_oracle_hadamard.py", "test_oracle_nvfp4_backward.py")

# (what the slip is, file, text, replacement, pin files expected to catch it)
MUTANTS = [
    # oracle.c: codecs, stochastic rounding, Philox, quantisers
    ("E2M1/E4M3 ties go to the odd code", "oracle.c",
     "return (lo & 1) ? hi : lo;", "return (lo & 1) ? lo : hi;", [CODECS]),
    ("E4M3 subnormals decoded one binade low", "oracle.c",
     "return ldexp((double)m, -9);", "return ldexp((double)m, -10);", [CODECS]),
    ("E8M0 exponent: amax exactly 448 * 2^e no longer fits", "oracle.c",
     "int e = (m <= 1.75) ? E - 8 : E - 7;", "int e = (m < 1.75) ? E - 8 : E - 7;", [CODECS]),
    ("stochastic rounding rounds up for u <= threshold", "oracle.c",
     "double r = ((double)u < thr) ? lo + q : lo;", "double r = ((double)u <= thr) ? lo + q : lo;", [CODECS]),
    ("Philox with nine rounds", "oracle.c",
     "for (int round = 0; round < 10; ++round)", "for (int round = 0; round < 9; ++round)", [CODECS]),
    ("Philox bumps the second key word by the first Weyl constant", "oracle.c",
     "k1 += PHILOX_W1;", "k1 += PHILOX_W0;", [CODECS]),
    ("random bits always taken from Philox word 0", "oracle.c",
     "uint32_t word = w[bit / 32];", "uint32_t word = w[0];", [CODECS]),
    ("NVFP4 outer scale without the factor 6", "oracle.c",
     "float s = amax / 2688.0f;", "float s = amax / 448.0f;", [QUANT]),
    ("NVFP4 codes scaled by the block scale only", "oracle.c",
     "float den = orc_e4m3_decode(sc) * s;", "float den = orc_e4m3_decode(sc);", [QUANT]),
    ("dequantisation drops the outer scale", "oracle.c",
     "return nvfp4_block_product(codes, sf, cols, r, c) * outer[r / group_rows];",
     "return nvfp4_block_product(codes, sf, cols, r, c);", [QUANT]),
    ("E4M3 stochastic rounding with two mantissa bits", "oracle.c",
     "double v = orc_sr_value(y, u, R, 3, -9);", "double v = orc_sr_value(y, u, R, 2, -9);", [CODECS]),
    ("E4M3 stochastic rounding with the subnormal step one binade high", "oracle.c",
     "double v = orc_sr_value(y, u, R, 3, -9);", "double v = orc_sr_value(y, u, R, 3, -8);", [CODECS, QUANT]),
    ("Philox multiplies the wrong counter word", "oracle.c",
     "uint64_t p1 = (uint64_t)PHILOX_M1 * c2;", "uint64_t p1 = (uint64_t)PHILOX_M1 * c1;", [CODECS]),
    ("E8M0 decode with bias 128", "oracle.c",
     "return ldexp(1.0, (int)c - 127);", "return ldexp(1.0, (int)c - 128);", [CODECS]),
    ("fp32 -> bf16 rounds ties up", "oracle.c",
     "u += 0x7fffu + lsb;", "u += 0x7fffu;", [CODECS, QUANT]),
    ("NVFP4 packs element 2j in the high nibble", "oracle.c",
     "cb[i / 2] = (uint8_t)(orc_e2m1_encode(v0) | (orc_e2m1_encode(v1) << 4));",
     "cb[i / 2] = (uint8_t)(orc_e2m1_encode(v1) | (orc_e2m1_encode(v0) << 4));", [QUANT]),
    ("NVFP4 block values read the scale of block c/32", "oracle.c",
     "(double)orc_e4m3_decode(sf[r * (cols / 16) + c / 16]);",
     "(double)orc_e4m3_decode(sf[r * (cols / 16) + c / 32]);", [GEMM]),
    ("MXFP8 dequantisation uses each row's first scale", "oracle.c",
     "orc_e8m0_decode(e8m0[r * nb + c / 32]);", "orc_e8m0_decode(e8m0[r * nb]);", [GEMM, QUANT]),
    ("column-wise MXFP8 takes amax over the transposed index", "oracle.c",
     "double a = fabs((double)bf16_to_f32(x[(b * 32 + t) * cols + c]));",
     "double a = fabs((double)bf16_to_f32(x[c * rows + b * 32 + t]));", [QUANT]),
    ("requantisation writes E8M0 with bias 126", "oracle.c",
     "out_e8m0[c * nb + b] = (uint8_t)(e + 127);", "out_e8m0[c * nb + b] = (uint8_t)(e + 126);", [QUANT]),
    ("NVFP4 backward quantiser: block scale of amax / (4s)", "oracle.c",
     "orc_e4m3_encode(bmax / (6.0f * s))", "orc_e4m3_encode(bmax / (4.0f * s))", [BWD]),
    ("NVFP4 backward quantiser ignores the stochastic-rounding flag", "oracle.c",
     "const uint8_t q = sr ? orc_e2m1_sr((double)y, orc_sr_bits(seed, stream, R, L), R)",
     "const uint8_t q = 0 ? orc_e2m1_sr((double)y, orc_sr_bits(seed, stream, R, L), R)", [BWD]),
    ("16x16 tile scale of amax / (3s)", "oracle.c",
     "orc_e4m3_encode(tmax / (6.0f * s))", "orc_e4m3_encode(tmax / (3.0f * s))", [BWD]),
    ("16x16 tile amax over half the tile's columns", "oracle.c",
     "for (int64_t c = tc * 16; c < tc * 16 + 16; ++c)", "for (int64_t c = tc * 16; c < tc * 16 + 8; ++c)", [BWD]),
    # __init__.py: GEMM references and glue
    ("NVFP4 GEMM drops the expert's outer scale", "__init__.py",
     "* a_outer[r0:r1, None].astype(np.float64) * float(b_outer[e])",
     "* a_outer[r0:r1, None].astype(np.float64)", [GEMM]),
    ("DGRAD multiplies every expert by expert 0's weights", "__init__.py",
     "Bv = mxfp8_dequantize(np.ascontiguousarray(b_codes[:, e * Kc:(e + 1) * Kc]),",
     "Bv = mxfp8_dequantize(np.ascontiguousarray(b_codes[:, 0:Kc]),", [GEMM]),
    ("WGRAD reads the first expert's scales for every expert", "__init__.py",
     "np.ascontiguousarray(a_e8[:, t0 // 32:t1 // 32]))", "np.ascontiguousarray(a_e8[:, 0:(t1 - t0) // 32]))",
     [GEMM]),
    ("routing puts an expert's tokens in decreasing order", "__init__.py",
     "    for t in range(T):                          # token order inside each expert",
     "    for t in reversed(range(T)):", [GEMM]),
    ("SwiGLU with gate and up swapped", "__init__.py",
     "a = _silu(h[:, :F]) * h[:, F:]", "a = _silu(h[:, F:]) * h[:, :F]", [GEMM]),
    ("SiLU derivative with a wrong sign", "__init__.py",
     "return s * (1.0 + g * (1.0 - s))", "return s * (1.0 - g * (1.0 - s))", [GEMM]),
    ("ungated activation squares the SiLU input", "__init__.py",
     "        a = _silu(h)\n", "        a = h * _silu(h)\n", [GEMM]),
    ("ungated backward uses SiLU instead of its derivative", "__init__.py",
     "dh = da * _dsilu(h)", "dh = da * _silu(h)", [GEMM]),
    ("combine drops the routing weights", "__init__.py",
     'out = np.einsum("tj,tjd->td", w.astype(np.float64), y[pos])', "out = y[pos].sum(axis=1)", [GEMM]),
    ("combine gradient drops the routing weights", "__init__.py",
     "dy[pos[:, j]] = w[:, j, None].astype(np.float64) * d", "dy[pos[:, j]] = d", [GEMM]),
    ("numpy fp32 -> bf16 rounds ties up", "__init__.py",
     "u = u + 0x7FFF + ((u >> 16) & 1)", "u = u + 0x7FFF", [CODECS, QUANT, GEMM]),
    ("fp64 -> bf16 rounds ties away from zero", "__init__.py",
     "r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)",
     "r = np.ldexp(np.trunc(np.ldexp(m, 8) + np.copysign(0.5, m)), e - 8)", [GEMM]),
    ("expert segments not padded to 128 rows", "__init__.py",
     "padded = (counts + align - 1) // align * align", "padded = counts", [GEMM]),
    ("S2F6 codes may reach -128", "__init__.py",
     "c = np.clip(np.rint(y), -127, 127).astype(np.int8)", "c = np.clip(np.rint(y), -128, 127).astype(np.int8)", [HAD]),
    ("gather takes the block scales of the previous token", "__init__.py",
     "osf[ok] = sf[src[ok]]", "osf[ok] = sf[np.maximum(src[ok] - 1, 0)]", [GEMM]),
    ("gather drops the outer scale", "__init__.py",
     "oo[ok] = outer[src[ok]]", "oo[ok] = 1.0", [GEMM]),
    ("sampled NVFP4 GEMM reads expert 0's weight rows", "__init__.py",
     "b = nvfp4_block_values(b_codes[e * N + n:e * N + n + 1], b_sf[e * N + n:e * N + n + 1])[0]",
     "b = nvfp4_block_values(b_codes[n:n + 1], b_sf[n:n + 1])[0]", [GEMM]),
    ("single requantised entry draws the bits of the wrong index", "__init__.py",
     "L = col * rows + row0 + t", "L = col * rows + t", [QUANT]),
    ("NVFP4 requantisation without the transpose", "__init__.py",
     "return nvfp4_quantize_f32(np.ascontiguousarray(xh.T), 1, sr, seed, stream, R)",
     "return nvfp4_quantize_f32(np.ascontiguousarray(xh.reshape(xh.shape[1], xh.shape[0])), 1, sr, seed, stream, R)",
     [BWD]),
    ("expert weight requantisation stacks untransposed experts", "__init__.py",
     "np.ascontiguousarray(xh.transpose(0, 2, 1).reshape(E * K, N))", "np.ascontiguousarray(xh.reshape(E * K, N))",
     [BWD]),
    ("NVFP4 wgrad drops the second operand's outer scales", "__init__.py",
     "C[e] = (Av[:, t0:t1] @ Bv[:, t0:t1].T) * ao[e][:, None] * bo[e][None, :]",
     "C[e] = (Av[:, t0:t1] @ Bv[:, t0:t1].T) * ao[e][:, None]", [BWD]),
    ("segment outer scales taken over the whole row", "__init__.py",
     "amax = np.abs(xt[:, t0:t1]).max(axis=1) if per_row else np.abs(xt[:, t0:t1]).max()",
     "amax = np.abs(xt).max(axis=1) if per_row else np.abs(xt[:, t0:t1]).max()", [BWD]),
    ("segment blocks take the next segment's scale", "__init__.py",
     "s_blk[:, t0 // 16:t1 // 16] = s[:, None] if per_row else s",
     "s_blk[:, t0 // 16 + 1:t1 // 16 + 1] = s[:, None] if per_row else s", [BWD]),
    ("tile-scaled transpose swaps the nibbles", "__init__.py",
     "return (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)", "return (q[:, 1::2] | (q[:, 0::2] << 4)).astype(np.uint8)",
     [BWD]),
    # __init__.py: Hadamard rotation and S2F6
    ("butterfly difference with the wrong sign", "__init__.py",
     "z = np.stack([a + b, a - b], axis=-2)", "z = np.stack([a + b, b - a], axis=-2)", [HAD]),
    ("S2F6 exponent: amax exactly (127/64) 2^e no longer fits", "__init__.py",
     "e = E1 if m2 <= S2F6_MAX else E1 + 1", "e = E1 if m2 < S2F6_MAX else E1 + 1", [HAD]),
    ("S2F6 codes with seven fractional bits", "__init__.py",
     "y = z.astype(np.float64) * np.ldexp(1.0, 6 - e)[..., None]",
     "y = z.astype(np.float64) * np.ldexp(1.0, 7 - e)[..., None]", [HAD]),
    ("sign mask read from the top bit down", "__init__.py",
     "bits = (words[:, None] >> np.arange(32, dtype=np.uint32)[None, :]) & 1",
     "bits = (words[:, None] >> np.arange(31, -1, -1, dtype=np.uint32)[None, :]) & 1", [HAD]),
    ("inverse rotation divides by 16", "__init__.py",
     "x = (zhat @ H.T).reshape(rows, cols) / 32.0", "x = (zhat @ H.T).reshape(rows, cols) / 16.0", [HAD]),
    ("S2F6 combine drops the routing weights", "__init__.py",
     'out = np.einsum("tj,tjd->td", w.astype(np.float64), xhat[pos])', "out = xhat[pos].sum(axis=1)", [HAD]),
]


def _copy_oracle(dst, mutant=None):
    os.makedirs(os.path.join(dst, "oracle"))
    for f in ("__init__.py", "oracle.c"):
        src = open(os.path.join(ROOT, "oracle", f)).read()
        if mutant is not None and mutant[1] == f:
            _, _, old, new, _ = mutant
            assert src.count(old) == 1, f"mutation site not unique in oracle/{f}: {old!r}"
            src = src.replace(old, new)
        open(os.path.join(dst, "oracle", f), "w").write(src)


def _run_pins(workdir, files):
    # the copy shadows the repository's oracle: it is first on sys.path (the
    # working directory), the repository second (for tests/ and its helpers)
    env = dict(os.environ, PYTHONPATH=ROOT, OMP_NUM_THREADS="1", PYTHONDONTWRITEBYTECODE="1")
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu",
           *[os.path.join(TESTS, f) for f in files]]
    r = subprocess.run(cmd, cwd=workdir, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler for the oracle")
    base = tmp_path_factory.mktemp("mutants")
    jobs = {"control": (None, [CODECS, QUANT, GEMM, HAD, BWD])}
    for i, m in enumerate(MUTANTS):
        jobs[i] = (m, m[4])
    dirs = {}
    for key, (m, _) in jobs.items():
        dirs[key] = str(base / f"m{key}")
        _copy_oracle(dirs[key], m)
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        fut = {key: ex.submit(_run_pins, dirs[key], files) for key, (_, files) in jobs.items()}
        return {key: f.result() for key, f in fut.items()}


def test_unmutated_copy_passes_every_pin(results):
    rc, out = results["control"]
    assert rc == 0, out


@pytest.mark.parametrize("i", range(len(MUTANTS)), ids=[m[0] for m in MUTANTS])
def test_pins_catch_the_planted_mistake(results, i):
    rc, out = results[i]
    assert rc == 1, f"pins did not fail on: {MUTANTS[i][0]} (pytest exit {rc})\n{out}"
