"""Pins of the combine-path oracle: 32-d random Hadamard rotation + S2F6.

[ai-primer §Quantized NVLink and BBBK]: expert outputs are rotated by a
32-dimensional random Hadamard transform and quantised to block-scaled S2F6
(two signed integer bits, six fractional bits) before the combine; the
rotation spreads an outlier's magnitude over the block.  Each pin checks the
oracle against something other than its own formula: the Kronecker-built
Sylvester matrix, H32 H32 = 32 I, a search over every exponent, hand-written
tie cases, the closed form of a one-hot block, the quantisation error bound
and a per-element loop over the combine.
"""
import numpy as np
import pytest

import oracle


def _popcount_hadamard(n):
    return np.array([[(-1.0) ** bin(a & b).count("1") for b in range(n)] for a in range(n)])


def test_butterflies_equal_the_sylvester_matrix_on_integers():
    rng = np.random.default_rng(0)
    x = rng.integers(-1000, 1001, size=(50, 32)).astype(np.float32)    # every partial sum is exact in fp32
    H = _popcount_hadamard(32)
    assert np.array_equal(oracle.sylvester_hadamard(32), H)
    assert np.array_equal(oracle.fwht32_f32(x).astype(np.float64), x.astype(np.float64) @ H.T)


def _sylvester_recursive_f32(x):
    """H_n x from the recursion H_2n = [[H_n, H_n], [H_n, -H_n]], each sum one
    fp32 rounding: H_2n [u; v] = [H_n u + H_n v; H_n u - H_n v]."""
    n = x.shape[-1]
    if n == 1:
        return x.astype(np.float32)
    u = _sylvester_recursive_f32(x[..., : n // 2])
    v = _sylvester_recursive_f32(x[..., n // 2:])
    return np.concatenate([np.float32(u + v), np.float32(u - v)], axis=-1)


def test_fp32_order_is_the_sylvester_recursion():
    """Reading R20 (evaluation order): on general fp32 inputs, where the order
    of the roundings shows, the butterflies give bit for bit the fp32
    evaluation of the Sylvester recursion that defines H32, and stay within
    the five-rounding error bound of the exact product."""
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((400, 32)) * 10.0 ** rng.uniform(-3, 3, (400, 1))).astype(np.float32)
    got = oracle.fwht32_f32(x)
    assert np.array_equal(got.view(np.uint32), _sylvester_recursive_f32(x).view(np.uint32))
    exact = x.astype(np.float64) @ _popcount_hadamard(32).T
    bound = 5 * 2.0 ** -24 * np.abs(x).astype(np.float64).sum(axis=-1, keepdims=True) * 1.0001
    assert np.all(np.abs(got - exact) <= bound)
    # a different order (h = 16 first) differs somewhere on these inputs: the pin has teeth
    z = x.copy()
    for h in (16, 8, 4, 2, 1):
        z = z.reshape(400, 32 // (2 * h), 2, h)
        z = np.stack([z[:, :, 0] + z[:, :, 1], z[:, :, 0] - z[:, :, 1]], axis=2).reshape(400, 32)
    assert not np.array_equal(z.view(np.uint32), got.view(np.uint32))


def test_transform_applied_twice_is_32_times_identity():
    rng = np.random.default_rng(1)
    x = rng.integers(-300, 301, size=(20, 32)).astype(np.float32)
    assert np.array_equal(oracle.fwht32_f32(oracle.fwht32_f32(x)), 32.0 * x)


def test_sign_masks_are_balanced_and_keyed():
    w = oracle.hadamard_sign_words(7, 3, 512)
    ones = sum(bin(int(v)).count("1") for v in w)
    assert abs(ones / (512 * 32) - 0.5) < 0.02
    assert len(set(w.tolist())) == 512
    assert not np.array_equal(w, oracle.hadamard_sign_words(8, 3, 512))
    assert not np.array_equal(w, oracle.hadamard_sign_words(7, 4, 512))
    s = oracle.hadamard_signs(7, 3, 64)
    assert set(np.unique(s)) <= {-1.0, 1.0} and s.shape == (64,)
    assert s[0] == (-1.0 if w[0] & 1 else 1.0) and s[33] == (-1.0 if (w[1] >> 1) & 1 else 1.0)


def _exponent_by_search(amax):
    if amax == 0.0:
        return -127
    for e in range(-127, 128):
        if amax <= (127.0 / 64.0) * 2.0 ** e:
            return e
    return 127


@pytest.mark.parametrize("amax", [0.0, 1.0, 127 / 64, np.nextafter(np.float32(127 / 64), np.float32(2)), 2.0, 1.9,
                                  3.0, 127 / 32, 0.75, 1e-30, 1e-40, 2.0 ** -149, 2.0 ** -126, 1e20, 3.0e38,
                                  float(np.finfo(np.float32).max)])
def test_exponent_is_the_smallest_that_fits(amax):
    assert oracle.s2f6_exponent(float(np.float32(amax))) == _exponent_by_search(float(np.float32(amax)))


def test_exponent_on_random_magnitudes():
    rng = np.random.default_rng(2)
    for a in (rng.standard_normal(2000) * 10.0 ** rng.uniform(-40, 38, 2000)).astype(np.float32):
        assert oracle.s2f6_exponent(abs(float(a))) == _exponent_by_search(abs(float(a)))


def _block_with_rotated_values(z, seed, stream):
    """fp32 x (one block) whose rotation is exactly z (z dyadic, small)."""
    sig = oracle.hadamard_signs(seed, stream, 32)
    x = (oracle.sylvester_hadamard(32) @ np.asarray(z, np.float64)) / 32.0 * sig
    assert np.array_equal(x.astype(np.float32).astype(np.float64), x)
    return x.astype(np.float32)[None, :]


def test_codes_round_half_to_even():
    # amax 127/64 gives e = 0, so a code is z * 64; half codes are ties
    z = np.zeros(32)
    z[0] = 127 / 64
    halves = [0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, 10.5, 11.5, -126.5]
    expect = [0, 2, 2, 4, 0, -2, -2, 10, 12, -126]
    z[1:1 + len(halves)] = np.array(halves) / 64
    x = _block_with_rotated_values(z, 5, 9)
    assert np.array_equal(oracle.fwht32_f32(x * oracle.hadamard_signs(5, 9, 32).astype(np.float32)), z[None, :])
    c, e = oracle.s2f6_quantize_hadamard(x, 5, 9)
    assert e[0, 0] == 127
    assert c[0, 0] == 127
    assert c[0, 1:1 + len(halves)].tolist() == expect
    assert np.all(c[0, 1 + len(halves):] == 0)


def test_one_hot_outlier_spreads_to_every_coordinate():
    # a single value A in a block rotates to +-A in all 32 coordinates
    for A in (1.0, 3.0, 1000.0, 7.3e-5):
        x = np.zeros((1, 64), np.float32)
        x[0, 40] = A
        c, e = oracle.s2f6_quantize_hadamard(x, 11, 0)
        eb = oracle.s2f6_exponent(float(np.float32(A)))
        assert e[0, 1] == eb + 127 and e[0, 0] == 0              # block 0 is zero: e = -127
        mag = np.rint(float(np.float32(A)) * 2.0 ** (6 - eb))
        assert np.all(np.abs(c[0, 32:].astype(np.float64)) == mag)
        assert np.all(c[0, :32] == 0)


def test_top_exponent_saturates_codes():
    # a one-hot block of the largest fp32 value rotates to |z| = (2 - 2^-23) 2^127
    # in every coordinate: e would be 128, clamps to 127, and 127.99... -> 127
    x = np.zeros((1, 32), np.float32)
    x[0, 3] = np.finfo(np.float32).max
    c, e = oracle.s2f6_quantize_hadamard(x, 0, 0)
    assert e[0, 0] == 127 + 127
    assert np.all(np.abs(c.astype(np.int64)) == 127)


def test_reconstruction_error_bound():
    rng = np.random.default_rng(3)
    rows, cols = 64, 256
    x = (rng.standard_t(3, (rows, cols)) * 10.0 ** rng.uniform(-3, 3, (rows, 1))).astype(np.float32)
    x[5, 17] = 5e4                                              # an outlier
    x[9] = 0
    c, e = oracle.s2f6_quantize_hadamard(x, 21, 4)
    xh = oracle.s2f6_dequantize_hadamard(c, e, 21, 4)
    err = np.linalg.norm((xh - x.astype(np.float64)).reshape(rows, cols // 32, 32), axis=-1)
    nrm = np.linalg.norm(x.astype(np.float64).reshape(rows, cols // 32, 32), axis=-1)
    step_half = np.ldexp(1.0, e.astype(np.int64) - 127 - 7)
    # per block: |zhat - z| <= half a code step in each of 32 coordinates, and
    # the inverse divides the 2-norm by sqrt(32); fp32 butterflies add < 1e-6
    assert np.all(err <= step_half + 1e-6 * nrm)
    assert np.all(xh[9] == 0)


def test_combine_matches_element_loops():
    rng = np.random.default_rng(4)
    M, D, T, k = 12, 64, 5, 3
    x = rng.standard_normal((M, D)).astype(np.float32)
    c, e = oracle.s2f6_quantize_hadamard(x, 2, 6)
    pos = rng.integers(0, M, size=(T, k)).astype(np.int32)
    w = rng.uniform(0, 1, size=(T, k)).astype(np.float32)
    words = oracle.hadamard_sign_words(2, 6, D // 32)
    want = np.zeros((T, D))
    for t in range(T):
        for j in range(k):
            r = pos[t, j]
            for d in range(D):
                blk, i = divmod(d, 32)
                acc = 0.0
                for b in range(32):
                    zhat = float(c[r, 32 * blk + b]) * 2.0 ** (int(e[r, blk]) - 127 - 6)
                    acc += (-1.0) ** bin(i & b).count("1") * zhat
                sign = -1.0 if (int(words[blk]) >> i) & 1 else 1.0
                want[t, d] += float(w[t, j]) * sign * acc / 32.0
    got = oracle.bf16_to_f32(oracle.combine_s2f6(c, e, pos, w, 2, 6)).astype(np.float64)
    assert np.array_equal(oracle.f64_to_bf16(want), oracle.combine_s2f6(c, e, pos, w, 2, 6))
    assert np.allclose(got, want, rtol=1e-2, atol=1e-6)
