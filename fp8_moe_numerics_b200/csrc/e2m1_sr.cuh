// e2m1_sr.cuh -- stochastic rounding onto the E2M1 grid (the four-bit
// backward's codes), shared by the NVFP4 quantisers.
//
// [ai-primer §NVFP4 forward, MXFP8 backward]: four bits in the backward pass
// is being explored; the rule taken here moves the MXFP8 recipe's stochastic
// rounding onto the E2M1 grid: with q the grid step at |y| and u the R-bit
// random integer of the element, |y| rounds up iff u < floor(frac(|y| / q) *
// 2^R); values past 6 saturate; the sign of y is kept, also on a zero.
#pragma once

#include "mx_common.cuh"

namespace {

// |E2M1 code| -> value (exact): 0, 0.5, 1, 1.5, 2, 3, 4, 6.
__device__ __forceinline__ float e2m1_mag(uint32_t m) {
    const uint32_t e = (m >> 1) & 3, f = m & 1;
    return e == 0 ? 0.5f * (float)f : __uint_as_float(((e + 126) << 23) | (f << 22));
}

// 2^n for -126 <= n <= 127 (exact).
__device__ __forceinline__ float pow2f(int n) { return __uint_as_float((uint32_t)(n + 127) << 23); }

// |y| rounded stochastically onto the E2M1 magnitudes with the R-bit random
// integer u: the grid step at |y| is q = 2^max(floor(log2 |y|) - 1, -1); |y|
// goes to lo = floor(|y| / q) q or lo + q, up iff u < floor(frac * 2^R) with
// frac = (|y| - lo) / q.  Every step is exact in fp32; the result is a grid
// magnitude, or 8 and above (saturated to 6 by the encoding).
template <int R>
__device__ __forceinline__ float e2m1_sr_magnitude(float y, uint32_t u) {
    const float ay = fabsf(y);
    if (ay == 0.0f) return 0.0f;
    const int fl = (int)((__float_as_uint(ay) >> 23) & 0xff) - 127;        // floor(log2 ay); -127 if subnormal
    const int Q = max(fl - 1, -1);
    const float inv_q = pow2f(-Q), q = pow2f(Q);
    const float lo = __fmul_rn(floorf(__fmul_rn(ay, inv_q)), q);
    const float frac = __fmul_rn(__fsub_rn(ay, lo), inv_q);
    const float thr = floorf(__fmul_rn(frac, (float)(1ull << R)));         // integer in [0, 2^R)
    return ((unsigned long long)u < __float2ull_rz(thr)) ? __fadd_rn(lo, q) : lo;
}

// Hardware stochastic rounding onto E2M1: sm_100a cvt.rs.satfinite.e2m1x4.f32
// d, {a, b, c, f}, rbits puts f's code in bits 3:0 of d and b's in bits 11:8.
// f adds the 16-bit random value rbits[23:16]:rbits[7:0], b the value
// rbits[31:24]:rbits[15:8], just below the kept E2M1 bit, and truncates (the
// carry rounds up).  With u the element's 16-bit integer, feeding 0xFFFF - u
// rounds up exactly when u < floor(frac * 2^16): the rule of
// e2m1_sr_magnitude<16>, signs and saturation included (established by
// comparing the instruction with the oracle on a B200).  a and c share b's and
// f's random bits and are not used.
// Two elements: y_even in f, y_odd in b; codes y_even | y_odd << 8.
__device__ __forceinline__ uint32_t cvt_rs_e2m1_pair(float y_even, float y_odd, uint32_t rbits) {
    uint16_t d;
    asm("cvt.rs.satfinite.e2m1x4.f32 %0, {%1, %2, %3, %4}, %5;"
        : "=h"(d) : "f"(0.0f), "f"(y_odd), "f"(0.0f), "f"(y_even), "r"(rbits));
    return d;
}
// rbits for elements 2k, 2k+1 whose 16-bit integers are the low and high
// halves of word w (R = 16).
__device__ __forceinline__ uint32_t rbits16_pair(uint32_t w) { return __byte_perm(~w, 0u, 0x3120); }
// R = 8: element j's 8-bit integer u enters as the 16-bit value (255 - u) << 8,
// which rounds up iff 256 u + 255 < floor(frac 2^16), i.e. iff u < floor(frac
// 2^8): the R = 8 rule.  Elements 4k .. 4k + 3 are the bytes of word w; h = 0
// takes the pair 4k, 4k + 1, h = 1 the pair 4k + 2, 4k + 3.
__device__ __forceinline__ uint32_t rbits8_pair(uint32_t w, int h) {
    return __byte_perm(~w, 0u, h ? 0x3244 : 0x1044);
}
// Eight code bytes from eight pair results (element 2j in the low nibble of byte j).
__device__ __forceinline__ uint2 pack_e2m1_pairs(const uint32_t d[8]) {
    uint32_t t[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t w = d[2 * k] | (d[2 * k + 1] << 16);     // codes in the low nibbles of bytes 0 .. 3
        t[k] = (w | (w >> 4)) & 0x00ff00ffu;                     // code bytes of the two pairs in bytes 0 and 2
    }
    return make_uint2(__byte_perm(t[0], t[1], 0x6420), __byte_perm(t[2], t[3], 0x6420));
}

// The eight code bytes of 16 scaled values y (element 2j in the low nibble of
// byte j), rounded stochastically with the random integers of linear indices
// L0 .. L0 + 15 (L0 a multiple of 16, so they are the fields of whole Philox
// blocks): R = 16 and 8 on the hardware instruction, R = 32 in exact software.
template <int R>
__device__ __forceinline__ uint2 e2m1_sr_codes(const float* y, uint64_t seed, uint64_t stream_id, uint64_t L0) {
    if constexpr (R == 16) {
        // elements 2k and 2k + 1 take the 16-bit halves of word k % 4 of Philox block k / 4
        uint32_t d[8];
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
            const uint4 rnd = philox4x32_10(L0 / 8 + blk, stream_id, seed);
            const uint32_t w[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
#pragma unroll
            for (int k = 0; k < 4; ++k)
                d[4 * blk + k] = cvt_rs_e2m1_pair(y[8 * blk + 2 * k], y[8 * blk + 2 * k + 1], rbits16_pair(w[k]));
        }
        return pack_e2m1_pairs(d);
    } else if constexpr (R == 8) {
        // one Philox block: elements 4k .. 4k + 3 are the bytes of word k
        const uint4 rnd = philox4x32_10(L0 / 16, stream_id, seed);
        const uint32_t w[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
        uint32_t d[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            d[2 * k] = cvt_rs_e2m1_pair(y[4 * k], y[4 * k + 1], rbits8_pair(w[k], 0));
            d[2 * k + 1] = cvt_rs_e2m1_pair(y[4 * k + 2], y[4 * k + 3], rbits8_pair(w[k], 1));
        }
        return pack_e2m1_pairs(d);
    } else {
        // magnitudes on the grid are encoded exactly; the sign of y is kept,
        // also where the magnitude is zero
        constexpr int kPer = 128 / R;
        uint32_t u[16];
#pragma unroll
        for (int blk = 0; blk < 16 / kPer; ++blk) {
            const uint4 rnd = philox4x32_10(L0 / kPer + blk, stream_id, seed);
#pragma unroll
            for (int f = 0; f < kPer; ++f) u[blk * kPer + f] = philox_field<R>(rnd, f);
        }
        float m[16];
        uint32_t sgn[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            m[i] = e2m1_sr_magnitude<R>(y[i], u[i]);
            sgn[i >> 3] |= (__float_as_uint(y[i]) >> 31) << (4 * (i & 7) + 3);
        }
        return make_uint2(cvt_e2m1x8(m) | sgn[0], cvt_e2m1x8(m + 8) | sgn[1]);
    }
}

}  // namespace
