// nvfp4_bwd.cu -- NVFP4 in the backward pass and the 16x16 shared-scale
// format (sm_100a).
//
// [ai-primer §NVFP4 forward, MXFP8 backward]: four-bit arithmetic in the
// backward pass is the lab's stated future work.  [ai-primer §Stochastic
// rounding across transposes]: a scale shared by each 16x16 tile was tried
// and rejected (one large value can force the tile's other values to zero).
//
// Readings taken where the pages are silent (the header states them in full):
//   - the forward quantiser's scale rules (outer s = amax / (6*448) per group
//     of rows, E4M3 block scale of amax_b / (6 s) per 16 values, to nearest);
//   - E2M1 element codes rounded stochastically: with q the grid step at |y|
//     and u the random integer of the element, round up iff
//     u < floor(frac(|y| / q) * 2^R); values past 6 saturate;
//   - the requantisation across the transpose gives the transposed tensor one
//     outer scale per row (or per expert for a weight stack), so that both
//     outer scales of every backward GEMM factor out of its contraction.
//
// Every step is one IEEE fp32 round-to-nearest operation in the order the
// oracle takes them; the stochastic rounding is done in software, exactly.
#include <type_traits>

#include "mx_common.cuh"

namespace {

constexpr int kThreads = 256;
constexpr float kOuterDiv = 2688.0f;              // 6 * 448

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

// Random integer of output element L (Philox4x32-10, counter (L / (128/R),
// stream), key seed; field L mod (128/R)).
template <int R>
__device__ __forceinline__ uint32_t sr_bits_at(uint64_t seed, uint64_t stream_id, uint64_t L) {
    constexpr int kPer = 128 / R;
    return philox_field<R>(philox4x32_10(L / kPer, stream_id, seed), (int)(L % kPer));
}

// One 16-value block: E4M3 scale of bmax / (6 s) (0 when s == 0) and the
// eight code bytes, element 2j in the low nibble of byte j.  L0 is the linear
// output index of element 0 (for the random integers).
template <int R, bool kSR>
__device__ __forceinline__ void quantize_block16(const float* v, float s, uint64_t seed, uint64_t stream_id,
                                                 uint64_t L0, uint32_t& scode, uint2& packed) {
    float bmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
    scode = s > 0.0f ? (cvt_e4m3x2(__fdiv_rn(bmax, __fmul_rn(6.0f, s)), 0.0f) & 0xffu) : 0u;
    packed = make_uint2(0u, 0u);
    if (scode == 0) return;
    const float inv = __fdiv_rn(1.0f, __fmul_rn(e4m3_to_f32(scode), s));
    float y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(v[i], inv);
    if constexpr (!kSR) {
        packed.x = cvt_e2m1x8(y);
        packed.y = cvt_e2m1x8(y + 8);
    } else {
        // magnitudes on the grid are encoded exactly; the sign of y is kept,
        // also where the magnitude is zero
        float m[16];
        uint32_t sgn[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            m[i] = e2m1_sr_magnitude<R>(y[i], sr_bits_at<R>(seed, stream_id, L0 + i));
            sgn[i >> 3] |= (__float_as_uint(y[i]) >> 31) << (4 * (i & 7) + 3);
        }
        packed = make_uint2(cvt_e2m1x8(m) | sgn[0], cvt_e2m1x8(m + 8) | sgn[1]);
    }
}

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) red[w] = v;
    __syncthreads();
    if (w == 0) {
        v = l < (int)(blockDim.x >> 5) ? red[l] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    }
    return v;                                     // valid in thread 0
}

// outer[g] = amax of group g (group_rows rows of a bf16 [rows, cols]) / 2688.
// One block per group; the group's words are read in 16-byte vectors.
__global__ void __launch_bounds__(kThreads)
group_outer_kernel(const uint16_t* __restrict__ x, int64_t cols, int64_t group_rows, float* __restrict__ outer) {
    __shared__ float red[kThreads / 32];
    const int64_t g = blockIdx.x;
    const uint4* src = reinterpret_cast<const uint4*>(x + g * group_rows * cols);
    const int64_t n = group_rows * cols / 8;
    float m = 0.0f;
    for (int64_t i = threadIdx.x; i < n; i += kThreads) {
        const uint4 u = __ldg(src + i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[k])), fabsf(bf16_hi(w[k]))));
    }
    m = block_reduce_max(m, red);
    if (threadIdx.x == 0) outer[g] = __fdiv_rn(m, kOuterDiv);
}

// One thread per 16-value block of a bf16 [rows, cols]: codes, scale byte.
template <int R, bool kSR>
__global__ void __launch_bounds__(kThreads)
nvfp4_quantize_sr_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t group_rows,
                         const float* __restrict__ outer, uint64_t seed, uint64_t stream_id, int sf_layout,
                         uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
    const int64_t S = cols / 16;
    const int64_t item = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (item >= rows * S) return;
    const int64_t r = item / S, b = item - r * S;
    const uint4* src = reinterpret_cast<const uint4*>(x + r * cols + b * 16);
    const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
    const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
    float v[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) { v[2 * k] = bf16_lo(w[k]); v[2 * k + 1] = bf16_hi(w[k]); }
    uint32_t scode;
    uint2 packed;
    quantize_block16<R, kSR>(v, __ldg(outer + r / group_rows), seed, stream_id, (uint64_t)(r * cols + b * 16),
                             scode, packed);
    *reinterpret_cast<uint2*>(codes + (r * cols + b * 16) / 2) = packed;
    sf[sf_offset(r, b, S, sf_layout)] = (uint8_t)scode;
}

// Dequantised NVFP4 element (r, c): (q * sf) * outer[r / group_rows], one
// fp32 rounding after the exact block product.
__device__ __forceinline__ float nvfp4_value(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf,
                                             const float* __restrict__ outer, int64_t rows, int64_t cols,
                                             int64_t group_rows, int in_layout, int64_t r, int64_t c) {
    const int64_t ci = (r * cols + c) / 2, si = sf_offset(r, c / 16, cols / 16, in_layout);
    if (!mx_in_range(ci, 1, rows * cols / 2) || !mx_in_range(si, 1, rows * (cols / 16)) ||
        !mx_in_range(r / group_rows, 1, rows / group_rows))
        return 0.0f;
    const uint32_t byte = __ldg(codes + ci);
    const uint32_t q = (c & 1) ? (byte >> 4) : (byte & 15u);
    const float qv = (q & 8) ? -e2m1_mag(q & 7) : e2m1_mag(q & 7);
    const float bp = __fmul_rn(qv, e4m3_to_f32(__ldg(sf + si)));
    return __fmul_rn(bp, __ldg(outer + r / group_rows));
}

// Pass 1 of the requantisation: amax of the dequantised input per output row
// (input column c of expert e: target e * cols + c) or per expert (target e).
// Block = 128 input rows x 64 columns, thread = one column over 32 rows; the
// block's maximum per target is merged with one atomicMax on the float bits
// (non-negative floats order like their bit patterns).  amax_bits holds zeros
// on entry.
__global__ void __launch_bounds__(kThreads)
requant_amax_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf,
                    const float* __restrict__ outer, int64_t rows, int64_t cols, int64_t group_rows, int in_layout,
                    int64_t rows_per_expert, int per_expert, uint32_t* __restrict__ amax_bits) {
    __shared__ float part[4][64];
    const int64_t r0 = (int64_t)blockIdx.y * 128, c0 = (int64_t)blockIdx.x * 64;
    const int cl = threadIdx.x & 63, rg = threadIdx.x >> 6;
    const int64_t c = c0 + cl;
    float m = 0.0f;
    for (int i = 0; i < 32; ++i)
        m = fmaxf(m, fabsf(nvfp4_value(codes, sf, outer, rows, cols, group_rows, in_layout, r0 + rg * 32 + i, c)));
    part[rg][cl] = m;
    __syncthreads();
    const int64_t e = r0 / rows_per_expert;
    if (!per_expert) {
        if (threadIdx.x < 64) {
            const float v = fmaxf(fmaxf(part[0][cl], part[1][cl]), fmaxf(part[2][cl], part[3][cl]));
            atomicMax(amax_bits + e * cols + c, __float_as_uint(v));
        }
    } else {
        __shared__ float red[kThreads / 32];
        const float v = block_reduce_max(part[rg][cl], red);
        if (threadIdx.x == 0) atomicMax(amax_bits + e, __float_as_uint(v));
    }
}

// amax bits -> outer scale, in place.
__global__ void amax_to_outer_kernel(float* __restrict__ v, int64_t n) {
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i < n) v[i] = __fdiv_rn(v[i], kOuterDiv);
}

// Pass 2: one thread per output block of 16.  Output row o = e * cols + c
// (input column c of expert e), output columns n0 .. n0 + 15 = the expert's
// input rows e * rows_per_expert + n0 ..; consecutive threads take
// consecutive c, so the input bytes of a row are read together.
template <int R, bool kSR>
__global__ void __launch_bounds__(kThreads)
requant_nvfp4_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf,
                     const float* __restrict__ outer, int64_t rows, int64_t cols, int64_t group_rows, int in_layout,
                     int64_t rows_per_expert, int per_expert, const float* __restrict__ out_outer, uint64_t seed,
                     uint64_t stream_id, int out_layout, uint8_t* __restrict__ out_codes,
                     uint8_t* __restrict__ out_sf) {
    const int64_t nb = rows_per_expert / 16;                   // output blocks per output row
    const int64_t E = rows / rows_per_expert;
    const int64_t item = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (item >= E * nb * cols) return;
    const int64_t c = item % cols, rest = item / cols;
    const int64_t b = rest % nb, e = rest / nb;
    const int64_t o = e * cols + c;
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        v[i] = nvfp4_value(codes, sf, outer, rows, cols, group_rows, in_layout, e * rows_per_expert + b * 16 + i, c);
    uint32_t scode;
    uint2 packed;
    const float s = __ldg(out_outer + (per_expert ? e : o));
    quantize_block16<R, kSR>(v, s, seed, stream_id, (uint64_t)(o * rows_per_expert + b * 16), scode, packed);
    if (mx_in_range((o * rows_per_expert + b * 16) / 2, 8, rows * cols / 2))
        *reinterpret_cast<uint2*>(out_codes + (o * rows_per_expert + b * 16) / 2) = packed;
    if (mx_in_range(sf_offset(o, b, nb, out_layout), 1, rows * cols / 16)) out_sf[sf_offset(o, b, nb, out_layout)] = (uint8_t)scode;
}

// 16x16 tiles: one warp per tile, lane l takes row l / 2 of the tile and its
// eight columns 8 (l % 2) ..; the tile amax is a warp reduction.
__global__ void __launch_bounds__(kThreads)
nvfp4_tile16_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t group_rows,
                    const float* __restrict__ outer, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf_tile) {
    const int64_t ntc = cols / 16;
    const int64_t tile = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    if (tile >= rows / 16 * ntc) return;                       // whole warps leave together
    const int lane = threadIdx.x & 31;
    const int64_t tr = tile / ntc, tc = tile - tr * ntc;
    const int64_t r = tr * 16 + (lane >> 1), c0 = tc * 16 + 8 * (lane & 1);
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + r * cols + c0));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    float v[8];
    float m = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        v[2 * k] = bf16_lo(w[k]);
        v[2 * k + 1] = bf16_hi(w[k]);
        m = fmaxf(m, fmaxf(fabsf(v[2 * k]), fabsf(v[2 * k + 1])));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float s = __ldg(outer + (tr * 16) / group_rows);
    const uint32_t scode = s > 0.0f ? (cvt_e4m3x2(__fdiv_rn(m, __fmul_rn(6.0f, s)), 0.0f) & 0xffu) : 0u;
    uint32_t packed = 0u;
    if (scode != 0) {
        const float inv = __fdiv_rn(1.0f, __fmul_rn(e4m3_to_f32(scode), s));
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = __fmul_rn(v[k], inv);
        packed = cvt_e2m1x8(v);
    }
    *reinterpret_cast<uint32_t*>(codes + (r * cols + c0) / 2) = packed;
    if (lane == 0) sf_tile[tr * ntc + tc] = (uint8_t)scode;
}

// ---------------------------------------------------------------------------
// The wgrad operands: the transpose [C, M] of a token-major [M, C] tensor
// with outer scales per expert segment of the tokens (seg [E+1], starts and
// lengths multiples of 128): per (segment, row) for dY^T, per segment for
// X^T.  Tokens past seg[E] (padding rows) quantise to zero.  The input is
// bf16 (the gradient) or the saved NVFP4 tensor (dequantised on load).
// ---------------------------------------------------------------------------
struct Bf16Src {
    const uint16_t* x;
    int64_t C;
    __device__ __forceinline__ float operator()(int64_t t, int64_t c) const {
        return __uint_as_float((uint32_t)__ldg(x + t * C + c) << 16);
    }
};
struct Nvfp4Src {
    const uint8_t* codes;
    const uint8_t* sf;
    const float* outer;
    int64_t M, C, group_rows;
    int layout;
    __device__ __forceinline__ float operator()(int64_t t, int64_t c) const {
        return nvfp4_value(codes, sf, outer, M, C, group_rows, layout, t, c);
    }
};

// Pass 1: block = 128 tokens x 64 columns of one segment (tiles at or past
// seg[E] do nothing); per-target maxima merged by atomicMax on the float bits.
template <typename Src>
__global__ void __launch_bounds__(kThreads)
segment_amax_kernel(Src src, const int64_t* __restrict__ seg, int64_t E, int64_t C, int per_row,
                    uint32_t* __restrict__ amax_bits) {
    __shared__ float part[4][64];
    __shared__ float red[kThreads / 32];
    const int64_t r0 = (int64_t)blockIdx.y * 128, c0 = (int64_t)blockIdx.x * 64;
    const int64_t end = __ldg(seg + E);
    if (r0 >= end) return;                                 // the whole block leaves together
    const int cl = threadIdx.x & 63, rg = threadIdx.x >> 6;
    const int64_t c = c0 + cl;
    float m = 0.0f;
    for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(src(r0 + rg * 32 + i, c)));
    part[rg][cl] = m;
    __syncthreads();
    int64_t lo = 0, hi = E;                                // seg[lo] <= r0 < seg[hi]
    while (hi - lo > 1) {
        const int64_t mid = (lo + hi) >> 1;
        if (__ldg(seg + mid) <= r0) lo = mid; else hi = mid;
    }
    if (per_row) {
        if (threadIdx.x < 64) {
            const float v = fmaxf(fmaxf(part[0][cl], part[1][cl]), fmaxf(part[2][cl], part[3][cl]));
            atomicMax(amax_bits + lo * C + c, __float_as_uint(v));
        }
    } else {
        const float v = block_reduce_max(part[rg][cl], red);
        if (threadIdx.x == 0) atomicMax(amax_bits + lo, __float_as_uint(v));
    }
}

// Pass 2: one thread per output block of 16 tokens; consecutive threads take
// consecutive columns c (output rows).
template <int R, bool kSR, typename Src>
__global__ void __launch_bounds__(kThreads)
segment_quantize_kernel(Src src, const int64_t* __restrict__ seg, int64_t E, int64_t M, int64_t C, int per_row,
                        const float* __restrict__ out_outer, uint64_t seed, uint64_t stream_id, int out_layout,
                        uint8_t* __restrict__ out_codes, uint8_t* __restrict__ out_sf) {
    const int64_t nb = M / 16;
    const int64_t item = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (item >= nb * C) return;
    const int64_t c = item % C, b = item / C;
    const int64_t t0 = b * 16;
    uint32_t scode = 0;
    uint2 packed = make_uint2(0u, 0u);
    if (t0 < __ldg(seg + E)) {
        int64_t lo = 0, hi = E;
        while (hi - lo > 1) {
            const int64_t mid = (lo + hi) >> 1;
            if (__ldg(seg + mid) <= t0) lo = mid; else hi = mid;
        }
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = src(t0 + i, c);
        const float s = __ldg(out_outer + (per_row ? lo * C + c : lo));
        quantize_block16<R, kSR>(v, s, seed, stream_id, (uint64_t)(c * M + t0), scode, packed);
    }
    if (mx_in_range((c * M + t0) / 2, 8, C * M / 2)) *reinterpret_cast<uint2*>(out_codes + (c * M + t0) / 2) = packed;
    if (mx_in_range(sf_offset(c, b, nb, out_layout), 1, C * M / 16)) out_sf[sf_offset(c, b, nb, out_layout)] = (uint8_t)scode;
}

template <bool kSR, typename F>
int dispatch_rbits(int rbits, F&& f) {
    if (!kSR) return f(std::integral_constant<int, 16>{});
    if (rbits == 8) return f(std::integral_constant<int, 8>{});
    if (rbits == 16) return f(std::integral_constant<int, 16>{});
    return f(std::integral_constant<int, 32>{});
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================

extern "C" int nvfp4_quantize_sr(const void* x, int64_t rows, int64_t cols, int64_t group_rows, int rounding,
                                 uint64_t seed, uint64_t stream_id, int rbits, uint8_t* codes, uint8_t* sf,
                                 float* outer, int sf_layout, cudaStream_t stream) {
    MX_NVTX_RANGE("nvfp4_quantize_sr");
    if (((!x || !codes || !sf || !outer) && rows > 0) || rows < 0 || cols <= 0 || cols % 16 || group_rows <= 0 ||
        rows % group_rows || !mx_aligned(x, 16) || !mx_aligned(codes, 16))
        return MX_EINVAL;
    if (rounding != MX_ROUND_RNE && rounding != MX_ROUND_SR) return MX_EINVAL;
    if (rounding == MX_ROUND_SR && rbits != 8 && rbits != 16 && rbits != 32) return MX_EINVAL;
    if (sf_layout != MX_SF_ROWMAJOR && sf_layout != MX_SF_MMA) return MX_EINVAL;
    if (sf_layout == MX_SF_MMA && (rows % 128 || cols % 64)) return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (rows == 0) return MX_OK;
    group_outer_kernel<<<(unsigned)(rows / group_rows), kThreads, 0, stream>>>(static_cast<const uint16_t*>(x), cols,
                                                                               group_rows, outer);
    mx_count_launch();
    const int64_t items = rows * (cols / 16);
    const unsigned grid = (unsigned)((items + kThreads - 1) / kThreads);
    auto launch = [&](auto kSRc) {
        constexpr bool kSR = decltype(kSRc)::value;
        return dispatch_rbits<kSR>(rbits, [&](auto Rc) {
            nvfp4_quantize_sr_kernel<decltype(Rc)::value, kSR><<<grid, kThreads, 0, stream>>>(
                static_cast<const uint16_t*>(x), rows, cols, group_rows, outer, seed, stream_id, sf_layout, codes,
                sf);
            mx_count_launch();
            return mx_launch_status();
        });
    };
    return rounding == MX_ROUND_SR ? launch(std::true_type{}) : launch(std::false_type{});
}

extern "C" int nvfp4_requant_transpose_sr(const uint8_t* codes, const uint8_t* sf, const float* outer, int64_t rows,
                                          int64_t cols, int64_t group_rows, int in_sf_layout, int64_t experts,
                                          int out_outer_per_expert, int rounding, uint64_t seed, uint64_t stream_id,
                                          int rbits, uint8_t* out_codes, uint8_t* out_sf, float* out_outer,
                                          int out_sf_layout, cudaStream_t stream) {
    MX_NVTX_RANGE("nvfp4_requant_transpose_sr");
    if (((!codes || !sf || !outer || !out_codes || !out_sf || !out_outer) && rows > 0) || rows < 0 || cols <= 0 ||
        cols % 64 || group_rows <= 0 || rows % group_rows || experts < 1 || rows % experts ||
        !mx_aligned(codes, 16) || !mx_aligned(out_codes, 16) || !mx_aligned(out_outer, 4))
        return MX_EINVAL;
    const int64_t rpe = rows / experts;
    if (rpe % 128) return MX_EINVAL;                          // pass 1 tiles of 128 rows stay inside an expert
    if (rounding != MX_ROUND_RNE && rounding != MX_ROUND_SR) return MX_EINVAL;
    if (rounding == MX_ROUND_SR && rbits != 8 && rbits != 16 && rbits != 32) return MX_EINVAL;
    for (int l : {in_sf_layout, out_sf_layout})
        if (l != MX_SF_ROWMAJOR && l != MX_SF_MMA) return MX_EINVAL;
    if (in_sf_layout == MX_SF_MMA && rows % 128) return MX_EINVAL;
    if (out_sf_layout == MX_SF_MMA && ((experts * cols) % 128 || rpe % 64)) return MX_EINVAL;
    if (out_outer_per_expert != 0 && out_outer_per_expert != 1) return MX_EINVAL;
    if (!out_outer_per_expert && experts != 1) return MX_EINVAL;   // per-row scales: one block (activations)
    if (int st = mx_check_device()) return st;
    if (rows == 0) return MX_OK;
    const int64_t n_outer = out_outer_per_expert ? experts : experts * cols;
    cudaError_t ce = cudaMemsetAsync(out_outer, 0, (size_t)n_outer * sizeof(float), stream);
    if (ce != cudaSuccess) return mx_set_cuda_error(ce);
    requant_amax_kernel<<<dim3((unsigned)(cols / 64), (unsigned)(rows / 128)), kThreads, 0, stream>>>(
        codes, sf, outer, rows, cols, group_rows, in_sf_layout, rpe, out_outer_per_expert,
        reinterpret_cast<uint32_t*>(out_outer));
    mx_count_launch();
    amax_to_outer_kernel<<<(unsigned)((n_outer + kThreads - 1) / kThreads), kThreads, 0, stream>>>(out_outer,
                                                                                                   n_outer);
    mx_count_launch();
    const int64_t items = experts * (rpe / 16) * cols;
    const unsigned grid = (unsigned)((items + kThreads - 1) / kThreads);
    auto launch = [&](auto kSRc) {
        constexpr bool kSR = decltype(kSRc)::value;
        return dispatch_rbits<kSR>(rbits, [&](auto Rc) {
            requant_nvfp4_kernel<decltype(Rc)::value, kSR><<<grid, kThreads, 0, stream>>>(
                codes, sf, outer, rows, cols, group_rows, in_sf_layout, rpe, out_outer_per_expert, out_outer, seed,
                stream_id, out_sf_layout, out_codes, out_sf);
            mx_count_launch();
            return mx_launch_status();
        });
    };
    return rounding == MX_ROUND_SR ? launch(std::true_type{}) : launch(std::false_type{});
}

extern "C" int nvfp4_quantize_tile16(const void* x, int64_t rows, int64_t cols, int64_t group_rows, uint8_t* codes,
                                     uint8_t* sf_tile, float* outer, cudaStream_t stream) {
    MX_NVTX_RANGE("nvfp4_quantize_tile16");
    if (((!x || !codes || !sf_tile || !outer) && rows > 0) || rows < 0 || cols <= 0 || cols % 16 || rows % 16 ||
        group_rows <= 0 || group_rows % 16 || rows % group_rows || !mx_aligned(x, 16) || !mx_aligned(codes, 16))
        return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (rows == 0) return MX_OK;
    group_outer_kernel<<<(unsigned)(rows / group_rows), kThreads, 0, stream>>>(static_cast<const uint16_t*>(x), cols,
                                                                               group_rows, outer);
    mx_count_launch();
    const int64_t warps = rows / 16 * (cols / 16);
    nvfp4_tile16_kernel<<<(unsigned)((warps * 32 + kThreads - 1) / kThreads), kThreads, 0, stream>>>(
        static_cast<const uint16_t*>(x), rows, cols, group_rows, outer, codes, sf_tile);
    mx_count_launch();
    return mx_launch_status();
}

namespace {

template <typename Src>
int segments_common(Src src, int64_t M, int64_t C, const int64_t* seg, int64_t E, int per_row, int rounding,
                    uint64_t seed, uint64_t stream_id, int rbits, uint8_t* out_codes, uint8_t* out_sf,
                    float* out_outer, int out_sf_layout, cudaStream_t stream) {
    const int64_t n_outer = per_row ? E * C : E;
    cudaError_t ce = cudaMemsetAsync(out_outer, 0, (size_t)n_outer * sizeof(float), stream);
    if (ce != cudaSuccess) return mx_set_cuda_error(ce);
    segment_amax_kernel<Src><<<dim3((unsigned)(C / 64), (unsigned)(M / 128)), kThreads, 0, stream>>>(
        src, seg, E, C, per_row, reinterpret_cast<uint32_t*>(out_outer));
    mx_count_launch();
    amax_to_outer_kernel<<<(unsigned)((n_outer + kThreads - 1) / kThreads), kThreads, 0, stream>>>(out_outer,
                                                                                                   n_outer);
    mx_count_launch();
    const int64_t items = (M / 16) * C;
    const unsigned grid = (unsigned)((items + kThreads - 1) / kThreads);
    auto launch = [&](auto kSRc) {
        constexpr bool kSR = decltype(kSRc)::value;
        return dispatch_rbits<kSR>(rbits, [&](auto Rc) {
            segment_quantize_kernel<decltype(Rc)::value, kSR, Src><<<grid, kThreads, 0, stream>>>(
                src, seg, E, M, C, per_row, out_outer, seed, stream_id, out_sf_layout, out_codes, out_sf);
            mx_count_launch();
            return mx_launch_status();
        });
    };
    return rounding == MX_ROUND_SR ? launch(std::true_type{}) : launch(std::false_type{});
}

int segments_check(int64_t M, int64_t C, const int64_t* seg, int64_t E, int per_row, int rounding, int rbits,
                   const uint8_t* out_codes, const uint8_t* out_sf, const float* out_outer, int out_sf_layout) {
    if (((!seg || !out_codes || !out_sf || !out_outer) && M > 0) || M < 0 || M % 128 || C <= 0 || C % 64 || E < 1 ||
        !mx_aligned(out_codes, 16) || !mx_aligned(out_outer, 4))
        return MX_EINVAL;
    if (per_row != 0 && per_row != 1) return MX_EINVAL;
    if (rounding != MX_ROUND_RNE && rounding != MX_ROUND_SR) return MX_EINVAL;
    if (rounding == MX_ROUND_SR && rbits != 8 && rbits != 16 && rbits != 32) return MX_EINVAL;
    if (out_sf_layout != MX_SF_ROWMAJOR && out_sf_layout != MX_SF_MMA) return MX_EINVAL;
    if (out_sf_layout == MX_SF_MMA && C % 128) return MX_EINVAL;
    return MX_OK;
}

}  // namespace

extern "C" int nvfp4_quantize_transpose_segments(const void* x, int64_t M, int64_t C, const int64_t* seg, int64_t E,
                                                 int per_row, int rounding, uint64_t seed, uint64_t stream_id,
                                                 int rbits, uint8_t* out_codes, uint8_t* out_sf, float* out_outer,
                                                 int out_sf_layout, cudaStream_t stream) {
    MX_NVTX_RANGE("nvfp4_quantize_transpose_segments");
    if ((!x && M > 0) || !mx_aligned(x, 16)) return MX_EINVAL;
    if (int st = segments_check(M, C, seg, E, per_row, rounding, rbits, out_codes, out_sf, out_outer, out_sf_layout))
        return st;
    if (int st = mx_check_device()) return st;
    if (M == 0) return MX_OK;
    return segments_common(Bf16Src{static_cast<const uint16_t*>(x), C}, M, C, seg, E, per_row, rounding, seed,
                           stream_id, rbits, out_codes, out_sf, out_outer, out_sf_layout, stream);
}

extern "C" int nvfp4_requant_transpose_segments(const uint8_t* codes, const uint8_t* sf, const float* outer,
                                                int in_sf_layout, int64_t group_rows, int64_t M, int64_t C,
                                                const int64_t* seg, int64_t E, int per_row, int rounding,
                                                uint64_t seed, uint64_t stream_id, int rbits, uint8_t* out_codes,
                                                uint8_t* out_sf, float* out_outer, int out_sf_layout,
                                                cudaStream_t stream) {
    MX_NVTX_RANGE("nvfp4_requant_transpose_segments");
    if (((!codes || !sf || !outer) && M > 0) || group_rows <= 0 || M % group_rows || !mx_aligned(codes, 16))
        return MX_EINVAL;
    if (in_sf_layout != MX_SF_ROWMAJOR && in_sf_layout != MX_SF_MMA) return MX_EINVAL;
    if (int st = segments_check(M, C, seg, E, per_row, rounding, rbits, out_codes, out_sf, out_outer, out_sf_layout))
        return st;
    if (int st = mx_check_device()) return st;
    if (M == 0) return MX_OK;
    return segments_common(Nvfp4Src{codes, sf, outer, M, C, group_rows, in_sf_layout}, M, C, seg, E, per_row, rounding,
                           seed, stream_id, rbits, out_codes, out_sf, out_outer, out_sf_layout, stream);
}

MX_BOUNDS_READER(mx_bounds_word_nvfp4_bwd)
