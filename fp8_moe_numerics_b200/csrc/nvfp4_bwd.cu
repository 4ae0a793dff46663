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
// oracle takes them.  The stochastic rounding runs on the hardware cvt.rs
// instruction for R = 16 and R = 8 (it computes the rule above exactly) and
// in exact software arithmetic for R = 32.
#include <type_traits>

#include "mx_common.cuh"
#include "requant_tile.cuh"
#include "e2m1_sr.cuh"

namespace {

constexpr int kThreads = 256;
constexpr float kOuterDiv = 2688.0f;              // 6 * 448

// One 16-value block: E4M3 scale of bmax / (6 s) (0 when s == 0) and the
// eight code bytes, element 2j in the low nibble of byte j.  L0 is the linear
// output index of element 0 (for the random integers), a multiple of 16.
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
        packed = e2m1_sr_codes<R>(y, seed, stream_id, L0);
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

// Dequantised NVFP4 values (q * sf) * outer[r / group_rows], one fp32
// rounding after the exact block product, of kN consecutive rows r0 .. r0 +
// kN - 1 at column c.  r0 is a multiple of kN (16 or 32), so the rows share
// one 32-row group of the MMA scale layout and their scale bytes sit 16 bytes
// apart (S apart in the row-major layout): the addresses are stepped, and
// the outer-scale group is found once when group_rows is a multiple of kN.
template <int kN>
__device__ __forceinline__ void nvfp4_column(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf,
                                             const float* __restrict__ outer, int64_t rows, int64_t cols,
                                             int64_t group_rows, int in_layout, int64_t r0, int64_t c, float* v) {
    const int64_t S = cols / 16;
    const int64_t c0i = (r0 * cols + c) / 2, s0i = sf_offset(r0, c / 16, S, in_layout);
    const int64_t s_step = in_layout == MX_SF_MMA ? 16 : S;
    const bool uniform = group_rows % kN == 0;
    const float so_uni = uniform && mx_in_range(r0 / group_rows, 1, rows / group_rows) ? __ldg(outer + r0 / group_rows)
                                                                                       : 0.0f;
    const int shift = (int)(c & 1) * 4;
#pragma unroll
    for (int i = 0; i < kN; ++i) {
        const int64_t ci = c0i + i * (cols / 2), si = s0i + i * s_step;
        const int64_t gi = uniform ? 0 : (group_rows == 1 ? r0 + i : (r0 + i) / group_rows);
        if (!mx_in_range(ci, 1, rows * cols / 2) || !mx_in_range(si, 1, rows * S) ||
            (!uniform && !mx_in_range(gi, 1, rows / group_rows))) {
            v[i] = 0.0f;
            continue;
        }
        const uint32_t q = (__ldg(codes + ci) >> shift) & 15u;
        const float qv = (q & 8) ? -e2m1_mag(q & 7) : e2m1_mag(q & 7);
        const float bp = __fmul_rn(qv, e4m3_to_f32(__ldg(sf + si)));
        v[i] = __fmul_rn(bp, uniform ? so_uni : __ldg(outer + gi));
    }
}

// Pass 1 of the requantisation with one outer scale per output row (input
// column c: target c): amax of the dequantised input down each column.
// Block = 128 input rows x 64 columns, thread = one column over 32 rows; the
// block's maximum per column is merged with one atomicMax on the float bits
// (non-negative floats order like their bit patterns).  amax_bits holds zeros
// on entry.
__global__ void __launch_bounds__(kThreads)
requant_amax_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf,
                    const float* __restrict__ outer, int64_t rows, int64_t cols, int64_t group_rows, int in_layout,
                    uint32_t* __restrict__ amax_bits) {
    __shared__ float part[4][64];
    const int64_t r0 = (int64_t)blockIdx.y * 128, c0 = (int64_t)blockIdx.x * 64;
    const int cl = threadIdx.x & 63, rg = threadIdx.x >> 6;
    const int64_t c = c0 + cl;
    float v[32];
    nvfp4_column<32>(codes, sf, outer, rows, cols, group_rows, in_layout, r0 + rg * 32, c, v);
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
    part[rg][cl] = m;
    __syncthreads();
    if (threadIdx.x < 64) {
        const float v = fmaxf(fmaxf(part[0][cl], part[1][cl]), fmaxf(part[2][cl], part[3][cl]));
        atomicMax(amax_bits + c, __float_as_uint(v));
    }
}

// amax bits -> outer scale, in place.
__global__ void amax_to_outer_kernel(float* __restrict__ v, int64_t n) {
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i < n) v[i] = __fdiv_rn(v[i], kOuterDiv);
}

// Largest |q * sf| over the 16 values of one block: the E2M1 magnitude codes
// (low three bits of each nibble) order like their values, so the block's
// largest code is found on the bytes (two 32-bit words) and decoded once.
__device__ __forceinline__ float block_max_product(uint32_t w0, uint32_t w1, uint32_t scode) {
    const uint32_t a = w0 & 0x77777777u, b = w1 & 0x77777777u;
    uint32_t m = __vmaxu4(__vmaxu4(a & 0x0f0f0f0fu, (a >> 4) & 0x0f0f0f0fu),
                          __vmaxu4(b & 0x0f0f0f0fu, (b >> 4) & 0x0f0f0f0fu));
    m = __vmaxu4(m, m >> 16);
    m = __vmaxu4(m, m >> 8);
    return __fmul_rn(e2m1_mag(m & 0xffu), e4m3_to_f32(scode));
}

// Pass 1 of the requantisations whose outer scale is one per group of input
// rows (an expert of a weight stack, a token segment): amax over the group
// of the dequantised values RN(q sf s_r).  RN is monotone, so a row's
// largest dequantised magnitude is RN(max |q sf| * s_r) with s_r the row's
// outer scale.  Block = 128 rows of one group, thread = one row: its 64-value
// chunks (32 code bytes, the 4 scale bytes of 4 blocks) at stride 2; the
// lanes of a warp take 32 consecutive rows, so the MMA layout's scale bytes of
// a warp are one 512-byte atom.  Kind kSeg: the groups are the segments seg
// (blocks at or past seg[E] do nothing); else groups of rpe rows.  amax_bits
// holds zeros on entry; the block's maximum goes in by one atomicMax on the
// float bits.
template <int kInLayout, bool kSeg>
__global__ void __launch_bounds__(kThreads)
group_amax_nvfp4_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf, bool sf_words,
                        const float* __restrict__ outer, int64_t rows, int64_t cols, int64_t group_rows, int64_t rpe,
                        const int64_t* __restrict__ seg, int64_t E, uint32_t* __restrict__ amax_bits) {
    __shared__ float red[kThreads / 32];
    const int64_t r0 = (int64_t)blockIdx.x * 128;
    int64_t target;
    if (kSeg) {
        if (r0 >= __ldg(seg + E)) return;                       // the whole block leaves together
        int64_t lo = 0, hi = E;                                 // seg[lo] <= r0 < seg[hi]
        while (hi - lo > 1) {
            const int64_t mid = (lo + hi) >> 1;
            if (__ldg(seg + mid) <= r0) lo = mid; else hi = mid;
        }
        target = lo;
    } else {
        target = r0 / rpe;
    }
    const int64_t r = r0 + (threadIdx.x & 127);
    const int64_t S = cols >> 4, nchunk = cols >> 6;
    float m = 0.0f;
#pragma unroll 2
    for (int64_t k = threadIdx.x >> 7; k < nchunk; k += 2) {
        const int64_t co = r * (cols >> 1) + 32 * k, so_ = sf_offset(r, 4 * k, S, kInLayout);
        uint4 c0 = make_uint4(0u, 0u, 0u, 0u), c1 = c0;
        uint32_t sw = 0;
        if (mx_in_range(co, 32, rows * (cols >> 1))) {
            c0 = __ldcs(reinterpret_cast<const uint4*>(codes + co));
            c1 = __ldcs(reinterpret_cast<const uint4*>(codes + co) + 1);
        }
        if (mx_in_range(so_, 4, rows * S)) {
            const uint8_t* sr = sf + so_;
            sw = sf_words ? __ldg(reinterpret_cast<const uint32_t*>(sr))
                          : (uint32_t)__ldg(sr) | (uint32_t)__ldg(sr + 1) << 8 | (uint32_t)__ldg(sr + 2) << 16 |
                                (uint32_t)__ldg(sr + 3) << 24;
        }
        m = fmaxf(m, fmaxf(fmaxf(block_max_product(c0.x, c0.y, sw & 0xffu), block_max_product(c0.z, c0.w, (sw >> 8) & 0xffu)),
                           fmaxf(block_max_product(c1.x, c1.y, (sw >> 16) & 0xffu), block_max_product(c1.z, c1.w, sw >> 24))));
    }
    const int64_t gi = group_rows == 1 ? r : r / group_rows;
    m = __fmul_rn(m, mx_in_range(gi, 1, rows / group_rows) ? __ldg(outer + gi) : 0.0f);
    m = block_reduce_max(m, red);
    if (threadIdx.x == 0) atomicMax(amax_bits + target, __float_as_uint(m));
}

// Pass 2 of the transposed NVFP4 quantisations, on the transposed tile (128
// input rows x 64 input columns).  Source kIn: a saved NVFP4 tensor with one
// outer scale per tile (kInNvfp4Tile) or per row (kInNvfp4Rows), or bf16
// (kInBf16).  Each thread takes 16 consecutive input rows (one output block)
// of one output row, twice: the 16 values as fp32 (NVFP4: the products p,
// then x = RN(p s_r) with the input row's outer scale s_r), then the output
// block's scale and codes as in the forward quantiser with the output row's
// outer scale.
//   Kind kSeg = false (a stack of experts of rpe rows each): output row
//   o = e * cols + c for input column c of expert e, its columns the expert's
//   rpe rows.  Kind kSeg = true (token segments): output row o = c, its
//   columns the M = rows tokens; tiles at or past seg[E] write zeros.
//   Outer scale of output row o: per group (expert or segment) when
//   out_per_group, else per output row (kSeg: per segment and column).
// The 8 scale bytes of an output row's tile are two aligned 4-byte words in
// either layout (n0 / 16 is a multiple of 8): lanes ^ 8 and ^ 16 hold a
// word's other bytes.
constexpr int kInNvfp4Tile = 0, kInNvfp4Rows = 1, kInBf16 = 2;

// Five blocks per SM where that needs no spills (all but the software R = 32 rounding),
// as for the MXFP8 requantisation's tile kernel.
template <int R, bool kSR, int kIn, bool kSeg>
__global__ void __launch_bounds__(kRqThreads, R == 32 ? 4 : 5)
requant_nvfp4_tile_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf, int in_layout, bool sf_words,
                          const float* __restrict__ outer, int64_t rows, int64_t cols, int64_t group_rows,
                          int64_t rpe, const int64_t* __restrict__ seg, int64_t E, int out_per_group,
                          const float* __restrict__ out_outer, uint64_t seed, uint64_t stream_id, int out_layout,
                          bool osf_words, uint8_t* __restrict__ out_codes, uint8_t* __restrict__ out_sf) {
    __shared__ __align__(1024) uint16_t T[kRqCols * kRqRows];
    __shared__ __align__(16) float so[kIn == kInNvfp4Rows ? kRqRows : 4];
    const int64_t c0 = (int64_t)blockIdx.x * kRqCols, r0 = (int64_t)blockIdx.y * kRqRows;
    const uint32_t tbase = smem_u32(T);
    int64_t grp, n0, out_cols, o_base;
    bool live = true;
    if (kSeg) {
        live = r0 < __ldg(seg + E);
        int64_t lo = 0, hi = E;
        if (live)
            while (hi - lo > 1) {
                const int64_t mid = (lo + hi) >> 1;
                if (__ldg(seg + mid) <= r0) lo = mid; else hi = mid;
            }
        grp = lo;
        n0 = r0;
        out_cols = rows;
        o_base = 0;
    } else {
        grp = r0 / rpe;
        n0 = r0 - grp * rpe;
        out_cols = rpe;
        o_base = grp * cols;
    }
    float s_uni = 0.0f;
    if (live) {
        if constexpr (kIn == kInBf16) {
            rq_load_tile_bf16(reinterpret_cast<const uint16_t*>(codes), rows, cols, r0, c0, tbase);
        } else {
            if (kIn == kInNvfp4Tile) {      // group_rows is a multiple of 128: one input outer scale per tile
                const int64_t gi = r0 / group_rows;
                if (mx_in_range(gi, 1, rows / group_rows)) s_uni = __ldg(outer + gi);
            }
            rq_load_tile<-1, kIn == kInNvfp4Rows>(codes, sf, sf_words, outer, rows, cols, group_rows, r0, c0, tbase,
                                                  so, in_layout);
        }
    }
    __syncthreads();
    const RqLane ln;
    const int64_t cg = c0 + ln.c, o = o_base + cg;
    const int64_t nb = out_cols >> 4;
    const int64_t n_out = rows * cols;                           // output elements
    float s_out = 0.0f;
    if (live) {
        const int64_t si = out_per_group ? grp : (kSeg ? grp * cols + cg : o);
        if (mx_in_range(si, 1, out_per_group ? E : E * cols)) s_out = __ldg(out_outer + si);
    }
#pragma unroll
    for (int it = 0; it < 2; ++it) {
        const int j = ln.chunk(it);
        uint32_t scode = 0;
        uint2 packed = make_uint2(0u, 0u);
        const int64_t L0 = o * out_cols + n0 + 16 * j;          // linear index of the block's first output element
        if (live) {
            uint32_t hw[8];
            rq_read16(tbase, ln.c, j, hw);
            float v[16];
            if constexpr (kIn == kInBf16) {
#pragma unroll
                for (int i = 0; i < 8; ++i) { v[2 * i] = bf16_lo(hw[i]); v[2 * i + 1] = bf16_hi(hw[i]); }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) h2_to_f32x2(hw[i], v[2 * i], v[2 * i + 1]);
            }
            if constexpr (kIn == kInNvfp4Rows) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 s4 = *reinterpret_cast<const float4*>(so + 16 * j + 4 * i);
                    v[4 * i] = __fmul_rn(v[4 * i], s4.x);
                    v[4 * i + 1] = __fmul_rn(v[4 * i + 1], s4.y);
                    v[4 * i + 2] = __fmul_rn(v[4 * i + 2], s4.z);
                    v[4 * i + 3] = __fmul_rn(v[4 * i + 3], s4.w);
                }
            } else if constexpr (kIn == kInNvfp4Tile) {
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(v[i], s_uni);
            }
            quantize_block16<R, kSR>(v, s_out, seed, stream_id, (uint64_t)L0, scode, packed);
        }
        if (mx_in_range(L0 / 2, 8, n_out / 2)) *reinterpret_cast<uint2*>(out_codes + L0 / 2) = packed;
        uint32_t word = scode << (8 * (2 * ln.q + ln.jj));
        word |= __shfl_xor_sync(0xffffffffu, word, 8);
        word |= __shfl_xor_sync(0xffffffffu, word, 16);
        const int64_t sfo = sf_offset(o, (n0 >> 4) + 4 * it, nb, out_layout);
        if (ln.jj == 0 && ln.q == 0 && mx_in_range(sfo, 4, n_out >> 4)) {
            uint8_t* dst = out_sf + sfo;
            if (osf_words) *reinterpret_cast<uint32_t*>(dst) = word;
            else { dst[0] = (uint8_t)word; dst[1] = (uint8_t)(word >> 8); dst[2] = (uint8_t)(word >> 16); dst[3] = (uint8_t)(word >> 24); }
        }
    }
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
struct Nvfp4Src {
    const uint8_t* codes;
    const uint8_t* sf;
    const float* outer;
    int64_t M, C, group_rows;
    int layout;
    template <int kN>
    __device__ __forceinline__ void column(int64_t t0, int64_t c, float* v) const {
        nvfp4_column<kN>(codes, sf, outer, M, C, group_rows, layout, t0, c, v);
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
    float v[32];
    src.template column<32>(r0 + rg * 32, c, v);
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
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

// Pass 1 of the bf16 source: amax per (segment, column) or per segment of a
// token-major bf16 [M, C].  |x| of a bf16 orders like its low 15 bits, so the
// maxima are taken on the bit patterns, two columns per 32-bit word.  Block =
// 128 tokens x 64 columns of one segment (blocks at or past seg[E] do
// nothing); thread (k = t % 8, g = t / 8) reads columns 8k .. 8k + 7 of rows
// 4g .. 4g + 3 (16 bytes each); lanes ^ 8 and ^ 16 hold the same columns.
__global__ void __launch_bounds__(kThreads)
segment_amax_bf16_kernel(const uint16_t* __restrict__ x, const int64_t* __restrict__ seg, int64_t E, int64_t M,
                         int64_t C, int per_row, uint32_t* __restrict__ amax_bits) {
    __shared__ uint4 part[kThreads / 32][8];
    __shared__ float red[kThreads / 32];
    const int64_t r0 = (int64_t)blockIdx.y * 128, c0 = (int64_t)blockIdx.x * 64;
    if (r0 >= __ldg(seg + E)) return;                      // the whole block leaves together
    const int k = threadIdx.x & 7, g = threadIdx.x >> 3;
    uint4 m = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t xi = (r0 + 4 * g + i) * C + c0 + 8 * k;
        if (!mx_in_range(xi, 8, M * C)) continue;
        const uint4 v = __ldcs(reinterpret_cast<const uint4*>(x + xi));
        m.x = __vmaxu2(m.x, v.x & 0x7fff7fffu);
        m.y = __vmaxu2(m.y, v.y & 0x7fff7fffu);
        m.z = __vmaxu2(m.z, v.z & 0x7fff7fffu);
        m.w = __vmaxu2(m.w, v.w & 0x7fff7fffu);
    }
#pragma unroll
    for (int o = 8; o <= 16; o <<= 1) {
        m.x = __vmaxu2(m.x, __shfl_xor_sync(0xffffffffu, m.x, o));
        m.y = __vmaxu2(m.y, __shfl_xor_sync(0xffffffffu, m.y, o));
        m.z = __vmaxu2(m.z, __shfl_xor_sync(0xffffffffu, m.z, o));
        m.w = __vmaxu2(m.w, __shfl_xor_sync(0xffffffffu, m.w, o));
    }
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane < 8) part[w][lane] = m;
    __syncthreads();
    int64_t lo = 0, hi = E;                                // seg[lo] <= r0 < seg[hi]
    while (hi - lo > 1) {
        const int64_t mid = (lo + hi) >> 1;
        if (__ldg(seg + mid) <= r0) lo = mid; else hi = mid;
    }
    // thread c < 64: column c0 + c is half (c & 1) of word (c / 2) % 4 of chunk c / 8
    float v = 0.0f;
    if (threadIdx.x < 64) {
        const int c = threadIdx.x, kk = c >> 3, wd = (c >> 1) & 3;
        uint32_t bits = 0;
#pragma unroll
        for (int ww = 0; ww < kThreads / 32; ++ww) {
            const uint4 p = part[ww][kk];
            const uint32_t word = wd == 0 ? p.x : wd == 1 ? p.y : wd == 2 ? p.z : p.w;
            bits = max(bits, (c & 1) ? word >> 16 : word & 0xffffu);
        }
        v = __uint_as_float(bits << 16);
    }
    if (per_row) {
        if (threadIdx.x < 64) atomicMax(amax_bits + lo * C + c0 + threadIdx.x, __float_as_uint(v));
    } else {
        v = block_reduce_max(v, red);
        if (threadIdx.x == 0) atomicMax(amax_bits + lo, __float_as_uint(v));
    }
}

template <bool kSR, typename F>
int dispatch_rbits(int rbits, F&& f) {
    if constexpr (!kSR) {
        return f(std::integral_constant<int, 16>{});
    } else {
        if (rbits == 8) return f(std::integral_constant<int, 8>{});
        if (rbits == 16) return f(std::integral_constant<int, 16>{});
        return f(std::integral_constant<int, 32>{});
    }
}

}  // namespace

// Pass 2 of the transposed NVFP4 quantisations: one tile per block, grid
// (cols / 64, rows / 128).  The source is bf16 (codes holds it) when sf is
// null, else NVFP4.
template <bool kSeg>
int launch_requant_nvfp4_tiles(const uint8_t* codes, const uint8_t* sf, int in_layout, bool sf_words,
                               const float* outer, int64_t rows, int64_t cols, int64_t group_rows, int64_t rpe,
                               const int64_t* seg, int64_t E, int out_per_group, const float* out_outer, int rounding,
                               uint64_t seed, uint64_t stream_id, int rbits, int out_layout, bool osf_words,
                               uint8_t* out_codes, uint8_t* out_sf, cudaStream_t stream) {
    const dim3 grid((unsigned)(cols / kRqCols), (unsigned)(rows / kRqRows));
    auto launch = [&](auto kSRc, auto in_kind) {
        constexpr bool kSR = decltype(kSRc)::value;
        constexpr int kIn = decltype(in_kind)::value;
        return dispatch_rbits<kSR>(rbits, [&](auto Rc) {
            requant_nvfp4_tile_kernel<decltype(Rc)::value, kSR, kIn, kSeg><<<grid, kRqThreads, 0, stream>>>(
                codes, sf, in_layout, sf_words, outer, rows, cols, group_rows, rpe, seg, E, out_per_group, out_outer,
                seed, stream_id, out_layout, osf_words, out_codes, out_sf);
            mx_count_launch();
            return mx_launch_status();
        });
    };
    auto by_source = [&](auto kSRc) {
        if constexpr (kSeg)
            if (!sf) return launch(kSRc, std::integral_constant<int, kInBf16>{});      // bf16 source
        if (group_rows % kRqRows) return launch(kSRc, std::integral_constant<int, kInNvfp4Rows>{});
        return launch(kSRc, std::integral_constant<int, kInNvfp4Tile>{});               // one outer scale per tile
    };
    return rounding == MX_ROUND_SR ? by_source(std::true_type{}) : by_source(std::false_type{});
}

// ===========================================================================
// C ABI
// ===========================================================================

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
    if (rows / 128 > 65535) return MX_EINVAL;                  // tile rows on the grid's y axis
    if (int st = mx_check_device()) return st;
    if (rows == 0) return MX_OK;
    const int64_t n_outer = out_outer_per_expert ? experts : experts * cols;
    cudaError_t ce = cudaMemsetAsync(out_outer, 0, (size_t)n_outer * sizeof(float), stream);
    if (ce != cudaSuccess) return mx_set_cuda_error(ce);
    const bool sf_words = mx_aligned(sf, 4), osf_words = mx_aligned(out_sf, 4);
    uint32_t* amax_bits = reinterpret_cast<uint32_t*>(out_outer);
    if (out_outer_per_expert) {
        auto amax = in_sf_layout == MX_SF_MMA ? group_amax_nvfp4_kernel<MX_SF_MMA, false>
                                              : group_amax_nvfp4_kernel<MX_SF_ROWMAJOR, false>;
        amax<<<(unsigned)(rows / 128), kThreads, 0, stream>>>(codes, sf, sf_words, outer, rows, cols, group_rows, rpe,
                                                             nullptr, experts, amax_bits);
    } else {
        requant_amax_kernel<<<dim3((unsigned)(cols / 64), (unsigned)(rows / 128)), kThreads, 0, stream>>>(
            codes, sf, outer, rows, cols, group_rows, in_sf_layout, amax_bits);
    }
    mx_count_launch();
    amax_to_outer_kernel<<<(unsigned)((n_outer + kThreads - 1) / kThreads), kThreads, 0, stream>>>(out_outer,
                                                                                                   n_outer);
    mx_count_launch();
    return launch_requant_nvfp4_tiles<false>(codes, sf, in_sf_layout, sf_words, outer, rows, cols, group_rows, rpe,
                                             nullptr, experts, out_outer_per_expert, out_outer, rounding, seed,
                                             stream_id, rbits, out_sf_layout, osf_words, out_codes, out_sf, stream);
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
    if (M / 128 > 65535) return MX_EINVAL;                     // tile rows on the grid's y axis
    if (int st = mx_check_device()) return st;
    if (M == 0) return MX_OK;
    const int64_t n_outer = per_row ? E * C : E;
    cudaError_t ce = cudaMemsetAsync(out_outer, 0, (size_t)n_outer * sizeof(float), stream);
    if (ce != cudaSuccess) return mx_set_cuda_error(ce);
    segment_amax_bf16_kernel<<<dim3((unsigned)(C / 64), (unsigned)(M / 128)), kThreads, 0, stream>>>(
        static_cast<const uint16_t*>(x), seg, E, M, C, per_row, reinterpret_cast<uint32_t*>(out_outer));
    mx_count_launch();
    amax_to_outer_kernel<<<(unsigned)((n_outer + kThreads - 1) / kThreads), kThreads, 0, stream>>>(out_outer,
                                                                                                   n_outer);
    mx_count_launch();
    return launch_requant_nvfp4_tiles<true>(static_cast<const uint8_t*>(x), nullptr, MX_SF_MMA, false, nullptr, M, C,
                                            1, M, seg, E, !per_row, out_outer, rounding, seed, stream_id, rbits,
                                            out_sf_layout, mx_aligned(out_sf, 4), out_codes, out_sf, stream);
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
    if (M / 128 > 65535) return MX_EINVAL;                     // tile rows on the grid's y axis
    if (int st = mx_check_device()) return st;
    if (M == 0) return MX_OK;
    const int64_t n_outer = per_row ? E * C : E;
    cudaError_t ce = cudaMemsetAsync(out_outer, 0, (size_t)n_outer * sizeof(float), stream);
    if (ce != cudaSuccess) return mx_set_cuda_error(ce);
    const bool sf_words = mx_aligned(sf, 4), osf_words = mx_aligned(out_sf, 4);
    uint32_t* amax_bits = reinterpret_cast<uint32_t*>(out_outer);
    if (!per_row) {
        auto amax = in_sf_layout == MX_SF_MMA ? group_amax_nvfp4_kernel<MX_SF_MMA, true>
                                              : group_amax_nvfp4_kernel<MX_SF_ROWMAJOR, true>;
        amax<<<(unsigned)(M / 128), kThreads, 0, stream>>>(codes, sf, sf_words, outer, M, C, group_rows, M, seg, E,
                                                          amax_bits);
    } else {
        segment_amax_kernel<Nvfp4Src><<<dim3((unsigned)(C / 64), (unsigned)(M / 128)), kThreads, 0, stream>>>(
            Nvfp4Src{codes, sf, outer, M, C, group_rows, in_sf_layout}, seg, E, C, 1, amax_bits);
    }
    mx_count_launch();
    amax_to_outer_kernel<<<(unsigned)((n_outer + kThreads - 1) / kThreads), kThreads, 0, stream>>>(out_outer,
                                                                                                   n_outer);
    mx_count_launch();
    return launch_requant_nvfp4_tiles<true>(codes, sf, in_sf_layout, sf_words, outer, M, C, group_rows, M, seg, E,
                                            !per_row, out_outer, rounding, seed, stream_id, rbits, out_sf_layout,
                                            osf_words, out_codes, out_sf, stream);
}

MX_BOUNDS_READER(mx_bounds_word_nvfp4_bwd)
