// requant_tile.cuh -- the dequantise-and-transpose front end shared by the
// requantisations of a saved NVFP4 tensor (to MXFP8 and to NVFP4).
//
// [ai-primer §Stochastic rounding across transposes]: the backward GEMMs
// need the transposes of the tensors the forward pass saved in NVFP4.  Both
// requantisations start the same way: an NVFP4 tile is decoded to its block
// products q*sf and stored transposed in shared memory, where the second
// phase reads each output row's values along the input's rows.
//
// One tile = 128 input rows x 64 input columns, 256 threads.  Each thread
// decodes 2 rows x 16 columns (one scale block per row) to the exact f16
// products q*sf (cvt e2m1x2 -> f16x2, one f16x2 multiply per pair; |q sf| <=
// 2688 and >= 2^-10 when nonzero, so f16 holds it exactly), and the warp
// stores its 16 x 64 products transposed with four stmatrix.trans (8 x 8
// blocks of 16-bit values).  The tile lives in shared memory as f16 [64
// cols][128 rows], 16-byte chunks XOR-swizzled by rq_swz() so that both
// phases are free of bank conflicts.
#pragma once

#include "mx_common.cuh"

namespace {

constexpr int kRqRows = 128, kRqCols = 64, kRqThreads = 256;

__device__ __forceinline__ int rq_swz(int c) { return ((c >> 4) & 3) | ((c & 1) << 2); }

__device__ __forceinline__ uint32_t h2_of_e4m3(uint32_t code) {
    uint32_t h2;
    const uint16_t in = (uint16_t)(code * 0x0101u);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return h2;
}
__device__ __forceinline__ uint32_t h2_of_e2m1(uint32_t byte_in_low) {
    uint32_t h2;
    asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(h2) : "r"(byte_in_low));
    return h2;
}
__device__ __forceinline__ uint32_t h2_mul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
// max(|a|, |b|) per lane; the sign bit is not meaningful (callers drop it).
__device__ __forceinline__ uint32_t h2_maxabs(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ void h2_to_f32x2(uint32_t h, float& lo, float& hi) {
    asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
        : "=f"(lo), "=f"(hi) : "r"(h));
}
__device__ __forceinline__ void stmatrix_x4_trans(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};"
                 :: "r"(addr), "r"(r0), "r"(r1), "r"(r2), "r"(r3) : "memory");
}
__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// Byte address in the tile of the 16-byte chunk holding input rows 8k .. 8k + 7
// of tile column c (k = 0 .. 15).
__device__ __forceinline__ uint32_t rq_chunk(uint32_t tbase, int c, int k) {
    return tbase + c * 256 + ((k ^ rq_swz(c)) << 4);
}

// Phase 1: the tile at (r0, c0) of an NVFP4 [rows, cols] (codes 16-byte
// aligned; sf in layout kInLayout, or in_layout when kInLayout is -1; its 4
// scale bytes of a tile row read as one word when sf_words) decoded into the
// transposed f16 tile at tbase.  With kPerRow the outer scale of every tile
// row goes to so[0 .. 127] (row r takes outer[r / group_rows]).  Loads past
// the buffers' extents (only in the bounds-checked build) read zeros.
template <int kInLayout, bool kPerRow>
__device__ __forceinline__ void rq_load_tile(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf,
                                             bool sf_words, const float* __restrict__ outer, int64_t rows,
                                             int64_t cols, int64_t group_rows, int64_t r0, int64_t c0,
                                             uint32_t tbase, float* so, int in_layout = MX_SF_MMA) {
    const int layout = kInLayout >= 0 ? kInLayout : in_layout;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    // lane (rho = lane / 4, b = lane % 4): rows 16w + rho and 16w + 8 + rho, code bytes 8b..8b+7 of the tile
    // row = columns 16b..16b+15 (scale block b of the tile)
    const int rho = lane >> 2, b = lane & 3;
    const int64_t S = cols >> 4;
    uint32_t pr[2][8];
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const int64_t r = r0 + 16 * w + 8 * g + rho;
        const int64_t co = r * (cols >> 1) + (c0 >> 1) + 8 * b, so_ = sf_offset(r, c0 >> 4, S, layout);
        uint2 cw = make_uint2(0u, 0u);
        uint32_t sw = 0;
        if (mx_in_range(co, 8, rows * (cols >> 1)))
            cw = __ldcs(reinterpret_cast<const uint2*>(codes + co));
        if (mx_in_range(so_, 4, rows * S)) {
            const uint8_t* sr = sf + so_;                            // the row's 4 scale bytes, consecutive
            sw = sf_words ? __ldg(reinterpret_cast<const uint32_t*>(sr))
                          : (uint32_t)__ldg(sr) | (uint32_t)__ldg(sr + 1) << 8 | (uint32_t)__ldg(sr + 2) << 16 |
                                (uint32_t)__ldg(sr + 3) << 24;
        }
        const uint32_t f = h2_of_e4m3((sw >> (8 * b)) & 0xffu);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) pr[g][kk] = h2_mul(h2_of_e2m1((kk < 4 ? cw.x : cw.y) >> (8 * (kk & 3))), f);
        if (kPerRow && b == 0) {
            const int64_t gi = group_rows == 1 ? r : r / group_rows;
            so[16 * w + 8 * g + rho] = mx_in_range(gi, 1, rows / group_rows) ? __ldg(outer + gi) : 0.0f;
        }
    }
    // stmatrix call n: 8-row group g = n / 2 of the warp's rows, column groups kappa = 4 (n % 2) + j for its
    // matrices j = 0..3.  Thread (rho, b) holds fragment row rho, fragment columns 2b, 2b+1 = tile columns
    // 16b + 2 kappa + {0, 1}; stored row m of matrix j (address from lane 8j + m) is tile column
    // 16 (m / 2) + 2 kappa + m % 2, its 8 values the 8 rows of chunk 2w + g.
    const int j = lane >> 3, m = lane & 7;
#pragma unroll
    for (int n = 0; n < 4; ++n) {
        const int g = n >> 1, kap = 4 * (n & 1) + j;
        const int c = 16 * (m >> 1) + 2 * kap + (m & 1);
        const int kb = 4 * (n & 1);
        stmatrix_x4_trans(rq_chunk(tbase, c, 2 * w + g), pr[g][kb], pr[g][kb + 1], pr[g][kb + 2], pr[g][kb + 3]);
    }
}

// Phase 1 for a bf16 [rows, cols] source (16-byte aligned rows): the tile at
// (r0, c0) stored transposed, same layout as the NVFP4 products.  Warp w takes
// rows 16w .. 16w + 15 as units n = 0 .. 3 (rows 16w + 8 (n / 2) .., column
// half h = n % 2); lane (rho, b) loads the 8 columns 16b + 8h .. 16b + 8h + 7
// of its row (16 bytes), so its register k holds columns 16b + 2 (4h + k) + {0,
// 1}: the fragment layout rq_load_tile's stmatrix calls take.
__device__ __forceinline__ void rq_load_tile_bf16(const uint16_t* __restrict__ x, int64_t rows, int64_t cols,
                                                  int64_t r0, int64_t c0, uint32_t tbase) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int rho = lane >> 2, b = lane & 3;
    uint4 v[4];
#pragma unroll
    for (int n = 0; n < 4; ++n) {
        const int64_t r = r0 + 16 * w + 8 * (n >> 1) + rho;
        const int64_t xi = r * cols + c0 + 16 * b + 8 * (n & 1);
        v[n] = mx_in_range(xi, 8, rows * cols) ? __ldcs(reinterpret_cast<const uint4*>(x + xi))
                                                : make_uint4(0u, 0u, 0u, 0u);
    }
    const int j = lane >> 3, m = lane & 7;
#pragma unroll
    for (int n = 0; n < 4; ++n) {
        const int c = 16 * (m >> 1) + 2 * (4 * (n & 1) + j) + (m & 1);
        stmatrix_x4_trans(rq_chunk(tbase, c, 2 * w + (n >> 1)), v[n].x, v[n].y, v[n].z, v[n].w);
    }
}

// Phase 2 lane map: lane (m = lane % 8, jj = (lane / 8) % 2, q = lane / 16) of
// warp w takes tile column (output row) c = 16 (m / 2) + 2w + m % 2 and, in
// its pass it = 0, 1, input rows 16j .. 16j + 15 with j = 2 (2 it + q) + jj.
struct RqLane {
    int m, jj, q, c;
    __device__ __forceinline__ RqLane() {
        const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
        m = lane & 7;
        jj = (lane >> 3) & 1;
        q = lane >> 4;
        c = 16 * (m >> 1) + 2 * w + (m & 1);
    }
    __device__ __forceinline__ int chunk(int it) const { return 2 * (2 * it + q) + jj; }
};

// The 16 f16 products of input rows 16j .. 16j + 15, tile column c.
__device__ __forceinline__ void rq_read16(uint32_t tbase, int c, int j, uint32_t hw[8]) {
    const uint4 v0 = lds_v4(rq_chunk(tbase, c, 2 * j));
    const uint4 v1 = lds_v4(rq_chunk(tbase, c, 2 * j + 1));
    hw[0] = v0.x; hw[1] = v0.y; hw[2] = v0.z; hw[3] = v0.w;
    hw[4] = v1.x; hw[5] = v1.y; hw[6] = v1.z; hw[7] = v1.w;
}

// max |p| over the 16 f16 products (as fp32, exact).
__device__ __forceinline__ float rq_maxabs16(const uint32_t hw[8]) {
    const uint32_t hm = h2_maxabs(h2_maxabs(h2_maxabs(hw[0], hw[1]), h2_maxabs(hw[2], hw[3])),
                                  h2_maxabs(h2_maxabs(hw[4], hw[5]), h2_maxabs(hw[6], hw[7])));
    float ml, mh;
    h2_to_f32x2(hm, ml, mh);
    return fmaxf(fabsf(ml), fabsf(mh));
}

}  // namespace
