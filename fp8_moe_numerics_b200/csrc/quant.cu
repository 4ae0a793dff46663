// quant.cu -- the NVFP4 quantiser (round-to-nearest and stochastic forms,
// SwiGLU fused in front for the activations), the MXFP8 quantiser (and its form
// that builds the combine's gradient rows itself), and the NVFP4 -> MXFP8
// stochastic requantisation across a transpose (sm_100a).
//
// All are written as HBM streams: 128-bit coalesced loads and stores, amax by
// packed-integer max and warp shuffles, every rounding decision taken by a PTX
// cvt or by exact integer arithmetic (see mx_common.cuh).
#include "mx_common.cuh"
#include "requant_tile.cuh"
#include "e2m1_sr.cuh"

#include <cuda.h>

namespace {

// Max of |bf16| over the 8 elements of a uint4, as the bf16 magnitude bits
// (integer order equals numeric order for non-NaN magnitudes).
__device__ __forceinline__ uint32_t absmax8_bf16(const uint4& v) {
    uint32_t m = __vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu);
    m = __vmaxu2(m, v.z & 0x7fff7fffu);
    m = __vmaxu2(m, v.w & 0x7fff7fffu);
    return max(m & 0xffffu, m >> 16);
}

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Random bits of the stochastically rounded form (nvfp4_quantize_sr): key,
// Philox stream and the linear index of the block's first element.
struct SrKey {
    uint64_t seed, stream;
};

// Quantise one 16-element block (two uint4 of bf16) with outer scale s > 0;
// ab_bits = the block's max |x| as bf16 magnitude bits (callers have it from
// the row amax).  Returns the E4M3 scale code; writes 8 bytes of E2M1 codes,
// to nearest or (kR > 0) rounded stochastically with kR random bits of the
// elements' linear indices L0 ...
template <int kR = 0>
__device__ __forceinline__ uint32_t nvfp4_block(const uint4& a, const uint4& b, uint32_t ab_bits, float s,
                                                uint2& packed, SrKey key = {}, uint64_t L0 = 0) {
    float ab = __uint_as_float(ab_bits << 16);
    float t = __fmul_rn(6.0f, s);
    float d = __fdiv_rn(ab, t);
    uint32_t sc = cvt_e4m3x2(d, 0.0f) & 0xffu;
    if (sc == 0) { packed = make_uint2(0u, 0u); return 0u; }
    float inv = __frcp_rn(__fmul_rn(e4m3_to_f32(sc), s));
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    const uint64_t inv2 = f2_pack(inv, inv);
    if constexpr (kR > 0) {
        float y[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            y[2 * i] = bf16_lo(w[i]);
            y[2 * i + 1] = bf16_hi(w[i]);
            mul2_rn(y[2 * i], y[2 * i + 1], inv2);
        }
        packed = e2m1_sr_codes<kR>(y, key.seed, key.stream, L0);
    } else {
        uint32_t word[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {                  // eight products (in pairs), then their code word
            float y[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                y[2 * i] = bf16_lo(w[4 * h + i]);
                y[2 * i + 1] = bf16_hi(w[4 * h + i]);
                mul2_rn(y[2 * i], y[2 * i + 1], inv2);
            }
            word[h] = cvt_e2m1x8(y);
        }
        packed = make_uint2(word[0], word[1]);
    }
    return sc;
}

// Codes and scale of block `blk` of `row` (outer scale s); every lane of the
// warp calls it, live or not, because the scale bytes of four consecutive
// blocks (in lanes 4m..4m+3) are merged by shuffles into one 32-bit store
// when `word_sf`.
template <int kLayout, int kR = 0>
__device__ __forceinline__ void emit_nvfp4_block(int64_t row, int64_t blk, int64_t nblk, bool active, float s,
                                                 const uint4& a, const uint4& b, uint32_t ab_bits,
                                                 uint8_t* __restrict__ crow, uint8_t* __restrict__ sf, bool word_sf,
                                                 int lane, SrKey key = {}) {
    uint2 packed = make_uint2(0u, 0u);
    uint32_t sc = 0;
    const bool live = active && blk < nblk;
    if (live && s > 0.0f) sc = nvfp4_block<kR>(a, b, ab_bits, s, packed, key, (uint64_t)((row * nblk + blk) * 16));
    if (live) *reinterpret_cast<uint2*>(crow + blk * 8) = packed;
    if (word_sf) {
        uint32_t w = sc << (8 * (lane & 3));
        w |= __shfl_xor_sync(0xffffffffu, w, 1);
        w |= __shfl_xor_sync(0xffffffffu, w, 2);
        if (live && (lane & 3) == 0) *reinterpret_cast<uint32_t*>(sf + sf_offset(row, blk, nblk, kLayout)) = w;
    } else if (live) {
        sf[sf_offset(row, blk, nblk, kLayout)] = (uint8_t)sc;
    }
}

// kTPR threads per row (a power of two, 16..256), 256 / kTPR rows per block.
// Thread j of a row handles the 16-element blocks j, j + kTPR, ... (kNB of
// them held in registers when the row fits, so each warp's loads cover
// contiguous bytes); longer rows are read twice.  The row amax is reduced by
// warp shuffles and, across the row's warps, through shared memory.  Scale
// bytes of four consecutive blocks are merged by shuffles into one 32-bit
// store when the row has a multiple of four blocks (`word_sf`).
// GROUP: the outer scale is per group of rows and `outer` already holds the
// group's amax bits (written by nvfp4_group_amax_kernel).
constexpr int kRowThreads = 256;

// Rows [block * 256/kTPR, +256/kTPR) of x, those below row_end.
template <int kTPR, int kNB, bool kGroup, int kLayout, int kR = 0>
__device__ __forceinline__ void quant_rows_block(const uint16_t* __restrict__ x, int64_t rows, int64_t row_end,
                                                 int64_t cols, int64_t group_rows, bool word_sf,
                                                 uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                                 float* __restrict__ outer, int64_t block, uint32_t* wmax,
                                                 SrKey key = {}) {
    constexpr int kRPB = kRowThreads / kTPR;
    const int lane = threadIdx.x & 31;
    const int j = threadIdx.x % kTPR;
    const int64_t row = block * kRPB + threadIdx.x / kTPR;
    const bool active = row < row_end;
    const int64_t nblk = cols >> 4;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (active ? row : 0) * cols);

    uint4 va[kNB], vb[kNB];
    uint32_t bmax[kNB];                                 // each block's max |x| (bf16 magnitude bits)
    uint32_t amax_bits = 0;
    const bool resident = nblk <= (int64_t)kTPR * kNB;
#pragma unroll
    for (int i = 0; i < kNB; ++i) {
        const int64_t blk = j + (int64_t)kTPR * i;
        va[i] = make_uint4(0, 0, 0, 0);
        vb[i] = va[i];
        if (active && resident && blk < nblk) {
            va[i] = __ldcs(xr + 2 * blk);
            vb[i] = __ldcs(xr + 2 * blk + 1);
        }
    }
#pragma unroll
    for (int i = 0; i < kNB; ++i) {
        bmax[i] = max(absmax8_bf16(va[i]), absmax8_bf16(vb[i]));
        amax_bits = max(amax_bits, bmax[i]);
    }
    if (active && !resident) {
        for (int64_t blk = j; blk < nblk; blk += kTPR)
            amax_bits = max(amax_bits, max(absmax8_bf16(xr[2 * blk]), absmax8_bf16(xr[2 * blk + 1])));
    }

    float s;
    if (kGroup) {
        const int64_t g = rows < ((int64_t)1 << 32) ? (int64_t)((uint32_t)row / (uint32_t)group_rows) : row / group_rows;
        s = active ? __fdiv_rn(outer[g], 2688.0f) : 0.0f;
    } else {
        if (kTPR >= 32) {
            amax_bits = warp_max_u32(amax_bits);
        } else {                                          // rows of kTPR lanes inside a warp
#pragma unroll
            for (int o = kTPR / 2; o > 0; o >>= 1) amax_bits = max(amax_bits, __shfl_xor_sync(0xffffffffu, amax_bits, o));
        }
        if (kTPR > 32) {
            if (lane == 0) wmax[threadIdx.x >> 5] = amax_bits;
            __syncthreads();
            const int w0 = (threadIdx.x / kTPR) * (kTPR / 32);
#pragma unroll
            for (int w = 0; w < kTPR / 32; ++w) amax_bits = max(amax_bits, wmax[w0 + w]);
        }
        s = __fdiv_rn(__uint_as_float(amax_bits << 16), 2688.0f);
        if (active && j == 0) outer[row] = s;
    }

    uint8_t* crow = codes + (active ? row : 0) * (cols >> 1);
    auto emit = [&](int64_t blk, const uint4& a, const uint4& b, uint32_t ab_bits) {
        emit_nvfp4_block<kLayout, kR>(row, blk, nblk, active, s, a, b, ab_bits, crow, sf, word_sf, lane, key);
    };
    if (resident) {
#pragma unroll
        for (int i = 0; i < kNB; ++i) emit(j + (int64_t)kTPR * i, va[i], vb[i], bmax[i]);
    } else {
        const int64_t nb_pad = (nblk + kTPR - 1) / kTPR * kTPR;   // every lane runs every shuffle
        for (int64_t blk = j; blk < nb_pad; blk += kTPR) {
            const bool in = active && blk < nblk;
            const uint4 a = in ? xr[2 * blk] : make_uint4(0, 0, 0, 0), b = in ? xr[2 * blk + 1] : make_uint4(0, 0, 0, 0);
            emit(blk, a, b, max(absmax8_bf16(a), absmax8_bf16(b)));
        }
    }
}

template <int kTPR, int kNB, bool kGroup, int kLayout, int kR = 0>
__global__ void __launch_bounds__(kRowThreads, kNB <= 4 ? 4 : 2)
nvfp4_quant_rows_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t group_rows,
                        bool word_sf, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, float* __restrict__ outer,
                        SrKey key) {
    __shared__ uint32_t wmax[kRowThreads / 32];
    quant_rows_block<kTPR, kNB, kGroup, kLayout, kR>(x, rows, rows, cols, group_rows, word_sf, codes, sf, outer,
                                                     (int64_t)blockIdx.x, wmax, key);
}

// SwiGLU fused into the per-token NVFP4 quantiser: the activation a =
// silu(g) * u of each element is formed in registers exactly as swiglu_fwd
// writes it (swiglu_word, bf16 round-to-nearest) and quantised as
// nvfp4_quant_rows_kernel quantises a bf16 row, so the result equals the two
// kernels run one after the other, without a's round trip through HBM.
// h = [g | u] (gated, [rows, 2F]) or [g] ([rows, F], u = 1).  Rows at or past
// *rows_valid are zero rows (codes 0, scales 0, outer 0).  Rows must fit in
// registers: F/16 <= 4 kTPR.
template <int kTPR, int kLayout>
__global__ void __launch_bounds__(kRowThreads, 4)
swiglu_nvfp4_rows_kernel(const uint16_t* __restrict__ h, int64_t rows, int64_t F, int gated, const int64_t* rows_valid,
                         bool word_sf, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                         float* __restrict__ outer) {
    constexpr int kNB = 4;
    constexpr int kRPB = kRowThreads / kTPR;
    __shared__ uint32_t wmax[kRowThreads / 32];
    const int lane = threadIdx.x & 31;
    const int j = threadIdx.x % kTPR;
    const int64_t row = (int64_t)blockIdx.x * kRPB + threadIdx.x / kTPR;
    const bool active = row < rows;
    const bool live = active && row < load_rows_valid(rows_valid, rows);
    const int64_t nblk = F >> 4;
    const int64_t hw = gated ? 2 * F : F;
    const uint4* gr = reinterpret_cast<const uint4*>(h + (live ? row : 0) * hw);
    const uint4* ur = reinterpret_cast<const uint4*>(h + (live ? row : 0) * hw + F);
    const uint4 one = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);   // bf16 1.0
    uint4 va[kNB], vb[kNB];
    uint32_t bmax[kNB];
    uint32_t amax_bits = 0;
#pragma unroll
    for (int i = 0; i < kNB; ++i) {
        const int64_t blk = j + (int64_t)kTPR * i;
        va[i] = make_uint4(0, 0, 0, 0);
        vb[i] = va[i];
        if (live && blk < nblk) {
            const uint4 g0 = __ldcs(gr + 2 * blk), g1 = __ldcs(gr + 2 * blk + 1);
            const uint4 u0 = gated ? __ldcs(ur + 2 * blk) : one, u1 = gated ? __ldcs(ur + 2 * blk + 1) : one;
            va[i] = make_uint4(swiglu_word(g0.x, u0.x), swiglu_word(g0.y, u0.y), swiglu_word(g0.z, u0.z),
                               swiglu_word(g0.w, u0.w));
            vb[i] = make_uint4(swiglu_word(g1.x, u1.x), swiglu_word(g1.y, u1.y), swiglu_word(g1.z, u1.z),
                               swiglu_word(g1.w, u1.w));
        }
        bmax[i] = max(absmax8_bf16(va[i]), absmax8_bf16(vb[i]));
        amax_bits = max(amax_bits, bmax[i]);
    }
    if (kTPR >= 32) {
        amax_bits = warp_max_u32(amax_bits);
    } else {
#pragma unroll
        for (int o = kTPR / 2; o > 0; o >>= 1) amax_bits = max(amax_bits, __shfl_xor_sync(0xffffffffu, amax_bits, o));
    }
    if (kTPR > 32) {
        if (lane == 0) wmax[threadIdx.x >> 5] = amax_bits;
        __syncthreads();
        const int w0 = (threadIdx.x / kTPR) * (kTPR / 32);
#pragma unroll
        for (int w = 0; w < kTPR / 32; ++w) amax_bits = max(amax_bits, wmax[w0 + w]);
    }
    const float s = __fdiv_rn(__uint_as_float(amax_bits << 16), 2688.0f);
    if (active && j == 0) outer[row] = s;
    uint8_t* crow = codes + (active ? row : 0) * (F >> 1);
#pragma unroll
    for (int i = 0; i < kNB; ++i)
        emit_nvfp4_block<kLayout>(row, j + (int64_t)kTPR * i, nblk, active, s, va[i], vb[i], bmax[i], crow, sf, word_sf,
                                  lane);
}

// amax over each group of rows, as fp32 bits, atomically max-ed into outer[g]
// (pre-zeroed).  blockIdx.y = group, blockIdx.x = chunk of the group's
// contiguous elements; each thread keeps four 16-byte loads in flight and the
// block issues one atomic.
constexpr int kAmaxThreads = 256, kAmaxUnroll = 4;

// One chunk [v0, v1) of group g's 16-byte vectors (streaming loads).
__device__ __forceinline__ void group_amax_chunk(const uint16_t* __restrict__ x, int64_t g, int64_t group_vec,
                                                 int64_t v0, int64_t v1, float* __restrict__ outer, uint32_t* wm) {
    const uint4* xv = reinterpret_cast<const uint4*>(x) + g * group_vec;
    uint32_t m = 0;
    for (int64_t v = v0 + threadIdx.x; v < v1; v += kAmaxThreads * kAmaxUnroll) {
        uint4 q[kAmaxUnroll];
#pragma unroll
        for (int u = 0; u < kAmaxUnroll; ++u) {
            const int64_t idx = v + (int64_t)u * kAmaxThreads;
            q[u] = idx < v1 ? __ldcs(xv + idx) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kAmaxUnroll; ++u) m = max(m, absmax8_bf16(q[u]));
    }
    m = warp_max_u32(m);
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = 0;
        for (int w = 0; w < kAmaxThreads / 32; ++w) b = max(b, wm[w]);
        atomicMax(reinterpret_cast<unsigned int*>(outer) + g, b << 16);
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kAmaxThreads)
nvfp4_group_amax_kernel(const uint16_t* __restrict__ x, int64_t ngroups, int64_t group_vec, int64_t chunk_vec,
                        float* __restrict__ outer) {
    __shared__ uint32_t wm[kAmaxThreads / 32];
    for (int64_t g = blockIdx.y; g < ngroups; g += gridDim.y) {
        const int64_t v0 = (int64_t)blockIdx.x * chunk_vec;
        group_amax_chunk(x, g, group_vec, v0, min(group_vec, v0 + chunk_vec), outer, wm);
    }
}

__global__ void nvfp4_group_finish_kernel(float* outer, int64_t ngroups) {
    int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g < ngroups) outer[g] = __fdiv_rn(outer[g], 2688.0f);
}

// ---------------------------------------------------------------------------
// Transpose tile of the register-prefetch MXFP8 quantiser: 128 rows x 64
// columns of the bf16 input.  Phase 1 loads the tile -- thread t owns row t/2, columns
// 32*(t%2) .. +31 -- and stores fp32 values transposed into shared memory
// T[c][r] (128 words per row c).  Phase 2: thread (c, g) takes output row c,
// elements r = 16g .. 16g+15 as four 16-byte chunks (8 threads cover the
// tile's 128 r of row c); lane pairs (g, g^1) form one 32-element MXFP8 block.
// Swizzle: the 16-byte chunk j of group g sits at chunk j ^ ((g/2)%4), and
// columns c >= 32 flip r's bit 4, so phase-1 scalar stores (16 rows x 2
// column halves per warp) and phase-2 16-byte loads (8 groups of one row per
// quarter warp) are both free of bank conflicts.
// ---------------------------------------------------------------------------
constexpr int kTR = 128, kTC = 64, kTileThreads = 256;
static_assert(kTR == kRqRows && kTC == kRqCols && kTileThreads == kRqThreads, "one tile shape");

__device__ __forceinline__ int tsw(int c, int r) {
    const int rs = (r & ~12) | ((((r >> 2) & 3) ^ ((r >> 5) & 3)) << 2);
    return c * kTR + (rs ^ ((c >> 5) << 4));
}

// Phase 2: from smem T to MXFP8 codes of the transposed output.
// kSR: stochastic rounding with kR random bits, else RNE.
template <bool kSR, int kR, int kLayout>
__device__ __forceinline__ void tile_emit_transposed(const float* T, int64_t rows, int64_t cols, int64_t r0, int64_t c0,
                                                     uint64_t seed, uint64_t stream_id,
                                                     uint8_t* __restrict__ out_codes, uint8_t* __restrict__ out_e8m0) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane & 7;
    const int64_t S = rows >> 5;                        // output scales per output row
#pragma unroll
    for (int it = 0; it < 2; ++it) {
        const int c = it * 32 + warp * 4 + (lane >> 3);
        float v[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 q = *reinterpret_cast<const float4*>(T + tsw(c, 16 * g + 4 * j));
            v[4 * j + 0] = q.x; v[4 * j + 1] = q.y; v[4 * j + 2] = q.z; v[4 * j + 3] = q.w;
        }
        float mf = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) mf = fmaxf(mf, fabsf(v[i]));
        mf = fmaxf(mf, __shfl_xor_sync(0xffffffffu, mf, 1));
        const int e = e8m0_exponent(mf);
        const SrBlock sb = sr_block(e);
        const int64_t cg = c0 + c;
        const int64_t rr = r0 + 16 * g;
        uint32_t w[4];
        if (kSR && kR == 16) {
            // hardware stochastic rounding, two elements per instruction
            const int64_t L0 = cg * rows + rr;          // output element index
            const float sc = exp2_neg(e);
            const uint64_t sc2 = f2_pack(sc, sc);
#pragma unroll
            for (int blk = 0; blk < 2; ++blk) {
                const uint4 rnd = philox4x32_10((uint64_t)(L0 / 8) + blk, stream_id, seed);
                const uint32_t wd[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
#pragma unroll
                for (int q = 0; q < 4; q += 2) {       // elements i..i+3 use words q, q+1
                    const int i = blk * 8 + 2 * q;
                    float a0 = v[i], a1 = v[i + 1], a2 = v[i + 2], a3 = v[i + 3];
                    mul2_rn(a0, a1, sc2);
                    mul2_rn(a2, a3, sc2);
                    w[blk * 2 + (q >> 1)] = cvt_rs16_e4m3_quad(a0, a1, a2, a3, wd[q], wd[q + 1]);
                }
            }
        } else if (kSR) {
            const int64_t L0 = cg * rows + rr;          // output element index
            constexpr int kPer = 128 / kR;              // elements per Philox block
#pragma unroll
            for (int blk = 0; blk < 16 / kPer + (16 % kPer ? 1 : 0); ++blk) {
                const uint4 rnd = philox4x32_10((uint64_t)(L0 / kPer) + blk, stream_id, seed);
#pragma unroll
                for (int jj = 0; jj < kPer && blk * kPer + jj < 16; ++jj) {
                    const int i = blk * kPer + jj;
                    const uint32_t code = e4m3_sr_code<kR>(v[i], sb, philox_field<kR>(rnd, jj));
                    if ((i & 3) == 0) w[i >> 2] = code; else w[i >> 2] |= code << (8 * (i & 3));
                }
            }
        } else {
            const float sc = exp2_neg(e);
            const uint64_t sc2 = f2_pack(sc, sc);
#pragma unroll
            for (int i = 0; i < 4; ++i)
            {
                float a0 = v[4 * i], a1 = v[4 * i + 1], a2 = v[4 * i + 2], a3 = v[4 * i + 3];
                mul2_rn(a0, a1, sc2);
                mul2_rn(a2, a3, sc2);
                w[i] = cvt_e4m3x4(a0, a1, a2, a3);
            }
        }
        if (mx_in_range(cg * rows + rr, 16, cols * rows))
            *reinterpret_cast<uint4*>(out_codes + cg * rows + rr) = make_uint4(w[0], w[1], w[2], w[3]);
        if ((g & 1) == 0 && mx_in_range(sf_offset(cg, rr >> 5, S, kLayout), 1, cols * S))
            out_e8m0[sf_offset(cg, rr >> 5, S, kLayout)] = (uint8_t)(e + 127);
    }
}

// MXFP8 quantisation of bf16 [rows, cols]: row-wise blocks (phase 1, straight
// from registers) and/or the transposed column-wise form (phase 2).  Blocks
// loop over 128x64 tiles (column tiles fastest) and load the next tile's
// values into registers before the current tile's transposed phase.
template <bool kRow, bool kCol, bool kSR, int kR, int kLayout>
__global__ void __launch_bounds__(kTileThreads, 4)
mxfp8_tile_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, const int64_t* rows_valid,
                  uint64_t seed, uint64_t stream_row, uint64_t stream_col,
                  uint8_t* __restrict__ row_codes, uint8_t* __restrict__ row_e8m0,
                  uint8_t* __restrict__ col_codes, uint8_t* __restrict__ col_e8m0) {
    __shared__ __align__(16) float T[kCol ? kTC * kTR : 4];
    const int64_t tiles_c = cols / kTC;
    const int64_t ntiles = tiles_c * ((load_rows_valid(rows_valid, rows) + kTR - 1) / kTR);
    int64_t tile = blockIdx.x;
    if (tile >= ntiles) return;
    const int t = threadIdx.x;
    const int rl = t >> 1, h = t & 1;
    uint4 q[4];
    auto fetch = [&](int64_t tl) {
        const int64_t c0 = (tl % tiles_c) * kTC, r = (tl / tiles_c) * kTR + rl;
        const uint4* src = reinterpret_cast<const uint4*>(x + r * cols + c0 + 32 * h);
#pragma unroll
        for (int i = 0; i < 4; ++i) q[i] = __ldcs(src + i);
    };
    fetch(tile);
    for (; tile < ntiles; tile += gridDim.x) {
        const int64_t c0 = (tile % tiles_c) * kTC, r0 = (tile / tiles_c) * kTR;
        const int64_t r = r0 + rl;
        float v[32];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t w[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) { v[8 * i + 2 * j] = bf16_lo(w[j]); v[8 * i + 2 * j + 1] = bf16_hi(w[j]); }
        }
        if (kRow) {
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) m = max(m, absmax8_bf16(q[i]));
            const int e = e8m0_exponent(__uint_as_float(m << 16));
            uint32_t w[8];
            const int64_t L0 = r * cols + c0 + 32 * h;
            if (kSR && kR == 16) {
                const float sc = exp2_neg(e);
                const uint64_t sc2 = f2_pack(sc, sc);
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) {
                    const uint4 rnd = philox4x32_10((uint64_t)(L0 / 8) + blk, stream_row, seed);
                    const uint32_t wd[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
#pragma unroll
                    for (int q = 0; q < 4; q += 2) {
                        const int i = blk * 8 + 2 * q;
                        float a0 = v[i], a1 = v[i + 1], a2 = v[i + 2], a3 = v[i + 3];
                        mul2_rn(a0, a1, sc2);
                        mul2_rn(a2, a3, sc2);
                        w[blk * 2 + (q >> 1)] = cvt_rs16_e4m3_quad(a0, a1, a2, a3, wd[q], wd[q + 1]);
                    }
                }
            } else if (kSR) {
                constexpr int kPer = 128 / kR;
#pragma unroll
                for (int blk = 0; blk < 32 / kPer; ++blk) {
                    const uint4 rnd = philox4x32_10((uint64_t)(L0 / kPer) + blk, stream_row, seed);
#pragma unroll
                    for (int jj = 0; jj < kPer; ++jj) {
                        const int i = blk * kPer + jj;
                        const uint32_t code = e4m3_sr_code<kR>(v[i], e, philox_field<kR>(rnd, jj));
                        if ((i & 3) == 0) w[i >> 2] = code; else w[i >> 2] |= code << (8 * (i & 3));
                    }
                }
            } else {
                const float sc = exp2_neg(e);
                const uint64_t sc2 = f2_pack(sc, sc);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                {
                    float a0 = v[4 * i], a1 = v[4 * i + 1], a2 = v[4 * i + 2], a3 = v[4 * i + 3];
                    mul2_rn(a0, a1, sc2);
                    mul2_rn(a2, a3, sc2);
                    w[i] = cvt_e4m3x4(a0, a1, a2, a3);
                }
            }
            uint4* dst = reinterpret_cast<uint4*>(row_codes + L0);
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
            row_e8m0[sf_offset(r, (c0 >> 5) + h, cols >> 5, kLayout)] = (uint8_t)(e + 127);
        }
        if (kCol) {
#pragma unroll
            for (int i = 0; i < 32; ++i) T[tsw(32 * h + i, rl)] = v[i];
            __syncthreads();
            if (tile + gridDim.x < ntiles) fetch(tile + gridDim.x);
            tile_emit_transposed<kSR, kR, kLayout>(T, rows, cols, r0, c0, seed, stream_col, col_codes, col_e8m0);
            __syncthreads();                               // T is rewritten by the next tile
        } else if (tile + gridDim.x < ntiles) {
            fetch(tile + gridDim.x);
        }
    }
}


// ---------------------------------------------------------------------------
// MXFP8 (RNE) row and column forms of the dispatch gradient, formed on the fly
// from the upstream gradient and the routing so that dY itself never goes
// through HBM.  The row form is mxfp8_tile_kernel's; the column form is the
// TMA quantiser's (the tile as bf16 column pairs in two buffers, one barrier
// per tile; measured on B200 5% faster than an fp32 tile with two barriers).
// Each thread's row is gathered from its token's row of dout (the next tile's
// loads issued before the current tile's transposed phase, their scaling at
// the top of the next iteration).  Every value is w * dout rounded to bf16 by
// the definition moe_dispatch_grad uses (scaled_bf16_word), so the codes equal
// those of moe_dispatch_grad and mxfp8_quantize run one after the other.
// Row p holds w[s] * dout[s / k] for s = src[p] >= 0, else zeros; a token's
// row is read by its k rows (kept in L2).
// ---------------------------------------------------------------------------
struct DispatchGradRows {
    const uint16_t* dout;
    const int32_t* src;
    const float* w;
    int64_t Tk, k, D;
    struct Raw {
        uint4 v[4];
        float wt;
        bool live;
    };
    // the thread's 32 columns c .. c + 31 of row r
    __device__ __forceinline__ void issue(int64_t r, int64_t c, int64_t valid, Raw& q) const {
        q.live = false;
        if (r >= valid) return;
        const int64_t s = __ldg(src + r);
        if (s < 0 || s >= Tk || !mx_in_range((s / k) * D + c, 32, (Tk / k) * D)) return;
        q.live = true;
        q.wt = w ? __ldg(w + s) : 1.0f;
        const uint4* vp = reinterpret_cast<const uint4*>(dout + (s / k) * D + c);
#pragma unroll
        for (int i = 0; i < 4; ++i) q.v[i] = __ldg(vp + i);
    }
    __device__ __forceinline__ void finish(const Raw& q, uint4* out) const {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            out[i] = q.live ? make_uint4(scaled_bf16_word(q.wt, q.v[i].x), scaled_bf16_word(q.wt, q.v[i].y),
                                         scaled_bf16_word(q.wt, q.v[i].z), scaled_bf16_word(q.wt, q.v[i].w))
                            : make_uint4(0u, 0u, 0u, 0u);
    }
};

// word (cp, r) of a transposed bf16 tile: columns 2cp, 2cp + 1 of row r (the TMA quantiser's layout)
__device__ __forceinline__ int dq_t2_word(int cp, int r) {
    int rr = r ^ ((cp >> 4) << 4);
    rr ^= ((rr >> 5) & 3) << 2;
    return cp * kTR + rr;
}

// Three blocks per SM (78-80 registers, no spills): measured on B200 10% faster than two (the
// gathers' latency is what bounds it) and than four (which spills).
template <int kLayout>
__global__ void __launch_bounds__(kTileThreads, 3)
dispatch_grad_mxfp8_kernel(DispatchGradRows src, int64_t rows, int64_t cols, const int64_t* rows_valid,
                           uint8_t* __restrict__ row_codes, uint8_t* __restrict__ row_e8m0,
                           uint8_t* __restrict__ col_codes, uint8_t* __restrict__ col_e8m0) {
    __shared__ __align__(16) uint32_t T2d[2 * (kTC / 2) * kTR];      // double-buffered bf16 column pairs
    // Row tiles vary fastest: the blocks in flight gather the same 64-column
    // slice of dout for rows of every expert, so that slice of all tokens (T x
    // 128 B, a few MB) stays in L2 while each token's k routed rows read it.
    // (Column tiles fastest, the blocks in flight read whole 8 KB token rows
    // and a token's other routed rows come back after they left L2.)
    const int64_t valid = load_rows_valid(rows_valid, rows);
    const int64_t tiles_r = (valid + kTR - 1) / kTR;
    const int64_t ntiles = (cols / kTC) * tiles_r;
    int64_t tile = blockIdx.x;
    if (tile >= ntiles) return;
    const int t = threadIdx.x;
    const int rl = t >> 1, h = t & 1;
    const int cp = t >> 3, g = t & 7;
    int buf = 0;
    DispatchGradRows::Raw raw;
    auto issue = [&](int64_t tl) { src.issue((tl % tiles_r) * kTR + rl, (tl / tiles_r) * kTC + 32 * h, valid, raw); };
    issue(tile);
    for (; tile < ntiles; tile += gridDim.x) {
        const int64_t c0 = (tile / tiles_r) * kTC, r0 = (tile % tiles_r) * kTR;
        const int64_t r = r0 + rl, c = c0 + 32 * h;
        uint4 q[4];
        src.finish(raw, q);
        float v[32];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t w[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) { v[8 * i + 2 * j] = bf16_lo(w[j]); v[8 * i + 2 * j + 1] = bf16_hi(w[j]); }
        }
        {                                                  // row-wise block, RNE (as mxfp8_tile_kernel)
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) m = max(m, absmax8_bf16(q[i]));
            const int e = e8m0_exponent(__uint_as_float(m << 16));
            const float sc = exp2_neg(e);
            const uint64_t sc2 = f2_pack(sc, sc);
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float a0 = v[4 * i], a1 = v[4 * i + 1], a2 = v[4 * i + 2], a3 = v[4 * i + 3];
                mul2_rn(a0, a1, sc2);
                mul2_rn(a2, a3, sc2);
                w[i] = cvt_e4m3x4(a0, a1, a2, a3);
            }
            if (mx_in_range(r * cols + c, 32, rows * cols)) {
                uint4* dst = reinterpret_cast<uint4*>(row_codes + r * cols + c);
                dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
            }
            if (mx_in_range(sf_offset(r, c >> 5, cols >> 5, kLayout), 1, rows * (cols >> 5)))
                row_e8m0[sf_offset(r, c >> 5, cols >> 5, kLayout)] = (uint8_t)(e + 127);
        }
        // column form: the tile as bf16 column pairs (the values are bf16 already), one barrier per
        // tile with two buffers, then thread (cp, g) emits 16 rows of columns 2cp and 2cp + 1
        uint32_t* Tb = T2d + buf * (kTC / 2) * kTR;
        {
            const uint32_t wq[16] = {q[0].x, q[0].y, q[0].z, q[0].w, q[1].x, q[1].y, q[1].z, q[1].w,
                                     q[2].x, q[2].y, q[2].z, q[2].w, q[3].x, q[3].y, q[3].z, q[3].w};
#pragma unroll
            for (int j = 0; j < 16; ++j) Tb[dq_t2_word(16 * h + j, rl)] = wq[j];
        }
        __syncthreads();
        if (tile + gridDim.x < ntiles) issue(tile + gridDim.x);
        uint32_t a[16];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const uint4 u = *reinterpret_cast<const uint4*>(Tb + dq_t2_word(cp, 16 * g + 4 * kk));
            a[4 * kk] = u.x; a[4 * kk + 1] = u.y; a[4 * kk + 2] = u.z; a[4 * kk + 3] = u.w;
        }
        const int64_t rr = r0 + 16 * g;
        const int64_t S = rows >> 5;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float cv[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) cv[m] = half ? bf16_hi(a[m]) : bf16_lo(a[m]);
            float mf = 0.0f;
#pragma unroll
            for (int m = 0; m < 16; ++m) mf = fmaxf(mf, fabsf(cv[m]));
            mf = fmaxf(mf, __shfl_xor_sync(0xffffffffu, mf, 1));
            const int e = e8m0_exponent(mf);
            const float sc = exp2_neg(e);
            const uint64_t sc2 = f2_pack(sc, sc);
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float a0 = cv[4 * i], a1 = cv[4 * i + 1], a2 = cv[4 * i + 2], a3 = cv[4 * i + 3];
                mul2_rn(a0, a1, sc2);
                mul2_rn(a2, a3, sc2);
                w[i] = cvt_e4m3x4(a0, a1, a2, a3);
            }
            const int64_t cg = c0 + 2 * cp + half;
            if (mx_in_range(cg * rows + rr, 16, cols * rows))
                *reinterpret_cast<uint4*>(col_codes + cg * rows + rr) = make_uint4(w[0], w[1], w[2], w[3]);
            if ((g & 1) == 0 && mx_in_range(sf_offset(cg, rr >> 5, S, kLayout), 1, cols * S))
                col_e8m0[sf_offset(cg, rr >> 5, S, kLayout)] = (uint8_t)(e + 127);
        }
        buf ^= 1;
    }
}

// ---------------------------------------------------------------------------
// MXFP8 quantiser (RNE), fed by TMA.  A persistent block of 8 consumer warps
// and one producer warp walks the same 128 x 64 tiles as mxfp8_tile_kernel.
// The producer's lane 0 keeps kQStages bf16 tiles in flight with 2-D TMA
// loads (128-byte swizzle) into a ring of shared-memory stages, so the
// consumers never wait on a global load of their own.  Per tile:
//   phase 1  thread (row t/2, half t%2) reads its 64 bytes of the row from the
//            stage, releases the stage, quantises them row-wise, and stores the
//            16 words (pairs of columns) into the transposed tile T2.
//   phase 2  after one barrier of the consumer warps, thread (column pair
//            t/8, row group t%8) reads 16 rows x 2 columns of T2 and emits two
//            16-row halves of column-wise MXFP8 blocks (lanes g, g^1 form one
//            32-row block).
// T2 is double-buffered, so the next tile's phase 1 needs no second barrier:
// a warp still in phase 2 of tile i reads the other buffer, and phase 1 of
// tile i+2 comes after every warp has passed tile i+1's barrier.  T2 holds
// word (cp, r) = columns 2cp, 2cp+1 of row r; column pairs 16..31 flip row
// bit 4 and every 4-word chunk index is XOR-ed with row/32, which keeps the
// phase-1 stores and the phase-2 16-byte loads free of bank conflicts.
// Waits are bounded (2 s): on expiry the status word records a timeout and
// the block stops.
// ---------------------------------------------------------------------------
#ifndef MX_Q_STAGES
#define MX_Q_STAGES 4          // bf16 tiles in flight per block
#endif
#ifndef MX_Q_MIN_BLOCKS
#define MX_Q_MIN_BLOCKS 2      // co-resident blocks per SM (bounds the registers)
#endif
constexpr int kQStages = MX_Q_STAGES;
constexpr int kQTileBytes = kTR * kTC * 2;                  // 16 KB of bf16
constexpr int kQThreads = kTileThreads + 32;
constexpr int kQSmemBytes = kQStages * kQTileBytes + 2 * kQTileBytes + 256 + 1024;
constexpr unsigned long long kQWaitLimitNs = 2ull * 1000ull * 1000ull * 1000ull;

__device__ __forceinline__ int t2_word(int cp, int r) {
    int rr = r ^ ((cp >> 4) << 4);
    rr ^= ((rr >> 5) & 3) << 2;
    return cp * kTR + rr;
}

__device__ __forceinline__ bool q_wait(uint64_t* bar, uint32_t parity, volatile int* abort, unsigned int* status) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = mx_globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort) return false;
        if (mx_globaltimer() - t0 > kQWaitLimitNs) {
            *abort = 1;
            atomicOr(status, 1u);
            return false;
        }
    }
    return true;
}

template <bool kRow, bool kCol, int kLayout>
__global__ void __launch_bounds__(kQThreads, MX_Q_MIN_BLOCKS)
mxfp8_tile_tma_kernel(const __grid_constant__ CUtensorMap tmX, int64_t rows, int64_t cols, const int64_t* rows_valid,
                      uint8_t* __restrict__ row_codes, uint8_t* __restrict__ row_e8m0, uint8_t* __restrict__ col_codes,
                      uint8_t* __restrict__ col_e8m0, unsigned int* status) {
    extern __shared__ uint8_t q_smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(q_smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = smem;                                              // SW128 tiles: 1024-byte aligned
    uint32_t* T2 = reinterpret_cast<uint32_t*>(smem + kQStages * kQTileBytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kQStages * kQTileBytes + 2 * kQTileBytes);
    uint64_t* empty = full + kQStages;
    volatile int* abort = reinterpret_cast<volatile int*>(empty + kQStages);
    volatile int* stop = abort + 1;                                      // [2], by tile parity
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tiles_c = cols / kTC;
    const int64_t ntiles = tiles_c * ((load_rows_valid(rows_valid, rows) + kTR - 1) / kTR);
    if ((int64_t)blockIdx.x >= ntiles) return;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kQStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], kTileThreads / 32); }
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
    }
    __syncthreads();

    if (warp == kTileThreads / 32) {                                     // producer
        if (lane == 0) {
            uint32_t it = 0;
            for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
                const int s = (int)(it % kQStages);
                if (!q_wait(&empty[s], ((it / kQStages) & 1) ^ 1, abort, status)) break;
                mbar_expect_tx(&full[s], kQTileBytes);
                const int c0 = (int)((tile % tiles_c) * kTC), r0 = (int)((tile / tiles_c) * kTR);
                asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                             " [%0], [%1, {%2, %3}], [%4];"
                             :: "r"(smem_u32(stages + s * kQTileBytes)), "l"(reinterpret_cast<uint64_t>(&tmX)),
                                "r"(c0), "r"(r0), "r"(smem_u32(&full[s])) : "memory");
            }
            // every issued copy lands before the block exits
            const unsigned long long t0 = mx_globaltimer();
            for (uint32_t k = it > kQStages ? it - kQStages : 0; k < it; ++k)
                while (!mbar_try_wait(&full[k % kQStages], (k / kQStages) & 1) &&
                       mx_globaltimer() - t0 < kQWaitLimitNs) {}
        }
        return;
    }

    const int t = threadIdx.x;
    const int rl = t >> 1, h = t & 1;
    const int cp = t >> 3, g = t & 7;
    uint32_t it = 0;
    int buf = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
        const int s = (int)(it % kQStages);
        // on a failed wait the warps still meet at this tile's barrier (a warp
        // leaving early would strand the others there) and stop after it
        const bool ok = q_wait(&full[s], (it / kQStages) & 1, abort, status);
        if (!kCol && !ok) break;
        const int64_t c0 = (tile % tiles_c) * kTC, r0 = (tile / tiles_c) * kTR;
        const uint8_t* st = stages + s * kQTileBytes + rl * 128;
        uint4 q[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) q[i] = *reinterpret_cast<const uint4*>(st + (((4 * h + i) ^ (rl & 7)) << 4));
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (kRow) {
            const int64_t r = r0 + rl;
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) m = max(m, absmax8_bf16(q[i]));
            const int e = e8m0_exponent(__uint_as_float(m << 16));
            const float sc = exp2_neg(e);
            const uint64_t sc2 = f2_pack(sc, sc);
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t qw[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
                float y[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    y[2 * j] = bf16_lo(qw[j]);
                    y[2 * j + 1] = bf16_hi(qw[j]);
                    mul2_rn(y[2 * j], y[2 * j + 1], sc2);
                }
                w[2 * i] = cvt_e4m3x4(y[0], y[1], y[2], y[3]);
                w[2 * i + 1] = cvt_e4m3x4(y[4], y[5], y[6], y[7]);
            }
            uint4* dst = reinterpret_cast<uint4*>(row_codes + r * cols + c0 + 32 * h);
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
            row_e8m0[sf_offset(r, (c0 >> 5) + h, cols >> 5, kLayout)] = (uint8_t)(e + 127);
        }
        if (kCol) {
            uint32_t* Tb = T2 + buf * (kTC / 2) * kTR;
            const uint32_t wq[16] = {q[0].x, q[0].y, q[0].z, q[0].w, q[1].x, q[1].y, q[1].z, q[1].w,
                                     q[2].x, q[2].y, q[2].z, q[2].w, q[3].x, q[3].y, q[3].z, q[3].w};
#pragma unroll
            for (int j = 0; j < 16; ++j) Tb[t2_word(16 * h + j, rl)] = wq[j];
            if (t == 0) stop[it & 1] = *abort;                             // one reading of the flag for all warps
            asm volatile("bar.sync 1, %0;" :: "n"(kTileThreads) : "memory");
            uint32_t a[16];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint4 v = *reinterpret_cast<const uint4*>(Tb + t2_word(cp, 16 * g + 4 * k));
                a[4 * k] = v.x; a[4 * k + 1] = v.y; a[4 * k + 2] = v.z; a[4 * k + 3] = v.w;
            }
            const int64_t rr = r0 + 16 * g;
            const int64_t S = rows >> 5;
#pragma unroll
            for (int half = 0; half < 2; ++half) {                        // column 2cp + half
                float v[16];
#pragma unroll
                for (int m = 0; m < 16; ++m) v[m] = half ? bf16_hi(a[m]) : bf16_lo(a[m]);
                float mf = 0.0f;
#pragma unroll
                for (int m = 0; m < 16; ++m) mf = fmaxf(mf, fabsf(v[m]));
                mf = fmaxf(mf, __shfl_xor_sync(0xffffffffu, mf, 1));
                const int e = e8m0_exponent(mf);
                const float sc = exp2_neg(e);
                const uint64_t sc2 = f2_pack(sc, sc);
                uint32_t w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                {
                    float a0 = v[4 * i], a1 = v[4 * i + 1], a2 = v[4 * i + 2], a3 = v[4 * i + 3];
                    mul2_rn(a0, a1, sc2);
                    mul2_rn(a2, a3, sc2);
                    w[i] = cvt_e4m3x4(a0, a1, a2, a3);
                }
                const int64_t cg = c0 + 2 * cp + half;
                *reinterpret_cast<uint4*>(col_codes + cg * rows + rr) = make_uint4(w[0], w[1], w[2], w[3]);
                if ((g & 1) == 0) col_e8m0[sf_offset(cg, rr >> 5, S, kLayout)] = (uint8_t)(e + 127);
            }
            buf ^= 1;
            if (stop[it & 1]) break;                                     // the same decision in every warp
        }
    }
}

// ---------------------------------------------------------------------------
// NVFP4 [rows, cols] -> dequantise -> transpose -> MXFP8 with stochastic
// rounding: one 128 x 64 input tile per block, 256 threads.
//   Phase 1 (rq_load_tile): the tile's exact f16 products q*sf, transposed
//   into shared memory.
//   Phase 2: each thread takes 16 consecutive rows of one output row, twice:
//   two 16-byte loads, f16 -> fp32, the outer scale (x = RN(p s)), the
//   32-row amax (the block's other half is in lane ^ 8), the E8M0 exponent e,
//   y = x 2^-e, and the rounding: R = 16 and R = 8 by cvt.rs (two values per
//   instruction), R = 32 by exact integer arithmetic on y.  With one
//   outer scale for the whole tile (expert weights) the amax is taken on the
//   f16 products (s > 0 is monotone) and the two products fold into one:
//   RN(RN(p s) 2^-e) = RN(p (s 2^-e)) whenever p s stays in fp32's normal
//   range, which s >= 2^-100 guarantees (|p| >= 2^-10); smaller s takes the
//   two products.
// ---------------------------------------------------------------------------
// cvt.rs on four values with their 16-bit random fields given as cvt.rs takes
// them (y0 in bits 15:0 of f01, y1 in bits 31:16, likewise y2, y3 in f23);
// codes packed y0 | y1 << 8 | y2 << 16 | y3 << 24.
__device__ __forceinline__ uint32_t cvt_rs_quad_fields(float y0, float y1, float y2, float y3, uint32_t f01,
                                                       uint32_t f23) {
    uint32_t d0, d1;
    asm("cvt.rs.satfinite.e4m3x4.f32 %0, {%1, %2, %3, %4}, %5;" : "=r"(d0) : "f"(0.0f), "f"(y1), "f"(0.0f), "f"(y0), "r"(f01));
    asm("cvt.rs.satfinite.e4m3x4.f32 %0, {%1, %2, %3, %4}, %5;" : "=r"(d1) : "f"(0.0f), "f"(y3), "f"(0.0f), "f"(y2), "r"(f23));
    return __byte_perm(d0, d1, 0x6420);
}

constexpr float kFoldMinScale = 7.888609052210118e-31f;          // 2^-100

// Five blocks per SM (48 registers, no spills): measured on B200 14% faster than four (62
// registers) on per-expert weights and 4% on per-row tensors; six spill.  The forms that
// would spill at five (R = 8, per-row scales into a row-major output) keep four.
template <int kR, int kOutLayout, bool kPerRow>
constexpr int rq_min_blocks() { return (kR == 8 || (kPerRow && kOutLayout == MX_SF_ROWMAJOR)) ? 4 : 5; }

template <int kR, int kInLayout, int kOutLayout, bool kPerRow>
__global__ void __launch_bounds__(kTileThreads, rq_min_blocks<kR, kOutLayout, kPerRow>())
requant_tile_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf, bool sf_words, bool e8_words,
                    const float* __restrict__ outer, int64_t rows, int64_t cols, int64_t group_rows, int group_shift,
                    const int64_t* rows_valid, uint64_t seed, uint64_t stream_id, uint8_t* __restrict__ out_codes,
                    uint8_t* __restrict__ out_e8m0) {
    __shared__ __align__(1024) uint16_t T[kTC * kTR];
    __shared__ __align__(16) float so[kPerRow ? kTR : 4];
    const int64_t c0 = (int64_t)blockIdx.x * kTC, r0 = (int64_t)blockIdx.y * kTR;
    if (r0 >= load_rows_valid(rows_valid, rows)) return;
    const uint32_t tbase = smem_u32(T);
    float s_uni = 0.0f;
    if (!kPerRow) {                   // group_rows is a multiple of 128: one outer scale per tile
        const int64_t gi = group_shift >= 0 ? (r0 >> group_shift) : (int64_t)((uint32_t)r0 / (uint32_t)group_rows);
        if (mx_in_range(gi, 1, rows / group_rows)) s_uni = __ldg(outer + gi);
    }
    rq_load_tile<kInLayout, kPerRow>(codes, sf, sf_words, outer, rows, cols, 1, r0, c0, tbase, so);
    __syncthreads();
    // ---------------- phase 2: lane (m = lane % 8, jj = (lane / 8) % 2, q = lane / 16) of warp w: output row
    // c = 16 (m / 2) + 2w + m % 2 of the tile, input rows 16j..16j+15 with j = 2 (2 it + q) + jj
    const RqLane ln;
    const int jj = ln.jj, q = ln.q, c = ln.c;
    const int64_t cg = c0 + c;
    const int64_t Se = rows >> 5;
    uint32_t e_bytes = 0;                               // E8M0 bytes of blocks q and 2 + q of this output row
#pragma unroll
    for (int it = 0; it < 2; ++it) {
        const int j = ln.chunk(it);
        uint32_t hw[8];
        rq_read16(tbase, c, j, hw);
        float y[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) h2_to_f32x2(hw[i], y[2 * i], y[2 * i + 1]);
        int e;
        if (kPerRow) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 s4 = *reinterpret_cast<const float4*>(so + 16 * j + 4 * i);
                mul2_rn(y[4 * i], y[4 * i + 1], f2_pack(s4.x, s4.y));
                mul2_rn(y[4 * i + 2], y[4 * i + 3], f2_pack(s4.z, s4.w));
            }
            float mf = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) mf = fmaxf(mf, fabsf(y[i]));
            mf = fmaxf(mf, __shfl_xor_sync(0xffffffffu, mf, 8));
            e = e8m0_exponent(mf);
            const float sc = exp2_neg(e);
            const uint64_t sc2 = f2_pack(sc, sc);
#pragma unroll
            for (int i = 0; i < 8; ++i) mul2_rn(y[2 * i], y[2 * i + 1], sc2);
        } else {
            float pm = rq_maxabs16(hw);
            pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, 8));
            e = e8m0_exponent(__fmul_rn(pm, s_uni));
            const bool fold = s_uni >= kFoldMinScale;
            const float s2 = fold ? __fmul_rn(s_uni, exp2_neg(e)) : s_uni;
            const uint64_t s22 = f2_pack(s2, s2);
#pragma unroll
            for (int i = 0; i < 8; ++i) mul2_rn(y[2 * i], y[2 * i + 1], s22);
            if (!fold) {
                const float sc = exp2_neg(e);
                const uint64_t sc2 = f2_pack(sc, sc);
#pragma unroll
                for (int i = 0; i < 8; ++i) mul2_rn(y[2 * i], y[2 * i + 1], sc2);
            }
        }
        const int64_t rr = r0 + 16 * j;
        const int64_t L0 = cg * rows + rr;              // linear index of the first output element
        uint32_t wo[4];
        if constexpr (kR == 16) {                       // the hardware stochastic rounding, two values per cvt
#pragma unroll
            for (int blk = 0; blk < 2; ++blk) {
                const uint4 rnd = philox4x32_10((uint64_t)(L0 / 8) + blk, stream_id, seed);
                wo[2 * blk] = cvt_rs16_e4m3_quad(y[8 * blk], y[8 * blk + 1], y[8 * blk + 2], y[8 * blk + 3], rnd.x,
                                                 rnd.y);
                wo[2 * blk + 1] = cvt_rs16_e4m3_quad(y[8 * blk + 4], y[8 * blk + 5], y[8 * blk + 6], y[8 * blk + 7],
                                                     rnd.z, rnd.w);
            }
        } else if constexpr (kR == 8) {
            // The same instruction with R = 8: element j's 8-bit integer u (byte j % 4 of word j / 4 of the
            // block) enters as the 16-bit field (255 - u) << 8.  cvt.rs rounds up iff 0xFFFF - field <
            // F16 = floor(frac 2^16), i.e. iff 256 u + 255 < F16, i.e. iff u < floor(F16 / 256) =
            // floor(frac 2^8): the R = 8 rule exactly.
            const uint4 rnd = philox4x32_10((uint64_t)(L0 / 16), stream_id, seed);
            const uint32_t nw[4] = {~rnd.x, ~rnd.y, ~rnd.z, ~rnd.w};
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
                wo[k4] = cvt_rs_quad_fields(y[4 * k4], y[4 * k4 + 1], y[4 * k4 + 2], y[4 * k4 + 3],
                                            __byte_perm(nw[k4], 0u, 0x1404), __byte_perm(nw[k4], 0u, 0x3424));
        } else {                                        // exact integer rounding of y = x 2^-e (block exponent 0)
            const SrBlock sb = sr_block(0);
            constexpr int kPer = 128 / kR;              // values per Philox block
#pragma unroll
            for (int blk = 0; blk < (16 + kPer - 1) / kPer; ++blk) {
                const uint4 rnd = philox4x32_10((uint64_t)(L0 / kPer) + blk, stream_id, seed);
#pragma unroll
                for (int f = 0; f < kPer && blk * kPer + f < 16; ++f) {
                    const int i = blk * kPer + f;
                    const uint32_t code = e4m3_sr_code<kR>(y[i], sb, philox_field<kR>(rnd, f));
                    if ((i & 3) == 0) wo[i >> 2] = code; else wo[i >> 2] |= code << (8 * (i & 3));
                }
            }
        }
        if (mx_in_range(cg * rows + rr, 16, cols * rows))
            *reinterpret_cast<uint4*>(out_codes + cg * rows + rr) = make_uint4(wo[0], wo[1], wo[2], wo[3]);
        e_bytes |= (uint32_t)(e + 127) << (16 * it);
    }
    // The tile's four E8M0 blocks of output row cg are 4 consecutive bytes in either layout (r0 / 32 is a
    // multiple of 4): lane q = 0 holds blocks 0 and 2, lane ^ 16 blocks 1 and 3; one 32-bit store.
    const uint32_t other = __shfl_xor_sync(0xffffffffu, e_bytes, 16);
    if (jj == 0 && q == 0 && mx_in_range(sf_offset(cg, r0 >> 5, Se, kOutLayout), 4, cols * Se)) {
        uint8_t* dst = out_e8m0 + sf_offset(cg, r0 >> 5, Se, kOutLayout);
        const uint32_t word = e_bytes | (other << 8);
        if (e8_words) *reinterpret_cast<uint32_t*>(dst) = word;
        else { dst[0] = (uint8_t)word; dst[1] = (uint8_t)(word >> 8); dst[2] = (uint8_t)(word >> 16); dst[3] = (uint8_t)(word >> 24); }
    }
}

template <typename F>
int dispatch_layout(int layout, F&& f) {
    if (layout == MX_SF_MMA) return f(std::integral_constant<int, MX_SF_MMA>());
    return f(std::integral_constant<int, MX_SF_ROWMAJOR>());
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================

namespace {

// The launches of nvfp4_quantize (kR = 0, codes to nearest) and of
// nvfp4_quantize_sr (kR random bits): one pass of the row kernel for per-row
// outer scales, else the group amax pass, the row kernel and the conversion
// of the group maxima to scales.  Arguments already validated.
template <int kR>
int nvfp4_quantize_launch(const void* x, int64_t rows, int64_t cols, int64_t group_rows, uint8_t* codes, uint8_t* sf,
                          float* outer, int sf_layout, SrKey key, cudaStream_t stream) {
    const uint16_t* xb = static_cast<const uint16_t*>(x);
    const int64_t ngroups = rows / group_rows;
    const int64_t nblk_row = cols / 16;
    // word-sized scale stores need four blocks per row and 4-byte aligned rows
    const bool word_sf = nblk_row % 4 == 0 && mx_aligned(sf, 4);
    return dispatch_layout(sf_layout, [&](auto L) {
        constexpr int kL = decltype(L)::value;
        auto run = [&](auto kGroupC) {
            constexpr bool kG = decltype(kGroupC)::value;
            auto go = [&](auto kern, int tpr) {
                const int64_t rpb = kRowThreads / tpr;
                kern<<<(unsigned)((rows + rpb - 1) / rpb), kRowThreads, 0, stream>>>(xb, rows, cols, group_rows, word_sf,
                                                                                       codes, sf, outer, key);
                mx_count_launch();
            };
            // four 16-element blocks (128 bytes) per thread in flight, 4 CTAs per SM:
            // 128 KB of loads outstanding per SM covers HBM latency under load
            if (nblk_row <= 64) go(nvfp4_quant_rows_kernel<16, 4, kG, kL, kR>, 16);
            else if (nblk_row <= 128) go(nvfp4_quant_rows_kernel<32, 4, kG, kL, kR>, 32);
            else if (nblk_row <= 256) go(nvfp4_quant_rows_kernel<64, 4, kG, kL, kR>, 64);
            else if (nblk_row <= 512) go(nvfp4_quant_rows_kernel<128, 4, kG, kL, kR>, 128);
            else if (nblk_row <= 1024) go(nvfp4_quant_rows_kernel<256, 4, kG, kL, kR>, 256);
            else go(nvfp4_quant_rows_kernel<256, 8, kG, kL, kR>, 256);
        };
        if (group_rows == 1) {
            run(std::false_type());
        } else {
            if (cudaMemsetAsync(outer, 0, sizeof(float) * ngroups, stream) != cudaSuccess) return mx_launch_status();
            const int64_t group_vec = group_rows * cols / 8;          // 16-byte vectors per group
            const int64_t chunk_vec = 16384;                            // 256 KiB per block
            const dim3 ag((unsigned)((group_vec + chunk_vec - 1) / chunk_vec), (unsigned)std::min<int64_t>(ngroups, 65535));
            nvfp4_group_amax_kernel<<<ag, kAmaxThreads, 0, stream>>>(xb, ngroups, group_vec, chunk_vec, outer);
            mx_count_launch();
            run(std::true_type());
            nvfp4_group_finish_kernel<<<(unsigned)((ngroups + 255) / 256), 256, 0, stream>>>(outer, ngroups);
            mx_count_launch();
        }
        return mx_launch_status();
    });
}

int nvfp4_quantize_check(const void* x, int64_t rows, int64_t cols, int64_t group_rows, const uint8_t* codes,
                         const uint8_t* sf, const float* outer, int sf_layout) {
    // an empty problem succeeds without touching memory (its pointers may be null)
    if (((!x || !codes || !sf || !outer) && rows > 0) || rows < 0 || cols <= 0 || cols % 16 || group_rows <= 0 ||
        rows % group_rows || !mx_aligned(x, 16) || !mx_aligned(codes, 16))
        return MX_EINVAL;
    if (sf_layout != MX_SF_ROWMAJOR && sf_layout != MX_SF_MMA) return MX_EINVAL;
    if (sf_layout == MX_SF_MMA && (rows % 128 || cols % 64)) return MX_EINVAL;
    return MX_OK;
}

}  // namespace

extern "C" int nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t group_rows, uint8_t* codes,
                              uint8_t* sf, float* outer, int sf_layout, cudaStream_t stream) {
    MX_NVTX_RANGE("nvfp4_quantize");
    if (int st = nvfp4_quantize_check(x, rows, cols, group_rows, codes, sf, outer, sf_layout)) return st;
    if (int st = mx_check_device()) return st;
    if (rows == 0) return MX_OK;
    return nvfp4_quantize_launch<0>(x, rows, cols, group_rows, codes, sf, outer, sf_layout, SrKey{}, stream);
}

// The four-bit backward's quantiser: the same scales, codes rounded
// stochastically (e2m1_sr.cuh) or to nearest.
extern "C" int nvfp4_quantize_sr(const void* x, int64_t rows, int64_t cols, int64_t group_rows, int rounding,
                                 uint64_t seed, uint64_t stream_id, int rbits, uint8_t* codes, uint8_t* sf,
                                 float* outer, int sf_layout, cudaStream_t stream) {
    MX_NVTX_RANGE("nvfp4_quantize_sr");
    if (int st = nvfp4_quantize_check(x, rows, cols, group_rows, codes, sf, outer, sf_layout)) return st;
    if (rounding != MX_ROUND_RNE && rounding != MX_ROUND_SR) return MX_EINVAL;
    if (rounding == MX_ROUND_SR && rbits != 8 && rbits != 16 && rbits != 32) return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (rows == 0) return MX_OK;
    const SrKey key{seed, stream_id};
    if (rounding == MX_ROUND_RNE)
        return nvfp4_quantize_launch<0>(x, rows, cols, group_rows, codes, sf, outer, sf_layout, key, stream);
    if (rbits == 8) return nvfp4_quantize_launch<8>(x, rows, cols, group_rows, codes, sf, outer, sf_layout, key, stream);
    if (rbits == 16)
        return nvfp4_quantize_launch<16>(x, rows, cols, group_rows, codes, sf, outer, sf_layout, key, stream);
    return nvfp4_quantize_launch<32>(x, rows, cols, group_rows, codes, sf, outer, sf_layout, key, stream);
}

extern "C" int swiglu_nvfp4_quantize(const void* h, int64_t rows, int64_t F, int gated, const int64_t* rows_valid,
                                     uint8_t* codes, uint8_t* sf, float* outer, int sf_layout, cudaStream_t stream) {
    MX_NVTX_RANGE("swiglu_nvfp4_quantize");
    if (((!h || !codes || !sf || !outer) && rows > 0) || rows < 0 || F <= 0 || F % 16 || F / 16 > 1024 ||
        !mx_aligned(h, 16) || !mx_aligned(codes, 16))
        return MX_EINVAL;
    if (sf_layout != MX_SF_ROWMAJOR && sf_layout != MX_SF_MMA) return MX_EINVAL;
    if (sf_layout == MX_SF_MMA && (rows % 128 || F % 64)) return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (rows == 0) return MX_OK;
    const int64_t nblk = F / 16;
    const bool word_sf = nblk % 4 == 0 && mx_aligned(sf, 4);
    const uint16_t* hb = static_cast<const uint16_t*>(h);
    return dispatch_layout(sf_layout, [&](auto L) {
        constexpr int kL = decltype(L)::value;
        auto go = [&](auto kern, int tpr) {
            const int64_t rpb = kRowThreads / tpr;
            kern<<<(unsigned)((rows + rpb - 1) / rpb), kRowThreads, 0, stream>>>(hb, rows, F, gated, rows_valid, word_sf,
                                                                                   codes, sf, outer);
            mx_count_launch();
        };
        if (nblk <= 64) go(swiglu_nvfp4_rows_kernel<16, kL>, 16);
        else if (nblk <= 128) go(swiglu_nvfp4_rows_kernel<32, kL>, 32);
        else if (nblk <= 256) go(swiglu_nvfp4_rows_kernel<64, kL>, 64);
        else if (nblk <= 512) go(swiglu_nvfp4_rows_kernel<128, kL>, 128);
        else go(swiglu_nvfp4_rows_kernel<256, kL>, 256);
        return mx_launch_status();
    });
}

extern "C" int mxfp8_quantize(const void* x, int64_t rows, int64_t cols, int rounding, uint64_t seed,
                              uint64_t stream_id, int rbits, const int64_t* rows_valid,
                              uint8_t* row_codes, uint8_t* row_e8m0, uint8_t* col_codes, uint8_t* col_e8m0,
                              int sf_layout, cudaStream_t stream) {
    MX_NVTX_RANGE("mxfp8_quantize");
    const bool do_row = row_codes != nullptr, do_col = col_codes != nullptr;
    if ((!x && rows > 0) || rows < 0 || cols <= 0 || rows % kTR || cols % 128 || !mx_aligned(x, 16)) return MX_EINVAL;
    if (rows == 0) return MX_OK;                        // nothing to compute in either form
    if (!do_row && !do_col) return MX_EINVAL;
    if ((do_row && (!row_e8m0 || !mx_aligned(row_codes, 16))) || (do_col && (!col_e8m0 || !mx_aligned(col_codes, 16))))
        return MX_EINVAL;
    if (rounding != MX_ROUND_RNE && rounding != MX_ROUND_SR) return MX_EINVAL;
    if (rounding == MX_ROUND_SR && rbits != 8 && rbits != 16 && rbits != 32) return MX_EINVAL;
    if (sf_layout != MX_SF_ROWMAJOR && sf_layout != MX_SF_MMA) return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const dim3 grid((unsigned)std::min<int64_t>((cols / kTC) * (rows / kTR), (int64_t)sms * 4));
    const uint64_t s_row = stream_id, s_col = do_row ? stream_id + 1 : stream_id;
    const uint16_t* xb = static_cast<const uint16_t*>(x);
    return dispatch_layout(sf_layout, [&](auto L) {
        constexpr int kL = decltype(L)::value;
        auto launch = [&](auto kRowC, auto kColC) {
            constexpr bool kRow = decltype(kRowC)::value, kCol = decltype(kColC)::value;
            if (rounding == MX_ROUND_RNE) {                 // TMA-fed form
                auto kern = mxfp8_tile_tma_kernel<kRow, kCol, kL>;
                CUtensorMap tm;
                unsigned int* status = nullptr;
                int occ = 0;
                if (mx_make_bf16_tile_map(&tm, x, rows, cols, kTC, kTR) == MX_OK &&
                    mx_status_word_address(&status) == MX_OK &&
                    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmemBytes) == cudaSuccess &&
                    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kQThreads, kQSmemBytes) == cudaSuccess &&
                    occ > 0) {
                    const dim3 qgrid((unsigned)std::min<int64_t>((cols / kTC) * (rows / kTR), (int64_t)sms * occ));
                    kern<<<qgrid, kQThreads, kQSmemBytes, stream>>>(tm, rows, cols, rows_valid, row_codes, row_e8m0,
                                                                    col_codes, col_e8m0, status);
                    mx_count_launch();
                    return;
                }
                cudaGetLastError();
            }
            if (rounding == MX_ROUND_RNE)
                mxfp8_tile_kernel<kRow, kCol, false, 8, kL><<<grid, kTileThreads, 0, stream>>>(
                    xb, rows, cols, rows_valid, seed, s_row, s_col, row_codes, row_e8m0, col_codes, col_e8m0);
            else if (rbits == 8)
                mxfp8_tile_kernel<kRow, kCol, true, 8, kL><<<grid, kTileThreads, 0, stream>>>(
                    xb, rows, cols, rows_valid, seed, s_row, s_col, row_codes, row_e8m0, col_codes, col_e8m0);
            else if (rbits == 16)
                mxfp8_tile_kernel<kRow, kCol, true, 16, kL><<<grid, kTileThreads, 0, stream>>>(
                    xb, rows, cols, rows_valid, seed, s_row, s_col, row_codes, row_e8m0, col_codes, col_e8m0);
            else
                mxfp8_tile_kernel<kRow, kCol, true, 32, kL><<<grid, kTileThreads, 0, stream>>>(
                    xb, rows, cols, rows_valid, seed, s_row, s_col, row_codes, row_e8m0, col_codes, col_e8m0);
            mx_count_launch();
        };
        if (do_row && do_col) launch(std::true_type(), std::true_type());
        else if (do_row) launch(std::true_type(), std::false_type());
        else launch(std::false_type(), std::true_type());
        return mx_launch_status();
    });
}

extern "C" int mxfp8_requant_transpose_sr(const uint8_t* codes, const uint8_t* sf, const float* outer,
                                          int64_t rows, int64_t cols, int64_t group_rows, int in_sf_layout,
                                          const int64_t* rows_valid, uint64_t seed, uint64_t stream_id, int rbits,
                                          uint8_t* out_codes, uint8_t* out_e8m0, int out_sf_layout,
                                          cudaStream_t stream) {
    MX_NVTX_RANGE("mxfp8_requant_transpose_sr");
    if (((!codes || !sf || !outer || !out_codes || !out_e8m0) && rows > 0) || rows < 0 || cols <= 0 || rows % kTR ||
        cols % kTC ||
        group_rows <= 0 || rows % group_rows || !mx_aligned(codes, 16) || !mx_aligned(out_codes, 16))
        return MX_EINVAL;
    if (rbits != 8 && rbits != 16 && rbits != 32) return MX_EINVAL;
    for (int l : {in_sf_layout, out_sf_layout})
        if (l != MX_SF_ROWMAJOR && l != MX_SF_MMA) return MX_EINVAL;
    if (out_sf_layout == MX_SF_MMA && (cols % 128 || rows % 128)) return MX_EINVAL;
    if (group_rows != 1 && group_rows % kTR) return MX_EINVAL;
    if (rows >= ((int64_t)1 << 31)) return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (rows == 0) return MX_OK;
    // one 128x64 tile per block: short independent blocks drift apart, so one
    // block's loads overlap another's rounding arithmetic (measured faster on
    // B200 than persistent blocks, which move through the phases in step)
    const dim3 grid((unsigned)(cols / kTC), (unsigned)(rows / kTR));
    // expert groups of a power-of-two size index their outer scale by a shift
    int gshift = -1;
    if (group_rows > 1 && (group_rows & (group_rows - 1)) == 0)
        for (gshift = 0; ((int64_t)1 << gshift) < group_rows; ++gshift) {}
    const bool sf_words = mx_aligned(sf, 4);            // a row's 4 scale bytes read as one word
    const bool e8_words = mx_aligned(out_e8m0, 4);      // an output row's 4 E8M0 bytes of a tile stored as one word
    return dispatch_layout(in_sf_layout, [&](auto Li) {
        return dispatch_layout(out_sf_layout, [&](auto Lo) {
            constexpr int kLi = decltype(Li)::value, kLo = decltype(Lo)::value;
            auto go = [&](auto Rc, auto per_row) {
                requant_tile_kernel<decltype(Rc)::value, kLi, kLo, decltype(per_row)::value>
                    <<<grid, kTileThreads, 0, stream>>>(codes, sf, sf_words, e8_words, outer, rows, cols, group_rows, gshift,
                                                         rows_valid, seed, stream_id, out_codes, out_e8m0);
            };
            auto by_r = [&](auto per_row) {
                if (rbits == 8) go(std::integral_constant<int, 8>(), per_row);
                else if (rbits == 16) go(std::integral_constant<int, 16>(), per_row);
                else go(std::integral_constant<int, 32>(), per_row);
            };
            if (group_rows == 1) by_r(std::true_type());
            else by_r(std::false_type());
            mx_count_launch();
            return mx_launch_status();
        });
    });
}

extern "C" int moe_dispatch_grad_mxfp8_quantize(const void* dout, const int32_t* src, const float* w, int64_t T,
                                                int64_t k, int64_t M_cap, int64_t D, const int64_t* rows_valid,
                                                uint8_t* row_codes, uint8_t* row_e8m0, uint8_t* col_codes,
                                                uint8_t* col_e8m0, int sf_layout, cudaStream_t stream) {
    MX_NVTX_RANGE("moe_dispatch_grad_mxfp8_quantize");
    if (((!dout || !src || !row_codes || !row_e8m0 || !col_codes || !col_e8m0) && M_cap > 0) || T < 0 || k <= 0 ||
        M_cap < 0 || M_cap % kTR || D <= 0 || D % 128 || !mx_aligned(dout, 16) || !mx_aligned(row_codes, 16) ||
        !mx_aligned(col_codes, 16))
        return MX_EINVAL;
    if (sf_layout != MX_SF_ROWMAJOR && sf_layout != MX_SF_MMA) return MX_EINVAL;
    if (T > ((int64_t)1 << 40) / k) return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (M_cap == 0) return MX_OK;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const DispatchGradRows rows_src{static_cast<const uint16_t*>(dout), src, w, T * k, k, D};
    return dispatch_layout(sf_layout, [&](auto L) {
        constexpr int kL = decltype(L)::value;
        auto kern = dispatch_grad_mxfp8_kernel<kL>;
        int occ = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kTileThreads, 0) != cudaSuccess || occ <= 0)
            occ = 2;
        const dim3 grid((unsigned)std::min<int64_t>((D / kTC) * (M_cap / kTR), (int64_t)sms * occ));
        kern<<<grid, kTileThreads, 0, stream>>>(rows_src, M_cap, D, rows_valid, row_codes, row_e8m0, col_codes,
                                                col_e8m0);
        mx_count_launch();
        return mx_launch_status();
    });
}

MX_BOUNDS_READER(mx_bounds_word_quant)
