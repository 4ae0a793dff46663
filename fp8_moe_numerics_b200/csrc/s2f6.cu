// s2f6.cu -- the combine path's 32-d random Hadamard rotation with
// block-scaled S2F6 quantisation, and the combine that reads it (sm_100a).
//
// [ai-primer §Quantized NVLink and BBBK]: expert outputs are rotated by a
// 32-dimensional random Hadamard transform and quantised into block-scaled
// S2F6 (eight-bit fixed point, two signed integer bits and six fractional
// bits) for the combine; the rotation spreads an outlier's magnitude over its
// block first.  The block arithmetic (s2f6_block_*: signs, rotation, exponent,
// codes) is in mx_common.cuh and shared with the GEMM epilogue that produces
// the same format directly from its accumulators.
//
// In both kernels one thread rotates a whole 32-value block in its registers:
// its 32 codes are 32 contiguous bytes and its exponent one byte; consecutive
// threads take consecutive blocks of a row so that every warp's loads and
// stores are contiguous.
#include "mx_common.cuh"

namespace {

constexpr int kThreads = 256;

// 2^n as fp32 for n in [-149, 127] (subnormal below -126); exact.
__device__ __forceinline__ float pow2_int(int n) {
    return n >= -126 ? __uint_as_float((uint32_t)(n + 127) << 23) : __uint_as_float(1u << (n + 149));
}

// Thread (row group g, column block jb) quantises MX_S2F6_ROWS rows of column
// block jb with one draw of the block's sign word; a warp covers 32
// consecutive column blocks, so each row's loads and stores stay contiguous.
// Measured on B200 (16384 x 4096, L2 flushed): 43 us for 1, 2 and 4 rows per
// thread alike -- the kernel is bound by HBM, not by Philox -- so one row,
// without register spills, is the default.
#ifndef MX_S2F6_ROWS
#define MX_S2F6_ROWS 1        // rows per thread (one sign word for all of them)
#endif
#ifndef MX_S2F6_MIN_BLOCKS
#define MX_S2F6_MIN_BLOCKS 5  // co-resident blocks per SM (bounds the registers)
#endif
constexpr int kRowsPerThread = MX_S2F6_ROWS;

__global__ void __launch_bounds__(kThreads, MX_S2F6_MIN_BLOCKS)
hadamard_s2f6_quantize_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t nbc, uint64_t seed,
                              uint64_t stream_id, uint8_t* __restrict__ codes, uint8_t* __restrict__ e8m0) {
    const int64_t item = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t groups = (rows + kRowsPerThread - 1) / kRowsPerThread;
    if (item >= groups * nbc) return;
    const int64_t g = item / nbc, jb = item - g * nbc;
    const uint32_t mask = hadamard_sign_word(seed, stream_id, (uint64_t)jb);
#pragma unroll 1
    for (int k = 0; k < kRowsPerThread; ++k) {
        const int64_t r = g * kRowsPerThread + k;
        if (r >= rows) break;
        const int64_t blk = r * nbc + jb;
        const uint4* src = reinterpret_cast<const uint4*>(x + blk * 32);
        uint32_t wq[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 u = __ldcs(src + q);
            wq[4 * q] = u.x; wq[4 * q + 1] = u.y; wq[4 * q + 2] = u.z; wq[4 * q + 3] = u.w;
        }
        uint32_t w[8];
        const int e = s2f6_block_mask_bf16(wq, mask, w);
        uint4* dst = reinterpret_cast<uint4*>(codes + blk * 32);
        __stcs(dst, make_uint4(w[0], w[1], w[2], w[3]));
        __stcs(dst + 1, make_uint4(w[4], w[5], w[6], w[7]));
        e8m0[blk] = (uint8_t)(e + 127);
    }
}

// int8 code in byte `i` of w, as an exact fp32 value: the sign-extended code
// is added to the bit pattern of 1.5 * 2^23, whose unit in the last place is
// 1, and the constant is subtracted again.
__device__ __forceinline__ float s2f6_code_value(uint32_t w, int i) {
    const int32_t c = (int32_t)(int8_t)(uint8_t)(w >> (8 * i));
    return __fsub_rn(__uint_as_float(0x4B400000u + (uint32_t)c), 12582912.0f);
}

// out[t, 32 jb ..] = sigma_jb (H32 u) / 32 with u = sum_j w[t, j] 2^(e_j - 6) c_j,
// the weighted sum of the k routed rows' codes taken in the rotated domain
// (the inverse rotation is linear), fp32, j in order; bf16 round to nearest.
__global__ void __launch_bounds__(kThreads)
moe_combine_s2f6_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ e8m0,
                        const int32_t* __restrict__ pos, const float* __restrict__ wts, int64_t T, int64_t k,
                        int64_t nbc, uint64_t seed, uint64_t stream_id, uint16_t* __restrict__ out) {
    const int64_t item = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (item >= T * nbc) return;
    const int64_t t = item / nbc, jb = item - t * nbc;
    float u[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) u[i] = 0.0f;
    for (int64_t j = 0; j < k; ++j) {
        const int64_t r = __ldg(pos + t * k + j);
        if (r < 0) continue;                               // entry left out by the routing
        const float wj = wts ? __ldg(wts + t * k + j) : 1.0f;
        const int e = (int)__ldg(e8m0 + r * nbc + jb) - 127;
        const float sc = __fmul_rn(wj, pow2_int(e - 6));
        const uint4* src = reinterpret_cast<const uint4*>(codes + (r * nbc + jb) * 32);
        const uint4 c0 = __ldg(src), c1 = __ldg(src + 1);
        const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int i = 0; i < 32; ++i) u[i] = __fmaf_rn(s2f6_code_value(cw[i >> 2], i & 3), sc, u[i]);
    }
    fwht32(u);
    apply_signs32(u, hadamard_sign_word(seed, stream_id, (uint64_t)jb));
    uint32_t o[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = pack_bf16x2(__fmul_rn(u[2 * i], 0.03125f), __fmul_rn(u[2 * i + 1], 0.03125f));
    uint4* dst = reinterpret_cast<uint4*>(out + item * 32);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================

extern "C" int hadamard_s2f6_quantize(const void* x, int64_t rows, int64_t cols, uint64_t seed, uint64_t stream_id,
                                      int8_t* codes, uint8_t* e8m0, cudaStream_t stream) {
    MX_NVTX_RANGE("hadamard_s2f6_quantize");
    if (((!x || !codes || !e8m0) && rows > 0) || rows < 0 || cols <= 0 || cols % 32 || !mx_aligned(x, 16) ||
        !mx_aligned(codes, 16))
        return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (rows == 0) return MX_OK;
    const int64_t items = (rows + kRowsPerThread - 1) / kRowsPerThread * (cols / 32);
    hadamard_s2f6_quantize_kernel<<<(unsigned)((items + kThreads - 1) / kThreads), kThreads, 0, stream>>>(
        static_cast<const uint16_t*>(x), rows, cols / 32, seed, stream_id, reinterpret_cast<uint8_t*>(codes), e8m0);
    mx_count_launch();
    return mx_launch_status();
}

extern "C" int moe_combine_s2f6(const int8_t* codes, const uint8_t* e8m0, const int32_t* pos, const float* w,
                                int64_t T, int64_t k, int64_t D, uint64_t seed, uint64_t stream_id, void* out,
                                cudaStream_t stream) {
    MX_NVTX_RANGE("moe_combine_s2f6");
    if (((!codes || !e8m0 || !pos || !out) && T > 0) || T < 0 || k < 1 || D <= 0 || D % 32 ||
        !mx_aligned(codes, 16) || !mx_aligned(out, 16))
        return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (T == 0) return MX_OK;
    const int64_t items = T * (D / 32);
    moe_combine_s2f6_kernel<<<(unsigned)((items + kThreads - 1) / kThreads), kThreads, 0, stream>>>(
        reinterpret_cast<const uint8_t*>(codes), e8m0, pos, w, T, k, D / 32, seed, stream_id,
        static_cast<uint16_t*>(out));
    mx_count_launch();
    return mx_launch_status();
}

MX_BOUNDS_READER(mx_bounds_word_s2f6)
