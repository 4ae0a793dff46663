// mx_common.cuh -- device helpers shared by the mxmoe kernels (sm_100a).
//
// Number formats ([ai-primer] "Inkling 2 Small uses four-bit training...",
// §Block scales and per-token activations): NVFP4 = E2M1 values with one E4M3
// scale per 16 values and an FP32 outer scale; MXFP8 = E4M3 values with one
// E8M0 scale per 32 values.  Conversions use the PTX `cvt` instructions
// (round-to-nearest-even, saturating to the largest finite value); the
// stochastic rounding and the E8M0 exponent are exact integer arithmetic on
// the fp32 bit patterns.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/mxmoe.h"

#include <nvtx3/nvToolsExt.h>

// One NVTX range per C-ABI call, named after the entry point: it marks the
// call's host side (validation and launches) in profiler timelines and costs
// a few nanoseconds when no profiling tool is attached (header-only NVTX3).
struct MxNvtxRange {
    explicit MxNvtxRange(const char* name) { nvtxRangePushA(name); }
    ~MxNvtxRange() { nvtxRangePop(); }
    MxNvtxRange(const MxNvtxRange&) = delete;
    MxNvtxRange& operator=(const MxNvtxRange&) = delete;
};
#define MX_NVTX_RANGE(name) MxNvtxRange mx_nvtx_range_(name)

// ---------------------------------------------------------------------------
// Host-side status helpers (defined in abi.cu)
// ---------------------------------------------------------------------------
int mx_set_cuda_error(cudaError_t e);   // records e, returns MX_ECUDA
int mx_check_device(void);              // MX_OK on sm_100, else MX_EUNSUPPORTED / MX_ECUDA
int mx_launch_status(void);             // cudaGetLastError -> MX_OK / MX_ECUDA
void mx_count_launch(void);             // one more kernel launched by this library (mx_kernel_launches)
int mx_status_word_address(unsigned int** out);   // device address of the bounded-wait status word
// Bits of the device status word: a bounded wait expired; a routing entry was
// out of range or repeated within its token.
constexpr unsigned int kStatusTimeout = 1u, kStatusBadRoute = 2u;
struct CUtensorMap_st;
int mx_make_bf16_tile_map(struct CUtensorMap_st* m, const void* base, int64_t rows, int64_t cols, int box_cols,
                          int box_rows);             // bf16 [rows, cols] TMA map, 128-byte swizzle

static inline bool mx_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ---------------------------------------------------------------------------
// Bounds-checked build.  Compiled with -DMX_DEBUG_BOUNDS (libmxmoe_debug.so,
// `python -m fp8_moe_numerics_b200.build --debug-bounds`), the kernels check
// the global indices they compute against the extent of the buffer the call's
// arguments give it: an access out of range is skipped and counted in a
// device word of its translation unit, which mx_debug_bounds_violations()
// reads and clears.  This replaces a memory checker that cannot run here.  In
// the normal build mx_in_range() is the constant true and the checks compile
// away.
// ---------------------------------------------------------------------------
#ifdef MX_DEBUG_BOUNDS
static __device__ unsigned int g_mx_bounds_word;           // one per translation unit
// [first, first + count) inside [0, extent)?  Counts a violation when not.
__device__ __forceinline__ bool mx_in_range(int64_t first, int64_t count, int64_t extent) {
    if (first >= 0 && count >= 0 && first + count <= extent) return true;
    atomicAdd(&g_mx_bounds_word, 1u);
    return false;
}
#define MX_BOUNDS_READER(name)                                                              \
    unsigned int name(bool clear) {                                                         \
        unsigned int v = 0, zero = 0;                                                       \
        if (cudaMemcpyFromSymbol(&v, g_mx_bounds_word, sizeof(v)) != cudaSuccess) return 0; \
        if (clear && v) cudaMemcpyToSymbol(g_mx_bounds_word, &zero, sizeof(zero));          \
        return v;                                                                           \
    }
#else
__device__ __forceinline__ constexpr bool mx_in_range(int64_t, int64_t, int64_t) { return true; }
#define MX_BOUNDS_READER(name) \
    unsigned int name(bool) { return 0u; }
#endif
// Per translation unit readers of the bounds word (defined in each .cu).
unsigned int mx_bounds_word_abi(bool clear);
unsigned int mx_bounds_word_quant(bool clear);
unsigned int mx_bounds_word_glue(bool clear);
unsigned int mx_bounds_word_gemm(bool clear);
unsigned int mx_bounds_word_s2f6(bool clear);
unsigned int mx_bounds_word_nvfp4_bwd(bool clear);

// ---------------------------------------------------------------------------
// Shared-memory addresses, mbarriers and the GPU clock
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Nanosecond wall clock of the GPU (bounded waits measure their limit on it).
__device__ __forceinline__ unsigned long long mx_globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------------------
// Scale-factor layouts
// ---------------------------------------------------------------------------
// MMA layout: 512-byte atoms of 128 rows x 4 scale columns; atom index
// (r/128)*(S/4) + s/4, byte (r%32)*16 + ((r%128)/32)*4 + s%4 inside it.
__host__ __device__ __forceinline__ int64_t sf_offset_mma(int64_t r, int64_t s, int64_t S) {
    return (((r >> 7) * (S >> 2) + (s >> 2)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (s & 3);
}
__host__ __device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t s, int64_t S, int layout) {
    return layout == MX_SF_MMA ? sf_offset_mma(r, s, S) : r * S + s;
}

// ---------------------------------------------------------------------------
// Element conversions (PTX cvt, sm_100a)
// ---------------------------------------------------------------------------
// Two fp32 -> one byte of two E2M1 codes; `lo` lands in the low nibble.
// Eight values -> one word of E2M1 codes: byte j holds v[2j] in its low nibble
// and v[2j+1] in its high nibble (RNE, satfinite); the four code bytes are
// packed by a vector mov, with byte 0 the least significant.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float* v) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out) : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return out;
}

// Two fp32 -> two E4M3 codes in a 16-bit value; `lo` in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(out) : "f"(lo), "f"(hi));
    return out;
}

// Four values -> E4M3 codes v0 | v1 << 8 | v2 << 16 | v3 << 24 (RNE, satfinite),
// the two code pairs packed by a vector mov.
__device__ __forceinline__ uint32_t cvt_e4m3x4(float v0, float v1, float v2, float v3) {
    uint32_t out;
    asm("{\n\t.reg .b16 h0, h1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h0, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h1, %4, %3;\n\t"
        "mov.b32 %0, {h0, h1};\n\t}"
        : "=r"(out) : "f"(v0), "f"(v1), "f"(v2), "f"(v3));
    return out;
}

// One E4M3 code -> fp32 (exact).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    uint32_t h2;
    uint16_t in = (uint16_t)((code & 0xff) * 0x0101u);   // same code in both lanes
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xffff)));
}

// Word of eight E2M1 codes -> four halves pairs (exact): h[j] holds the codes
// of byte j (low nibble first); the bytes are unpacked by a vector mov.
__device__ __forceinline__ void e2m1x8_to_h2x4(uint32_t w, __half2* h) {
    uint32_t r0, r1, r2, r3;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(w));
    h[0] = *reinterpret_cast<__half2*>(&r0);
    h[1] = *reinterpret_cast<__half2*>(&r1);
    h[2] = *reinterpret_cast<__half2*>(&r2);
    h[3] = *reinterpret_cast<__half2*>(&r3);
}

// E4M3 code -> half (exact: E4M3 is a subset of fp16).
__device__ __forceinline__ __half e4m3_to_h(uint32_t code) {
    uint32_t h2;
    uint16_t in = (uint16_t)((code & 0xff) * 0x0101u);   // same code in both lanes
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __ushort_as_half((unsigned short)(h2 & 0xffff));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// sigmoid with the fast exponential and division intrinsics: a few fp32 ulp,
// far below the bf16 rounding that follows (results stay within one bf16
// rounding of the exact value); exp overflow gives sigmoid 0, as it should.
__device__ __forceinline__ float sigmoid_f(float g) { return __fdividef(1.0f, 1.0f + __expf(-g)); }
__device__ __forceinline__ float silu_f(float g) { return g * sigmoid_f(g); }

// Two SwiGLU outputs silu(g) * u, each rounded to bf16, from two bf16 pairs
// (the one definition the standalone and the fused-quantiser kernels share).
__device__ __forceinline__ uint32_t swiglu_word(uint32_t g, uint32_t u) {
    return pack_bf16x2(silu_f(bf16_lo(g)) * bf16_lo(u), silu_f(bf16_hi(g)) * bf16_hi(u));
}

__device__ __forceinline__ float dsilu_f(float g) {
    const float s = sigmoid_f(g);
    return s * (1.0f + g * (1.0f - s));
}

// The SwiGLU backward of two elements from bf16 pairs of the gate g, the up
// projection u and the upstream gradient d: dg = d u silu'(g) and du =
// d silu(g), each rounded to bf16 (the one definition the standalone kernel
// and the fused MXFP8 quantiser share).
__device__ __forceinline__ uint32_t swiglu_bwd_gate_word(uint32_t g, uint32_t u, uint32_t d) {
    return pack_bf16x2(bf16_lo(d) * bf16_lo(u) * dsilu_f(bf16_lo(g)), bf16_hi(d) * bf16_hi(u) * dsilu_f(bf16_hi(g)));
}
__device__ __forceinline__ uint32_t swiglu_bwd_up_word(uint32_t g, uint32_t d) {
    return pack_bf16x2(bf16_lo(d) * silu_f(bf16_lo(g)), bf16_hi(d) * silu_f(bf16_hi(g)));
}

// The dispatch gradient of two elements: w * dout, rounded to bf16.
__device__ __forceinline__ uint32_t scaled_bf16_word(float w, uint32_t v) {
    return pack_bf16x2(w * bf16_lo(v), w * bf16_hi(v));
}

// ---------------------------------------------------------------------------
// MXFP8 block exponent: smallest e with amax <= 448 * 2^e, clamped to
// [-127, 127]; -127 for amax == 0.  448 = 1.75 * 2^8, so for a normal
// amax = 1.f * 2^E the answer is E-8 when 1.f <= 1.75, else E-7.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int e8m0_exponent(float amax) {
    uint32_t b = __float_as_uint(amax) & 0x7fffffffu;
    int eb = (int)(b >> 23);
    if (eb == 0) return -127;                    // zero or fp32-subnormal: E <= -127
    int E = eb - 127;
    int e = ((b & 0x7fffffu) <= 0x600000u) ? E - 8 : E - 7;
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^-e as an fp32 (e in [-127, 127]); 2^-127 is the subnormal 0x00200000.
__device__ __forceinline__ float exp2_neg(int e) {
    int k = 127 - e;                             // biased exponent of 2^-e
    return k >= 1 ? __uint_as_float((uint32_t)k << 23) : __uint_as_float(0x00200000u);
}

// ---------------------------------------------------------------------------
// Stochastic rounding of y = xh * 2^-e onto the E4M3 grid, exactly.
// xh is any finite fp32.  With y = M * 2^p (M the 24-bit significand), the
// quantum is 2^Q, Q = max(floor(log2 y) - 3, -9); the sh = Q - p bits of M
// below the quantum are dropped and the value rounds up iff
// u < floor(rem * 2^R / 2^sh).  The E4M3 code of units * 2^Q is
// (Q + 9) * 8 + units for every Q >= -9 (codes are monotone in magnitude, so a
// carry into the next binade is the next code).  Caller guarantees |y| <= 448.
//
// Fast path: xh normal and y >= 2^-6 (E4M3 normal range) means sh = 20, so
// the code is the top 11 magnitude bits of xh re-biased, plus the carry
// decided by the top R of the 20 dropped bits.  `sr_block` precomputes the
// per-block constants.
// ---------------------------------------------------------------------------
struct SrBlock {
    int lo_eb;        // smallest fp32 biased exponent taking the fast path
    uint32_t off;     // (e + 120) << 3
    int e;
};

__device__ __forceinline__ SrBlock sr_block(int e) {
    SrBlock b;
    b.lo_eb = max(1, e + 121);
    b.off = (uint32_t)(e + 120) << 3;
    b.e = e;
    return b;
}

template <int R>
__device__ __noinline__ uint32_t e4m3_sr_general(uint32_t mag, int e, uint32_t u) {
    if (mag == 0) return 0u;
    const uint32_t eb = mag >> 23;
    const uint32_t M = eb ? ((mag & 0x7fffffu) | 0x800000u) : mag;
    const int p = (eb ? (int)eb - 150 : -149) - e;     // exponent of M's unit bit in y
    const int fl = p + (31 - __clz(M));                // floor(log2 y)
    const int Q = fl - 3 < -9 ? -9 : fl - 3;
    const int sh = Q - p;                              // >= -3
    uint32_t units;
    if (sh <= 0) {
        units = M << (-sh);                            // on the grid already
    } else {
        const uint32_t lo = sh >= 32 ? 0u : (M >> sh);
        const uint32_t rem = sh >= 32 ? M : (M & ((1u << sh) - 1u));
        uint32_t thr;
        if (sh >= R) {
            const int d = sh - R;
            thr = d >= 32 ? 0u : (rem >> d);
        } else {
            thr = rem << (R - sh);                     // rem < 2^sh, so < 2^R
        }
        units = lo + (u < thr ? 1u : 0u);
    }
    return (uint32_t)((Q + 9) * 8 + (int)units);
}

template <int R>
__device__ __forceinline__ uint32_t e4m3_sr_code(float xh, const SrBlock& b, uint32_t u) {
    const uint32_t bits = __float_as_uint(xh);
    const uint32_t sign = (bits >> 24) & 0x80u;
    const uint32_t mag = bits & 0x7fffffffu;
    const uint32_t rem = mag & 0xfffffu;
    const uint32_t thr = R <= 20 ? (rem >> (20 - R)) : (rem << (R - 20));
    uint32_t code = (mag >> 20) - b.off + (u < thr ? 1u : 0u);
    if ((int)(mag >> 23) < b.lo_eb) code = e4m3_sr_general<R>(mag, b.e, u);
    return sign | code;
}

template <int R>
__device__ __forceinline__ uint32_t e4m3_sr_code(float xh, int e, uint32_t u) {
    return e4m3_sr_code<R>(xh, sr_block(e), u);
}

// ---------------------------------------------------------------------------
// Hardware stochastic rounding (sm_100a cvt.rs) onto E4M3.
// cvt.rs.satfinite.e4m3x4.f32 d, {a, b, c, f}, rbits puts f's code in byte 0
// and b's in byte 2; f adds rbits[15:0] and b adds rbits[31:16] as 16 random
// bits just below the kept E4M3 bits and truncates (the carry rounds up).  With
// u the 16-bit value of the stream, feeding 0xFFFF - u rounds up exactly when
// u < floor(frac * 2^16): the rule of e4m3_sr_code<16>, in one instruction
// (established by comparing the instruction with the oracle on a B200).  The
// a and c lanes are not used: their random bits are not independent of b's
// and f's.  Inputs must be |y| <= 448.
//
// Four consecutive elements: y0, y1 take the low and high halves of random
// word u01, y2, y3 those of u23; the codes are packed
// y0 | y1 << 8 | y2 << 16 | y3 << 24 by one byte permute.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cvt_rs16_e4m3_quad(float y0, float y1, float y2, float y3, uint32_t u01,
                                                       uint32_t u23) {
    uint32_t d0, d1;
    asm("cvt.rs.satfinite.e4m3x4.f32 %0, {%1, %2, %3, %4}, %5;"
        : "=r"(d0) : "f"(0.0f), "f"(y1), "f"(0.0f), "f"(y0), "r"(~u01));
    asm("cvt.rs.satfinite.e4m3x4.f32 %0, {%1, %2, %3, %4}, %5;"
        : "=r"(d1) : "f"(0.0f), "f"(y3), "f"(0.0f), "f"(y2), "r"(~u23));
    return __byte_perm(d0, d1, 0x6420);
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): ten rounds of the
// multiply / cross / key-add network; the key advances by the Weyl constants
// between rounds.  counter = (g lo, g hi, stream lo, stream hi),
// key = (seed lo, seed hi).
// ---------------------------------------------------------------------------
// Each multiply is written as its 32-bit low and high halves and the key is
// advanced by one add per round: measured on B200, 47 warp-instructions per
// call against 74 for the same function through 64-bit products and
// key + r * W per round.
__device__ __forceinline__ uint4 philox4x32_10(uint64_t g, uint64_t stream, uint64_t seed) {
    uint32_t c0 = (uint32_t)g, c1 = (uint32_t)(g >> 32), c2 = (uint32_t)stream, c3 = (uint32_t)(stream >> 32);
    uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        uint32_t lo0, hi0, lo1, hi1;
        asm("mul.lo.u32 %0, %2, %3;\n\tmul.hi.u32 %1, %2, %3;" : "=r"(lo0), "=r"(hi0) : "r"(0xD2511F53u), "r"(c0));
        asm("mul.lo.u32 %0, %2, %3;\n\tmul.hi.u32 %1, %2, %3;" : "=r"(lo1), "=r"(hi1) : "r"(0xCD9E8D57u), "r"(c2));
        const uint32_t n0 = hi1 ^ c1 ^ k0;
        const uint32_t n2 = hi0 ^ c3 ^ k1;
        c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
        k0 += 0x9E3779B9u;                                   // the Weyl sequence of the key
        k1 += 0xBB67AE85u;
    }
    return make_uint4(c0, c1, c2, c3);
}

// R-bit random integer j (0 <= j < 128/R) of a Philox block.
template <int R>
__device__ __forceinline__ uint32_t philox_field(const uint4& w, int j) {
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
    if (R == 32) return words[j];
    int bit = j * R;
    return (words[bit >> 5] >> (bit & 31)) & ((1u << (R & 31)) - 1u);
}

__device__ __forceinline__ int64_t load_rows_valid(const int64_t* rows_valid, int64_t rows) {
    if (!rows_valid) return rows;
    int64_t v = *rows_valid;
    return v < rows ? v : rows;
}

// ---------------------------------------------------------------------------
// Combine path ([ai-primer §Quantized NVLink and BBBK]): expert outputs are
// rotated by a 32-dimensional random Hadamard transform and quantised to
// block-scaled S2F6, eight-bit fixed point with two signed integer bits and
// six fractional bits.  Per 32-column block j of a row: z = H32 (sigma_j x),
// H32 the unnormalised Sylvester matrix, sigma_j flipping coordinate i when
// bit i of hadamard_sign_word(j) is set; one E8M0 exponent e per block (the
// smallest with amax|z| <= (127/64) 2^e, in [-127, 127]); int8 codes
// c = RNE(z 2^(6-e)) in [-127, 127].  The inverse is x = sigma_j (H32 z) / 32.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t hadamard_sign_word(uint64_t seed, uint64_t stream, uint64_t j) {
    return philox4x32_10(j, stream, seed).x;
}

// Two fp32 lanes in one 64-bit register, for sm_100a's packed f32x2
// arithmetic: each lane of add/sub/mul/fma .rn.f32x2 is one IEEE
// round-to-nearest operation, so a packed op gives the two scalar results.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// (a * s, b * s) with s2 = (s, s): two round-to-nearest products, one instruction.
__device__ __forceinline__ void mul2_rn(float& a, float& b, uint64_t s2) {
    f2_unpack(f2_mul(f2_pack(a, b), s2), a, b);
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// Smallest integer e with amax <= (127/64) 2^e, clamped to [-127, 127]
// (-127 for amax == 0); amax finite and >= 0.  A subnormal amax is first
// scaled by 2^64 (exact) so its exponent field is meaningful.
__device__ __forceinline__ int s2f6_exponent(float amax) {
    if (amax == 0.0f) return -127;
    int adj = 0;
    if (amax < 1.17549435e-38f) {
        amax = __fmul_rn(amax, 18446744073709551616.0f);
        adj = 64;
    }
    const uint32_t b = __float_as_uint(amax);
    int e = (int)(b >> 23) - 127 - adj;
    if ((b & 0x7fffffu) > 0x7e0000u) ++e;               // significand above 127/64 = 1.111111b
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// Codes of one block from its rotated values in pairs P[q] = (z_2q, z_2q+1):
// c_i = RNE(z_i 2^(6-e)) clamped to [-127, 127], packed four per word (code i
// in byte i%4 of word i/4, two's complement).  One fma adds 1.5 * 2^23 to the
// exactly scaled value, so the sum rounds once to the nearest integer (ties
// to even) and its low byte is the code.  kClamp: e == 127, where 127.99..
// can occur; kTiny: 2^(6-e) is not finite in fp32, so 2^64 of it is applied
// first (exactly).
template <bool kClamp, bool kTiny>
__device__ __forceinline__ void s2f6_codes_pairs(const uint64_t* P, float scale, uint32_t* words) {
    const float magic = 12582912.0f;
    const uint64_t S2 = f2_pack(scale, scale), M2 = f2_pack(magic, magic);
    const uint64_t T2 = f2_pack(18446744073709551616.0f, 18446744073709551616.0f);
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        float y[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint64_t z = kTiny ? f2_mul(P[2 * w + h], T2) : P[2 * w + h];
            f2_unpack(f2_fma(z, S2, M2), y[2 * h], y[2 * h + 1]);
        }
        uint32_t b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (kClamp) y[i] = fminf(fmaxf(y[i], magic - 127.0f), magic + 127.0f);
            b[i] = __float_as_uint(y[i]);
        }
        words[w] = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    }
}

// Stages 2..16 of the rotation on pairs P[q] = (z_2q, z_2q+1) -- stage h
// pairs element i with i + h, i.e. pair q with pair q + h/2 -- then the
// block's exponent and codes.  Returns e.
__device__ __forceinline__ int s2f6_finish(uint64_t* P, uint32_t* words) {
#pragma unroll
    for (int h2 = 1; h2 < 16; h2 <<= 1) {
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            if ((q & h2) == 0) {
                const uint64_t a = P[q], b = P[q + h2];
                P[q] = f2_add(a, b);
                P[q + h2] = f2_sub(a, b);
            }
        }
    }
    float amax = 0.0f;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        float a, b;
        f2_unpack(P[q], a, b);
        amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
    }
    const int e = s2f6_exponent(amax);
    const int sh = 6 - e;                               // in [-121, 133]
    if (sh > 126) s2f6_codes_pairs<false, true>(P, __uint_as_float((uint32_t)(sh - 64 + 127) << 23), words);
    else if (e == 127) s2f6_codes_pairs<true, false>(P, __uint_as_float((uint32_t)(sh + 127) << 23), words);
    else s2f6_codes_pairs<false, false>(P, __uint_as_float((uint32_t)(sh + 127) << 23), words);
    return e;
}

// One 32-value block v (fp32, unrotated): negated where bit i of `mask` is
// set, rotated by H32 (stage h = 1 on scalars into pairs, stages 2..16 on
// pairs -- the same adds in the same order as one scalar butterfly network),
// then its exponent and codes.  Returns e.
__device__ __forceinline__ int s2f6_block_mask(const float* v, uint32_t mask, uint32_t* words) {
    uint64_t P[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        const float a = __uint_as_float(__float_as_uint(v[2 * q]) ^ ((mask << (31 - 2 * q)) & 0x80000000u));
        const float b = __uint_as_float(__float_as_uint(v[2 * q + 1]) ^ ((mask << (30 - 2 * q)) & 0x80000000u));
        P[q] = f2_pack(__fadd_rn(a, b), __fsub_rn(a, b));
    }
    return s2f6_finish(P, words);
}

// The same block read straight from 16 words of bf16 pairs (word q holds
// values 2q and 2q+1), without first widening all 32 values.
__device__ __forceinline__ int s2f6_block_mask_bf16(const uint32_t* wq, uint32_t mask, uint32_t* words) {
    uint64_t P[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        const float a = __uint_as_float((wq[q] << 16) ^ ((mask << (31 - 2 * q)) & 0x80000000u));
        const float b = __uint_as_float((wq[q] & 0xffff0000u) ^ ((mask << (30 - 2 * q)) & 0x80000000u));
        P[q] = f2_pack(__fadd_rn(a, b), __fsub_rn(a, b));
    }
    return s2f6_finish(P, words);
}

// The same block with v first multiplied by `scale`, the signs given as a
// table sig[i] = +-1.0f (16-byte aligned): x_i = v_i (sig_i scale), which is
// sig_i RN(v_i scale) exactly.
__device__ __forceinline__ int s2f6_block_scaled(const float* v, float scale, const float* sig, uint32_t* words) {
    const uint64_t S2 = f2_pack(scale, scale);
    uint64_t P[16];
#pragma unroll
    for (int q4 = 0; q4 < 8; ++q4) {
        const float4 sg = *reinterpret_cast<const float4*>(sig + 4 * q4);
        const uint64_t s01 = f2_mul(f2_pack(sg.x, sg.y), S2), s23 = f2_mul(f2_pack(sg.z, sg.w), S2);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int q = 2 * q4 + h;
            float a, b;
            f2_unpack(f2_mul(f2_pack(v[2 * q], v[2 * q + 1]), h ? s23 : s01), a, b);
            P[q] = f2_pack(__fadd_rn(a, b), __fsub_rn(a, b));
        }
    }
    return s2f6_finish(P, words);
}

// Scalar forms, used where no pairs are at hand (the combine's inverse).
// Negate v[i] where bit i of `mask` is set (exact).
__device__ __forceinline__ void apply_signs32(float* v, uint32_t mask) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(__float_as_uint(v[i]) ^ ((mask << (31 - i)) & 0x80000000u));
}

// Unnormalised Walsh-Hadamard transform of 32 values in registers: stages
// h = 1, 2, 4, 8, 16, each pair (i, i + h) with i & h == 0 becoming
// (a + b, a - b), one fp32 round-to-nearest add each.
__device__ __forceinline__ void fwht32(float* v) {
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if ((i & h) == 0) {
                const float a = v[i], b = v[i + h];
                v[i] = __fadd_rn(a, b);
                v[i + h] = __fsub_rn(a, b);
            }
        }
    }
}
