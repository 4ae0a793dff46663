/*
 * oracle.c -- plain, slow CPU reference for the NVFP4-forward / MXFP8-backward
 * expert-layer numerics.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no source with the CUDA library and includes no CUDA header.
 *
 * Sources (web pages on Thinking Machines' "End-to-End 4-Bit Training"):
 *   [P2] "Inkling 2 Small uses four-bit training, Thinking Machines reports 8%
 *        and 20% savings" (ai-primer.com), sections
 *        "NVFP4 forward, MXFP8 backward", "Block scales and per-token
 *        activations" (format table), "Stochastic rounding across transposes".
 *   [P3] aibuzzwire.news article on "End-to-End 4-Bit Training",
 *        section "Why Fewer Bits Means Faster Training".
 * Where the pages are silent the reading taken is stated beside the code.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -fPIC
 * -shared.  Every float operation below is a single IEEE round-to-nearest-even
 * operation; no FMA contraction is allowed (-ffp-contract=off).
 *
 * Parity status per function is listed in the header of oracle/__init__.py.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>
#include <stdlib.h>

#define ORC_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* bf16 <-> fp32                                                             */
/* ------------------------------------------------------------------------ */

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 is the top half of an fp32: widening is exact. */
static float bf16_to_f32(uint16_t b) { return bits_to_f32((uint32_t)b << 16); }

/* fp32 -> bf16 round-to-nearest-even on the 16 dropped bits. */
ORC_API uint16_t orc_f32_to_bf16(float f) {
    uint32_t u = f32_to_bits(f);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x40);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------ */
/* Element codecs.                                                           */
/* [P2 §Block scales and per-token activations]: NVFP4 = four-bit values     */
/* with one eight-bit E4M3 scale per 16 values; MXFP8 = 8-bit values with a  */
/* shared scale per 32 (8.25 bits/value).  The bit layouts are the OCP       */
/* microscaling definitions: E2M1 (bias 1, max 6), E4M3 "fn" (bias 7, max    */
/* 448, no infinities, S.1111.111 is NaN), E8M0 (2^(c-127), 0xFF NaN).       */
/* ------------------------------------------------------------------------ */

/* Magnitude of an E2M1 code (low three bits). */
static double e2m1_mag(int c) {
    int e = (c >> 1) & 3, m = c & 1;
    if (e == 0) return 0.5 * m;                  /* subnormal: m * 2^-1 */
    return ldexp(1.0 + 0.5 * m, e - 1);          /* (1.m) * 2^(e-1) */
}

/* Magnitude of an E4M3 code (low seven bits; 0x7f is NaN and never used). */
static double e4m3_mag(int c) {
    int e = (c >> 3) & 15, m = c & 7;
    if (e == 0) return ldexp((double)m, -9);     /* subnormal: m/8 * 2^-6 */
    return ldexp(8.0 + m, e - 10);               /* (1 + m/8) * 2^(e-7) */
}

ORC_API float orc_e2m1_decode(uint8_t c) {
    double v = e2m1_mag(c & 7);
    return (float)((c & 8) ? -v : v);
}

ORC_API float orc_e4m3_decode(uint8_t c) {
    if ((c & 0x7f) == 0x7f) return NAN;
    double v = e4m3_mag(c & 0x7f);
    return (float)((c & 0x80) ? -v : v);
}

ORC_API double orc_e8m0_decode(uint8_t c) {
    if (c == 0xff) return NAN;
    return ldexp(1.0, (int)c - 127);
}

/*
 * Round |x| to the nearest magnitude of a monotone code table mag(0..n_max),
 * ties to the code with an even last mantissa bit, values above the largest
 * finite magnitude clamp to it ("satfinite").  The search is a bisection for
 * the largest code not above |x|, then a comparison with its successor; the
 * differences are exact in double because every operand is an fp32 value or
 * a short dyadic rational.
 */
static int rne_code(double ax, double (*mag)(int), int n_max) {
    if (ax >= mag(n_max)) return n_max;
    int lo = 0, hi = n_max;                      /* mag(lo) <= ax < mag(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (mag(mid) <= ax) lo = mid; else hi = mid;
    }
    double dlo = ax - mag(lo), dhi = mag(hi) - ax;
    if (dlo < dhi) return lo;
    if (dhi < dlo) return hi;
    return (lo & 1) ? hi : lo;                   /* tie: even mantissa bit */
}

/* E2M1, round-to-nearest-even, saturating, sign kept (negative -> 0x8 | c). */
ORC_API uint8_t orc_e2m1_encode(float x) {
    int c = rne_code(fabs((double)x), e2m1_mag, 7);
    return (uint8_t)(c | (signbit(x) ? 8 : 0));
}

/* E4M3, round-to-nearest-even, saturating to 448, sign kept. */
ORC_API uint8_t orc_e4m3_encode(float x) {
    int c = rne_code(fabs((double)x), e4m3_mag, 0x7e);
    return (uint8_t)(c | (signbit(x) ? 0x80 : 0));
}

ORC_API void orc_e2m1_encode_array(const float* x, int64_t n, uint8_t* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(x[i]);
}

ORC_API void orc_e4m3_encode_array(const float* x, int64_t n, uint8_t* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(x[i]);
}

/* Round-to-nearest on an arbitrary sorted grid (the toy two-value format of
 * [P3 §Why Fewer Bits Means Faster Training]); ties go to the lower value. */
ORC_API double orc_round_nearest_on_grid(double x, const double* grid, int n) {
    double best = grid[0];
    for (int i = 1; i < n; ++i)
        if (fabs(x - grid[i]) < fabs(x - best)) best = grid[i];
    return best;
}

/* ------------------------------------------------------------------------ */
/* Philox4x32-10, written from Salmon, Moraes, Dror, Shaw, "Parallel Random  */
/* Numbers: As Easy as 1, 2, 3" (SC'11): each round multiplies counter words */
/* 0 and 2 by the two round constants, crosses the high halves with words    */
/* 1 and 3 and the key, and the key is advanced by the two Weyl constants    */
/* between rounds.  The pages only say "stochastic rounding"; the generator  */
/* is a reading taken here (a counter-based stream the GPU can reproduce).   */
/* ------------------------------------------------------------------------ */

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

ORC_API void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += PHILOX_W0; k1 += PHILOX_W1; }
        uint64_t p0 = (uint64_t)PHILOX_M0 * c0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * c2;
        uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        uint32_t n1 = (uint32_t)p1;
        uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        uint32_t n3 = (uint32_t)p0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/*
 * The random integer u in [0, 2^R) used for output element L of one call.
 * Reading taken (pages silent): block g = L / (128/R) of the stream is one
 * Philox call with counter (g_lo, g_hi, stream_lo, stream_hi) and key
 * (seed_lo, seed_hi); element j = L mod (128/R) takes bits [jR mod 32, +R)
 * of output word floor(jR/32).
 */
ORC_API uint32_t orc_sr_bits(uint64_t seed, uint64_t stream, int R, uint64_t L) {
    uint64_t per = 128u / (uint64_t)R;
    uint64_t g = L / per, j = L % per;
    uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), (uint32_t)stream, (uint32_t)(stream >> 32)};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t w[4];
    orc_philox4x32_10(ctr, key, w);
    uint64_t bit = j * (uint64_t)R;
    uint32_t word = w[bit / 32];
    if (R == 32) return word;
    return (word >> (bit % 32)) & ((1u << R) - 1u);
}

/* ------------------------------------------------------------------------ */
/* Stochastic rounding onto a minifloat grid.                                */
/* [P2 §Stochastic rounding across transposes]: a value between two grid    */
/* points goes up with probability equal to its fractional distance, so the  */
/* expectation is preserved (4.5 on the E2M1 grid -> 4 w.p. 0.75, 6 w.p.     */
/* 0.25).  Reading taken for the discrete rule: with R random bits u, round  */
/* up iff u < floor(frac * 2^R).  All arithmetic is exact in double: y is an */
/* fp32 value times a power of two, the quantum is a power of two.           */
/* mbits = mantissa bits, qmin = exponent of the smallest subnormal step.    */
/* Returns the signed grid value.                                            */
/* ------------------------------------------------------------------------ */

ORC_API double orc_sr_value(double y, uint32_t u, int R, int mbits, int qmin) {
    double ay = fabs(y);
    if (ay == 0.0) return y;                     /* keeps the sign of zero */
    int E2;
    (void)frexp(ay, &E2);                        /* ay = f * 2^E2, f in [0.5,1) */
    int fl = E2 - 1;                             /* floor(log2 ay) */
    int Q = fl - mbits;
    if (Q < qmin) Q = qmin;
    double q = ldexp(1.0, Q);
    double lo = floor(ay / q) * q;
    double frac = (ay - lo) / q;                 /* exact, in [0,1) */
    double thr = floor(ldexp(frac, R));          /* floor(frac * 2^R) */
    double r = ((double)u < thr) ? lo + q : lo;
    return signbit(y) ? -r : r;
}

/* SR onto the E4M3 grid (|y| <= 448 is guaranteed by the caller's scale). */
ORC_API uint8_t orc_e4m3_sr(double y, uint32_t u, int R) {
    double v = orc_sr_value(y, u, R, 3, -9);
    return orc_e4m3_encode((float)v);            /* v is on the grid: exact */
}

/* SR onto the E2M1 grid (used by the worked-example pin). */
ORC_API uint8_t orc_e2m1_sr(double y, uint32_t u, int R) {
    double v = orc_sr_value(y, u, R, 1, -1);
    return orc_e2m1_encode((float)v);
}

/* ------------------------------------------------------------------------ */
/* NVFP4 quantisation.                                                       */
/* [P2 §Block scales and per-token activations]: E2M1 codes, one E4M3 scale  */
/* per 16 consecutive values along a row, plus an FP32 outer scale: one per  */
/* token for activations, one per expert for weights.                        */
/* Readings taken (pages give no formula):                                   */
/*   s   = amax / (6 * 448)            (outer scale; 0 if amax == 0)         */
/*   sf  = E4M3_rne_sat(amax_b / (6 * s))     per 16-block                   */
/*   q_i = E2M1_rne_sat(x_i * (1 / (sf * s)))  (codes 0 if sf == 0)          */
/* Codes are packed two per byte, element 2j in the low nibble.              */
/* group_rows = rows sharing one outer scale (1: per token; N: per expert).  */
/* sf is written row-major [rows][cols/16]; outer has rows/group_rows items. */
/* ------------------------------------------------------------------------ */

ORC_API void orc_nvfp4_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t group_rows,
                                uint8_t* codes, uint8_t* sf, float* outer) {
    int64_t ngroups = rows / group_rows;
    int64_t nblk = cols / 16;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t g = 0; g < ngroups; ++g) {
        const uint16_t* xg = x + g * group_rows * cols;
        float amax = 0.0f;
        for (int64_t i = 0; i < group_rows * cols; ++i) {
            float a = fabsf(bf16_to_f32(xg[i]));
            if (a > amax) amax = a;
        }
        float s = amax / 2688.0f;                /* 2688 = 6 * 448 */
        outer[g] = s;
        for (int64_t r = g * group_rows; r < (g + 1) * group_rows; ++r) {
            for (int64_t b = 0; b < nblk; ++b) {
                const uint16_t* xb = x + r * cols + b * 16;
                uint8_t* cb = codes + (r * cols + b * 16) / 2;
                float ab = 0.0f;
                for (int i = 0; i < 16; ++i) {
                    float a = fabsf(bf16_to_f32(xb[i]));
                    if (a > ab) ab = a;
                }
                uint8_t sc = 0;
                if (s > 0.0f) {
                    float t = 6.0f * s;
                    float d = ab / t;
                    sc = orc_e4m3_encode(d);
                }
                sf[r * nblk + b] = sc;
                if (sc == 0) { memset(cb, 0, 8); continue; }
                float den = orc_e4m3_decode(sc) * s;
                float inv = 1.0f / den;
                for (int i = 0; i < 16; i += 2) {
                    float v0 = bf16_to_f32(xb[i]) * inv;
                    float v1 = bf16_to_f32(xb[i + 1]) * inv;
                    cb[i / 2] = (uint8_t)(orc_e2m1_encode(v0) | (orc_e2m1_encode(v1) << 4));
                }
            }
        }
    }
}

/* q * sf of NVFP4 element (r, c): exact in fp32 (at most 6 significant bits). */
static float nvfp4_block_product(const uint8_t* codes, const uint8_t* sf, int64_t cols, int64_t r, int64_t c) {
    uint8_t byte = codes[(r * cols + c) / 2];
    uint8_t q = (c & 1) ? (byte >> 4) : (byte & 15);
    return orc_e2m1_decode(q) * orc_e4m3_decode(sf[r * (cols / 16) + c / 16]);
}

/* Dequantised NVFP4 value: (q * sf) * s, one fp32 rounding. */
static float nvfp4_value(const uint8_t* codes, const uint8_t* sf, const float* outer,
                         int64_t cols, int64_t group_rows, int64_t r, int64_t c) {
    return nvfp4_block_product(codes, sf, cols, r, c) * outer[r / group_rows];
}

ORC_API void orc_nvfp4_dequantize(const uint8_t* codes, const uint8_t* sf, const float* outer,
                                  int64_t rows, int64_t cols, int64_t group_rows, float* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            out[r * cols + c] = nvfp4_value(codes, sf, outer, cols, group_rows, r, c);
}

/* ------------------------------------------------------------------------ */
/* MXFP8 shared scale.                                                       */
/* Reading taken (pages say only "MXFP8"; the E8M0-per-32 form is the OCP    */
/* MX format): the block exponent e is the smallest integer with             */
/* amax <= 448 * 2^e, clamped to [-127, 127]; e = -127 for an all-zero       */
/* block.  No element is clipped, so stochastic rounding stays unbiased.     */
/* Returns e.                                                                */
/* ------------------------------------------------------------------------ */

ORC_API int orc_e8m0_exponent(double amax) {
    if (amax == 0.0) return -127;
    int E2;
    double f = frexp(amax, &E2);                 /* amax = f * 2^E2, f in [0.5,1) */
    double m = 2.0 * f;                          /* amax = m * 2^(E2-1), m in [1,2) */
    int E = E2 - 1;
    int e = (m <= 1.75) ? E - 8 : E - 7;         /* 448 = 1.75 * 2^8 */
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* ------------------------------------------------------------------------ */
/* Re-quantisation of a saved NVFP4 tensor to MXFP8 across a transpose.      */
/* [P2 §Stochastic rounding across transposes]: dequantise the saved tensor, */
/* transpose in higher precision, re-quantise to MXFP8 with stochastic       */
/* rounding.  Readings taken: dequantisation in fp32; the input [rows, cols] */
/* becomes out[c][r] (the full transpose, [cols, rows]); blocks of 32 run    */
/* along r.  Expert segments start at multiples of 32 rows, so no block      */
/* crosses an expert and a per-expert transpose is a column range of this    */
/* one.  group_rows = rows sharing one outer scale (1 for activations, N for */
/* an expert weight stack [E*N, K]).  Scales row-major [cols][rows/32].      */
/* Random bits: orc_sr_bits with L = c*rows + r, the output element index.   */
/* ------------------------------------------------------------------------ */

ORC_API void orc_mxfp8_requant_transpose_sr(const uint8_t* codes, const uint8_t* sf, const float* outer,
                                            int64_t rows, int64_t cols, int64_t group_rows,
                                            uint64_t seed, uint64_t stream, int R,
                                            uint8_t* out_codes, uint8_t* out_e8m0) {
    int64_t nb = rows / 32;
    #pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < cols; ++c) {
        for (int64_t b = 0; b < nb; ++b) {
            float xh[32];
            double amax = 0.0;
            for (int t = 0; t < 32; ++t) {
                xh[t] = nvfp4_value(codes, sf, outer, cols, group_rows, b * 32 + t, c);
                if (fabs((double)xh[t]) > amax) amax = fabs((double)xh[t]);
            }
            int e = orc_e8m0_exponent(amax);
            out_e8m0[c * nb + b] = (uint8_t)(e + 127);
            for (int t = 0; t < 32; ++t) {
                int64_t L = c * rows + b * 32 + t;
                double y = ldexp((double)xh[t], -e);            /* exact */
                out_codes[L] = orc_e4m3_sr(y, orc_sr_bits(seed, stream, R, (uint64_t)L), R);
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* MXFP8 quantisation of a bf16 gradient ([P2 §NVFP4 forward, MXFP8          */
/* backward]: gradients are computed with MXFP8 matrix multiplications).     */
/* Reading taken: same E8M0 rule; E4M3 round-to-nearest-even by default      */
/* (sr = 1 uses the stochastic rule and stream above).                       */
/* Row-wise form: blocks of 32 along each row, codes [rows][cols], scales    */
/* row-major [rows][cols/32].                                                */
/* ------------------------------------------------------------------------ */

static uint8_t mx_round(double y, int sr, uint64_t seed, uint64_t stream, int R, uint64_t L) {
    if (!sr) return orc_e4m3_encode((float)y);  /* y is an fp32 value times 2^-e: exact cast */
    return orc_e4m3_sr(y, orc_sr_bits(seed, stream, R, L), R);
}

ORC_API void orc_mxfp8_quantize_rows(const uint16_t* x, int64_t rows, int64_t cols, int sr,
                                     uint64_t seed, uint64_t stream, int R,
                                     uint8_t* codes, uint8_t* e8m0) {
    int64_t nb = cols / 32;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            double amax = 0.0;
            for (int t = 0; t < 32; ++t) {
                double a = fabs((double)bf16_to_f32(x[r * cols + b * 32 + t]));
                if (a > amax) amax = a;
            }
            int e = orc_e8m0_exponent(amax);
            e8m0[r * nb + b] = (uint8_t)(e + 127);
            for (int t = 0; t < 32; ++t) {
                int64_t L = r * cols + b * 32 + t;
                double y = ldexp((double)bf16_to_f32(x[L]), -e);
                codes[L] = mx_round(y, sr, seed, stream, R, (uint64_t)L);
            }
        }
    }
}

/* Column-wise form: out[c][r] = the transpose, blocks of 32 along r (the
 * rows of x), scales row-major [cols][rows/32].  Expert segments start at
 * multiples of 32 rows, so each expert's transposed block is a column range. */
ORC_API void orc_mxfp8_quantize_cols(const uint16_t* x, int64_t rows, int64_t cols,
                                     int sr, uint64_t seed, uint64_t stream, int R,
                                     uint8_t* codes, uint8_t* e8m0) {
    int64_t nb = rows / 32;
    #pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < cols; ++c) {
        for (int64_t b = 0; b < nb; ++b) {
            double amax = 0.0;
            for (int t = 0; t < 32; ++t) {
                double a = fabs((double)bf16_to_f32(x[(b * 32 + t) * cols + c]));
                if (a > amax) amax = a;
            }
            int e = orc_e8m0_exponent(amax);
            e8m0[c * nb + b] = (uint8_t)(e + 127);
            for (int t = 0; t < 32; ++t) {
                int64_t L = c * rows + b * 32 + t;
                double y = ldexp((double)bf16_to_f32(x[(b * 32 + t) * cols + c]), -e);
                codes[L] = mx_round(y, sr, seed, stream, R, (uint64_t)L);
            }
        }
    }
}

/* Dequantised MXFP8 value q * 2^e, exact in fp64. */
ORC_API void orc_mxfp8_dequantize(const uint8_t* codes, const uint8_t* e8m0, int64_t rows, int64_t cols,
                                  double* out) {
    int64_t nb = cols / 32;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            out[r * cols + c] = (double)orc_e4m3_decode(codes[r * cols + c]) *
                                orc_e8m0_decode(e8m0[r * nb + c / 32]);
}

/* NVFP4 dequantised to fp64 *without* the outer scale: q * sf exactly.  The
 * GEMM oracle sums these in fp64 and applies the outer scales afterwards. */
ORC_API void orc_nvfp4_block_values(const uint8_t* codes, const uint8_t* sf, int64_t rows, int64_t cols,
                                    double* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            uint8_t byte = codes[(r * cols + c) / 2];
            uint8_t q = (c & 1) ? (byte >> 4) : (byte & 15);
            out[r * cols + c] = (double)orc_e2m1_decode(q) * (double)orc_e4m3_decode(sf[r * (cols / 16) + c / 16]);
        }
}

/* ------------------------------------------------------------------------ */
/* NVFP4 in the backward pass: the pages' stated future work ([P2 §NVFP4     */
/* forward, MXFP8 backward]: four-bit arithmetic in the backward pass is     */
/* being explored; a first NVFP4 forward+backward attempt cost too much).    */
/* Readings taken (pages silent): the scale rules of orc_nvfp4_quantize      */
/* (outer s = amax / (6*448) per group of rows, one E4M3 scale of            */
/* amax_b / (6s) per 16 consecutive values of a row, both round-to-nearest); */
/* the element code is E2M1 of x / (sf*s), rounded stochastically with the   */
/* random integer of linear element index L = r*cols + c (orc_sr_bits,       */
/* orc_e2m1_sr; values past 6 saturate) when sr != 0, to nearest even       */
/* otherwise.  The input is fp32, so that a dequantised, transposed tensor   */
/* is re-quantised without an intermediate bf16 rounding.                    */
/* ------------------------------------------------------------------------ */
/* One block of 16 fp32 values under outer scale s: E4M3 scale code (0 when  */
/* s == 0 or the block is zero) and eight code bytes, element 2j in the low  */
/* nibble of byte j; L0 is the linear output index of element 0.             */
static uint8_t nvfp4_block_f32(const float* xb, float s, int sr, uint64_t seed, uint64_t stream, int R,
                               uint64_t L0, uint8_t* cb) {
    float bmax = 0.0f;
    for (int i = 0; i < 16; ++i)
        if (fabsf(xb[i]) > bmax) bmax = fabsf(xb[i]);
    const uint8_t scode = (s > 0.0f) ? orc_e4m3_encode(bmax / (6.0f * s)) : 0;
    memset(cb, 0, 8);
    if (scode == 0) return 0;
    const float inv = 1.0f / (orc_e4m3_decode(scode) * s);
    for (int i = 0; i < 16; ++i) {
        const float y = xb[i] * inv;
        const uint64_t L = L0 + (uint64_t)i;
        const uint8_t q = sr ? orc_e2m1_sr((double)y, orc_sr_bits(seed, stream, R, L), R)
                             : orc_e2m1_encode(y);
        cb[i / 2] |= (uint8_t)((i & 1) ? (q << 4) : q);
    }
    return scode;
}

ORC_API void orc_nvfp4_quantize_f32(const float* x, int64_t rows, int64_t cols, int64_t group_rows, int sr,
                                    uint64_t seed, uint64_t stream, int R,
                                    uint8_t* codes, uint8_t* sf, float* outer) {
    const int64_t nblk = cols / 16;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t g = 0; g < rows / group_rows; ++g) {
        float gmax = 0.0f;
        for (int64_t i = g * group_rows * cols; i < (g + 1) * group_rows * cols; ++i)
            if (fabsf(x[i]) > gmax) gmax = fabsf(x[i]);
        const float s = gmax / (6.0f * 448.0f);
        outer[g] = s;
        for (int64_t r = g * group_rows; r < (g + 1) * group_rows; ++r)
            for (int64_t b = 0; b < nblk; ++b)
                sf[r * nblk + b] = nvfp4_block_f32(x + r * cols + b * 16, s, sr, seed, stream, R,
                                                   (uint64_t)(r * cols + b * 16), codes + (r * cols + b * 16) / 2);
    }
}

/* The same blocks with the outer scale of each block given (s_blk, row-major */
/* [rows][cols/16]): for outer scales that change along a row, as those of a */
/* transposed tensor taken per expert segment of its columns.                */
ORC_API void orc_nvfp4_quantize_f32_block_outer(const float* x, int64_t rows, int64_t cols, const float* s_blk,
                                                int sr, uint64_t seed, uint64_t stream, int R,
                                                uint8_t* codes, uint8_t* sf) {
    const int64_t nblk = cols / 16;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nblk; ++b)
            sf[r * nblk + b] = nvfp4_block_f32(x + r * cols + b * 16, s_blk[r * nblk + b], sr, seed, stream, R,
                                               (uint64_t)(r * cols + b * 16), codes + (r * cols + b * 16) / 2);
}

/* ------------------------------------------------------------------------ */
/* The rejected alternative ([P2 §Stochastic rounding across transposes]):   */
/* one scale shared by each 16x16 tile, so that both orientations of the     */
/* tensor hold the same codes, at the price of outlier sensitivity (one      */
/* large value can force the tile's other values to round to zero).          */
/* Readings taken: the tile scale is E4M3 of tile_amax / (6s) with the outer */
/* scale s of orc_nvfp4_quantize_f32, one per group_rows rows (a multiple of */
/* 16, so that no tile straddles two outer scales); codes round to nearest   */
/* even.  sf_tile is row-major [rows/16][cols/16].                           */
/* ------------------------------------------------------------------------ */
ORC_API void orc_nvfp4_quantize_tile16(const float* x, int64_t rows, int64_t cols, int64_t group_rows,
                                       uint8_t* codes, uint8_t* sf_tile, float* outer) {
    const int64_t ntc = cols / 16;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t g = 0; g < rows / group_rows; ++g) {
        float gmax = 0.0f;
        for (int64_t i = g * group_rows * cols; i < (g + 1) * group_rows * cols; ++i)
            if (fabsf(x[i]) > gmax) gmax = fabsf(x[i]);
        const float s = gmax / (6.0f * 448.0f);
        outer[g] = s;
        for (int64_t tr = g * group_rows / 16; tr < (g + 1) * group_rows / 16; ++tr) {
            for (int64_t tc = 0; tc < ntc; ++tc) {
                float tmax = 0.0f;
                for (int64_t r = tr * 16; r < tr * 16 + 16; ++r)
                    for (int64_t c = tc * 16; c < tc * 16 + 16; ++c)
                        if (fabsf(x[r * cols + c]) > tmax) tmax = fabsf(x[r * cols + c]);
                const uint8_t scode = (s > 0.0f) ? orc_e4m3_encode(tmax / (6.0f * s)) : 0;
                sf_tile[tr * ntc + tc] = scode;
                const float inv = scode ? 1.0f / (orc_e4m3_decode(scode) * s) : 0.0f;
                for (int64_t r = tr * 16; r < tr * 16 + 16; ++r) {
                    uint8_t* cb = codes + (r * cols + tc * 16) / 2;
                    memset(cb, 0, 8);
                    if (scode == 0) continue;
                    for (int i = 0; i < 16; ++i) {
                        const uint8_t q = orc_e2m1_encode(x[r * cols + tc * 16 + i] * inv);
                        cb[i / 2] |= (uint8_t)((i & 1) ? (q << 4) : q);
                    }
                }
            }
        }
    }
}
