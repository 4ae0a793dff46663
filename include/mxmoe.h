/*
 * mxmoe.h -- C ABI of the B200 (sm_100a) library for 4-bit mixture-of-experts
 * training numerics: NVFP4 forward expert GEMMs, and MXFP8 backward GEMMs fed by
 * a dequantise -> transpose -> stochastic-rounding requantisation of the saved
 * NVFP4 tensors.
 *
 * The method is the one reported for Thinking Machines' "End-to-End 4-Bit
 * Training" (Inkling 2 Small).  Citations name the web page and its section:
 *   [ai-primer] "Inkling 2 Small uses four-bit training, Thinking Machines
 *               reports 8% and 20% savings" (ai-primer.com)
 *   [hermes]    "Thinking Machines' Inkling 2 Small Trains a 594B Model in 68
 *               Hours" (hermes-ai.net)
 *
 * Conventions for every entry point
 *   - Pointers marked "device" are CUDA device pointers owned by the caller;
 *     the library allocates no memory and keeps no pointer after returning.
 *   - Work is enqueued asynchronously on `stream`; outputs are valid after the
 *     stream is synchronised.  Nothing is synchronised inside a call.
 *   - Return value: MX_OK, or MX_EINVAL (bad argument; checked on the host
 *     before any launch, nothing is written), MX_ECUDA (launch failure;
 *     mx_last_cuda_error() gives the cudaError_t), MX_EUNSUPPORTED (device is
 *     not sm_100 or a mode that is not built).  Device-side bounded waits that
 *     expire are reported later by mx_sync_status() as MX_ETIMEOUT.
 *   - An empty problem (rows == 0, M_cap == 0, T == 0) succeeds without
 *     touching memory, and the pointers of its empty arrays may be NULL; a
 *     weight-gradient GEMM without routed rows writes zeros to its output.
 *   - bf16 tensors are row-major, 2 bytes per element.
 *   - NVFP4 tensor [rows, cols]: codes u8 [rows, cols/2] (E2M1, element 2j in
 *     the low nibble of byte j), E4M3 block scales (one per 16 consecutive
 *     elements of a row), fp32 outer scales (one per group of `group_rows`
 *     rows: 1 = per token, N = per expert matrix of N rows).
 *   - MXFP8 tensor [rows, cols]: codes u8 [rows, cols] (E4M3), E8M0 block
 *     scales (one per 32 consecutive elements of a row; value 2^(byte-127)).
 *   - Scale layouts (`sf_layout`):
 *       MX_SF_ROWMAJOR: scale (r, s) at byte r*S + s, S = cols/block.
 *       MX_SF_MMA: the tcgen05 block-scaled MMA layout.  Rows come in groups
 *         of 128 and scale columns in groups of 4; each (row group, column
 *         group) is a 512-byte atom stored at atom index
 *         (r/128)*(S/4) + s/4, and (r, s) sits at byte
 *         (r%32)*16 + ((r%128)/32)*4 + s%4 of its atom.  Needs rows % 128 == 0
 *         and S % 4 == 0.
 *   - Expert-major row buffers: `seg_offsets` (device, int64 [E+1]) gives the
 *     first row of each expert; every segment length is a multiple of 128
 *     (empty experts have length 0); seg_offsets[E] = M_pad <= M_cap, the
 *     allocated row count.  Rows in [M_pad, M_cap) belong to no expert.
 */
#ifndef MXMOE_H
#define MXMOE_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MX_API __attribute__((visibility("default")))
#else
#define MX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum { MX_OK = 0, MX_EINVAL = 1, MX_ECUDA = 2, MX_ETIMEOUT = 3, MX_EUNSUPPORTED = 4, MX_EDATA = 5 };
enum { MX_SF_ROWMAJOR = 0, MX_SF_MMA = 1 };
enum { MX_OUT_F32 = 0, MX_OUT_BF16 = 1 };
enum { MX_ROUND_RNE = 0, MX_ROUND_SR = 1 };
enum { MX_GEMM_DGRAD = 0, MX_GEMM_WGRAD = 1 };

/* Library version, for the bindings' sanity check. */
MX_API int mx_version(void);

/* cudaError_t of the last MX_ECUDA returned on this host thread. */
MX_API int mx_last_cuda_error(void);

/* Kernels this library has launched in this process so far (all threads,
 * all devices), for accounting by callers; the pages have no counterpart. */
MX_API unsigned long long mx_kernel_launches(void);

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device: MX_ETIMEOUT if a bounded wait inside a GEMM kernel
 * expired since the last call (that kernel's output is then undefined);
 * otherwise MX_EDATA if a routing call since the last call met an expert id
 * outside [0, E) or the same id twice in one token (those entries were left
 * out, see moe_route) or a row-group permutation met a group index past its
 * input; MX_ECUDA if the synchronisation failed; else MX_OK. */
MX_API int mx_sync_status(cudaStream_t stream);

/* Failure-detection self-test: one kernel waits on a barrier that nothing
 * completes, gives up after `limit_us` microseconds (1 .. 10^7) the way the
 * GEMM kernels' bounded waits do, and records MX_ETIMEOUT in the device status
 * word; the next mx_sync_status() returns MX_ETIMEOUT and clears it.  Nothing
 * faults and the context stays usable.  MX_EINVAL for a limit out of range.
 * The pages have no counterpart. */
MX_API int mx_wait_selftest(int64_t limit_us, cudaStream_t stream);

/* Bounds-checked build (libmxmoe_debug.so, built with -DMX_DEBUG_BOUNDS): the
 * kernels check the global indices they compute against the extents their
 * call's arguments give the buffers, skip an access out of range and count
 * it.  mx_debug_bounds_build() is 1 in that library and 0 in libmxmoe.so;
 * mx_debug_bounds_violations() synchronises nothing, reads the counts of
 * everything that has completed (the caller synchronises first), clears them
 * when `clear` is nonzero, and is always 0 in libmxmoe.so.  The pages have no
 * counterpart: it stands in for a memory checker. */
MX_API int mx_debug_bounds_build(void);
MX_API unsigned long long mx_debug_bounds_violations(int clear);

/* Bytes of a scale array of `rows` x `cols` elements with one scale per
 * `block` (16 or 32) elements in `sf_layout`; 0 if the shape is not allowed
 * for that layout. */
MX_API size_t mx_sf_bytes(int64_t rows, int64_t cols, int block, int sf_layout);

/* --------------------------------------------------------------------------
 * nvfp4_quantize -- bf16 [rows, cols] -> NVFP4.
 * [ai-primer §Block scales and per-token activations]: E2M1 values, one E4M3
 * scale per 16-value block, an FP32 outer scale per token (activations,
 * group_rows = 1) or per expert (weights [E*N, K], group_rows = N).
 * Per group: s = amax/2688 (2688 = 6*448, s = 0 for an all-zero group); per
 * block: sf = E4M3_rne_satfinite(amax_block / (6*s)); codes =
 * E2M1_rne_satfinite(x * (1/(sf*s))), all zero when sf == 0.  Every step is
 * one IEEE fp32 round-to-nearest operation.
 *   x      device bf16 [rows, cols]
 *   codes  device u8 [rows, cols/2];  sf device u8 mx_sf_bytes(rows,cols,16,sf_layout)
 *   outer  device f32 [rows/group_rows]
 * Requires cols % 16 == 0 (cols % 64 == 0 and rows % 128 == 0 for MX_SF_MMA),
 * rows % group_rows == 0, 16-byte aligned x and codes.
 * ------------------------------------------------------------------------ */
MX_API int nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t group_rows,
                   uint8_t* codes, uint8_t* sf, float* outer, int sf_layout, cudaStream_t stream);

/* --------------------------------------------------------------------------
 * mxfp8_requant_transpose_sr -- saved NVFP4 [rows, cols] -> MXFP8 transpose.
 * [ai-primer §Stochastic rounding across transposes]: dequantise the saved
 * tensor, transpose in higher precision, re-quantise to MXFP8 with stochastic
 * rounding so represented values are preserved in expectation.
 * Dequantised value: (q*sf)*s in fp32.  Output out[c][r] ([cols, rows]) with
 * one E8M0 scale per 32 consecutive r: e = smallest integer with
 * amax <= 448*2^e (clamped to [-127,127], -127 for a zero block); element
 * y = x*2^-e rounded onto the E4M3 grid stochastically: with the quantum q of
 * y's binade, round up iff u < floor(frac(y/q) * 2^rbits), u the rbits-bit
 * random integer of output element L = c*rows + r.
 * Random stream: Philox4x32-10 (Salmon et al., SC'11), key = (seed lo, seed
 * hi), counter = (g lo, g hi, stream_id lo, stream_id hi) with
 * g = L / (128/rbits); element L takes bits [j*rbits mod 32, +rbits) of word
 * floor(j*rbits/32), j = L mod (128/rbits).
 * Expert segments start at multiples of 32 rows, so each expert's transposed
 * block is a column range [seg_e, seg_e+1) of the output.
 *   codes/sf/outer  device NVFP4 input (sf in in_sf_layout), outer per
 *                   group_rows rows (1 for activations, N for a weight stack)
 *   out_codes       device u8 [cols, rows]
 *   out_e8m0        device u8 mx_sf_bytes(cols, rows, 32, out_sf_layout)
 *   rows_valid      device int64 or NULL: only r < *rows_valid are read and
 *                   written (an expert-major buffer passes &seg_offsets[E])
 * Requires rows % 128 == 0, cols % 64 == 0, rbits in {8, 16, 32}, group_rows 1
 * or a multiple of 128, rows < 2^31.
 * ------------------------------------------------------------------------ */
MX_API int mxfp8_requant_transpose_sr(const uint8_t* codes, const uint8_t* sf, const float* outer,
                               int64_t rows, int64_t cols, int64_t group_rows, int in_sf_layout,
                               const int64_t* rows_valid, uint64_t seed, uint64_t stream_id, int rbits,
                               uint8_t* out_codes, uint8_t* out_e8m0, int out_sf_layout, cudaStream_t stream);

/* --------------------------------------------------------------------------
 * mxfp8_quantize -- bf16 [rows, cols] -> MXFP8, row-wise and/or column-wise.
 * [ai-primer §NVFP4 forward, MXFP8 backward]: gradients are computed with
 * MXFP8 matrix multiplications.  Same E8M0 rule as above; rounding
 * MX_ROUND_RNE (E4M3 round-to-nearest-even) or MX_ROUND_SR (the stochastic
 * rule and stream above, L = index in the output written).
 *   row_codes [rows, cols], row_e8m0 (rows x cols, block 32): blocks along rows
 *   col_codes [cols, rows], col_e8m0 (cols x rows, block 32): the transpose,
 *     blocks along the original columns' length (tokens)
 * Either output pair may be NULL (not produced).  With both and SR, the
 * column-wise form uses stream_id + 1.  rows_valid as above.
 * Requires rows % 128 == 0, cols % 128 == 0.
 * ------------------------------------------------------------------------ */
MX_API int mxfp8_quantize(const void* x, int64_t rows, int64_t cols, int rounding, uint64_t seed,
                   uint64_t stream_id, int rbits, const int64_t* rows_valid,
                   uint8_t* row_codes, uint8_t* row_e8m0, uint8_t* col_codes, uint8_t* col_e8m0,
                   int sf_layout, cudaStream_t stream);

/* --------------------------------------------------------------------------
 * grouped_gemm_nvfp4 -- forward expert GEMM on tcgen05 block-scaled MMA.
 * [ai-primer §NVFP4 forward, MXFP8 backward]: forward expert-layer matmuls in
 * NVFP4 with a dedicated kernel.
 * For rows r of expert e (seg_offsets[e] <= r < seg_offsets[e+1]):
 *   out[r, n] = a_outer[r] * b_outer[e] * sum_k (qa*sfa)[r,k] * (qb*sfb)[e*N+n,k]
 * accumulated in fp32; bf16 output is the round-to-nearest of the fp32 value.
 *   A: NVFP4 [M_cap, K], sf MX_SF_MMA, outer per row
 *   B: NVFP4 [E*N, K] (expert weight stack), sf MX_SF_MMA, outer per expert
 *   out: [M_cap, N] f32 or bf16 (out_dtype); rows >= seg_offsets[E] untouched
 * Requires K % 256 == 0, N % 128 == 0, M_cap % 128 == 0, 1 <= E.
 * Enqueues one kernel on `stream`, or two when N % 256 == 0 and E <= 768: CTA
 * pairs over 256-row tiles, then single CTAs for the experts' leftover
 * 128-row tiles (the same holds for grouped_gemm_nvfp4_s2f6 and for
 * grouped_gemm_mxfp8's DGRAD mode).
 * ------------------------------------------------------------------------ */
MX_API int grouped_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_outer,
                       const uint8_t* b_codes, const uint8_t* b_sf, const float* b_outer,
                       const int64_t* seg_offsets, int64_t E, int64_t M_cap, int64_t N, int64_t K,
                       void* out, int out_dtype, cudaStream_t stream);

/* --------------------------------------------------------------------------
 * grouped_gemm_mxfp8 -- backward expert GEMMs on tcgen05 block-scaled MMA.
 * [ai-primer §Stochastic rounding across transposes]: gradients come from
 * MXFP8 matrix multiplications of the re-quantised tensors.
 * MX_GEMM_DGRAD (input gradient), contraction length K (the forward N):
 *   A: MXFP8 [M_cap, K] (row-wise gradient), B: MXFP8 [N, E*K] (the
 *   transposed weight stack; expert e = columns [e*K, (e+1)*K)),
 *   out[r, n] = sum_k A[r,k] * B[n, e*K+k] for rows r of expert e; out [M_cap, N];
 *   rows >= seg_offsets[E] untouched.
 * MX_GEMM_WGRAD (weight gradient), contraction over each expert's tokens:
 *   A: MXFP8 [N, M_cap], B: MXFP8 [K, M_cap] (column-wise forms),
 *   out[e, n, k] = sum over t in segment e of A[n,t] * B[k,t]; out [E, N, K];
 *   an empty expert gets zeros.
 * All scales MX_SF_MMA.  Requires K % 128 == 0 and N % 128 == 0 (DGRAD);
 * N % 128 == 0, K % 128 == 0, M_cap % 128 == 0 (WGRAD).
 * ------------------------------------------------------------------------ */
MX_API int grouped_gemm_mxfp8(int mode, const uint8_t* a_codes, const uint8_t* a_e8m0,
                       const uint8_t* b_codes, const uint8_t* b_e8m0,
                       const int64_t* seg_offsets, int64_t E, int64_t M_cap, int64_t N, int64_t K,
                       void* out, int out_dtype, cudaStream_t stream);

/* --------------------------------------------------------------------------
 * Expert-layer glue (routing permutation, NVFP4 dispatch, SwiGLU, combine).
 * [ai-primer §Quantized NVLink and BBBK]: tokens travel to their experts in
 * NVFP4 and the backward pass reuses the quantised forward activations;
 * [hermes §594B weights, 17B at work]: each token uses 8 of 384 experts.
 * ------------------------------------------------------------------------ */

/* Scratch bytes moe_route needs for T tokens and E experts. */
MX_API size_t mx_route_workspace_bytes(int64_t T, int64_t E);

/* moe_route -- top-k expert ids -> expert-major row order.
 *   topk       device int32 [T, k], distinct ids in [0, E) per token
 *   seg_offsets device int64 [E+1] out: segment starts, each segment padded
 *              to a multiple of 128 rows
 *   src        device int32 [M_cap] out: t*k + j of the assignment stored at
 *              that row, -1 for padding rows and rows >= seg_offsets[E]
 *   pos        device int32 [T, k] out: row of assignment (t, j)
 *   workspace  device, mx_route_workspace_bytes(T, E) bytes of scratch
 * Rows of one expert are in increasing token order.  M_cap must be at least
 * T*k + 127*E rounded up to 128; (E+1)*8 <= 48 KiB; T*k < 2^31.
 * An entry whose id is outside [0, E), or repeats an id of an earlier entry of
 * the same token, is left out: it takes no row, its pos is -1 (moe_combine,
 * moe_combine_s2f6 and moe_dispatch_grad skip such entries), and the next
 * mx_sync_status() returns MX_EDATA.  Nothing is read or written outside the
 * buffers above.  The launches stop at the first launch failure (MX_ECUDA). */
MX_API int moe_route(const int32_t* topk, int64_t T, int64_t k, int64_t E, int64_t M_cap,
              int64_t* seg_offsets, int32_t* src, int32_t* pos,
              void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* moe_route_aligned -- moe_route with each segment padded to a multiple of
 * `align` rows (128 or 256; 256 for the NVFP4 wgrad GEMM, whose K-stage holds
 * 256 tokens).  M_cap must be a multiple of align and at least T*k +
 * (align-1)*E rounded up to align.  With align = 128 it is moe_route. */
MX_API int moe_route_aligned(const int32_t* topk, int64_t T, int64_t k, int64_t E, int64_t align, int64_t M_cap,
                             int64_t* seg_offsets, int32_t* src, int32_t* pos,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* moe_route_static -- moe_route without a caller-provided workspace.
 * The pages describe nothing like this; it exists for callers that cannot
 * allocate device memory for scratch (for example code running inside an
 * allocator or memory-pool callback, or a host runtime that owns every device
 * allocation).  The scratch is a fixed 1 MiB array inside the library's device
 * image, held by every GPU that loads the library until the process exits.
 * Arguments and outputs are those of moe_route.  Returns MX_EINVAL when
 * mx_route_workspace_bytes(T, E) exceeds 1 MiB.  Allocates nothing and frees
 * nothing.  The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * Every call uses the same array, and each call writes every scratch word it
 * reads, so no clearing is needed; calls that can overlap on the GPU (other
 * streams, other host threads) race on the array and give undefined results. */
MX_API int moe_route_static(const int32_t* topk, int64_t T, int64_t k, int64_t E, int64_t M_cap,
                            int64_t* seg_offsets, int32_t* src, int32_t* pos, cudaStream_t stream);

/* moe_permute_row_groups -- reorder an expert-major row buffer by whole
 * groups of 128 rows (the unit every expert segment is padded to).
 * [ai-primer §Quantized NVLink and BBBK]: tokens travel to the GPU holding
 * their expert in NVFP4 and come back through the combine; in that exchange
 * rows arrive grouped by source rank, and this call regroups them by expert
 * (and back) without touching their bytes.
 *   in         device, ngroups_in groups of group_bytes bytes (one array of a
 *              row buffer: codes, MMA-layout scales, outer scales, bf16 rows...)
 *   out        device, ngroups_out groups of group_bytes bytes
 *   group_src  device int32 [ngroups_out]: input group of output group g, or
 *              -1 for a group of zeros
 * An index >= ngroups_in is written as zeros and the next mx_sync_status()
 * returns MX_EDATA.  Requires group_bytes % 16 == 0 and 16-byte aligned
 * in/out; in and out must not overlap. */
MX_API int moe_permute_row_groups(const void* in, int64_t ngroups_in, void* out, int64_t ngroups_out,
                                  int64_t group_bytes, const int32_t* group_src, cudaStream_t stream);

/* nvfp4_gather_rows -- dispatch per-token NVFP4 rows into expert-major order:
 * row p of the output is row src[p]/k of the input (zeros when src[p] < 0).
 * Input sf MX_SF_ROWMAJOR, output sf MX_SF_MMA.  Writes all M_cap rows.
 * Requires cols % 64 == 0, M_cap % 128 == 0. */
MX_API int nvfp4_gather_rows(const uint8_t* codes, const uint8_t* sf, const float* outer,
                      const int32_t* src, int64_t k, int64_t M_cap, int64_t cols,
                      uint8_t* out_codes, uint8_t* out_sf, float* out_outer, cudaStream_t stream);

/* swiglu_fwd -- a = silu(g)*u (gated: g = h[:, :F], u = h[:, F:]) or
 * a = silu(h) (not gated), fp32 math, bf16 round-to-nearest output.
 *   h device bf16 [rows, 2F or F];  a device bf16 [rows, F]
 * Rows >= *rows_valid (when rows_valid != NULL) are written as zero. */
MX_API int swiglu_fwd(const void* h, int64_t rows, int64_t F, int gated, const int64_t* rows_valid,
               void* a, cudaStream_t stream);

/* swiglu_bwd -- dh from h and da (analytic derivative of swiglu_fwd). */
MX_API int swiglu_bwd(const void* h, const void* da, int64_t rows, int64_t F, int gated,
               const int64_t* rows_valid, void* dh, cudaStream_t stream);

/* swiglu_nvfp4_quantize -- swiglu_fwd fused into nvfp4_quantize (per-token
 * outer scale, group_rows = 1): each a = silu(g)*u is rounded to bf16 exactly
 * as swiglu_fwd rounds it and quantised exactly as nvfp4_quantize quantises a
 * bf16 row, so the outputs equal those two calls in sequence while a never
 * reaches HBM ([ai-primer §NVFP4 forward, MXFP8 backward]: both expert GEMMs
 * of the forward pass take NVFP4 operands).  h bf16 [rows, 2F] (gated, g then
 * u) or [rows, F]; rows at or past *rows_valid (when rows_valid != NULL)
 * quantise as zero rows.  Outputs as nvfp4_quantize of [rows, F].  F % 16 ==
 * 0 and F <= 16384 (F % 64 == 0 and rows % 128 == 0 for MX_SF_MMA); h and
 * codes 16-byte aligned; else MX_EINVAL. */
MX_API int swiglu_nvfp4_quantize(const void* h, int64_t rows, int64_t F, int gated, const int64_t* rows_valid,
                                 uint8_t* codes, uint8_t* sf, float* outer, int sf_layout, cudaStream_t stream);

/* moe_combine -- out[t] = sum_j w[t,j] * y[pos[t,j]], fp32 accumulation,
 * bf16 output.  y device bf16 [*, D], pos int32 [T, k], w f32 [T, k] (NULL:
 * all weights 1). */
MX_API int moe_combine(const void* y, const int32_t* pos, const float* w, int64_t T, int64_t k, int64_t D,
                void* out, cudaStream_t stream);

/* moe_dispatch_grad -- gradient of moe_combine w.r.t. y:
 * dy[p] = w[src[p]] * dout[src[p]/k] (bf16), zero rows where src[p] < 0.
 * dout bf16 [T, D]; src int32 [M_cap] and pos int32 [T, k] as written by
 * moe_route (pos[t*k + j] is the row of token t's j-th copy, so
 * src[pos[i]] == i); w fp32 [T, k] or NULL (all ones); dy bf16 [M_cap, D].
 * Writes all M_cap rows, reading each token's row of dout once.  dout and dy
 * 16-byte aligned, D a multiple of 8; else MX_EINVAL. */
MX_API int moe_dispatch_grad(const void* dout, const int32_t* src, const int32_t* pos, const float* w, int64_t T,
                             int64_t k, int64_t M_cap, int64_t D, void* dy, cudaStream_t stream);

/* moe_dispatch_grad_mxfp8_quantize -- moe_dispatch_grad fused into the
 * gradient quantiser that follows it ([ai-primer §NVFP4 forward, MXFP8
 * backward]: the gradients enter the backward GEMMs as MXFP8).  Writes what
 * moe_dispatch_grad(dout, src, ., w) followed by mxfp8_quantize (MX_ROUND_RNE,
 * both forms, the same rows_valid) of dy [M_cap, D] writes, byte for byte,
 * without dy reaching HBM: each row is gathered from its token's row of dout
 * and scaled as moe_dispatch_grad scales it.  Outputs as mxfp8_quantize:
 * row_codes [M_cap, D], row_e8m0, col_codes [D, M_cap], col_e8m0
 * (sf_layout); row tiles at or past *rows_valid are not written.  Requires
 * M_cap % 128 == 0, D % 128 == 0, k >= 1, all four outputs, dout and codes
 * 16-byte aligned; else MX_EINVAL. */
MX_API int moe_dispatch_grad_mxfp8_quantize(const void* dout, const int32_t* src, const float* w, int64_t T,
                                            int64_t k, int64_t M_cap, int64_t D, const int64_t* rows_valid,
                                            uint8_t* row_codes, uint8_t* row_e8m0, uint8_t* col_codes,
                                            uint8_t* col_e8m0, int sf_layout, cudaStream_t stream);

/* --------------------------------------------------------------------------
 * Combine path in S2F6.  [ai-primer §Quantized NVLink and BBBK]: expert
 * outputs are rotated by a 32-dimensional random Hadamard transform and
 * quantised into block-scaled S2F6 (eight-bit fixed point, two signed integer
 * bits and six fractional bits) for the combine, the transform and the
 * quantisation folded into the output GEMM's epilogue.  The pages give the
 * format's bit split only; the readings taken here:
 *   rotation  per 32-column block j of a row, z = H32 (sigma_j * x): H32 the
 *             unnormalised Sylvester-Hadamard matrix (H[a][b] =
 *             (-1)^popcount(a & b)), evaluated as five butterfly stages
 *             h = 1, 2, 4, 8, 16 of fp32 adds (a, b) -> (a + b, a - b) on the
 *             pairs (i, i + h), i & h == 0; sigma_j negates coordinate i when
 *             bit i of word 0 of Philox4x32-10(counter (j lo, j hi, stream_id
 *             lo, stream_id hi), key (seed lo, seed hi)) is set.  The inverse
 *             is x = sigma_j * (H32 z) / 32.
 *   scale     one E8M0 byte per block, e + 127 with e the smallest integer
 *             such that max|z| <= (127/64) * 2^e, clamped to [-127, 127]
 *             (-127 for a zero block).
 *   codes     int8 c = round-half-even(z * 2^(6-e)) clamped to [-127, 127];
 *             value c * 2^(e-6).
 * Layout: codes int8 [rows, cols] row-major, exponents u8 [rows, cols/32]
 * row-major.  Inputs finite.
 * ------------------------------------------------------------------------ */

/* hadamard_s2f6_quantize -- bf16 x [rows, cols] -> S2F6 codes and exponents
 * (the unfused form: x holds bf16 expert outputs).  cols % 32 == 0, x and
 * codes 16-byte aligned; else MX_EINVAL.  rows == 0 succeeds without touching
 * memory. */
MX_API int hadamard_s2f6_quantize(const void* x, int64_t rows, int64_t cols, uint64_t seed, uint64_t stream_id,
                                  int8_t* codes, uint8_t* e8m0, cudaStream_t stream);

/* grouped_gemm_nvfp4_s2f6 -- grouped_gemm_nvfp4 with the S2F6 epilogue: each
 * output row's fp32 values (those the MX_OUT_F32 form would store) are rotated
 * and quantised per 32-column block as above, in the registers that drain
 * the accumulator.  Arguments and requirements as grouped_gemm_nvfp4, the
 * output being codes int8 [M_cap, N] and e8m0 u8 [M_cap, N/32] (rows of
 * padding hold codes of zero sums).  codes 16-byte and e8m0 8-byte aligned;
 * else MX_EINVAL. */
MX_API int grouped_gemm_nvfp4_s2f6(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_outer,
                                   const uint8_t* b_codes, const uint8_t* b_sf, const float* b_outer,
                                   const int64_t* seg_offsets, int64_t E, int64_t M_cap, int64_t N, int64_t K,
                                   uint64_t seed, uint64_t stream_id, int8_t* codes, uint8_t* e8m0,
                                   cudaStream_t stream);

/* moe_combine_s2f6 -- moe_combine reading S2F6 rows: out[t] =
 * sum_j w[t,j] * xhat(pos[t,j]), xhat the rotated-back dequantised row.  The
 * sum is taken in the rotated domain (u = sum_j w_j 2^(e_j - 6) c_j, fp32,
 * j in order) and rotated back once per token block; bf16 round-to-nearest
 * output [T, D].  w NULL: all weights 1.  D % 32 == 0, codes and out 16-byte
 * aligned; else MX_EINVAL. */
MX_API int moe_combine_s2f6(const int8_t* codes, const uint8_t* e8m0, const int32_t* pos, const float* w,
                            int64_t T, int64_t k, int64_t D, uint64_t seed, uint64_t stream_id, void* out,
                            cudaStream_t stream);

/* --------------------------------------------------------------------------
 * NVFP4 in the backward pass, and the 16x16 shared-scale format.
 * [ai-primer §NVFP4 forward, MXFP8 backward]: four-bit arithmetic in the
 * backward pass is the lab's stated future work.  [ai-primer §Stochastic
 * rounding across transposes]: a scale shared by each 16x16 tile keeps both
 * orientations' codes equal but was rejected as outlier-sensitive.  The pages
 * give no rule; the readings taken here:
 *   scales    those of nvfp4_quantize: outer s = amax / 2688 per group of
 *             rows, E4M3 block scale RNE(amax_b / (6 s)) per 16 values;
 *   rounding  MX_ROUND_RNE: E2M1 of y = x * (1 / (sf s)) to nearest even, as
 *             nvfp4_quantize; MX_ROUND_SR: with q the E2M1 step at |y|
 *             (2^max(floor(log2|y|) - 1, -1)), lo = floor(|y| / q) q, round
 *             up to lo + q iff u < floor(((|y| - lo) / q) 2^rbits), u the
 *             rbits-bit random integer of the output element (the Philox
 *             stream of mxfp8_requant_transpose_sr, L = the element's linear
 *             index in the output); magnitudes past 6 saturate; the sign of y
 *             is kept, also on a zero.
 * ------------------------------------------------------------------------ */

/* nvfp4_quantize_sr -- bf16 [rows, cols] -> NVFP4 with the rounding above
 * (the gradient operands of an NVFP4 backward).  Arguments, layouts and
 * requirements as nvfp4_quantize, plus rounding, seed, stream_id and rbits
 * (8, 16 or 32 for MX_ROUND_SR).  With MX_ROUND_RNE the outputs equal those
 * of nvfp4_quantize. */
MX_API int nvfp4_quantize_sr(const void* x, int64_t rows, int64_t cols, int64_t group_rows, int rounding,
                             uint64_t seed, uint64_t stream_id, int rbits, uint8_t* codes, uint8_t* sf,
                             float* outer, int sf_layout, cudaStream_t stream);

/* nvfp4_requant_transpose_sr -- saved NVFP4 -> NVFP4 of its transpose.
 * The input [rows, cols] (codes, sf in in_sf_layout, outer per group_rows
 * rows) holds `experts` stacked blocks of rows / experts rows each (1 for an
 * activation tensor, E for an expert weight stack [E*N, K]; per-row outer
 * scales take experts = 1).  Each value is
 * dequantised ((q * sf) * outer, fp32), each block is transposed, and the
 * result [experts * cols, rows / experts] (block e's transpose in rows
 * e*cols ..) is quantised with the rounding above, blocks of 16 along the old
 * rows.  Outer scales: one per output row (out_outer_per_expert = 0; out_outer
 * [experts * cols]) or one per expert (1; out_outer [experts]).  With
 * experts = E this gives the stack of W_e^T that grouped_gemm_nvfp4 takes as
 * B for the NVFP4 input gradient (output width K).
 *   out_codes device u8 [experts*cols, rows/experts/2]; out_sf device u8
 *   mx_sf_bytes(experts*cols, rows/experts, 16, out_sf_layout)
 * Requires cols % 64 == 0, rows / experts % 128 == 0, rows % group_rows == 0,
 * rows <= 65535 * 128 (rows % 128 == 0 for an MX_SF_MMA input;
 * experts*cols % 128 == 0 for an MX_SF_MMA output), 16-byte aligned codes
 * and out_codes.  out_outer is
 * written twice (the per-target maxima, then the scales) by the calls this
 * entry point enqueues. */
MX_API int nvfp4_requant_transpose_sr(const uint8_t* codes, const uint8_t* sf, const float* outer, int64_t rows,
                                      int64_t cols, int64_t group_rows, int in_sf_layout, int64_t experts,
                                      int out_outer_per_expert, int rounding, uint64_t seed, uint64_t stream_id,
                                      int rbits, uint8_t* out_codes, uint8_t* out_sf, float* out_outer,
                                      int out_sf_layout, cudaStream_t stream);

/* nvfp4_quantize_tile16 -- bf16 [rows, cols] -> NVFP4 with one E4M3 scale per
 * 16x16 tile: scale RNE(tile_amax / (6 s)), codes RNE; outer s = amax / 2688
 * per group_rows rows (a multiple of 16).  Both orientations of the tensor
 * hold the same codes.
 *   codes device u8 [rows, cols/2]; sf_tile device u8 [rows/16, cols/16]
 *   row-major; outer device f32 [rows/group_rows]
 * Requires rows % 16 == 0, cols % 16 == 0, group_rows % 16 == 0, 16-byte
 * aligned x and codes. */
MX_API int nvfp4_quantize_tile16(const void* x, int64_t rows, int64_t cols, int64_t group_rows, uint8_t* codes,
                                 uint8_t* sf_tile, float* outer, cudaStream_t stream);

/* The wgrad operands of an NVFP4 backward: NVFP4 of the transpose [C, M] of a
 * token-major [M, C] tensor in expert-major row order (seg [E+1] from
 * moe_route: segment starts and lengths multiples of 128), blocks of 16 along
 * the tokens, with outer scales per expert segment so that the wgrad GEMM
 * applies a per-row times a per-expert factor: per (segment, row) when
 * per_row = 1 (out_outer [E, C], for dY^T), per segment when per_row = 0
 * (out_outer [E], for X^T).  Each scale is the segment's amax / 2688; rounding
 * as above with L = c*M + t; tokens at or past seg[E] quantise to zero.
 *   out_codes device u8 [C, M/2]; out_sf device u8 mx_sf_bytes(C, M, 16,
 *   out_sf_layout); out_outer written twice (maxima, then scales).
 * Requires M % 128 == 0, C % 64 == 0 (C % 128 == 0 for an MX_SF_MMA output),
 * 16-byte aligned inputs and out_codes.  Segment boundaries off multiples of
 * 128 give wrong scales (no out-of-bounds access). */
MX_API int nvfp4_quantize_transpose_segments(const void* x, int64_t M, int64_t C, const int64_t* seg, int64_t E,
                                             int per_row, int rounding, uint64_t seed, uint64_t stream_id,
                                             int rbits, uint8_t* out_codes, uint8_t* out_sf, float* out_outer,
                                             int out_sf_layout, cudaStream_t stream);

/* The same from a saved NVFP4 tensor [M, C] (codes, sf in in_sf_layout, outer
 * per group_rows rows), each value dequantised ((q * sf) * outer, fp32).
 * Also requires M <= 65535 * 128 and 16-byte aligned codes. */
MX_API int nvfp4_requant_transpose_segments(const uint8_t* codes, const uint8_t* sf, const float* outer,
                                            int in_sf_layout, int64_t group_rows, int64_t M, int64_t C,
                                            const int64_t* seg, int64_t E, int per_row, int rounding,
                                            uint64_t seed, uint64_t stream_id, int rbits, uint8_t* out_codes,
                                            uint8_t* out_sf, float* out_outer, int out_sf_layout,
                                            cudaStream_t stream);

/* grouped_gemm_nvfp4_wgrad -- the NVFP4 weight gradient on tcgen05
 * block-scaled MMA (kind::mxf4nvf4, the MXFP8 WGRAD tile schedule).
 *   A: NVFP4 [N, M_cap] (dY^T, codes [N, M_cap/2], sf MX_SF_MMA), a_outer
 *      [E*N] per (segment, row); B: NVFP4 [K, M_cap] (X^T), b_outer [E] per
 *      segment -- as nvfp4_quantize_transpose_segments /
 *      nvfp4_requant_transpose_segments write them;
 *   out[e, n, k] = a_outer[e*N + n] * b_outer[e] * sum over the tokens t of
 *      segment e of (qa*sfa)[n, t] * (qb*sfb)[k, t], fp32 accumulate; out
 *      [E, N, K] f32 or bf16; an empty expert gets zeros.
 * Requires segments at multiples of 256 tokens (a K-stage of NVFP4 holds 256
 * tokens; other boundaries give wrong sums, no out-of-bounds access),
 * M_cap % 256 == 0, N % 128 == 0, K % 128 == 0, 16-byte aligned operands. */
MX_API int grouped_gemm_nvfp4_wgrad(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_outer,
                                    const uint8_t* b_codes, const uint8_t* b_sf, const float* b_outer,
                                    const int64_t* seg_offsets, int64_t E, int64_t M_cap, int64_t N, int64_t K,
                                    void* out, int out_dtype, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MXMOE_H */
