// glue.cu -- expert-layer glue around the quantisers and GEMMs: routing
// permutation, NVFP4 dispatch gather, SiLU / SwiGLU, combine and its gradient.
//
// [ai-primer] "Inkling 2 Small uses four-bit training...", §Quantized NVLink and
// BBBK: tokens travel to their routed experts in NVFP4 and the backward pass
// reuses the quantised forward activations -- here the per-token NVFP4 rows are
// quantised once and gathered into expert-major order.
#include "mx_common.cuh"

#include <algorithm>
#include <mutex>

namespace {

constexpr int kChunk = 256;   // tokens per routing chunk

// Whether entry j of token t names an expert: an id in [0, E) that no earlier
// entry of the same token names.  Other entries are left out of the routing
// (their pos is -1) and flag the device status word.
__device__ __forceinline__ bool route_entry_valid(const int32_t* __restrict__ topk, int64_t t, int64_t k, int64_t j,
                                                  int64_t E) {
    const int32_t id = topk[t * k + j];
    if ((uint64_t)(uint32_t)id >= (uint64_t)E || id < 0) return false;
    for (int64_t i = 0; i < j; ++i)
        if (topk[t * k + i] == id) return false;
    return true;
}

// Per-chunk expert histogram: hist[c][e].
__global__ void route_count_kernel(const int32_t* __restrict__ topk, int64_t T, int64_t k, int64_t E,
                                   int32_t* __restrict__ hist, unsigned int* __restrict__ status) {
    extern __shared__ int32_t h[];
    for (int64_t e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    const int64_t t = (int64_t)blockIdx.x * kChunk + threadIdx.x;
    if (t < T)
        for (int64_t j = 0; j < k; ++j) {
            if (route_entry_valid(topk, t, k, j, E)) atomicAdd(&h[topk[t * k + j]], 1);
            else atomicOr(status, kStatusBadRoute);
        }
    __syncthreads();
    for (int64_t e = threadIdx.x; e < E; e += blockDim.x)
        if (mx_in_range((int64_t)blockIdx.x * E + e, 1, (int64_t)gridDim.x * E)) hist[(int64_t)blockIdx.x * E + e] = h[e];
}

// Totals, kAlign-padded exclusive scan into seg_offsets, and per-(chunk,
// expert) base rows written back over hist.
template <int kAlign>
__global__ void route_scan_kernel(int32_t* __restrict__ hist, int32_t* __restrict__ counts, int64_t nchunks,
                                  int64_t E, int64_t* __restrict__ seg) {
    extern __shared__ int64_t start[];   // [E + 1]
    for (int64_t e = threadIdx.x; e < E; e += blockDim.x) {
        int64_t c = 0;
        for (int64_t ch = 0; ch < nchunks; ++ch) c += hist[ch * E + e];
        counts[e] = (int32_t)c;
        start[e + 1] = (c + kAlign - 1) / kAlign * kAlign;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        start[0] = 0;
        for (int64_t e = 0; e < E; ++e) start[e + 1] += start[e];
    }
    __syncthreads();
    for (int64_t e = threadIdx.x; e <= E; e += blockDim.x) seg[e] = start[e];
    for (int64_t e = threadIdx.x; e < E; e += blockDim.x) {
        int64_t run = start[e];
        for (int64_t ch = 0; ch < nchunks; ++ch) {
            const int32_t c = hist[ch * E + e];
            hist[ch * E + e] = (int32_t)run;
            run += c;
        }
    }
}

// One warp per chunk: rows handed out in token order.  For each group of 32
// tokens a shared bitmask per expert marks the lanes that chose it; a lane's
// rank is the number of lower lanes in that mask.
__global__ void route_scatter_kernel(const int32_t* __restrict__ topk, int64_t T, int64_t k, int64_t E,
                                     int64_t M_cap, const int32_t* __restrict__ base, int32_t* __restrict__ src,
                                     int32_t* __restrict__ pos) {
    extern __shared__ uint32_t sm[];
    uint32_t* mask = sm;                                   // [E]
    int32_t* run = reinterpret_cast<int32_t*>(sm + E);     // [E]
    const int lane = threadIdx.x;
    for (int64_t e = lane; e < E; e += 32) { mask[e] = 0; run[e] = base[(int64_t)blockIdx.x * E + e]; }
    __syncwarp();
    const uint32_t below = (1u << lane) - 1u;
    for (int gi = 0; gi < kChunk / 32; ++gi) {
        const int64_t t = (int64_t)blockIdx.x * kChunk + gi * 32 + lane;
        const bool act = t < T;
        uint32_t valid = 0;   // bit j: entry j of this lane's token names an expert
        if (act)
            for (int64_t j = 0; j < k; ++j)
                if (route_entry_valid(topk, t, k, j, E)) {
                    valid |= 1u << j;
                    atomicOr(&mask[topk[t * k + j]], 1u << lane);
                }
        __syncwarp();
        if (act)
            for (int64_t j = 0; j < k; ++j) {
                if (!(valid >> j & 1u)) { pos[t * k + j] = -1; continue; }
                const int32_t e = topk[t * k + j];
                const int32_t p = run[e] + __popc(mask[e] & below);
                pos[t * k + j] = p;
                if (mx_in_range(p, 1, M_cap)) src[p] = (int32_t)(t * k + j);
            }
        __syncwarp();
        if (act)
            for (int64_t j = 0; j < k; ++j) {
                if (!(valid >> j & 1u)) continue;
                const int32_t e = topk[t * k + j];
                const uint32_t m = mask[e];
                if ((m & below) == 0) { run[e] += __popc(m); mask[e] = 0; }
            }
        __syncwarp();
    }
}

// src = -1 on each expert's padding rows and on rows >= seg[E].
__global__ void route_pad_kernel(const int64_t* __restrict__ seg, const int32_t* __restrict__ counts, int64_t E,
                                 int64_t M_cap, int32_t* __restrict__ src) {
    const int64_t e = blockIdx.x;
    int64_t a, b;
    if (e < E) { a = seg[e] + counts[e]; b = seg[e + 1]; }
    else { a = seg[E]; b = M_cap; }
    for (int64_t p = a + threadIdx.x; p < b; p += blockDim.x)
        if (mx_in_range(p, 1, M_cap)) src[p] = -1;
}

// One warp per output row.
__global__ void gather_rows_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf,
                                   const float* __restrict__ outer, const int32_t* __restrict__ src, int64_t k,
                                   int64_t M_cap, int64_t cols, uint8_t* __restrict__ out_codes,
                                   uint8_t* __restrict__ out_sf, float* __restrict__ out_outer) {
    const int lane = threadIdx.x & 31;
    const int64_t p = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (p >= M_cap) return;
    const int32_t sidx = src[p];
    const int64_t t = sidx < 0 ? -1 : sidx / k;
    const int64_t n16 = cols / 32;                         // uint4 of codes per row
    const uint4* ci = reinterpret_cast<const uint4*>(codes + (t < 0 ? 0 : t) * (cols / 2));
    uint4* co = reinterpret_cast<uint4*>(out_codes + p * (cols / 2));
    for (int64_t i = lane; i < n16; i += 32) co[i] = t < 0 ? make_uint4(0, 0, 0, 0) : __ldg(ci + i);
    const int64_t S = cols / 16;
    for (int64_t a = lane; a < S / 4; a += 32) {
        const uint32_t v = t < 0 ? 0u : __ldg(reinterpret_cast<const uint32_t*>(sf + t * S) + a);
        *reinterpret_cast<uint32_t*>(out_sf + sf_offset_mma(p, 4 * a, S)) = v;
    }
    if (lane == 0) out_outer[p] = t < 0 ? 0.0f : outer[t];
}


// 8 outputs per thread.
__global__ void swiglu_fwd_kernel(const uint16_t* __restrict__ h, int64_t rows, int64_t F, int gated,
                                  const int64_t* rows_valid, uint16_t* __restrict__ a) {
    const int64_t nv = F / 8;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows * nv) return;
    const int64_t r = i / nv, c = (i % nv) * 8;
    uint4 o = make_uint4(0, 0, 0, 0);
    if (r < load_rows_valid(rows_valid, rows)) {
        const int64_t hw = gated ? 2 * F : F;
        const uint4 gv = *reinterpret_cast<const uint4*>(h + r * hw + c);
        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
        uint32_t uw[4] = {0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u};   // bf16 1.0
        if (gated) {
            const uint4 uv = *reinterpret_cast<const uint4*>(h + r * hw + F + c);
            uw[0] = uv.x; uw[1] = uv.y; uw[2] = uv.z; uw[3] = uv.w;
        }
        uint32_t ow[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            ow[j] = swiglu_word(gw[j], uw[j]);
        o = make_uint4(ow[0], ow[1], ow[2], ow[3]);
    }
    *reinterpret_cast<uint4*>(a + r * F + c) = o;
}

__global__ void swiglu_bwd_kernel(const uint16_t* __restrict__ h, const uint16_t* __restrict__ da, int64_t rows,
                                  int64_t F, int gated, const int64_t* rows_valid, uint16_t* __restrict__ dh) {
    const int64_t nv = F / 8;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows * nv) return;
    const int64_t r = i / nv, c = (i % nv) * 8;
    const int64_t hw = gated ? 2 * F : F;
    uint4 og = make_uint4(0, 0, 0, 0), ou = make_uint4(0, 0, 0, 0);
    if (r < load_rows_valid(rows_valid, rows)) {
        const uint4 gv = *reinterpret_cast<const uint4*>(h + r * hw + c);
        const uint4 dv = *reinterpret_cast<const uint4*>(da + r * F + c);
        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, dw[4] = {dv.x, dv.y, dv.z, dv.w};
        uint32_t uw[4] = {0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u};
        if (gated) {
            const uint4 uv = *reinterpret_cast<const uint4*>(h + r * hw + F + c);
            uw[0] = uv.x; uw[1] = uv.y; uw[2] = uv.z; uw[3] = uv.w;
        }
        uint32_t wg[4], wu[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            wg[j] = swiglu_bwd_gate_word(gw[j], uw[j], dw[j]);
            wu[j] = swiglu_bwd_up_word(gw[j], dw[j]);
        }
        og = make_uint4(wg[0], wg[1], wg[2], wg[3]);
        ou = make_uint4(wu[0], wu[1], wu[2], wu[3]);
    }
    *reinterpret_cast<uint4*>(dh + r * hw + c) = og;
    if (gated) *reinterpret_cast<uint4*>(dh + r * hw + F + c) = ou;
}

// One block per token; 8 bf16 per thread per step.
__global__ void combine_kernel(const uint16_t* __restrict__ y, const int32_t* __restrict__ pos,
                               const float* __restrict__ w, int64_t k, int64_t D, uint16_t* __restrict__ out) {
    const int64_t t = blockIdx.x;
    for (int64_t c = threadIdx.x * 8; c < D; c += blockDim.x * 8) {
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int64_t j = 0; j < k; ++j) {
            const int32_t p = pos[t * k + j];
            if (p < 0) continue;                           // entry left out by the routing
            const float wj = w ? w[t * k + j] : 1.0f;
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(y + (int64_t)p * D + c));
            const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc[2 * q] += wj * bf16_lo(vw[q]);
                acc[2 * q + 1] += wj * bf16_hi(vw[q]);
            }
        }
        *reinterpret_cast<uint4*>(out + t * D + c) = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                                                pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    }
}

// Blocks [0, T): token t's row of dout is read once (streaming) and written,
// scaled by w[t, j], to its k rows pos[t, j].  Blocks from T on: 32 rows of
// the buffer each, a warp per row, writing zeros to the rows with src < 0
// (expert padding and the tail past the last segment).
constexpr int kDispatchThreads = 128;

__global__ void __launch_bounds__(kDispatchThreads)
dispatch_grad_kernel(const uint16_t* __restrict__ dout, const int32_t* __restrict__ src, const int32_t* __restrict__ pos,
                     const float* __restrict__ w, int64_t T, int64_t k, int64_t M_cap, int64_t D,
                     uint16_t* __restrict__ dy) {
    __shared__ int32_t sp[32];
    __shared__ float sw[32];
    const int64_t b = blockIdx.x;
    if (b < T) {
        if (threadIdx.x < k) {
            sp[threadIdx.x] = pos[b * k + threadIdx.x];
            sw[threadIdx.x] = w ? w[b * k + threadIdx.x] : 1.0f;
        }
        __syncthreads();
        for (int64_t c = threadIdx.x * 8; c < D; c += kDispatchThreads * 8) {
            const uint4 v = __ldcs(reinterpret_cast<const uint4*>(dout + b * D + c));
            for (int64_t j = 0; j < k; ++j) {
                if (sp[j] < 0 || !mx_in_range((int64_t)sp[j] * D + c, 8, M_cap * D)) continue;   // left out
                const float wj = sw[j];
                const uint4 o = make_uint4(scaled_bf16_word(wj, v.x), scaled_bf16_word(wj, v.y),
                                           scaled_bf16_word(wj, v.z), scaled_bf16_word(wj, v.w));
                *reinterpret_cast<uint4*>(dy + (int64_t)sp[j] * D + c) = o;
            }
        }
    } else {
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        for (int i = 0; i < 8; ++i) {
            const int64_t p = (b - T) * 32 + warp * 8 + i;
            if (p >= M_cap || src[p] >= 0) continue;
            for (int64_t c = lane * 8; c < D; c += 32 * 8)
                *reinterpret_cast<uint4*>(dy + p * D + c) = make_uint4(0, 0, 0, 0);
        }
    }
}

}  // namespace

namespace {

// The routing launches (count, kAlign-padded scan, scatter, padding rows)
// after the entry point's checks.
template <int kAlign>
int route_launch(const int32_t* topk, int64_t T, int64_t k, int64_t E, int64_t M_cap, int64_t* seg_offsets,
                 int32_t* src, int32_t* pos, void* workspace, cudaStream_t stream) {
    const int64_t nchunks = (T + kChunk - 1) / kChunk;
    int32_t* hist = static_cast<int32_t*>(workspace);
    int32_t* counts = hist + nchunks * E;
    unsigned int* status = nullptr;
    if (int st = mx_status_word_address(&status)) return st;
    // Each launch reads what the previous one wrote: stop at the first failure.
    if (nchunks > 0) {
        route_count_kernel<<<(unsigned)nchunks, kChunk, E * sizeof(int32_t), stream>>>(topk, T, k, E, hist, status);
        mx_count_launch();
        if (int st = mx_launch_status()) return st;
    }
    route_scan_kernel<kAlign><<<1, 1024, (E + 1) * sizeof(int64_t), stream>>>(hist, counts, nchunks, E, seg_offsets);
    mx_count_launch();
    if (int st = mx_launch_status()) return st;
    if (nchunks > 0) {
        route_scatter_kernel<<<(unsigned)nchunks, 32, 2 * E * sizeof(uint32_t), stream>>>(topk, T, k, E, M_cap, hist,
                                                                                          src, pos);
        mx_count_launch();
        if (int st = mx_launch_status()) return st;
    }
    route_pad_kernel<<<(unsigned)(E + 1), 256, 0, stream>>>(seg_offsets, counts, E, M_cap, src);
    mx_count_launch();
    return mx_launch_status();
}

// Largest dynamic shared memory of the routing launches: the scan's
// (E + 1) int64 starts (the count needs 4E bytes, the scatter 8E).
constexpr int64_t kRouteSmemLimit = 48 * 1024;

// Arguments of a routing call apart from its workspace.
int route_check_args(const int32_t* topk, int64_t T, int64_t k, int64_t E, int64_t align, int64_t M_cap,
                     const int64_t* seg_offsets, const int32_t* src, const int32_t* pos) {
    if (((!topk || !pos) && T > 0) || !seg_offsets || !src || T < 0 || k <= 0 || k > 32 || E <= 0 || M_cap < 0 ||
        M_cap % align)
        return MX_EINVAL;
    if ((E + 1) * (int64_t)sizeof(int64_t) > kRouteSmemLimit || T >= ((int64_t)1 << 31) / k) return MX_EINVAL;
    const int64_t need_rows = (T * k + (align - 1) * E + align - 1) / align * align;
    return M_cap < need_rows ? MX_EINVAL : MX_OK;
}

int route_check(const int32_t* topk, int64_t T, int64_t k, int64_t E, int64_t align, int64_t M_cap,
                const int64_t* seg_offsets, const int32_t* src, const int32_t* pos, const void* workspace,
                size_t workspace_bytes) {
    if (int st = route_check_args(topk, T, k, E, align, M_cap, seg_offsets, src, pos)) return st;
    if (!workspace || workspace_bytes < mx_route_workspace_bytes(T, E)) return MX_EINVAL;
    return MX_OK;
}

}  // namespace

extern "C" int moe_route(const int32_t* topk, int64_t T, int64_t k, int64_t E, int64_t M_cap, int64_t* seg_offsets,
                         int32_t* src, int32_t* pos, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    MX_NVTX_RANGE("moe_route");
    if (int st = route_check(topk, T, k, E, 128, M_cap, seg_offsets, src, pos, workspace, workspace_bytes)) return st;
    if (int st = mx_check_device()) return st;
    return route_launch<128>(topk, T, k, E, M_cap, seg_offsets, src, pos, workspace, stream);
}

extern "C" int moe_route_aligned(const int32_t* topk, int64_t T, int64_t k, int64_t E, int64_t align, int64_t M_cap,
                                 int64_t* seg_offsets, int32_t* src, int32_t* pos, void* workspace,
                                 size_t workspace_bytes, cudaStream_t stream) {
    MX_NVTX_RANGE("moe_route_aligned");
    if (align != 128 && align != 256) return MX_EINVAL;
    if (int st = route_check(topk, T, k, E, align, M_cap, seg_offsets, src, pos, workspace, workspace_bytes))
        return st;
    if (int st = mx_check_device()) return st;
    return align == 128 ? route_launch<128>(topk, T, k, E, M_cap, seg_offsets, src, pos, workspace, stream)
                        : route_launch<256>(topk, T, k, E, M_cap, seg_offsets, src, pos, workspace, stream);
}

extern "C" int nvfp4_gather_rows(const uint8_t* codes, const uint8_t* sf, const float* outer, const int32_t* src,
                                 int64_t k, int64_t M_cap, int64_t cols, uint8_t* out_codes, uint8_t* out_sf,
                                 float* out_outer, cudaStream_t stream) {
    MX_NVTX_RANGE("nvfp4_gather_rows");
    if (((!codes || !sf || !outer || !src || !out_codes || !out_sf || !out_outer) && M_cap > 0) || k <= 0 || M_cap < 0 ||
        M_cap % 128 || cols <= 0 || cols % 64 || !mx_aligned(codes, 16) || !mx_aligned(out_codes, 16) ||
        !mx_aligned(sf, 4) || !mx_aligned(out_sf, 4))
        return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (M_cap == 0) return MX_OK;
    gather_rows_kernel<<<(unsigned)((M_cap + 7) / 8), 256, 0, stream>>>(codes, sf, outer, src, k, M_cap, cols,
                                                                       out_codes, out_sf, out_outer);
    mx_count_launch();
    return mx_launch_status();
}

extern "C" int swiglu_fwd(const void* h, int64_t rows, int64_t F, int gated, const int64_t* rows_valid, void* a,
                          cudaStream_t stream) {
    MX_NVTX_RANGE("swiglu_fwd");
    if (!h || !a || rows < 0 || F <= 0 || F % 8 || !mx_aligned(h, 16) || !mx_aligned(a, 16)) return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    const int64_t n = rows * (F / 8);
    if (n == 0) return MX_OK;
    swiglu_fwd_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(static_cast<const uint16_t*>(h), rows, F,
                                                                        gated, rows_valid, static_cast<uint16_t*>(a));
    mx_count_launch();
    return mx_launch_status();
}

extern "C" int swiglu_bwd(const void* h, const void* da, int64_t rows, int64_t F, int gated, const int64_t* rows_valid,
                          void* dh, cudaStream_t stream) {
    MX_NVTX_RANGE("swiglu_bwd");
    if (!h || !da || !dh || rows < 0 || F <= 0 || F % 8 || !mx_aligned(h, 16) || !mx_aligned(da, 16) ||
        !mx_aligned(dh, 16))
        return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    const int64_t n = rows * (F / 8);
    if (n == 0) return MX_OK;
    swiglu_bwd_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(
        static_cast<const uint16_t*>(h), static_cast<const uint16_t*>(da), rows, F, gated, rows_valid,
        static_cast<uint16_t*>(dh));
    mx_count_launch();
    return mx_launch_status();
}

extern "C" int moe_combine(const void* y, const int32_t* pos, const float* w, int64_t T, int64_t k, int64_t D,
                           void* out, cudaStream_t stream) {
    MX_NVTX_RANGE("moe_combine");
    if (!y || !pos || !out || T < 0 || k <= 0 || D <= 0 || D % 8 || !mx_aligned(y, 16) || !mx_aligned(out, 16))
        return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (T == 0) return MX_OK;
    combine_kernel<<<(unsigned)T, 128, 0, stream>>>(static_cast<const uint16_t*>(y), pos, w, k, D,
                                                    static_cast<uint16_t*>(out));
    mx_count_launch();
    return mx_launch_status();
}

extern "C" int moe_dispatch_grad(const void* dout, const int32_t* src, const int32_t* pos, const float* w, int64_t T,
                                 int64_t k, int64_t M_cap, int64_t D, void* dy, cudaStream_t stream) {
    MX_NVTX_RANGE("moe_dispatch_grad");
    if (!dout || !src || !pos || !dy || T < 0 || k <= 0 || k > 32 || M_cap < 0 || D <= 0 || D % 8 ||
        !mx_aligned(dout, 16) || !mx_aligned(dy, 16))
        return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (M_cap == 0) return MX_OK;
    const int64_t blocks = T + (M_cap + 31) / 32;
    dispatch_grad_kernel<<<(unsigned)blocks, kDispatchThreads, 0, stream>>>(
        static_cast<const uint16_t*>(dout), src, pos, w, T, k, M_cap, D, static_cast<uint16_t*>(dy));
    mx_count_launch();
    return mx_launch_status();
}

// ===========================================================================
// moe_permute_row_groups -- moves whole 128-row groups of an expert-major
// buffer (the unit every expert segment is padded to) from one order into
// another: the reordering of the expert-parallel exchange, where rows arrive
// grouped by source rank and the expert GEMMs want them grouped by expert.
// ===========================================================================
namespace {

constexpr int kPermuteThreads = 256;

// Output group g = input group group_src[g] (group_vec 16-byte vectors each),
// or zeros where group_src[g] < 0; an index past the input is written as zeros
// and flags the device status word.
__global__ void __launch_bounds__(kPermuteThreads)
permute_row_groups_kernel(const uint4* __restrict__ in, int64_t ngroups_in, uint4* __restrict__ out,
                          int64_t ngroups_out, int64_t group_vec, const int32_t* __restrict__ group_src,
                          unsigned int* __restrict__ status) {
    const int64_t total = ngroups_out * group_vec;
    for (int64_t v = (int64_t)blockIdx.x * kPermuteThreads + threadIdx.x; v < total;
         v += (int64_t)gridDim.x * kPermuteThreads) {
        const int64_t g = v / group_vec, i = v - g * group_vec;
        const int32_t sg = __ldg(group_src + g);
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (sg >= 0 && sg < ngroups_in) val = __ldcs(in + sg * group_vec + i);
        else if (sg >= 0 && i == 0) atomicOr(status, kStatusBadRoute);
        out[v] = val;
    }
}

}  // namespace

extern "C" int moe_permute_row_groups(const void* in, int64_t ngroups_in, void* out, int64_t ngroups_out,
                                      int64_t group_bytes, const int32_t* group_src, cudaStream_t stream) {
    MX_NVTX_RANGE("moe_permute_row_groups");
    if (((!out || !group_src) && ngroups_out > 0) || (!in && ngroups_in > 0) || ngroups_in < 0 || ngroups_out < 0 ||
        group_bytes <= 0 || group_bytes % 16 || !mx_aligned(in, 16) || !mx_aligned(out, 16))
        return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (ngroups_out == 0) return MX_OK;
    unsigned int* status = nullptr;
    if (int st = mx_status_word_address(&status)) return st;
    const int64_t total = ngroups_out * (group_bytes / 16);
    const int64_t blocks = std::min<int64_t>((total + kPermuteThreads - 1) / kPermuteThreads, 148 * 16);
    permute_row_groups_kernel<<<(unsigned)blocks, kPermuteThreads, 0, stream>>>(
        static_cast<const uint4*>(in), ngroups_in, static_cast<uint4*>(out), ngroups_out, group_bytes / 16, group_src,
        status);
    mx_count_launch();
    return mx_launch_status();
}

// ===========================================================================
// moe_route_static -- moe_route for callers that cannot allocate device memory
// ===========================================================================
// Some callers cannot hand this library a scratch buffer: code running inside
// a custom allocator or memory-pool callback, or an embedding runtime that owns
// every device allocation and forbids new ones.  For them the routing scratch
// (per-chunk expert histograms and per-expert counts) lives in this fixed
// array, part of the library's device image: every GPU that loads the library
// holds these bytes until the process exits.
//
// Every word of the scratch that a call reads is written earlier in the same
// call, so nothing has to be cleared between calls.  Calls share the array:
// two calls that may run at the same time on the GPU (different streams, or
// different host threads, without ordering between them) race on it and give
// undefined results.
namespace {

constexpr size_t kRouteStaticScratchBytes = size_t(1) << 20;   // 1 MiB
static __device__ __align__(256) int32_t g_route_scratch[kRouteStaticScratchBytes / sizeof(int32_t)];

std::mutex g_route_scratch_mutex;
void* g_route_scratch_ptr[64] = {nullptr};

// Device address of the scratch array on the current device, looked up once
// per device (the array's host-side name is not a device address).
int route_scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return mx_set_cuda_error(e);
    if (dev < 0 || dev >= 64) return MX_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_route_scratch_mutex);
    if (!g_route_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess || !p) return mx_set_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
        g_route_scratch_ptr[dev] = p;
    }
    *out = g_route_scratch_ptr[dev];
    return MX_OK;
}

}  // namespace

extern "C" int moe_route_static(const int32_t* topk, int64_t T, int64_t k, int64_t E, int64_t M_cap,
                                int64_t* seg_offsets, int32_t* src, int32_t* pos, cudaStream_t stream) {
    MX_NVTX_RANGE("moe_route_static");
    if (int st = route_check_args(topk, T, k, E, 128, M_cap, seg_offsets, src, pos)) return st;
    if (mx_route_workspace_bytes(T, E) > kRouteStaticScratchBytes) return MX_EINVAL;   // beyond the fixed scratch
    if (int st = mx_check_device()) return st;
    void* scratch = nullptr;
    if (int st = route_scratch_address(&scratch)) return st;
    return moe_route(topk, T, k, E, M_cap, seg_offsets, src, pos, scratch, kRouteStaticScratchBytes, stream);
}

MX_BOUNDS_READER(mx_bounds_word_glue)
