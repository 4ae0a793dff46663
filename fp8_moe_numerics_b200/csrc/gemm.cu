// gemm.cu -- grouped expert GEMMs on 5th-generation tensor cores (sm_100a).
//
// [ai-primer] "Inkling 2 Small uses four-bit training...", §NVFP4 forward,
// MXFP8 backward: forward expert matmuls run in NVFP4 through a dedicated
// kernel; gradients use MXFP8 matmuls (§Stochastic rounding across
// transposes).  One persistent, warp-specialised kernel template serves both:
//
//   warp 0      TMA producer: operand tiles by cp.async.bulk.tensor (128-byte
//               swizzle) into a ring of 4 shared-memory stages (mbarriers)
//   warp 1      MMA issuer: allocates TMEM, issues block-scaled tcgen05.mma
//               (kind::mxf4nvf4 block16 for NVFP4, kind::mxf8f6f4 block32 for
//               MXFP8), commits stage release / accumulator-ready
//   warps 4-7   scale loaders: each stage's scale atoms from global memory
//               into a ring of 4 TMEM scale regions with tcgen05.st (measured
//               on B200: tcgen05.cp of scales stalls the MMA pipe ~24 cycles
//               per atom, tcgen05.st from registers runs beside it)
//   warps 8-15  epilogue: tcgen05.ld of the fp32 accumulator into registers,
//               early accumulator release, outer scales (NVFP4), conversion,
//               128-bit stores overlapping the next tile's main loop
//
// Tile: 128 rows (MMA M) x kBN columns (MMA N), 128 bytes of K per stage
// (256 FP4 or 128 FP8 values = 4 MMAs of 32 bytes each).  Every mbarrier wait
// is bounded: on expiry the kernel records MX_ETIMEOUT in a device status
// word, stops issuing work, drains its own copies and frees its TMEM.
#include "mx_common.cuh"

#include <cuda.h>

#include <algorithm>
#include <cstring>
#include <mutex>

__device__ unsigned int g_mx_status_word = 0;

namespace {

constexpr int kKindNVFP4 = 0, kKindMXFP8 = 1;
constexpr int kModeRows = 0, kModeWgrad = 1;
constexpr int kBM = 128;
constexpr int kStageBytesK = 128;       // bytes of K per stage (one 128B swizzle atom)
constexpr int kThreads = 512;           // 16 warps: producer, MMA, 2 idle, 4 scale loaders, 8 epilogue
constexpr int kTmemCols = 512;
constexpr unsigned long long kWaitLimitNs = 2ull * 1000ull * 1000ull * 1000ull;    // 2 s

struct GemmArgs {
    const uint8_t* sfa;       // A scale atoms (MMA layout)
    const uint8_t* sfb;       // B scale atoms (MMA layout)
    const float* a_outer;     // NVFP4: per-row outer scale of A
    const float* b_outer;     // NVFP4: per-expert outer scale of B
    const int64_t* seg;       // [E+1]
    void* out;
    int64_t E, M_cap, N, K;   // problem sizes as in the C ABI
    int64_t sfa_groups;       // scale-column groups (of 4) per 128-row group of A
    int64_t sfb_groups;       // same for B
    int64_t ldo;              // output row stride (elements)
};

// ---------------------------------------------------------------------------
// PTX wrappers
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

// Bounded wait: false (and the abort flag / status word set) on expiry or when
// another role of this CTA has already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicOr(&g_mx_status_word, 1u);
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];"
                 :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(smem_u32(bar)) : "memory");
}

// Shared-memory matrix descriptor (tcgen05): start address >> 4 in bits
// [0,14), leading byte offset >> 4 in [16,30), stride byte offset >> 4 in
// [32,46), descriptor version 1 in [46,48), layout type in [61,64)
// (0 = no swizzle, 2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3fffu);
    d |= (uint64_t)((lbo >> 4) & 0x3fffu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3fffu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)(layout & 7u) << 61;
    return d;
}

// K-major operand, 128-byte swizzle: 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t operand_desc(uint32_t saddr) { return smem_desc(saddr, 16, 1024, 2); }
// Instruction descriptor of a block-scaled MMA with M = 128, N = n, K-major
// A and B: formats in bits [7,10) and [10,13), N>>3 in [17,23), scale format
// in bit 23 (0 = UE4M3, 1 = UE8M0), M>>4 in [24,29), scale-factor byte ids of
// A in [29,31) and of B in [4,6).
__device__ __forceinline__ uint32_t idesc_block_scaled(uint32_t fmt, uint32_t scale_fmt, int n, uint32_t sfa_id,
                                                       uint32_t sfb_id) {
    return (sfb_id << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(n >> 3) << 17) | (scale_fmt << 23) |
           ((uint32_t)(kBM >> 4) << 24) | (sfa_id << 29);
}

template <int kKind>
__device__ __forceinline__ void mma_block_scaled(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    if (kKind == kKindNVFP4) {
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "setp.ne.b32 p, %4, 0;\n\t"
                     "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
                     :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
                     : "memory");
    } else {
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "setp.ne.b32 p, %4, 0;\n\t"
                     "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
                     :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
                     : "memory");
    }
}

// 32 columns of fp32 for this thread's TMEM lane, waited for inside the asm.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, float* v) {
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
                   "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
                   "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr) : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// ---------------------------------------------------------------------------
// Tile scheduling shared by all roles
// ---------------------------------------------------------------------------
struct Tile {
    int64_t e;          // expert
    int64_t row0;       // first output row (ROWS: token row; WGRAD: row of out viewed as [E*N, K])
    int64_t col0;       // first output column
    int64_t a_y;        // A tile row coordinate
    int64_t b_y;        // B tile row coordinate
    int64_t k0_bytes;   // first K byte of the contraction (A and B x coordinate base)
    int64_t b_x0;       // B x coordinate base (DGRAD: e*K)
    int64_t k_tiles;    // stages of 128 K-bytes
    int64_t sfa_atom0;  // first SFA atom of the tile's first stage
    int64_t sfb_atom0;  // first SFB atom (row group 0)
};

__device__ __forceinline__ int64_t find_expert(const int64_t* seg, int64_t E, int64_t row) {
    int64_t lo = 0, hi = E;                      // seg[lo] <= row < seg[hi]
    while (hi - lo > 1) {
        const int64_t mid = (lo + hi) >> 1;
        if (__ldg(seg + mid) <= row) lo = mid; else hi = mid;
    }
    return lo;
}

template <int kKind, int kMode, int kBN>
__device__ __forceinline__ int64_t total_tiles(const GemmArgs& p) {
    if (kMode == kModeRows) return (__ldg(p.seg + p.E) / kBM) * (p.N / kBN);
    return p.E * (p.N / kBM) * (p.K / kBN);
}

template <int kKind, int kMode, int kBN>
__device__ __forceinline__ Tile make_tile(const GemmArgs& p, int64_t idx) {
    Tile t;
    const int64_t spg = kKind == kKindNVFP4 ? 4 : 1;   // scale atoms per stage per 128-row group
    if (kMode == kModeRows) {
        const int64_t n_tiles = p.N / kBN;
        const int64_t mt = idx / n_tiles, nt = idx % n_tiles;
        t.row0 = mt * kBM;
        t.col0 = nt * kBN;
        t.e = find_expert(p.seg, p.E, t.row0);
        const int64_t kbytes = kKind == kKindNVFP4 ? p.K / 2 : p.K;
        t.k_tiles = kbytes / kStageBytesK;
        t.k0_bytes = 0;
        t.a_y = t.row0;
        t.sfa_atom0 = mt * p.sfa_groups;
        if (kKind == kKindNVFP4) {                      // B = weight stack [E*N, K]
            t.b_y = t.e * p.N + t.col0;
            t.b_x0 = 0;
            t.sfb_atom0 = (t.b_y / kBM) * p.sfb_groups;
        } else {                                        // DGRAD: B = [N, E*K]
            t.b_y = t.col0;
            t.b_x0 = t.e * p.K;
            t.sfb_atom0 = (t.b_y / kBM) * p.sfb_groups + t.e * p.K / 128;
        }
        (void)spg;
    } else {                                            // WGRAD: out [E, N, K]
        const int64_t nt_n = p.N / kBM, nt_k = p.K / kBN;
        t.e = idx / (nt_n * nt_k);
        const int64_t rem = idx % (nt_n * nt_k);
        const int64_t tn = rem / nt_k, tk = rem % nt_k;
        const int64_t s0 = __ldg(p.seg + t.e), s1 = __ldg(p.seg + t.e + 1);
        t.row0 = t.e * p.N + tn * kBM;
        t.col0 = tk * kBN;
        t.k_tiles = (s1 - s0) / kStageBytesK;
        t.k0_bytes = s0;
        t.b_x0 = 0;
        t.a_y = tn * kBM;
        t.b_y = tk * kBN;
        t.sfa_atom0 = t.a_y / kBM * p.sfa_groups + s0 / 128;
        t.sfb_atom0 = t.b_y / kBM * p.sfb_groups + s0 / 128;
    }
    return t;
}

template <int kKind, int kBN>
struct Smem {
    static constexpr int kA = kBM * kStageBytesK;                       // 16 KB
    static constexpr int kB = kBN * kStageBytesK;                       // 16 / 32 KB
    static constexpr int kAtomsA = kKind == kKindNVFP4 ? 4 : 1;         // scale atoms per stage, 128-row group
    static constexpr int kAtomsB = kAtomsA * (kBN / 128);
    static constexpr int kSfa = kAtomsA * 512;
    static constexpr int kSfb = kAtomsB * 512;
    static constexpr int kStageTx = kA + kB + kSfa + kSfb;             // bytes the TMA engine delivers per stage
    static constexpr int kStage = (kStageTx + 1023) / 1024 * 1024;      // stage stride: keeps every SW128 tile 1024-aligned
    static constexpr int kStaging = 8 * 4096;                           // epilogue: one 64x32 bf16 box per warp
    static constexpr int kStages = (kStage * 6 + kStaging <= 220 * 1024) ? 6
                                 : (kStage * 4 + kStaging <= 220 * 1024) ? 4 : 3;
    static constexpr int kStagingOff = kStages * kStage;
    static_assert(kStage % 1024 == 0 && kStagingOff % 1024 == 0, "128-byte swizzle needs 1024-byte aligned tiles");
    static constexpr int kBarOff = kStagingOff + kStaging;
    static constexpr int kBytes = kBarOff + 512 + 1024;                  // + barriers + alignment slack
    // TMEM: accumulator buffer(s), then one scale region per stage
    static constexpr int kSfaCols = 4 * kAtomsA;
    static constexpr int kSfbCols = 4 * kAtomsB;
    static constexpr int kSfRegion = kSfaCols + kSfbCols;
    static constexpr int kAccBufs = (2 * kBN + kStages * kSfRegion <= kTmemCols) ? 2 : 1;
    static constexpr int kSfCol = kAccBufs * kBN;
    static_assert(kSfCol + kStages * kSfRegion <= kTmemCols, "TMEM budget");
};

__device__ __forceinline__ void tmem_st_32x32b_x4(uint32_t taddr, const uint4& v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};"
                 :: "r"(taddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

template <int kKind, int kMode, int kBN, bool kOutBF16>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmOut, const GemmArgs p) {
    using L = Smem<kKind, kBN>;
    constexpr int kStages = L::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);   // operands landed
    uint64_t* sf_full = full + kStages;                                 // scales written to TMEM
    uint64_t* empty = sf_full + kStages;                                // stage consumed by the MMAs
    uint64_t* acc_full = empty + kStages;        // [2]: accumulator buffer b ready
    uint64_t* acc_empty = acc_full + 2;          // [2]: accumulator buffer b drained
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t total = total_tiles<kKind, kMode, kBN>(p);
    if ((int64_t)blockIdx.x >= total) return;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&sf_full[s], 4);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 8); }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
        if (kOutBF16) asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(&tmOut)) : "memory");
    }
    if (warp == 1) tmem_alloc(tmem_base_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (A, B)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_phase[kStages];
            bool issued[kStages];
            for (int s = 0; s < kStages; ++s) { issued[s] = false; issued_phase[s] = 0; }
            bool ok = true;
            for (int64_t idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
                const Tile t = make_tile<kKind, kMode, kBN>(p, idx);
                for (int64_t kt = 0; kt < t.k_tiles; ++kt) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    uint8_t* sa = smem + stage * L::kStage;
                    uint8_t* sb = sa + L::kA;
                    uint8_t* ssfa = sb + L::kB;
                    uint8_t* ssfb = ssfa + L::kSfa;
                    mbar_expect_tx(&full[stage], (uint32_t)L::kStageTx);
                    const int kx = (int)(t.k0_bytes + kt * kStageBytesK);
                    tma_load_2d(sa, &tmA, &full[stage], kx, (int)t.a_y);
                    tma_load_2d(sb, &tmB, &full[stage], (int)t.b_x0 + kx, (int)t.b_y);
                    bulk_load(ssfa, p.sfa + (t.sfa_atom0 + kt * L::kAtomsA) * 512, L::kSfa, &full[stage]);
#pragma unroll
                    for (int h = 0; h < kBN / 128; ++h)
                        bulk_load(ssfb + h * L::kAtomsA * 512, p.sfb + (t.sfb_atom0 + h * p.sfb_groups + kt * L::kAtomsA) * 512,
                                  L::kAtomsA * 512, &full[stage]);
                    issued[stage] = true;
                    issued_phase[stage] = phase;
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
            }
            // drain: every issued copy has landed before shared memory is released
            for (int s = 0; s < kStages; ++s)
                if (issued[s]) {
                    const unsigned long long t0 = globaltimer();
                    while (!mbar_try_wait(&full[s], issued_phase[s]) && globaltimer() - t0 < kWaitLimitNs) {}
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kFmt = kKind == kKindNVFP4 ? 1u : 0u;      // E2M1 / E4M3
            constexpr uint32_t kScaleFmt = kKind == kKindNVFP4 ? 0u : 1u; // UE4M3 / UE8M0
            int stage = 0, buf = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int64_t idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
                const Tile t = make_tile<kKind, kMode, kBN>(p, idx);
                if (!mbar_wait(&acc_empty[buf], acc_phase ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)(buf * kBN);
                for (int64_t kt = 0; kt < t.k_tiles; ++kt) {
                    if (!mbar_wait(&full[stage], phase, abort_flag) || !mbar_wait(&sf_full[stage], phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint8_t* sa = smem + stage * L::kStage;
                    const uint8_t* sb = sa + L::kA;
                    const uint32_t sfa = tmem + L::kSfCol + stage * L::kSfRegion;
                    const uint32_t sfb = sfa + L::kSfaCols;
                    const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sb);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t sfa_t, sfb_t, id;
                        if (kKind == kKindNVFP4) {
                            sfa_t = sfa + 4 * j;
                            sfb_t = sfb + (kBN / 32) * j;
                            id = idesc_block_scaled(kFmt, kScaleFmt, kBN, 0, 0);
                        } else {
                            sfa_t = sfa | ((uint32_t)j << 30);
                            sfb_t = sfb | ((uint32_t)j << 30);
                            id = idesc_block_scaled(kFmt, kScaleFmt, kBN, (uint32_t)j, (uint32_t)j);
                        }
                        mma_block_scaled<kKind>(acc, operand_desc(a0 + 32 * j), operand_desc(b0 + 32 * j), id,
                                                sfa_t, sfb_t, (kt > 0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&acc_full[buf]);
                if (++buf == L::kAccBufs) { buf = 0; acc_phase ^= 1u; }
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ scale movers
        // The stage's scale atoms arrive in shared memory with the operands.
        // Warp q copies them into its own TMEM lane quarter with tcgen05.st:
        // lane l of an atom holds 16 bytes = 4 columns (rows l, l+32, l+64,
        // l+96 of the 128-row group), the replicated layout the block-scaled
        // MMA reads in every quarter.  tcgen05.st from registers does not
        // occupy the tensor pipe (tcgen05.cp would, ~24 cycles per atom).
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int64_t idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
            const Tile t = make_tile<kKind, kMode, kBN>(p, idx);
            for (int64_t kt = 0; kt < t.k_tiles; ++kt) {
                if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                const uint8_t* ssfa = smem + stage * L::kStage + L::kA + L::kB;
                const uint8_t* ssfb = ssfa + L::kSfa;
                uint4 va[L::kAtomsA], vb[L::kAtomsB];
#pragma unroll
                for (int j = 0; j < L::kAtomsA; ++j) va[j] = reinterpret_cast<const uint4*>(ssfa + j * 512)[lane];
#pragma unroll
                for (int j = 0; j < L::kAtomsB; ++j) vb[j] = reinterpret_cast<const uint4*>(ssfb + j * 512)[lane];
                tc_fence_after();
                const uint32_t sfa = tmem + lane_base + L::kSfCol + stage * L::kSfRegion;
                const uint32_t sfb = sfa + L::kSfaCols;
#pragma unroll
                for (int j = 0; j < L::kAtomsA; ++j) tmem_st_32x32b_x4(sfa + 4 * j, va[j]);
#pragma unroll
                for (int h = 0; h < kBN / 128; ++h)
#pragma unroll
                    for (int j = 0; j < L::kAtomsA; ++j)
                        tmem_st_32x32b_x4(sfb + (kBN / 32) * j + 4 * h, vb[h * L::kAtomsA + j]);
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_full[stage]);
                if (++stage == kStages) { stage = 0; phase ^= 1u; }
            }
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ epilogue
        // Eight warps: warp w reads TMEM lane quarter w%4 (the hardware lets a
        // warp touch only its own 32 lanes) and column half (w-8)/4.  bf16
        // output: each 32-column chunk is scaled and packed as it arrives, the
        // accumulator is released after the last chunk, and the stores overlap
        // the next tile's main loop.  fp32 output stores chunk by chunk and
        // releases the accumulator afterwards.
        constexpr int kCols = kBN / 2;
        const int q = warp & 3;
        const int half = (warp - 8) >> 2;
        const int r = q * 32 + lane;
        const int cb = half * kCols;
        uint32_t acc_phase = 0;
        int buf = 0;
        for (int64_t idx = blockIdx.x; idx < total; idx += gridDim.x) {
            const Tile t = make_tile<kKind, kMode, kBN>(p, idx);
            if (!mbar_wait(&acc_full[buf], acc_phase, abort_flag)) break;
            tc_fence_after();
            float scale = 1.0f;
            if (kKind == kKindNVFP4) scale = __ldg(p.a_outer + t.row0 + r) * __ldg(p.b_outer + t.e);
            const int64_t orow = t.row0 + r;
            const uint32_t taddr = tmem + (uint32_t)(buf * kBN) + ((uint32_t)(q * 32) << 16) + cb;
            if (kOutBF16) {
                // 32 rows x kCols bf16 per warp, written by TMA tensor stores of
                // 64-column boxes staged in this warp's 4 KB of shared memory
                // (128-byte swizzle: 16-byte chunk c of row r at c ^ (r % 8)).
                uint8_t* stg = smem + L::kStagingOff + (warp - 8) * 4096;
                const uint32_t srow = smem_u32(stg) + (uint32_t)lane * 128u;
                const int ox = (int)(t.col0 + cb), oy = (int)(t.row0 + q * 32);
                if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");   // previous tile's box
                __syncwarp();
                uint32_t pk[kCols > 64 ? kCols / 2 - 32 : 1];  // columns 64.. held until the staging buffer frees
#pragma unroll
                for (int c = 0; c < kCols; c += 32) {
                    float v[32];
                    if (t.k_tiles > 0) tmem_ld_32x32b_x32(taddr + c, v);
                    else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = 0.0f;
                    }
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i] * scale, v[2 * i + 1] * scale);
                        w[i] = *reinterpret_cast<uint32_t*>(&b);
                    }
                    if (c < 64) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint32_t chunk = (uint32_t)((c / 8 + i) ^ (lane & 7));
                            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                         :: "r"(srow + chunk * 16u), "r"(w[4 * i]), "r"(w[4 * i + 1]), "r"(w[4 * i + 2]),
                                            "r"(w[4 * i + 3]) : "memory");
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) pk[(c - 64) / 2 + i] = w[i];
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[buf]);
                // box 0 (columns 0..63 of this warp's block)
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) {
                    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
                                 :: "l"(reinterpret_cast<uint64_t>(&tmOut)), "r"(ox), "r"(oy), "r"(smem_u32(stg)) : "memory");
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                }
                __syncwarp();
                if (kCols > 64) {
                    // box 1 (columns 64..127) from registers
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t chunk = (uint32_t)(i ^ (lane & 7));
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                     :: "r"(srow + chunk * 16u), "r"(pk[4 * i]), "r"(pk[4 * i + 1]), "r"(pk[4 * i + 2]),
                                        "r"(pk[4 * i + 3]) : "memory");
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) {
                        asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
                                     :: "l"(reinterpret_cast<uint64_t>(&tmOut)), "r"(ox + 64), "r"(oy), "r"(smem_u32(stg)) : "memory");
                        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                    }
                }
            } else {
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow * p.ldo + t.col0 + cb);
#pragma unroll 1
                for (int c = 0; c < kCols; c += 32) {
                    float v[32];
                    if (t.k_tiles > 0) tmem_ld_32x32b_x32(taddr + c, v);
                    else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = 0.0f;
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[c / 4 + i] = make_float4(v[4 * i] * scale, v[4 * i + 1] * scale, v[4 * i + 2] * scale,
                                                     v[4 * i + 3] * scale);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[buf]);
            }
            if (++buf == L::kAccBufs) { buf = 0; acc_phase ^= 1u; }
        }
        if (kOutBF16 && lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 2-D uint8 tensor [rows, inner] (row stride = inner bytes), box [box_rows, 128 B], 128-byte swizzle.
int make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t inner, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return MX_EUNSUPPORTED;
    const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)inner};
    const cuuint32_t box[2] = {(cuuint32_t)kStageBytesK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MX_OK : MX_EINVAL;
}

// bf16 output [rows, cols] (row stride cols), box 64 x 32, 128-byte swizzle.
int make_out_map(CUtensorMap* m, void* base, int64_t rows, int64_t cols) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return MX_EUNSUPPORTED;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64, 32};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MX_OK : MX_EINVAL;
}

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

template <int kKind, int kMode, int kBN, bool kOutBF16>
int launch(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mo, const GemmArgs& args, int64_t max_tiles,
           cudaStream_t stream) {
    using L = Smem<kKind, kBN>;
    auto kern = grouped_gemm_kernel<kKind, kMode, kBN, kOutBF16>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes) != cudaSuccess)
        return mx_launch_status();
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(max_tiles, num_sms()));
    kern<<<(unsigned)grid, kThreads, L::kBytes, stream>>>(ma, mb, mo, args);
    return mx_launch_status();
}

// Tile width: 256 columns (one accumulator) whenever the output width allows
// it; 128 columns (two accumulators) otherwise.  Measured on B200, the wide
// tile is faster even for short K loops: it halves the A traffic per flop.
template <int kKind, int kMode>
int dispatch(int64_t out_cols, int64_t out_rows, int64_t k_stages, int out_dtype, const CUtensorMap& ma256,
             const CUtensorMap& mb256, const CUtensorMap& ma128, const CUtensorMap& mb128, const GemmArgs& args,
             int64_t tiles128, cudaStream_t stream) {
    CUtensorMap mo;
    memset(&mo, 0, sizeof(mo));
    if (out_dtype == MX_OUT_BF16)
        if (int st = make_out_map(&mo, args.out, out_rows, out_cols)) return st;
    (void)k_stages;
    const bool wide = out_cols % 256 == 0;
    const bool bf16 = out_dtype == MX_OUT_BF16;
    if (wide)
        return bf16 ? launch<kKind, kMode, 256, true>(ma256, mb256, mo, args, tiles128 / 2, stream)
                    : launch<kKind, kMode, 256, false>(ma256, mb256, mo, args, tiles128 / 2, stream);
    return bf16 ? launch<kKind, kMode, 128, true>(ma128, mb128, mo, args, tiles128, stream)
                : launch<kKind, kMode, 128, false>(ma128, mb128, mo, args, tiles128, stream);
}

}  // namespace

extern "C" int mx_sync_status(cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return mx_set_cuda_error(e);
    unsigned int word = 0, zero = 0;
    if ((e = cudaMemcpyFromSymbol(&word, g_mx_status_word, sizeof(word))) != cudaSuccess) return mx_set_cuda_error(e);
    if (word && (e = cudaMemcpyToSymbol(g_mx_status_word, &zero, sizeof(zero))) != cudaSuccess)
        return mx_set_cuda_error(e);
    return word ? MX_ETIMEOUT : MX_OK;
}

extern "C" int grouped_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_outer,
                                  const uint8_t* b_codes, const uint8_t* b_sf, const float* b_outer,
                                  const int64_t* seg_offsets, int64_t E, int64_t M_cap, int64_t N, int64_t K,
                                  void* out, int out_dtype, cudaStream_t stream) {
    if (!a_codes || !a_sf || !a_outer || !b_codes || !b_sf || !b_outer || !seg_offsets || !out || E < 1 ||
        M_cap < 0 || M_cap % 128 || N <= 0 || N % 128 || K <= 0 || K % 256)
        return MX_EINVAL;
    if (out_dtype != MX_OUT_F32 && out_dtype != MX_OUT_BF16) return MX_EINVAL;
    if (!mx_aligned(a_codes, 16) || !mx_aligned(b_codes, 16) || !mx_aligned(a_sf, 16) || !mx_aligned(b_sf, 16) ||
        !mx_aligned(out, 16))
        return MX_EINVAL;
    if (M_cap >= (int64_t)1 << 31 || E * N >= (int64_t)1 << 31 || K / 2 >= (int64_t)1 << 31) return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (M_cap == 0) return MX_OK;
    CUtensorMap ma, mb, mb2;
    if (int st = make_map(&ma, a_codes, M_cap, K / 2, kBM)) return st;
    if (int st = make_map(&mb, b_codes, E * N, K / 2, 128)) return st;
    if (N % 256 == 0)
        if (int st = make_map(&mb2, b_codes, E * N, K / 2, 256)) return st;
    GemmArgs a{};
    a.sfa = a_sf; a.sfb = b_sf; a.a_outer = a_outer; a.b_outer = b_outer; a.seg = seg_offsets; a.out = out;
    a.E = E; a.M_cap = M_cap; a.N = N; a.K = K;
    a.sfa_groups = K / 64; a.sfb_groups = K / 64; a.ldo = N;
    return dispatch<kKindNVFP4, kModeRows>(N, M_cap, K / 2 / kStageBytesK, out_dtype, ma, mb2, ma, mb, a,
                                           (M_cap / kBM) * (N / 128), stream);
}

extern "C" int grouped_gemm_mxfp8(int mode, const uint8_t* a_codes, const uint8_t* a_e8m0, const uint8_t* b_codes,
                                  const uint8_t* b_e8m0, const int64_t* seg_offsets, int64_t E, int64_t M_cap,
                                  int64_t N, int64_t K, void* out, int out_dtype, cudaStream_t stream) {
    if (!a_codes || !a_e8m0 || !b_codes || !b_e8m0 || !seg_offsets || !out || E < 1 || M_cap < 0 || M_cap % 128 ||
        N <= 0 || N % 128 || K <= 0 || K % 128)
        return MX_EINVAL;
    if (mode != MX_GEMM_DGRAD && mode != MX_GEMM_WGRAD) return MX_EINVAL;
    if (out_dtype != MX_OUT_F32 && out_dtype != MX_OUT_BF16) return MX_EINVAL;
    if (!mx_aligned(a_codes, 16) || !mx_aligned(b_codes, 16) || !mx_aligned(a_e8m0, 16) || !mx_aligned(b_e8m0, 16) ||
        !mx_aligned(out, 16))
        return MX_EINVAL;
    if (M_cap >= (int64_t)1 << 31 || E * K >= (int64_t)1 << 31 || N >= (int64_t)1 << 31) return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (M_cap == 0 && mode == MX_GEMM_DGRAD) return MX_OK;
    CUtensorMap ma, mb;
    GemmArgs a{};
    a.sfa = a_e8m0; a.sfb = b_e8m0; a.seg = seg_offsets; a.out = out;
    a.E = E; a.M_cap = M_cap; a.N = N; a.K = K;
    if (mode == MX_GEMM_DGRAD) {
        // A [M_cap, K], B [N, E*K]; out [M_cap, N]
        CUtensorMap mb2;
        if (int st = make_map(&ma, a_codes, M_cap, K, kBM)) return st;
        if (int st = make_map(&mb, b_codes, N, E * K, 128)) return st;
        if (N % 256 == 0)
            if (int st = make_map(&mb2, b_codes, N, E * K, 256)) return st;
        a.sfa_groups = K / 128; a.sfb_groups = E * K / 128; a.ldo = N;
        return dispatch<kKindMXFP8, kModeRows>(N, M_cap, K / kStageBytesK, out_dtype, ma, mb2, ma, mb, a,
                                               (M_cap / kBM) * (N / 128), stream);
    }
    // WGRAD: A [N, M_cap], B [K, M_cap]; out [E, N, K]
    if (M_cap == 0) return MX_EINVAL;
    CUtensorMap mb2;
    if (int st = make_map(&ma, a_codes, N, M_cap, kBM)) return st;
    if (int st = make_map(&mb, b_codes, K, M_cap, 128)) return st;
    if (K % 256 == 0)
        if (int st = make_map(&mb2, b_codes, K, M_cap, 256)) return st;
    a.sfa_groups = M_cap / 128; a.sfb_groups = M_cap / 128; a.ldo = K;
    return dispatch<kKindMXFP8, kModeWgrad>(K, E * N, 0, out_dtype, ma, mb2, ma, mb, a, E * (N / kBM) * (K / 128), stream);
}
