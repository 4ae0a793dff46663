// gemm.cu -- grouped expert GEMMs on 5th-generation tensor cores (sm_100a).
//
// [ai-primer] "Inkling 2 Small uses four-bit training...", §NVFP4 forward,
// MXFP8 backward: forward expert matmuls run in NVFP4 through a dedicated
// kernel; gradients use MXFP8 matmuls (§Stochastic rounding across
// transposes).  One persistent, warp-specialised kernel template serves both:
//
//   warp 0      TMA producer: operand tiles by cp.async.bulk.tensor (128-byte
//               swizzle) and the stage's scale atoms by cp.async.bulk into a
//               ring of 3-6 shared-memory stages (as many as fit beside the
//               epilogue staging), completion on mbarriers
//   warp 1      MMA issuer: allocates TMEM, issues block-scaled tcgen05.mma
//               (kind::mxf4nvf4 block16 for NVFP4, kind::mxf8f6f4 block32 for
//               MXFP8), commits stage release / accumulator-ready
//   warps 4-7   scale movers: each stage's scale atoms from shared memory
//               into a ring of TMEM scale regions with tcgen05.st (measured
//               on B200: tcgen05.cp of scales stalls the MMA pipe ~24 cycles
//               per atom, tcgen05.st from registers runs beside it)
//   warps 8-15  epilogue: tcgen05.ld of the fp32 accumulator into registers,
//               early release of the chunks the next tile's accumulator
//               shares, outer scales (NVFP4), conversion, 32 x 32 boxes
//               staged in shared memory and written by TMA tensor stores
//               while the next tile's main loop runs
//
// Tile: 128 rows (MMA M) x kBN columns (MMA N) per CTA, 128 bytes of K per
// stage (256 FP4 or 128 FP8 values = 4 MMAs of 32 bytes each).  Where the
// shape allows, CTA pairs (cta_group::2) compute 256 x 256 tiles, each CTA
// loading its 128 rows of A and half of B; row-mode calls add a single-CTA
// tail kernel with 128 x 256 tiles for the experts' leftover row tiles (see
// the tile scheduling below).  Every mbarrier wait is bounded: on expiry the
// kernel records MX_ETIMEOUT in a device status word, stops issuing work,
// drains its own copies and frees its TMEM.
#include "mx_common.cuh"

#include <cuda.h>

#include <algorithm>
#include <cstring>
#include <mutex>

__device__ unsigned int g_mx_status_word = 0;

namespace {

constexpr int kKindNVFP4 = 0, kKindMXFP8 = 1;
constexpr int kOutTypeF32 = 0, kOutTypeBF16 = 1, kOutTypeS2F6 = 2;   // epilogue output
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
    uint8_t* e8m0_out;        // S2F6 output: one exponent per 32 outputs of a row
    uint64_t seed, stream_id; // S2F6 output: key and stream of the rotation's signs
    int64_t sfa_atoms, sfb_atoms, a_outer_n;   // extents of the scale arrays (512-byte atoms) and of a_outer
    int64_t tail_min_items;   // ROWS, 256-wide tiles: fewest tail items that make the tail kernel pay
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
// Bounded wait: false (and the abort flag / status word set) on expiry or when
// another role of this CTA has already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit_ns) {
            *abort_flag = 1;
            atomicOr(&g_mx_status_word, kStatusTimeout);
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

// Operand tile of a CTA pair: lands in this CTA's shared memory, its bytes
// are counted on the leader CTA's mbarrier (a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];"
                 :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
                 : "memory");
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// shared::cluster address of the variable at the same offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_to_rank(const void* p, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    return a;
}

// Arrive on a barrier of another CTA of the cluster.  CTA-scope release: what
// the arrival publishes is TMEM state, already ordered by tcgen05.wait and
// tcgen05.fence; a cluster-scope release would add a memory fence per call.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" :: "r"(bar_cluster) : "memory");
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <bool kPair>
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    if (kPair) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
}

template <bool kPair>
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    if (kPair)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
    else
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive on `bar` once every MMA issued so far has completed.  A pair's
// leader signals the barrier at the same offset in both CTAs.
template <bool kPair>
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    if (kPair)
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                     :: "r"(smem_u32(bar)), "h"((uint16_t)0x3) : "memory");
    else
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
// Instruction descriptor of a block-scaled MMA with M = m, N = n, K-major
// A and B: formats in bits [7,10) and [10,13), N>>3 in [17,23), scale format
// in bit 23 (0 = UE4M3, 1 = UE8M0), M>>4 in [24,29), scale-factor byte ids of
// A in [29,31) and of B in [4,6).
__device__ __forceinline__ uint32_t idesc_block_scaled(uint32_t fmt, uint32_t scale_fmt, int m, int n, uint32_t sfa_id,
                                                       uint32_t sfb_id) {
    return (sfb_id << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(n >> 3) << 17) | (scale_fmt << 23) |
           ((uint32_t)(m >> 4) << 24) | (sfa_id << 29);
}

// One block-scaled MMA.  kPair: issued by the leader of a CTA pair, M = 256
// with 128 rows of A and half of B's rows in each CTA's shared memory, each
// CTA's accumulator and scale factors in its own TMEM.
template <int kKind, bool kPair>
__device__ __forceinline__ void mma_block_scaled(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
#define MX_MMA_ASM(GROUP, KIND)                                                                                  \
    asm volatile("{\n\t.reg .pred p;\n\t"                                                                      \
                 "setp.ne.b32 p, %4, 0;\n\t"                                                                     \
                 "tcgen05.mma.cta_group::" GROUP ".kind::" KIND " [%0], %1, %2, %3, [%5], [%6], p;\n\t}"          \
                 :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),             \
                    "r"(sfb_tmem)                                                                                 \
                 : "memory")
    if (kKind == kKindNVFP4) {
        if (kPair) MX_MMA_ASM("2", "mxf4nvf4.block_scale.block16");
        else MX_MMA_ASM("1", "mxf4nvf4.block_scale.block16");
    } else {
        if (kPair) MX_MMA_ASM("2", "mxf8f6f4.block_scale.block32");
        else MX_MMA_ASM("1", "mxf8f6f4.block_scale.block32");
    }
#undef MX_MMA_ASM
}

// Two 32-column loads in flight at once, waited for inside the same asm so no
// use of the registers can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld2_32x32b_x32(uint32_t taddr0, uint32_t taddr1, float* v0, float* v1) {
    uint32_t a[32], b[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
                 "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
                 "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]),
                   "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]),
                   "=r"(a[16]), "=r"(a[17]), "=r"(a[18]), "=r"(a[19]), "=r"(a[20]), "=r"(a[21]), "=r"(a[22]), "=r"(a[23]),
                   "=r"(a[24]), "=r"(a[25]), "=r"(a[26]), "=r"(a[27]), "=r"(a[28]), "=r"(a[29]), "=r"(a[30]), "=r"(a[31]),
                   "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]), "=r"(b[6]), "=r"(b[7]),
                   "=r"(b[8]), "=r"(b[9]), "=r"(b[10]), "=r"(b[11]), "=r"(b[12]), "=r"(b[13]), "=r"(b[14]), "=r"(b[15]),
                   "=r"(b[16]), "=r"(b[17]), "=r"(b[18]), "=r"(b[19]), "=r"(b[20]), "=r"(b[21]), "=r"(b[22]), "=r"(b[23]),
                   "=r"(b[24]), "=r"(b[25]), "=r"(b[26]), "=r"(b[27]), "=r"(b[28]), "=r"(b[29]), "=r"(b[30]), "=r"(b[31])
                 : "r"(taddr0), "r"(taddr1) : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) { v0[i] = __uint_as_float(a[i]); v1[i] = __uint_as_float(b[i]); }
}

// ---------------------------------------------------------------------------
// Tile scheduling shared by all roles
// ---------------------------------------------------------------------------
// A work item is one output tile.  Single-CTA items are 128 rows x kBN
// columns.  Pair items are 256 rows x kBN columns: CTA rank r of the pair owns
// rows [128 r, 128 r + 128) of the tile and loads half of B's kBN rows.  In
// ROWS mode with 256-wide tiles a call runs two kernels, the pair kernel and
// the tail kernel (single CTAs, 128 x 256 tiles); segments are padded to 128
// rows, not 256, so an expert with an odd tile count has one row tile left
// over after its full pairs.  That tile goes either
//  - to the tail kernel, which needs one SM and 1.5 times a pair CTA's bytes
//    per stage for it, or
//  - to a half pair in the pair kernel, whose CTA 1 recomputes CTA 0's rows
//    (valid memory, no special case in the pipeline) and stores nothing: two
//    SMs' operand feed for 128 rows, but spread over the pair kernel's
//    waves and next to the expert's other row pairs, whose weight tiles are
//    still in L2.
// Both kernels take the same decision from seg: the tail kernel gets every
// leftover tile when that makes at least tail_min_items items (measured on
// B200: a few waves, or its last partial wave, its launch and its weight
// re-reads cost more than the half pairs save), else none.  Both scan their
// per-expert item counts into a shared-memory prefix at start-up, so items
// form a dense list.  ROWS calls with 128-wide tiles walk the row tiles
// directly.
constexpr int kMaxPairExperts = 768;    // prefix capacity (shared memory)

// The single-CTA kernel with 256-wide tiles exists only as the ROWS tail kernel.
template <int kMode, int kBN, bool kPair>
constexpr bool kRowsTail = kMode == kModeRows && !kPair && kBN == 256;

struct Tile {
    bool store;         // false: CTA 1 of a half pair (recomputes CTA 0's rows)
    int64_t e;          // expert
    int64_t row0;       // first output row of this CTA (ROWS: token row; WGRAD: row of out viewed as [E*N, K])
    int64_t col0;       // first output column
    int64_t a_y;        // A tile row coordinate (this CTA's 128 rows)
    int64_t b_y;        // B tile row coordinate (this CTA's share of the kBN rows)
    int64_t k0_bytes;   // first K byte of the contraction (A and B x coordinate base)
    int64_t b_x0;       // B x coordinate base (DGRAD: e*K)
    int64_t k_tiles;    // stages of 128 K-bytes
    int64_t sfa_atom0;  // first SFA atom of the tile's first stage
    int64_t sfb_atom0;  // first SFB atom (row group 0 of the kBN columns)
};

__device__ __forceinline__ int64_t find_expert(const int64_t* seg, int64_t E, int64_t row) {
    int64_t lo = 0, hi = E;                      // seg[lo] <= row < seg[hi]
    while (hi - lo > 1) {
        const int64_t mid = (lo + hi) >> 1;
        if (__ldg(seg + mid) <= row) lo = mid; else hi = mid;
    }
    return lo;
}

template <int kMode, int kBN, bool kPair>
__device__ __forceinline__ int64_t total_tiles(const GemmArgs& p, const int32_t* pfx) {
    if (kMode == kModeRows)
        return ((kPair || kRowsTail<kMode, kBN, kPair>) ? (int64_t)pfx[p.E] : __ldg(p.seg + p.E) / kBM) * (p.N / kBN);
    return p.E * (p.N / (kPair ? 2 * kBM : kBM)) * (p.K / kBN);
}

// ROWS pair and tail kernels: pfx[e] = items of experts 0..e-1 (pfx[E] =
// all).  With the split (see above) an expert's items are its full row pairs
// (pair kernel) and its leftover row tile (tail kernel); without it, its
// row pairs including a final half pair, and nothing.  Called by the whole
// block.
template <bool kTail>
__device__ __forceinline__ void build_row_prefix(const GemmArgs& p, int32_t* pfx) {
    int64_t n_odd = 0;                          // experts with an odd tile count
    for (int64_t e0 = 0; e0 < p.E; e0 += blockDim.x) {
        const int64_t e = e0 + threadIdx.x;
        const int64_t tiles = e < p.E ? (__ldg(p.seg + e + 1) - __ldg(p.seg + e)) / kBM : 0;
        n_odd += __syncthreads_count((int)(tiles & 1));
    }
    const bool split = n_odd * (p.N / 256) >= p.tail_min_items;
    for (int64_t e = threadIdx.x; e < p.E; e += blockDim.x) {
        const int64_t tiles = (__ldg(p.seg + e + 1) - __ldg(p.seg + e)) / kBM;
        pfx[e + 1] = (int32_t)(kTail ? (split ? (tiles & 1) : 0) : (split ? tiles / 2 : (tiles + 1) / 2));
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int32_t carry = 0;
        for (int64_t b = 0; b < p.E; b += 32) {
            const int64_t e = b + lane;
            int32_t v = e < p.E ? pfx[e + 1] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            if (e < p.E) pfx[e + 1] = carry + v;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) pfx[0] = 0;
    }
    __syncthreads();
}

template <int kKind, int kMode, int kBN, bool kPair>
__device__ __forceinline__ Tile make_tile(const GemmArgs& p, int64_t idx, uint32_t rank, const int32_t* pfx) {
    Tile t;
    t.store = true;
    const int64_t half = kPair ? (int64_t)rank * kBM : 0;      // this CTA's row offset inside a pair item
    const int64_t b_half = kPair ? (int64_t)rank * (kBN / 2) : 0;
    if (kMode == kModeRows) {
        const int64_t n_tiles = p.N / kBN;
        const int64_t mt = idx / n_tiles, nt = idx % n_tiles;
        int64_t base;
        if (kPair || kRowsTail<kMode, kBN, kPair>) {
            int lo = 0, hi = (int)p.E;                   // last expert with pfx[e] <= mt
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (pfx[mid] <= mt) lo = mid; else hi = mid;
            }
            t.e = lo;
            base = kPair ? __ldg(p.seg + t.e) + (mt - pfx[t.e]) * (2 * kBM) : __ldg(p.seg + t.e + 1) - kBM;
            if (kPair) t.store = rank == 0 || base + kBM < __ldg(p.seg + t.e + 1);
        } else {
            base = mt * kBM;
            t.e = find_expert(p.seg, p.E, base);
        }
        const int64_t a_row = t.store ? base + half : base;
        t.row0 = base + half;
        t.col0 = nt * kBN;
        const int64_t kbytes = kKind == kKindNVFP4 ? p.K / 2 : p.K;
        t.k_tiles = kbytes / kStageBytesK;
        t.k0_bytes = 0;
        t.a_y = a_row;
        t.sfa_atom0 = (a_row / kBM) * p.sfa_groups;
        if (kKind == kKindNVFP4) {                      // B = weight stack [E*N, K]
            const int64_t b_first = t.e * p.N + t.col0;
            t.b_y = b_first + b_half;
            t.b_x0 = 0;
            t.sfb_atom0 = (b_first / kBM) * p.sfb_groups;
        } else {                                        // DGRAD: B = [N, E*K]
            t.b_y = t.col0 + b_half;
            t.b_x0 = t.e * p.K;
            t.sfb_atom0 = (t.col0 / kBM) * p.sfb_groups + t.e * p.K / 128;
        }
    } else {                                            // WGRAD: out [E, N, K]
        const int64_t rows = kPair ? 2 * kBM : kBM;
        const int64_t nt_n = p.N / rows, nt_k = p.K / kBN;
        t.e = idx / (nt_n * nt_k);
        const int64_t rem = idx % (nt_n * nt_k);
        // the dimension with fewer tiles varies fastest: a wave of items then
        // re-streams the smaller set of operand row blocks
        const bool k_outer = nt_k >= nt_n;
        const int64_t tn = k_outer ? rem % nt_n : rem / nt_k, tk = k_outer ? rem / nt_n : rem % nt_k;
        const int64_t s0 = __ldg(p.seg + t.e), s1 = __ldg(p.seg + t.e + 1);
        t.a_y = tn * rows + half;
        t.row0 = t.e * p.N + t.a_y;
        t.col0 = tk * kBN;
        t.b_x0 = 0;
        t.b_y = t.col0 + b_half;
        if constexpr (kKind == kKindNVFP4) {
            // two tokens per K-byte: a stage holds 256 tokens, a scale atom
            // 64 (segments are multiples of 256 tokens)
            t.k_tiles = (s1 - s0) / (2 * kStageBytesK);
            t.k0_bytes = s0 / 2;
            t.sfa_atom0 = t.a_y / kBM * p.sfa_groups + s0 / 64;
            t.sfb_atom0 = t.col0 / kBM * p.sfb_groups + s0 / 64;
        } else {
            t.k_tiles = (s1 - s0) / kStageBytesK;
            t.k0_bytes = s0;
            t.sfa_atom0 = t.a_y / kBM * p.sfa_groups + s0 / 128;
            t.sfb_atom0 = t.col0 / kBM * p.sfb_groups + s0 / 128;
        }
    }
    return t;
}

// Shared-memory and TMEM budget of one CTA.  A stage holds 128 K-bytes of A
// (128 rows), of B (kBN rows, or kBN/2 for a pair) and the stage's scale
// atoms: SFA for this CTA's 128 rows and SFB for all kBN columns (each CTA of
// a pair keeps a full copy: the MMA reads B's scales from every CTA's TMEM).
//
// TMEM (512 columns): two accumulator buffers of kBN columns at 0 and
// kAccStride, then a ring of kSfSlots scale regions.  When 2 kBN columns do
// not fit beside the scales the buffers overlap in kOvChunks 32-column chunks:
// the epilogue drains those first and releases them, so the next tile's MMAs
// wait for a fraction of the drain instead of all of it.  NVFP4 pairs keep
// only two scale regions (a ring released by MMA commits, decoupled from the
// shared-memory stages) to make that overlap small.
constexpr int kSmemLimit = 227 * 1024;
template <int kKind, int kBN, bool kPair, int kOut>
struct Smem {
    static constexpr int kA = kBM * kStageBytesK;                       // 16 KB
    static constexpr int kB = (kPair ? kBN / 2 : kBN) * kStageBytesK;
    static constexpr int kAtomsA = kKind == kKindNVFP4 ? 4 : 1;         // scale atoms per stage, 128-row group
    static constexpr int kAtomsB = kAtomsA * (kBN / 128);
    static constexpr int kSfa = kAtomsA * 512;
    static constexpr int kSfb = kAtomsB * 512;
    static constexpr int kAbTx = kA + kB;                               // operand bytes per stage and CTA
    static constexpr int kSfTx = kSfa + kSfb;
    static constexpr int kStage = (kAbTx + kSfTx + 1023) / 1024 * 1024;  // stride keeps every SW128 tile 1024-aligned
    static constexpr int kSfaCols = 4 * kAtomsA;
    static constexpr int kSfbCols = 4 * kAtomsB;
    static constexpr int kSfRegion = kSfaCols + kSfbCols;
    // per-expert item prefix: pair kernels and the ROWS tail kernel (the only
    // single-CTA kernel with 256-wide tiles)
    static constexpr int kPfxBytes = (kPair || kBN == 256) ? 4 * (kMaxPairExperts + 4) : 0;
    // S2F6: the rotation's signs (+-1.0f) of every output column, N <= 4096
    static constexpr int kMaskWords = kOut == kOutTypeS2F6 ? 4096 : 0;
    static constexpr int kFixed = 512 + kPfxBytes + 4 * kMaskWords + 1024;   // barriers + prefix + masks + slack
    static constexpr int stages_for(int staging) {
        for (int s = 6; s > 2; --s)
            if (s * kStage + staging + kFixed <= kSmemLimit) return s;
        return 2;
    }
    // Epilogue staging, 8 warps: fp32 boxes need 4 KB each; bf16 boxes are 2 KB
    // and get two buffers per warp unless giving up the second buys a
    // pipeline stage (operands in flight are what bound these kernels).
    static constexpr bool kOneBox = kOut == kOutTypeBF16 && stages_for(8 * 2048) > stages_for(8 * 4096);
    // S2F6 boxes are 32 rows x 32 bytes: two 1 KB buffers per warp, then the
    // tile's E8M0 bytes (128 rows x 8 bytes, two buffers).
    static constexpr int kWarpStaging = kOut == kOutTypeS2F6 ? 2048 : (kOneBox ? 2048 : 4096);
    static constexpr int kE8Bytes = kOut == kOutTypeS2F6 ? 2 * kBM * (kBN / 32) : 0;
    static constexpr int kStaging = 8 * kWarpStaging + kE8Bytes;
    static constexpr int kStages = stages_for(kStaging);
    static constexpr int kStagingOff = kStages * kStage;
    static_assert(kStage % 1024 == 0 && kStagingOff % 1024 == 0, "128-byte swizzle needs 1024-byte aligned tiles");
    static constexpr int kBarOff = kStagingOff + kStaging;
    static constexpr int kPfxOff = kBarOff + 512;
    static constexpr int kMaskOff = kPfxOff + kPfxBytes;
    static constexpr int kBytes = kMaskOff + 4 * kMaskWords + 1024;
    static_assert(kBytes <= kSmemLimit, "shared memory budget");
    // TMEM
    static constexpr int kSfSlots = (kBN == 256 && kKind == kKindNVFP4) ? 2 : kStages;
    static constexpr int kSfCols = kSfSlots * kSfRegion;
    static constexpr int kAccStride = (kTmemCols - kBN - kSfCols) / 32 * 32 < kBN
                                    ? (kTmemCols - kBN - kSfCols) / 32 * 32 : kBN;
    static constexpr int kOvChunks = (kBN - kAccStride) / 32;           // chunks shared by the two buffers
    static constexpr int kSfCol = kAccStride + kBN;
    static_assert(kSfCol + kSfCols <= kTmemCols && kAccStride > 0, "TMEM budget");
    static_assert(kOvChunks <= 4, "shared chunks must fall in the epilogue's first load group");
};

__device__ __forceinline__ void tmem_st_32x32b_x4(uint32_t taddr, const uint4& v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};"
                 :: "r"(taddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// Bounded wait for phase `parity` of a local barrier against a shared deadline
// (used only while draining at exit).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, unsigned long long t0) {
    while (!mbar_try_wait(bar, parity) && globaltimer() - t0 < kWaitLimitNs) {}
}

template <int kKind, int kMode, int kBN, int kOut, bool kPair>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmOut, const GemmArgs p) {
    using L = Smem<kKind, kBN, kPair, kOut>;
    constexpr int kStages = L::kStages;
    constexpr int kSlots = L::kSfSlots;
    constexpr bool kSfRing = kSlots < kStages;                          // scale regions released by MMA commits
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);   // operands landed (pair: leader's counts both CTAs)
    uint64_t* empty = full + kStages;                                   // stage consumed by the MMAs
    uint64_t* sf_landed = empty + kStages;                              // pair: this CTA's scale atoms landed
    uint64_t* sf_full = sf_landed + kStages;                            // [kSlots] scales in TMEM (pair: both CTAs)
    uint64_t* sf_free = sf_full + kSlots;                               // [kSlots] scale region read by the MMAs
    uint64_t* acc_full = sf_free + kSlots;       // [2]: accumulator buffer b ready
    uint64_t* acc_free = acc_full + 2;           // [2]: see the epilogue (pair: both CTAs report)
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(acc_free + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);
    uint64_t* e8_ready = acc_free + 3;           // [4][2] S2F6: warp 12 + q wrote its E8M0 bytes into buffer b

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = kPair ? cluster_ctarank() : 0u;
    const int64_t first = kPair ? (int64_t)(blockIdx.x >> 1) : (int64_t)blockIdx.x;
    const int64_t stride = kPair ? (int64_t)(gridDim.x >> 1) : (int64_t)gridDim.x;
    int32_t* pfx = reinterpret_cast<int32_t*>(smem + L::kPfxOff);
    static_assert(kPair || kBN == 128 || kRowsTail<kMode, kBN, kPair>, "single-CTA 256-wide tiles: ROWS tail only");
    if ((kPair && kMode == kModeRows) || kRowsTail<kMode, kBN, kPair>) build_row_prefix<!kPair>(p, pfx);
    const int64_t total = total_tiles<kMode, kBN, kPair>(p, pfx);
    if (first >= total) return;                                         // uniform across a pair

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_landed[s], 1);
        }
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(&sf_full[s], kPair ? 8 : 4);
            mbar_init(&sf_free[s], 1);
        }
        for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_free[b], kPair ? 16 : 8); }
        for (int qq = 0; qq < 8; ++qq) mbar_init(&e8_ready[qq], 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
        asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(&tmOut)) : "memory");
    }
    if (kPair) cluster_sync();                  // the peer's barriers exist before anything arrives on them
    if (warp == 1) tmem_alloc<kPair>(tmem_base_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_phase[kStages];
            bool issued[kStages];
            for (int s = 0; s < kStages; ++s) { issued[s] = false; issued_phase[s] = 0; }
            bool ok = true;
            for (int64_t idx = first; idx < total && ok; idx += stride) {
                const Tile t = make_tile<kKind, kMode, kBN, kPair>(p, idx, rank, pfx);
                for (int64_t kt = 0; kt < t.k_tiles; ++kt) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    uint8_t* sa = smem + stage * L::kStage;
                    uint8_t* sb = sa + L::kA;
                    uint8_t* ssfa = sb + L::kB;
                    uint8_t* ssfb = ssfa + L::kSfa;
                    const int kx = (int)(t.k0_bytes + kt * kStageBytesK);
                    uint64_t* sf_bar = &full[stage];
                    if (kPair) {
                        // A and B count on the leader's barrier (it expects both CTAs' bytes);
                        // the scale atoms on this CTA's own barrier for its scale movers.
                        const uint32_t lead_full = map_to_rank(&full[stage], 0);
                        if (rank == 0) mbar_expect_tx(&full[stage], (uint32_t)(2 * L::kAbTx));
                        tma_load_2d_pair(sa, &tmA, lead_full, kx, (int)t.a_y);
                        tma_load_2d_pair(sb, &tmB, lead_full, (int)t.b_x0 + kx, (int)t.b_y);
                        sf_bar = &sf_landed[stage];
                        mbar_expect_tx(sf_bar, (uint32_t)L::kSfTx);
                    } else {
                        mbar_expect_tx(&full[stage], (uint32_t)(L::kAbTx + L::kSfTx));
                        tma_load_2d(sa, &tmA, &full[stage], kx, (int)t.a_y);
#pragma unroll
                        for (int h = 0; h < kBN / 128; ++h)      // B boxes are 128 rows
                            tma_load_2d(sb + h * 128 * kStageBytesK, &tmB, &full[stage], (int)t.b_x0 + kx,
                                        (int)t.b_y + 128 * h);
                    }
                    // (in the bounds-checked build an atom range past its array is read from atom 0
                    // instead, so that the barrier still completes; the violation is counted)
                    const int64_t fa = t.sfa_atom0 + kt * L::kAtomsA;
                    bulk_load(ssfa, p.sfa + (mx_in_range(fa, L::kAtomsA, p.sfa_atoms) ? fa : 0) * 512, L::kSfa, sf_bar);
#pragma unroll
                    for (int h = 0; h < kBN / 128; ++h) {
                        const int64_t fb = t.sfb_atom0 + h * p.sfb_groups + kt * L::kAtomsA;
                        bulk_load(ssfb + h * L::kAtomsA * 512,
                                  p.sfb + (mx_in_range(fb, L::kAtomsA, p.sfb_atoms) ? fb : 0) * 512, L::kAtomsA * 512,
                                  sf_bar);
                    }
                    issued[stage] = true;
                    issued_phase[stage] = phase;
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
            }
            // drain: every copy this CTA issued has landed before its shared
            // memory is released (a pair's operand bytes are counted on the
            // leader; once the MMAs consumed a stage, its copies had landed)
            const unsigned long long t0 = globaltimer();
            for (int s = 0; s < kStages; ++s)
                if (issued[s]) {
                    if (kPair) {
                        drain_wait(&sf_landed[s], issued_phase[s], t0);
                        if (rank == 0) drain_wait(&full[s], issued_phase[s], t0);
                        else drain_wait(&empty[s], issued_phase[s], t0);
                    } else {
                        drain_wait(&full[s], issued_phase[s], t0);
                    }
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (a pair's leader only)
        // Tile i accumulates into buffer i & 1.  With disjoint buffers it
        // waits until tile i-2 left its buffer; with overlapping buffers until
        // tile i-1's shared chunks were drained (which implies the former).
        if (lane == 0 && rank == 0) {
            constexpr uint32_t kFmt = kKind == kKindNVFP4 ? 1u : 0u;      // E2M1 / E4M3
            constexpr uint32_t kScaleFmt = kKind == kKindNVFP4 ? 0u : 1u; // UE4M3 / UE8M0
            constexpr int kM = kPair ? 2 * kBM : kBM;
            int stage = 0, slot = 0;
            uint32_t phase = 0, sphase = 0, it = 0;
            bool ok = true;
            for (int64_t idx = first; idx < total && ok; idx += stride) {
                const Tile t = make_tile<kKind, kMode, kBN, kPair>(p, idx, rank, pfx);
                if (L::kOvChunks > 0) {
                    if (it > 0 && !mbar_wait(&acc_free[(it - 1) & 1], ((it - 1) >> 1) & 1u, abort_flag)) break;
                } else {
                    if (!mbar_wait(&acc_free[it & 1], ((it >> 1) & 1u) ^ 1u, abort_flag)) break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)((it & 1) * L::kAccStride);
                for (int64_t kt = 0; kt < t.k_tiles; ++kt) {
                    if (!mbar_wait(&full[stage], phase, abort_flag) || !mbar_wait(&sf_full[slot], sphase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint8_t* sa = smem + stage * L::kStage;
                    const uint8_t* sb = sa + L::kA;
                    const uint32_t sfa = tmem + L::kSfCol + slot * L::kSfRegion;
                    const uint32_t sfb = sfa + L::kSfaCols;
                    const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sb);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t sfa_t, sfb_t, id;
                        if (kKind == kKindNVFP4) {
                            sfa_t = sfa + 4 * j;
                            sfb_t = sfb + (kBN / 32) * j;
                            id = idesc_block_scaled(kFmt, kScaleFmt, kM, kBN, 0, 0);
                        } else {
                            sfa_t = sfa | ((uint32_t)j << 30);
                            sfb_t = sfb | ((uint32_t)j << 30);
                            id = idesc_block_scaled(kFmt, kScaleFmt, kM, kBN, (uint32_t)j, (uint32_t)j);
                        }
                        mma_block_scaled<kKind, kPair>(acc, operand_desc(a0 + 32 * j), operand_desc(b0 + 32 * j), id,
                                                       sfa_t, sfb_t, (kt > 0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit<kPair>(&empty[stage]);
                    if (kSfRing) tc_commit<kPair>(&sf_free[slot]);
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                    if (++slot == kSlots) { slot = 0; sphase ^= 1u; }
                }
                if (!ok) break;
                tc_commit<kPair>(&acc_full[it & 1]);
                ++it;
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
        // In a pair each CTA fills its own TMEM and reports to the leader.
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        int stage = 0, slot = 0;
        uint32_t phase = 0, sphase = 0;
        bool ok = true;
        for (int64_t idx = first; idx < total && ok; idx += stride) {
            const Tile t = make_tile<kKind, kMode, kBN, kPair>(p, idx, rank, pfx);
            for (int64_t kt = 0; kt < t.k_tiles; ++kt) {
                if (!mbar_wait(kPair ? &sf_landed[stage] : &full[stage], phase, abort_flag)) { ok = false; break; }
                const uint8_t* ssfa = smem + stage * L::kStage + L::kA + L::kB;
                const uint8_t* ssfb = ssfa + L::kSfa;
                uint4 va[L::kAtomsA], vb[L::kAtomsB];
#pragma unroll
                for (int j = 0; j < L::kAtomsA; ++j) va[j] = reinterpret_cast<const uint4*>(ssfa + j * 512)[lane];
#pragma unroll
                for (int j = 0; j < L::kAtomsB; ++j) vb[j] = reinterpret_cast<const uint4*>(ssfb + j * 512)[lane];
                if (kSfRing && !mbar_wait(&sf_free[slot], sphase ^ 1u, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t sfa = tmem + lane_base + L::kSfCol + slot * L::kSfRegion;
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
                if (lane == 0) {
                    if (kPair) mbar_arrive_cluster(map_to_rank(&sf_full[slot], 0));
                    else mbar_arrive(&sf_full[slot]);
                }
                if (++stage == kStages) { stage = 0; phase ^= 1u; }
                if (++slot == kSlots) { slot = 0; sphase ^= 1u; }
            }
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ epilogue
        // Eight warps: warp w reads TMEM lane quarter w%4 (a warp may touch
        // only its own 32 lanes) and every other 32-column chunk of the tile
        // (parity (w-8)/4), in a drain order that puts the chunks shared with
        // the other accumulator buffer first.  Chunks are loaded two at a
        // time; after the first pair (which holds every shared chunk) the warp
        // reports on acc_free, then converts, stages each chunk as one 32x32
        // box in shared memory and writes it with a TMA tensor store.  bf16
        // boxes (64-byte rows, 64-byte swizzle) alternate between two 2 KB
        // buffers, or use one when the second would cost a pipeline stage;
        // fp32 boxes (128-byte rows, 128-byte swizzle) use one 4 KB buffer.  A
        // pair's CTAs each drain their own 128 rows.
        constexpr int kChunks = kBN / 32;
        constexpr int kOv = L::kOvChunks;
        const int q = warp & 3;
        const int h = (warp - 8) >> 2;
        const int r = q * 32 + lane;
        uint8_t* stg = smem + L::kStagingOff + (warp - 8) * L::kWarpStaging;
        // S2F6: the E8M0 bytes of the tile's rows, [128][kBN / 32] per buffer;
        // warp 8 + q stores each row's group of kBN / 32 bytes once warp 12 + q
        // reported its half on e8_ready[q][buffer], one store per row instead
        // of one per byte.  Buffers (and their barriers) alternate by stored
        // tile: warp 12 + q reaches the next use of a buffer only after warp
        // 8 + q released the tile that follows it, which it does after the
        // store, so a barrier never runs a phase ahead of its waiter.
        uint8_t* e8s = smem + L::kStagingOff + 8 * L::kWarpStaging;
        uint32_t n_stored = 0;
        const uint32_t acc_free_lead[2] = {kPair ? map_to_rank(&acc_free[0], 0) : 0u,
                                           kPair ? map_to_rank(&acc_free[1], 0) : 0u};
        uint32_t it = 0, nbox = 0;
        // S2F6: the rotation's signs of every output column as +-1.0f, once per
        // CTA (the eight epilogue warps fill the table, then meet on named
        // barrier 1); wider outputs take each block's mask word instead
        float* signs = reinterpret_cast<float*>(smem + L::kMaskOff);
        const bool sign_table = kOut == kOutTypeS2F6 && p.ldo <= L::kMaskWords;
        if (sign_table) {
            for (int64_t j = threadIdx.x - 256; j < (p.ldo >> 5); j += 256) {
                const uint32_t m = hadamard_sign_word(p.seed, p.stream_id, (uint64_t)j);
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4*>(signs + 32 * j + i) =
                        make_float4((m >> i) & 1 ? -1.0f : 1.0f, (m >> (i + 1)) & 1 ? -1.0f : 1.0f,
                                    (m >> (i + 2)) & 1 ? -1.0f : 1.0f, (m >> (i + 3)) & 1 ? -1.0f : 1.0f);
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
        }
        // NVFP4: each tile's outer scales (a per-row and a per-expert fp32) are
        // loaded one tile ahead, so their latency overlaps the previous drain.
        auto tile_scale = [&](const Tile& tt) -> float {
            return (kKind == kKindNVFP4 && mx_in_range(tt.row0 + r, 1, p.a_outer_n))
                       ? __ldg(p.a_outer + tt.row0 + r) * __ldg(p.b_outer + tt.e) : 1.0f;
        };
        Tile t_next = make_tile<kKind, kMode, kBN, kPair>(p, first, rank, pfx);
        float scale_next = tile_scale(t_next);
        for (int64_t idx = first; idx < total; idx += stride) {
            const Tile t = t_next;
            const float scale = scale_next;
            if (idx + stride < total) {
                t_next = make_tile<kKind, kMode, kBN, kPair>(p, idx + stride, rank, pfx);
                scale_next = tile_scale(t_next);
            }
            const int b = (int)(it & 1);
            if (!mbar_wait(&acc_full[b], (it >> 1) & 1u, abort_flag)) break;
            tc_fence_after();
            auto release = [&]() {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (kPair) mbar_arrive_cluster(acc_free_lead[b]);
                    else mbar_arrive(&acc_free[b]);
                }
            };
            if (!t.store) {                                     // half pair: nothing to store
                release();
                ++it;
                continue;
            }
            const uint32_t tbase = tmem + (uint32_t)(b * L::kAccStride) + ((uint32_t)(q * 32) << 16);
            const int oy = (int)(t.row0 + q * 32);
#pragma unroll
            for (int g = 0; g < kChunks / 4; ++g) {
                int col[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int j = h + 4 * g + 2 * u;                // drain position
                    col[u] = 32 * (b == 0 ? (j < kOv ? kChunks - kOv + j : j - kOv) : j);
                }
                float v[2][32];
                if (t.k_tiles > 0) {
                    tmem_ld2_32x32b_x32(tbase + (uint32_t)col[0], tbase + (uint32_t)col[1], v[0], v[1]);
                } else {
#pragma unroll
                    for (int u = 0; u < 2; ++u)
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[u][i] = 0.0f;
                }
                if (g == (kOv > 0 ? 0 : kChunks / 4 - 1)) release();
                if constexpr (kOut == kOutTypeS2F6) {
                    // Each thread holds 32 consecutive outputs of its row: one
                    // rotation block.  Scale, rotate and quantise it in registers,
                    // stage the warp's 32 rows x 32 codes as one box (two 1 KB
                    // buffers per warp) and write it with a TMA tensor store; the
                    // exponent byte goes straight to global memory.
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int64_t ocol = t.col0 + col[u];
                        uint32_t w[8];
                        int e;
                        if (sign_table) {
                            e = s2f6_block_scaled(v[u], scale, signs + ocol, w);
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[u][i] = v[u][i] * scale;
                            e = s2f6_block_mask(v[u], hadamard_sign_word(p.seed, p.stream_id, (uint64_t)(ocol >> 5)), w);
                        }
                        uint8_t* box = stg + (nbox & 1u) * 1024;
                        if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                        __syncwarp();
                        const uint32_t row = smem_u32(box) + (uint32_t)lane * 32u;
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                     :: "r"(row), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]) : "memory");
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                     :: "r"(row + 16u), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]) : "memory");
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                        __syncwarp();
                        if (lane == 0) {
                            asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
                                         :: "l"(reinterpret_cast<uint64_t>(&tmOut)), "r"((int)ocol), "r"(oy),
                                            "r"(smem_u32(box)) : "memory");
                            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                        }
                        ++nbox;
                        e8s[(n_stored & 1u) * (L::kE8Bytes / 2) + r * (kBN / 32) + (col[u] >> 5)] = (uint8_t)(e + 127);
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        uint8_t* box;
                        if (kOut == kOutTypeBF16) {
                            if (L::kOneBox) {
                                box = stg;
                                if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                            } else {
                                box = stg + (nbox & 1u) * 2048;
                                if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                            }
                            __syncwarp();
                            const uint32_t row = smem_u32(box) + (uint32_t)lane * 64u;
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                uint32_t w[4];
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    __nv_bfloat162 bb = __floats2bfloat162_rn(v[u][8 * c + 2 * i] * scale,
                                                                              v[u][8 * c + 2 * i + 1] * scale);
                                    w[i] = *reinterpret_cast<uint32_t*>(&bb);
                                }
                                const uint32_t sw = (uint32_t)(c ^ ((lane >> 1) & 3));
                                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                             :: "r"(row + sw * 16u), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]) : "memory");
                            }
                        } else {
                            box = stg;
                            if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                            __syncwarp();
                            const uint32_t row = smem_u32(box) + (uint32_t)lane * 128u;
#pragma unroll
                            for (int c = 0; c < 8; ++c) {
                                const uint32_t sw = (uint32_t)(c ^ (lane & 7));
                                asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};"
                                             :: "r"(row + sw * 16u), "f"(v[u][4 * c] * scale), "f"(v[u][4 * c + 1] * scale),
                                                "f"(v[u][4 * c + 2] * scale), "f"(v[u][4 * c + 3] * scale) : "memory");
                            }
                        }
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                        __syncwarp();
                        if (lane == 0) {
                            asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
                                         :: "l"(reinterpret_cast<uint64_t>(&tmOut)), "r"((int)t.col0 + col[u]), "r"(oy),
                                            "r"(smem_u32(box)) : "memory");
                            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                        }
                        ++nbox;
                    }
                }
            }
            if (kOut == kOutTypeS2F6) {
                const uint8_t* src = e8s + (n_stored & 1u) * (L::kE8Bytes / 2) + r * (kBN / 32);
                uint64_t* ready = &e8_ready[2 * q + (n_stored & 1u)];
                if (h == 1) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(ready);
                } else {
                    if (!mbar_wait(ready, (n_stored >> 1) & 1u, abort_flag)) break;
                    static_assert(kBN / 32 == 8 || kBN / 32 == 4, "E8M0 group of a tile row: one 8- or 4-byte store");
                    uint8_t* dst = p.e8m0_out + (t.row0 + r) * (p.ldo >> 5) + (t.col0 >> 5);
                    if (kBN / 32 == 8) *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(src);
                    else *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<const uint32_t*>(src);
                }
                ++n_stored;
            }
            ++it;
        }
        if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }

    // Teardown: every MMA has completed (the epilogue saw each accumulator's
    // commit) and every TMEM read is done before the columns are freed; a
    // pair frees its joint allocation only once both CTAs are here.
    tc_fence_before();
    __syncthreads();
    if (kPair) cluster_sync();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc<kPair>(tmem, kTmemCols);
    }
}

// The bounded wait on a barrier that nothing completes: exercises the expiry
// path (status word set, kernel returns) without a fault or a hang.
__global__ void wait_selftest_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, &abort_flag, limit_ns);
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

// Output [rows, cols] (row stride cols), box 32 x 32: bf16 with 64-byte rows
// and 64-byte swizzle, fp32 with 128-byte rows and 128-byte swizzle.
// S2F6 codes [rows, cols] int8, box 32 x 32 (32-byte rows, no swizzle).
int make_s2f6_map(CUtensorMap* m, void* base, int64_t rows, int64_t cols) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return MX_EUNSUPPORTED;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols};
    const cuuint32_t box[2] = {32, 32};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MX_OK : MX_EINVAL;
}

int make_out_map(CUtensorMap* m, void* base, int64_t rows, int64_t cols, bool bf16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return MX_EUNSUPPORTED;
    const cuuint64_t esize = bf16 ? 2 : 4;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * esize};
    const cuuint32_t box[2] = {32, 32};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    bf16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MX_OK : MX_EINVAL;
}

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

// Largest grid of co-resident CTA pairs for one pair kernel on this device.
template <typename Kern>
int max_pairs(Kern kern, const cudaLaunchConfig_t& cfg) {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (cached[dev] > 0) return cached[dev];
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters <= 0) {
        (void)cudaGetLastError();
        clusters = num_sms() / 2;
    }
    cached[dev] = clusters;
    return clusters;
}

template <int kKind, int kMode, int kBN, int kOut, bool kPair>
int launch(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mo, const GemmArgs& args, int64_t items,
           cudaStream_t stream) {
    using L = Smem<kKind, kBN, kPair, kOut>;
    auto kern = grouped_gemm_kernel<kKind, kMode, kBN, kOut, kPair>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes) != cudaSuccess)
        return mx_launch_status();
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = L::kBytes;
    cfg.stream = stream;
    int64_t slots = num_sms();
    if (kPair) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cfg.gridDim = dim3(2);
        slots = max_pairs(kern, cfg);
    }
    const int64_t n = std::max<int64_t>(1, std::min<int64_t>(items, slots));
    cfg.gridDim = dim3((unsigned)(kPair ? 2 * n : n));
    if (cudaLaunchKernelEx(&cfg, kern, ma, mb, mo, args) != cudaSuccess) return mx_launch_status();
    mx_count_launch();
    return mx_launch_status();
}

constexpr int kOutS2F6Dtype = -2;                      // internal out_dtype of grouped_gemm_nvfp4_s2f6

// CTA pairs with 256 x 256 output tiles wherever the shape allows (measured
// on B200: halving each CTA's B traffic per flop and the deeper pipeline it
// buys lift the tensor pipe's duty cycle); in ROWS mode the pair kernel is
// followed by the tail kernel (single CTAs, 128 x 256 tiles), which takes the
// experts' leftover row tiles when there are enough of them.  Other shapes use
// single CTAs with 128 x 128 tiles and two accumulators.  items_* bound the
// kernels' item counts (grid sizes).
template <int kKind, int kMode, int kOut>
int launch_wide(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mo, const GemmArgs& args,
                int64_t items_pair, int64_t items_tail, cudaStream_t stream) {
    if (int st = launch<kKind, kMode, 256, kOut, true>(ma, mb, mo, args, items_pair, stream)) return st;
    if constexpr (kMode == kModeRows)
        return launch<kKind, kMode, 256, kOut, false>(ma, mb, mo, args, items_tail, stream);
    return MX_OK;
}

// The tail kernel runs the leftover row tiles when they fill at least this
// many waves of single CTAs (measured on B200 at the 384- and 64-expert
// layers: 11 waves gain 2%, 2.3 waves lose 2% against half pairs).
constexpr int64_t kTailMinWaves = 4;

template <int kKind, int kMode>
int dispatch(bool pair, int64_t out_rows, int64_t out_cols, int out_dtype, const CUtensorMap& ma,
             const CUtensorMap& mb, GemmArgs args, int64_t items_pair, int64_t items_single,
             cudaStream_t stream) {
    // ROWS tail items: at most one row tile per expert and 256-wide column tile
    const int64_t items_tail = std::min(args.E, args.M_cap / kBM) * (args.N / 256);
    args.tail_min_items = kTailMinWaves * num_sms();
    CUtensorMap mo;
    if (out_dtype == kOutS2F6Dtype) {
        if constexpr (kKind == kKindNVFP4 && kMode == kModeRows) {
            if (int st = make_s2f6_map(&mo, args.out, out_rows, out_cols)) return st;
            return pair ? launch_wide<kKind, kMode, kOutTypeS2F6>(ma, mb, mo, args, items_pair, items_tail, stream)
                        : launch<kKind, kMode, 128, kOutTypeS2F6, false>(ma, mb, mo, args, items_single, stream);
        } else {
            return MX_EINVAL;
        }
    }
    const bool bf16 = out_dtype == MX_OUT_BF16;
    if (int st = make_out_map(&mo, args.out, out_rows, out_cols, bf16)) return st;
    if (pair)
        return bf16 ? launch_wide<kKind, kMode, kOutTypeBF16>(ma, mb, mo, args, items_pair, items_tail, stream)
                    : launch_wide<kKind, kMode, kOutTypeF32>(ma, mb, mo, args, items_pair, items_tail, stream);
    return bf16 ? launch<kKind, kMode, 128, kOutTypeBF16, false>(ma, mb, mo, args, items_single, stream)
                : launch<kKind, kMode, 128, kOutTypeF32, false>(ma, mb, mo, args, items_single, stream);
}

}  // namespace

extern "C" int mx_sync_status(cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return mx_set_cuda_error(e);
    unsigned int word = 0, zero = 0;
    if ((e = cudaMemcpyFromSymbol(&word, g_mx_status_word, sizeof(word))) != cudaSuccess) return mx_set_cuda_error(e);
    if (word && (e = cudaMemcpyToSymbol(g_mx_status_word, &zero, sizeof(zero))) != cudaSuccess)
        return mx_set_cuda_error(e);
    if (word & kStatusTimeout) return MX_ETIMEOUT;
    return word ? MX_EDATA : MX_OK;
}

// Device address of the status word on the current device, looked up once per
// device; kernels in other translation units take it as an argument.
static std::mutex g_status_addr_mutex;
static unsigned int* g_status_addr[64] = {nullptr};

int mx_status_word_address(unsigned int** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return mx_set_cuda_error(e);
    if (dev < 0 || dev >= 64) return MX_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_status_addr_mutex);
    if (!g_status_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_mx_status_word);
        if (e != cudaSuccess || !p) return mx_set_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
        g_status_addr[dev] = static_cast<unsigned int*>(p);
    }
    *out = g_status_addr[dev];
    return MX_OK;
}

// bf16 [rows, cols] (row stride cols), box box_rows x box_cols, 128-byte swizzle
// (box_cols * 2 == 128).
int mx_make_bf16_tile_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return MX_EUNSUPPORTED;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MX_OK : MX_EINVAL;
}

extern "C" int mx_wait_selftest(int64_t limit_us, cudaStream_t stream) {
    MX_NVTX_RANGE("mx_wait_selftest");
    if (limit_us <= 0 || limit_us > 10 * 1000 * 1000) return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    wait_selftest_kernel<<<1, 32, 0, stream>>>((unsigned long long)limit_us * 1000ull);
    mx_count_launch();
    return mx_launch_status();
}

extern "C" int grouped_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_outer,
                                  const uint8_t* b_codes, const uint8_t* b_sf, const float* b_outer,
                                  const int64_t* seg_offsets, int64_t E, int64_t M_cap, int64_t N, int64_t K,
                                  void* out, int out_dtype, cudaStream_t stream) {
    MX_NVTX_RANGE("grouped_gemm_nvfp4");
    if (((!a_codes || !a_sf || !a_outer || !b_codes || !b_sf || !b_outer || !seg_offsets || !out) && M_cap > 0) || E < 1 ||
        M_cap < 0 || M_cap % 128 || N <= 0 || N % 128 || K <= 0 || K % 256)
        return MX_EINVAL;
    if (out_dtype != MX_OUT_F32 && out_dtype != MX_OUT_BF16) return MX_EINVAL;
    if (!mx_aligned(a_codes, 16) || !mx_aligned(b_codes, 16) || !mx_aligned(a_sf, 16) || !mx_aligned(b_sf, 16) ||
        !mx_aligned(out, 16))
        return MX_EINVAL;
    if (M_cap >= (int64_t)1 << 31 || E * N >= (int64_t)1 << 31 || K / 2 >= (int64_t)1 << 31) return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (M_cap == 0) return MX_OK;
    CUtensorMap ma, mb;
    if (int st = make_map(&ma, a_codes, M_cap, K / 2, kBM)) return st;
    if (int st = make_map(&mb, b_codes, E * N, K / 2, 128)) return st;
    GemmArgs a{};
    a.sfa = a_sf; a.sfb = b_sf; a.a_outer = a_outer; a.b_outer = b_outer; a.seg = seg_offsets; a.out = out;
    a.E = E; a.M_cap = M_cap; a.N = N; a.K = K;
    a.sfa_groups = K / 64; a.sfb_groups = K / 64; a.ldo = N;
    a.sfa_atoms = M_cap / 128 * a.sfa_groups; a.sfb_atoms = E * N / 128 * a.sfb_groups; a.a_outer_n = M_cap;
    return dispatch<kKindNVFP4, kModeRows>(N % 256 == 0 && E <= kMaxPairExperts, M_cap, N, out_dtype, ma, mb, a, (M_cap / kBM) * (N / 256),
                                           (M_cap / kBM) * (N / 128), stream);
}

extern "C" int grouped_gemm_nvfp4_s2f6(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_outer,
                                       const uint8_t* b_codes, const uint8_t* b_sf, const float* b_outer,
                                       const int64_t* seg_offsets, int64_t E, int64_t M_cap, int64_t N, int64_t K,
                                       uint64_t seed, uint64_t stream_id, int8_t* codes, uint8_t* e8m0,
                                       cudaStream_t stream) {
    MX_NVTX_RANGE("grouped_gemm_nvfp4_s2f6");
    if (((!a_codes || !a_sf || !a_outer || !b_codes || !b_sf || !b_outer || !seg_offsets || !codes || !e8m0) &&
         M_cap > 0) || E < 1 || M_cap < 0 || M_cap % 128 || N <= 0 || N % 128 || K <= 0 || K % 256)
        return MX_EINVAL;
    if (!mx_aligned(a_codes, 16) || !mx_aligned(b_codes, 16) || !mx_aligned(a_sf, 16) || !mx_aligned(b_sf, 16) ||
        !mx_aligned(codes, 16) || !mx_aligned(e8m0, 8))
        return MX_EINVAL;
    if (M_cap >= (int64_t)1 << 31 || E * N >= (int64_t)1 << 31 || K / 2 >= (int64_t)1 << 31) return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (M_cap == 0) return MX_OK;
    CUtensorMap ma, mb;
    if (int st = make_map(&ma, a_codes, M_cap, K / 2, kBM)) return st;
    if (int st = make_map(&mb, b_codes, E * N, K / 2, 128)) return st;
    GemmArgs a{};
    a.sfa = a_sf; a.sfb = b_sf; a.a_outer = a_outer; a.b_outer = b_outer; a.seg = seg_offsets; a.out = codes;
    a.E = E; a.M_cap = M_cap; a.N = N; a.K = K;
    a.sfa_groups = K / 64; a.sfb_groups = K / 64; a.ldo = N;
    a.sfa_atoms = M_cap / 128 * a.sfa_groups; a.sfb_atoms = E * N / 128 * a.sfb_groups; a.a_outer_n = M_cap;
    a.e8m0_out = e8m0; a.seed = seed; a.stream_id = stream_id;
    return dispatch<kKindNVFP4, kModeRows>(N % 256 == 0 && E <= kMaxPairExperts, M_cap, N, kOutS2F6Dtype, ma, mb, a,
                                           (M_cap / kBM) * (N / 256), (M_cap / kBM) * (N / 128), stream);
}

extern "C" int grouped_gemm_mxfp8(int mode, const uint8_t* a_codes, const uint8_t* a_e8m0, const uint8_t* b_codes,
                                  const uint8_t* b_e8m0, const int64_t* seg_offsets, int64_t E, int64_t M_cap,
                                  int64_t N, int64_t K, void* out, int out_dtype, cudaStream_t stream) {
    MX_NVTX_RANGE("grouped_gemm_mxfp8");
    if (((!a_codes || !a_e8m0 || !b_codes || !b_e8m0 || !seg_offsets) && M_cap > 0) || !out || E < 1 || M_cap < 0 ||
        M_cap % 128 ||
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
    if (M_cap == 0) {                                   // WGRAD without routed rows: every dW_e is zero
        const cudaError_t e = cudaMemsetAsync(out, 0, (size_t)(E * N * K) * (out_dtype == MX_OUT_BF16 ? 2 : 4), stream);
        return e == cudaSuccess ? MX_OK : mx_set_cuda_error(e);
    }
    CUtensorMap ma, mb;
    GemmArgs a{};
    a.sfa = a_e8m0; a.sfb = b_e8m0; a.seg = seg_offsets; a.out = out;
    a.E = E; a.M_cap = M_cap; a.N = N; a.K = K;
    if (mode == MX_GEMM_DGRAD) {
        // A [M_cap, K], B [N, E*K]; out [M_cap, N]
        if (int st = make_map(&ma, a_codes, M_cap, K, kBM)) return st;
        if (int st = make_map(&mb, b_codes, N, E * K, 128)) return st;
        a.sfa_groups = K / 128; a.sfb_groups = E * K / 128; a.ldo = N;
        a.sfa_atoms = M_cap / 128 * a.sfa_groups; a.sfb_atoms = N / 128 * a.sfb_groups; a.a_outer_n = M_cap;
        return dispatch<kKindMXFP8, kModeRows>(N % 256 == 0 && E <= kMaxPairExperts, M_cap, N, out_dtype, ma, mb, a,
                                               (M_cap / kBM) * (N / 256), (M_cap / kBM) * (N / 128), stream);
    }
    // WGRAD: A [N, M_cap], B [K, M_cap]; out [E, N, K]
    if (int st = make_map(&ma, a_codes, N, M_cap, kBM)) return st;
    if (int st = make_map(&mb, b_codes, K, M_cap, 128)) return st;
    a.sfa_groups = M_cap / 128; a.sfb_groups = M_cap / 128; a.ldo = K;
    a.sfa_atoms = N / 128 * a.sfa_groups; a.sfb_atoms = K / 128 * a.sfb_groups; a.a_outer_n = E * N;
    const bool pair = N % 256 == 0 && K % 256 == 0;
    return dispatch<kKindMXFP8, kModeWgrad>(pair, E * N, K, out_dtype, ma, mb, a, E * (N / 256) * (K / 256),
                                            E * (N / 128) * (K / 128), stream);
}

// NVFP4 weight gradient (the NVFP4 backward's wgrad): A [N, M_cap] and B
// [K, M_cap] in NVFP4 along the tokens (codes [rows, M_cap/2], scales in the
// MMA layout), outer scales per expert segment: a_outer [E*N] (segment,
// row), b_outer [E].  out[e, n, k] = a_outer[e*N + n] * b_outer[e] * sum over
// the tokens of segment e.  Segments must be multiples of 256 tokens (a
// K-stage of NVFP4 holds 256); other boundaries give wrong sums, no
// out-of-bounds access.
extern "C" int grouped_gemm_nvfp4_wgrad(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_outer,
                                        const uint8_t* b_codes, const uint8_t* b_sf, const float* b_outer,
                                        const int64_t* seg_offsets, int64_t E, int64_t M_cap, int64_t N, int64_t K,
                                        void* out, int out_dtype, cudaStream_t stream) {
    MX_NVTX_RANGE("grouped_gemm_nvfp4_wgrad");
    if (((!a_codes || !a_sf || !a_outer || !b_codes || !b_sf || !b_outer || !seg_offsets) && M_cap > 0) || !out ||
        E < 1 || M_cap < 0 || M_cap % 256 || N <= 0 || N % 128 || K <= 0 || K % 128)
        return MX_EINVAL;
    if (out_dtype != MX_OUT_F32 && out_dtype != MX_OUT_BF16) return MX_EINVAL;
    if (!mx_aligned(a_codes, 16) || !mx_aligned(b_codes, 16) || !mx_aligned(a_sf, 16) || !mx_aligned(b_sf, 16) ||
        !mx_aligned(out, 16))
        return MX_EINVAL;
    if (M_cap >= (int64_t)1 << 31 || E * N >= (int64_t)1 << 31 || K >= (int64_t)1 << 31) return MX_EINVAL;
    if (int st = mx_check_device()) return st;
    if (M_cap == 0) {                                   // no routed rows: every dW_e is zero
        const cudaError_t e = cudaMemsetAsync(out, 0, (size_t)(E * N * K) * (out_dtype == MX_OUT_BF16 ? 2 : 4), stream);
        return e == cudaSuccess ? MX_OK : mx_set_cuda_error(e);
    }
    CUtensorMap ma, mb;
    if (int st = make_map(&ma, a_codes, N, M_cap / 2, kBM)) return st;
    if (int st = make_map(&mb, b_codes, K, M_cap / 2, 128)) return st;
    GemmArgs a{};
    a.sfa = a_sf; a.sfb = b_sf; a.a_outer = a_outer; a.b_outer = b_outer; a.seg = seg_offsets; a.out = out;
    a.E = E; a.M_cap = M_cap; a.N = N; a.K = K;
    a.sfa_groups = M_cap / 64; a.sfb_groups = M_cap / 64; a.ldo = K;
    a.sfa_atoms = N / 128 * a.sfa_groups; a.sfb_atoms = K / 128 * a.sfb_groups; a.a_outer_n = E * N;
    const bool pair = N % 256 == 0 && K % 256 == 0;
    return dispatch<kKindNVFP4, kModeWgrad>(pair, E * N, K, out_dtype, ma, mb, a, E * (N / 256) * (K / 256),
                                            E * (N / 128) * (K / 128), stream);
}

MX_BOUNDS_READER(mx_bounds_word_gemm)
