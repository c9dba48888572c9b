// gemm.cu -- block-scaled NVFP4 GEMM and MoE grouped GEMM on the sm_100a
// tensor cores (tcgen05, kind::mxf4nvf4, 16-element UE4M3 block scales).
//
// D[i][j] = ga * gb * sum_k (e2m1(a_ik) sa(i,k/16)) (e2m1(b_jk) sb(j,k/16)),
// FP32 accumulation in tensor memory (asector.ru, "Nvidia dobivaetsya uspekha
// s 4-bitnym formatom NVFP4", section "NVFP4 and Blackwell": the tensor cores
// compute with scaling and high-precision accumulation; iitak.ru, "Thinking
// Machines uskorila obuchenie Inkling 2 Small 4-bitnymi chislami", section
// "Details": NVFP4 in the expert layers -> the grouped form).
//
// Structure: persistent CTA pairs (clusters of 2, one CTA per SM, 448
// threads each).  A pair computes a 256x256 output tile with the two-SM form
// of the MMA (cta_group::2): each CTA stages its own 128 rows of A and 128 of
// the 256 rows of B, so each SM moves half the B tile and the tensor cores of
// the pair read one copy of it.  Per CTA:
//   warp 0      TMA producer: this CTA's A/B boxes (128-byte swizzled, 4-bit
//               codes two per byte; completing on the leader CTA's barrier,
//               which expects both CTAs' bytes) and its scale atoms (own 128
//               A rows: one 1D bulk copy; all 256 B rows: one 4D box; both on
//               its own barrier, issued before the stage's code tiles so the
//               scale writers' work overlaps the tiles' flight) into a 5-stage
//               ring.
//   warps 2..5  scale writers, one per tensor-memory lane quadrant: each lane
//               loads row i of the stage's 512-byte scale atoms from shared
//               memory and writes them into its quadrant of this CTA's tensor
//               memory with tcgen05.st, then arrives on the leader's barrier
//               of the stage (the one the code tiles complete on).  The
//               tensor pipe spends no cycles on scale copies.
//   warp 1      leader CTA only: one elected thread waits on that one barrier
//               per stage (both CTAs' tiles landed, both CTAs' scales written:
//               one wait instead of two shortens its per-stage path, 658 -> 615
//               cycles per stage at long K) and issues 4 MMAs of 256x256x64, then
//               commits the stage to both CTAs' producers and, after the last
//               K stage, the accumulator to both epilogues.
//   warps 6..13 epilogue: tcgen05.ld of this CTA's 128x256 FP32 accumulator
//               half (two warps per lane quadrant, converted as it is loaded),
//               release of the accumulator to the leader, then stores.  BF16
//               rows are turned around in a 2 KB staging block per warp so
//               that each store instruction writes whole 32-byte sectors of 8
//               rows instead of a 16-byte piece of 32 rows.
// Every mbarrier wait is bounded (2 s); a timeout sets the workspace status
// word and the kernel winds down instead of hanging.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace nvfp4 {

// Operand formats.  NVFP4: E2M1 codes, one UE4M3 scale per 16 elements
// (kind::mxf4nvf4, block16).  MXFP8: E4M3 codes, one UE8M0 scale per 32
// elements (kind::mxf8f6f4, block32) -- the backward-pass format of the
// recipe on the iitak page, "How it works".  MXFP4: E2M1 codes, one UE8M0
// scale per 32 elements (kind::mxf4, block32) -- the OCP format the pages
// compare NVFP4 against (hightech page; asector page, "NVFP4 and Blackwell").
enum : int { kFmtNVFP4 = 0, kFmtMXFP8 = 1, kFmtMXFP4 = 2 };

constexpr int BM = 128;                    // A rows per CTA; a CTA pair covers 2 * BM
constexpr int kMmaM = 2 * BM;              // M of the two-SM MMA
constexpr int kMaxStages = 8;
constexpr int kMaxAccStages = 2;
#ifndef NVFP4_GEMM_EPI_WARPS
#define NVFP4_GEMM_EPI_WARPS 8
#endif
constexpr int kEpiWarps = NVFP4_GEMM_EPI_WARPS;     // epilogue warps per CTA (8 or 16)
constexpr int kGemmThreads = 32 * (6 + kEpiWarps);  // producer, MMA, 4 scale writers, epilogue
static_assert(kEpiWarps == 8 || kEpiWarps == 16, "epilogue warps: 8 or 16");

constexpr int kTmemCols = 512;
constexpr int kMaxGemmGroups = 256;
constexpr int kEpiStageBytes = 2048;  // per epilogue warp: 32 rows x 64 bytes of BF16
constexpr int kSmemLimit = 232448;    // 227 KB of dynamic shared memory per CTA

struct GemmShared {
    uint64_t full[kMaxStages];      // leader: A/B codes of both CTAs landed
    uint64_t sf_full[kMaxStages];   // this CTA's scale atoms landed
    uint64_t empty[kMaxStages];     // the stage's MMAs completed (both CTAs)
    uint64_t acc_full[kMaxAccStages];
    uint64_t acc_empty[kMaxAccStages];
    uint32_t tmem_base;
    int32_t total_tiles;
    int32_t cum_tiles[kMaxGemmGroups + 1];
    int32_t group_start[kMaxGemmGroups + 1];
    int32_t group_sfblk[kMaxGemmGroups + 1];  // first padded 128-row scale block of a group
};

constexpr int kSmemShared = (int)((sizeof(GemmShared) + 1023) / 1024 * 1024);

// Tile and pipeline geometry of one (format, tile width) variant.  Every stage
// holds 128 bytes of K per operand row -- one 128-byte swizzle row, 256 FP4 or
// 128 FP8 elements -- and is consumed by 4 MMAs that each step 32 bytes along K
// (K = 64 for FP4, K = 32 for FP8).
//  - kBN = 256: one 256x256 FP32 accumulator (256 tensor-memory columns) per
//    pair; the next tile's MMAs wait until the epilogue has read it.
//  - kBN = 128: two 256x128 accumulators used in turn, so the MMAs of tile t+1
//    run while the epilogue drains tile t.
// Scale atoms (512 bytes: 128 rows x 4 scale bytes) per 128 rows and stage:
// four for NVFP4 (16 scales per row), two for MXFP4 (8), one for MXFP8 (4).  In
// tensor memory each atom takes 4 columns per 128 rows (column c, lane i: row
// 32c + i's 4 bytes, in every lane quadrant).
template <int kFmt, int kBN>
struct GemmCfg {
    static constexpr int BN = kBN;
    static constexpr int kBRows = kBN / 2;  // B rows staged by each CTA
    static constexpr int kBlocksN = kBN / 128;
    static constexpr int kSfAtoms = kFmt == kFmtNVFP4 ? 4 : kFmt == kFmtMXFP4 ? 2 : 1;
    static constexpr int kKStage = kFmt == kFmtMXFP8 ? 128 : 256;  // K elements per stage
    static constexpr int kKAtom = kFmt == kFmtNVFP4 ? 64 : 128;    // K elements per scale atom
    static constexpr int kA_Bytes = BM * 128;
    static constexpr int kB_Bytes = kBRows * 128;
    static constexpr int kSFA_Bytes = kSfAtoms * 512;
    static constexpr int kSFB_Bytes = kSfAtoms * 512 * kBlocksN;
    // stages start on 1024-byte boundaries (the 128-byte swizzle repeats every 1024)
    static constexpr int kStageBytes = (kA_Bytes + kB_Bytes + kSFA_Bytes + kSFB_Bytes + 1023) / 1024 * 1024;
    static constexpr uint32_t kPairCodeTx = 2u * (kA_Bytes + kB_Bytes);  // the leader's full barrier
    static constexpr int kAccStages = kBN == 256 ? 1 : 2;
    static constexpr int kTmemSF = kAccStages * kBN;  // scale regions follow the accumulators
    static constexpr int kSfColsA = kSfAtoms * 4;
    static constexpr int kSfCols = kSfColsA + kSfAtoms * 4 * kBlocksN;  // written per stage
    static constexpr int kSfStride = (kSfCols + 15) / 16 * 16;            // columns per stage region
    static constexpr int kStagesBySmem =
        (kSmemLimit - kSmemShared - kEpiWarps * kEpiStageBytes - 1024) / kStageBytes;
    static constexpr int kStagesByTmem = (kTmemCols - kTmemSF) / kSfStride;
    static constexpr int kStages = kStagesBySmem < kStagesByTmem
                                       ? (kStagesBySmem < kMaxStages ? kStagesBySmem : kMaxStages)
                                       : (kStagesByTmem < kMaxStages ? kStagesByTmem : kMaxStages);
    static constexpr size_t kSmemBytes =
        (size_t)kStages * kStageBytes + kSmemShared + kEpiWarps * kEpiStageBytes + 1024;
    static_assert(kStages >= 4, "pipeline too shallow");
    static_assert(kTmemSF + kStages * kSfStride <= kTmemCols, "tensor memory overflow");
    static_assert(kSmemBytes <= (size_t)kSmemLimit, "shared memory overflow");
};

struct GemmArgs {
    const uint8_t* sfa;
    const uint8_t* sfb;
    const float* ga;  // NVFP4 tensor scales (unused for MXFP8)
    const float* gb;
    void* D;
    int64_t M, N, K, ldd;
    int bf16_out;
    // grouped form
    int grouped;
    int G;
    const int32_t* group_offsets;
    int64_t total_rows;
    uint32_t* status;
    unsigned long long* cycles;  // workspace: SM cycles of the longest CTA of this call
    float* amax_out;  // optional: max |D| (as stored), atomically accumulated
    uint64_t wait_ns;  // limit of every barrier wait (2 s; shorter under the test hook)
    int no_copies;     // test hook: the producers issue no copy (see wait_test_hook)
};

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address, in the cluster's shared window, of the variable at p in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank)
{
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_addr(p)), "r"(rank));
    return out;
}

// All threads of both CTAs: arrive and wait (release / acquire at cluster scope).
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// Arrive on a barrier of either CTA of the pair (release at CTA scope, as the
// tcgen05 fences around it order the tensor-memory work; a cluster-scope
// release would add a memory barrier to every stage).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster_addr)
{
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster_addr)
                 : "memory");
}

// Pair-form TMA load: the box lands in this CTA's shared memory and its bytes
// are counted on the barrier at `bar` (a cluster address: the leader's).  No
// multicast.  x is a multiple of 128 bytes at every call site.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, int32_t x,
                                                 int32_t y, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Four-dimensional TMA tile load completing on `bar` (x = 0 at every call site).
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int32_t x, int32_t y,
                                            int32_t z, int32_t w, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], "
        "[%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_addr(bar))
        : "memory");
}

// Tensor memory of the pair: one warp with the same index in each CTA.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive (once the issuing thread's earlier tcgen05 operations completed) on
// the barrier at the same offset in both CTAs of the pair.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
        "[%0], %1;" ::"r"(smem_addr(bar)),
        "h"((uint16_t)0x3)
        : "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, 8-row
// groups 1024 bytes apart (start, LBO and SBO in 16-byte units; version 1).
__device__ __forceinline__ uint64_t desc_sw128(const void* p)
{
    const uint64_t start = (smem_addr(p) >> 4) & 0x3FFFu;
    return start | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of a block-scaled MMA, M = 256 (the pair), N = kBN,
// both operands K-major, dense.  NVFP4: A/B format E2M1 (1), UE4M3 scales
// (bit 23 clear).  MXFP8: A/B format E4M3 (0), UE8M0 scales (bit 23 set).
// MXFP4: E2M1 (1), UE8M0.  sf_id is the first byte of each 32-bit scale column
// the MMA reads: an MXFP8 MMA (K 32) reads byte sf_id = 0..3, an MXFP4 MMA
// (K 64) the two bytes from sf_id = 0 or 2; NVFP4 reads all four (sf_id 0).
template <int kFmt, int kBN>
__host__ __device__ constexpr uint32_t make_idesc(uint32_t sf_id)
{
    const uint32_t fmt = kFmt == kFmtMXFP8 ? 0u : 1u;
    const uint32_t e8m0 = kFmt == kFmtNVFP4 ? 0u : 1u;
    return (sf_id << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(kBN >> 3) << 17) | (e8m0 << 23) |
           ((uint32_t)(kMmaM >> 4) << 24) | (sf_id << 29);
}

template <int kFmt>
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                       uint32_t accumulate)
{
    if constexpr (kFmt == kFmtNVFP4) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
            "}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
            : "memory");
    } else if constexpr (kFmt == kFmtMXFP8) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
            "}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
            "}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
            : "memory");
    }
}

#define TMEM_LD_32(taddr, r)                                                                       \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12," \
                 "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, "  \
                 "[%32];"                                                                          \
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),         \
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),       \
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]),   \
                   "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),   \
                   "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),   \
                   "=r"(r[30]), "=r"(r[31])                                                        \
                 : "r"(taddr))


__device__ __forceinline__ uint4 lds128(const void* p)
{
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(smem_addr(p)));
    return r;
}
#define TMEM_ST_16(taddr, v) asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr), "r"((v)[0]), "r"((v)[1]), "r"((v)[2]), "r"((v)[3]), "r"((v)[4]), "r"((v)[5]), "r"((v)[6]), "r"((v)[7]), "r"((v)[8]), "r"((v)[9]), "r"((v)[10]), "r"((v)[11]), "r"((v)[12]), "r"((v)[13]), "r"((v)[14]), "r"((v)[15]) : "memory")
#define TMEM_ST_32(taddr, v) asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr), "r"((v)[0]), "r"((v)[1]), "r"((v)[2]), "r"((v)[3]), "r"((v)[4]), "r"((v)[5]), "r"((v)[6]), "r"((v)[7]), "r"((v)[8]), "r"((v)[9]), "r"((v)[10]), "r"((v)[11]), "r"((v)[12]), "r"((v)[13]), "r"((v)[14]), "r"((v)[15]), "r"((v)[16]), "r"((v)[17]), "r"((v)[18]), "r"((v)[19]), "r"((v)[20]), "r"((v)[21]), "r"((v)[22]), "r"((v)[23]), "r"((v)[24]), "r"((v)[25]), "r"((v)[26]), "r"((v)[27]), "r"((v)[28]), "r"((v)[29]), "r"((v)[30]), "r"((v)[31]) : "memory")
#define TMEM_ST_8(taddr, v) asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"((v)[0]), "r"((v)[1]), "r"((v)[2]), "r"((v)[3]), "r"((v)[4]), "r"((v)[5]), "r"((v)[6]), "r"((v)[7]) : "memory")
#define TMEM_ST_4(taddr, v) asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"((v)[0]), "r"((v)[1]), "r"((v)[2]), "r"((v)[3]) : "memory")

// One lane's N consecutive 32-bit tensor-memory columns from v (warp-wide).
template <int N>
__device__ __forceinline__ void tmem_store_words(uint32_t taddr, const uint32_t* v)
{
    if constexpr (N == 48) {
        TMEM_ST_16(taddr, v);
        TMEM_ST_32(taddr + 16, (v + 16));
    } else if constexpr (N == 32) {
        TMEM_ST_32(taddr, v);
    } else if constexpr (N == 16) {
        TMEM_ST_16(taddr, v);
    } else if constexpr (N == 24) {
        TMEM_ST_16(taddr, v);
        TMEM_ST_8(taddr + 16, (v + 16));
    } else if constexpr (N == 12) {
        TMEM_ST_8(taddr, v);
        TMEM_ST_4(taddr + 8, (v + 8));
    } else if constexpr (N == 8) {
        TMEM_ST_8(taddr, v);
    } else {
        static_assert(N == 0, "unsupported scale-column count");
    }
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- scheduling
struct TileCoord {
    int group;       // expert (0 when dense)
    int64_t row0;    // first A row of the pair's 256-row tile
    int64_t row_end; // one past the last valid A row
    int64_t sf_blk;  // 128-row scale block of the tile's first half
    int64_t n0;
};

template <int kBN>
__device__ __forceinline__ TileCoord tile_coord(const GemmArgs& a, const GemmShared* sh, int t)
{
    TileCoord c;
    const int64_t tiles_n = (a.N + kBN - 1) / kBN;
    if (!a.grouped) {
        const int64_t tiles_m = (a.M + kMmaM - 1) / kMmaM;
        const int64_t band = 8 * tiles_n;  // 8 M tiles share a band: B tiles reused from L2
        const int64_t g = t / band, first_m = g * 8;
        const int64_t gm = min((int64_t)8, tiles_m - first_m);
        const int64_t r = t - g * band;
        const int64_t mt = first_m + r % gm, nt = r / gm;
        c.group = 0;
        c.row0 = mt * kMmaM;
        c.row_end = a.M;
        c.sf_blk = 2 * mt;
        c.n0 = nt * kBN;
    } else {
        int lo = 0, hi = a.G - 1;  // e with cum[e] <= t < cum[e+1]
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (sh->cum_tiles[mid] <= t)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int64_t local = t - sh->cum_tiles[lo];
        const int64_t mt = local / tiles_n, nt = local - mt * tiles_n;
        c.group = lo;
        c.row0 = sh->group_start[lo] + mt * kMmaM;
        c.row_end = sh->group_start[lo + 1];
        c.sf_blk = sh->group_sfblk[lo] + 2 * mt;
        c.n0 = nt * kBN;
    }
    return c;
}

// ---------------------------------------------------------------- kernel
template <int kFmt, int kBN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                const __grid_constant__ CUtensorMap map_sfb, GemmArgs a)
{
    using C = GemmCfg<kFmt, kBN>;
    constexpr int kS = C::kStages;
    constexpr int kAcc = C::kAccStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    GemmShared* sh = reinterpret_cast<GemmShared*>(smem + kS * C::kStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();  // 0: leader (issues the MMAs), 1: peer
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    uint8_t* epi_stage = smem + kS * C::kStageBytes + kSmemShared;
    const long long t_entry = clock64();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kS; ++s) {
            // leader: its producer's expect_tx (both CTAs' code bytes) and the 8 scale
            // writers of the pair (scales in tensor memory); peer: unused
            mbar_init(&sh->full[s], 9);
            mbar_init(&sh->sf_full[s], 1);   // this CTA's producer
            mbar_init(&sh->empty[s], 1);     // the leader's MMA commit, multicast to both
        }
        for (int b = 0; b < kAcc; ++b) {
            mbar_init(&sh->acc_full[b], 1);
            mbar_init(&sh->acc_empty[b], 2 * kEpiWarps);  // leader: epilogue warps of both CTAs
        }
        fence_barrier_init();
        // tile table (both CTAs compute the same one)
        const int64_t tiles_n = (a.N + kBN - 1) / kBN;
        if (!a.grouped) {
            sh->total_tiles = (int32_t)(((a.M + kMmaM - 1) / kMmaM) * tiles_n);
        } else {
            int32_t cum = 0, blk = 0;
            for (int e = 0; e <= a.G; ++e) {
                const int32_t st = a.group_offsets[e];
                sh->group_start[e] = st;
                sh->cum_tiles[e] = cum;
                sh->group_sfblk[e] = blk;
                if (e < a.G) {
                    const int32_t cnt = a.group_offsets[e + 1] - st;
                    const int32_t mt = cnt > 0 ? (cnt + kMmaM - 1) / kMmaM : 0;
                    cum += mt * (int32_t)tiles_n;
                    blk += cnt > 0 ? (cnt + BM - 1) / BM : 0;
                }
            }
            sh->total_tiles = cum;
        }
    }
    if (warp == 1) tmem_alloc_pair(&sh->tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers initialised and tensor memory allocated
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;
    const int total = sh->total_tiles;
    const int64_t kstages = a.K / C::kKStage;
    const int64_t k_atoms = a.K / C::kKAtom;  // scale atoms per 128-row block
    bool failed = false;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_b)) : "memory");
            if (kBN == 256)
                asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_sfb)) : "memory");
            const int64_t nblk = (a.N + 127) / 128;  // 128-row scale blocks per group of B
            uint32_t it = 0;
            for (int t = pair; t < total && !failed && !a.no_copies; t += n_pairs) {
                const TileCoord c = tile_coord<kBN>(a, sh, t);
                // This CTA's A rows; a half past the group's (or matrix's) end
                // reads rows it never stores, and the leader's scale block
                // instead of one that may not exist.
                const int64_t a_row = c.row0 + (int64_t)BM * rank;
                const int64_t sfa_blk = c.sf_blk + ((rank == 1 && a_row < c.row_end) ? 1 : 0);
                const int64_t b_row = (int64_t)c.group * a.N + c.n0 + (int64_t)C::kBRows * rank;
                const int64_t nb0 = c.n0 / 128;
                for (int64_t ks = 0; ks < kstages; ++ks, ++it) {
                    const int s = (int)(it % kS);
                    const uint32_t ph = (it / kS) & 1u;
                    if (!mbar_wait(&sh->empty[s], ph ^ 1u, a.wait_ns)) {
                        record_status(a.status, NVFP4_ERR_TIMEOUT);
                        failed = true;
                        break;
                    }
                    uint8_t* st = smem + s * C::kStageBytes;
                    // this CTA's scale atoms first (they land first, and the scale
                    // writers' work overlaps the code tiles' flight): kSfAtoms
                    // consecutive atoms per 128-row block
                    uint8_t* sf = st + C::kA_Bytes + C::kB_Bytes;
                    mbar_arrive_expect_tx(&sh->sf_full[s], C::kSFA_Bytes + C::kSFB_Bytes);
                    bulk_copy_g2s(sf, a.sfa + (sfa_blk * k_atoms + ks * C::kSfAtoms) * 512,
                                  C::kSFA_Bytes, &sh->sf_full[s]);
                    if constexpr (kBN == 256) {
                        // both 128-row blocks of B's scales in one box (a block past
                        // the operand's end reads as zeros)
                        tma_load_4d(sf + C::kSFA_Bytes, &map_sfb, 0, (int32_t)ks, (int32_t)nb0,
                                    c.group, &sh->sf_full[s]);
                    } else {
                        // the tile's one 128-row block (n0 is a multiple of 128 and
                        // below N, so the block exists)
                        bulk_copy_g2s(sf + C::kSFA_Bytes,
                                      a.sfb + (((int64_t)c.group * nblk + nb0) * k_atoms +
                                               ks * C::kSfAtoms) * 512,
                                      C::kSFB_Bytes, &sh->sf_full[s]);
                    }
                    if (leader) mbar_arrive_expect_tx(&sh->full[s], C::kPairCodeTx);
                    const uint32_t fb = cluster_addr(&sh->full[s], 0);
                    tma_load_2d_pair(st, &map_a, (int32_t)(ks * 128), (int32_t)a_row, fb);
                    tma_load_2d_pair(st + C::kA_Bytes, &map_b, (int32_t)(ks * 128), (int32_t)b_row, fb);
                }
            }
            // Drain: the last stages' copies have landed once their MMAs
            // completed (the CTA's shared memory must outlive them).
            const uint32_t first = it > (uint32_t)kS ? it - kS : 0u;
            for (uint32_t j = first; j < it; ++j)
                (void)mbar_wait(&sh->empty[j % kS], (j / kS) & 1u, a.wait_ns);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader CTA)
        if (leader && lane == 0) {
            uint32_t it = 0, tcount = 0;
            for (int t = pair; t < total && !failed; t += n_pairs, ++tcount) {
                const uint32_t buf = tcount % kAcc, aph = (tcount / kAcc) & 1u;
                // wait until both epilogues drained this accumulator's previous tile
                if (!mbar_wait(&sh->acc_empty[buf], aph ^ 1u, a.wait_ns)) {
                    record_status(a.status, NVFP4_ERR_TIMEOUT);
                    failed = true;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + buf * (uint32_t)kBN;
                for (int64_t ks = 0; ks < kstages; ++ks, ++it) {
                    const int s = (int)(it % kS);
                    const uint32_t ph = (it / kS) & 1u;
                    if (!mbar_wait(&sh->full[s], ph, a.wait_ns)) {  // codes landed, scales written
                        record_status(a.status, NVFP4_ERR_TIMEOUT);
                        failed = true;
                        break;
                    }
                    tc_fence_after();
                    uint8_t* st = smem + s * C::kStageBytes;
                    const uint32_t t_sfa = tmem + C::kTmemSF + (uint32_t)s * C::kSfStride;
                    const uint32_t t_sfb = t_sfa + C::kSfColsA;
                    const uint64_t ad = desc_sw128(st), bd = desc_sw128(st + C::kA_Bytes);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        // +32 bytes along K inside the swizzled row: 64 FP4 or 32 FP8
                        // elements.  NVFP4: atom j's columns; MXFP8: byte j of the
                        // stage's one atom; MXFP4: bytes 2(j%2), 2(j%2)+1 of atom j/2.
                        const uint32_t aj = kFmt == kFmtNVFP4 ? (uint32_t)j
                                            : kFmt == kFmtMXFP4 ? (uint32_t)(j >> 1) : 0u;
                        const uint32_t sf_id = kFmt == kFmtNVFP4 ? 0u
                                               : kFmt == kFmtMXFP4 ? 2u * (uint32_t)(j & 1)
                                                                   : (uint32_t)j;
                        tc_mma<kFmt>(d_tmem, ad + 2 * j, bd + 2 * j, make_idesc<kFmt, kBN>(sf_id),
                                     t_sfa + 4 * aj, t_sfb + 4 * C::kBlocksN * aj,
                                     (ks > 0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit_pair(&sh->empty[s]);  // both CTAs' stage free once these MMAs completed
                }
                if (failed) break;
                tc_commit_pair(&sh->acc_full[buf]);
            }
        }
    } else if (warp < 6) {
        // ------------------------------------------------ scale writers (warps 2..5, both CTAs)
        // Each warp writes its lane quadrant of the stage's scale columns in
        // this CTA's tensor memory with tcgen05.st: lane i gets row i of every
        // 512-byte atom (the layout a broadcast copy would produce in each
        // quadrant).  Completion is reported to the leader, whose MMAs read
        // both CTAs' scales.
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        uint32_t it = 0;
        for (int t = pair; t < total && !failed; t += n_pairs) {
            for (int64_t ks = 0; ks < kstages; ++ks, ++it) {
                const int s = (int)(it % kS);
                const uint32_t ph = (it / kS) & 1u;
                bool ok = true;
                if (lane == 0) ok = mbar_wait(&sh->sf_full[s], ph, a.wait_ns);
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) {
                    if (lane == 0) record_status(a.status, NVFP4_ERR_TIMEOUT);
                    failed = true;
                    break;
                }
                const uint8_t* sfa_s = smem + s * C::kStageBytes + C::kA_Bytes + C::kB_Bytes;
                const uint8_t* sfb_s = sfa_s + C::kSFA_Bytes;  // [block][atom][512]
                uint32_t v[C::kSfCols];
#pragma unroll
                for (int j = 0; j < C::kSfAtoms; ++j) {
                    const uint4 x = lds128(sfa_s + j * 512 + lane * 16);
                    v[4 * j] = x.x, v[4 * j + 1] = x.y, v[4 * j + 2] = x.z, v[4 * j + 3] = x.w;
#pragma unroll
                    for (int bb = 0; bb < C::kBlocksN; ++bb) {
                        const uint4 y = lds128(sfb_s + (bb * C::kSfAtoms + j) * 512 + lane * 16);
                        const int o = C::kSfColsA + 4 * (j * C::kBlocksN + bb);
                        v[o] = y.x, v[o + 1] = y.y, v[o + 2] = y.z, v[o + 3] = y.w;
                    }
                }
                tmem_store_words<C::kSfCols>(tmem + lane_base + C::kTmemSF + (uint32_t)s * C::kSfStride, v);
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(cluster_addr(&sh->full[s], 0));
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 6..13, both CTAs)
        constexpr int kCols = kBN / (kEpiWarps / 4);  // accumulator columns per warp
        constexpr int kChunks = kCols / 32;
        const int quad = warp & 3;                   // TMEM lanes 32*quad .. 32*quad+31
        const int col0 = ((warp - 6) >> 2) * kCols;
        uint8_t* stg = epi_stage + (warp - 6) * kEpiStageBytes;
        float out_max = 0.0f;                            // max |D| stored by this thread
        uint32_t tcount = 0;
        for (int t = pair; t < total; t += n_pairs, ++tcount) {
            const TileCoord c = tile_coord<kBN>(a, sh, t);
            const uint32_t buf = tcount % kAcc, aph = (tcount / kAcc) & 1u;
            const bool ok = mbar_wait(&sh->acc_full[buf], aph, a.wait_ns);
            if (!ok) {
                if (lane == 0) record_status(a.status, NVFP4_ERR_TIMEOUT);
                break;
            }
            tc_fence_after();
            const uint32_t tbase =
                tmem + ((uint32_t)(32 * quad) << 16) + buf * (uint32_t)kBN + (uint32_t)col0;
            const float alpha = kFmt == kFmtNVFP4 ? __fmul_rn(a.ga[0], a.gb[c.group]) : 1.0f;
            const int64_t row = c.row0 + (int64_t)BM * rank + 32 * quad + lane;
            const bool row_ok = row < c.row_end;
            if (a.bf16_out) {
                // kCols columns in 32-column loads, converted to bf16 pairs as they
                // arrive (two loads in flight per wait for 64-column warps): the
                // accumulator is released before any store.
                uint32_t packed[16 * kChunks];
                constexpr int kPer = (kChunks == 2 && kEpiWarps == 8) ? 2 : 1;
#pragma unroll
                for (int hh = 0; hh < kChunks; hh += kPer) {
                    uint32_t r[32 * kPer];
#pragma unroll
                    for (int q = 0; q < kPer; ++q) TMEM_LD_32(tbase + 32 * (hh + q), (r + 32 * q));
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16 * kPer; ++i) {
                        float x0, x1;  // two IEEE products, as two __fmul_rn
                        mul2(x0, x1, __uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]), alpha, alpha);
                        const __nv_bfloat162 p = __floats2bfloat162_rn(x0, x1);
                        packed[16 * hh + i] = *reinterpret_cast<const uint32_t*>(&p);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(cluster_addr(&sh->acc_empty[buf], 0));  // accumulator drained
                const int64_t cbase = c.n0 + col0;
                // max |D| of this lane's stored (rounded) values, after the accumulator
                // is released: only when asked for, and off the drain's critical path
                if (a.amax_out && row_ok) {
#pragma unroll
                    for (int g = 0; g < 4 * kChunks; ++g)
                        if (cbase + 8 * g < a.N) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const uint32_t w = packed[4 * g + i];
                                out_max = absmax3(out_max, __uint_as_float(w << 16),
                                                  __uint_as_float(w & 0xFFFF0000u));
                            }
                        }
                }
                const int64_t rowbase = c.row0 + (int64_t)BM * rank + 32 * quad;
                // 32-column chunks through a 64-byte-swizzled 32x64-byte staging
                // block: each lane writes its row, then 8 rows x 64 bytes leave
                // per store instruction (whole 32-byte sectors).
#pragma unroll
                for (int hh = 0; hh < kChunks; ++hh) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        st_shared_v4(stg + lane * 64 + 16 * (q ^ ((lane >> 1) & 3)),
                                     make_uint4(packed[16 * hh + 4 * q], packed[16 * hh + 4 * q + 1],
                                                packed[16 * hh + 4 * q + 2], packed[16 * hh + 4 * q + 3]));
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = 8 * i + (lane >> 2), q = lane & 3;
                        const uint4 v = lds128(stg + r * 64 + 16 * (q ^ ((r >> 1) & 3)));
                        const int64_t grow = rowbase + r, col = cbase + 32 * hh + 8 * q;
                        if (grow < c.row_end && col < a.N)
                            *reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.D) + grow * a.ldd + col) = v;
                    }
                    __syncwarp();
                }
                continue;
            }
            // FP32 output: rounds of 32 columns, each stored before the next
            // load; the accumulator is released after the last load.
#pragma unroll 1
            for (int hh = 0; hh < kChunks; ++hh) {
                uint32_t r[32];
                TMEM_LD_32(tbase + 32 * hh, r);
                tmem_ld_wait();
                if (hh == kChunks - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(cluster_addr(&sh->acc_empty[buf], 0));  // accumulator drained
                }
                if (!row_ok) continue;
                const int64_t cbase = c.n0 + col0 + 32 * hh;
                float* drow = static_cast<float*>(a.D) + row * a.ldd + cbase;
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    const float x0 = __fmul_rn(__uint_as_float(r[4 * v]), alpha);
                    const float x1 = __fmul_rn(__uint_as_float(r[4 * v + 1]), alpha);
                    const float x2 = __fmul_rn(__uint_as_float(r[4 * v + 2]), alpha);
                    const float x3 = __fmul_rn(__uint_as_float(r[4 * v + 3]), alpha);
                    if (cbase + 4 * v < a.N) {
                        *reinterpret_cast<float4*>(drow + 4 * v) = make_float4(x0, x1, x2, x3);
                        out_max = absmax3(out_max, absmax3(x0, x1, x2), x3);
                    }
                }
            }
        }
        // max |D| over this thread's stored values -> one atomic per warp.  For
        // bf16 output the max is rounded like the values were: rounding is
        // monotonic, so that is the max of the stored values.
        if (a.amax_out) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) out_max = fmaxf(out_max, __shfl_xor_sync(0xffffffffu, out_max, o));
            if (a.bf16_out) out_max = __bfloat162float(__float2bfloat16_rn(out_max));
            if (lane == 0) atomicMax(reinterpret_cast<uint32_t*>(a.amax_out), __float_as_uint(out_max));
        }
    }

    // Neither CTA leaves (or frees the pair's tensor memory) before both are done.
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
    if (threadIdx.x == 0) atomicMax(a.cycles, (unsigned long long)(clock64() - t_entry));
}

// ---------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_tiled()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, []() {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// [rows, kbytes] uint8 matrix, box 128 bytes x box_rows, 128-byte swizzle.
static bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t kbytes, int box_rows)
{
    auto fn = encode_tiled();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)kbytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)kbytes};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// B's scales in the tensor-core layout, [G][nblk][k_atoms][512 bytes], seen
// as 8-byte elements: {one K stage's atoms, K stages, nblk, G}; a box is one
// stage of two consecutive row blocks (the 256-wide tile).
static bool make_sfb_map(CUtensorMap* m, const void* sfb, int64_t G, int64_t N, int64_t K,
                         int k_stage, int k_atom, int stage_atoms)
{
    auto fn = encode_tiled();
    if (!fn) return false;
    const int64_t nblk = (N + 127) / 128, k_atoms = K / k_atom;
    const cuuint32_t inner = (cuuint32_t)(stage_atoms * 64);  // 8-byte elements per stage
    cuuint64_t dims[4] = {inner, (cuuint64_t)(K / k_stage), (cuuint64_t)nblk, (cuuint64_t)G};
    cuuint64_t strides[3] = {(cuuint64_t)stage_atoms * 512u, (cuuint64_t)(k_atoms * 512),
                             (cuuint64_t)(nblk * k_atoms * 512)};
    cuuint32_t box[4] = {inner, 1u, 2u, 1u};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 4, const_cast<void*>(sfb), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct GemmDevice {
    int sms = 0;
    int pairs = 0;  // CTA pairs that are resident at once
    bool ok = false;
};

template <int kFmt, int kBN>
static GemmDevice& gemm_device(int dev)
{
    static GemmDevice infos[64];
    static std::once_flag flags[64];
    std::call_once(flags[dev & 63], [dev]() {
        GemmDevice& d = infos[dev & 63];
        using C = GemmCfg<kFmt, kBN>;
        auto fn = gemm_kernel<kFmt, kBN>;
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess || prop.major != 10) return;
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)C::kSmemBytes) != cudaSuccess)
            return;
        d.sms = prop.multiProcessorCount;
        // Pairs need two SMs of one cluster-capable group: ask how many fit
        // at once, so that the persistent grid never waits for a second wave.
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(d.sms & ~1));
        cfg.blockDim = dim3(kGemmThreads);
        cfg.dynamicSmemBytes = C::kSmemBytes;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, fn, &cfg) != cudaSuccess || clusters < 1)
            return;
        d.pairs = std::min(clusters, d.sms / 2);
        d.ok = true;
    });
    return infos[dev & 63];
}

static bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kGemmWorkspace = 256;

// Output-tile width.  256 (one accumulator) moves the fewest operand bytes per
// FLOP; 128 (two accumulators) hides the epilogue's drain but moves 1.5x the
// operand bytes per FLOP, and measured 30-45% slower on every shape of the
// workloads (dense, grouped, MXFP8), so 256 is the default.
// NVFP4_GEMM_TILE_N=128 or 256 in the environment overrides the choice (read
// on every call).
static int pick_tile_n(bool grouped, int64_t K, int k_stage)
{
    if (const char* e = getenv("NVFP4_GEMM_TILE_N")) {
        if (!strcmp(e, "128")) return 128;
        if (!strcmp(e, "256")) return 256;
    }
    (void)grouped;
    (void)K;
    (void)k_stage;
    return 256;  // measured faster for every shape of the workloads, dense and grouped
}

template <int kFmt, int kBN>
static nvfp4_status launch_variant(const void* qa, const void* qb, GemmArgs& a, int64_t a_rows,
                                   int64_t b_rows, int64_t max_tiles_m, cudaStream_t st)
{
    using C = GemmCfg<kFmt, kBN>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    wait_test_hook(&a.wait_ns, &a.no_copies);
    GemmDevice& info = gemm_device<kFmt, kBN>(dev);
    if (!info.ok) return NVFP4_ERR_UNSUPPORTED;
    const int64_t kbytes = kFmt == kFmtMXFP8 ? a.K : a.K / 2;
    CUtensorMap ma, mb, msf;
    memset(&msf, 0, sizeof(msf));
    if (!make_map(&ma, qa, a_rows, kbytes, BM) || !make_map(&mb, qb, b_rows, kbytes, C::kBRows))
        return NVFP4_ERR_CUDA;
    if (kBN == 256 &&
        !make_sfb_map(&msf, a.sfb, a.G, a.N, a.K, C::kKStage, C::kKAtom, C::kSfAtoms))
        return NVFP4_ERR_CUDA;
    // the status word and the cycle count report this call only; the output amax starts at 0
    if (cudaMemsetAsync(a.status, 0, 16, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (a.amax_out && cudaMemsetAsync(a.amax_out, 0, 4, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    const int64_t tiles = max_tiles_m * ((a.N + kBN - 1) / kBN);
    const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, info.pairs));
    gemm_kernel<kFmt, kBN><<<2 * pairs, kGemmThreads, C::kSmemBytes, st>>>(ma, mb, msf, a);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

template <int kFmt>
static nvfp4_status launch_gemm(const void* qa, const void* qb, GemmArgs& a, int64_t a_rows,
                                int64_t b_rows, int64_t max_tiles_m, cudaStream_t st)
{
    if (pick_tile_n(a.grouped != 0, a.K, GemmCfg<kFmt, 256>::kKStage) == 128)
        return launch_variant<kFmt, 128>(qa, qb, a, a_rows, b_rows, max_tiles_m, st);
    return launch_variant<kFmt, 256>(qa, qb, a, a_rows, b_rows, max_tiles_m, st);
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" size_t nvfp4_gemm_workspace_size(int64_t, int64_t, int64_t) { return kGemmWorkspace; }

// SM clock cycles, from entry to exit, of the longest-running CTA of the last
// GEMM call given this workspace (bytes 16..23).  Divided by the call's
// CUDA-event time it gives the SM clock the call ran at.
extern "C" nvfp4_status nvfp4_gemm_cycles(void* workspace, void* stream, uint64_t* cycles)
{
    if (!workspace || !cycles) return NVFP4_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned long long v = 0;
    const unsigned long long* src = static_cast<const unsigned long long*>(workspace) + 2;
    if (cudaMemcpyAsync(&v, src, 8, cudaMemcpyDeviceToHost, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return NVFP4_ERR_CUDA;
    *cycles = v;
    return NVFP4_OK;
}

// Checks shared by the dense GEMMs; k_mult is the K granularity of a stage.
static nvfp4_status check_dense(const uint8_t* qa, const uint8_t* sfa, const uint8_t* qb,
                                const uint8_t* sfb, int64_t M, int64_t N, int64_t K, int64_t k_mult,
                                int out_dtype, void* D, int64_t ldd, float* amax_out,
                                void* workspace, size_t ws_bytes)
{
    if (!qa || !sfa || !qb || !sfb || !D) return NVFP4_ERR_INVALID_ARG;
    if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0 || M % 16 || N % 16 || K % k_mult || ldd < N) return NVFP4_ERR_SHAPE;
    if (M > (int64_t)1 << 31 || N > (int64_t)1 << 31) return NVFP4_ERR_SHAPE;
    const int esz = out_dtype == NVFP4_OUT_BF16 ? 2 : 4;
    if (!al16(qa) || !al16(qb) || !al16(sfa) || !al16(sfb) || !al16(D) || (ldd * esz) % 16 ||
        (reinterpret_cast<uintptr_t>(amax_out) & 3u))
        return NVFP4_ERR_ALIGN;
    if (!workspace || ws_bytes < kGemmWorkspace) return NVFP4_ERR_WORKSPACE;
    if (!al16(workspace)) return NVFP4_ERR_ALIGN;
    return NVFP4_OK;
}

extern "C" nvfp4_status nvfp4_gemm(const uint8_t* qa, const uint8_t* sfa, const float* ga,
                                   const uint8_t* qb, const uint8_t* sfb, const float* gb,
                                   int64_t M, int64_t N, int64_t K, int out_dtype, void* D,
                                   int64_t ldd, float* amax_out, void* workspace, size_t ws_bytes,
                                   void* stream)
{
    if (!ga || !gb) return NVFP4_ERR_INVALID_ARG;
    const nvfp4_status chk = check_dense(qa, sfa, qb, sfb, M, N, K, 256, out_dtype, D, ldd,
                                         amax_out, workspace, ws_bytes);
    if (chk != NVFP4_OK) return chk;
    GemmArgs a{};
    a.sfa = sfa;
    a.sfb = sfb;
    a.ga = ga;
    a.gb = gb;
    a.D = D;
    a.M = M;
    a.N = N;
    a.K = K;
    a.ldd = ldd;
    a.bf16_out = out_dtype == NVFP4_OUT_BF16;
    a.grouped = 0;
    a.G = 1;
    a.status = static_cast<uint32_t*>(workspace) + 2;
    a.cycles = static_cast<unsigned long long*>(workspace) + 2;
    a.amax_out = amax_out;
    return launch_gemm<kFmtNVFP4>(qa, qb, a, M, N, (M + kMmaM - 1) / kMmaM,
                                  static_cast<cudaStream_t>(stream));
}

extern "C" nvfp4_status mxfp8_gemm(const uint8_t* qa, const uint8_t* sfa, const uint8_t* qb,
                                   const uint8_t* sfb, int64_t M, int64_t N, int64_t K,
                                   int out_dtype, void* D, int64_t ldd, float* amax_out,
                                   void* workspace, size_t ws_bytes, void* stream)
{
    const nvfp4_status chk = check_dense(qa, sfa, qb, sfb, M, N, K, 128, out_dtype, D, ldd,
                                         amax_out, workspace, ws_bytes);
    if (chk != NVFP4_OK) return chk;
    GemmArgs a{};
    a.sfa = sfa;
    a.sfb = sfb;
    a.D = D;
    a.M = M;
    a.N = N;
    a.K = K;
    a.ldd = ldd;
    a.bf16_out = out_dtype == NVFP4_OUT_BF16;
    a.grouped = 0;
    a.G = 1;
    a.status = static_cast<uint32_t*>(workspace) + 2;
    a.cycles = static_cast<unsigned long long*>(workspace) + 2;
    a.amax_out = amax_out;
    return launch_gemm<kFmtMXFP8>(qa, qb, a, M, N, (M + kMmaM - 1) / kMmaM,
                                  static_cast<cudaStream_t>(stream));
}

extern "C" nvfp4_status mxfp4_gemm(const uint8_t* qa, const uint8_t* sfa, const uint8_t* qb,
                                   const uint8_t* sfb, int64_t M, int64_t N, int64_t K,
                                   int out_dtype, void* D, int64_t ldd, float* amax_out,
                                   void* workspace, size_t ws_bytes, void* stream)
{
    const nvfp4_status chk = check_dense(qa, sfa, qb, sfb, M, N, K, 256, out_dtype, D, ldd,
                                         amax_out, workspace, ws_bytes);
    if (chk != NVFP4_OK) return chk;
    GemmArgs a{};
    a.sfa = sfa;
    a.sfb = sfb;
    a.D = D;
    a.M = M;
    a.N = N;
    a.K = K;
    a.ldd = ldd;
    a.bf16_out = out_dtype == NVFP4_OUT_BF16;
    a.grouped = 0;
    a.G = 1;
    a.status = static_cast<uint32_t*>(workspace) + 2;
    a.cycles = static_cast<unsigned long long*>(workspace) + 2;
    a.amax_out = amax_out;
    return launch_gemm<kFmtMXFP4>(qa, qb, a, M, N, (M + kMmaM - 1) / kMmaM,
                                  static_cast<cudaStream_t>(stream));
}

extern "C" nvfp4_status nvfp4_grouped_gemm(int G, const int32_t* group_offsets, int64_t total_rows,
                                           const uint8_t* qa, const uint8_t* sfa, const float* ga,
                                           const uint8_t* qb, const uint8_t* sfb, const float* gb,
                                           int64_t N, int64_t K, int out_dtype, void* D,
                                           float* amax_out, void* workspace, size_t ws_bytes,
                                           void* stream)
{
    if (G < 1 || G > kMaxGemmGroups || !group_offsets || !qa || !sfa || !ga || !qb || !sfb ||
        !gb || !D)
        return NVFP4_ERR_INVALID_ARG;
    if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
    if (total_rows <= 0 || N <= 0 || K <= 0 || N % 128 || K % 256) return NVFP4_ERR_SHAPE;
    if (total_rows > (int64_t)1 << 31 || (int64_t)G * N > (int64_t)1 << 31) return NVFP4_ERR_SHAPE;
    if (!al16(qa) || !al16(qb) || !al16(sfa) || !al16(sfb) || !al16(D) ||
        (reinterpret_cast<uintptr_t>(amax_out) & 3u))
        return NVFP4_ERR_ALIGN;
    if (!workspace || ws_bytes < kGemmWorkspace) return NVFP4_ERR_WORKSPACE;
    if (!al16(workspace)) return NVFP4_ERR_ALIGN;
    GemmArgs a{};
    a.sfa = sfa;
    a.sfb = sfb;
    a.ga = ga;
    a.gb = gb;
    a.D = D;
    a.M = total_rows;
    a.N = N;
    a.K = K;
    a.ldd = N;
    a.bf16_out = out_dtype == NVFP4_OUT_BF16;
    a.grouped = 1;
    a.G = G;
    a.group_offsets = group_offsets;
    a.total_rows = total_rows;
    a.status = static_cast<uint32_t*>(workspace) + 2;
    a.cycles = static_cast<unsigned long long*>(workspace) + 2;
    a.amax_out = amax_out;
    // upper bound on M tiles: every group may add one partial tile
    return launch_gemm<kFmtNVFP4>(qa, qb, a, total_rows, (int64_t)G * N,
                                  (total_rows + kMmaM - 1) / kMmaM + G,
                                  static_cast<cudaStream_t>(stream));
}
