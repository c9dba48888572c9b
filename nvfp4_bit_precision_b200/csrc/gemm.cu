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
//               memory with tcgen05.st, then reports to the leader.  The
//               tensor pipe spends no cycles on scale copies.
//   warp 1      leader CTA only: one elected thread waits for a stage's tiles
//               and both CTAs' scales and issues 4 MMAs of 256x256x64, then
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
#include <mutex>

#include "common.cuh"

namespace nvfp4 {

constexpr int BM = 128;                    // A rows per CTA; a CTA pair covers 2 * BM
constexpr int kMmaM = 2 * BM;              // M of the two-SM MMA
constexpr int BN = 256;                    // output columns per tile
constexpr int BK = 256;                    // elements per stage (128 bytes per row)
constexpr int kGemmStages = 5;
constexpr int kA_Bytes = BM * BK / 2;          // 16 KB
constexpr int kB_Bytes = (BN / 2) * BK / 2;    // 16 KB: this CTA's half of the B tile
constexpr int kSFA_Bytes = BM * BK / 16;       // 2 KB: 4 atoms of 512 B (this CTA's rows)
constexpr int kSFB_Bytes = BN * BK / 16;       // 4 KB: 2 row blocks x 4 atoms (all of B)
constexpr int kStageBytes = kA_Bytes + kB_Bytes + kSFA_Bytes + kSFB_Bytes;
constexpr uint32_t kPairCodeTx = 2u * (kA_Bytes + kB_Bytes);  // the leader's full barrier
constexpr int kGemmThreads = 448;  // producer, MMA, 4 scale writers, 8 epilogue warps
// Tensor memory: the 128x256 FP32 accumulator in columns 0..255, then one
// 48-column scale region per pipeline stage (SFA 4 x 4 columns, SFB 4 x 8).
// Within a region, column 4j + c of every lane quadrant holds, in lane i, the
// four scales of row 32c + i for K-group j (SFA) -- row i of the K-group's
// 512-byte atom; SFB keeps rows 0..127 at 16 + 8j + c, rows 128..255 at
// 16 + 8j + 4 + c.
constexpr int kTmemCols = 512;
constexpr int kTmemSF = 256;
constexpr int kTmemSFStage = 48;
static_assert(kTmemSF + kGemmStages * kTmemSFStage <= kTmemCols, "tensor memory overflow");
constexpr int kMaxGemmGroups = 256;
constexpr int kEpiStageBytes = 2048;  // per epilogue warp: 32 rows x 64 bytes of BF16

struct GemmArgs {
    const uint8_t* sfa;
    const uint8_t* sfb;
    const float* ga;
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
    float* amax_out;  // optional: max |D| (as stored), atomically accumulated
};

struct GemmShared {
    uint64_t full[kGemmStages];      // leader: A/B codes of both CTAs landed
    uint64_t sf_full[kGemmStages];   // this CTA's scale atoms landed
    uint64_t empty[kGemmStages];     // the stage's MMAs completed (both CTAs)
    uint64_t sf_ready[kGemmStages];  // leader: both CTAs' scales are in tensor memory
    uint64_t acc_full;
    uint64_t acc_empty;
    uint32_t tmem_base;
    int32_t total_tiles;
    int32_t cum_tiles[kMaxGemmGroups + 1];
    int32_t group_start[kMaxGemmGroups + 1];
    int32_t group_sfblk[kMaxGemmGroups + 1];  // first padded 128-row scale block of a group
};

constexpr int kSmemShared = (int)((sizeof(GemmShared) + 1023) / 1024 * 1024);

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

// Instruction descriptor: kind::mxf4nvf4, A/B E2M1 (format 1), UE4M3 scales,
// both K-major, M = 256 (the pair), N = 256, dense, K = 64 per instruction.
__host__ __device__ constexpr uint32_t make_idesc()
{
    return (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kMmaM >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                       uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
        "}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
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
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- scheduling
struct TileCoord {
    int group;       // expert (0 when dense)
    int64_t row0;    // first A row of the pair's 256-row tile
    int64_t row_end; // one past the last valid A row
    int64_t sf_blk;  // 128-row scale block of the tile's first half
    int64_t n0;
};

__device__ __forceinline__ TileCoord tile_coord(const GemmArgs& a, const GemmShared* sh, int t)
{
    TileCoord c;
    const int64_t tiles_n = (a.N + BN - 1) / BN;
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
        c.n0 = nt * BN;
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
        c.n0 = nt * BN;
    }
    return c;
}

// ---------------------------------------------------------------- kernel
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                const __grid_constant__ CUtensorMap map_sfb, GemmArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    GemmShared* sh = reinterpret_cast<GemmShared*>(smem + kGemmStages * kStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();  // 0: leader (issues the MMAs), 1: peer
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    uint8_t* epi_stage = smem + kGemmStages * kStageBytes + kSmemShared;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(&sh->full[s], 1);      // leader: its producer's expect_tx; peer: unused
            mbar_init(&sh->sf_full[s], 1);   // this CTA's producer
            mbar_init(&sh->empty[s], 1);     // the leader's MMA commit, multicast to both
            mbar_init(&sh->sf_ready[s], 8);  // leader: 4 scale writers of each CTA
        }
        mbar_init(&sh->acc_full, 1);
        mbar_init(&sh->acc_empty, 16);       // leader: 8 epilogue warps of each CTA
        fence_barrier_init();
        // tile table (both CTAs compute the same one)
        const int64_t tiles_n = (a.N + BN - 1) / BN;
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
    const int64_t kstages = a.K / BK;
    const int64_t k64 = a.K / 64;  // scale atoms per 128-row block
    bool failed = false;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_b)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_sfb)) : "memory");
            uint32_t it = 0;
            for (int t = pair; t < total && !failed; t += n_pairs) {
                const TileCoord c = tile_coord(a, sh, t);
                // This CTA's A rows; a half past the group's (or matrix's) end
                // reads rows it never stores, and the leader's scale block
                // instead of one that may not exist.
                const int64_t a_row = c.row0 + (int64_t)BM * rank;
                const int64_t sfa_blk = c.sf_blk + ((rank == 1 && a_row < c.row_end) ? 1 : 0);
                const int64_t b_row = (int64_t)c.group * a.N + c.n0 + (int64_t)(BN / 2) * rank;
                const int64_t nb0 = c.n0 / 128;
                for (int64_t ks = 0; ks < kstages; ++ks, ++it) {
                    const int s = (int)(it % kGemmStages);
                    const uint32_t ph = (it / kGemmStages) & 1u;
                    if (!mbar_wait(&sh->empty[s], ph ^ 1u)) {
                        record_status(a.status, NVFP4_ERR_TIMEOUT);
                        failed = true;
                        break;
                    }
                    uint8_t* st = smem + s * kStageBytes;
                    // this CTA's scale atoms first (they land first, and the scale
                    // writers' work overlaps the code tiles' flight): 4 consecutive
                    // atoms (2 KB) per 128-row block
                    uint8_t* sf = st + kA_Bytes + kB_Bytes;
                    mbar_arrive_expect_tx(&sh->sf_full[s], kSFA_Bytes + kSFB_Bytes);
                    bulk_copy_g2s(sf, a.sfa + (sfa_blk * k64 + ks * 4) * 512, kSFA_Bytes, &sh->sf_full[s]);
                    // both 128-row blocks of B's scales in one box (a block past
                    // the operand's end reads as zeros)
                    tma_load_4d(sf + kSFA_Bytes, &map_sfb, 0, (int32_t)ks, (int32_t)nb0, c.group,
                                &sh->sf_full[s]);
                    if (leader) mbar_arrive_expect_tx(&sh->full[s], kPairCodeTx);
                    const uint32_t fb = cluster_addr(&sh->full[s], 0);
                    tma_load_2d_pair(st, &map_a, (int32_t)(ks * (BK / 2)), (int32_t)a_row, fb);
                    tma_load_2d_pair(st + kA_Bytes, &map_b, (int32_t)(ks * (BK / 2)), (int32_t)b_row, fb);
                }
            }
            // Drain: the last stages' copies have landed once their MMAs
            // completed (the CTA's shared memory must outlive them).
            const uint32_t first = it > (uint32_t)kGemmStages ? it - kGemmStages : 0u;
            for (uint32_t j = first; j < it; ++j)
                (void)mbar_wait(&sh->empty[j % kGemmStages], (j / kGemmStages) & 1u);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader CTA)
        if (leader && lane == 0) {
            const uint32_t idesc = make_idesc();
            uint32_t it = 0, tcount = 0;
            for (int t = pair; t < total && !failed; t += n_pairs, ++tcount) {
                // wait until both epilogues drained the accumulator of the previous tile
                if (!mbar_wait(&sh->acc_empty, (tcount & 1u) ^ 1u)) {
                    record_status(a.status, NVFP4_ERR_TIMEOUT);
                    failed = true;
                    break;
                }
                tc_fence_after();
                for (int64_t ks = 0; ks < kstages; ++ks, ++it) {
                    const int s = (int)(it % kGemmStages);
                    const uint32_t ph = (it / kGemmStages) & 1u;
                    if (!mbar_wait(&sh->full[s], ph) || !mbar_wait(&sh->sf_ready[s], ph)) {
                        record_status(a.status, NVFP4_ERR_TIMEOUT);
                        failed = true;
                        break;
                    }
                    tc_fence_after();
                    uint8_t* st = smem + s * kStageBytes;
                    const uint32_t t_sfa = tmem + kTmemSF + (uint32_t)s * kTmemSFStage;
                    const uint32_t t_sfb = t_sfa + 16;
                    const uint64_t ad = desc_sw128(st), bd = desc_sw128(st + kA_Bytes);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        // +32 bytes (64 four-bit elements) along K inside the swizzled row
                        tc_mma(tmem, ad + 2 * j, bd + 2 * j, idesc, t_sfa + 4 * j, t_sfb + 8 * j,
                               (ks > 0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit_pair(&sh->empty[s]);  // both CTAs' stage free once these MMAs completed
                }
                if (failed) break;
                tc_commit_pair(&sh->acc_full);
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
                const int s = (int)(it % kGemmStages);
                const uint32_t ph = (it / kGemmStages) & 1u;
                bool ok = true;
                if (lane == 0) ok = mbar_wait(&sh->sf_full[s], ph);
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) {
                    if (lane == 0) record_status(a.status, NVFP4_ERR_TIMEOUT);
                    failed = true;
                    break;
                }
                const uint8_t* sfa_s = smem + s * kStageBytes + kA_Bytes + kB_Bytes;
                const uint8_t* sfb_s = sfa_s + kSFA_Bytes;
                uint32_t v[48];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 x = lds128(sfa_s + j * 512 + lane * 16);
                    v[4 * j] = x.x, v[4 * j + 1] = x.y, v[4 * j + 2] = x.z, v[4 * j + 3] = x.w;
                    const uint4 lo = lds128(sfb_s + j * 512 + lane * 16);
                    const uint4 hi = lds128(sfb_s + kSFB_Bytes / 2 + j * 512 + lane * 16);
                    v[16 + 8 * j] = lo.x, v[17 + 8 * j] = lo.y, v[18 + 8 * j] = lo.z, v[19 + 8 * j] = lo.w;
                    v[20 + 8 * j] = hi.x, v[21 + 8 * j] = hi.y, v[22 + 8 * j] = hi.z, v[23 + 8 * j] = hi.w;
                }
                const uint32_t taddr = tmem + lane_base + kTmemSF + (uint32_t)s * kTmemSFStage;
                TMEM_ST_16(taddr, v);
                TMEM_ST_32(taddr + 16, (v + 16));
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(cluster_addr(&sh->sf_ready[s], 0));
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 6..13, both CTAs)
        const int quad = warp & 3;                   // TMEM lanes 32*quad .. 32*quad+31
        const int col0 = ((warp - 6) >> 2) * (BN / 2);  // 0 or 128
        const uint32_t acc_empty_leader = cluster_addr(&sh->acc_empty, 0);
        uint8_t* stg = epi_stage + (warp - 6) * kEpiStageBytes;
        float out_max = 0.0f;                            // max |D| stored by this thread
        uint32_t tcount = 0;
        for (int t = pair; t < total; t += n_pairs, ++tcount) {
            const TileCoord c = tile_coord(a, sh, t);
            const bool ok = mbar_wait(&sh->acc_full, tcount & 1u);
            if (!ok) {
                if (lane == 0) record_status(a.status, NVFP4_ERR_TIMEOUT);
                break;
            }
            tc_fence_after();
            const uint32_t tbase = tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)col0;
            const float alpha = __fmul_rn(a.ga[0], a.gb[c.group]);
            const int64_t row = c.row0 + (int64_t)BM * rank + 32 * quad + lane;
            const bool row_ok = row < c.row_end;
            if (a.bf16_out) {
                // 128 columns in four 32-column loads, each converted to bf16
                // pairs at once: the accumulator is released before any store
                // with at most 32 + 64 registers of data live.
                uint32_t packed[64];
                float m_all = 0.0f;  // max |x| over the 128 columns (before rounding)
#pragma unroll
                for (int hh = 0; hh < 4; ++hh) {
                    uint32_t r[32];
                    TMEM_LD_32(tbase + 32 * hh, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float x0 = __fmul_rn(__uint_as_float(r[2 * i]), alpha);
                        const float x1 = __fmul_rn(__uint_as_float(r[2 * i + 1]), alpha);
                        m_all = absmax3(m_all, x0, x1);
                        const __nv_bfloat162 p = __floats2bfloat162_rn(x0, x1);
                        packed[16 * hh + i] = *reinterpret_cast<const uint32_t*>(&p);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acc_empty_leader);  // accumulator drained
                const int64_t cbase = c.n0 + col0;
                // max |D| of this lane's row (rounded values where the N tail cuts the row)
                if (row_ok) {
                    if (cbase + 128 <= a.N) {
                        out_max = fmaxf(out_max, m_all);
                    } else {
#pragma unroll
                        for (int g = 0; g < 16; ++g)
                            if (cbase + 8 * g < a.N) {
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    const uint32_t w = packed[4 * g + i];
                                    out_max = absmax3(out_max, __uint_as_float(w << 16),
                                                      __uint_as_float(w & 0xFFFF0000u));
                                }
                            }
                    }
                }
                const int64_t rowbase = c.row0 + (int64_t)BM * rank + 32 * quad;
                // 32-column chunks through a 64-byte-swizzled 32x64-byte staging
                // block: each lane writes its row, then 8 rows x 64 bytes leave
                // per store instruction (whole 32-byte sectors).
#pragma unroll
                for (int hh = 0; hh < 4; ++hh) {
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
            // FP32 output: four rounds of 32 columns, each stored before the
            // next load; the accumulator is released after the last load.
#pragma unroll 1
            for (int hh = 0; hh < 4; ++hh) {
                uint32_t r[32];
                TMEM_LD_32(tbase + 32 * hh, r);
                tmem_ld_wait();
                if (hh == 3) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(acc_empty_leader);  // accumulator drained
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

// B's scales in the tensor-core layout, [G][nblk][K/64 atoms][512 bytes], seen
// as 8-byte elements: {256 (one K stage's 4 atoms), K/256 stages, nblk, G}; a
// box is one stage of two consecutive row blocks.
static bool make_sfb_map(CUtensorMap* m, const void* sfb, int64_t G, int64_t N, int64_t K)
{
    auto fn = encode_tiled();
    if (!fn) return false;
    const int64_t nblk = (N + 127) / 128, k64 = K / 64;
    cuuint64_t dims[4] = {256u, (cuuint64_t)(K / BK), (cuuint64_t)nblk, (cuuint64_t)G};
    cuuint64_t strides[3] = {2048u, (cuuint64_t)(k64 * 512), (cuuint64_t)(nblk * k64 * 512)};
    cuuint32_t box[4] = {256u, 1u, 2u, 1u};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 4, const_cast<void*>(sfb), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static size_t gemm_smem_bytes() { return (size_t)kGemmStages * kStageBytes + kSmemShared + 8 * kEpiStageBytes + 1024; }

struct GemmDevice {
    int sms = 0;
    int pairs = 0;  // CTA pairs that are resident at once
    bool ok = false;
};

static GemmDevice& gemm_device(int dev)
{
    static GemmDevice infos[64];
    static std::once_flag flags[64];
    std::call_once(flags[dev & 63], [dev]() {
        GemmDevice& d = infos[dev & 63];
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess || prop.major != 10) return;
        if (cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gemm_smem_bytes()) != cudaSuccess)
            return;
        d.sms = prop.multiProcessorCount;
        // Pairs need two SMs of one cluster-capable group: ask how many fit
        // at once, so that the persistent grid never waits for a second wave.
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(d.sms & ~1));
        cfg.blockDim = dim3(kGemmThreads);
        cfg.dynamicSmemBytes = gemm_smem_bytes();
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, gemm_kernel, &cfg) != cudaSuccess || clusters < 1)
            return;
        d.pairs = std::min(clusters, d.sms / 2);
        d.ok = true;
    });
    return infos[dev & 63];
}

static bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kGemmWorkspace = 256;

}  // namespace nvfp4

using namespace nvfp4;

extern "C" size_t nvfp4_gemm_workspace_size(int64_t, int64_t, int64_t) { return kGemmWorkspace; }

static nvfp4_status launch_gemm(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& msf, GemmArgs& a,
                                int64_t max_tiles, cudaStream_t st)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    GemmDevice& info = gemm_device(dev);
    if (!info.ok) return NVFP4_ERR_UNSUPPORTED;
    // the status word reports this call only; the output amax starts at 0
    if (cudaMemsetAsync(a.status, 0, 4, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (a.amax_out && cudaMemsetAsync(a.amax_out, 0, 4, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(max_tiles, info.pairs));
    gemm_kernel<<<2 * pairs, kGemmThreads, gemm_smem_bytes(), st>>>(ma, mb, msf, a);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

extern "C" nvfp4_status nvfp4_gemm(const uint8_t* qa, const uint8_t* sfa, const float* ga,
                                   const uint8_t* qb, const uint8_t* sfb, const float* gb,
                                   int64_t M, int64_t N, int64_t K, int out_dtype, void* D,
                                   int64_t ldd, float* amax_out, void* workspace, size_t ws_bytes,
                                   void* stream)
{
    if (!qa || !sfa || !ga || !qb || !sfb || !gb || !D) return NVFP4_ERR_INVALID_ARG;
    if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0 || M % 16 || N % 16 || K % BK || ldd < N) return NVFP4_ERR_SHAPE;
    if (M > (int64_t)1 << 31 || N > (int64_t)1 << 31) return NVFP4_ERR_SHAPE;
    const int esz = out_dtype == NVFP4_OUT_BF16 ? 2 : 4;
    if (!al16(qa) || !al16(qb) || !al16(sfa) || !al16(sfb) || !al16(D) || (ldd * esz) % 16 ||
        (reinterpret_cast<uintptr_t>(amax_out) & 3u))
        return NVFP4_ERR_ALIGN;
    if (!workspace || ws_bytes < kGemmWorkspace) return NVFP4_ERR_WORKSPACE;
    if (!al16(workspace)) return NVFP4_ERR_ALIGN;
    CUtensorMap ma, mb;
    if (!make_map(&ma, qa, M, K / 2, BM) || !make_map(&mb, qb, N, K / 2, BN / 2)) return NVFP4_ERR_CUDA;
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
    a.amax_out = amax_out;
    CUtensorMap msf;
    if (!make_sfb_map(&msf, sfb, 1, N, K)) return NVFP4_ERR_CUDA;
    const int64_t tiles = ((M + kMmaM - 1) / kMmaM) * ((N + BN - 1) / BN);
    return launch_gemm(ma, mb, msf, a, tiles, static_cast<cudaStream_t>(stream));
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
    if (total_rows <= 0 || N <= 0 || K <= 0 || N % 128 || K % BK) return NVFP4_ERR_SHAPE;
    if (total_rows > (int64_t)1 << 31 || (int64_t)G * N > (int64_t)1 << 31) return NVFP4_ERR_SHAPE;
    if (!al16(qa) || !al16(qb) || !al16(sfa) || !al16(sfb) || !al16(D) ||
        (reinterpret_cast<uintptr_t>(amax_out) & 3u))
        return NVFP4_ERR_ALIGN;
    if (!workspace || ws_bytes < kGemmWorkspace) return NVFP4_ERR_WORKSPACE;
    if (!al16(workspace)) return NVFP4_ERR_ALIGN;
    CUtensorMap ma, mb;
    if (!make_map(&ma, qa, total_rows, K / 2, BM) || !make_map(&mb, qb, (int64_t)G * N, K / 2, BN / 2))
        return NVFP4_ERR_CUDA;
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
    a.amax_out = amax_out;
    // upper bound on tiles: every group may add one partial M tile
    CUtensorMap msf;
    if (!make_sfb_map(&msf, sfb, G, N, K)) return NVFP4_ERR_CUDA;
    const int64_t tiles = ((total_rows + kMmaM - 1) / kMmaM + G) * ((N + BN - 1) / BN);
    return launch_gemm(ma, mb, msf, a, tiles, static_cast<cudaStream_t>(stream));
}
