// quantize.cu -- NVFP4 / MXFP8 quantisation and NVFP4 dequantisation on sm_100a.
//
// Two HBM-bound passes over 128x128 bf16 tiles, each a persistent grid whose
// warp 0 keeps a 2-stage ring of tiles in flight (TMA boxes with the 128-byte
// swizzle for dense input, per-row bulk copies for a gather) while all eight
// warps compute from shared memory:
//   1. amax_kernel: max |x| and, when the columnwise Hadamard is on, max
//      |RHT(x)| over the columnwise 16-vectors; one atomicMax per CTA
//      (amax_rows_kernel, with direct loads, when rows are gathered).
//   2. quant_kernel: walks the tiles in the reverse order of pass 1 (the tail
//      pass 1 left in L2 is read first) and produces, from one staged copy,
//      the rowwise codes/scales, the columnwise (transposed, optionally
//      Hadamard-rotated) codes/scales and the MXFP8 copies, with Philox
//      stochastic rounding in registers, 16-byte vector stores, and the
//      transposed MXFP8 codes written through per-warp shared-memory staging
//      and TMA stores.
//
// Format and steps: asector.ru, "Nvidia dobivaetsya uspekha s 4-bitnym
// formatom NVFP4" ("NVFP4 and Blackwell": E2M1, 16-element local scale plus a
// per-tensor scale, RNE and stochastic rounding; "Experiments and comparison
// with FP8": 2D weight scales, random Hadamard transforms), and iitak.ru,
// "Thinking Machines uskorila obuchenie Inkling 2 Small 4-bitnymi chislami"
// ("Details": -54 -> -6 with multiplier 9; "How it works": transposed blocks,
// 16x16 squares, random re-rounding, MXFP8 backward).
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <mutex>

#include "common.cuh"

namespace nvfp4 {

constexpr int kTileRows = 128;
constexpr int kTileCols = 128;
constexpr int kPitch = kTileCols * 2 + 16;  // bytes per staged row (+16 breaks bank aliasing)
constexpr int kTileBytes = kTileRows * kPitch;
constexpr int kStages = 2;
// Per-warp staging of the transposed outputs of a warp's 64 columns x 32 rows,
// each written out with one TMA store per warp and tile: MXFP8 codes (32
// bytes per column) and NVFP4 columnwise codes (16 bytes per column).
constexpr int kMxStageBytes = 64 * 32;
constexpr int kQcStageBytes = 64 * 16;
// Both passes run 8 warps per CTA, 2 CTAs per SM.  (Measured: 12-warp CTAs at
// 80 registers, with the rowwise and columnwise work on separate warps, made
// the fused gradient pass 13% slower.)
constexpr int kQuantThreads = 256;
constexpr int kColWarps = 8;
constexpr int kAmaxThreads = 256;
constexpr int kMaxGroups = 256;  // MoE groups per call (the grouped GEMM's limit too)

struct QArgs {
    const uint16_t* x;
    int64_t rows, cols, ld;
    int rounding, scaling, outputs, rht, sf_layout;
    uint64_t seed;
    uint32_t offset;
    const float* amax_in;
    const uint32_t* amax_ws;
    const int32_t* row_index;
    int64_t src_rows;
    const int32_t* group_offsets;
    int num_groups;
    int mx_outputs, mx_rounding;
    uint8_t *q_row, *sf_row;
    float* g_row;
    uint8_t *q_col, *sf_col;
    float* g_col;
    uint8_t *mx_q_row, *mx_sf_row, *mx_q_col, *mx_sf_col;
    uint32_t* status;
    int64_t tiles_c, n_tiles;
    PhiloxKeys pk;  // round keys of `seed`
    int mx_staged;  // MXFP8 columnwise codes go through shared memory and TMA stores
    int qc_staged;  // NVFP4 columnwise codes likewise (rows a multiple of 32)
    int mx_mma;     // MXFP8 scale bytes in the tensor-core tiled layout
    uint64_t wait_ns;  // limit of every barrier wait (2 s; shorter under the test hook)
    int no_copies;     // test hook: the producer issues no copy (see wait_test_hook)
};

// Offset of the E8M0 byte of 32-block b of row r, in a [rows, nblk] scale
// tensor: row-major, or the tensor cores' 128x4 atoms (the NVFP4 tiled layout
// with 32-element blocks).
__device__ __forceinline__ int64_t mx_sf_off(const QArgs& a, int64_t r, int64_t b, int64_t nblk)
{
    return a.mx_mma ? sf_mma_offset(r, b, nblk) : r * nblk + b;
}

__device__ __forceinline__ uint4 ld_global_v4(const void* p)
{
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint2 ld_global_v2(const void* p)
{
    uint2 r;
    asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}

__device__ __forceinline__ uint4 ld_shared_v4(const void* p)
{
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(smem_addr(p)));
    return r;
}

__device__ __forceinline__ uint32_t ld_shared_u32(const void* p)
{
    uint32_t r;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(smem_addr(p)));
    return r;
}

// Source row of output row r (gather); an out-of-range index is reported and
// replaced by row 0 so that every access stays inside x.
__device__ __forceinline__ int64_t source_row(const QArgs& a, int64_t r)
{
    if (!a.row_index) return r;
    const int64_t s = a.row_index[r];
    if (s < 0 || s >= a.src_rows) {
        record_status(a.status, NVFP4_ERR_INDEX);
        return 0;
    }
    return s;
}

// Tile row of a tile index: the host caps the tile count at 2^31 - 1, so a
// 32-bit division does (a 64-bit one costs several times the instructions).
__device__ __forceinline__ int64_t tile_row(const QArgs& a, int64_t tile)
{
    return (int64_t)((uint32_t)tile / (uint32_t)a.tiles_c);
}

__device__ __forceinline__ float warp_max16(float v)
{
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// --------------------------------------------------------------------------
// Tile staging and block quantisation, shared by the passes.
// --------------------------------------------------------------------------
struct QShared {
    // RN(S / d) for every scale byte (d its E4M3 value; 0 where d = 0), for
    // the rowwise [0] and columnwise [1] global scales: the per-block
    // division becomes a table lookup with the same result.
    float rtab[2][128];
    int32_t n_groups;
    int32_t group_start[kMaxGroups + 1];   // output-row offsets
    int32_t group_padded[kMaxGroups + 1];  // padded scale-row offsets
};

// Padded scale row of output row r (MoE layout); identity when dense.
__device__ __forceinline__ int64_t padded_row(const QShared* sh, bool grouped, int64_t r)
{
    if (!grouped) return r;
    int lo = 0, hi = sh->n_groups - 1;  // find e with start[e] <= r < start[e+1]
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sh->group_start[mid] <= r)
            lo = mid;
        else
            hi = mid - 1;
    }
    return r - sh->group_start[lo] + sh->group_padded[lo];
}

// Staged tile layouts.
//  kTma (dense input): two TMA boxes of 128 rows x 64 columns (128 bytes per
//    row) with the 128-byte swizzle -- 16-byte chunk q of a row sits at chunk
//    q ^ (row & 7) -- so both the rowwise 16-byte reads (8 rows per quarter
//    warp) and the columnwise 4-byte reads are bank-conflict free.
//  rows (gather): one bulk copy per row, rows kPitch bytes apart.
// Address of the 16-byte chunk holding columns 8q .. 8q+7 of tile row r.
template <bool kTma>
__device__ __forceinline__ const uint8_t* chunk_addr(const uint8_t* T, int r, int q)
{
    if (kTma) return T + (q >> 3) * (kTileRows * 128) + r * 128 + (((q & 7) ^ (r & 7)) << 4);
    return T + r * kPitch + q * 16;
}

template <bool kTma>
__device__ __forceinline__ void issue_tile(const QArgs& a, const CUtensorMap* map, int64_t tile,
                                           uint8_t* buf, uint64_t* bar, int lane)
{
    const int64_t tr = tile_row(a, tile), tc = tile - tr * a.tiles_c;
    const int64_t r0 = tr * kTileRows, c0 = tc * kTileCols;
    if (kTma) {
        // one box per 64-column panel; rows and columns past the tensor read as 0
        if (lane == 0) {
            const bool second = c0 + 64 < a.cols;
            mbar_arrive_expect_tx(bar, (second ? 2u : 1u) * kTileRows * 128u);
            tma_load_2d(buf, map, (int32_t)c0, (int32_t)r0, bar);
            if (second) tma_load_2d(buf + kTileRows * 128, map, (int32_t)(c0 + 64), (int32_t)r0, bar);
        }
        return;
    }
    const int nrows = (int)(a.rows - r0 < kTileRows ? a.rows - r0 : kTileRows);
    const uint32_t row_bytes = (uint32_t)(a.cols - c0 < kTileCols ? a.cols - c0 : kTileCols) * 2u;
    if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)nrows * row_bytes);
    __syncwarp();
    for (int i = lane; i < nrows; i += 32) {
        const int64_t sr = source_row(a, r0 + i);
        bulk_copy_g2s(buf + i * kPitch, a.x + sr * a.ld + c0, row_bytes, bar);
    }
}

__device__ __forceinline__ void unpack8(const uint4& p, float* v)
{
    v[0] = bf16_lo(p.x);
    v[1] = bf16_hi(p.x);
    v[2] = bf16_lo(p.y);
    v[3] = bf16_hi(p.y);
    v[4] = bf16_lo(p.z);
    v[5] = bf16_hi(p.z);
    v[6] = bf16_lo(p.w);
    v[7] = bf16_hi(p.w);
}

// RN(a / 6) for a >= 0.  Markstein's corrected quotient (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000 processor",
// IBM J. Res. Develop. 34(1), 1990): q0 = RN(a z) with z = RN(1/6), the
// remainder a - 6 q0 exactly in one fused multiply-add, then RN(q0 + r z).
// Checked against the IEEE division for every non-negative float: equal for
// every a >= 2^-120; below that (quotients near the subnormal range) the
// division itself is used.
__device__ __forceinline__ float div6_rn(float a)
{
    if (a < 7.52316384526264005100e-37f) return __fdiv_rn(a, 6.0f);  // 2^-120
    const float z = 0.16666667163372039794921875f;                    // RN(1/6)
    const float q0 = __fmul_rn(a, z);
    const float r = __fmaf_rn(-q0, 6.0f, a);
    return __fmaf_rn(r, z, q0);
}

// Quantisation of 16-value blocks given their (possibly 2D-reduced) amax:
// scale byte = E4M3_RNE((amax_b / 6) * S), r = RN(S / d) from the per-CTA table,
// codes = RNE or SR of x * r.  times4: v and amax_b hold 4x the values (Hadamard
// path without its factor 1/4); the factor is applied here exactly: amax_b/4
// never rounds, and v*(r/4) == (v/4)*r whenever r/4 is a normal float
// (otherwise the division is done per element).
// Two blocks at once (v and w, with their amax): both scale bytes from one
// paired E4M3 conversion and both Philox blocks computed side by side.  Returns
// the scale bytes (v's in bits 0..7, w's in bits 8..15); the codes go to
// cv0/cv1 and cw0/cw1.  With use_pre the two blocks' Philox words are given (pre_v,
// pre_w: the same words the call would compute from idx_v and idx_w).
__device__ __forceinline__ uint32_t quant_block16x2(float (&v)[16], float (&w)[16], float am_v,
                                                    float am_w, float S, const float* rtab,
                                                    bool times4, bool sr, const PhiloxKeys& pk,
                                                    uint32_t offset, uint32_t stream,
                                                    uint64_t idx_v, uint64_t idx_w, uint32_t& cv0,
                                                    uint32_t& cv1, uint32_t& cw0, uint32_t& cw1,
                                                    bool use_pre = false, U4 pre_v = U4{},
                                                    U4 pre_w = U4{})
{
    if (times4) {
        am_v = __fmul_rn(am_v, 0.25f);
        am_w = __fmul_rn(am_w, 0.25f);
    }
    const float sv = __fmul_rn(div6_rn(am_v), S);
    const float sw = __fmul_rn(div6_rn(am_w), S);
    const uint32_t bytes = e4m3x2_rne_sat(sw, sv) & 0xFFFFu;
    float rv = rtab[bytes & 0xFFu], rw = rtab[bytes >> 8];  // RN(S / d); 0 when d = 0
    if (times4) {
        if (rv >= 7.52316384526264005100e-37f) {  // 2^-120: r/4 stays normal
            rv = __fmul_rn(rv, 0.25f);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(v[i], 0.25f);
        }
        if (rw >= 7.52316384526264005100e-37f) {
            rw = __fmul_rn(rw, 0.25f);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) w[i] = __fmul_rn(w[i], 0.25f);
        }
    }
    if (times4) {
        // after the Hadamard butterflies the values sit in (v_i, w_i) register
        // pairs: one packed multiply per such pair needs no re-pairing
#pragma unroll
        for (int i = 0; i < 16; ++i) mul2(v[i], w[i], v[i], w[i], rv, rw);
    } else {
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            mul2(v[i], v[i + 1], v[i], v[i + 1], rv, rv);
            mul2(w[i], w[i + 1], w[i], w[i + 1], rw, rw);
        }
    }
    if (sr) {
        // one Philox call per 16-element block: word q drives elements 4q..4q+3
        U4 a, b;
        if (use_pre) {
            a = pre_v;
            b = pre_w;
        } else {
            const uint64_t jv = idx_v >> 4, jw = idx_w >> 4;
            philox4x32_10_keyed_x2(static_cast<uint32_t>(jv), static_cast<uint32_t>(jv >> 32),
                                   static_cast<uint32_t>(jw), static_cast<uint32_t>(jw >> 32), stream,
                                   offset, pk, a, b);
        }
        cv0 = e2m1x4_sr(v + 0, a.x) | (e2m1x4_sr(v + 4, a.y) << 16);
        cv1 = e2m1x4_sr(v + 8, a.z) | (e2m1x4_sr(v + 12, a.w) << 16);
        cw0 = e2m1x4_sr(w + 0, b.x) | (e2m1x4_sr(w + 4, b.y) << 16);
        cw1 = e2m1x4_sr(w + 8, b.z) | (e2m1x4_sr(w + 12, b.w) << 16);
    } else {
        cv0 = e2m1x8_rne(v);
        cv1 = e2m1x8_rne(v + 8);
        cw0 = e2m1x8_rne(w);
        cw1 = e2m1x8_rne(w + 8);
    }
    return bytes;
}

// MXFP8 of 32 values: returns the E8M0 byte, writes 32 code bytes to out[8].
__device__ __forceinline__ uint32_t mx_block32(const float* v, bool sr, const PhiloxKeys& pk,
                                               uint32_t offset, uint64_t idx, uint32_t* out)
{
    const float am = absmax16(v + 16, absmax16(v, 0.0f));
    // floor(log2 amax) - 8 from the exponent field; subnormal or zero amax -> -127
    const int ef = (int)((__float_as_uint(am) >> 23) & 0xFFu);
    const int e = max(ef - 127 - 8, -127);
    const float scale = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, exact
    if (sr) {
        U4 w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) w[q] = sr_block8(pk, offset, 2u, (idx >> 3) + q);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            float y[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                y[i] = e4m3_sr_value(__fmul_rn(v[4 * k + i], scale),
                                     u16_of(w[(4 * k + i) >> 3], (4 * k + i) & 7));
            out[k] = e4m3x2_rne_sat(y[1], y[0]) | (e4m3x2_rne_sat(y[3], y[2]) << 16);
        }
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            float y[4];
            mul2(y[0], y[1], v[4 * k], v[4 * k + 1], scale, scale);
            mul2(y[2], y[3], v[4 * k + 2], v[4 * k + 3], scale, scale);
            out[k] = e4m3x2_rne_sat(y[1], y[0]) | (e4m3x2_rne_sat(y[3], y[2]) << 16);
        }
    }
    return (uint32_t)(e + 127);
}

// E8M0 exponent of an MXFP8 block with absolute maximum am (OCP rule:
// floor(log2 am) - 8, clamped to -127; subnormal or zero am -> -127) and the
// exact scale 2^-e the elements are multiplied by.
__device__ __forceinline__ int mx_exponent(float am, float& scale)
{
    const int ef = (int)((__float_as_uint(am) >> 23) & 0xFFu);
    const int e = max(ef - 127 - 8, -127);
    scale = __uint_as_float((uint32_t)(127 - e) << 23);
    return e;
}

// 8 consecutive elements of one MXFP8 block -> 8 E4M3 bytes (element 0 in the
// low byte).  SR: 16-bit uniforms from the Philox block w of these 8 elements.
__device__ __forceinline__ uint2 mx_convert8(const float (&v)[8], float scale, bool sr, const U4& w)
{
    float y[8];
    if (sr) {
#pragma unroll
        for (int i = 0; i < 8; ++i) y[i] = e4m3_sr_value(__fmul_rn(v[i], scale), u16_of(w, i));
    } else {
#pragma unroll
        for (int i = 0; i < 8; i += 2) mul2(y[i], y[i + 1], v[i], v[i + 1], scale, scale);
    }
    return make_uint2(e4m3x2_rne_sat(y[1], y[0]) | (e4m3x2_rne_sat(y[3], y[2]) << 16),
                      e4m3x2_rne_sat(y[5], y[4]) | (e4m3x2_rne_sat(y[7], y[6]) << 16));
}

__device__ __forceinline__ void store_codes32(uint8_t* dst, const uint32_t (&c)[8], bool vec16)
{
    if (vec16) {
        reinterpret_cast<uint4*>(dst)[0] = make_uint4(c[0], c[1], c[2], c[3]);
        reinterpret_cast<uint4*>(dst)[1] = make_uint4(c[4], c[5], c[6], c[7]);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            reinterpret_cast<uint2*>(dst)[i] = make_uint2(c[2 * i], c[2 * i + 1]);
    }
}

// --------------------------------------------------------------------------
// Pass 1: global amax (dense input).  The same 128x128 TMA tiles and 2-stage
// copy ring as pass 2, walked in the opposite order; each thread takes one column pair over 32
// rows (two 16-row blocks): max |x| for the rowwise and 2D scales and, with the
// Hadamard on, max |RHT(x)| over the columnwise 16-vectors.  One atomicMax per
// CTA on the float bit pattern.
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(kAmaxThreads, 2)
    amax_kernel(const __grid_constant__ CUtensorMap map_x, QArgs a, uint32_t* amax_out)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* tiles = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kTileBytes);
    uint64_t* empty = full + kStages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kAmaxThreads / 32);
        }
        fence_barrier_init();
    }
    __syncthreads();
    const bool rht = a.rht != 0;
    const uint32_t signs = rht ? rht_sign_bits(a.seed) : 0u;
    const int64_t first = blockIdx.x;
    const int64_t my_count =
        first < a.n_tiles ? (a.n_tiles - first + gridDim.x - 1) / gridDim.x : 0;
    auto tile_of = [&](int64_t k) { return first + k * (int64_t)gridDim.x; };
    int64_t issued = 0;
    const bool produce = warp == 0 && !a.no_copies;
    if (produce) {
        for (; issued < my_count && issued < kStages - 1; ++issued)
            issue_tile<true>(a, &map_x, tile_of(issued), tiles + (issued % kStages) * kTileBytes,
                             &full[issued % kStages], lane);
    }
    const int cp = 32 * (warp & 1) + lane;  // column pair 0..63
    const int rgrp = warp >> 1;              // 32-row group 0..3
    float mr = 0.0f, mc = 0.0f;
    int64_t k = 0;
    for (; k < my_count; ++k) {
        const int stage = (int)(k % kStages);
        if (produce && issued < my_count) {
            const int s = (int)(issued % kStages);
            bool ok = true;
            if (issued >= kStages) ok = mbar_wait(&empty[s], (uint32_t)((issued / kStages - 1) & 1), a.wait_ns);
            if (!ok) {
                if (lane == 0) record_status(a.status, NVFP4_ERR_TIMEOUT);
                break;
            }
            issue_tile<true>(a, &map_x, tile_of(issued), tiles + s * kTileBytes, &full[s], lane);
            ++issued;
        }
        if (!mbar_wait(&full[stage], (uint32_t)((k / kStages) & 1), a.wait_ns)) {
            if (lane == 0) record_status(a.status, NVFP4_ERR_TIMEOUT);
            break;
        }
        const uint8_t* T = tiles + stage * kTileBytes;
        const int64_t tile = tile_of(k);
        const int64_t tr = tile_row(a, tile), tc = tile - tr * a.tiles_c;
        const int64_t cg0 = tc * kTileCols + 2 * cp;
        const int64_t rbase = tr * kTileRows + 32 * rgrp;
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
            // positions past the tensor hold zeros (rows) or stale bytes (an
            // uncopied second panel): skip them
            if (cg0 >= a.cols || rbase + 16 * sub >= a.rows) continue;
            float va[16], vb[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t w =
                    ld_shared_u32(chunk_addr<true>(T, 32 * rgrp + 16 * sub + i, cp >> 2) + 4 * (cp & 3));
                unpack_bf16x2(w, ((signs >> i) & 1u) << 31, va[i], vb[i]);  // |x| unaffected
            }
            mr = absmax16(vb, absmax16(va, mr));
            if (rht) {
                hadamard16x2_times4(va, vb);  // 4x the transform; the 1/4 is applied once below
                mc = absmax16(vb, absmax16(va, mc));
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
    }
    if (warp == 0) {
        for (int64_t j = k + 1; j < issued; ++j)
            (void)mbar_wait(&full[j % kStages], (uint32_t)((j / kStages) & 1), a.wait_ns);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, o));
        mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
    }
    __shared__ float red[2][kAmaxThreads / 32];
    if (lane == 0) {
        red[0][warp] = mr;
        red[1][warp] = mc;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kAmaxThreads / 32; ++w) {
            mr = fmaxf(mr, red[0][w]);
            mc = fmaxf(mc, red[1][w]);
        }
        mc = __fmul_rn(mc, 0.25f);  // the transform's factor 1/4 (exact)
        // non-negative floats order like their bit patterns
        atomicMax(&amax_out[0], __float_as_uint(mr));
        atomicMax(&amax_out[1], __float_as_uint(mc));
    }
}

// Pass 1 for a gather: rows come from row_index, so tiles would be staged by
// one small copy per row; direct loads of 16 rows x 4 columns per thread (16
// in flight) serve it better.
__global__ void __launch_bounds__(256, 2) amax_rows_kernel(QArgs a, uint32_t* amax_out)
{
    const bool rht = a.rht != 0;
    const uint32_t signs = rht ? rht_sign_bits(a.seed) : 0u;
    float mr = 0.0f, mc = 0.0f;
    const int64_t ncg = a.cols / 4;
    const int64_t units = (a.rows / 16) * ncg;
    for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < units;
         u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t rb = u / ncg, cg = u - rb * ncg;
        uint2 raw[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            raw[i] = ld_global_v2(a.x + source_row(a, rb * 16 + i) * a.ld + cg * 4);
        // columns 2p and 2p+1 form one packed pair; row i's sign flip (the
        // Hadamard's D) is applied while unpacking -- |x| is unaffected
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            float va[16], vb[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                unpack_bf16x2(p == 0 ? raw[i].x : raw[i].y, ((signs >> i) & 1u) << 31, va[i], vb[i]);
            mr = absmax16(vb, absmax16(va, mr));
            if (rht) {
                hadamard16x2_times4(va, vb);
                mc = absmax16(vb, absmax16(va, mc));
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, o));
        mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
    }
    __shared__ float red[2][8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        red[0][warp] = mr;
        red[1][warp] = mc;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < 8; ++w) {
            mr = fmaxf(mr, red[0][w]);
            mc = fmaxf(mc, red[1][w]);
        }
        mc = __fmul_rn(mc, 0.25f);  // the transform's factor 1/4 (exact)
        atomicMax(&amax_out[0], __float_as_uint(mr));
        atomicMax(&amax_out[1], __float_as_uint(mc));
    }
}

// --------------------------------------------------------------------------
// Pass 2: fused quantisation.
// --------------------------------------------------------------------------
// Compile-time variants of the fused pass.  Each switch is off, on, or read
// from the call's arguments (run time).  Variant 0 reads every switch at run
// time; the others fix the switches for the tensor roles of the training
// recipe (asector.ru, "Experiments and comparison with FP8": 2D weight scales
// and random Hadamard transforms for outlier gradients; iitak.ru, "How it
// works": 16x16 weight squares, random re-rounding and the MXFP8 backward):
//   1 gradients:   rowwise SR, columnwise Hadamard + SR, MXFP8 columnwise RNE
//   2 activations: rowwise RNE, columnwise Hadamard RNE
//   3 weights:     16x16 2D scales, both directions, RNE
//   4 MoE rows:    rowwise RNE only (gather and groups at run time)
//   5 MXFP8 rows:  MXFP8 rowwise only (the expert outputs of the MoE combine)
// Fixed switches let the compiler drop the unused branches and the registers
// they hold; results are identical to variant 0.
enum : int8_t { kOff = 0, kOn = 1, kRt = 2 };
struct QSpec {
    int8_t nv_row, nv_col, mx_row, mx_col, sr, mx_sr, rht, two_d, groups;
};
constexpr int kNumSpecs = 6;
constexpr QSpec kSpecs[kNumSpecs] = {
    {kRt, kRt, kRt, kRt, kRt, kRt, kRt, kRt, kRt},
    {kOn, kOn, kOff, kOn, kOn, kOff, kOn, kOff, kOff},
    {kOn, kOn, kOff, kOff, kOff, kRt, kOn, kOff, kOff},
    {kOn, kOn, kOff, kOff, kOff, kRt, kOff, kOn, kOff},
    {kOn, kOff, kOff, kOff, kOff, kRt, kRt, kOff, kRt},
    {kOff, kOff, kOn, kOff, kOff, kRt, kOff, kOff, kOff},
};
template <bool B>
struct BoolC {
    static constexpr bool value = B;
};

__host__ __device__ constexpr bool spec_pick(int8_t s, bool run_time)
{
    return s == kRt ? run_time : s == kOn;
}

template <bool kTma, int kSpec>
__global__ void __launch_bounds__(kQuantThreads, 2)
    quant_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_mx,
                 const __grid_constant__ CUtensorMap map_qc, const __grid_constant__ QArgs a)
{
    constexpr QSpec sp = kSpecs[kSpec];
    extern __shared__ uint8_t smem_raw[];
    // the swizzled TMA boxes need 1024-byte alignment
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* tiles = smem;
    uint8_t* mx_stage_all = smem + kStages * kTileBytes;
    uint8_t* qc_stage_all = mx_stage_all + kColWarps * kMxStageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(qc_stage_all + kColWarps * kQcStageBytes);
    QShared* sh = reinterpret_cast<QShared*>(reinterpret_cast<uint8_t*>(bars) + 64);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars[s], 1);                              // full: producer + tx bytes
            mbar_init(&bars[kStages + s], kQuantThreads / 32);  // empty: one arrival per warp
        }
        fence_barrier_init();
    }
    const bool grouped = spec_pick(sp.groups, a.group_offsets != nullptr);
    if (grouped) {
        if (threadIdx.x == 0) {
            sh->n_groups = a.num_groups;
            int32_t pad = 0;
            for (int e = 0; e <= a.num_groups; ++e) {
                const int32_t st = a.group_offsets[e];
                sh->group_start[e] = st;
                sh->group_padded[e] = pad;
                if (e < a.num_groups) {
                    const int32_t cnt = a.group_offsets[e + 1] - st;
                    pad += ((cnt + 127) / 128) * 128;
                }
            }
        }
    }
    __syncthreads();

    const bool nv_row = spec_pick(sp.nv_row, (a.outputs & NVFP4_ROWWISE) != 0);
    const bool nv_col = spec_pick(sp.nv_col, (a.outputs & NVFP4_COLWISE) != 0);
    const bool mx_row = spec_pick(sp.mx_row, (a.mx_outputs & NVFP4_ROWWISE) != 0);
    const bool mx_col = spec_pick(sp.mx_col, (a.mx_outputs & NVFP4_COLWISE) != 0);
    const bool sr = spec_pick(sp.sr, a.rounding == NVFP4_SR);
    const bool mx_sr = spec_pick(sp.mx_sr, a.mx_rounding == NVFP4_SR);
    const bool two_d = spec_pick(sp.two_d, a.scaling == NVFP4_2D16x16);
    const bool rht = spec_pick(sp.rht, a.rht != 0);
    const bool mma_sf = a.sf_layout == NVFP4_SF_MMA;

    float S_row = 1.0f, g_row = 1.0f, S_col = 1.0f, g_col = 1.0f;
    if (nv_row || nv_col) {
        float amax_r, amax_c;
        if (a.amax_in) {
            amax_r = a.amax_in[0];
            amax_c = a.amax_in[1];
        } else {
            amax_r = __uint_as_float(a.amax_ws[0]);
            amax_c = rht ? __uint_as_float(a.amax_ws[1]) : amax_r;
        }
        global_scales(amax_r, S_row, g_row);
        global_scales(amax_c, S_col, g_col);
        if (blockIdx.x == 0 && threadIdx.x == 0) {
            if (nv_row) *a.g_row = g_row;
            if (nv_col) *a.g_col = g_col;
        }
        for (int t = threadIdx.x; t < 256; t += blockDim.x) {
            const float d = e4m3_value((uint32_t)(t & 127));
            sh->rtab[t >> 7][t & 127] = d != 0.0f ? __fdiv_rn(t < 128 ? S_row : S_col, d) : 0.0f;
        }
        __syncthreads();
    }
    const uint32_t signs = (nv_col && rht) ? rht_sign_bits(a.seed) : 0u;

    const int64_t first = blockIdx.x;
    const int64_t my_count =
        first < a.n_tiles ? (a.n_tiles - first + gridDim.x - 1) / gridDim.x : 0;
    auto tile_of = [&](int64_t k) { return a.n_tiles - 1 - (first + k * (int64_t)gridDim.x); };

    // Stage ring: full[s] completes when tile data landed, empty[s] when all 8
    // warps are done with it.  Warp 0 keeps two tiles in flight ahead of the
    // tile it computes; no CTA-wide barrier, so warps drift apart freely.
    uint64_t* full = bars;
    uint64_t* empty = bars + kStages;
    int64_t issued = 0;  // tiles whose copies warp 0 has issued
    const bool produce = warp == 0 && !a.no_copies;
    if (produce) {
        for (; issued < my_count && issued < kStages - 1; ++issued)
            issue_tile<kTma>(a, &map_x, tile_of(issued), tiles + (issued % kStages) * kTileBytes,
                             &full[issued % kStages], lane);
    }

    const bool q_row_vec = (a.cols % 32) == 0;
    const bool q_col_vec = (a.rows % 32) == 0;
    const bool sf_row_vec = mma_sf || (a.cols % 64) == 0;
    const bool sf_col_vec = mma_sf || (a.rows % 32) == 0;  // 2 scale bytes per column store

    int64_t k = 0;
    for (; k < my_count; ++k) {
        const int stage = (int)(k % kStages);
        if (produce && issued < my_count) {
            // refill the stage tile `issued - kStages` used, once every warp released it
            const int s = (int)(issued % kStages);
            bool ok = true;
            if (issued >= kStages)
                ok = mbar_wait(&empty[s], (uint32_t)((issued / kStages - 1) & 1), a.wait_ns);
            if (!ok) {
                if (lane == 0) record_status(a.status, NVFP4_ERR_TIMEOUT);
                break;
            }
            issue_tile<kTma>(a, &map_x, tile_of(issued), tiles + s * kTileBytes, &full[s], lane);
            ++issued;
        }
        if (!mbar_wait(&full[stage], (uint32_t)((k / kStages) & 1), a.wait_ns)) {
            if (lane == 0) record_status(a.status, NVFP4_ERR_TIMEOUT);
            break;
        }
        const uint8_t* T = tiles + stage * kTileBytes;
        const int64_t tile = tile_of(k);
        const int64_t tr = tile_row(a, tile), tc = tile - tr * a.tiles_c;
        const int64_t r0 = tr * kTileRows, c0 = tc * kTileCols;
        // A tile wholly inside the tensor runs a copy of the body compiled
        // without the edge predicates (every check below is then a constant);
        // tiles on an edge run the general copy.  Same results either way.
        const bool full_tile = r0 + kTileRows <= a.rows && c0 + kTileCols <= a.cols;
        auto tile_body = [&](auto full_c) {
            constexpr bool kFull = decltype(full_c)::value;

            // ---------------- rowwise: thread = (row, 64-column half) ----------
            if (nv_row || mx_row) {
                const int rl = 16 * warp + (lane & 15);
                const int h = lane >> 4;
                const int64_t rg = r0 + rl;
                const bool rvalid = kFull || rg < a.rows;
                const int64_t cbase = c0 + 64 * h;
                // Shared-memory reads are unconditional: positions past the tensor
                // hold zeros (TMA) or stale bytes (gather), and blocks made of them
                // are never stored; 1D blocks and 16x16 tiles never mix valid and
                // invalid elements because rows and cols are multiples of 16.
                if (nv_row) {
                    uint32_t codes[8];
                    uint32_t sfw = 0;
                    bool all_valid = true;
                    // the random words of the thread's four blocks (consecutive
                    // counters), four Philox chains side by side
                    U4 rnd[4] = {};
                    if (sr) philox4x32_10_keyed_x4((uint64_t)(rg * a.cols + cbase) >> 4, 0u, a.offset, a.pk, rnd);
    #pragma unroll
                    for (int bp = 0; bp < 4; bp += 2) {  // two 16-blocks at a time
                        const int64_t cg = cbase + 16 * bp;
                        all_valid &= kFull || (rvalid && cg + 16 < a.cols);
                        float v[16], w[16];
                        unpack8(ld_shared_v4(chunk_addr<kTma>(T, rl, 8 * h + 2 * bp)), v);
                        unpack8(ld_shared_v4(chunk_addr<kTma>(T, rl, 8 * h + 2 * bp + 1)), v + 8);
                        unpack8(ld_shared_v4(chunk_addr<kTma>(T, rl, 8 * h + 2 * bp + 2)), w);
                        unpack8(ld_shared_v4(chunk_addr<kTma>(T, rl, 8 * h + 2 * bp + 3)), w + 8);
                        float amv = absmax16(v, 0.0f), amw = absmax16(w, 0.0f);
                        if (two_d) {
                            amv = warp_max16(amv);
                            amw = warp_max16(amw);
                        }
                        const uint64_t idx = (uint64_t)(rg * a.cols + cg);
                        const uint32_t bytes = quant_block16x2(
                            v, w, amv, amw, S_row, sh->rtab[0], false, sr && (kFull || (rvalid && cg < a.cols)), a.pk,
                            a.offset, 0u, idx, idx + 16, codes[2 * bp], codes[2 * bp + 1],
                            codes[2 * bp + 2], codes[2 * bp + 3], sr, rnd[bp], rnd[bp + 1]);
                        sfw |= bytes << (8 * bp);
                    }
                    if (all_valid) {
                        store_codes32(a.q_row + rg * (a.cols / 2) + cbase / 2, codes, q_row_vec);
                        const int64_t b0 = cbase / 16;
                        const int64_t off = mma_sf ? sf_mma_offset(padded_row(sh, grouped, rg), b0, a.cols / 16)
                                                   : rg * (a.cols / 16) + b0;
                        if (sf_row_vec) {
                            *reinterpret_cast<uint32_t*>(a.sf_row + off) = sfw;
                        } else {
    #pragma unroll
                            for (int blk = 0; blk < 4; ++blk) a.sf_row[off + blk] = (sfw >> (8 * blk)) & 0xFFu;
                        }
                    } else if (rvalid) {
    #pragma unroll
                        for (int blk = 0; blk < 4; ++blk) {
                            const int64_t cg = cbase + 16 * blk;
                            if (cg >= a.cols) continue;
                            *reinterpret_cast<uint2*>(a.q_row + rg * (a.cols / 2) + cg / 2) =
                                make_uint2(codes[2 * blk], codes[2 * blk + 1]);
                            const int64_t off = mma_sf ? sf_mma_offset(padded_row(sh, grouped, rg), cg / 16, a.cols / 16)
                                                       : rg * (a.cols / 16) + cg / 16;
                            a.sf_row[off] = (sfw >> (8 * blk)) & 0xFFu;
                        }
                    }
                }
                if (mx_row && rvalid) {
    #pragma unroll 1
                    for (int part = 0; part < 2; ++part) {
                        const int64_t cg = cbase + 32 * part;
                        if (!kFull && cg >= a.cols) continue;
                        float v[32];
    #pragma unroll
                        for (int q = 0; q < 4; ++q)
                            unpack8(ld_shared_v4(chunk_addr<kTma>(T, rl, 8 * h + 4 * part + q)), v + 8 * q);
                        uint32_t out[8];
                        const uint32_t e8 = mx_block32(v, mx_sr, a.pk, a.offset,
                                                       (uint64_t)(rg * a.cols + cg), out);
                        uint4* dst = reinterpret_cast<uint4*>(a.mx_q_row + rg * a.cols + cg);
                        dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
                        dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
                        a.mx_sf_row[mx_sf_off(a, rg, cg / 32, a.cols / 32)] = (uint8_t)e8;
                    }
                }
            }

            // ---------------- columnwise: thread = (column pair, 32-row group) --
            // One 32-bit shared load per row gives both columns of the pair; the
            // pair's two Hadamard transforms run in the two lanes of f32x2.
            if (nv_col || mx_col) {
                const int cp = 32 * (warp & 1) + lane;  // column pair 0..63
                const int rgrp = warp >> 1;              // 32-row group 0..3
                const int64_t cg0 = c0 + 2 * cp;         // columns cg0, cg0 + 1
                const bool cvalid = kFull || cg0 < a.cols;  // cols is even: the pair is whole
                const int64_t rbase = r0 + 32 * rgrp;
                // the pair's 4 bytes: chunk cp/4 of each row, byte 4*(cp%4) within it
                // shared addresses of the pair's word in rows j = 0..7 of the group (TMA
                // tiles: the swizzle depends on row & 7); row i is row i & 7 plus
                // (i >> 3) * 8 rows, a constant offset
                uint32_t pw_base[8];
                {
                    const int q = cp >> 2;
                    const uint32_t b0 = smem_addr(T) + 4u * (cp & 3);
    #pragma unroll
                    for (int j = 0; j < 8; ++j)
                        pw_base[j] = kTma ? b0 + (q >> 3) * (kTileRows * 128) + (32 * rgrp + j) * 128 +
                                                (((q & 7) ^ j) << 4)
                                          : b0 + (32 * rgrp + j) * kPitch + q * 16;
                }
                auto pair_word = [&](int i) -> uint32_t {
                    uint32_t r;
                    asm volatile("ld.shared.u32 %0, [%1];"
                                 : "=r"(r)
                                 : "r"(pw_base[i & 7] + (i >> 3) * (kTma ? 8 * 128 : 8 * kPitch)));
                    return r;
                };
                // MXFP8 columnwise: the 32-row block's amax of each column is
                // gathered while the NVFP4 pass below unpacks the rows (the
                // Hadamard's sign flips leave |x| alone); the conversion then
                // re-reads the rows 8 at a time.  rows is a multiple of 32 here.
                float mxa = 0.0f, mxb = 0.0f;
                const int64_t cwarp = c0 + 64 * (warp & 1);  // first column of the warp
                uint8_t* stg_qc = qc_stage_all + warp * kQcStageBytes;
                const bool qc_staged = kTma && nv_col && a.qc_staged;
                if (kTma && (a.mx_staged || qc_staged)) {
                    if (lane == 0) bulk_wait_read0();  // this warp's previous stores have read its staging
                    __syncwarp();
                }
                if (kFull || rbase < a.rows) {
                    // rows is a multiple of 16: both 16-row blocks exist, or (at the
                    // bottom edge) only the first.  The first block's codes wait in
                    // registers so each column gets one 16-byte store.
                    const bool two = kFull || rbase + 32 <= a.rows;
                    const int64_t b0 = rbase / 16;
                    uint32_t keep0 = 0, keep1 = 0, keep2 = 0, keep3 = 0, keep_sf = 0;
    #pragma unroll
                    for (int sub = 0; sub < 2; ++sub) {
                        if (sub == 1 && !two) break;
                        const int64_t rg = rbase + 16 * sub;
                        float va[16], vb[16];
    #pragma unroll
                        for (int i = 0; i < 16; ++i)
                            unpack_bf16x2(pair_word(16 * sub + i), rht ? ((signs >> i) & 1u) << 31 : 0u,
                                          va[i], vb[i]);
                        if (mx_col) {
                            mxa = absmax16(va, mxa);
                            mxb = absmax16(vb, mxb);
                        }
                        if (!nv_col) continue;
                        if (rht) hadamard16x2_times4(va, vb);
                        float ama = absmax16(va, 0.0f), amb = absmax16(vb, 0.0f);
                        if (two_d) {  // 16x16 tile = 8 column pairs (lanes) x 16 rows
                            float m = fmaxf(ama, amb);
    #pragma unroll
                            for (int o = 1; o < 8; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                            ama = amb = m;
                        }
                        uint32_t ca0, ca1, cb0, cb1;
                        const uint32_t bab = quant_block16x2(
                            va, vb, ama, amb, S_col, sh->rtab[1], rht, sr && cvalid, a.pk, a.offset, 1u,
                            (uint64_t)(cg0 * a.rows + rg), (uint64_t)((cg0 + 1) * a.rows + rg), ca0, ca1,
                            cb0, cb1);
                        const uint32_t ba = bab & 0xFFu, bb = bab >> 8;
                        if (!cvalid) continue;
                        if (two && sub == 0) {
                            keep0 = ca0, keep1 = ca1, keep2 = cb0, keep3 = cb1;
                            keep_sf = ba | (bb << 8);
                            continue;
                        }
                        uint8_t* da = a.q_col + cg0 * (a.rows / 2) + rbase / 2;
                        uint8_t* db = da + a.rows / 2;
                        const int64_t offa = mma_sf ? sf_mma_offset(cg0, b0, a.rows / 16)
                                                    : cg0 * (a.rows / 16) + b0;
                        const int64_t offb = mma_sf ? sf_mma_offset(cg0 + 1, b0, a.rows / 16)
                                                    : offa + a.rows / 16;
                        if (!two) {  // a lone 16-row block: 8 code bytes and one scale per column
                            *reinterpret_cast<uint2*>(da) = make_uint2(ca0, ca1);
                            *reinterpret_cast<uint2*>(db) = make_uint2(cb0, cb1);
                            a.sf_col[offa] = (uint8_t)ba;
                            a.sf_col[offb] = (uint8_t)bb;
                        } else {
                            if (qc_staged) {  // buffer row 2*lane + h = column cg0 + h
                                st_shared_v4(stg_qc + (2 * lane) * 16, make_uint4(keep0, keep1, ca0, ca1));
                                st_shared_v4(stg_qc + (2 * lane + 1) * 16, make_uint4(keep2, keep3, cb0, cb1));
                            } else if (q_col_vec) {
                                *reinterpret_cast<uint4*>(da) = make_uint4(keep0, keep1, ca0, ca1);
                                *reinterpret_cast<uint4*>(db) = make_uint4(keep2, keep3, cb0, cb1);
                            } else {
                                reinterpret_cast<uint2*>(da)[0] = make_uint2(keep0, keep1);
                                reinterpret_cast<uint2*>(da)[1] = make_uint2(ca0, ca1);
                                reinterpret_cast<uint2*>(db)[0] = make_uint2(keep2, keep3);
                                reinterpret_cast<uint2*>(db)[1] = make_uint2(cb0, cb1);
                            }
                            const uint32_t sfa = (keep_sf & 0xFFu) | (ba << 8);
                            const uint32_t sfb = (keep_sf >> 8) | (bb << 8);
                            if (sf_col_vec) {
                                *reinterpret_cast<uint16_t*>(a.sf_col + offa) = (uint16_t)sfa;
                                *reinterpret_cast<uint16_t*>(a.sf_col + offb) = (uint16_t)sfb;
                            } else {
                                a.sf_col[offa] = (uint8_t)sfa;
                                a.sf_col[offa + 1] = (uint8_t)(sfa >> 8);
                                a.sf_col[offb] = (uint8_t)sfb;
                                a.sf_col[offb + 1] = (uint8_t)(sfb >> 8);
                            }
                        }
                    }
                }
                if (qc_staged && (kFull || (rbase < a.rows && cwarp < a.cols))) {
                    // this warp's 64 columns x 32 rows of NVFP4 codes (16 bytes per
                    // column) out with one TMA store, clipped at the tensor edge
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&map_qc, stg_qc, (int32_t)(rbase / 2), (int32_t)cwarp);
                        bulk_commit();
                    }
                }
                if (kTma && mx_col && a.mx_staged) {
                    // This warp's 64 columns x 32 rows of codes go to its staging
                    // buffer (row 2*lane + h of the buffer = column cg0 + h) and out
                    // with one TMA store; the store clips what lies past the tensor.
                    if (kFull || (rbase < a.rows && cwarp < a.cols)) {
                        uint8_t* stg = mx_stage_all + warp * kMxStageBytes;
                        float sa, sb;
                        const int ea = mx_exponent(mxa, sa), eb = mx_exponent(mxb, sb);
                        const int64_t ia = cg0 * a.rows + rbase, ib = ia + a.rows;  // element indices
    #pragma unroll
                        for (int g2 = 0; g2 < 2; ++g2) {  // 16 rows per pass
                            uint2 ca[2], cb[2];
    #pragma unroll
                            for (int gg = 0; gg < 2; ++gg) {
                                const int g = 2 * g2 + gg;
                                float va[8], vb[8];
    #pragma unroll
                                for (int i = 0; i < 8; ++i) {
                                    const uint32_t w = pair_word(8 * g + i);
                                    va[i] = bf16_lo(w);
                                    vb[i] = bf16_hi(w);
                                }
                                U4 wa{}, wb{};
                                if (mx_sr) {
                                    wa = sr_block8(a.pk, a.offset, 2u, (uint64_t)(ia >> 3) + g);
                                    wb = sr_block8(a.pk, a.offset, 2u, (uint64_t)(ib >> 3) + g);
                                }
                                ca[gg] = mx_convert8(va, sa, mx_sr, wa);
                                cb[gg] = mx_convert8(vb, sb, mx_sr, wb);
                            }
                            st_shared_v4(stg + (2 * lane) * 32 + 16 * g2,
                                         make_uint4(ca[0].x, ca[0].y, ca[1].x, ca[1].y));
                            st_shared_v4(stg + (2 * lane + 1) * 32 + 16 * g2,
                                         make_uint4(cb[0].x, cb[0].y, cb[1].x, cb[1].y));
                        }
                        if (cvalid) {
                            a.mx_sf_col[mx_sf_off(a, cg0, rbase / 32, a.rows / 32)] = (uint8_t)(ea + 127);
                            a.mx_sf_col[mx_sf_off(a, cg0 + 1, rbase / 32, a.rows / 32)] = (uint8_t)(eb + 127);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&map_mx, stg, (int32_t)rbase, (int32_t)cwarp);
                            bulk_commit();
                        }
                    }
                } else if (mx_col && cvalid && (kFull || rbase < a.rows)) {
                    float sa, sb;
                    const int ea = mx_exponent(mxa, sa), eb = mx_exponent(mxb, sb);
                    const int64_t ia = cg0 * a.rows + rbase, ib = ia + a.rows;  // element indices
                    uint8_t* qa = a.mx_q_col + ia;
                    uint8_t* qb = a.mx_q_col + ib;
    #pragma unroll 2
                    for (int g = 0; g < 4; ++g) {
                        float va[8], vb[8];
    #pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const uint32_t w = pair_word(8 * g + i);
                            va[i] = bf16_lo(w);
                            vb[i] = bf16_hi(w);
                        }
                        U4 wa{}, wb{};
                        if (mx_sr) {
                            wa = sr_block8(a.pk, a.offset, 2u, (uint64_t)(ia >> 3) + g);
                            wb = sr_block8(a.pk, a.offset, 2u, (uint64_t)(ib >> 3) + g);
                        }
                        *reinterpret_cast<uint2*>(qa + 8 * g) = mx_convert8(va, sa, mx_sr, wa);
                        *reinterpret_cast<uint2*>(qb + 8 * g) = mx_convert8(vb, sb, mx_sr, wb);
                    }
                    a.mx_sf_col[mx_sf_off(a, cg0, rbase / 32, a.rows / 32)] = (uint8_t)(ea + 127);
                    a.mx_sf_col[mx_sf_off(a, cg0 + 1, rbase / 32, a.rows / 32)] = (uint8_t)(eb + 127);
                }
            }
        };
        if (full_tile)
            tile_body(BoolC<true>{});
        else
            tile_body(BoolC<false>{});
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);  // this warp is done with the stage
    }
    // This warp's staged stores must finish before the CTA's shared memory
    // goes away.
    if (kTma && lane == 0) bulk_wait_all();
    // Copies issued for tiles this CTA did not consume (only after a timeout)
    // must land before the CTA's shared memory goes away.
    if (warp == 0) {
        for (int64_t j = k + 1; j < issued; ++j)
            (void)mbar_wait(&full[j % kStages], (uint32_t)((j / kStages) & 1), a.wait_ns);
    }
}

// --------------------------------------------------------------------------
// MoE dispatch of quantised rows: output row i = source row row_index[i]
// (codes and scale bytes), scales rewritten from the dense tiled layout into
// the grouped tiled layout.  One CTA per (group, 128-row block), the blocks the
// grouped GEMM tiles over, so each CTA writes whole 512-byte scale atoms.
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(512) gather_rows_kernel(
    const uint8_t* q_src, const uint8_t* sf_src, int64_t src_rows, int64_t k,
    const int32_t* row_index, int64_t rows, const int32_t* group_offsets, int G, uint8_t* q_dst,
    uint8_t* sf_dst, uint32_t* status)
{
    // locate this CTA's (group, block): group e has ceil(count/128) blocks.
    // The offsets come into shared memory in one parallel load; warp 0 then
    // scans 32 groups per step (block counts, inclusive shuffle scan, ballot).
    __shared__ int s_e, s_t, s_pad_blk;
    __shared__ int32_t s_off[kMaxGroups + 1];
    if (group_offsets) {
        for (int g = threadIdx.x; g <= G; g += blockDim.x) s_off[g] = group_offsets[g];
        __syncthreads();
    }
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int e = -1, t = 0, pad_blk = 0;
        const int b = blockIdx.x;
        if (!group_offsets) {
            if ((int64_t)b * 128 < rows) e = 0, t = b;
        } else {
            int before = 0;  // blocks of the groups already scanned
            for (int g0 = 0; g0 < G; g0 += 32) {
                const int g = g0 + lane;
                const int nb = g < G ? (s_off[g + 1] - s_off[g] + 127) / 128 : 0;
                int incl = nb;
                for (int d = 1; d < 32; d <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, incl, d);
                    if (lane >= d) incl += v;
                }
                const unsigned hit = __ballot_sync(0xffffffffu, b < before + incl && b >= before + incl - nb && nb > 0);
                if (hit) {
                    const int src = __ffs(hit) - 1;
                    const int excl = before + __shfl_sync(0xffffffffu, incl - nb, src);
                    e = g0 + src;
                    t = b - excl;
                    pad_blk = excl;
                    break;
                }
                before += __shfl_sync(0xffffffffu, incl, 31);
            }
        }
        if (lane == 0) {
            s_e = e;
            s_t = t;
            s_pad_blk = pad_blk;
        }
    }
    __syncthreads();
    const int e = s_e;
    if (e < 0) return;
    const int64_t g0 = group_offsets ? group_offsets[e] : 0;
    const int64_t g1 = group_offsets ? group_offsets[e + 1] : rows;
    const int64_t r0 = g0 + 128 * (int64_t)s_t;
    const int nr = (int)(g1 - r0 < 128 ? g1 - r0 : 128);
    const int64_t dst_blk = s_pad_blk + s_t;  // padded 128-row scale block
    const int64_t k16 = k / 16, k64 = k / 64, chunks = k / 32;  // 16-byte code chunks per row

    __shared__ int64_t s_src[128];
    for (int i = threadIdx.x; i < nr; i += blockDim.x) {
        int64_t s = row_index[r0 + i];
        if (s < 0 || s >= src_rows) {
            record_status(status, NVFP4_ERR_INDEX);
            s = 0;
        }
        s_src[i] = s;
    }
    __syncthreads();
    // codes: one warp per two rows at a time, its lanes on consecutive 16-byte
    // vectors, four loads per row in flight per lane before their stores
    {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const int nwarps = blockDim.x >> 5;
        for (int i = warp; i < nr; i += 2 * nwarps) {
            // rows i and i + nwarps: both rows' loads in flight before their stores
            const int i2 = i + nwarps;
            const bool two = i2 < nr;
            const uint4* __restrict__ src = reinterpret_cast<const uint4*>(q_src + s_src[i] * (k / 2));
            uint4* __restrict__ dst = reinterpret_cast<uint4*>(q_dst + (r0 + i) * (k / 2));
            const uint4* __restrict__ src2 =
                reinterpret_cast<const uint4*>(q_src + s_src[two ? i2 : i] * (k / 2));
            uint4* __restrict__ dst2 = reinterpret_cast<uint4*>(q_dst + (r0 + (two ? i2 : i)) * (k / 2));
            int64_t c = lane;
            for (; c + 96 < chunks; c += 128) {
                const uint4 v0 = src[c], v1 = src[c + 32], v2 = src[c + 64], v3 = src[c + 96];
                uint4 u0, u1, u2, u3;
                if (two) u0 = src2[c], u1 = src2[c + 32], u2 = src2[c + 64], u3 = src2[c + 96];
                dst[c] = v0;
                dst[c + 32] = v1;
                dst[c + 64] = v2;
                dst[c + 96] = v3;
                if (two) {
                    dst2[c] = u0;
                    dst2[c + 32] = u1;
                    dst2[c + 64] = u2;
                    dst2[c + 96] = u3;
                }
            }
            for (; c < chunks; c += 32) {
                dst[c] = src[c];
                if (two) dst2[c] = src2[c];
            }
        }
    }
    // scales: 4 bytes (one row's four 16-blocks of a 64-column group) per
    // word; consecutive threads write consecutive words of a destination atom
    // (word w holds row (w >> 2) + 32 * (w & 3)), eight loads in flight each
    const int total = 128 * (int)k64;  // <= 2^29 (k <= 2^28): no index below overflows
    for (int base = threadIdx.x; base < total; base += 8 * blockDim.x) {
        uint32_t v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int idx = base + u * blockDim.x;
            const int w = idx & 127, i = (w >> 2) | ((w & 3) << 5);
            if (idx < total && i < nr)
                v[u] = *reinterpret_cast<const uint32_t*>(sf_src + sf_mma_offset(s_src[i], 4 * (idx >> 7), k16));
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int idx = base + u * blockDim.x;
            const int w = idx & 127, i = (w >> 2) | ((w & 3) << 5);
            if (idx < total && i < nr)
                *reinterpret_cast<uint32_t*>(sf_dst + sf_mma_offset(dst_blk * 128 + i, 4 * (idx >> 7), k16)) = v[u];
        }
    }
}

// --------------------------------------------------------------------------
// Dequantisation: x_hat = (e2m1(code) * d) * g.
// --------------------------------------------------------------------------
__device__ __forceinline__ void e2m1x2_to_f32(uint32_t byte, float& lo, float& hi)
{
    uint32_t h2;
    const uint16_t b = static_cast<uint16_t>(byte & 0xFFu);
    asm("{\n\t.reg .b8 b0, b1;\n\tmov.b16 {b0, b1}, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b0;\n\t}"
        : "=r"(h2)
        : "h"(b));
    lo = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
    hi = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
}

__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* q, const uint8_t* sf,
                                                      const float* gp, int64_t rows, int64_t cols,
                                                      int mma_sf, int bf16_out, void* out)
{
    const float g = *gp;
    const int64_t nb = rows * (cols / 16);
    for (int64_t blk = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; blk < nb;
         blk += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = blk / (cols / 16), b = blk - r * (cols / 16);
        const uint2 c = *reinterpret_cast<const uint2*>(q + r * (cols / 2) + b * 8);
        const int64_t off = mma_sf ? sf_mma_offset(r, b, cols / 16) : r * (cols / 16) + b;
        const float d = e4m3_value(sf[off]);
        float v[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t word = i < 4 ? c.x : c.y;
            float lo, hi;
            e2m1x2_to_f32((word >> (8 * (i & 3))) & 0xFFu, lo, hi);
            v[2 * i] = __fmul_rn(__fmul_rn(lo, d), g);
            v[2 * i + 1] = __fmul_rn(__fmul_rn(hi, d), g);
        }
        if (bf16_out) {
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const __nv_bfloat162 p = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
                w[i] = *reinterpret_cast<const uint32_t*>(&p);
            }
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + r * cols + b * 16);
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + r * cols + b * 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
    }
}

// --------------------------------------------------------------------------
// Host side.
// --------------------------------------------------------------------------
struct DeviceInfo {
    int sms = 0;
    int quant_blocks_per_sm = 0;
    bool ok = false;
};

static size_t quant_smem_bytes()
{
    return (size_t)kStages * kTileBytes + kColWarps * (kMxStageBytes + kQcStageBytes) + 64 +
           sizeof(QShared) + 1024;  // + alignment slack
}

// Tensor map of the bf16 input for the TMA tile path: boxes of 128 rows x 64
// columns (128 bytes) with the 128-byte swizzle.
static bool make_input_map(CUtensorMap* m, const void* x, int64_t rows, int64_t cols, int64_t ld)
{
    auto fn = encode_tiled_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
    cuuint32_t box[2] = {64u, (cuuint32_t)kTileRows};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

using QuantKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, QArgs);

// The compiled variants: TMA tiles for dense input, row copies for the gather
// (which only variants 0 and 4 serve).  nullptr where none is built.
static QuantKernel quant_variant(bool tma, int spec)
{
    switch (spec) {
    case 0: return tma ? quant_kernel<true, 0> : quant_kernel<false, 0>;
    case 1: return tma ? quant_kernel<true, 1> : nullptr;
    case 2: return tma ? quant_kernel<true, 2> : nullptr;
    case 3: return tma ? quant_kernel<true, 3> : nullptr;
    case 4: return tma ? quant_kernel<true, 4> : quant_kernel<false, 4>;
    case 5: return tma ? quant_kernel<true, 5> : nullptr;
    }
    return nullptr;
}

// First compiled variant whose fixed switches agree with the call (variant 0
// agrees with every call).
static int pick_variant(const QArgs& a, bool tma)
{
    auto agrees = [](int8_t s, bool v) { return s == kRt || (s == kOn) == v; };
    for (int v = 1; v < kNumSpecs; ++v) {
        const QSpec& q = kSpecs[v];
        if (quant_variant(tma, v) && agrees(q.nv_row, (a.outputs & NVFP4_ROWWISE) != 0) &&
            agrees(q.nv_col, (a.outputs & NVFP4_COLWISE) != 0) &&
            agrees(q.mx_row, (a.mx_outputs & NVFP4_ROWWISE) != 0) &&
            agrees(q.mx_col, (a.mx_outputs & NVFP4_COLWISE) != 0) &&
            agrees(q.sr, a.rounding == NVFP4_SR) && agrees(q.mx_sr, a.mx_rounding == NVFP4_SR) &&
            agrees(q.rht, a.rht != 0) && agrees(q.two_d, a.scaling == NVFP4_2D16x16) &&
            agrees(q.groups, a.group_offsets != nullptr))
            return v;
    }
    return 0;
}

// Store map of a transposed output [cols, inner] (u8, inner bytes contiguous):
// boxes of box_inner bytes x 64 columns, no swizzle.  inner is a multiple of
// 16 (MXFP8 codes: inner = rows, box 32; NVFP4 codes: inner = rows / 2, box 16).
static bool make_store_map(CUtensorMap* m, const void* q, int64_t inner, int64_t cols, uint32_t box_inner)
{
    auto fn = encode_tiled_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)cols};
    cuuint64_t strides[1] = {(cuuint64_t)inner};
    cuuint32_t box[2] = {box_inner, 64u};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(q), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static DeviceInfo& device_info(int dev)
{
    static DeviceInfo infos[64];
    static std::once_flag flags[64];
    std::call_once(flags[dev & 63], [dev]() {
        DeviceInfo& d = infos[dev & 63];
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return;
        if (prop.major != 10) return;
        d.sms = prop.multiProcessorCount;
        int blocks = 1 << 30;
        for (int tma = 0; tma < 2; ++tma) {
            for (int v = 0; v < kNumSpecs; ++v) {
                const QuantKernel fn = quant_variant(tma != 0, v);
                if (!fn) continue;
                int nb = 0;
                if (cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)quant_smem_bytes()) != cudaSuccess ||
                    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, kQuantThreads,
                                                                  quant_smem_bytes()) != cudaSuccess ||
                    nb < 1)
                    return;
                blocks = std::min(blocks, nb);
            }
        }
        for (const void* fn : {reinterpret_cast<const void*>(amax_kernel)}) {
            int nb = 0;
            if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)quant_smem_bytes()) != cudaSuccess ||
                cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, kAmaxThreads,
                                                              quant_smem_bytes()) != cudaSuccess ||
                nb < 1)
                return;
            blocks = std::min(blocks, nb);
        }
        d.quant_blocks_per_sm = blocks;
        d.ok = true;
    });
    return infos[dev & 63];
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kQuantWorkspace = 256;

}  // namespace nvfp4

using namespace nvfp4;

extern "C" size_t nvfp4_sf_mma_bytes(int64_t rows, int64_t k)
{
    if (rows <= 0 || k <= 0) return 0;
    return (size_t)((rows + 127) / 128) * 128 * (size_t)(((k / 16) + 3) / 4) * 4;
}

extern "C" size_t mxfp8_sf_mma_bytes(int64_t rows, int64_t k)
{
    if (rows <= 0 || k <= 0) return 0;
    return (size_t)((rows + 127) / 128) * 128 * (size_t)(((k / 32) + 3) / 4) * 4;
}

extern "C" size_t nvfp4_sf_mma_grouped_bytes(int64_t total_rows, int num_groups, int64_t k)
{
    if (total_rows < 0 || num_groups <= 0 || k <= 0) return 0;
    const int64_t padded = ((total_rows + 127) / 128) * 128 + 128 * (int64_t)num_groups;
    return (size_t)padded * (size_t)(((k / 16) + 3) / 4) * 4;
}

extern "C" size_t nvfp4_quantize_workspace_size(int64_t, int64_t, const nvfp4_quant_params*)
{
    return kQuantWorkspace;
}

static nvfp4_status launch_quant(QArgs& a, bool need_amax, void* workspace, cudaStream_t st)
{
    philox_round_keys(a.seed, &a.pk);
    wait_test_hook(&a.wait_ns, &a.no_copies);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    DeviceInfo& info = device_info(dev);
    if (!info.ok) return NVFP4_ERR_UNSUPPORTED;
    a.tiles_c = (a.cols + kTileCols - 1) / kTileCols;
    a.n_tiles = ((a.rows + kTileRows - 1) / kTileRows) * a.tiles_c;
    if (a.n_tiles > 0x7FFFFFFFll) return NVFP4_ERR_SHAPE;  // tile indices are 31-bit on the device
    if (workspace) {
        // amax words (when computed) and the status word start at zero on every call
        uint32_t* ws = static_cast<uint32_t*>(workspace);
        if (cudaMemsetAsync(need_amax ? ws : ws + 2, 0, need_amax ? 12 : 4, st) != cudaSuccess)
            return NVFP4_ERR_CUDA;
    }
    const int64_t grid = std::min<int64_t>(a.n_tiles, (int64_t)info.sms * info.quant_blocks_per_sm);
    CUtensorMap map;
    memset(&map, 0, sizeof(map));
    const bool tma = !a.row_index;  // dense input: TMA tiles; the gather reads rows one by one
    if (tma && !make_input_map(&map, a.x, a.rows, a.cols, a.ld)) return NVFP4_ERR_CUDA;
    if (need_amax) {
        uint32_t* amax = static_cast<uint32_t*>(workspace);
        a.amax_ws = amax;
        if (tma) {
            amax_kernel<<<(int)grid, kAmaxThreads, quant_smem_bytes(), st>>>(map, a, amax);
        } else {
            const int64_t units = (a.rows / 16) * (a.cols / 4);  // 16 rows x 4 columns each
            const int blocks = (int)std::max<int64_t>(
                1, std::min<int64_t>((units + 255) / 256, (int64_t)info.sms * 8));
            amax_rows_kernel<<<blocks, 256, 0, st>>>(a, amax);
        }
        if (cudaGetLastError() != cudaSuccess) return NVFP4_ERR_CUDA;
    }
    const QuantKernel fn = quant_variant(tma, pick_variant(a, tma));
    CUtensorMap map_mx;
    memset(&map_mx, 0, sizeof(map_mx));
    a.mx_staged = 0;
    if (tma && (a.mx_outputs & NVFP4_COLWISE)) {
        if (!make_store_map(&map_mx, a.mx_q_col, a.rows, a.cols, 32)) return NVFP4_ERR_CUDA;
        a.mx_staged = 1;
    }
    CUtensorMap map_qc;
    memset(&map_qc, 0, sizeof(map_qc));
    a.qc_staged = 0;
    if (tma && (a.outputs & NVFP4_COLWISE) && a.rows % 32 == 0) {
        if (!make_store_map(&map_qc, a.q_col, a.rows / 2, a.cols, 16)) return NVFP4_ERR_CUDA;
        a.qc_staged = 1;
    }
    void* args[] = {&map, &map_mx, &map_qc, &a};
    if (cudaLaunchKernel(reinterpret_cast<const void*>(fn), dim3((unsigned)grid), dim3(kQuantThreads),
                         args, quant_smem_bytes(), st) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

extern "C" nvfp4_status nvfp4_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                       const nvfp4_quant_params* p, uint8_t* q_row,
                                       uint8_t* sf_row, float* g_row, uint8_t* q_col,
                                       uint8_t* sf_col, float* g_col, void* workspace,
                                       size_t ws_bytes, void* stream)
{
    if (!x_bf16 || !p) return NVFP4_ERR_INVALID_ARG;
    // MXFP8 rowwise alone quantises every row on its own: any row count will do
    const bool mx_rows_only = p->outputs == 0 && p->mx_outputs == NVFP4_ROWWISE;
    if (rows <= 0 || cols <= 0 || (rows % 16 && !mx_rows_only) || cols % 16 || ld < cols)
        return NVFP4_ERR_SHAPE;
    if (!aligned16(x_bf16) || (ld * 2) % 16) return NVFP4_ERR_ALIGN;
    if (p->rounding != NVFP4_RNE && p->rounding != NVFP4_SR) return NVFP4_ERR_INVALID_ARG;
    if (p->mx_rounding != NVFP4_RNE && p->mx_rounding != NVFP4_SR) return NVFP4_ERR_INVALID_ARG;
    if (p->scaling != NVFP4_1D16 && p->scaling != NVFP4_2D16x16) return NVFP4_ERR_INVALID_ARG;
    if (p->sf_layout != NVFP4_SF_ROWMAJOR && p->sf_layout != NVFP4_SF_MMA) return NVFP4_ERR_INVALID_ARG;
    if (p->outputs & ~3 || p->mx_outputs & ~3) return NVFP4_ERR_INVALID_ARG;
    if (p->rht_colwise != 0 && p->rht_colwise != 1) return NVFP4_ERR_INVALID_ARG;
    if (p->outputs == 0 && p->mx_outputs == 0) return NVFP4_ERR_INVALID_ARG;
    const bool nv_row = p->outputs & NVFP4_ROWWISE, nv_col = p->outputs & NVFP4_COLWISE;
    if (nv_row && (!q_row || !sf_row || !g_row)) return NVFP4_ERR_INVALID_ARG;
    if (nv_col && (!q_col || !sf_col || !g_col)) return NVFP4_ERR_INVALID_ARG;
    if ((nv_row && (!aligned16(q_row) || !aligned16(sf_row))) ||
        (nv_col && (!aligned16(q_col) || !aligned16(sf_col))))
        return NVFP4_ERR_ALIGN;
    if (p->sf_layout == NVFP4_SF_MMA && ((nv_row && cols % 64) || (nv_col && rows % 64)))
        return NVFP4_ERR_SHAPE;
    if (p->mx_sf_layout != NVFP4_SF_ROWMAJOR && p->mx_sf_layout != NVFP4_SF_MMA)
        return NVFP4_ERR_INVALID_ARG;
    if (p->mx_sf_layout == NVFP4_SF_MMA &&
        (((p->mx_outputs & NVFP4_ROWWISE) && cols % 128) || ((p->mx_outputs & NVFP4_COLWISE) && rows % 128)))
        return NVFP4_ERR_SHAPE;
    if (p->mx_outputs & NVFP4_ROWWISE) {
        if (cols % 32) return NVFP4_ERR_SHAPE;
        if (!p->mx_q_row || !p->mx_sf_row) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(p->mx_q_row)) return NVFP4_ERR_ALIGN;
    }
    if (p->mx_outputs & NVFP4_COLWISE) {
        if (rows % 32) return NVFP4_ERR_SHAPE;
        if (!p->mx_q_col || !p->mx_sf_col) return NVFP4_ERR_INVALID_ARG;
        if (!aligned16(p->mx_q_col)) return NVFP4_ERR_ALIGN;
    }
    if (p->row_index && p->src_rows <= 0) return NVFP4_ERR_INVALID_ARG;
    if (p->group_offsets) {
        if (p->sf_layout != NVFP4_SF_MMA || !nv_row || p->num_groups < 1 ||
            p->num_groups > kMaxGroups)
            return NVFP4_ERR_INVALID_ARG;
    }
    const bool need_amax = (nv_row || nv_col) && !p->amax_in;
    if (need_amax && (!workspace || ws_bytes < kQuantWorkspace)) return NVFP4_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return NVFP4_ERR_ALIGN;

    QArgs a{};
    a.x = static_cast<const uint16_t*>(x_bf16);
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.rounding = p->rounding;
    a.scaling = p->scaling;
    a.outputs = p->outputs;
    a.rht = p->rht_colwise;
    a.sf_layout = p->sf_layout;
    a.seed = p->seed;
    a.offset = p->offset;
    a.amax_in = p->amax_in;
    a.row_index = p->row_index;
    a.src_rows = p->src_rows;
    a.group_offsets = p->group_offsets;
    a.num_groups = p->num_groups;
    a.mx_outputs = p->mx_outputs;
    a.mx_rounding = p->mx_rounding;
    a.q_row = q_row;
    a.sf_row = sf_row;
    a.g_row = g_row;
    a.q_col = q_col;
    a.sf_col = sf_col;
    a.g_col = g_col;
    a.mx_q_row = p->mx_q_row;
    a.mx_sf_row = p->mx_sf_row;
    a.mx_q_col = p->mx_q_col;
    a.mx_sf_col = p->mx_sf_col;
    a.mx_mma = p->mx_sf_layout == NVFP4_SF_MMA;
    a.status = workspace ? static_cast<uint32_t*>(workspace) + 2 : nullptr;
    return launch_quant(a, need_amax, workspace, static_cast<cudaStream_t>(stream));
}

// --------------------------------------------------------------------------
// Allocation-free quantisation.
//
// Some callers cannot hand the library a workspace: code running under a host
// framework whose device memory is fully reserved by its own caching
// allocator, or latency-critical paths that must never reach cudaMalloc
// (which can synchronise the whole device).  For them nvfp4_quantize_noalloc
// keeps the quantiser's scratch (two amax words and the status word) in the
// file-scope array below instead of a caller buffer.  Every GPU that loads
// this library holds the array until the process exits.
// --------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = 256;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array on device `dev`, looked up with that device
// current (host code only sees a stand-in symbol, never the device address).
// Only a successful lookup is kept: a failed one (for example, attempted during
// a stream capture) is tried again on the next call instead of failing every
// later call on that device.
static void* noalloc_scratch(int dev)
{
    static std::atomic<void*> ptrs[64];
    void* p = ptrs[dev].load(std::memory_order_acquire);
    if (p) return p;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    p = ptrs[dev].load(std::memory_order_relaxed);
    if (!p && cudaGetSymbolAddress(&p, g_noalloc_scratch) == cudaSuccess && p)
        ptrs[dev].store(p, std::memory_order_release);
    return ptrs[dev].load(std::memory_order_relaxed);
}

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void* x_bf16, int64_t rows, int64_t cols,
                                               int64_t ld, const nvfp4_quant_params* p,
                                               uint8_t* q_row, uint8_t* sf_row, float* g_row,
                                               uint8_t* q_col, uint8_t* sf_col, float* g_col,
                                               void* stream)
{
    if (nvfp4_quantize_workspace_size(rows, cols, p) > kNoAllocScratchBytes)
        return NVFP4_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (dev < 0 || dev >= 64) return NVFP4_ERR_UNSUPPORTED;
    void* scratch = noalloc_scratch(dev);
    if (!scratch) return NVFP4_ERR_CUDA;
    return nvfp4_quantize(x_bf16, rows, cols, ld, p, q_row, sf_row, g_row, q_col, sf_col, g_col,
                          scratch, kNoAllocScratchBytes, stream);
}

extern "C" nvfp4_status nvfp4_quantize_noalloc_status(void* stream)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (dev < 0 || dev >= 64) return NVFP4_ERR_UNSUPPORTED;
    void* scratch = noalloc_scratch(dev);
    if (!scratch) return NVFP4_ERR_CUDA;
    return nvfp4_workspace_status(scratch, stream);
}

extern "C" nvfp4_status mxfp8_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                       int directions, int rounding, uint64_t seed,
                                       uint32_t offset, uint8_t* q_row, uint8_t* e8_row,
                                       uint8_t* q_col, uint8_t* e8_col, void* stream)
{
    nvfp4_quant_params p{};
    p.rounding = NVFP4_RNE;
    p.mx_outputs = directions;
    p.mx_rounding = rounding;
    p.seed = seed;
    p.offset = offset;
    p.mx_q_row = q_row;
    p.mx_sf_row = e8_row;
    p.mx_q_col = q_col;
    p.mx_sf_col = e8_col;
    if (directions == 0 || (directions & ~3)) return NVFP4_ERR_INVALID_ARG;
    return nvfp4_quantize(x_bf16, rows, cols, ld, &p, nullptr, nullptr, nullptr, nullptr, nullptr,
                          nullptr, nullptr, 0, stream);
}

extern "C" nvfp4_status nvfp4_gather_rows(const uint8_t* q_src, const uint8_t* sf_src,
                                          int64_t src_rows, int64_t k, const int32_t* row_index,
                                          int64_t rows, const int32_t* group_offsets,
                                          int num_groups, uint8_t* q_dst, uint8_t* sf_dst,
                                          void* workspace, size_t ws_bytes, void* stream)
{
    if (!q_src || !sf_src || !row_index || !q_dst || !sf_dst) return NVFP4_ERR_INVALID_ARG;
    if (src_rows <= 0 || rows <= 0 || k <= 0 || k % 64 || k > (int64_t(1) << 28)) return NVFP4_ERR_SHAPE;
    if (group_offsets && (num_groups < 1 || num_groups > kMaxGroups)) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(q_src) || !aligned16(q_dst) || (reinterpret_cast<uintptr_t>(sf_src) & 3) ||
        (reinterpret_cast<uintptr_t>(sf_dst) & 3))
        return NVFP4_ERR_ALIGN;
    if (workspace && (ws_bytes < kQuantWorkspace || !aligned16(workspace))) return NVFP4_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (!device_info(dev).ok) return NVFP4_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t* status = workspace ? static_cast<uint32_t*>(workspace) + 2 : nullptr;
    if (status && cudaMemsetAsync(status, 0, 4, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    const int64_t blocks = (rows + 127) / 128 + (group_offsets ? num_groups : 0);
    gather_rows_kernel<<<(int)blocks, 512, 0, st>>>(q_src, sf_src, src_rows, k, row_index, rows,
                                                    group_offsets, num_groups, q_dst, sf_dst,
                                                    status);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

extern "C" nvfp4_status nvfp4_dequantize(const uint8_t* q, const uint8_t* sf, const float* g,
                                         int64_t rows, int64_t cols, int sf_layout, int out_dtype,
                                         void* out, void* stream)
{
    if (!q || !sf || !g || !out) return NVFP4_ERR_INVALID_ARG;
    if (rows <= 0 || cols <= 0 || cols % 16) return NVFP4_ERR_SHAPE;
    if (sf_layout != NVFP4_SF_ROWMAJOR && sf_layout != NVFP4_SF_MMA) return NVFP4_ERR_INVALID_ARG;
    if (sf_layout == NVFP4_SF_MMA && cols % 64) return NVFP4_ERR_SHAPE;
    if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(q) & 7u) || !aligned16(out)) return NVFP4_ERR_ALIGN;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    DeviceInfo& info = device_info(dev);
    if (!info.ok) return NVFP4_ERR_UNSUPPORTED;
    const int64_t nb = rows * (cols / 16);
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((nb + 255) / 256, (int64_t)info.sms * 8));
    dequant_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        q, sf, g, rows, cols, sf_layout == NVFP4_SF_MMA, out_dtype == NVFP4_OUT_BF16, out);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

extern "C" nvfp4_status nvfp4_workspace_status(void* workspace, void* stream)
{
    if (!workspace) return NVFP4_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    uint32_t* word = static_cast<uint32_t*>(workspace) + 2;
    if (cudaMemcpyAsync(&v, word, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (v != 0 && cudaMemsetAsync(word, 0, 4, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    return static_cast<nvfp4_status>(v);
}

extern "C" const char* nvfp4_status_string(nvfp4_status s)
{
    switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_SHAPE: return "unsupported shape";
    case NVFP4_ERR_ALIGN: return "pointer or leading dimension not 16-byte aligned";
    case NVFP4_ERR_UNSUPPORTED: return "unsupported device or combination";
    case NVFP4_ERR_CUDA: return "CUDA runtime error";
    case NVFP4_ERR_TIMEOUT: return "device wait timed out";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
    case NVFP4_ERR_INDEX: return "gather index out of range";
    }
    return "unknown status";
}

extern "C" int nvfp4_version(void) { return 200; }
