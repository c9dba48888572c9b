// mxfp4.cu -- MXFP4 quantisation (OCP Microscaling, 32-element blocks, E8M0
// scale, E2M1 elements), both directions from one staged copy of the input.
//
// MXFP4 is the 4-bit format the pages measure NVFP4 against (hightech.plus,
// "Novyi 4-bitnyi metod obucheniya BYaM ne ustupaet 8-bitnomu": existing
// 4-bit formats such as MXFP4 fall short of 8-bit accuracy; asector.ru,
// "Nvidia dobivaetsya uspekha s 4-bitnym formatom NVFP4", section "NVFP4 and
// Blackwell": Blackwell's tensor cores take MXFP8, MXFP6, MXFP4 and NVFP4, and
// the comparison with the Open Compute Project's MXFP4, which NVFP4 beats).
// The pages do not restate the format, so the OCP MX v1.0 definition is used:
// per block e = clamp(floor(log2 amax) - 2, -127, 127), 2 being the largest
// E2M1 exponent (6 = 1.5 * 2^2); scale byte e + 127 (amax 0 -> e = -127);
// element = E2M1 of x * 2^-e, round-to-nearest-even, saturating at +-6.
// There is no tensor scale.
//
// Persistent CTAs walk 64 x 128 tiles; each tile is copied into one of two
// shared-memory buffers with 16-byte cp.async while the CTA quantises the
// other.  Warps 0..3 quantise the tile's columns (thread = column pair x
// 32-row block, one 32-bit shared load per row gives both columns) into a
// staging block, from which lane pairs store each column's 32 code bytes as
// one whole sector; warps 4..7 quantise its rows (thread = one 32-block of a
// row; four lanes cover a row's 64 code bytes, so every store instruction
// writes whole sectors).  Values stay packed as bf16 pairs and are unpacked
// where they are used.  The kernel is
// HBM-bound: 2 bytes read and 0.5 + 1/32 written per element and direction.
#include "common.cuh"

#include <mutex>

namespace nvfp4 {
namespace {

constexpr int kMx4TileRows = 64;
constexpr int kMx4TileCols = 128;
constexpr int kMx4Pitch = kMx4TileCols * 2 + 16;  // bytes per staged row (+16 staggers banks)
constexpr int kMx4Threads = 256;

struct Mx4Args {
    const uint16_t* x;
    int64_t rows, cols, ld;
    uint8_t* q_row;
    uint8_t* e8_row;
    uint8_t* q_col;
    uint8_t* e8_col;
    int64_t tiles_r, tiles_c;
    int mma_sf;  // scale bytes in the tensor cores' tiled layout (128x4 atoms of 32-blocks)
};

// Offset of the E8M0 byte of 32-block b of row r in a [rows, nblk] scale tensor.
__device__ __forceinline__ int64_t mx4_sf_off(const Mx4Args& a, int64_t r, int64_t b, int64_t nblk)
{
    return a.mma_sf ? sf_mma_offset(r, b, nblk) : r * nblk + b;
}

// E8M0 byte of a block with absolute maximum am, and the exact factor 2^-e
// its elements are multiplied by.  floor(log2 am) is the unbiased exponent
// field for a normal am; a subnormal or zero am has field 0 and lands on the
// clamp (-127).  The largest finite am gives e = 125, inside the clamp.
__device__ __forceinline__ uint32_t mx4_scale(float am, float& factor)
{
    const int ef = (int)((__float_as_uint(am) >> 23) & 0xFFu);
    const int e = max(ef - 127 - 2, -127);
    factor = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e: exponent field 2..254
    return (uint32_t)(e + 127);
}

// Eight values, given as four bf16 pairs (element 0 in the low half), times
// the block factor -> eight codes (element 0 in the low nibble).
__device__ __forceinline__ uint32_t mx4_codes8(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                               float f)
{
    float y[8];
    mul2(y[0], y[1], bf16_lo(w0), bf16_hi(w0), f, f);
    mul2(y[2], y[3], bf16_lo(w1), bf16_hi(w1), f, f);
    mul2(y[4], y[5], bf16_lo(w2), bf16_hi(w2), f, f);
    mul2(y[6], y[7], bf16_lo(w3), bf16_hi(w3), f, f);
    return e2m1x8_rne(y);
}

// Copy tile t into `buf` (64 rows of 16 chunks of 8 elements); chunks past the
// tensor are zero-filled without reading and only feed blocks never stored.
__device__ __forceinline__ void mx4_issue_tile(const Mx4Args& a, int64_t t, uint8_t* buf)
{
    const int64_t tr = (uint32_t)t / (uint32_t)a.tiles_c, tcol = t - tr * a.tiles_c;  // t < 2^31
    const int64_t r0 = tr * kMx4TileRows, c0 = tcol * kMx4TileCols;
#pragma unroll
    for (int i = threadIdx.x; i < kMx4TileRows * 16; i += kMx4Threads) {
        const int r = i >> 4, q = i & 15;
        const bool in = r0 + r < a.rows && c0 + 8 * q < a.cols;
        const uint16_t* src = in ? a.x + (r0 + r) * a.ld + c0 + 8 * q : a.x;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                         smem_addr(buf + r * kMx4Pitch + 16 * q)),
                     "l"(src), "r"(in ? 16 : 0)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

constexpr int kMx4StgPitch = 48;  // bytes per staged column: 32 code bytes + 16 (banks)

__device__ __forceinline__ void mx4_tile(const Mx4Args& a, int64_t t, const uint8_t* tile,
                                         uint8_t* stg, uint8_t* stg_e8)
{
    const int64_t tr = (uint32_t)t / (uint32_t)a.tiles_c, tcol = t - tr * a.tiles_c;  // t < 2^31
    const int64_t r0 = tr * kMx4TileRows, c0 = tcol * kMx4TileCols;
    // valid extent of the tile: multiples of 32 (rows and cols are)
    const int nr = a.rows - r0 < kMx4TileRows ? (int)(a.rows - r0) : kMx4TileRows;
    const int nc = a.cols - c0 < kMx4TileCols ? (int)(a.cols - c0) : kMx4TileCols;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < 4) {
        if (!a.q_col) return;
        // columnwise: column pair cp (columns 2cp, 2cp + 1), 32-row block rb
        const int cp = 32 * (warp & 1) + lane, rb = warp >> 1;
        if (2 * cp < nc && 32 * rb < nr) {
        uint32_t w[32];
        float ma = 0.0f, mb = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            w[i] = *reinterpret_cast<const uint32_t*>(tile + (32 * rb + i) * kMx4Pitch + 4 * cp);
            ma = absmax3(ma, bf16_lo(w[i]), 0.0f);
            mb = absmax3(mb, bf16_hi(w[i]), 0.0f);
        }
        float fa, fb;
        const uint32_t ea = mx4_scale(ma, fa), eb = mx4_scale(mb, fb);
        uint32_t ca[4], cb[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            // column a = low halves, column b = high halves of rows 8g .. 8g+7
            float y[8];
#pragma unroll
            for (int i = 0; i < 8; i += 2)
                mul2(y[i], y[i + 1], bf16_lo(w[8 * g + i]), bf16_lo(w[8 * g + i + 1]), fa, fa);
            ca[g] = e2m1x8_rne(y);
#pragma unroll
            for (int i = 0; i < 8; i += 2)
                mul2(y[i], y[i + 1], bf16_hi(w[8 * g + i]), bf16_hi(w[8 * g + i + 1]), fb, fb);
            cb[g] = e2m1x8_rne(y);
        }
        // stage: column 2cp + h, rows 32rb .. 32rb+31 -> 16 bytes at 16 rb
        *reinterpret_cast<uint4*>(stg + (2 * cp) * kMx4StgPitch + 16 * rb) = make_uint4(ca[0], ca[1], ca[2], ca[3]);
        *reinterpret_cast<uint4*>(stg + (2 * cp + 1) * kMx4StgPitch + 16 * rb) = make_uint4(cb[0], cb[1], cb[2], cb[3]);
        stg_e8[(2 * cp) * 2 + rb] = (uint8_t)ea;
        stg_e8[(2 * cp + 1) * 2 + rb] = (uint8_t)eb;
        }
        // the four column warps' staged codes -> whole 32-byte sectors: lanes
        // 2k and 2k+1 store the two halves of one column's 64 rows
        asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int i = threadIdx.x + 128 * j;  // 16-byte chunk: column i/2, half i%2
            const int c = i >> 1, h = i & 1;
            if (c < nc && 32 * h < nr)
                *reinterpret_cast<uint4*>(a.q_col + (c0 + c) * (a.rows / 2) + r0 / 2 + 16 * h) =
                    *reinterpret_cast<const uint4*>(stg + c * kMx4StgPitch + 16 * h);
        }
        {
            const int c = threadIdx.x;  // 0..127: column c's scale bytes
            if (c < nc) {
                a.e8_col[mx4_sf_off(a, c0 + c, r0 / 32, a.rows / 32)] = stg_e8[2 * c];
                if (nr > 32) a.e8_col[mx4_sf_off(a, c0 + c, r0 / 32 + 1, a.rows / 32)] = stg_e8[2 * c + 1];
            }
        }
    } else {
        if (!a.q_row) return;
        // rowwise: block blk (32 columns) of row r, for r = t/4 and t/4 + 32
        const int u = threadIdx.x - 128;
        const int blk = u & 3;
        if (32 * blk >= nc) return;
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
            const int r = (u >> 2) + 32 * pass;
            if (r >= nr) break;
            uint4 p[4];
            float m = 0.0f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                p[q] = *reinterpret_cast<const uint4*>(tile + r * kMx4Pitch + 64 * blk + 16 * q);
                m = absmax3(m, bf16_lo(p[q].x), bf16_hi(p[q].x));
                m = absmax3(m, bf16_lo(p[q].y), bf16_hi(p[q].y));
                m = absmax3(m, bf16_lo(p[q].z), bf16_hi(p[q].z));
                m = absmax3(m, bf16_lo(p[q].w), bf16_hi(p[q].w));
            }
            float f;
            const uint32_t e8 = mx4_scale(m, f);
            const int64_t row = r0 + r, cg = c0 + 32 * blk;
            *reinterpret_cast<uint4*>(a.q_row + row * (a.cols / 2) + cg / 2) =
                make_uint4(mx4_codes8(p[0].x, p[0].y, p[0].z, p[0].w, f),
                           mx4_codes8(p[1].x, p[1].y, p[1].z, p[1].w, f),
                           mx4_codes8(p[2].x, p[2].y, p[2].z, p[2].w, f),
                           mx4_codes8(p[3].x, p[3].y, p[3].z, p[3].w, f));
            a.e8_row[mx4_sf_off(a, row, cg / 32, a.cols / 32)] = (uint8_t)e8;
        }
    }
}

__global__ void __launch_bounds__(kMx4Threads, 3) mxfp4_kernel(const Mx4Args a)
{
    __shared__ __align__(16) uint8_t tiles[2][kMx4TileRows * kMx4Pitch];
    __shared__ __align__(16) uint8_t stg[kMx4TileCols * kMx4StgPitch];
    __shared__ uint8_t stg_e8[kMx4TileCols * 2];
    const int64_t n_tiles = a.tiles_r * a.tiles_c;
    int64_t t = blockIdx.x;
    if (t >= n_tiles) return;
    mx4_issue_tile(a, t, tiles[0]);
    for (int k = 0; t < n_tiles; ++k, t += gridDim.x) {
        const int64_t nt = t + gridDim.x;
        if (nt < n_tiles) {
            mx4_issue_tile(a, nt, tiles[(k + 1) & 1]);
            asm volatile("cp.async.wait_group 1;" ::: "memory");  // tile t has landed
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        mx4_tile(a, t, tiles[k & 1], stg, stg_e8);
        __syncthreads();  // buffer k & 1 is refilled two tiles later
    }
}

bool aligned16_ptr(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Resident CTAs per device (the persistent grid); 0 when the device is not sm_100.
int mx4_grid(int dev)
{
    static int grids[64];
    static std::once_flag flags[64];
    std::call_once(flags[dev & 63], [dev]() {
        int major = 0, sms = 0, per_sm = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            major != 10 ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, mxfp4_kernel, kMx4Threads, 0) !=
                cudaSuccess)
            return;
        grids[dev & 63] = sms * (per_sm > 0 ? per_sm : 1);
    });
    return grids[dev & 63];
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status mxfp4_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                       int directions, int sf_layout, uint8_t* q_row,
                                       uint8_t* e8_row, uint8_t* q_col, uint8_t* e8_col,
                                       void* stream)
{
    if (!x_bf16 || directions == 0 || (directions & ~3)) return NVFP4_ERR_INVALID_ARG;
    if (sf_layout != NVFP4_SF_ROWMAJOR && sf_layout != NVFP4_SF_MMA) return NVFP4_ERR_INVALID_ARG;
    const bool row = (directions & NVFP4_ROWWISE) != 0, col = (directions & NVFP4_COLWISE) != 0;
    if ((row && (!q_row || !e8_row)) || (col && (!q_col || !e8_col))) return NVFP4_ERR_INVALID_ARG;
    if (rows <= 0 || cols <= 0 || rows % 32 || cols % 32 || ld < cols) return NVFP4_ERR_SHAPE;
    if (sf_layout == NVFP4_SF_MMA && ((row && cols % 128) || (col && rows % 128))) return NVFP4_ERR_SHAPE;
    if (rows > ((int64_t)1 << 31) || cols > ((int64_t)1 << 31)) return NVFP4_ERR_SHAPE;
    if (!aligned16_ptr(x_bf16) || ld % 8 || (row && !aligned16_ptr(q_row)) ||
        (col && !aligned16_ptr(q_col)))
        return NVFP4_ERR_ALIGN;
    const int64_t tiles_r = (rows + kMx4TileRows - 1) / kMx4TileRows;
    const int64_t tiles_c = (cols + kMx4TileCols - 1) / kMx4TileCols;
    if (tiles_r * tiles_c > 0x7FFFFFFFll) return NVFP4_ERR_SHAPE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    const int grid = mx4_grid(dev);
    if (grid <= 0) return NVFP4_ERR_UNSUPPORTED;
    Mx4Args a{};
    a.x = static_cast<const uint16_t*>(x_bf16);
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.q_row = row ? q_row : nullptr;
    a.e8_row = row ? e8_row : nullptr;
    a.q_col = col ? q_col : nullptr;
    a.e8_col = col ? e8_col : nullptr;
    a.tiles_r = tiles_r;
    a.tiles_c = tiles_c;
    a.mma_sf = sf_layout == NVFP4_SF_MMA;
    const int64_t n_tiles = tiles_r * tiles_c;
    mxfp4_kernel<<<(unsigned)(n_tiles < grid ? n_tiles : grid), kMx4Threads, 0,
                   static_cast<cudaStream_t>(stream)>>>(a);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
