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
// One CTA per 64 x 128 tile: the tile is loaded once into shared memory with
// coalesced 16-byte loads; warps 0..3 quantise its columns (thread = column
// pair x 32-row block, one 32-bit shared load per row gives both columns),
// warps 4..7 its rows (thread = row x 64-column half, two blocks).  The
// kernel is HBM-bound: 2 bytes read and 0.5 + 1/32 written per element and
// direction.
#include "common.cuh"

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
    int64_t tiles_c;
};

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p)
{
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
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

// 32 values -> 16 code bytes (element 0 in the low nibble of byte 0).
__device__ __forceinline__ uint4 mx4_codes(const float (&v)[32], float factor)
{
    uint32_t c[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        float y[8];
#pragma unroll
        for (int i = 0; i < 8; i += 2) mul2(y[i], y[i + 1], v[8 * g + i], v[8 * g + i + 1], factor, factor);
        c[g] = e2m1x8_rne(y);
    }
    return make_uint4(c[0], c[1], c[2], c[3]);
}

__global__ void __launch_bounds__(kMx4Threads) mxfp4_kernel(const Mx4Args a)
{
    __shared__ __align__(16) uint8_t tile[kMx4TileRows * kMx4Pitch];
    const int64_t tr = blockIdx.x / a.tiles_c, tcol = blockIdx.x - tr * a.tiles_c;
    const int64_t r0 = tr * kMx4TileRows, c0 = tcol * kMx4TileCols;
    // valid extent of the tile: multiples of 32 (rows and cols are)
    const int nr = a.rows - r0 < kMx4TileRows ? (int)(a.rows - r0) : kMx4TileRows;
    const int nc = a.cols - c0 < kMx4TileCols ? (int)(a.cols - c0) : kMx4TileCols;

    // 64 rows x 16 chunks of 8 elements; chunks past the tensor are zeros
    // and only ever feed blocks that are not stored.
#pragma unroll
    for (int i = threadIdx.x; i < kMx4TileRows * 16; i += kMx4Threads) {
        const int r = i >> 4, q = i & 15;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < nr && 8 * q < nc) v = ldg_nc_v4(a.x + (r0 + r) * a.ld + c0 + 8 * q);
        *reinterpret_cast<uint4*>(tile + r * kMx4Pitch + 16 * q) = v;
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < 4) {
        if (!a.q_col) return;
        // columnwise: column pair cp (columns 2cp, 2cp + 1), 32-row block rb
        const int cp = 32 * (warp & 1) + lane, rb = warp >> 1;
        if (2 * cp >= nc || 32 * rb >= nr) return;
        float va[32], vb[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(tile + (32 * rb + i) * kMx4Pitch + 4 * cp);
            va[i] = bf16_lo(w);
            vb[i] = bf16_hi(w);
        }
        float fa, fb;
        const uint32_t ea = mx4_scale(absmax16(va + 16, absmax16(va, 0.0f)), fa);
        const uint32_t eb = mx4_scale(absmax16(vb + 16, absmax16(vb, 0.0f)), fb);
        const int64_t col = c0 + 2 * cp, rr = r0 + 32 * rb;
        *reinterpret_cast<uint4*>(a.q_col + col * (a.rows / 2) + rr / 2) = mx4_codes(va, fa);
        *reinterpret_cast<uint4*>(a.q_col + (col + 1) * (a.rows / 2) + rr / 2) = mx4_codes(vb, fb);
        a.e8_col[col * (a.rows / 32) + rr / 32] = (uint8_t)ea;
        a.e8_col[(col + 1) * (a.rows / 32) + rr / 32] = (uint8_t)eb;
    } else {
        if (!a.q_row) return;
        // rowwise: row r, 64-column half h (two 32-blocks)
        const int t = threadIdx.x - 128;
        const int r = t >> 1, h = t & 1;
        if (r >= nr) return;
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
            const int cb = 64 * h + 32 * blk;
            if (cb >= nc) break;
            float v[32];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 p = *reinterpret_cast<const uint4*>(tile + r * kMx4Pitch + 2 * cb + 16 * q);
                v[8 * q + 0] = bf16_lo(p.x), v[8 * q + 1] = bf16_hi(p.x);
                v[8 * q + 2] = bf16_lo(p.y), v[8 * q + 3] = bf16_hi(p.y);
                v[8 * q + 4] = bf16_lo(p.z), v[8 * q + 5] = bf16_hi(p.z);
                v[8 * q + 6] = bf16_lo(p.w), v[8 * q + 7] = bf16_hi(p.w);
            }
            float f;
            const uint32_t e8 = mx4_scale(absmax16(v + 16, absmax16(v, 0.0f)), f);
            const int64_t row = r0 + r, cg = c0 + cb;
            *reinterpret_cast<uint4*>(a.q_row + row * (a.cols / 2) + cg / 2) = mx4_codes(v, f);
            a.e8_row[row * (a.cols / 32) + cg / 32] = (uint8_t)e8;
        }
    }
}

bool aligned16_ptr(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status mxfp4_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                       int directions, uint8_t* q_row, uint8_t* e8_row,
                                       uint8_t* q_col, uint8_t* e8_col, void* stream)
{
    if (!x_bf16 || directions == 0 || (directions & ~3)) return NVFP4_ERR_INVALID_ARG;
    const bool row = (directions & NVFP4_ROWWISE) != 0, col = (directions & NVFP4_COLWISE) != 0;
    if ((row && (!q_row || !e8_row)) || (col && (!q_col || !e8_col))) return NVFP4_ERR_INVALID_ARG;
    if (rows <= 0 || cols <= 0 || rows % 32 || cols % 32 || ld < cols) return NVFP4_ERR_SHAPE;
    if (rows > ((int64_t)1 << 31) || cols > ((int64_t)1 << 31)) return NVFP4_ERR_SHAPE;
    if (!aligned16_ptr(x_bf16) || ld % 8 || (row && !aligned16_ptr(q_row)) ||
        (col && !aligned16_ptr(q_col)))
        return NVFP4_ERR_ALIGN;
    const int64_t tiles_r = (rows + kMx4TileRows - 1) / kMx4TileRows;
    const int64_t tiles_c = (cols + kMx4TileCols - 1) / kMx4TileCols;
    if (tiles_r * tiles_c > 0x7FFFFFFFll) return NVFP4_ERR_SHAPE;
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (major != 10) return NVFP4_ERR_UNSUPPORTED;
    Mx4Args a{};
    a.x = static_cast<const uint16_t*>(x_bf16);
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.q_row = row ? q_row : nullptr;
    a.e8_row = row ? e8_row : nullptr;
    a.q_col = col ? q_col : nullptr;
    a.e8_col = col ? e8_col : nullptr;
    a.tiles_c = tiles_c;
    mxfp4_kernel<<<(unsigned)(tiles_r * tiles_c), kMx4Threads, 0, static_cast<cudaStream_t>(stream)>>>(a);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
