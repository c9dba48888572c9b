// moe_comm.cu -- the receiving end of the MXFP8-compressed expert combine.
//
// In expert-parallel MoE training the expert outputs travel back to the
// tokens' ranks; the iitak.ru page ("Thinking Machines uskorila obuchenie
// Inkling 2 Small 4-bitnymi chislami", section "But") has them cross NVLink at
// 8.25 bits per number (an 8-bit element plus an 8-bit scale per 32) instead of
// 16, because compute outran the link.  The sender quantises its rows with
// mxfp8_quantize (rowwise, OCP MX v1.0); after the exchange each rank combines
// the k expert rows of every token:
//   out[t][c] = sum_{j<k} w[t][j] * (e4m3(q[r][c]) * 2^(e8[r][c/32] - 127)),
//   r = slot_row[t][j] (rows with slot_row < 0 are skipped),
// in FP32, one rounding for each product and one for each sum, j in order (so
// the result does not depend on thread scheduling), then RNE to bf16.
#include "common.cuh"

#include <algorithm>
#include <mutex>

namespace nvfp4 {
namespace {

// E4M3 byte -> its value (exact) through the hardware FP8 -> FP16 conversion.
__device__ __forceinline__ void e4m3x2_to_f32(uint32_t two, float& lo, float& hi)
{
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(two)));
    lo = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
    hi = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
}

// 2^(byte - 127) for an E8M0 byte 0..254 (byte 0 is 2^-127, a subnormal float).
__device__ __forceinline__ float e8m0_value(uint32_t b)
{
    return b >= 1 ? __uint_as_float(b << 23) : __uint_as_float(0x00400000u);
}

// One thread = 16 consecutive columns of one token.  The token's slots are
// taken four at a time: their row indices, weights and scale bytes, then their
// 16-byte code loads, are all issued before any is used, so four loads per
// thread are in flight; the sum still runs over j in order.
__global__ void __launch_bounds__(256) mxfp8_combine_kernel(
    const uint8_t* __restrict__ q, const uint8_t* __restrict__ e8, int64_t rows, int64_t cols,
    const int32_t* __restrict__ slot_row, const float* __restrict__ weight, int64_t tokens, int k,
    uint16_t* __restrict__ out, uint32_t* status)
{
    const int64_t groups = cols / 16;
    for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < tokens * groups;
         u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = u / groups, c0 = (u - t * groups) * 16;
        float acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
        for (int j0 = 0; j0 < k; j0 += 4) {
            int32_t r[4];
            float w[4], sc[4];
            uint4 codes[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                r[jj] = j0 + jj < k ? slot_row[t * k + j0 + jj] : -1;
                if (r[jj] >= rows) {
                    record_status(status, NVFP4_ERR_INDEX);
                    r[jj] = -1;
                }
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                if (r[jj] < 0) continue;
                w[jj] = weight[t * k + j0 + jj];
                sc[jj] = e8m0_value(e8[r[jj] * (cols / 32) + c0 / 32]);
                codes[jj] = *reinterpret_cast<const uint4*>(q + r[jj] * cols + c0);
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                if (r[jj] < 0) continue;
                const uint32_t words[4] = {codes[jj].x, codes[jj].y, codes[jj].z, codes[jj].w};
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    float lo, hi;
                    e4m3x2_to_f32((words[p >> 1] >> (16 * (p & 1))) & 0xFFFFu, lo, hi);
                    // the element value is exact: an E4M3 value times a power of two
                    acc[2 * p] = __fadd_rn(acc[2 * p], __fmul_rn(w[jj], __fmul_rn(lo, sc[jj])));
                    acc[2 * p + 1] = __fadd_rn(acc[2 * p + 1], __fmul_rn(w[jj], __fmul_rn(hi, sc[jj])));
                }
            }
        }
        uint32_t packed[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * p], acc[2 * p + 1]);
            packed[p] = *reinterpret_cast<const uint32_t*>(&b);
        }
        uint4* dst = reinterpret_cast<uint4*>(out + t * cols + c0);
        dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    }
}

int combine_grid(int dev)
{
    static int grids[64];
    static std::once_flag flags[64];
    std::call_once(flags[dev & 63], [dev]() {
        int major = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            major != 10 || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return;
        grids[dev & 63] = sms * 8;
    });
    return grids[dev & 63];
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status mxfp8_combine(const uint8_t* q, const uint8_t* e8, int64_t rows,
                                      int64_t cols, const int32_t* slot_row, const float* weight,
                                      int64_t tokens, int k, void* out_bf16, void* workspace,
                                      size_t ws_bytes, void* stream)
{
    if (!slot_row || !weight || !out_bf16 || k < 1 || k > 64) return NVFP4_ERR_INVALID_ARG;
    if (rows < 0 || tokens < 0 || cols <= 0 || cols % 32) return NVFP4_ERR_SHAPE;
    if (rows > 0 && (!q || !e8)) return NVFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(q) & 15u) || (reinterpret_cast<uintptr_t>(out_bf16) & 15u) ||
        (reinterpret_cast<uintptr_t>(slot_row) & 3u) || (reinterpret_cast<uintptr_t>(weight) & 3u))
        return NVFP4_ERR_ALIGN;
    if (workspace && (ws_bytes < 16 || (reinterpret_cast<uintptr_t>(workspace) & 15u)))
        return NVFP4_ERR_WORKSPACE;
    if (tokens == 0) return NVFP4_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    const int grid = combine_grid(dev);
    if (grid <= 0) return NVFP4_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t* status = workspace ? static_cast<uint32_t*>(workspace) + 2 : nullptr;
    if (status && cudaMemsetAsync(status, 0, 4, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    const int64_t units = tokens * (cols / 16);
    const int blocks = (int)std::min<int64_t>((units + 255) / 256, grid);
    mxfp8_combine_kernel<<<blocks, 256, 0, st>>>(q, e8, rows, cols, slot_row, weight, tokens, k,
                                                 static_cast<uint16_t*>(out_bf16), status);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
