// Batch-1 bf16 GEMV, the consumer of a decoded weight block (eq_gemv_bf16).
//
// EntQuant technical summary (gist.science 2601.22787), section 2
// "inference-time decoding": decoded weights land in a buffer that the
// block's forward kernels read right after; at batch 1 the forward of a
// linear layer is y = W x.  This kernel streams W once from HBM (16-byte
// loads, four in flight per lane), keeps x in L1/L2, multiplies and sums in
// fp32 and reduces across the warp: one warp per output row.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "eqw_internal.h"

namespace {

constexpr int kRowsPerCta = 8;

__device__ __forceinline__ float dot8(const uint4 w, const uint4 x) {
    const __nv_bfloat162 *a = reinterpret_cast<const __nv_bfloat162 *>(&w);
    const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&x);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 fa = __bfloat1622float2(a[i]);
        const float2 fb = __bfloat1622float2(b[i]);
        s = fmaf(fa.x, fb.x, s);
        s = fmaf(fa.y, fb.y, s);
    }
    return s;
}

__global__ void __launch_bounds__(kRowsPerCta * 32)
eq_gemv_bf16_kernel(const uint4 *__restrict__ w, const uint4 *__restrict__ x, float *__restrict__ y,
                    uint32_t rows, uint32_t vec_per_row) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t row = blockIdx.x * kRowsPerCta + (threadIdx.x >> 5);
    if (row >= rows) return;
    const uint4 *wr = w + (size_t)row * vec_per_row;
    float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
    uint32_t v = lane;
    for (; v + 96 < vec_per_row; v += 128) {
        const uint4 w0 = __ldcs(wr + v), w1 = __ldcs(wr + v + 32), w2 = __ldcs(wr + v + 64), w3 = __ldcs(wr + v + 96);
        acc0 += dot8(w0, __ldg(x + v));
        acc1 += dot8(w1, __ldg(x + v + 32));
        acc2 += dot8(w2, __ldg(x + v + 64));
        acc3 += dot8(w3, __ldg(x + v + 96));
    }
    for (; v < vec_per_row; v += 32) acc0 += dot8(__ldcs(wr + v), __ldg(x + v));
    float acc = (acc0 + acc1) + (acc2 + acc3);
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, d);
    if (lane == 0) y[row] = acc;
}

}  // namespace

extern "C" EQW_API int eq_gemv_bf16(const void *d_w, const void *d_x, float *d_y, uint32_t rows, uint32_t cols,
                                    cudaStream_t s) {
    const eqw::NvtxScope nvtx_range("eq_gemv_bf16");
    if (!rows) return EQ_OK;
    if (!d_w || !d_x || !d_y || cols % 8) return EQ_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(d_w) % 16 || reinterpret_cast<uintptr_t>(d_x) % 16) return EQ_ERR_INVALID_ARG;
    const uint32_t grid = (rows + kRowsPerCta - 1) / kRowsPerCta;
    eq_gemv_bf16_kernel<<<grid, kRowsPerCta * 32, 0, s>>>(static_cast<const uint4 *>(d_w),
                                                          static_cast<const uint4 *>(d_x), d_y, rows, cols / 8);
    return cudaGetLastError() == cudaSuccess ? EQ_OK : EQ_ERR_CUDA;
}
