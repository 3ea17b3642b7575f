// Prefill consumer on the 5th-generation tensor cores: eq_gemm_symbols.
//
// EntQuant technical summary (gist.science 2601.22787), section 4: the decode
// overhead is amortised at long sequences, where the forward pass of a linear
// layer is a GEMM over many tokens.  Here the weights arrive as the decoded
// 1-byte symbols (eq_decode_symbols: Int8 or E4M3 codes, half the bytes of
// bf16) plus the container's per-row scales and super weights:
//   Y[t, r] = scale[r] * sum_c X[t, c] * value(sym[r, c])
//             + sum over super weights (r, c, v) of bf16(v) * X[t, c]
// X is bf16 [tokens, cols], Y fp32 [tokens, rows], both row-major.  Every
// Int8 / E4M3 value is exact in bf16, so each tile of symbols is widened
// exactly to bf16 in shared memory and multiplied with tcgen05.mma
// (kind::f16, bf16 x bf16, fp32 accumulator in tensor memory); the row scale
// is applied once per output in the epilogue and the (rare) super weights by
// a small second kernel.
//
// Kernel eq_gemm_symbols_kernel, one CTA per 128 x 128 output tile, 4 warps:
//   stage      K slab of 64: all threads copy the X tile (16-byte loads) and
//              widen the symbol tile into shared memory in the canonical
//              K-major layout without swizzle (8 x 16-byte core matrices,
//              K-adjacent cores 128 B apart, 8-row groups 1024 B apart);
//              two stages alternate so the copy of slab s+1 overlaps the
//              tensor-core work on slab s
//   MMA        one thread issues 4 x tcgen05.mma (M 128, N 128, K 16) per
//              slab and tcgen05.commit to the stage's mbarrier
//   epilogue   warp w reads accumulator lanes 32w..32w+31 with tcgen05.ld,
//              multiplies by the row scales and stores fp32
// Every mbarrier wait is bounded; on expiry the CTA records EQ_DEV_TIMEOUT,
// still releases its tensor memory and stops.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>

#include "eqw_device.cuh"

namespace {

#ifndef EQ_GEMM_THREADS
#define EQ_GEMM_THREADS 256
#endif
constexpr int kGemmThreads = EQ_GEMM_THREADS;  // 4 or 8 warps
// One token tile of 128 per CTA and two stages is the configuration verified
// on the GPU.  Two token halves per CTA (two accumulators fed by one widened
// weight tile) raised an illegal-instruction error there, cause not found;
// it is not used.
#ifndef EQ_GEMM_HALVES
#define EQ_GEMM_HALVES 1
#endif
#ifndef EQ_GEMM_STAGES
#define EQ_GEMM_STAGES 2
#endif
static_assert(EQ_GEMM_HALVES == 1, "two token halves per CTA faulted on the GPU and are not used");
constexpr uint32_t kMmaM = 128;                        // tokens per MMA (accumulator lanes)
constexpr uint32_t kHalves = EQ_GEMM_HALVES;           // MMAs per widened weight tile
constexpr uint32_t kTileM = kMmaM * kHalves;           // tokens per CTA tile
constexpr uint32_t kTileN = 128;                       // weight rows per tile (MMA N, accumulator columns)
constexpr uint32_t kTileK = 64;                        // K per stage
constexpr uint32_t kMmaK = 16;                         // K per tcgen05.mma (bf16)
constexpr uint32_t kStageBytesA = kTileM * kTileK * 2;  // 16 KiB per 128 tokens
constexpr uint32_t kStageBytesB = kTileN * kTileK * 2;  // 16 KiB
constexpr uint32_t kStages = EQ_GEMM_STAGES;
constexpr uint32_t kTmemCols = kTileN * kHalves;        // one fp32 accumulator per token half
constexpr size_t kGemmSmem = kStages * (kStageBytesA + kStageBytesB) + 1024;

struct GemmParams {
    const uint16_t *x;        // bf16 [tokens, cols]
    const uint8_t *sym;       // [rows, cols]
    const float *scales;      // [rows]
    float *y;                 // [tokens, rows]
    int32_t *status;
    uint32_t tokens, rows, cols;
    uint32_t dtype;
};

#ifndef EQ_GEMM_SWIZZLE
#define EQ_GEMM_SWIZZLE 1
#endif

// Shared-memory matrix descriptor (tcgen05), K-major: start address, leading
// byte offset, stride byte offset (between 8-row groups), all in 16-byte
// units; version 1; layout type 2 = 128-byte swizzle, 0 = none.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;                        // descriptor version for tcgen05
    if (EQ_GEMM_SWIZZLE) d |= (uint64_t)2 << 61;   // 128-byte swizzle (base offset 0: tiles 1024-aligned)
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N and M of the tile.
constexpr uint32_t kInstrDesc = (1u << 4)                 // D format fp32
                              | (1u << 7)                 // A format bf16
                              | (1u << 10)                // B format bf16
                              | ((kTileN >> 3) << 17)     // N / 8
                              | ((kTileM >> 4) << 24);    // M / 16

// Byte offset of the 16-byte chunk k8 (bf16 8 k8 .. 8 k8 + 7) of tile row `row`.
// 128-byte swizzle: each 64-element row is one 128-byte line, 8-row groups are
// 1024 bytes apart, and chunk k8 of row r sits at chunk position k8 ^ (r % 8).
// Without swizzle: core matrices of 8 rows x 16 bytes, core (row / 8, k8) at
// ((row / 8) * 8 + k8) * 128 with rows 16 bytes apart inside it.
__device__ __forceinline__ uint32_t tile_offset(uint32_t row, uint32_t k8) {
    if (EQ_GEMM_SWIZZLE) return (row >> 3) * 1024u + (row & 7u) * 128u + ((k8 ^ (row & 7u)) << 4);
    return ((row >> 3) * (kTileK / 8) + k8) * 128u + (row & 7u) * 16u;
}

// Descriptor of K step kk (16 bf16) of a tile at `buf`: 128-byte swizzle
// advances the start by 32 bytes per step (the hardware applies the XOR),
// LBO unused (1), SBO 1024; without swizzle two 128-byte cores per step,
// LBO 128 (K-adjacent cores), SBO 1024 (8-row groups).
__device__ __forceinline__ uint64_t tile_desc(uint32_t buf, uint32_t kk) {
    if (EQ_GEMM_SWIZZLE) return smem_desc(buf + kk * 32u, 16u, 1024u);
    return smem_desc(buf + kk * 256u, 128u, 1024u);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// 16 symbol bytes -> 16 bf16 (exact), as two 16-byte vectors.
template <int DT>
__device__ __forceinline__ void widen16(uint4 b, uint4 &lo, uint4 &hi) {
    const uint32_t w[4] = {b.x, b.y, b.z, b.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t src = w[i / 2] >> (16 * (i & 1));
        const float f0 = symbol_value<DT>(src & 0xFFu), f1 = symbol_value<DT>((src >> 8) & 0xFFu);
        o[i] = pack_bf16x2(make_float2(f0, f1));
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(da), "l"(db), "r"(kInstrDesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

// 32 consecutive fp32 accumulator columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

template <int DT>
__global__ void __launch_bounds__(kGemmThreads) eq_gemm_symbols_kernel(const __grid_constant__ GemmParams P) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t mbar_s[kStages];
    __shared__ uint32_t tmem_base_s;
    const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
    const uint32_t n0 = blockIdx.x * kTileN;   // weight rows (outputs)
    const uint32_t m0 = blockIdx.y * kTileM;   // tokens
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    // stage s: A tile at base + s * (A + B bytes), B tile right after it; its mbarrier at mbar0 + 8 s
    auto bufA = [&](uint32_t st) { return base + st * (kStageBytesA + kStageBytesB); };
    auto bufB = [&](uint32_t st) { return base + st * (kStageBytesA + kStageBytesB) + kStageBytesA; };
    const uint32_t mbar0 = smem_u32(&mbar_s[0]);

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&tmem_base_s)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (uint32_t st = 0; st < kStages; ++st) mbar_init(mbar0 + 8 * st, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;

    const uint32_t n_slabs = P.cols / kTileK;
    // per thread: kXv 16-byte chunks of the X tile and kBv of the symbol tile
    constexpr uint32_t kXv = kTileM * (kTileK / 8) / kGemmThreads;
    constexpr uint32_t kBv = kTileN * (kTileK / 16) / kGemmThreads;
    uint4 xr[kXv], br[kBv];
    // global -> registers for slab `it` (issued one slab ahead of its use)
    auto fetch = [&](uint32_t it) {
        const uint32_t k0 = it * kTileK;
#pragma unroll
        for (uint32_t i = 0; i < kXv; ++i) {
            const uint32_t e = tid + i * kGemmThreads, r = e >> 3, k8 = e & 7u;
            xr[i] = m0 + r < P.tokens
                        ? __ldg(reinterpret_cast<const uint4 *>(P.x + (size_t)(m0 + r) * P.cols + k0) + k8)
                        : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (uint32_t i = 0; i < kBv; ++i) {
            const uint32_t e = tid + i * kGemmThreads, r = e >> 2, c = e & 3u;
            br[i] = __ldg(reinterpret_cast<const uint4 *>(P.sym + (size_t)(n0 + r) * P.cols + k0) + c);
        }
    };
    if (n_slabs) fetch(0);
    bool ok = true;
    for (uint32_t it = 0; it < n_slabs && ok; ++it) {
        const uint32_t s = it % kStages;
        if (it >= kStages) {  // the MMAs that read this stage kStages slabs ago must be done
            // commit number (it - kStages) / kStages of stage s, i.e. the completion of that parity
            ok = mbar_wait_bounded(mbar0 + 8 * s, ((it - kStages) / kStages) & 1u);
            if (!__syncthreads_and(ok)) {
                ok = false;
                break;
            }
        }
        // registers -> stage s: the X tile as is, the symbol tile widened to bf16
#pragma unroll
        for (uint32_t i = 0; i < kXv; ++i) {
            const uint32_t e = tid + i * kGemmThreads;
            st_shared_v4(bufA(s) + tile_offset(e >> 3, e & 7u), xr[i]);
        }
#pragma unroll
        for (uint32_t i = 0; i < kBv; ++i) {
            const uint32_t e = tid + i * kGemmThreads, r = e >> 2, c = e & 3u;
            uint4 lo, hi;
            widen16<DT>(br[i], lo, hi);
            st_shared_v4(bufB(s) + tile_offset(r, 2 * c), lo);
            st_shared_v4(bufB(s) + tile_offset(r, 2 * c + 1), hi);
        }
        if (it + 1 < n_slabs) fetch(it + 1);  // in flight during the barrier and the MMAs
        fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor core
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < kTileK / kMmaK; ++kk) {
                const uint64_t db = tile_desc(bufB(s), kk);
#pragma unroll
                for (uint32_t h = 0; h < kHalves; ++h)  // token half h: A rows 128h.., accumulator columns 128h..
                    tc_mma(tmem + h * kTileN, tile_desc(bufA(s) + h * (kMmaM * kTileK * 2), kk), db,
                           (it | kk) != 0u);
            }
            tc_commit(mbar0 + 8 * s);
        }
    }
    // all MMAs done: the last commit of the last slab covers every earlier MMA of thread 0
    if (ok && n_slabs) {
        // the last commit of every stage (the very last one covers all MMAs of thread 0)
        for (uint32_t j = 0; j < kStages && j < n_slabs && ok; ++j) {
            const uint32_t it = n_slabs - 1 - j;
            ok = mbar_wait_bounded(mbar0 + 8 * (it % kStages), (it / kStages) & 1u);
        }
        ok = __syncthreads_and(ok);
    }
    tc_fence_after();
    if (ok) {
        // warp w may read accumulator lanes 32 (w % 4) .. + 31; the warps that
        // share a lane quarter split the accumulator columns (kHalves x 128)
        constexpr uint32_t kWarps = kGemmThreads / 32, kColsPerWarp = kTmemCols * 4 / kWarps;
        const uint32_t quarter = warp & 3u, c_first = (warp >> 2) * (kColsPerWarp / 32);
#pragma unroll 1
        for (uint32_t c = c_first; c < c_first + kColsPerWarp / 32; ++c) {
            const uint32_t h = c / (kTileN / 32), cn = c % (kTileN / 32);  // token half, column chunk
            const uint32_t m = m0 + h * kMmaM + quarter * 32u + lane;
            uint32_t r[32];
            tmem_ld32(tmem + ((quarter * 32u) << 16) + c * 32u, r);
            if (m < P.tokens) {
                float4 *dst = reinterpret_cast<float4 *>(P.y + (size_t)m * P.rows + n0 + cn * 32u);
                const float4 *sc = reinterpret_cast<const float4 *>(P.scales + n0 + cn * 32u);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 s4 = __ldg(sc + q);
                    dst[q] = make_float4(__fmul_rn(__uint_as_float(r[4 * q]), s4.x),
                                         __fmul_rn(__uint_as_float(r[4 * q + 1]), s4.y),
                                         __fmul_rn(__uint_as_float(r[4 * q + 2]), s4.z),
                                         __fmul_rn(__uint_as_float(r[4 * q + 3]), s4.w));
                }
            }
        }
    } else if (tid == 0) {
        atomicOr(P.status, EQ_DEV_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    }
}

// Super weights: Y[t, r] += bf16(v) * X[t, c], one thread per (super weight, token).
__global__ void eq_gemm_outliers_kernel(const uint32_t *rec, uint32_t n_out, const uint16_t *x, uint32_t tokens,
                                        uint32_t rows, uint32_t cols, float *y, int32_t *status) {
    const uint64_t t = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (uint64_t)n_out * tokens) return;
    const uint32_t o = (uint32_t)(t / tokens), tok = (uint32_t)(t % tokens);
    const uint32_t r = rec[3 * o], c = rec[3 * o + 1];
    if (r >= rows || c >= cols) {
        atomicOr(status, EQ_DEV_BAD_OUTLIER);
        return;
    }
    const float w = __bfloat162float(__float2bfloat16_rn(__uint_as_float(rec[3 * o + 2])));
    const float xv = __uint_as_float((uint32_t)x[(size_t)tok * cols + c] << 16);
    atomicAdd(y + (size_t)tok * rows + r, __fmul_rn(w, xv));
}

bool g_gemm_attr_set[128][2];

}  // namespace

extern "C" EQW_API int eq_gemm_symbols(const eq_model *m, uint32_t matrix, const void *d_sym, const void *d_x,
                                       uint32_t tokens, float *d_y, int32_t *d_status, cudaStream_t s) {
    if (!m || !d_status || matrix >= m->mats.size()) return EQ_ERR_INVALID_ARG;
    const MatrixDesc &d = m->mats[matrix];
    const eq_matrix_info &in = d.info;
    if (!tokens || !in.rows || !in.cols) return EQ_OK;
    if (in.rows % kTileN || in.cols % kTileK) return EQ_ERR_UNSUPPORTED;
    if (!d_sym || !d_x || !d_y) return EQ_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(d_sym) % 16 || reinterpret_cast<uintptr_t>(d_x) % 16 ||
        reinterpret_cast<uintptr_t>(d_y) % 16 || d.scales_off % 16)
        return EQ_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return EQ_ERR_CUDA;
    GemmParams P{};
    P.x = static_cast<const uint16_t *>(d_x);
    P.sym = static_cast<const uint8_t *>(d_sym);
    P.scales = reinterpret_cast<const float *>(m->d_blob + d.scales_off);
    P.y = d_y;
    P.status = d_status;
    P.tokens = tokens;
    P.rows = in.rows;
    P.cols = in.cols;
    P.dtype = in.dtype;
    auto fn = in.dtype == EQ_INT8 ? eq_gemm_symbols_kernel<EQ_INT8> : eq_gemm_symbols_kernel<EQ_E4M3>;
    bool &attr = g_gemm_attr_set[dev][in.dtype - 1];
    if (!attr) {
        if (cudaFuncSetAttribute(reinterpret_cast<const void *>(fn), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kGemmSmem) != cudaSuccess)
            return EQ_ERR_CUDA;
        attr = true;
    }
    const dim3 grid(in.rows / kTileN, (tokens + kTileM - 1) / kTileM);
    fn<<<grid, kGemmThreads, kGemmSmem, s>>>(P);
    if (cudaGetLastError() != cudaSuccess) return EQ_ERR_CUDA;
    if (in.n_outliers) {
        const uint64_t n = (uint64_t)in.n_outliers * tokens;
        eq_gemm_outliers_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
            reinterpret_cast<const uint32_t *>(m->d_blob + d.outliers_off), in.n_outliers,
            static_cast<const uint16_t *>(d_x), tokens, in.rows, in.cols, d_y, d_status);
        if (cudaGetLastError() != cudaSuccess) return EQ_ERR_CUDA;
    }
    return EQ_OK;
}
