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
// Kernel eq_gemm_symbols_kernel, one CTA per 256-token x 128-row output tile
// (two token halves sharing each widened weight tile), 8 producer warps and
// one MMA warp:
//   producers  per K slab of 64: one TMA tensor copy of the token tile
//              (issued by thread 0, 128-byte swizzle: the K-major layout the
//              MMA reads, 16-byte chunk c of row r at chunk position
//              c ^ (r % 8), 8-row groups 1024 B apart) and cp.async copies of
//              the symbol bytes into a staging area, issued kAhead slabs
//              ahead into a ring of kStages stages; once a thread's copies of
//              a slab have landed it widens its own symbol chunks into the
//              swizzled bf16 tile and its warp arrives on the stage's "full"
//              mbarrier (which also waits for the tensor copy's bytes); a
//              stage is refilled only after its "empty" barrier says the
//              tensor core is done with it
//   MMA warp   one lane waits for "full", issues 4 x 2 tcgen05.mma (M 128,
//              N 128, K 16; token half h into the fp32 accumulator in TMEM
//              columns 128 h .. 128 h + 127) and tcgen05.commit to the
//              stage's "empty" barrier; a last commit to "done" releases the
//              epilogue
//   epilogue   producer warp w reads accumulator lanes 32 (w % 4) with
//              tcgen05.ld, multiplies by the row scales and stores fp32
// Every mbarrier wait is bounded; on expiry the CTA records EQ_DEV_TIMEOUT,
// still releases its tensor memory and stops.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>

#include "eqw_device.cuh"

namespace {

#ifndef EQ_GEMM_THREADS
#define EQ_GEMM_THREADS 256
#endif
#ifndef EQ_GEMM_TMEM_A
#define EQ_GEMM_TMEM_A 1
#endif
constexpr int kGemmThreads = EQ_GEMM_THREADS;  // 4 or 8 warps
// Token halves per CTA: each widened weight tile feeds kHalves MMAs of 128
// tokens into kHalves accumulators (one instruction shape, M = 128, whatever
// the CTA's token tile).
#ifndef EQ_GEMM_HALVES
#define EQ_GEMM_HALVES 2
#endif
#ifndef EQ_GEMM_STAGES
#define EQ_GEMM_STAGES 4
#endif
static_assert(EQ_GEMM_HALVES >= 1 && EQ_GEMM_HALVES <= 4, "one to four 128-token parts per CTA");
constexpr uint32_t kMmaM = 128;                        // tokens per MMA (accumulator lanes)
constexpr uint32_t kHalves = EQ_GEMM_HALVES;           // MMAs per widened weight tile
constexpr uint32_t kTileM = kMmaM * kHalves;           // tokens per CTA tile
#ifndef EQ_GEMM_TILE_N
#define EQ_GEMM_TILE_N 128
#endif
constexpr uint32_t kTileN = EQ_GEMM_TILE_N;            // weight rows per tile (MMA N, accumulator columns)
static_assert(kTileN % 16 == 0 && kTileN >= 16 && kTileN <= 256, "cta_group::1 MMA with M = 128: N in 16..256");
#ifndef EQ_GEMM_K
#define EQ_GEMM_K 64
#endif
constexpr uint32_t kTileK = EQ_GEMM_K;                 // K per stage: 64 (128-byte rows) or 32 (64-byte rows)
static_assert(kTileK == 64 || kTileK == 32, "K per stage");
constexpr uint32_t kRowBytes = kTileK * 2;             // one bf16 tile row = one swizzle row
constexpr uint32_t kAtomBytes = 8 * kRowBytes;         // 8-row swizzle atom (SBO)
constexpr uint32_t kMmaK = 16;                         // K per tcgen05.mma (bf16)
constexpr uint32_t kStageBytesA = kTileM * kTileK * 2;  // 16 KiB per 128 tokens
constexpr uint32_t kStageBytesB = kTileN * kTileK * 2;  // 16 KiB
constexpr uint32_t kStages = EQ_GEMM_STAGES;
#ifndef EQ_GEMM_AHEAD
#define EQ_GEMM_AHEAD 2
#endif
constexpr uint32_t kAhead = EQ_GEMM_AHEAD;              // slabs whose copies are in flight ahead of use
static_assert(kAhead < kStages, "a stage is refilled only after its previous slab's MMAs");
constexpr uint32_t kStageBytesS = kTileN * kTileK;      // 8 KiB of symbol bytes (staging)
constexpr uint32_t kStageBytes = kStageBytesA + kStageBytesB + kStageBytesS;
constexpr uint32_t kTmemCols = kTileN * kHalves;        // one fp32 accumulator per token part
// tcgen05.alloc takes a power of two of at least 32 columns
constexpr uint32_t kTmemAlloc = kTmemCols <= 32 ? 32 : kTmemCols <= 64 ? 64 : kTmemCols <= 128 ? 128
                              : kTmemCols <= 256 ? 256 : 512;
static_assert(kTmemCols <= 512, "tensor memory has 512 columns");
constexpr size_t kGemmSmem = kStages * kStageBytes + 1024;

struct GemmParams {
    CUtensorMap tmap_x;       // bf16 [tokens, cols], box kTileK x 128 (one per token part), swizzled
    const uint16_t *x;        // bf16 [tokens, cols]
    const uint8_t *sym;       // [rows, cols]
    const float *scales;      // [rows]
    float *y;                 // [tokens, rows]
    int32_t *status;
    uint32_t tokens, rows, cols;
    uint32_t dtype;
};


// Shared-memory matrix descriptor (tcgen05), K-major: start address, leading
// byte offset, stride byte offset (between 8-row groups), all in 16-byte
// units; version 1; layout type 2 = 128-byte swizzle, 0 = none.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;                        // descriptor version for tcgen05
    // layout type: 2 = 128-byte swizzle (K 64), 4 = 64-byte swizzle (K 32); base
    // offset 0: every tile starts on a 1024-byte boundary
    d |= (uint64_t)(kTileK == 64 ? 2 : 4) << 61;
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N and M of one MMA.  M is the instruction's 128, not the CTA's
// token tile: cta_group::1 takes M = 64 or 128 only, and an M field of 256
// here is an illegal instruction on the GPU.
static_assert(kMmaM == 64 || kMmaM == 128, "cta_group::1 MMA shape");
constexpr uint32_t kInstrDesc = (1u << 4)                 // D format fp32
                              | (1u << 7)                 // A format bf16
                              | (1u << 10)                // B format bf16
                              | ((kTileN >> 3) << 17)     // N / 8
                              | ((kMmaM >> 4) << 24);     // M / 16

// Byte offset of the 16-byte chunk k8 (bf16 8 k8 .. 8 k8 + 7) of tile row
// `row` in the swizzled K-major layout: one tile row per swizzle row, 8-row
// atoms kAtomBytes apart, and chunk k8 of row r at chunk position
// k8 ^ (r % 8) (128-byte swizzle) or k8 ^ ((r / 2) % 4) (64-byte swizzle):
// the XOR of the offset's bits 4.. with its bits 7.. that both the TMA copy
// and the MMA's descriptors apply.
__device__ __forceinline__ uint32_t tile_offset(uint32_t row, uint32_t k8) {
    const uint32_t sw = kTileK == 64 ? (row & 7u) : ((row >> 1) & 3u);
    return (row >> 3) * kAtomBytes + (row & 7u) * kRowBytes + ((k8 ^ sw) << 4);
}

// Descriptor of K step kk (16 bf16) of a tile at `buf`: the start advances by
// 32 bytes per step inside the swizzle row (the hardware applies the XOR),
// LBO unused (16), SBO = one 8-row atom.
__device__ __forceinline__ uint64_t tile_desc(uint32_t buf, uint32_t kk) {
    return smem_desc(buf + kk * 32u, 16u, kAtomBytes);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// 16 symbol bytes -> 16 bf16 (exact), as two 16-byte vectors, without the
// conversion pipe.  Int8: with the sign bit flipped, byte u = v + 128 placed
// under the exponent of 2^23 (bits 0x4B0000uu) is the float 2^23 + 128 + v,
// so one exact fp32 subtraction gives v, whose bf16 is the float's upper
// half (v has at most 8 significant bits).  E4M3: the 7 exponent/mantissa
// bits at bit 20 and the sign at bit 31 are value * 2^-120 as an fp32
// (subnormal codes included), and * 2^120 is exact; again the upper half is
// the bf16 (3 mantissa bits).  Pairs are packed with one byte permute.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

template <int DT>
__device__ __forceinline__ float byte_value(uint32_t w, uint32_t i) {
    if constexpr (DT == EQ_INT8) {
        // bytes of (w ^ 0x80808080) and 0x4B000000: byte i, then 0x00, 0x00, 0x4B
        const uint32_t bits = prmt(w, 0x4B000000u, 0x7440u | i);
        return __fadd_rn(__uint_as_float(bits), -8388736.0f);  // - (2^23 + 128)
    } else {
        const uint32_t b = (w >> (8 * i)) & 0xFFu;
        return __fmul_rn(__uint_as_float(((b & 0x80u) << 24) | ((b & 0x7Fu) << 20)), 0x1p120f);
    }
}

template <int DT>
__device__ __forceinline__ void widen16(uint4 b, uint4 &lo, uint4 &hi) {
    uint32_t w[4] = {b.x, b.y, b.z, b.w};
    if constexpr (DT == EQ_INT8) {
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] ^= 0x80808080u;
    }
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t src = w[i / 2];
        const uint32_t j = 2 * (i & 1);  // bytes j, j + 1 of the word
        const float f0 = byte_value<DT>(src, j), f1 = byte_value<DT>(src, j + 1);
        // upper halves of f0 (low bf16) and f1 (high bf16)
        o[i] = prmt(__float_as_uint(f0), __float_as_uint(f1), 0x7632u);
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

// 16-byte asynchronous copy global -> shared (src_bytes 0: zero fill).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Warp-specialised mainloop: kProducerWarps warps fill a ring of kStages
// shared-memory stages (token tile copied, symbol tile widened) and arrive on
// the stage's "full" barrier (one arrival per warp); the MMA warp's first lane
// waits for "full", issues the slab's 4 MMAs and commits them to the stage's
// "empty" barrier, which the producers wait on before refilling the stage; a
// final commit to "done" releases the epilogue.  No block-wide barrier runs
// inside the loop.
template <int DT>
__global__ void __launch_bounds__(kGemmThreads + 32, 1) eq_gemm_symbols_kernel(const __grid_constant__ GemmParams P) {
    constexpr uint32_t kProducerWarps = kGemmThreads / 32;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full_s[kStages], empty_s[kStages], done_s;
    __shared__ uint32_t tmem_base_s;
    const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
    const bool mma_warp = warp == kProducerWarps;
    // token tiles vary fastest, so the blocks that read one weight tile run
    // together and it comes from DRAM once (the token matrix stays in L2)
    const uint32_t n0 = blockIdx.y * kTileN;   // weight rows (outputs)
    const uint32_t m0 = blockIdx.x * kTileM;   // tokens
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    // stage st: token tile (swizzled bf16), widened symbol tile (swizzled bf16), symbol bytes (staging)
    auto bufA = [&](uint32_t st) { return base + st * kStageBytes; };
    auto bufB = [&](uint32_t st) { return base + st * kStageBytes + kStageBytesA; };
    auto bufS = [&](uint32_t st) { return base + st * kStageBytes + kStageBytesA + kStageBytesB; };
    const uint32_t full0 = smem_u32(&full_s[0]), empty0 = smem_u32(&empty_s[0]), done = smem_u32(&done_s);

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&tmem_base_s)), "r"(kTmemAlloc) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (uint32_t st = 0; st < kStages; ++st) {
            mbar_init(full0 + 8 * st, kProducerWarps + 1u);  // + the token tile's expect_tx arrival
            mbar_init(empty0 + 8 * st, 1);
        }
        mbar_init(done, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    const uint32_t n_slabs = P.cols / kTileK;
    bool ok = true;

    if (!mma_warp) {
        // per thread: kBv 16-byte chunks of the symbol tile (kSymChunks per row)
        constexpr uint32_t kSymChunks = kTileK / 16;
        constexpr uint32_t kBv = kTileN * kSymChunks / kGemmThreads;
        // this thread's copies of slab `it` into stage `st`
        auto issue = [&](uint32_t it, uint32_t st) {
            const uint32_t k0 = it * kTileK;
            // token tile: one TMA tensor copy (x = k0 is a multiple of 64
            // elements, 128 bytes; rows past the last token read as zeros),
            // completing on the stage's "full" barrier
            if (tid == 0) {
                mbar_expect_tx(full0 + 8 * st, kStageBytesA);
#pragma unroll
                for (uint32_t h = 0; h < kHalves; ++h)  // one 128-token box per part
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                        " [%0], [%1, {%2, %3}], [%4];" ::"r"(bufA(st) + h * kMmaM * kRowBytes),
                        "l"(reinterpret_cast<uint64_t>(&P.tmap_x)), "r"(k0), "r"(m0 + h * kMmaM),
                        "r"(full0 + 8 * st)
                        : "memory");
            }
#pragma unroll
            for (uint32_t i = 0; i < kBv; ++i) {
                const uint32_t e = tid + i * kGemmThreads, r = e / kSymChunks, c = e % kSymChunks;
                cp_async16(bufS(st) + e * 16u, P.sym + (size_t)(n0 + r) * P.cols + k0 + 16 * c, 16u);
            }
        };
        // the first kAhead slabs go to stages that start out free
        for (uint32_t it = 0; it < kAhead; ++it) {
            if (it < n_slabs) issue(it, it % kStages);
            cp_async_commit();
        }
        for (uint32_t it = 0; it < n_slabs; ++it) {
            const uint32_t s = it % kStages;
            const uint32_t ahead = it + kAhead;
            if (ahead < n_slabs) {
                const uint32_t sa = ahead % kStages;
                // stage sa last held slab ahead - kStages: wait until its MMAs are done
                // (the decision is warp-uniform: the __syncwarp below needs every lane)
                if (ahead >= kStages &&
                    !__all_sync(0xFFFFFFFFu, mbar_wait_bounded(empty0 + 8 * sa, ((ahead - kStages) / kStages) & 1u))) {
                    ok = false;
                    break;
                }
                issue(ahead, sa);
            }
            cp_async_commit();            // one group per slab, empty past the end
            cp_async_wait<kAhead>();      // this thread's copies of slab `it` have landed
            // widen this thread's own symbol chunks of slab `it`
#pragma unroll
            for (uint32_t i = 0; i < kBv; ++i) {
                const uint32_t e = tid + i * kGemmThreads, r = e / kSymChunks, c = e % kSymChunks;
                uint4 lo, hi;
                widen16<DT>(ld_shared_v4(bufS(s) + e * 16u), lo, hi);
                st_shared_v4(bufB(s) + tile_offset(r, 2 * c), lo);
                st_shared_v4(bufB(s) + tile_offset(r, 2 * c + 1), hi);
            }
            fence_proxy_async_smem();  // copies and stores -> visible to the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(full0 + 8 * s);
        }
        cp_async_wait<0>();
    } else if (lane == 0) {
        for (uint32_t it = 0; it < n_slabs; ++it) {
            const uint32_t s = it % kStages;
            if (!mbar_wait_bounded(full0 + 8 * s, (it / kStages) & 1u)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < kTileK / kMmaK; ++kk)
#pragma unroll
                for (uint32_t h = 0; h < kHalves; ++h)  // half h: tokens 128 h .., accumulator columns 128 h ..
                    tc_mma(tmem + h * kTileN, tile_desc(bufA(s) + h * kMmaM * kRowBytes, kk),
                           tile_desc(bufB(s), kk), (it | kk) != 0u);
            tc_commit(empty0 + 8 * s);
        }
        tc_commit(done);  // completes when every MMA issued above has
    }
    if (!mma_warp) {
        ok = mbar_wait_bounded(done, 0u) && ok;
        tc_fence_after();
        if (__all_sync(0xFFFFFFFFu, ok)) {
            // warp w reads accumulator lanes 32 (w % 4) .. + 31; warps sharing a
            // lane quarter split the columns (half h = columns 128 h ..)
            constexpr uint32_t kColsPerWarp = kTmemCols * 4 / kProducerWarps;
            const uint32_t quarter = warp & 3u, c_first = (warp >> 2) * (kColsPerWarp / 32);
#pragma unroll 1
            for (uint32_t c = c_first; c < c_first + kColsPerWarp / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tmem + ((quarter * 32u) << 16) + c * 32u, r);
                const uint32_t half = c * 32u / kTileN, n_off = c * 32u % kTileN;
                const uint32_t m = m0 + half * kMmaM + quarter * 32u + lane;
                if (m < P.tokens) {
                    float4 *dst = reinterpret_cast<float4 *>(P.y + (size_t)m * P.rows + n0 + n_off);
                    const float4 *sc = reinterpret_cast<const float4 *>(P.scales + n0 + n_off);
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
        }
    }
    if (!ok) atomicOr(P.status, EQ_DEV_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemAlloc)
                     : "memory");
    }
}

// ---- weights in tensor memory -------------------------------------------------------
// eq_gemm_tm_kernel: the same product with the roles of the operands swapped
// and the widened weights never in shared memory.  One CTA per 128-row x
// 256-token output tile; the MMA is M = 128 weight rows (A, read from tensor
// memory) x N = 256 tokens (B, the TMA-copied token tile in shared memory),
// K 16, fp32 accumulator in tensor memory (128 lanes x 256 columns: lane =
// weight row, column = token).  Per K slab of 64:
//   producers  thread (w, l) of the 8 producer warps owns weight row
//              32 (w % 4) + l and half w / 4 of the slab's 64 columns: it
//              loads its 32 symbol bytes straight into registers (one slab
//              ahead), widens them exactly to bf16 and stores them with
//              tcgen05.st into its own tensor-memory lane, in the stage's 16
//              columns of that half (two bf16 per 32-bit column, the lower K
//              index in the low half); thread 0 also issues the token tile's
//              two TMA tensor copies (128 tokens each)
//   MMA warp   one lane waits for "full", issues the slab's 4 MMAs (A from
//              tensor memory, B from the swizzled token tile) and commits them
//              to the stage's "empty" barrier
//   epilogue   thread (w, l) reads its weight row's 128 accumulator columns
//              of half w / 4 (tcgen05.ld), multiplies by its row's scale and
//              stores them, one token column at a time (a warp's 32 lanes
//              write 32 consecutive outputs of one token)
// Shared memory per slab: the token tile written once (32 KB) and read once by
// the MMAs (32 KB), against 128 KB in eq_gemm_symbols_kernel.
constexpr uint32_t kTmTileN = 128;                     // weight rows per CTA (MMA M)
constexpr uint32_t kTmTileT = 256;                     // tokens per CTA (MMA N)
constexpr uint32_t kTmK = 64;                          // K per slab
constexpr uint32_t kTmStages = 4;
constexpr uint32_t kTmBBytes = kTmTileT * kTmK * 2;    // 32 KB token tile per stage
constexpr uint32_t kTmAccCols = kTmTileT;              // fp32 accumulator columns
constexpr uint32_t kTmACols = kTmK / 2;                // tensor-memory columns of one stage's weights
constexpr uint32_t kTmAlloc = 512;                     // accumulator + kTmStages weight stages, rounded up
static_assert(kTmAccCols + kTmStages * kTmACols <= kTmAlloc, "tensor memory columns");
static_assert(kTileK == kTmK, "token map box: 64 columns");
constexpr size_t kTmSmem = kTmStages * kTmBBytes + 1024;
constexpr uint32_t kTmInstrDesc = (1u << 4)                  // D format fp32
                                | (1u << 7)                  // A format bf16
                                | (1u << 10)                 // B format bf16
                                | ((kTmTileT >> 3) << 17)    // N / 8
                                | ((kTmTileN >> 4) << 24);   // M / 16

__device__ __forceinline__ void tc_mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(tmem_d), "r"(tmem_a), "l"(db), "r"(kTmInstrDesc), "r"(accumulate)
        : "memory");
}

// 16 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
        ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
          "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

template <int DT>
__global__ void __launch_bounds__(kGemmThreads + 32, 1) eq_gemm_tm_kernel(const __grid_constant__ GemmParams P) {
    constexpr uint32_t kProducerWarps = kGemmThreads / 32;
    static_assert(kProducerWarps == 8, "two producer warps per tensor-memory lane quarter");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full_s[kTmStages], empty_s[kTmStages], done_s;
    __shared__ uint32_t tmem_base_s;
    const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
    const bool mma_warp = warp == kProducerWarps;
    // token tiles vary fastest, so the blocks that read one weight tile run together
    const uint32_t n0 = blockIdx.y * kTmTileN;  // weight rows
    const uint32_t m0 = blockIdx.x * kTmTileT;  // tokens
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    auto bufB = [&](uint32_t st) { return base + st * kTmBBytes; };
    const uint32_t full0 = smem_u32(&full_s[0]), empty0 = smem_u32(&empty_s[0]), done = smem_u32(&done_s);

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&tmem_base_s)), "r"(kTmAlloc) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (uint32_t st = 0; st < kTmStages; ++st) {
            mbar_init(full0 + 8 * st, kProducerWarps + 1u);  // + the token tile's expect_tx arrival
            mbar_init(empty0 + 8 * st, 1);
        }
        mbar_init(done, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;                 // lane 0, first allocated column
    const uint32_t tmem_a = tmem + kTmAccCols;         // weight stages follow the accumulator
    const uint32_t n_slabs = P.cols / kTmK;
    bool ok = true;

    if (!mma_warp) {
        const uint32_t quarter = warp & 3u, half = warp >> 2;
        const uint32_t lane_base = (quarter * 32u) << 16;
        const uint8_t *src = P.sym + (size_t)(n0 + quarter * 32u + lane) * P.cols + half * 32u;
        uint4 cur0 = ldg_nc_v4(src), cur1 = ldg_nc_v4(src + 16);
        for (uint32_t it = 0; it < n_slabs; ++it) {
            const uint32_t s = it % kTmStages;
            uint4 nx0 = cur0, nx1 = cur1;
            if (it + 1 < n_slabs) {  // next slab's symbols, one slab ahead
                nx0 = ldg_nc_v4(src + (size_t)(it + 1) * kTmK);
                nx1 = ldg_nc_v4(src + (size_t)(it + 1) * kTmK + 16);
            }
            // stage s last held slab it - kTmStages: wait until its MMAs are done
            if (it >= kTmStages) {
                if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(empty0 + 8 * s, ((it - kTmStages) / kTmStages) & 1u))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            if (tid == 0) {
                // token tile: two TMA tensor copies of 128 tokens (x = k0, a multiple of
                // 64 elements; rows past the last token read as zeros)
                mbar_expect_tx(full0 + 8 * s, kTmBBytes);
#pragma unroll
                for (uint32_t h = 0; h < 2; ++h)
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                        " [%0], [%1, {%2, %3}], [%4];" ::"r"(bufB(s) + h * kMmaM * kRowBytes),
                        "l"(reinterpret_cast<uint64_t>(&P.tmap_x)), "r"(it * kTmK), "r"(m0 + h * kMmaM),
                        "r"(full0 + 8 * s)
                        : "memory");
            }
            // this row's 32 symbols of the slab, widened exactly, into its tensor-memory lane
            uint4 lo0, hi0, lo1, hi1;
            widen16<DT>(cur0, lo0, hi0);
            widen16<DT>(cur1, lo1, hi1);
            const uint32_t v[16] = {lo0.x, lo0.y, lo0.z, lo0.w, hi0.x, hi0.y, hi0.z, hi0.w,
                                    lo1.x, lo1.y, lo1.z, lo1.w, hi1.x, hi1.y, hi1.z, hi1.w};
            tmem_st16(tmem_a + lane_base + s * kTmACols + half * (kTmACols / 2), v);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(full0 + 8 * s);
            cur0 = nx0;
            cur1 = nx1;
        }
    } else if (lane == 0) {
        for (uint32_t it = 0; it < n_slabs; ++it) {
            const uint32_t s = it % kTmStages;
            if (!mbar_wait_bounded(full0 + 8 * s, (it / kTmStages) & 1u)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < kTmK / kMmaK; ++kk)
                tc_mma_ts(tmem, tmem_a + s * kTmACols + kk * (kMmaK / 2), tile_desc(bufB(s), kk), (it | kk) != 0u);
            tc_commit(empty0 + 8 * s);
        }
        tc_commit(done);  // completes when every MMA issued above has
    }
    if (!mma_warp) {
        ok = mbar_wait_bounded(done, 0u) && ok;
        tc_fence_after();
        if (__all_sync(0xFFFFFFFFu, ok)) {
            // thread (w, l): weight row 32 (w % 4) + l, tokens 128 (w / 4) ..
            const uint32_t quarter = warp & 3u, half = warp >> 2;
            const uint32_t r = n0 + quarter * 32u + lane;
            const float sc = __ldg(P.scales + r);
#pragma unroll 1
            for (uint32_t c = 0; c < kTmAccCols / 2; c += 32) {
                uint32_t acc[32];
                tmem_ld32(tmem + ((quarter * 32u) << 16) + half * (kTmAccCols / 2) + c, acc);
                const uint32_t t0 = m0 + half * (kTmAccCols / 2) + c;
#pragma unroll
                for (uint32_t j = 0; j < 32; ++j)
                    if (t0 + j < P.tokens) P.y[(size_t)(t0 + j) * P.rows + r] = __fmul_rn(__uint_as_float(acc[j]), sc);
            }
        }
    }
    if (!ok) atomicOr(P.status, EQ_DEV_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmAlloc)
                     : "memory");
    }
}

// Failure-path check of the GEMM's waits: the GEMM's own set-up (TMEM
// allocation, "full" / "empty" / "done" barriers with its arrival counts) and
// exit path (status flag, TMEM release), but no producer ever arrives on
// "full", so the MMA lane's bounded wait must give up; it then arrives on
// "done" itself, the producers pass it (or give up on it) and the block
// returns with EQ_DEV_TIMEOUT set and its TMEM freed.
__global__ void __launch_bounds__(kGemmThreads + 32, 1) eq_gemm_wait_timeout_kernel(int32_t *status) {
    constexpr uint32_t kProducerWarps = kGemmThreads / 32;
    __shared__ __align__(8) uint64_t full_s[kStages], empty_s[kStages], done_s;
    __shared__ uint32_t tmem_base_s;
    const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
    const uint32_t full0 = smem_u32(&full_s[0]), empty0 = smem_u32(&empty_s[0]), done = smem_u32(&done_s);
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&tmem_base_s)), "r"(kTmemAlloc) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (uint32_t st = 0; st < kStages; ++st) {
            mbar_init(full0 + 8 * st, kProducerWarps + 1u);
            mbar_init(empty0 + 8 * st, 1);
        }
        mbar_init(done, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    bool ok = true;
    if (warp == kProducerWarps) {
        if (lane == 0) {
            ok = mbar_wait_bounded(full0, 0u);  // nothing arrives: gives up after the limit
            mbar_arrive(done);                  // releases the producers (synchronous: nothing left in flight)
        }
    } else {
        ok = mbar_wait_bounded(done, 0u);
    }
    if (!ok) atomicOr(status, EQ_DEV_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemAlloc)
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

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Tensor map of the token matrix: inner dimension cols (K), outer tokens;
// box kTileK x kTileM with the swizzle the MMA descriptors expect.
int encode_token_map(CUtensorMap *map, const void *x, uint32_t tokens, uint32_t cols) {
    auto enc = tensor_map_encoder();
    if (!enc) return EQ_ERR_CUDA;
    const cuuint64_t dims[2] = {cols, tokens};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2u};
    const cuuint32_t box[2] = {kTileK, kMmaM};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE,
                           kTileK == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? EQ_OK : EQ_ERR_CUDA;
}

}  // namespace

extern "C" EQW_API int eq_gemm_symbols(const eq_model *m, uint32_t matrix, const void *d_sym, const void *d_x,
                                       uint32_t tokens, float *d_y, int32_t *d_status, cudaStream_t s) {
    const eqw::NvtxScope nvtx_range("eq_gemm_symbols");
    if (!m || !d_status || matrix >= m->mats.size()) return EQ_ERR_INVALID_ARG;
    const MatrixDesc &d = m->mats[matrix];
    const eq_matrix_info &in = d.info;
    if (!tokens || !in.rows || !in.cols) return EQ_OK;
    if (in.rows % kTileN || in.cols % kTileK || in.rows / kTileN > 65535u) return EQ_ERR_UNSUPPORTED;
    if (!d_sym || !d_x || !d_y) return EQ_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(d_sym) % 16 || reinterpret_cast<uintptr_t>(d_x) % 16 ||
        reinterpret_cast<uintptr_t>(d_y) % 16 || d.scales_off % 16)
        return EQ_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return EQ_ERR_CUDA;
    GemmParams P{};
    if (const int rc = encode_token_map(&P.tmap_x, d_x, tokens, in.cols)) return rc;
    P.x = static_cast<const uint16_t *>(d_x);
    P.sym = static_cast<const uint8_t *>(d_sym);
    P.scales = reinterpret_cast<const float *>(m->d_blob + d.scales_off);
    P.y = d_y;
    P.status = d_status;
    P.tokens = tokens;
    P.rows = in.rows;
    P.cols = in.cols;
    P.dtype = in.dtype;
#if EQ_GEMM_TMEM_A
    auto fn = in.dtype == EQ_INT8 ? eq_gemm_tm_kernel<EQ_INT8> : eq_gemm_tm_kernel<EQ_E4M3>;
    const size_t smem = kTmSmem;
    const dim3 grid((tokens + kTmTileT - 1) / kTmTileT, in.rows / kTmTileN);
#else
    auto fn = in.dtype == EQ_INT8 ? eq_gemm_symbols_kernel<EQ_INT8> : eq_gemm_symbols_kernel<EQ_E4M3>;
    const size_t smem = kGemmSmem;
    const dim3 grid((tokens + kTileM - 1) / kTileM, in.rows / kTileN);
#endif
    bool &attr = g_gemm_attr_set[dev][in.dtype - 1];
    if (!attr) {
        if (cudaFuncSetAttribute(reinterpret_cast<const void *>(fn), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return EQ_ERR_CUDA;
        attr = true;
    }
    fn<<<grid, kGemmThreads + 32, smem, s>>>(P);
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

extern "C" EQW_API int eq_selftest_gemm_wait_timeout(int32_t *d_status, cudaStream_t s) {
    if (!d_status) return EQ_ERR_INVALID_ARG;
    eq_gemm_wait_timeout_kernel<<<1, kGemmThreads + 32, 0, s>>>(d_status);
    return cudaGetLastError() == cudaSuccess ? EQ_OK : EQ_ERR_CUDA;
}
