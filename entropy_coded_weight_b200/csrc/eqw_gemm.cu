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
// Int8 / E4M3 value is exact in bf16, so each slab of symbols is widened
// exactly to bf16 and multiplied with tcgen05.mma (kind::f16, bf16 x bf16,
// fp32 accumulator in tensor memory); the row scale is applied once per
// output in the epilogue and the (rare) super weights by a small second
// kernel.
//
// Two kernels, chosen per launch by the host:
//   eq_gemm_symbols_pair_kernel  (tcgen05.mma.cta_group::2, M = 256 over a pair
//                                of CTAs on two SMs) for 256-token tiles when
//                                every matrix has a multiple of 256 rows; it is
//                                described where it is defined, below;
//   eq_gemm_symbols_kernel       (cta_group::1, M = 128) otherwise, and with
//                                128-token tiles for inputs of <= 128 tokens.
//
// Kernel eq_gemm_symbols_kernel: a persistent launch (one CTA per SM) over the
// 128-row x 256-token output tiles of up to 8 matrices of one weight type (a
// transformer block's projections in one launch; the matrix with the longest
// K first, CTA b taking tiles b, b + grid, ...).  The MMA is M = 128 weight
// rows (A, read from tensor memory) x N = 256 tokens (B, in shared memory) x
// K 16, with the fp32 accumulator in tensor memory (128 lanes x 256 columns:
// lane = weight row, column = token).  Three roles per CTA, over a ring of 5
// stages (one K slab of 64 each):
//   loader     one lane of warp 9: for each slab, once the stage's "empty"
//              barrier says the tensor core is done with it, arms the stage's
//              "load" barrier and issues three TMA tensor copies: the token
//              tile (two boxes of 128 tokens x 64 bf16, 128-byte swizzle: the
//              K-major layout the MMA's B descriptor reads, 16-byte chunk c of
//              row r at chunk c ^ (r % 8), 8-row groups 1024 B apart) and the
//              symbol tile (128 rows x 64 bytes, 64-byte swizzle)
//   producers  warps 0-7; thread (w, l) owns weight row 32 (w % 4) + l and
//              half w / 4 of the slab's 64 columns: after "load" it reads its
//              32 symbol bytes from the symbol tile (conflict-free thanks to
//              the swizzle), widens them exactly to bf16 and stores them with
//              tcgen05.st into its own tensor-memory lane, in the stage's 16
//              columns of that half (two bf16 per 32-bit column, the lower K
//              index in the low half); the warp arrives on the stage's "full"
//              barrier once the store has completed (checked one slab later,
//              so that the store's latency overlaps the next slab's work)
//   MMA warp   one lane waits for "full" (and "load"), issues the slab's 4
//              MMAs and tcgen05.commits them to the stage's "empty" barrier; a
//              commit to "done" after a tile's last slab releases the epilogue
//   epilogue   the producers: thread (w, l) reads its weight row's 128
//              accumulator columns of half w / 4 (tcgen05.ld), multiplies by
//              the row's scale and stores them one token column at a time (a
//              warp's 32 lanes write 32 consecutive outputs of one token), then
//              arrives on "acc_free", which the MMA lane waits for before the
//              next tile's first MMA; the stage ring runs on across tiles, so
//              the loader fetches the next tile's first slabs meanwhile
// Shared memory per stage: 32 KB token tile + 8 KB symbol tile; the widened
// weights never touch it.
// Every mbarrier wait is bounded; on expiry the CTA records EQ_DEV_TIMEOUT,
// still releases its tensor memory and stops.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "eqw_device.cuh"

namespace {

constexpr uint32_t kProducerWarps = 8;                 // two per tensor-memory lane quarter
constexpr uint32_t kParts = kProducerWarps / 4;        // producer warps sharing a lane quarter's slab
constexpr int kGemmThreads = (kProducerWarps + 2) * 32; // + the MMA warp and the loader warp
constexpr uint32_t kTileN = 128;                       // weight rows per CTA (MMA M, accumulator lanes)
constexpr uint32_t kTileK = 64;                        // K per slab (128-byte rows: the 128-byte swizzle)
constexpr uint32_t kBoxT = 128;                        // tokens per TMA box
constexpr uint32_t kRowBytes = kTileK * 2;             // one bf16 token row of a slab = one swizzle row
constexpr uint32_t kAtomBytes = 8 * kRowBytes;         // 8-row swizzle atom (SBO)
constexpr uint32_t kMmaK = 16;                         // K per tcgen05.mma (bf16)
constexpr uint32_t kWBytes = kTileN * kTileK;          // symbol tile of a stage, 8 KB
constexpr uint32_t kACols = kTileK / 2;                // tensor-memory columns of one stage's weights
constexpr uint32_t kPartBytes = kTileK / kParts;       // symbol bytes one producer thread widens per slab
constexpr uint32_t kPartCols = kACols / kParts;        // tensor-memory columns it stores them in
static_assert(kParts == 2 || kParts == 4, "a producer thread takes 32 or 16 bytes of its row's slab");
constexpr uint32_t kTmemAlloc = 512;                   // accumulator + the weight stages, rounded up

// The token-tile width TT (MMA N) fixes the rest: 256 tokens for long inputs
// (5 stages of 32 + 8 KB), 128 for short ones (8 stages of 16 + 8 KB: the
// weights are then read once, and the MMA does no work on absent tokens).
template <uint32_t TT>
struct GemmShape {
    static_assert(TT == 128 || TT == 256, "token tile");
    static constexpr uint32_t kTileT = TT;                       // tokens per tile (MMA N, accumulator columns)
    static constexpr uint32_t kStages = TT == 256 ? 5 : 8;
    static constexpr uint32_t kXBytes = TT * kTileK * 2;         // token tile of a stage
    static constexpr uint32_t kStageBytes = kXBytes + kWBytes;   // both land on the stage's "load" barrier
    static constexpr uint32_t kAccCols = TT;                     // fp32 accumulator columns
    static constexpr size_t kSmem = kStages * kStageBytes + 1024;
    // instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
    // K-major, N = TT tokens, M = 128 weight rows (cta_group::1 takes M = 64
    // or 128 only)
    static constexpr uint32_t kInstrDesc = (1u << 4)             // D format fp32
                                         | (1u << 7)             // A format bf16
                                         | (1u << 10)            // B format bf16
                                         | ((TT >> 3) << 17)     // N / 8
                                         | ((kTileN >> 4) << 24);  // M / 16
    static_assert(kAccCols + kStages * kACols <= kTmemAlloc, "tensor memory columns");
    static_assert(kSmem <= 227u * 1024u, "shared memory per block");
    static_assert(kTileN == 128 && TT % 16 == 0 && TT <= 256, "cta_group::1 MMA shape");
};

constexpr uint32_t kMaxGemmJobs = 8;
constexpr uint32_t kNarrowTokens = 128;  // inputs up to this many tokens take the 128-token tile  // matrices per launch (a transformer block has 7)

// One matrix of a launch: its tiles are [first_tile, first_tile + rows / 128 *
// token tiles), weight-row tile major, token tile fastest.
struct GemmJob {
    CUtensorMap tmap_x;       // bf16 [tokens, cols] input of this matrix, box kTileK x kBoxT, 128-byte swizzle
    CUtensorMap tmap_w;       // uint8 [rows, cols] symbols, box kTileK x kTileN, 64-byte swizzle
    const uint8_t *sym;       // [rows, cols]
    const float *scales;      // [rows]
    float *y;                 // [tokens, rows]
    uint32_t rows, cols;
    uint32_t first_tile;
    uint32_t pad;
};

struct GemmParams {
    int32_t *status;
    uint32_t tokens;
    uint32_t t_tiles;         // token tiles per weight-row tile
    uint32_t n_jobs;
    uint32_t total_tiles;
    GemmJob jobs[kMaxGemmJobs];
};
static_assert(sizeof(GemmParams) <= 4096, "kernel parameter space");

// Shared-memory matrix descriptor (tcgen05), K-major: start address, leading
// byte offset, stride byte offset (between 8-row groups), all in 16-byte
// units; version 1; layout type 2 = 128-byte swizzle, 0 = none.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;                        // descriptor version for tcgen05
    // layout type 2 = 128-byte swizzle; base offset 0: every tile starts on a
    // 1024-byte boundary
    d |= (uint64_t)2 << 61;
    return d;
}


// Descriptor of K step kk (16 bf16) of a tile at `buf`: the start advances by
// 32 bytes per step inside the swizzle row (the hardware applies the XOR),
// LBO unused (16), SBO = one 8-row atom.
__device__ __forceinline__ uint64_t tile_desc(uint32_t buf, uint32_t kk) {
    return smem_desc(buf + kk * 32u, 16u, kAtomBytes);
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

// Non-blocking check that the phase with parity `parity` has completed (acquire).
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

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

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(tmem_d), "r"(tmem_a), "l"(db), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 16 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
        ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
          "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// 8 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t *v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
                   "r"(v[7])
                 : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 16-byte chunk c (0..3) of weight row `row` in a slab's 64-byte-swizzled
// symbol tile (chunk c of row r is stored at chunk c ^ ((r >> 1) & 3) of the
// row): the 32 lanes of a warp (32 consecutive rows) reading the same c hit 8
// distinct 16-byte bank groups per 128 bytes, no conflicts.
__device__ __forceinline__ uint4 lds_sym16(uint32_t tile, uint32_t row, uint32_t c) {
    const uint32_t addr = tile + row * kTileK + ((c ^ ((row >> 1) & 3u)) << 4);
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

template <int DT, uint32_t TT>
__global__ void __launch_bounds__(kGemmThreads, 1) eq_gemm_symbols_kernel(const __grid_constant__ GemmParams P) {
    using S = GemmShape<TT>;
    constexpr uint32_t kStages = S::kStages, kStageBytes = S::kStageBytes, kXBytes = S::kXBytes;
    constexpr uint32_t kTileT = S::kTileT, kAccCols = S::kAccCols;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t load_s[kStages], full_s[kStages], empty_s[kStages], done_s, acc_free_s;
    __shared__ uint32_t tmem_base_s;
    __shared__ volatile uint32_t abort_s;  // a bounded wait gave up: every role stops
    const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    auto bufB = [&](uint32_t st) { return base + st * kStageBytes; };            // token tile
    auto bufW = [&](uint32_t st) { return base + st * kStageBytes + kXBytes; };  // symbol tile
    const uint32_t load0 = smem_u32(&load_s[0]), full0 = smem_u32(&full_s[0]), empty0 = smem_u32(&empty_s[0]);
    const uint32_t done = smem_u32(&done_s), acc_free = smem_u32(&acc_free_s);

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&tmem_base_s)), "r"(kTmemAlloc) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (uint32_t st = 0; st < kStages; ++st) {
            mbar_init(load0 + 8 * st, 1);              // the loader's expect_tx arrival + the copies' bytes
            mbar_init(full0 + 8 * st, kProducerWarps);  // every producer warp has stored its weights
            mbar_init(empty0 + 8 * st, 1);             // tcgen05.commit of the stage's MMAs
        }
        mbar_init(done, 1);
        mbar_init(acc_free, kProducerWarps);  // every producer warp has read its accumulator part
        fence_mbar_init();
        abort_s = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;        // lane 0, first allocated column
    const uint32_t tmem_a = tmem + kAccCols;  // weight stages follow the accumulator
    bool ok = true;
    uint32_t g = 0;  // slabs so far in this CTA: stage g % kStages, phase g / kStages
    uint32_t st = 0, sph = 0, st_prev = 0;  // g % kStages, (g / kStages) & 1 and the previous slab's stage

    if (warp < kProducerWarps) {
        // ---- producers: symbols (shared) -> bf16 -> tensor memory; the tile's epilogue ----
        const uint32_t quarter = warp & 3u, part = warp >> 2;
        const uint32_t row = quarter * 32u + lane;  // weight row within the tile = tensor-memory lane
        const uint32_t lane_base = (quarter * 32u) << 16;
        uint32_t ti = 0, jb = 0;
        for (uint32_t tile = blockIdx.x; tile < P.total_tiles; tile += gridDim.x, ++ti) {
            if (__any_sync(0xFFFFFFFFu, abort_s != 0u)) break;
            while (jb + 1 < P.n_jobs && tile >= P.jobs[jb + 1].first_tile) ++jb;
            const GemmJob &J = P.jobs[jb];
            const uint32_t local = tile - J.first_tile;
            const uint32_t n0 = (local / P.t_tiles) * kTileN, m0 = (local % P.t_tiles) * kTileT;
            const uint32_t n_slabs = J.cols / kTileK;
            for (uint32_t it = 0; it < n_slabs; ++it, ++g) {
                const uint32_t s = st;
                if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(load0 + 8 * s, sph))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // this thread's kPartBytes symbols of the slab, widened exactly
                uint32_t v[kPartCols];
#pragma unroll
                for (uint32_t j = 0; j < kPartBytes / 16; ++j) {
                    uint4 lo, hi;
                    widen16<DT>(lds_sym16(bufW(s), row, part * (kPartBytes / 16) + j), lo, hi);
                    v[8 * j + 0] = lo.x, v[8 * j + 1] = lo.y, v[8 * j + 2] = lo.z, v[8 * j + 3] = lo.w;
                    v[8 * j + 4] = hi.x, v[8 * j + 5] = hi.y, v[8 * j + 6] = hi.z, v[8 * j + 7] = hi.w;
                }
                // the previous slab's tensor-memory store has had this slab's work to complete
                if (it > 0) {
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(full0 + 8 * st_prev);
                }
                const uint32_t ta = tmem_a + lane_base + s * kACols + part * kPartCols;
                if constexpr (kPartCols == 16) {
                    tmem_st16(ta, v);
                } else {
                    tmem_st8(ta, v);
                }
                st_prev = st;
                if (++st == kStages) {
                    st = 0;
                    sph ^= 1u;
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (!ok) break;
            if (lane == 0) mbar_arrive(full0 + 8 * st_prev);
            // epilogue: thread (w, l) holds weight row 32 (w % 4) + l and part w / 4 of the tile's tokens
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(done, ti & 1u))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t r = n0 + row;
            const float sc = __ldg(J.scales + r);
#pragma unroll 1
            for (uint32_t c = 0; c < kAccCols / kParts; c += 32) {
                uint32_t acc[32];
                tmem_ld32(tmem + lane_base + part * (kAccCols / kParts) + c, acc);
                const uint32_t t0 = m0 + part * (kAccCols / kParts) + c;
#pragma unroll
                for (uint32_t j = 0; j < 32; ++j)
                    if (t0 + j < P.tokens) J.y[(size_t)(t0 + j) * J.rows + r] = __fmul_rn(__uint_as_float(acc[j]), sc);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_free);  // the MMA warp may overwrite the accumulator
        }
    } else if (warp == kProducerWarps && lane == 0) {
        // ---- MMA issuer ----
        // One lane issues every MMA, so its loop is kept short: one wait per slab ("full": the
        // producers arrive only after they have seen the slab's copies land on "load"), the stage
        // and phase kept incrementally, and the descriptors advanced by adding to their address
        // field (16-byte units, well below its 14-bit limit for any shared-memory address).
        const uint64_t desc0 = tile_desc(bufB(0), 0);
        uint32_t ti = 0, n_done = 0, s = 0, ph = 0;  // stage and phase of the next slab
        bool ready = false;  // the next slab's "full" phase was already seen complete
        for (uint32_t tile = blockIdx.x, jb = 0; tile < P.total_tiles; tile += gridDim.x, ++ti) {
            while (jb + 1 < P.n_jobs && tile >= P.jobs[jb + 1].first_tile) ++jb;
            const uint32_t n_slabs = P.jobs[jb].cols / kTileK;
            // the previous tile's epilogue must have read the accumulator
            if (abort_s || (ti > 0 && !mbar_wait_bounded(acc_free, (ti - 1) & 1u))) {
                ok = false;
                break;
            }
            tc_fence_after();
            for (uint32_t it = 0; it < n_slabs; ++it) {
                if (!ready && !mbar_wait_bounded(full0 + 8 * s, ph)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t db = desc0 + ((s * kStageBytes) >> 4);
                const uint32_t ta = tmem_a + s * kACols;
#pragma unroll
                for (uint32_t kk = 0; kk < kTileK / kMmaK; ++kk)  // K step kk: +32 bytes, 2 descriptor units
                    tc_mma_ts(tmem, ta + kk * (kMmaK / 2), db + 2u * kk, S::kInstrDesc, (it | kk) != 0u);
                const uint32_t s_next = s + 1 == kStages ? 0u : s + 1, ph_next = s + 1 == kStages ? ph ^ 1u : ph;
                // peek (non-blocking) at the next slab's barrier while this slab's commit goes out
                ready = mbar_test(full0 + 8 * s_next, ph_next);
                tc_commit(empty0 + 8 * s);
                s = s_next;
                ph = ph_next;
            }
            tc_commit(done);  // completes when every MMA issued above has
            ++n_done;
            if (!ok) break;
        }
        // no MMA may still be running when the tensor memory is released
        if (n_done > 0 && !mbar_wait_bounded(done, (n_done - 1) & 1u)) ok = false;
    } else if (warp == kProducerWarps + 1 && lane == 0) {
        // ---- loader: the token tile and the symbol tile of every slab, kStages ahead ----
        for (uint32_t tile = blockIdx.x, jb = 0; tile < P.total_tiles && ok; tile += gridDim.x) {
            while (jb + 1 < P.n_jobs && tile >= P.jobs[jb + 1].first_tile) ++jb;
            const GemmJob &J = P.jobs[jb];
            const uint32_t local = tile - J.first_tile;
            const uint32_t n0 = (local / P.t_tiles) * kTileN, m0 = (local % P.t_tiles) * kTileT;
            const uint32_t n_slabs = J.cols / kTileK;
            const uint64_t map_x = reinterpret_cast<uint64_t>(&J.tmap_x);
            const uint64_t map_w = reinterpret_cast<uint64_t>(&J.tmap_w);
            for (uint32_t it = 0; it < n_slabs; ++it, ++g) {
                const uint32_t s = st;
                // stage s last held slab g - kStages (phase sph ^ 1): its MMAs (and so its producers) are done
                if (g >= kStages && (abort_s || !mbar_wait_bounded(empty0 + 8 * s, sph ^ 1u))) {
                    ok = false;
                    break;
                }
                mbar_expect_tx(load0 + 8 * s, kStageBytes);
                // token tile: two boxes of 128 tokens (x = k0, a multiple of 64 elements; rows past
                // the last token read as zeros); symbol tile: 128 rows x 64 bytes (x = k0 bytes)
#pragma unroll
                for (uint32_t h = 0; h < kTileT / kBoxT; ++h)
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                        " [%0], [%1, {%2, %3}], [%4];" ::"r"(bufB(s) + h * kBoxT * kRowBytes),
                        "l"(map_x), "r"(it * kTileK), "r"(m0 + h * kBoxT), "r"(load0 + 8 * s)
                        : "memory");
                asm volatile(
                    "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                    " [%0], [%1, {%2, %3}], [%4];" ::"r"(bufW(s)), "l"(map_w), "r"(it * kTileK), "r"(n0),
                    "r"(load0 + 8 * s)
                    : "memory");
                if (++st == kStages) {
                    st = 0;
                    sph ^= 1u;
                }
            }
        }
        // no copy may still be writing shared memory when the block exits: wait (bounded) for
        // the last copy issued to each stage; at normal exit they have all been consumed already
        for (uint32_t k = g > kStages ? g - kStages : 0; k < g; ++k)
            if (!mbar_wait_bounded(load0 + 8 * (k % kStages), (k / kStages) & 1u)) ok = false;
    }
    if (!ok) {
        abort_s = 1;
        atomicOr(P.status, EQ_DEV_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemAlloc)
                     : "memory");
    }
}

// ---- 2-SM variant (cta_group::2) -----------------------------------------------------
// For 256-token tiles over matrices whose rows are a multiple of 256, a
// cluster of two CTAs (one per SM of a pair) computes 256 weight rows x 256
// tokens with tcgen05.mma.cta_group::2 (M = 256): CTA r of the pair holds
// weight rows 128 r .. + 127 of the tile in its tensor memory (A, widened by
// its own producers), tokens 128 r .. + 127 of the tile in its shared memory
// (half of B), and the accumulator of its 128 weight rows for all 256 tokens.
// Each SM thus keeps half the token tile of the one-SM kernel per slab (16
// KB): 8 stages fit where 5 did, and the one lane that issues the MMAs (in CTA
// 0) issues half as many per FLOP.
//   loader     (each CTA) after its own "empty" (arrived by CTA 0's commit,
//              multicast to both CTAs), its token half (one 128-token box) and
//              its 128-row symbol tile, on its own "load" barrier
//   producers  (each CTA) widen as in the one-SM kernel, then arrive on CTA
//              0's "full" barrier (16 arrivals: 8 warps in each CTA)
//   MMA lane   (CTA 0) waits for "full", issues the slab's 4 MMAs and commits
//              them to "empty" in both CTAs; after a tile, to "done" in both
//   epilogue   (each CTA) its 128 rows x 256 tokens, then arrives on CTA 0's
//              "acc_free" (16 arrivals)
// Both CTAs take part in the same two cluster barriers (after set-up, before
// releasing the tensor memory); every other wait is bounded.
constexpr uint32_t kPairStages = 8;
constexpr uint32_t kPairXBytes = kBoxT * kTileK * 2;          // this CTA's 128 tokens of a slab, 16 KB
constexpr uint32_t kPairStageBytes = kPairXBytes + kWBytes;    // + its 128-row symbol tile
constexpr uint32_t kPairAcc = 256;                             // accumulator columns (tokens)
constexpr size_t kPairSmem = kPairStages * kPairStageBytes + 1024;
constexpr uint32_t kPairInstrDesc = (1u << 4) | (1u << 7) | (1u << 10)  // fp32 D, bf16 A and B, K-major
                                  | ((kPairAcc >> 3) << 17)              // N / 8
                                  | ((2 * kTileN >> 4) << 24);           // M / 16, M = 256 over the pair
static_assert(kPairAcc + kPairStages * kACols <= kTmemAlloc, "tensor memory columns");
static_assert(kPairSmem + 1024 <= 227u * 1024u, "shared memory per block");

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Every thread of both CTAs.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The shared::cluster address of the variable at `local` in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}

// Arrive on a barrier given by its shared::cluster address (possibly the other
// CTA's), with the default semantics.  What it publishes is the arriving
// warp's tensor-memory stores (ordered by tcgen05.wait::st and
// tcgen05.fence::before_thread_sync) and reads of the accumulator, not data
// in memory, so no cluster-wide release is needed.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

__device__ __forceinline__ bool mbar_poll_cluster(uint32_t bar, uint32_t parity, bool blocking) {
    uint32_t ok;
    if (blocking)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
    return ok != 0;
}

// Bounded wait on a local barrier that threads of the other CTA (or CTA 0's
// commits) arrive on.
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity) {
    if (mbar_poll_cluster(bar, parity, true)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_poll_cluster(bar, parity, true)) return true;
        if (clock64() - t0 > kWaitCycles) return false;
    }
}

__device__ __forceinline__ void tc_mma_ts_pair(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(tmem_d), "r"(tmem_a), "l"(db), "r"(kPairInstrDesc), "r"(accumulate)
        : "memory");
}

// Arrives (when every MMA issued so far by this thread has completed) on the
// barrier at shared-memory offset `bar` in both CTAs of the pair.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\t"
        "mov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}"
        ::"r"(bar)
        : "memory");
}

template <int DT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    eq_gemm_symbols_pair_kernel(const __grid_constant__ GemmParams P) {
    constexpr uint32_t kStages = kPairStages, kStageBytes = kPairStageBytes;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t load_s[kStages], full_s[kStages], empty_s[kStages], done_s, acc_free_s;
    __shared__ uint32_t tmem_base_s;
    __shared__ volatile uint32_t abort_s;
    const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
    const uint32_t rank = cluster_rank();
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    auto bufB = [&](uint32_t st) { return base + st * kStageBytes; };                // this CTA's token half
    auto bufW = [&](uint32_t st) { return base + st * kStageBytes + kPairXBytes; };  // its symbol tile
    const uint32_t load0 = smem_u32(&load_s[0]), full0 = smem_u32(&full_s[0]), empty0 = smem_u32(&empty_s[0]);
    const uint32_t done = smem_u32(&done_s), acc_free = smem_u32(&acc_free_s);

    if (warp == 0) {  // the same warp in both CTAs allocates, collectively
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&tmem_base_s)), "r"(kTmemAlloc) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (uint32_t st = 0; st < kStages; ++st) {
            mbar_init(load0 + 8 * st, 1);                   // this CTA's expect_tx arrival + its copies
            mbar_init(full0 + 8 * st, 2 * kProducerWarps);  // (CTA 0) the producer warps of both CTAs
            mbar_init(empty0 + 8 * st, 1);                  // CTA 0's commit
        }
        mbar_init(done, 1);
        mbar_init(acc_free, 2 * kProducerWarps);
        fence_mbar_init();
        abort_s = 0;
    }
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers initialised and tensor memory allocated
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    const uint32_t tmem_a = tmem + kPairAcc;
    const uint32_t n_clusters = gridDim.x / 2, cl = blockIdx.x / 2;
    bool ok = true;

    if (warp < kProducerWarps) {
        // ---- producers (both CTAs) ----
        const uint32_t quarter = warp & 3u, part = warp >> 2;
        const uint32_t row = quarter * 32u + lane;
        const uint32_t lane_base = (quarter * 32u) << 16;
        const uint32_t full_c0 = cluster_addr(full0, 0), acc_free_c0 = cluster_addr(acc_free, 0);
        uint32_t st = 0, sph = 0, st_prev = 0, ti = 0, jb = 0;
        for (uint32_t tile = cl; tile < P.total_tiles; tile += n_clusters, ++ti) {
            if (__any_sync(0xFFFFFFFFu, abort_s != 0u)) break;
            while (jb + 1 < P.n_jobs && tile >= P.jobs[jb + 1].first_tile) ++jb;
            const GemmJob &J = P.jobs[jb];
            const uint32_t local = tile - J.first_tile;
            const uint32_t n0 = (local / P.t_tiles) * (2 * kTileN) + rank * kTileN, m0 = (local % P.t_tiles) * kPairAcc;
            const uint32_t n_slabs = J.cols / kTileK;
            for (uint32_t it = 0; it < n_slabs; ++it) {
                const uint32_t s = st;
                if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(load0 + 8 * s, sph))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t v[kPartCols];
#pragma unroll
                for (uint32_t j = 0; j < kPartBytes / 16; ++j) {
                    uint4 lo, hi;
                    widen16<DT>(lds_sym16(bufW(s), row, part * (kPartBytes / 16) + j), lo, hi);
                    v[8 * j + 0] = lo.x, v[8 * j + 1] = lo.y, v[8 * j + 2] = lo.z, v[8 * j + 3] = lo.w;
                    v[8 * j + 4] = hi.x, v[8 * j + 5] = hi.y, v[8 * j + 6] = hi.z, v[8 * j + 7] = hi.w;
                }
                if (it > 0) {  // the previous slab's store has completed: tell CTA 0's MMA lane
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(full_c0 + 8 * st_prev);
                }
                const uint32_t ta = tmem_a + lane_base + s * kACols + part * kPartCols;
                if constexpr (kPartCols == 16) {
                    tmem_st16(ta, v);
                } else {
                    tmem_st8(ta, v);
                }
                st_prev = st;
                if (++st == kStages) {
                    st = 0;
                    sph ^= 1u;
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (!ok) break;
            if (lane == 0) mbar_arrive_cluster(full_c0 + 8 * st_prev);
            // epilogue: this CTA's 128 weight rows, part w / 4 of the tile's 256 tokens
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_cluster(done, ti & 1u))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t r = n0 + row;
            const float sc = __ldg(J.scales + r);
#pragma unroll 1
            for (uint32_t c = 0; c < kPairAcc / kParts; c += 32) {
                uint32_t acc[32];
                tmem_ld32(tmem + lane_base + part * (kPairAcc / kParts) + c, acc);
                const uint32_t t0 = m0 + part * (kPairAcc / kParts) + c;
#pragma unroll
                for (uint32_t j = 0; j < 32; ++j)
                    if (t0 + j < P.tokens) J.y[(size_t)(t0 + j) * J.rows + r] = __fmul_rn(__uint_as_float(acc[j]), sc);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_free_c0);
        }
    } else if (warp == kProducerWarps && lane == 0 && rank == 0) {
        // ---- MMA lane (CTA 0) ----
        const uint64_t desc0 = tile_desc(bufB(0), 0);
        uint32_t ti = 0, n_done = 0, s = 0, ph = 0;
        bool ready = false;
        for (uint32_t tile = cl, jb = 0; tile < P.total_tiles; tile += n_clusters, ++ti) {
            while (jb + 1 < P.n_jobs && tile >= P.jobs[jb + 1].first_tile) ++jb;
            const uint32_t n_slabs = P.jobs[jb].cols / kTileK;
            if (abort_s || (ti > 0 && !mbar_wait_cluster(acc_free, (ti - 1) & 1u))) {
                ok = false;
                break;
            }
            tc_fence_after();
            for (uint32_t it = 0; it < n_slabs; ++it) {
                if (!ready && !mbar_wait_cluster(full0 + 8 * s, ph)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t db = desc0 + ((s * kStageBytes) >> 4);
                const uint32_t ta = tmem_a + s * kACols;
#pragma unroll
                for (uint32_t kk = 0; kk < kTileK / kMmaK; ++kk)
                    tc_mma_ts_pair(tmem, ta + kk * (kMmaK / 2), db + 2u * kk, (it | kk) != 0u);
                const uint32_t s_next = s + 1 == kStages ? 0u : s + 1, ph_next = s + 1 == kStages ? ph ^ 1u : ph;
                ready = mbar_poll_cluster(full0 + 8 * s_next, ph_next, false);
                tc_commit_pair(empty0 + 8 * s);
                s = s_next;
                ph = ph_next;
            }
            tc_commit_pair(done);
            ++n_done;
            if (!ok) break;
        }
        if (n_done > 0 && !mbar_wait_cluster(done, (n_done - 1) & 1u)) ok = false;
    } else if (warp == kProducerWarps + 1 && lane == 0) {
        // ---- loader (both CTAs) ----
        uint32_t st = 0, sph = 0, g = 0;
        for (uint32_t tile = cl, jb = 0; tile < P.total_tiles && ok; tile += n_clusters) {
            while (jb + 1 < P.n_jobs && tile >= P.jobs[jb + 1].first_tile) ++jb;
            const GemmJob &J = P.jobs[jb];
            const uint32_t local = tile - J.first_tile;
            const uint32_t n0 = (local / P.t_tiles) * (2 * kTileN) + rank * kTileN;
            const uint32_t m0 = (local % P.t_tiles) * kPairAcc + rank * kBoxT;  // this CTA's token half
            const uint32_t n_slabs = J.cols / kTileK;
            const uint64_t map_x = reinterpret_cast<uint64_t>(&J.tmap_x);
            const uint64_t map_w = reinterpret_cast<uint64_t>(&J.tmap_w);
            for (uint32_t it = 0; it < n_slabs; ++it, ++g) {
                const uint32_t s = st;
                if (g >= kStages && (abort_s || !mbar_wait_cluster(empty0 + 8 * s, sph ^ 1u))) {
                    ok = false;
                    break;
                }
                mbar_expect_tx(load0 + 8 * s, kStageBytes);
                asm volatile(
                    "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                    " [%0], [%1, {%2, %3}], [%4];" ::"r"(bufB(s)), "l"(map_x), "r"(it * kTileK), "r"(m0),
                    "r"(load0 + 8 * s)
                    : "memory");
                asm volatile(
                    "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                    " [%0], [%1, {%2, %3}], [%4];" ::"r"(bufW(s)), "l"(map_w), "r"(it * kTileK), "r"(n0),
                    "r"(load0 + 8 * s)
                    : "memory");
                if (++st == kStages) {
                    st = 0;
                    sph ^= 1u;
                }
            }
        }
        for (uint32_t k = g > kStages ? g - kStages : 0; k < g; ++k)
            if (!mbar_wait_bounded(load0 + 8 * (k % kStages), (k / kStages) & 1u)) ok = false;
    }
    if (!ok) {
        abort_s = 1;
        atomicOr(P.status, EQ_DEV_TIMEOUT);
    }
    tc_fence_before();
    cluster_sync_all();  // no MMA of CTA 0 reads this CTA's memory any more
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemAlloc)
                     : "memory");
    }
}

// Failure-path check of the GEMM's waits: the GEMM's own set-up (TMEM
// allocation, "load" / "full" / "empty" / "done" barriers with their arrival
// counts, the GEMM's block size) and exit path (status flag, TMEM release),
// but no producer ever arrives on "full", so the MMA lane's bounded wait must
// give up; it then arrives on "done" itself, the producers pass it (or give up
// on it) and the block returns with EQ_DEV_TIMEOUT set and its TMEM freed.
__global__ void __launch_bounds__(kGemmThreads, 1) eq_gemm_wait_timeout_kernel(int32_t *status) {
    constexpr uint32_t kStages = GemmShape<256>::kStages;
    __shared__ __align__(8) uint64_t load_s[kStages], full_s[kStages], empty_s[kStages], done_s;
    __shared__ uint32_t tmem_base_s;
    const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
    const uint32_t load0 = smem_u32(&load_s[0]), full0 = smem_u32(&full_s[0]), empty0 = smem_u32(&empty_s[0]);
    const uint32_t done = smem_u32(&done_s);
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&tmem_base_s)), "r"(kTmemAlloc) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (uint32_t st = 0; st < kStages; ++st) {
            mbar_init(load0 + 8 * st, 1);
            mbar_init(full0 + 8 * st, kProducerWarps);
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
    } else if (warp < kProducerWarps) {
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

bool g_gemm_attr_set[128][2][3];  // device, weight type, kernel (128-token, 256-token, 2-SM)

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
// box kTileK x kBoxT with the swizzle the MMA descriptors expect.
int encode_token_map(CUtensorMap *map, const void *x, uint32_t tokens, uint32_t cols) {
    auto enc = tensor_map_encoder();
    if (!enc) return EQ_ERR_CUDA;
    const cuuint64_t dims[2] = {cols, tokens};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2u};
    const cuuint32_t box[2] = {kTileK, kBoxT};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? EQ_OK : EQ_ERR_CUDA;
}

// Tensor map of a matrix's symbols: inner dimension cols, outer rows; box
// kTileK bytes x kTileN rows with the 64-byte swizzle the producers read.
int encode_symbol_map(CUtensorMap *map, const void *sym, uint32_t rows, uint32_t cols) {
    auto enc = tensor_map_encoder();
    if (!enc) return EQ_ERR_CUDA;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols};
    const cuuint32_t box[2] = {kTileK, kTileN};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(sym), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? EQ_OK : EQ_ERR_CUDA;
}

}  // namespace

namespace {

struct GemmRequest {
    uint32_t matrix;
    const void *sym, *x;
    float *y;
};

// Checks one request against its matrix; EQ_OK, or the error the entry point returns.
int check_request(const eq_model *m, const GemmRequest &q) {
    if (q.matrix >= m->mats.size()) return EQ_ERR_INVALID_ARG;
    const MatrixDesc &d = m->mats[q.matrix];
    const eq_matrix_info &in = d.info;
    if (!in.rows || !in.cols) return EQ_OK;
    if (in.rows % kTileN || in.cols % kTileK || in.rows / kTileN > 65535u) return EQ_ERR_UNSUPPORTED;
    if (!q.sym || !q.x || !q.y) return EQ_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(q.sym) % 16 || reinterpret_cast<uintptr_t>(q.x) % 16 ||
        reinterpret_cast<uintptr_t>(q.y) % 16 || d.scales_off % 16)
        return EQ_ERR_INVALID_ARG;
    return EQ_OK;
}

// One persistent launch per weight type over the tiles of all requests of that
// type (at most kMaxGemmJobs per launch), longest K first so that the static
// round-robin tile order ends with the short tiles; then the super weights.
int gemm_launch(const eq_model *m, const GemmRequest *req, uint32_t n, uint32_t tokens, int32_t *d_status,
                cudaStream_t s) {
    if (!m || !d_status || (n && !req)) return EQ_ERR_INVALID_ARG;
    for (uint32_t i = 0; i < n; ++i)
        if (const int rc = check_request(m, req[i])) return rc;
    if (!tokens) return EQ_OK;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return EQ_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return EQ_ERR_CUDA;
    if (m->sm_limit && m->sm_limit < (uint32_t)sms) sms = (int)m->sm_limit;
    // short inputs (<= 128 tokens) take the 128-token tile: each weight tile is read once and the
    // MMA does no work on absent tokens
    const bool narrow = tokens <= kNarrowTokens;
    const uint32_t tile_t = narrow ? 128u : 256u;
    const size_t smem = narrow ? GemmShape<128>::kSmem : GemmShape<256>::kSmem;
    const uint32_t t_tiles = (tokens + tile_t - 1) / tile_t;
    for (int dt = EQ_INT8; dt <= EQ_E4M3; ++dt) {
        std::vector<uint32_t> order;
        for (uint32_t i = 0; i < n; ++i) {
            const eq_matrix_info &in = m->mats[req[i].matrix].info;
            if (in.dtype == dt && in.rows && in.cols) order.push_back(i);
        }
        std::stable_sort(order.begin(), order.end(), [&](uint32_t a, uint32_t b) {
            return m->mats[req[a].matrix].info.cols > m->mats[req[b].matrix].info.cols;
        });
        auto fn = dt == EQ_INT8 ? (narrow ? eq_gemm_symbols_kernel<EQ_INT8, 128> : eq_gemm_symbols_kernel<EQ_INT8, 256>)
                                : (narrow ? eq_gemm_symbols_kernel<EQ_E4M3, 128> : eq_gemm_symbols_kernel<EQ_E4M3, 256>);
        for (size_t at = 0; at < order.size(); at += kMaxGemmJobs) {
            const size_t end = std::min(order.size(), at + kMaxGemmJobs);
            // the 2-SM kernel: 256-token tiles, every matrix a whole number of 256-row tiles
            bool pair = !narrow && sms >= 2;
            for (size_t k = at; k < end && pair; ++k) pair = m->mats[req[order[k]].matrix].info.rows % (2 * kTileN) == 0;
            const uint32_t tile_rows = pair ? 2 * kTileN : kTileN;
            GemmParams P{};
            P.status = d_status;
            P.tokens = tokens;
            P.t_tiles = t_tiles;
            uint64_t tiles = 0;
            for (size_t k = at; k < end; ++k) {
                const GemmRequest &q = req[order[k]];
                const MatrixDesc &d = m->mats[q.matrix];
                GemmJob &J = P.jobs[P.n_jobs++];
                if (const int rc = encode_token_map(&J.tmap_x, q.x, tokens, d.info.cols)) return rc;
                if (const int rc = encode_symbol_map(&J.tmap_w, q.sym, d.info.rows, d.info.cols)) return rc;
                J.sym = static_cast<const uint8_t *>(q.sym);
                J.scales = reinterpret_cast<const float *>(m->d_blob + d.scales_off);
                J.y = q.y;
                J.rows = d.info.rows;
                J.cols = d.info.cols;
                J.first_tile = (uint32_t)tiles;
                tiles += (uint64_t)(d.info.rows / tile_rows) * t_tiles;
            }
            if (tiles > 0xFFFFFFFFull - (uint64_t)sms) return EQ_ERR_UNSUPPORTED;
            P.total_tiles = (uint32_t)tiles;
            const int variant = pair ? 2 : narrow ? 0 : 1;
            const void *kfn = pair ? reinterpret_cast<const void *>(dt == EQ_INT8 ? eq_gemm_symbols_pair_kernel<EQ_INT8>
                                                                                  : eq_gemm_symbols_pair_kernel<EQ_E4M3>)
                                   : reinterpret_cast<const void *>(fn);
            const size_t ksmem = pair ? kPairSmem : smem;
            bool &attr = g_gemm_attr_set[dev][dt - 1][variant];
            if (!attr) {
                if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ksmem) != cudaSuccess)
                    return EQ_ERR_CUDA;
                attr = true;
            }
            if (pair) {
                const uint32_t clusters = (uint32_t)std::min<uint64_t>(tiles, (uint64_t)(sms / 2));
                auto pfn = dt == EQ_INT8 ? eq_gemm_symbols_pair_kernel<EQ_INT8> : eq_gemm_symbols_pair_kernel<EQ_E4M3>;
                pfn<<<2 * clusters, kGemmThreads, ksmem, s>>>(P);
            } else {
                const uint32_t grid = std::min<uint64_t>(tiles, (uint64_t)sms);
                fn<<<grid, kGemmThreads, smem, s>>>(P);
            }
            if (cudaGetLastError() != cudaSuccess) return EQ_ERR_CUDA;
        }
    }
    for (uint32_t i = 0; i < n; ++i) {
        const MatrixDesc &d = m->mats[req[i].matrix];
        const eq_matrix_info &in = d.info;
        if (!in.n_outliers || !in.rows || !in.cols) continue;
        const uint64_t cnt = (uint64_t)in.n_outliers * tokens;
        eq_gemm_outliers_kernel<<<(unsigned)((cnt + 255) / 256), 256, 0, s>>>(
            reinterpret_cast<const uint32_t *>(m->d_blob + d.outliers_off), in.n_outliers,
            static_cast<const uint16_t *>(req[i].x), tokens, in.rows, in.cols, req[i].y, d_status);
        if (cudaGetLastError() != cudaSuccess) return EQ_ERR_CUDA;
    }
    return EQ_OK;
}

}  // namespace

extern "C" EQW_API int eq_gemm_symbols(const eq_model *m, uint32_t matrix, const void *d_sym, const void *d_x,
                                       uint32_t tokens, float *d_y, int32_t *d_status, cudaStream_t s) {
    const eqw::NvtxScope nvtx_range("eq_gemm_symbols");
    const GemmRequest q{matrix, d_sym, d_x, d_y};
    return gemm_launch(m, &q, 1, tokens, d_status, s);
}

extern "C" EQW_API int eq_gemm_symbols_block(const eq_model *m, uint32_t layer, const void *const *d_syms,
                                             const void *const *d_xs, uint32_t tokens, float *const *d_ys,
                                             uint32_t count, int32_t *d_status, cudaStream_t s) {
    const eqw::NvtxScope nvtx_range("eq_gemm_symbols_block");
    if (!m || layer >= m->n_layers) return EQ_ERR_INVALID_ARG;
    const uint32_t first = m->layer_first[layer], n = m->layer_count[layer];
    if (count != n || (n && (!d_syms || !d_xs || !d_ys))) return EQ_ERR_INVALID_ARG;
    std::vector<GemmRequest> req(n);
    for (uint32_t i = 0; i < n; ++i) req[i] = GemmRequest{first + i, d_syms[i], d_xs[i], d_ys[i]};
    return gemm_launch(m, req.data(), n, tokens, d_status, s);
}

extern "C" EQW_API int eq_selftest_gemm_wait_timeout(int32_t *d_status, cudaStream_t s) {
    if (!d_status) return EQ_ERR_INVALID_ARG;
    eq_gemm_wait_timeout_kernel<<<1, kGemmThreads, 0, s>>>(d_status);
    return cudaGetLastError() == cudaSuccess ? EQ_OK : EQ_ERR_CUDA;
}
