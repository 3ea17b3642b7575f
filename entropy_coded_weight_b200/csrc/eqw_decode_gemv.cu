// Fused decode + batch-1 GEMV of entropy-coded weights: eq_decode_gemv_block,
// eq_decode_gemv_matrix.
//
// EntQuant technical summary (gist.science 2601.22787), section 2
// "inference-time decoding": a block's weights are expanded into a buffer just
// before its forward kernels read them, and at batch 1 a linear layer's
// forward is y = W x; section 5 expects large speed-ups from dedicated fused
// kernels.
// Here the buffer disappears: each warp decodes its chunk exactly as
// eq_decode_kernel does (staging ring, interleaved rANS step, shared slot
// table, rank-mode dequant) and, after every 8 steps, multiplies the 8 weights
// a lane holds by the matching 8 entries of x, so no weight leaves the
// registers.  HBM traffic per weight falls from the compressed read plus a
// bf16 write and a bf16 read (about 4.3 bytes at 2.1 bits per weight) to the
// compressed read alone (about 0.27 bytes).
//
// Arithmetic, per matrix:
//   w[r, c] = bf16(fp32(value(sym) * scale[r])), both roundings to nearest
//             even -- the bits eq_decode_block writes -- so w * x (bf16 * bf16)
//             is exact in fp32;
//   each lane sums its products in fp32 with fused multiply-adds into two
//   accumulators (even and odd columns); at the end of a row segment (the
//   part of a row inside one chunk) the warp adds its 32 lane sums with a
//   butterfly of shuffles, lane 0 adds the row's super weights w_o * x[c]
//   that fall in the segment (the stream carries value zero at their
//   positions), and adds the segment sum to y[r] with one fp32 atomic add.
// A row of at most 65536 columns spans at most two chunks, so y[r] is the sum
// of at most two segment sums in either order: the result is deterministic.
//
// Requires cols % 256 == 0 for every non-empty matrix: a 256-symbol group then
// never crosses a row, every chunk holds whole groups, and one 16-byte load
// of x per lane and group serves its 8 weights.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "eqw_device.cuh"

namespace {

#ifndef EQ_GEMV_WARPS
#define EQ_GEMV_WARPS EQ_SHARED_WARPS
#endif
#ifndef EQ_GEMV_MIN_CTAS
#define EQ_GEMV_MIN_CTAS 1
#endif
#ifndef EQ_GEMV_FMA2
#define EQ_GEMV_FMA2 1
#endif
constexpr int kGemvWarps = EQ_GEMV_WARPS;       // warps per block, shared-table kernel
constexpr int kGemvMinCtas = EQ_GEMV_MIN_CTAS;  // register budget: blocks of kGemvWarps per SM

struct GemvJob {
    const uint64_t *chunk_index;  // absolute record offsets, n_chunks + 1 entries
    const float *scales;          // fp32 [rows]
    const uint4 *x;               // bf16 [cols], 8 per 16-byte vector
    float *y;                     // fp32 [rows], zero when the launch starts
    const uint32_t *outliers;     // {row, col, value bits} x n_out, ascending linear index
    uint64_t n_elems;
    uint32_t cols;
    uint32_t rows;
    uint32_t n_chunks;
    uint32_t chunk0;              // always 0: every chunk of the matrix is decoded here
    uint32_t begin;               // first launch-wide work unit (tile or chunk) of this matrix
    uint32_t n_out;
};

struct GemvParams {
    const uint8_t *blob;
    uint64_t blob_len;
    int32_t *status;
    uint32_t n_mats;
    uint32_t total_units;
    uint32_t tile_warps;          // shared-table kernels: warps that take chunks of a tile (assign_tiles)
    uint32_t tile_chains;         // shared-table kernels: chunks per warp in a tile, 1 or 2 (assign_tiles)
    GemvJob mats[kMaxMatsPerLaunch];
};

// fp32 -> nearest bf16 (ties to even) -> fp32, exact.
__device__ __forceinline__ float bf16_round(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

// The two bf16 of a 32-bit word as fp32 (exact).
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// a0 += w0 * x0, a1 += w1 * x1, each a fused multiply-add rounded to nearest even.
__device__ __forceinline__ void fma_pair(float &a0, float &a1, float w0, float w1, float x0, float x1) {
#if EQ_GEMV_FMA2
    unsigned long long A, Wp, X;
    asm("mov.b64 %0, {%1, %2};" : "=l"(A) : "f"(a0), "f"(a1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(Wp) : "f"(w0), "f"(w1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(X) : "f"(x0), "f"(x1));
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(A) : "l"(Wp), "l"(X));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(A));
#else
    a0 = fmaf(w0, x0, a0);
    a1 = fmaf(w1, x1, a1);
#endif
}

__device__ __forceinline__ uint32_t vec_word(const uint4 &v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Super weights of one row segment: outliers with linear index in [lo, hi)
// (a binary search over the ascending list, then a scan), each adding
// bf16(v) * x[c] to `a`.
__device__ __noinline__ float add_outliers(int32_t *status, const GemvJob &M, uint64_t lo, uint64_t hi, float a) {
    const uint32_t *rec = M.outliers;
    uint32_t b = 0, e = M.n_out;
    while (b < e) {
        const uint32_t mid = (b + e) / 2;
        const uint64_t lin = (uint64_t)rec[3 * mid] * M.cols + rec[3 * mid + 1];
        if (lin < lo) b = mid + 1;
        else e = mid;
    }
    const uint16_t *x16 = reinterpret_cast<const uint16_t *>(M.x);
    for (; b < M.n_out; ++b) {
        const uint32_t r = rec[3 * b], c = rec[3 * b + 1];
        if (r >= M.rows || c >= M.cols) {
            atomicOr(status, EQ_DEV_BAD_OUTLIER);
            break;
        }
        if ((uint64_t)r * M.cols + c >= hi) break;
        a = fmaf(bf16_round(__uint_as_float(rec[3 * b + 2])), __uint_as_float((uint32_t)x16[c] << 16), a);
    }
    return a;
}

// End of a row segment [lo, hi) of row `row`: warp sum, super weights, y[row] +=.
__device__ __forceinline__ void flush_segment(int32_t *status, const GemvJob &M, uint32_t row, uint64_t lo,
                                              uint64_t hi, float a, uint32_t lane) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) a += __shfl_xor_sync(kFull, a, d);
    if (lane == 0) {
        if (M.n_out) a = add_outliers(status, M, lo, hi, a);
        atomicAdd(M.y + row, a);
    }
}

// One 256-symbol group times x.  BY_RANK: the slot entry's low 5 bits name
// the lane holding the weight (lane r holds bf16(value(rank r) * scale));
// otherwise `w` is the row scale and the weight is formed from the symbol.
template <int DT, bool BY_RANK, uint32_t CODEC>
__device__ __forceinline__ void group_dot(uint32_t lut, uint32_t ring, uint32_t &pw, CodecState<CODEC> &x,
                                          uint32_t lt, float w, const uint4 *xp, float &a0, float &a1) {
    const uint4 xv = __ldg(xp);
    const uint32_t rp0 = ring + (pw & (kRingBytes - 1));
    uint32_t rp = rp0;
#pragma unroll
    for (int r = 0; r < 8; r += 2) {
        const uint32_t e0 = codec_step<CODEC>(lut, rp, x, lt);
        const uint32_t e1 = codec_step<CODEC>(lut, rp, x, lt);
        float w0, w1;
        if constexpr (BY_RANK) {
            w0 = __shfl_sync(kFull, w, e0);
            w1 = __shfl_sync(kFull, w, e1);
        } else {
            w0 = bf16_round(dequant1<DT>(e0, w));
            w1 = bf16_round(dequant1<DT>(e1, w));
        }
        const uint32_t u = vec_word(xv, r / 2);
        fma_pair(a0, a1, w0, w1, bf_lo(u), bf_hi(u));
    }
    pw += rp - rp0;
}

// Runs of groups within one row, two groups per ring check (the ring keeps
// two groups' worth of words resident past each check).
template <int DT, bool BY_RANK, uint32_t CODEC>
__device__ __forceinline__ void run_dot(uint32_t lut, uint32_t ring, uint32_t mbar, RingCtl *ctl, uint32_t &pw,
                                        uint32_t &limit, CodecState<CODEC> &x, uint32_t lt, float w,
                                        const uint4 *xp, uint32_t run, float &a0, float &a1) {
    uint32_t i = 0;
    while (i < run) {
        if (pw >= limit) {
            limit = ring_service(ctl, ring, mbar, pw);
            if (ctl->dead) return;
        }
        if (i + 1 < run) {
            do {
                group_dot<DT, BY_RANK, CODEC>(lut, ring, pw, x, lt, w, xp, a0, a1);
                group_dot<DT, BY_RANK, CODEC>(lut, ring, pw, x, lt, w, xp + kGroupSyms / 8, a0, a1);
                i += 2;
                xp += 2 * kGroupSyms / 8;
            } while (i + 1 < run && pw < limit);
        } else {
            group_dot<DT, BY_RANK, CODEC>(lut, ring, pw, x, lt, w, xp, a0, a1);
            i += 1;
            xp += kGroupSyms / 8;
        }
    }
}

// One chunk (its slot table ready at `lut`, or a single symbol `single`).
// Returns false if a bounded wait gave up (the warp must stop).
template <int DT, uint32_t CODEC>
__device__ __forceinline__ bool gemv_body(int32_t *status, const GemvJob &M, uint64_t first, const ChunkHead &h,
                                          bool single_sym, uint32_t single, uint32_t lut, uint32_t ring,
                                          uint32_t mbar, RingCtl *ctl, uint32_t lane, uint32_t lt, bool by_rank,
                                          uint32_t lane_sym) {
    const uint32_t n_groups = h.n / kGroupSyms;
    uint32_t row = (uint32_t)(first / M.cols);
    uint32_t col = (uint32_t)(first - (uint64_t)row * M.cols);
    CodecState<CODEC> x = codec_start<CODEC>(h.x);
    if (single_sym) {
        // rANS f = 4096 / Huffman length 0: the states never change and there are no words
        if (h.n_words != 0 || !__all_sync(kFull, CODEC == kCodecHuffman || h.x == kStateLow)) {
            flag(status, EQ_DEV_BAD_END);
            return true;
        }
        for (uint32_t g = 0; g < n_groups;) {
            const uint32_t run = min((M.cols - col) / kGroupSyms, n_groups - g);
            const float w = bf16_round(dequant1<DT>(single, __ldg(M.scales + row)));
            const uint4 *xp = M.x + col / 8 + lane;
            float a0 = 0.f, a1 = 0.f;
            for (uint32_t i = 0; i < run; ++i, xp += kGroupSyms / 8) {
                const uint4 xv = __ldg(xp);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    a0 = fmaf(w, bf_lo(vec_word(xv, q)), a0);
                    a1 = fmaf(w, bf_hi(vec_word(xv, q)), a1);
                }
            }
            const uint64_t lo = (uint64_t)row * M.cols + col;
            flush_segment(status, M, row, lo, lo + (uint64_t)run * kGroupSyms, a0 + a1, lane);
            g += run;
            col += run * kGroupSyms;
            if (col == M.cols) {
                col = 0;
                ++row;
            }
        }
        return true;
    }
    ring_start(ctl, h);
    __syncwarp();
    uint32_t limit = h.n_words ? 0u : kNoLimit;
    uint32_t pw = 0;
    const float vraw = symbol_value<DT>(lane_sym);
    for (uint32_t g = 0; g < n_groups && !ctl->dead;) {
        const uint32_t run = min((M.cols - col) / kGroupSyms, n_groups - g);
        const float s = __ldg(M.scales + row);
        const uint4 *xp = M.x + col / 8 + lane;
        float a0 = 0.f, a1 = 0.f;
        if (by_rank)
            run_dot<DT, true, CODEC>(lut, ring, mbar, ctl, pw, limit, x, lt, bf16_round(__fmul_rn(vraw, s)), xp,
                                     run, a0, a1);
        else
            run_dot<DT, false, CODEC>(lut, ring, mbar, ctl, pw, limit, x, lt, s, xp, run, a0, a1);
        const uint64_t lo = (uint64_t)row * M.cols + col;
        flush_segment(status, M, row, lo, lo + (uint64_t)run * kGroupSyms, a0 + a1, lane);
        g += run;
        col += run * kGroupSyms;
        if (col == M.cols) {
            col = 0;
            ++row;
        }
    }
    if (!ring_drain(ctl, mbar)) {
        flag(status, EQ_DEV_TIMEOUT);
        return false;
    }
    if (!__all_sync(kFull, codec_done(x)) || pw != 2u * h.n_words) flag(status, EQ_DEV_BAD_END);
    return true;
}

// Two full chunks per warp in lockstep (rank mode, cols % 512 == 0), as in
// the decode kernel; each chain keeps its own row, weights and accumulators.
template <uint32_t CODEC>
struct DotChain {
    CodecState<CODEC> x;
    uint32_t pw, limit, row, col;
    float w, a0, a1;
    const uint4 *xp;
};

template <uint32_t CODEC>
__device__ __forceinline__ void group2_dot(uint32_t lut, uint32_t ringA, uint32_t ringB, DotChain<CODEC> &A,
                                           DotChain<CODEC> &B, uint32_t lt) {
    const uint4 xa = __ldg(A.xp), xb = __ldg(B.xp);
    const uint32_t a0 = ringA + (A.pw & (kRingBytes - 1));
    const uint32_t b0 = ringB + (B.pw & (kRingBytes - 1));
    uint32_t ra = a0, rb = b0;
#pragma unroll
    for (int r = 0; r < 8; r += 2) {
        const uint32_t ea0 = codec_step<CODEC>(lut, ra, A.x, lt);
        const uint32_t eb0 = codec_step<CODEC>(lut, rb, B.x, lt);
        const uint32_t ea1 = codec_step<CODEC>(lut, ra, A.x, lt);
        const uint32_t eb1 = codec_step<CODEC>(lut, rb, B.x, lt);
        const uint32_t ua = vec_word(xa, r / 2), ub = vec_word(xb, r / 2);
        fma_pair(A.a0, A.a1, __shfl_sync(kFull, A.w, ea0), __shfl_sync(kFull, A.w, ea1), bf_lo(ua), bf_hi(ua));
        fma_pair(B.a0, B.a1, __shfl_sync(kFull, B.w, eb0), __shfl_sync(kFull, B.w, eb1), bf_lo(ub), bf_hi(ub));
    }
    A.pw += ra - a0;
    B.pw += rb - b0;
    A.xp += kGroupSyms / 8;
    B.xp += kGroupSyms / 8;
}

template <uint32_t CODEC>
__device__ __forceinline__ void chain_row(const GemvJob &M, DotChain<CODEC> &C, float vraw, uint32_t lane) {
    C.w = bf16_round(__fmul_rn(vraw, __ldg(M.scales + C.row)));
    C.xp = M.x + C.col / 8 + lane;
    C.a0 = C.a1 = 0.f;
}

// After a pair of groups: at the end of a row, flush the segment and move on.
template <uint32_t CODEC>
__device__ __forceinline__ void chain_advance(int32_t *status, const GemvJob &M, DotChain<CODEC> &C, uint64_t first,
                                              float vraw, uint32_t lane) {
    C.col += 2 * kGroupSyms;
    if (C.col == M.cols) {
        const uint64_t base = (uint64_t)C.row * M.cols;
        flush_segment(status, M, C.row, base > first ? base : first, base + M.cols, C.a0 + C.a1, lane);
        C.col = 0;
        ++C.row;
        if (C.row < M.rows) chain_row(M, C, vraw, lane);
    }
}

template <int DT, uint32_t CODEC>
__device__ __forceinline__ bool gemv_pair(int32_t *status, const GemvJob &M, const ChunkHead &hA, const ChunkHead &hB,
                                          uint64_t firstA, uint64_t firstB, uint32_t lut, uint32_t ringA,
                                          uint32_t ringB, uint32_t mbarA, uint32_t mbarB, RingCtl *ctlA,
                                          RingCtl *ctlB, uint32_t lane, uint32_t lt, uint32_t lane_sym) {
    ring_start(ctlA, hA);
    ring_start(ctlB, hB);
    __syncwarp();
    const float vraw = symbol_value<DT>(lane_sym);
    DotChain<CODEC> A, B;
    A.x = codec_start<CODEC>(hA.x);
    B.x = codec_start<CODEC>(hB.x);
    A.pw = B.pw = 0;
    A.limit = hA.n_words ? 0u : kNoLimit;
    B.limit = hB.n_words ? 0u : kNoLimit;
    A.row = (uint32_t)(firstA / M.cols);
    A.col = (uint32_t)(firstA - (uint64_t)A.row * M.cols);
    B.row = (uint32_t)(firstB / M.cols);
    B.col = (uint32_t)(firstB - (uint64_t)B.row * M.cols);
    chain_row(M, A, vraw, lane);
    chain_row(M, B, vraw, lane);
    constexpr uint32_t kPairs = kChunkSyms / (2 * kGroupSyms);
    for (uint32_t q = 0; q < kPairs; ++q) {
        if (A.pw >= A.limit) A.limit = ring_service(ctlA, ringA, mbarA, A.pw);
        if (B.pw >= B.limit) B.limit = ring_service(ctlB, ringB, mbarB, B.pw);
        if (ctlA->dead || ctlB->dead) break;
        group2_dot(lut, ringA, ringB, A, B, lt);
        group2_dot(lut, ringA, ringB, A, B, lt);
        chain_advance(status, M, A, firstA, vraw, lane);
        chain_advance(status, M, B, firstB, vraw, lane);
    }
    // a chunk that ends inside a row leaves a partial segment
    if (A.col != 0) {
        const uint64_t base = (uint64_t)A.row * M.cols;
        flush_segment(status, M, A.row, base > firstA ? base : firstA, base + A.col, A.a0 + A.a1, lane);
    }
    if (B.col != 0) {
        const uint64_t base = (uint64_t)B.row * M.cols;
        flush_segment(status, M, B.row, base > firstB ? base : firstB, base + B.col, B.a0 + B.a1, lane);
    }
    const bool okA = ring_drain(ctlA, mbarA);
    const bool okB = ring_drain(ctlB, mbarB);
    if (!okA || !okB) {
        flag(status, EQ_DEV_TIMEOUT);
        return false;
    }
    if (!__all_sync(kFull, codec_done(A.x)) || A.pw != 2u * hA.n_words) flag(status, EQ_DEV_BAD_END);
    if (!__all_sync(kFull, codec_done(B.x)) || B.pw != 2u * hB.n_words) flag(status, EQ_DEV_BAD_END);
    return true;
}

// Same work distribution as eq_decode_kernel (row-uniform layout only):
// SHARED = one slot table per block over tiles of P.tile_warps x chains chunks,
// otherwise one table per warp and chunk.
template <int WARPS, bool SHARED, int DT, uint32_t CODEC>
__global__ void __launch_bounds__(WARPS * 32, SHARED ? kGemvMinCtas : 1)
    eq_decode_gemv_kernel(const __grid_constant__ GemvParams P) {
    constexpr uint32_t LAYOUT = kRowUniform;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = threadIdx.x >> 5;
    const WarpSmem<WARPS, SHARED> S(smem_raw, warp, lane);
    constexpr uint32_t C = WarpSmem<WARPS, SHARED>::C;
    RingCtl *ctl = S.ctl;
    const uint32_t lt = lanemask_lt();

    if constexpr (SHARED) {
        uint32_t cur_mat = kNoLimit;
        for (uint32_t unit = blockIdx.x; unit < P.total_units; unit += gridDim.x) {
            const uint32_t mi = job_of(P, unit);
            const GemvJob &M = P.mats[mi];
            const uint32_t TW = P.tile_warps, TC = P.tile_chains;
            const uint32_t k0 = (unit - M.begin) * TW * TC;
            if (mi != cur_mat) {
                shared_table_rebuild<WARPS, LAYOUT, CODEC>(P, M, k0, lane, warp, S);
                cur_mat = mi;
            }
            const uint32_t np = S.blk[0];
            const uint32_t lane_sym = S.ref_entries[lane < np ? lane : 0] & 0xFFu;
            ChunkHead hc[C];
            bool have[C];
            for (uint32_t c = 0; c < C; ++c) {
                const uint32_t k = k0 + warp + c * TW;
                have[c] = c < TC && warp < TW && k < M.n_chunks && !ctl[0].dead && !ctl[C - 1].dead;
                if (have[c]) have[c] = shared_chunk_head<CODEC>(P, M, k, lane, np, S, hc[c]);
            }
            if constexpr (C == 2) {
                if (have[0] && have[1] && rank_mode<LAYOUT>(np) && hc[0].n == kChunkSyms &&
                    hc[1].n == kChunkSyms && M.cols % (2 * kGroupSyms) == 0) {
                    gemv_pair<DT, CODEC>(P.status, M, hc[0], hc[1], (uint64_t)(k0 + warp) * kChunkSyms,
                                  (uint64_t)(k0 + warp + TW) * kChunkSyms, S.lut_addr, S.ring,
                                  S.ring + kRingStride, S.mbar, S.mbar + 8 * kRingSegs, ctl, ctl + 1, lane, lt,
                                  lane_sym);
                    __syncwarp();
                    continue;
                }
            }
            for (uint32_t c = 0; c < C; ++c) {
                if (!have[c] || ctl->dead) continue;
                gemv_body<DT, CODEC>(P.status, M, (uint64_t)(k0 + warp + c * TW) * kChunkSyms, hc[c], np == 1,
                              S.ref_entries[0] & 0xFFu, S.lut_addr, S.ring, S.mbar, ctl, lane, lt,
                              rank_mode<LAYOUT>(np), lane_sym);
                __syncwarp();
            }
        }
    } else {
        const uint32_t stride = gridDim.x * WARPS;
        for (uint32_t c = blockIdx.x * WARPS + warp; c < P.total_units && !ctl->dead; c += stride) {
            const GemvJob &M = P.mats[job_of(P, c)];
            const uint32_t k = c - M.begin;
            ChunkHead h;
            if (!load_head<CODEC>(P, M, k, lane, h)) continue;
            const uint32_t *tab = reinterpret_cast<const uint32_t *>(h.rec + kHeadBytes<CODEC>);
            __syncwarp();  // the previous chunk's reads of the slot table are done
            const bool by_rank = rank_mode<LAYOUT>(h.n_present);
            if (!warp_table<CODEC>(tab, h.n_present, lane, nullptr, nullptr, S.lut, by_rank)) {
                flag(P.status, EQ_DEV_BAD_TABLE);
                continue;
            }
            __syncwarp();
            gemv_body<DT, CODEC>(P.status, M, (uint64_t)k * kChunkSyms, h, h.n_present == 1, tab[0] & 0xFFu, S.lut_addr,
                          S.ring, S.mbar, ctl, lane, lt, by_rank, tab[lane < h.n_present ? lane : 0] & 0xFFu);
            __syncwarp();
        }
    }
}

// y_i = 0 for every matrix of a launch (the fused kernel only adds).
struct ZeroParams {
    float *y[kMaxMatsPerLaunch];
    uint32_t rows[kMaxMatsPerLaunch];
    uint32_t n;
};

__global__ void eq_zero_rows_kernel(const __grid_constant__ ZeroParams Z) {
    for (uint32_t j = 0; j < Z.n; ++j)
        for (uint32_t r = blockIdx.x * blockDim.x + threadIdx.x; r < Z.rows[j]; r += gridDim.x * blockDim.x)
            Z.y[j][r] = 0.f;
}

// ---- host side ---------------------------------------------------------------------

// variants: [codec][shared][dtype - 1]
struct GemvSetup {
    bool ready = false;
    int sms = 0;
    KernelSetup<GemvParams> k[2][2][2];
};
std::mutex g_gemv_mu;
GemvSetup g_gemv_setup[128];

template <int DT, uint32_t CODEC>
int setup_variant(GemvSetup &d) {
    int rc = setup_kernel(d.k[CODEC][1][DT - 1], eq_decode_gemv_kernel<kGemvWarps, true, DT, CODEC>, kGemvWarps,
                          Smem<kGemvWarps, true>::kBytes, 1);
    if (rc) return rc;
    return setup_kernel(d.k[CODEC][0][DT - 1], eq_decode_gemv_kernel<kPrivateWarps, false, DT, CODEC>,
                        kPrivateWarps, Smem<kPrivateWarps, false>::kBytes, kPrivateWarps);
}

int gemv_setup(GemvSetup **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return EQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_gemv_mu);
    GemvSetup &d = g_gemv_setup[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return EQ_ERR_CUDA;
        int rc;
        if ((rc = setup_variant<EQ_INT8, kCodecRans>(d)) || (rc = setup_variant<EQ_E4M3, kCodecRans>(d)) ||
            (rc = setup_variant<EQ_INT8, kCodecHuffman>(d)) || (rc = setup_variant<EQ_E4M3, kCodecHuffman>(d)))
            return rc;
        d.ready = true;
    }
    *out = &d;
    return EQ_OK;
}

// Checks for matrices [first, first + count): x 16-byte aligned, y present,
// cols % 256 == 0 for every non-empty matrix.
int check_gemv_args(const eq_model *m, uint32_t first, uint32_t count, const void *const *xs, float *const *ys) {
    for (uint32_t i = 0; i < count; ++i) {
        const eq_matrix_info &in = m->mats[first + i].info;
        if (in.rows && !ys[i]) return EQ_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(ys[i]) % 4) return EQ_ERR_INVALID_ARG;
        if (in.rows && in.cols) {
            if (!xs[i] || reinterpret_cast<uintptr_t>(xs[i]) % 16) return EQ_ERR_INVALID_ARG;
            if (in.cols % kGroupSyms) return EQ_ERR_UNSUPPORTED;
        }
    }
    return EQ_OK;
}

// y_i = W_i x_i for matrices [first, first + count): per group of up to 16
// matrices one launch zeroing their y, then one launch per kernel variant
// (table scope x dtype) present.
int launch_gemv(const eq_model *m, uint32_t first, uint32_t count, const void *const *xs, float *const *ys,
                int32_t *d_status, cudaStream_t s) {
    int rc = check_gemv_args(m, first, count, xs, ys);
    if (rc) return rc;
    GemvSetup *dev = nullptr;
    if ((rc = gemv_setup(&dev))) return rc;
    const int sms = m->sm_limit && m->sm_limit < (uint32_t)dev->sms ? (int)m->sm_limit : dev->sms;
    for (uint32_t base = 0; base < count; base += kMaxMatsPerLaunch) {
        const uint32_t cnt = std::min<uint32_t>(kMaxMatsPerLaunch, count - base);
        ZeroParams Z{};
        uint32_t max_rows = 0;
        for (uint32_t i = 0; i < cnt; ++i) {
            const uint32_t rows = m->mats[first + base + i].info.rows;
            if (!rows) continue;
            Z.y[Z.n] = ys[base + i];
            Z.rows[Z.n++] = rows;
            max_rows = std::max(max_rows, rows);
        }
        if (Z.n) {
            eq_zero_rows_kernel<<<std::min<uint32_t>((max_rows + 255) / 256, 4u * dev->sms), 256, 0, s>>>(Z);
            if (cudaGetLastError() != cudaSuccess) return EQ_ERR_CUDA;
        }
        GemvParams P[2][2][2];
        for (auto &a : P)
            for (auto &b : a)
                for (auto &c : b) {
                    c = GemvParams{};
                    c.blob = m->d_blob;
                    c.blob_len = m->len;
                    c.status = d_status;
                }
        for (uint32_t i = 0; i < cnt; ++i) {
            const MatrixDesc &d = m->mats[first + base + i];
            if (d.info.n_chunks == 0) continue;
            const int sh = d.info.uniform_table ? 1 : 0;
            GemvParams &Pv = P[d.codec][sh][d.info.dtype - 1];
            GemvJob &J = Pv.mats[Pv.n_mats++];
            J.chunk_index = reinterpret_cast<const uint64_t *>(m->d_blob + d.chunk_index_off);
            J.scales = reinterpret_cast<const float *>(m->d_blob + d.scales_off);
            J.x = static_cast<const uint4 *>(xs[base + i]);
            J.y = ys[base + i];
            J.outliers = reinterpret_cast<const uint32_t *>(m->d_blob + d.outliers_off);
            J.n_elems = (uint64_t)d.info.rows * d.info.cols;
            J.cols = d.info.cols;
            J.rows = d.info.rows;
            J.n_chunks = d.info.n_chunks;
            J.chunk0 = 0;
            J.begin = Pv.total_units;
            J.n_out = d.info.n_outliers;
            Pv.total_units += d.info.n_chunks;  // per-chunk units; shared-table launches are re-tiled below
        }
        for (int co = 0; co < 2; ++co)
            for (int dt = 0; dt < 2; ++dt)
                assign_tiles(P[co][1][dt], (uint32_t)(sms * dev->k[co][1][dt].ctas_per_sm), kGemvWarps,
                             EQ_CHAINS);
        for (int co = 0; co < 2; ++co)
            for (int sh = 0; sh < 2; ++sh)
                for (int dt = 0; dt < 2; ++dt)
                    if ((rc = launch(dev->k[co][sh][dt], sms, P[co][sh][dt], s))) return rc;
    }
    return EQ_OK;
}

}  // namespace

extern "C" EQW_API int eq_decode_gemv_matrix(const eq_model *m, uint32_t matrix, const void *d_x, float *d_y,
                                             int32_t *d_status, cudaStream_t s) {
    const eqw::NvtxScope nvtx_range("eq_decode_gemv_matrix");
    if (!m || !d_status || matrix >= m->mats.size()) return EQ_ERR_INVALID_ARG;
    return launch_gemv(m, matrix, 1, &d_x, &d_y, d_status, s);
}

extern "C" EQW_API int eq_decode_gemv_block(const eq_model *m, uint32_t layer, const void *const *d_x,
                                            float *const *d_y, uint32_t count, int32_t *d_status, cudaStream_t s) {
    const eqw::NvtxScope nvtx_range("eq_decode_gemv_block");
    if (!m || !d_status || layer >= m->n_layers || !d_x || !d_y) return EQ_ERR_INVALID_ARG;
    if (count != m->layer_count[layer]) return EQ_ERR_INVALID_ARG;
    return launch_gemv(m, m->layer_first[layer], count, d_x, d_y, d_status, s);
}
