// Decode kernels for entropy-coded weights on B200 (sm_100a) and their
// C-ABI launchers: eq_decode_matrix, eq_decode_block, eq_decode_model_stream.
//
// EntQuant technical summary (gist.science 2601.22787), section 2
// "inference-time decoding": the compressed bitstream stays in GPU memory and
// a parallel ANS decoder expands one transformer block's weights into a
// buffer just before that block runs, densely interleaved with the forward
// kernels.  Section 2 "super weights": Int8 outliers are kept outside the
// entropy-coded stream.  EntroLLM technical overview, "parallel decoding
// strategy": independent chunks decode concurrently.
//
// Kernel KB2, eq_rans_decode_dequant_kernel (persistent, one warp per chunk):
//   prologue  load the chunk's frequency list, check it, expand it into a
//             4096-slot table in shared memory: slot -> (f, slot - cum, sym)
//             packed in one u32, so every decoded symbol costs one LDS;
//   staging   the chunk's 16-bit renormalisation words stream into a 2 KB
//             shared-memory ring in 512-byte segments with TMA bulk copies
//             (cp.async.bulk, mbarrier completion, no multicast), issued up
//             to four segments ahead by lane 0;
//   decode    each lane owns one of the 32 interleaved rANS states; a step is
//             slot = x & 4095; x = f * (x >> 12) + (slot - cum); if x < 2^16
//             the lane takes the next word, its position found from a warp
//             ballot and a popcount of the lower lanes;
//   dequant   lane l decodes symbols 8l .. 8l+7 of every 256-symbol group, so
//             after 8 steps it holds 8 consecutive outputs: value * row scale
//             (fp32, round to nearest even), packed to bf16 (round to nearest
//             even) and written with one 16-byte store; the warp's 32 stores
//             cover 512 contiguous bytes.
// Kernel KB3, eq_outlier_scatter_kernel: out[r * cols + c] = bf16(v) for the
// super weights, launched after KB2 on the same stream.
//
// No tensor cores: nothing here is a dense contraction.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>

#include "eqw_internal.h"

using namespace eqw;

namespace {

constexpr int kWarpsPerCta = 4;
constexpr int kThreads = kWarpsPerCta * 32;
constexpr uint32_t kSegWords = 256;  // one staging segment: 512 bytes
constexpr uint32_t kSegBytes = 2 * kSegWords;
constexpr uint32_t kRingSegs = 4;
constexpr uint32_t kRingWords = kSegWords * kRingSegs;
constexpr uint32_t kFull = 0xFFFFFFFFu;
// Bounded wait for a staged copy: about one second of SM clocks, after which
// the warp records EQ_DEV_TIMEOUT and stops instead of spinning forever.
constexpr long long kWaitCycles = 2000000000LL;

struct __align__(16) WarpSmem {
    uint32_t lut[kProbTotal];     // 16 KB: (f << 20) | ((slot - cum) << 8) | sym
    uint16_t ring[kRingWords];    // 2 KB of staged renormalisation words
    uint64_t mbar[kRingSegs];     // one mbarrier per ring segment
};
constexpr size_t kSmemBytes = sizeof(WarpSmem) * kWarpsPerCta;

struct MatJob {
    const uint64_t *chunk_index;  // absolute record offsets, n_chunks + 1 entries
    const float *scales;          // fp32 [rows]
    uint16_t *out;                // bf16 bits, row-major [rows, cols]
    uint64_t n_elems;
    uint32_t cols;
    uint32_t n_chunks;
    uint32_t chunk_begin;         // first launch-wide chunk id of this matrix
    uint32_t dtype;
    uint32_t aligned;             // cols % 8 == 0 and out 16-byte aligned
    uint32_t pad;
};

struct DecodeParams {
    const uint8_t *blob;
    uint64_t blob_len;
    int32_t *status;
    uint32_t n_mats;
    uint32_t total_chunks;
    MatJob mats[kMaxMatsPerLaunch];
};

struct ScatterJob {
    const uint32_t *rec;  // {row, col, value bits} x n_out
    uint16_t *out;
    uint32_t rows, cols, n_out, begin;
};

struct ScatterParams {
    int32_t *status;
    uint32_t n_jobs;
    uint32_t total;
    ScatterJob jobs[kMaxMatsPerLaunch];
};

// ---- PTX helpers: mbarrier + bulk copy (TMA, 1-D, no multicast) -------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > kWaitCycles) return false;
    }
}

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// ---- number formats -------------------------------------------------------------
// Int8: two's complement.  E4M3 (OCP E4M3FN, bias 7): placing the 7 exponent
// and mantissa bits at bit 20 of an fp32 gives value * 2^-120 exactly
// (subnormal inputs included), and multiplying by 2^120 is exact.
template <int DT>
__device__ __forceinline__ float symbol_value(uint32_t s) {
    if constexpr (DT == EQ_INT8) {
        return static_cast<float>(static_cast<int8_t>(s & 0xFFu));
    } else {
        const uint32_t b = ((s & 0x80u) << 24) | ((s & 0x7Fu) << 20);
        return __fmul_rn(__uint_as_float(b), 0x1p120f);
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint16_t to_bf16(float v) {
    __nv_bfloat16 h = __float2bfloat16_rn(v);
    return *reinterpret_cast<uint16_t *>(&h);
}

__device__ __forceinline__ void flag(int32_t *status, int32_t bits) {
    if ((threadIdx.x & 31) == 0) atomicOr(status, bits);
}

// Staging ring for one chunk's words (warp-uniform bookkeeping).
struct Ring {
    const uint8_t *payload;
    uint32_t pbytes;   // payload bytes padded to 16
    uint32_t n_segs;
    uint32_t issued;
    uint32_t ready;
    uint32_t phase;    // bit k: parity of the next completion of mbar[k]
};

__device__ __forceinline__ void ring_issue(WarpSmem &S, Ring &R, uint32_t lane) {
    const uint32_t s = R.issued++;
    if (lane == 0) {
        const uint32_t bytes = min(kSegBytes, R.pbytes - s * kSegBytes);
        uint64_t *bar = &S.mbar[s % kRingSegs];
        mbar_expect_tx(bar, bytes);
        bulk_load(&S.ring[(s % kRingSegs) * kSegWords], R.payload + (size_t)s * kSegBytes, bytes, bar);
    }
}

// Keep up to four segments in flight and make sure words [p, p + 256) are
// resident.  Returns false if a wait gave up.
__device__ __forceinline__ bool ring_prepare(WarpSmem &S, Ring &R, uint32_t p, uint32_t lane) {
    if (R.n_segs == 0) return true;
    const uint32_t horizon = (p / kSegWords) + kRingSegs;
    if (R.issued < R.n_segs && R.issued < horizon) {
        // the slots being refilled were read through the generic proxy
        __syncwarp();
        fence_proxy_async_smem();
        do {
            ring_issue(S, R, lane);
        } while (R.issued < R.n_segs && R.issued < horizon);
    }
    uint32_t need = (p + kSegWords - 1) / kSegWords;
    if (need >= R.n_segs) need = R.n_segs - 1;
    while (R.ready <= need && R.ready < R.issued) {
        const uint32_t slot = R.ready % kRingSegs;
        const bool ok = mbar_wait_bounded(&S.mbar[slot], (R.phase >> slot) & 1u);
        R.phase ^= 1u << slot;
        ++R.ready;
        if (!__all_sync(kFull, ok)) return false;
    }
    return true;
}

// Wait for every copy still in flight (bounded) so the ring can be reused.
__device__ __forceinline__ bool ring_drain(WarpSmem &S, Ring &R) {
    bool all_ok = true;
    while (R.ready < R.issued) {
        const uint32_t slot = R.ready % kRingSegs;
        const bool ok = mbar_wait_bounded(&S.mbar[slot], (R.phase >> slot) & 1u);
        R.phase ^= 1u << slot;
        ++R.ready;
        all_ok = __all_sync(kFull, ok) && all_ok;
    }
    return all_ok;
}

// Row and column of this lane's next 8 outputs (aligned layouts only).
struct RowCursor {
    uint32_t row;
    uint32_t col;
};

template <int DT>
__device__ __forceinline__ void store8_aligned(const MatJob &M, uint64_t idx, const RowCursor &rc,
                                               const uint32_t (&sy)[8]) {
    const float sc = __ldg(M.scales + rc.row);
    uint4 o;
    o.x = pack_bf16x2(__fmul_rn(symbol_value<DT>(sy[0]), sc), __fmul_rn(symbol_value<DT>(sy[1]), sc));
    o.y = pack_bf16x2(__fmul_rn(symbol_value<DT>(sy[2]), sc), __fmul_rn(symbol_value<DT>(sy[3]), sc));
    o.z = pack_bf16x2(__fmul_rn(symbol_value<DT>(sy[4]), sc), __fmul_rn(symbol_value<DT>(sy[5]), sc));
    o.w = pack_bf16x2(__fmul_rn(symbol_value<DT>(sy[6]), sc), __fmul_rn(symbol_value<DT>(sy[7]), sc));
    *reinterpret_cast<uint4 *>(M.out + idx) = o;
}

// Element-wise store of up to 8 outputs starting at idx (ragged shapes and tails).
template <int DT>
__device__ __forceinline__ void store8_generic(const MatJob &M, uint64_t idx, uint32_t count,
                                               const uint32_t (&sy)[8]) {
#pragma unroll
    for (uint32_t r = 0; r < 8; ++r) {
        if (r < count) {
            const uint64_t i = idx + r;
            const float sc = __ldg(M.scales + i / M.cols);
            M.out[i] = to_bf16(__fmul_rn(symbol_value<DT>(sy[r]), sc));
        }
    }
}

__device__ __forceinline__ void advance(RowCursor &rc, uint32_t cols) {
    rc.col += kGroupSyms;
    while (rc.col >= cols) {
        rc.col -= cols;
        ++rc.row;
    }
}

// One full 256-symbol group: 8 steps of all 32 lanes.
__device__ __forceinline__ void decode_group(const WarpSmem &S, uint32_t &x, uint32_t &p, uint32_t lt,
                                             uint32_t (&sy)[8]) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const uint32_t e = S.lut[x & (kProbTotal - 1)];
        x = (e >> 20) * (x >> kProbBits) + ((e >> 8) & 0xFFFu);
        sy[r] = e & 0xFFu;
        const bool need = x < kStateLow;
        const uint32_t b = __ballot_sync(kFull, need);
        if (need) x = (x << 16) | S.ring[(p + __popc(b & lt)) & (kRingWords - 1)];
        p += __popc(b);
    }
}

// The last, partial group: lane l is active at step r while 8l + r < rem.
__device__ __forceinline__ void decode_tail(const WarpSmem &S, uint32_t &x, uint32_t &p, uint32_t lt,
                                            uint32_t lane, uint32_t rem, uint32_t (&sy)[8]) {
#pragma unroll
    for (uint32_t r = 0; r < 8; ++r) {
        const bool active = lane * kGroup + r < rem;
        bool need = false;
        if (active) {
            const uint32_t e = S.lut[x & (kProbTotal - 1)];
            x = (e >> 20) * (x >> kProbBits) + ((e >> 8) & 0xFFFu);
            sy[r] = e & 0xFFu;
            need = x < kStateLow;
        }
        const uint32_t b = __ballot_sync(kFull, need);
        if (need) x = (x << 16) | S.ring[(p + __popc(b & lt)) & (kRingWords - 1)];
        p += __popc(b);
    }
}

// Returns false only if a bounded wait for staged words gave up: the warp's
// ring state is then unknown and it must not take further chunks.
template <int DT, bool ALIGNED>
__device__ __forceinline__ bool decode_chunk(const DecodeParams &P, const MatJob &M, uint32_t k, WarpSmem &S, uint32_t &phase,
                             uint32_t lane, uint32_t lt) {
    const uint64_t first = (uint64_t)k * kChunkSyms;
    const uint64_t rem_all = M.n_elems - first;
    const uint32_t n_expect = rem_all < kChunkSyms ? (uint32_t)rem_all : kChunkSyms;
    const uint64_t off = M.chunk_index[k];
    const uint64_t end = M.chunk_index[k + 1];
    if ((off & 15) || end > P.blob_len || end < off + kRecordHeadBytes + 16) {
        flag(P.status, EQ_DEV_BAD_HEADER);
        return true;
    }
    const uint8_t *rec = P.blob + off;
    const uint4 head = *reinterpret_cast<const uint4 *>(rec);
    const uint32_t n = head.x, n_words = head.y, n_present = head.z;
    const uint32_t table_bytes = (kRecordHeadBytes + 4 * n_present + 15) & ~15u;
    if (n != n_expect || n_present < 1 || n_present > 256 ||
        off + table_bytes + ((2ull * n_words + 15) & ~15ull) != end) {
        flag(P.status, EQ_DEV_BAD_HEADER);
        return true;
    }
    uint32_t x = reinterpret_cast<const uint32_t *>(rec + 16)[lane];
    if (!__all_sync(kFull, x >= kStateLow)) {
        flag(P.status, EQ_DEV_BAD_STATE);
        return true;
    }

    // ---- table: check it and expand it into the slot table ----
    const uint32_t *tab = reinterpret_cast<const uint32_t *>(rec + kRecordHeadBytes);
    uint32_t run = 0;
    int prev_sym = -1;
    bool ok = true;
    uint32_t single_sym = 0;
    for (uint32_t base = 0; base < n_present; base += 32) {
        const uint32_t i = base + lane;
        const bool have = i < n_present;
        const uint32_t e = have ? tab[i] : 0u;
        const uint32_t f = e >> 16, sym = e & 0xFFu;
        bool good = !have || ((e & 0xFF00u) == 0 && f >= 1 && f <= kProbTotal);
        const int left = __shfl_up_sync(kFull, (int)sym, 1);
        if (have && (int)sym <= (lane == 0 ? prev_sym : left)) good = false;
        uint32_t inc = f;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t t = __shfl_up_sync(kFull, inc, d);
            if (lane >= (uint32_t)d) inc += t;
        }
        const uint32_t cum = run + inc - f;
        ok = __all_sync(kFull, good) && ok;
        const uint32_t cnt = min(32u, n_present - base);
        if (n_present > 1) {
            for (uint32_t q = 0; q < cnt; ++q) {
                const uint32_t fq = __shfl_sync(kFull, f, q);
                const uint32_t cq = __shfl_sync(kFull, cum, q);
                const uint32_t sq = __shfl_sync(kFull, sym, q);
                for (uint32_t t = lane; t < fq; t += 32) {
                    const uint32_t slot = cq + t;
                    if (slot < kProbTotal && fq < kProbTotal) S.lut[slot] = (fq << 20) | (t << 8) | sq;
                }
            }
        } else {
            single_sym = __shfl_sync(kFull, sym, 0);
        }
        prev_sym = __shfl_sync(kFull, (int)sym, cnt - 1);
        run += __shfl_sync(kFull, inc, 31);
    }
    if (!ok || run != kProbTotal) {
        flag(P.status, EQ_DEV_BAD_TABLE);
        return true;
    }

    const uint32_t n_full = n / kGroupSyms;
    const uint32_t tail = n % kGroupSyms;
    RowCursor rc{0, 0};
    if (ALIGNED) {
        const uint64_t e0 = first + kGroup * lane;
        rc.row = (uint32_t)(e0 / M.cols);
        rc.col = (uint32_t)(e0 - (uint64_t)rc.row * M.cols);
    }

    // ---- single-symbol chunk: no payload, every state stays at 2^16 ----
    if (n_present == 1) {
        if (n_words != 0 || !__all_sync(kFull, x == kStateLow)) {
            flag(P.status, EQ_DEV_BAD_END);
            return true;
        }
        uint32_t sy[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) sy[r] = single_sym;
        for (uint32_t g = 0; g < n_full; ++g) {
            const uint64_t idx = first + (uint64_t)g * kGroupSyms + kGroup * lane;
            if (ALIGNED) {
                store8_aligned<DT>(M, idx, rc, sy);
                advance(rc, M.cols);
            } else {
                store8_generic<DT>(M, idx, 8, sy);
            }
        }
        if (tail) {
            const uint32_t mine = tail > kGroup * lane ? min(8u, tail - kGroup * lane) : 0u;
            store8_generic<DT>(M, first + (uint64_t)n_full * kGroupSyms + kGroup * lane, mine, sy);
        }
        return true;
    }

    // ---- stream the words and decode ----
    __syncwarp();
    Ring R;
    R.payload = rec + table_bytes;
    R.pbytes = (2u * n_words + 15u) & ~15u;
    R.n_segs = (R.pbytes + kSegBytes - 1) / kSegBytes;
    R.issued = 0;
    R.ready = 0;
    R.phase = phase;

    uint32_t p = 0;
    bool alive = true;
    for (uint32_t g = 0; g < n_full; ++g) {
        if (!ring_prepare(S, R, p, lane)) {
            alive = false;
            break;
        }
        uint32_t sy[8];
        decode_group(S, x, p, lt, sy);
        const uint64_t idx = first + (uint64_t)g * kGroupSyms + kGroup * lane;
        if (ALIGNED) {
            store8_aligned<DT>(M, idx, rc, sy);
            advance(rc, M.cols);
        } else {
            store8_generic<DT>(M, idx, 8, sy);
        }
    }
    if (alive && tail) {
        if (!ring_prepare(S, R, p, lane)) {
            alive = false;
        } else {
            uint32_t sy[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            decode_tail(S, x, p, lt, lane, tail, sy);
            const uint32_t mine = tail > kGroup * lane ? min(8u, tail - kGroup * lane) : 0u;
            store8_generic<DT>(M, first + (uint64_t)n_full * kGroupSyms + kGroup * lane, mine, sy);
        }
    }
    const bool drained = ring_drain(S, R);
    phase = R.phase;
    if (!alive || !drained) {
        flag(P.status, EQ_DEV_TIMEOUT);
        return false;
    }
    // a valid stream returns every state to 2^16 and consumes exactly n_words
    if (!__all_sync(kFull, x == kStateLow) || p != n_words) flag(P.status, EQ_DEV_BAD_END);
    return true;
}

__global__ void __launch_bounds__(kThreads) eq_rans_decode_dequant_kernel(const __grid_constant__ DecodeParams P) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = threadIdx.x >> 5;
    WarpSmem &S = reinterpret_cast<WarpSmem *>(smem_raw)[warp];
    if (lane == 0) {
        for (uint32_t i = 0; i < kRingSegs; ++i) mbar_init(&S.mbar[i], 1);
        fence_mbar_init();
    }
    __syncwarp();
    const uint32_t lt = lanemask_lt();
    uint32_t phase = 0;
    const uint32_t stride = gridDim.x * kWarpsPerCta;
    for (uint32_t c = blockIdx.x * kWarpsPerCta + warp; c < P.total_chunks; c += stride) {
        uint32_t mi = 0;
        while (mi + 1 < P.n_mats && c >= P.mats[mi + 1].chunk_begin) ++mi;
        const MatJob &M = P.mats[mi];
        const uint32_t k = c - M.chunk_begin;
        bool go;
        if (M.dtype == EQ_INT8) {
            go = M.aligned ? decode_chunk<EQ_INT8, true>(P, M, k, S, phase, lane, lt)
                           : decode_chunk<EQ_INT8, false>(P, M, k, S, phase, lane, lt);
        } else {
            go = M.aligned ? decode_chunk<EQ_E4M3, true>(P, M, k, S, phase, lane, lt)
                           : decode_chunk<EQ_E4M3, false>(P, M, k, S, phase, lane, lt);
        }
        __syncwarp();
        if (!go) break;
    }
}

__global__ void eq_outlier_scatter_kernel(const __grid_constant__ ScatterParams P) {
    const uint32_t t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= P.total) return;
    uint32_t j = 0;
    while (j + 1 < P.n_jobs && t >= P.jobs[j + 1].begin) ++j;
    const ScatterJob &J = P.jobs[j];
    const uint32_t *r = J.rec + 3ull * (t - J.begin);
    const uint32_t row = r[0], col = r[1];
    const float v = __uint_as_float(r[2]);
    if (row >= J.rows || col >= J.cols) {
        atomicOr(P.status, EQ_DEV_BAD_OUTLIER);
        return;
    }
    J.out[(uint64_t)row * J.cols + col] = to_bf16(v);
}

// ---- host side ---------------------------------------------------------------------

struct DeviceSetup {
    bool ready = false;
    int sms = 0;
    int ctas_per_sm = 0;
};
std::mutex g_setup_mu;
DeviceSetup g_setup[128];

int device_setup(DeviceSetup **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return EQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    DeviceSetup &d = g_setup[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return EQ_ERR_CUDA;
        if (cudaFuncSetAttribute(eq_rans_decode_dequant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemBytes) != cudaSuccess)
            return EQ_ERR_CUDA;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.ctas_per_sm, eq_rans_decode_dequant_kernel, kThreads,
                                                          kSmemBytes) != cudaSuccess ||
            d.ctas_per_sm < 1)
            return EQ_ERR_CUDA;
        d.ready = true;
    }
    *out = &d;
    return EQ_OK;
}

// Decode matrices [first, first + count) of the model into outs[i].
int launch_decode(const eq_model *m, uint32_t first, uint32_t count, uint16_t *const *outs, int32_t *d_status,
                  cudaStream_t s) {
    DeviceSetup *dev = nullptr;
    int rc = device_setup(&dev);
    if (rc) return rc;
    for (uint32_t base = 0; base < count; base += kMaxMatsPerLaunch) {
        const uint32_t cnt = std::min<uint32_t>(kMaxMatsPerLaunch, count - base);
        DecodeParams P{};
        P.blob = m->d_blob;
        P.blob_len = m->len;
        P.status = d_status;
        ScatterParams Q{};
        Q.status = d_status;
        uint32_t chunks = 0, n_out = 0;
        for (uint32_t i = 0; i < cnt; ++i) {
            const MatrixDesc &d = m->mats[first + base + i];
            if (d.info.n_chunks == 0) continue;
            MatJob &J = P.mats[P.n_mats++];
            J.chunk_index = reinterpret_cast<const uint64_t *>(m->d_blob + d.chunk_index_off);
            J.scales = reinterpret_cast<const float *>(m->d_blob + d.scales_off);
            J.out = outs[base + i];
            J.n_elems = (uint64_t)d.info.rows * d.info.cols;
            J.cols = d.info.cols;
            J.n_chunks = d.info.n_chunks;
            J.chunk_begin = chunks;
            J.dtype = d.info.dtype;
            J.aligned = (d.info.cols % kGroup == 0) && (reinterpret_cast<uintptr_t>(J.out) % 16 == 0);
            chunks += d.info.n_chunks;
            if (d.info.n_outliers) {
                ScatterJob &O = Q.jobs[Q.n_jobs++];
                O.rec = reinterpret_cast<const uint32_t *>(m->d_blob + d.outliers_off);
                O.out = outs[base + i];
                O.rows = d.info.rows;
                O.cols = d.info.cols;
                O.n_out = d.info.n_outliers;
                O.begin = n_out;
                n_out += d.info.n_outliers;
            }
        }
        P.total_chunks = chunks;
        Q.total = n_out;
        if (chunks) {
            const uint32_t want = (chunks + kWarpsPerCta - 1) / kWarpsPerCta;
            const uint32_t grid = std::min<uint32_t>(want, (uint32_t)(dev->sms * dev->ctas_per_sm));
            eq_rans_decode_dequant_kernel<<<grid, kThreads, kSmemBytes, s>>>(P);
            if (cudaGetLastError() != cudaSuccess) return EQ_ERR_CUDA;
        }
        if (n_out) {
            eq_outlier_scatter_kernel<<<(n_out + 127) / 128, 128, 0, s>>>(Q);
            if (cudaGetLastError() != cudaSuccess) return EQ_ERR_CUDA;
        }
    }
    return EQ_OK;
}

}  // namespace

extern "C" EQW_API int eq_decode_matrix(const eq_model *m, uint32_t matrix, void *d_out, size_t out_bytes,
                                        int32_t *d_status, cudaStream_t s) {
    if (!m || !d_status || matrix >= m->mats.size()) return EQ_ERR_INVALID_ARG;
    const eq_matrix_info &in = m->mats[matrix].info;
    const uint64_t need = 2ull * in.rows * in.cols;
    if (need && (!d_out || reinterpret_cast<uintptr_t>(d_out) % 2)) return EQ_ERR_INVALID_ARG;
    if (out_bytes < need) return EQ_ERR_NOSPACE;
    uint16_t *out = static_cast<uint16_t *>(d_out);
    return launch_decode(m, matrix, 1, &out, d_status, s);
}

extern "C" EQW_API int eq_decode_block(const eq_model *m, uint32_t layer, void *d_out, size_t out_bytes,
                                       int32_t *d_status, cudaStream_t s) {
    if (!m || !d_status || layer >= m->n_layers) return EQ_ERR_INVALID_ARG;
    const uint32_t first = m->layer_first[layer], count = m->layer_count[layer];
    size_t offs[256];
    std::vector<size_t> big;
    size_t *o = offs;
    if (count > 256) {
        big.resize(count);
        o = big.data();
    }
    size_t total = 0;
    int rc = eq_block_layout(m, layer, o, count, &total);
    if (rc) return rc;
    if (total && (!d_out || reinterpret_cast<uintptr_t>(d_out) % 16)) return EQ_ERR_INVALID_ARG;
    if (out_bytes < total) return EQ_ERR_NOSPACE;
    std::vector<uint16_t *> outs(count);
    for (uint32_t i = 0; i < count; ++i)
        outs[i] = reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(d_out) + o[i]);
    return launch_decode(m, first, count, outs.data(), d_status, s);
}

extern "C" EQW_API int eq_decode_model_stream(const eq_model *m, uint32_t layer, void *const d_buf[2],
                                              size_t buf_bytes, int32_t *d_status, cudaStream_t decode_stream,
                                              cudaEvent_t const ev_free[2], cudaEvent_t const ev_ready[2]) {
    if (!m || !d_buf || !ev_free || !ev_ready || layer >= m->n_layers) return EQ_ERR_INVALID_ARG;
    const uint32_t b = layer & 1u;
    if (!ev_ready[b]) return EQ_ERR_INVALID_ARG;
    if (ev_free[b] && cudaStreamWaitEvent(decode_stream, ev_free[b], 0) != cudaSuccess) return EQ_ERR_CUDA;
    int rc = eq_decode_block(m, layer, d_buf[b], buf_bytes, d_status, decode_stream);
    if (rc) return rc;
    if (cudaEventRecord(ev_ready[b], decode_stream) != cudaSuccess) return EQ_ERR_CUDA;
    return EQ_OK;
}
