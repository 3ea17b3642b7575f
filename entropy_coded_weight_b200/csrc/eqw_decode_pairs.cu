// KP, eq_decode_pairs_kernel: the decode kernel for the common case of
// eqw_decode.cu's KB2 -- matrices whose chunks all carry one frequency table
// with 2..32 distinct symbols (rank-mode dequant), rows a multiple of 512
// symbols, bf16 output -- decoded two full chunks per warp in lockstep.
//
// EntQuant technical summary (gist.science 2601.22787), section 2
// "inference-time decoding": a block's compressed weights are expanded into a
// bf16 buffer just before the block runs; EntroLLM technical overview,
// "parallel decoding strategy": independent chunks decode concurrently.
//
// Same format, same step and dequant arithmetic as KB2 (bit-identical
// output); what differs:
//   work split   the launch's chunk pairs (chunks 2i, 2i+1 of a matrix) are cut
//                into one contiguous range per block, so every SM gets the
//                same number of pairs to within one; a range touches at most
//                kPairTables matrices, whose slot tables are all built once at
//                block start -- no barrier after that.  KB2's fixed tiles of 48
//                chunks leave a 70B-shape block's last round 84 % full.
//   word ring    the same 2 KB TMA-fed ring per chain (four 512-byte segments
//                plus a mirror of segment 0), with its counters in registers
//                and segments numbered across the chain's chunks, so the
//                slot and the mbarrier phase of a segment follow from its
//                number; the service (one bulk copy issued, one segment
//                waited per 512 bytes consumed) is inline code.
//   loop         runs of iterations between row changes carry no row checks,
//                and one test covers both chains' ring limits.
// A matrix's chunks that do not form full pairs (an odd last chunk, a short
// tail chunk) are left to KB2 (eq_decode.cu launches it for the remainder), as
// are launches with fewer pairs than warps (latency-bound: KB2 spreads those
// over more warps, one chain each).
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>
#include <utility>
#include <vector>

#include "eqw_device.cuh"
#include "eqw_pairs.h"

namespace {

#ifndef EQ_PAIR_WARPS
#define EQ_PAIR_WARPS 24
#endif
constexpr int kPairWarps = EQ_PAIR_WARPS;
constexpr uint32_t kPairTables = 3;        // matrices one block's range may touch
constexpr uint32_t kQPerChunk = kChunkSyms / (2 * kGroupSyms);  // iterations of two groups

struct PairJob {
    const uint64_t *chunk_index;  // absolute record offsets, n_chunks + 1 entries
    const float *scales;          // fp32 [rows]
    uint16_t *out;                // bf16 bits, row-major [rows, cols]
    uint32_t cols, rows;
    uint32_t first_pair;          // launch-wide index of this matrix's first pair
    uint32_t n_pairs;             // pairs decoded here: chunks [0, 2 n_pairs)
};

struct PairParams {
    const uint8_t *blob;
    uint64_t blob_len;
    int32_t *status;
    uint32_t n_mats;
    uint32_t total_pairs;
    PairJob mats[kMaxMatsPerLaunch];
};

template <int WARPS, int C>
struct PairSmem {
    static constexpr uint32_t kChains = C * WARPS;
    static constexpr uint32_t kRingOff = kPairTables * kLutBytes;
    static constexpr uint32_t kMbarOff = kRingOff + kChains * kRingStride;
    static constexpr uint32_t kSrcOff = kMbarOff + kChains * kRingSegs * 8;
    static constexpr uint32_t kRefOff = kSrcOff + kChains * 16;  // per table: 32 entries, 32 cum
    static constexpr uint32_t kMetaOff = kRefOff + kPairTables * 64 * 4;      // per table: n_present (0: invalid)
    static constexpr uint32_t kBytes = kMetaOff + kPairTables * 4;
};
constexpr int kTuple = 2;  // chunks decoded in lockstep per warp
static_assert(PairSmem<kPairWarps, kTuple>::kBytes <= 227 * 1024, "pair kernel shared memory");
static_assert(PairSmem<kPairWarps, kTuple>::kRingOff % 128 == 0, "ring alignment");

template <class Params>
__device__ __forceinline__ uint32_t pair_job(const Params &P, uint32_t pair, uint32_t from) {
    uint32_t mi = from;
    while (mi + 1 < P.n_mats && pair >= P.mats[mi + 1].first_pair) ++mi;
    return mi;
}

// Ring bookkeeping of one chain.  Segments are numbered across the chain's
// chunks (a chunk's payload starts on a fresh segment), so segment g always
// lands in slot g % 4 and its completion is the (g / 4)-th phase of that slot's
// mbarrier: the wait parity is bit 2 of g, nothing to track.  Byte positions P
// count in the same frame (P = 512 g + offset within segment g).
struct RingRegs {
    uint32_t issued;  // next segment to copy
    uint32_t ready;   // next segment to wait for
};

// Where a chain's ring refills from: the chunk's payload, its size and the
// number of its first segment.
struct TupleSrc {
    const uint8_t *payload;
    uint32_t pbytes;  // payload bytes rounded up to 16
    uint32_t g0;      // frame number of the payload's first segment
};

// Service of one chain's ring: copy the segments whose slots hold only bytes
// before P, then wait until bytes [P, P + kSpan) are resident.  Returns the
// position at which the ring next needs service.  A wait that gives up sets
// `dead` and leaves that segment not ready, so the drain waits for it again.
__device__ __forceinline__ uint32_t tuple_service(RingRegs &R, uint32_t P, uint32_t gend, uint32_t ring,
                                                  uint32_t mbar, const TupleSrc *src, bool &dead, int32_t *status) {
    const uint32_t horizon = min(gend, P / kSegBytes + kRingSegs);
    if (R.issued < horizon) {
        __syncwarp();
        fence_proxy_async_smem();  // the slots being refilled were read through the generic proxy
        if ((threadIdx.x & 31u) == 0) {
            const uint32_t g0 = src->g0, pbytes = src->pbytes;
            const uint8_t *payload = src->payload;
            for (uint32_t g = R.issued; g < horizon; ++g) {
                const uint32_t off = (g - g0) * kSegBytes;
                const uint32_t bytes = min(kSegBytes, pbytes - off);
                const uint32_t slot = g % kRingSegs;
                check(status, off < pbytes && off + bytes <= pbytes && bytes % 16 == 0);
                mbar_expect_tx(mbar + 8 * slot, slot == 0 ? 2 * bytes : bytes);
                bulk_load(ring + slot * kSegBytes, payload + off, bytes, mbar + 8 * slot);
                if (slot == 0) bulk_load(ring + kRingBytes, payload + off, bytes, mbar);
            }
        }
        R.issued = horizon;
    }
    const uint32_t need = min(R.issued, (P + kSpan - 1) / kSegBytes + 1);  // segments below `need` resident
    while (R.ready < need) {
        const uint32_t slot = R.ready % kRingSegs;
        if (!__all_sync(kFull, mbar_wait_bounded(mbar + 8 * slot, (R.ready / kRingSegs) & 1u))) {
            dead = true;
            return kNoLimit;
        }
        ++R.ready;
    }
    uint32_t lim = R.ready < gend ? R.ready * kSegBytes - (kSpan - 1) : kNoLimit;
    if (R.issued < gend) lim = min(lim, (R.issued - (kRingSegs - 1)) * kSegBytes);
    return lim;
}

// Wait (bounded) for every copy of this chain still in flight.
__device__ __forceinline__ bool tuple_drain(RingRegs &R, uint32_t mbar) {
    bool ok = true;
    for (; R.ready < R.issued; ++R.ready)
        ok = __all_sync(kFull, mbar_wait_bounded(mbar + 8 * (R.ready % kRingSegs), (R.ready / kRingSegs) & 1u)) &&
             ok;
    return ok;
}

// Chunk k's header checked against the directory and its frequency list
// against the block's reference list for the matrix.
template <uint32_t CODEC>
__device__ __forceinline__ bool pair_head(const PairParams &P, const PairJob &M, uint32_t k, uint32_t lane,
                                          uint32_t np, const uint32_t *ref, ChunkHead &h) {
    const uint64_t off = M.chunk_index[k];
    const uint64_t end = M.chunk_index[k + 1];
    if ((off & 15) || end > P.blob_len || end < off + kHeadBytes<CODEC> + 16) {
        flag(P.status, EQ_DEV_BAD_HEADER);
        return false;
    }
    h.rec = P.blob + off;
    const uint4 head = *reinterpret_cast<const uint4 *>(h.rec);
    h.n = head.x;
    h.n_words = head.y;
    h.n_present = head.z;
    h.table_bytes = (kHeadBytes<CODEC> + 4 * h.n_present + 15) & ~15u;
    if (h.n != kChunkSyms || h.n_present != np || off + h.table_bytes + ((2ull * h.n_words + 15) & ~15ull) != end) {
        flag(P.status, h.n_present != np ? EQ_DEV_BAD_TABLE : EQ_DEV_BAD_HEADER);
        return false;
    }
    const uint32_t *tab = reinterpret_cast<const uint32_t *>(h.rec + kHeadBytes<CODEC>);
    const bool same = lane >= np || tab[lane] == ref[lane];
    if (!__all_sync(kFull, same)) {
        flag(P.status, EQ_DEV_BAD_TABLE);
        return false;
    }
    if constexpr (CODEC == kCodecHuffman) {
        h.x = 0;
    } else {
        h.x = reinterpret_cast<const uint32_t *>(h.rec + 16)[lane];
        if (!__all_sync(kFull, h.x >= kStateLow)) {
            flag(P.status, EQ_DEV_BAD_STATE);
            return false;
        }
    }
    return true;
}

// One chain's decode state in the hot loop.
// One chain's decode state in the hot loop.
template <uint32_t CODEC>
struct TupleChain {
    CodecState<CODEC> x;
    uint32_t P;      // consumed payload bytes, in the ring's frame
    uint32_t limit;  // P at which the ring next needs service
    uint32_t gend;   // frame number one past the chunk's last segment
    RingRegs R;
    uint32_t row;    // output row of the current group
    uint32_t qrow;   // iteration at which the row next changes
    float vr;        // this lane's rank value times the row scale
    uint16_t *dst;
};

// One 256-symbol group of all C chains, interleaved step by step; each lane's
// 8 dequantised outputs of a chain leave as one 16-byte store (at byte offset
// byte_off from the chain's current output position).
template <uint32_t CODEC, int C>
__device__ __forceinline__ void tuple_group(uint32_t lut, uint32_t ring0, TupleChain<CODEC> (&ch)[C], uint32_t lt,
                                            uint32_t byte_off, int32_t *status) {
    uint32_t r0[C], rp[C], o[C][4];
#pragma unroll
    for (int c = 0; c < C; ++c) rp[c] = r0[c] = ring0 + c * kRingStride + (ch[c].P & (kRingBytes - 1));
#pragma unroll
    for (int r = 0; r < 8; r += 2) {
        uint32_t e0[C], e1[C];
#pragma unroll
        for (int c = 0; c < C; ++c) e0[c] = codec_step<CODEC>(lut, rp[c], ch[c].x, lt);
#pragma unroll
        for (int c = 0; c < C; ++c) e1[c] = codec_step<CODEC>(lut, rp[c], ch[c].x, lt);
#pragma unroll
        for (int c = 0; c < C; ++c)
            o[c][r / 2] = pack_bf16x2(make_float2(__shfl_sync(kFull, ch[c].vr, e0[c]),
                                                  __shfl_sync(kFull, ch[c].vr, e1[c])));
    }
#pragma unroll
    for (int c = 0; c < C; ++c) {
        // every word read lay in [r0, rp]: inside this chain's ring and its mirror
        check(status, rp[c] + 2 <= ring0 + c * kRingStride + kRingStride);
        st_global_v4(reinterpret_cast<uint16_t *>(reinterpret_cast<uint8_t *>(ch[c].dst) + byte_off),
                     make_uint4(o[c][0], o[c][1], o[c][2], o[c][3]));
        ch[c].P += rp[c] - r0[c];
    }
}

// Decode chunks k0 .. k0 + C - 1 of matrix M (all full) in lockstep.  R[c] and
// g[c] carry chain c's ring counters and next free frame segment in and out.
// Returns false if a bounded wait gave up (the warp must stop).
template <uint32_t CODEC, int C>
__device__ __forceinline__ bool decode_tuple(int32_t *status, const PairJob &M, const ChunkHead (&h)[C], uint32_t k0,
                                             uint32_t lut, uint32_t ring0, uint32_t mbar0, TupleSrc *src,
                                             uint32_t lane, uint32_t lt, float vraw, RingRegs (&R)[C],
                                             uint32_t (&g)[C]) {
    TupleChain<CODEC> ch[C];
    uint32_t g0[C];
    const uint32_t qpr = M.cols / (2 * kGroupSyms);  // iterations per row
#pragma unroll
    for (int c = 0; c < C; ++c) {
        const uint32_t pb = (2u * h[c].n_words + 15u) & ~15u;
        if (lane == 0) {
            src[c].payload = h[c].rec + h[c].table_bytes;
            src[c].pbytes = pb;
            src[c].g0 = g[c];
        }
        const uint64_t first = (uint64_t)(k0 + c) * kChunkSyms;
        g0[c] = g[c];
        ch[c].x = codec_start<CODEC>(h[c].x);
        ch[c].P = g[c] * kSegBytes;
        ch[c].gend = g[c] + (pb + kSegBytes - 1) / kSegBytes;
        ch[c].R = R[c];
        ch[c].limit = pb ? 0u : kNoLimit;
        ch[c].row = (uint32_t)(first / M.cols);
        ch[c].qrow = (uint32_t)(M.cols - (first - (uint64_t)ch[c].row * M.cols)) / (2 * kGroupSyms);
        ch[c].vr = __fmul_rn(vraw, __ldg(M.scales + ch[c].row));
        ch[c].dst = M.out + first + kGroup * lane;
    }
    __syncwarp();
    bool dead = false;
    uint32_t q = 0;
    while (q < kQPerChunk && !dead) {
        // a run of iterations up to the next row change of any chain
        uint32_t qe = kQPerChunk;
#pragma unroll
        for (int c = 0; c < C; ++c) qe = min(qe, ch[c].qrow);
        for (; q < qe; ++q) {
            bool svc = false;
#pragma unroll
            for (int c = 0; c < C; ++c) svc = svc || ch[c].P >= ch[c].limit;
            if (svc) {
#pragma unroll
                for (int c = 0; c < C; ++c)
                    if (ch[c].P >= ch[c].limit)
                        ch[c].limit = tuple_service(ch[c].R, ch[c].P, ch[c].gend, ring0 + c * kRingStride,
                                                    mbar0 + 8 * kRingSegs * c, src + c, dead, status);
                if (dead) break;
            }
            tuple_group<CODEC, C>(lut, ring0, ch, lt, 0, status);
            tuple_group<CODEC, C>(lut, ring0, ch, lt, 2 * kGroupSyms, status);
#pragma unroll
            for (int c = 0; c < C; ++c) {
#if EQ_CHECKED
                // the words consumed were waited for; the two stores lay inside the matrix
                const uint32_t pb = (2u * h[c].n_words + 15u) & ~15u;
                const uint32_t resident = ch[c].R.ready < ch[c].gend ? ch[c].R.ready * kSegBytes : g0[c] * kSegBytes + pb;
                check(status, ch[c].P <= resident);
                check(status, (uint64_t)(ch[c].dst - M.out) + 2 * kGroupSyms - kGroup * lane <=
                                  (uint64_t)M.rows * M.cols);
#endif
                ch[c].dst += 2 * kGroupSyms;
            }
        }
#pragma unroll
        for (int c = 0; c < C; ++c)
            if (ch[c].qrow == q) {
                ch[c].qrow += qpr;
                if (++ch[c].row < M.rows) ch[c].vr = __fmul_rn(vraw, __ldg(M.scales + ch[c].row));
            }
    }
    bool drained = true;
#pragma unroll
    for (int c = 0; c < C; ++c) {
        drained = tuple_drain(ch[c].R, mbar0 + 8 * kRingSegs * c) && drained;
        R[c] = ch[c].R;
        g[c] = ch[c].R.issued;  // the next chunk starts on a fresh segment
    }
    if (dead || !drained) {
        flag(status, EQ_DEV_TIMEOUT);
        return false;
    }
    // a valid stream returns every state to its start value and consumes exactly n_words
    bool ok = true;
#pragma unroll
    for (int c = 0; c < C; ++c) ok = ok && codec_done(ch[c].x) && ch[c].P - g0[c] * kSegBytes == 2u * h[c].n_words;
    if (!__all_sync(kFull, ok)) flag(status, EQ_DEV_BAD_END);
    return true;
}

template <int WARPS, int C, int DT, uint32_t CODEC>
__global__ void __launch_bounds__(WARPS * 32, 1) eq_decode_pairs_kernel(const __grid_constant__ PairParams P) {
    extern __shared__ __align__(1024) unsigned char smem[];
    using L = PairSmem<WARPS, C>;
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = threadIdx.x >> 5;
    const uint32_t base = smem_u32(smem);
    const uint32_t ring0 = base + L::kRingOff + warp * C * kRingStride;
    const uint32_t mbar0 = base + L::kMbarOff + warp * C * kRingSegs * 8;
    TupleSrc *src = reinterpret_cast<TupleSrc *>(smem + L::kSrcOff) + C * warp;
    uint32_t *ref = reinterpret_cast<uint32_t *>(smem + L::kRefOff);
    uint32_t *meta = reinterpret_cast<uint32_t *>(smem + L::kMetaOff);
    if (lane == 0) {
        for (uint32_t i = 0; i < C * kRingSegs; ++i) mbar_init(mbar0 + 8 * i, 1);
        fence_mbar_init();
    }
    // this block's contiguous range of the launch's tuples
    const uint32_t p0 = (uint32_t)((uint64_t)blockIdx.x * P.total_pairs / gridDim.x);
    const uint32_t p1 = (uint32_t)((uint64_t)(blockIdx.x + 1) * P.total_pairs / gridDim.x);
    if (p0 >= p1) return;
    const uint32_t m_lo = pair_job(P, p0, 0);
    const uint32_t nt = pair_job(P, p1 - 1, m_lo) - m_lo + 1;  // <= kPairTables (checked by the host)

    // reference frequency list of each matrix in the range: that of the range's
    // first chunk of the matrix, checked; every chunk decoded is compared with it
    if (warp < nt) {
        const PairJob &M = P.mats[m_lo + warp];
        const uint32_t k = C * (max(p0, M.first_pair) - M.first_pair);
        const uint64_t off = M.chunk_index[k];
        bool ok = (off & 15) == 0 && off + kHeadBytes<CODEC> + 16 <= P.blob_len;
        uint32_t np = 0;
        if (ok) {
            np = reinterpret_cast<const uint32_t *>(P.blob + off)[2];
            ok = np >= 2 && np <= 32 && off + kHeadBytes<CODEC> + 4ull * np <= P.blob_len;
        }
        if (ok)
            ok = warp_table<CODEC>(reinterpret_cast<const uint32_t *>(P.blob + off + kHeadBytes<CODEC>), np, lane,
                                   ref + 64 * warp, ref + 64 * warp + 32, nullptr, false);
        if (!ok) flag(P.status, EQ_DEV_BAD_TABLE);
        if (lane == 0) meta[warp] = ok ? np : 0u;
    }
    __syncthreads();
    for (uint32_t j = 0; j < nt; ++j) {
        const uint32_t np = meta[j];
        uint32_t *lut = reinterpret_cast<uint32_t *>(smem) + j * kProbTotal;
        for (uint32_t i = 0; i < np; ++i) {
            const uint32_t e = ref[64 * j + i], c = ref[64 * j + 32 + i];
            const uint32_t f = entry_slots<CODEC>(e);
            for (uint32_t t = threadIdx.x; t < f; t += WARPS * 32)
                if (c + t < kProbTotal && f < kProbTotal) lut[c + t] = slot_entry<CODEC>(e, f, t, i);
        }
    }
    __syncthreads();
    for (uint32_t j = 0; j < nt; ++j)
        if (meta[j]) check_table<CODEC>(P.status, reinterpret_cast<uint32_t *>(smem) + j * kProbTotal, threadIdx.x,
                                        WARPS * 32);

    const uint32_t lt = lanemask_lt();
    RingRegs R[C];  // ring counters and frame position carry over from tuple to tuple
    uint32_t g[C];
#pragma unroll
    for (int c = 0; c < C; ++c) R[c].issued = R[c].ready = g[c] = 0;
    uint32_t mi = m_lo;
    for (uint32_t p = p0 + warp; p < p1; p += WARPS) {
        mi = pair_job(P, p, mi);
        const uint32_t j = mi - m_lo;
        const uint32_t np = meta[j];
        if (!np) continue;
        const PairJob &M = P.mats[mi];
        const uint32_t k0 = C * (p - M.first_pair);
        ChunkHead h[C];
        bool ok = true;
#pragma unroll
        for (int c = 0; c < C; ++c) ok = ok && pair_head<CODEC>(P, M, k0 + c, lane, np, ref + 64 * j, h[c]);
        if (!ok) continue;
        const float vraw = symbol_value<DT>(ref[64 * j + (lane < np ? lane : 0)] & 0xFFu);
        if (!decode_tuple<CODEC, C>(P.status, M, h, k0, base + j * kLutBytes, ring0, mbar0, src, lane, lt, vraw, R, g))
            break;
    }
}

// ---- host ----------------------------------------------------------------------------

struct PairSetup {
    bool ready = false;
    KernelSetup<PairParams> k[2][2];  // [codec][dtype - 1]
};
std::mutex g_pair_mu;
PairSetup g_pair[128];

template <int DT, uint32_t CODEC>
int pair_setup_one(PairSetup &d) {
    return setup_kernel(d.k[CODEC][DT - 1], eq_decode_pairs_kernel<kPairWarps, kTuple, DT, CODEC>, kPairWarps,
                        PairSmem<kPairWarps, kTuple>::kBytes, 1);
}

int pair_setup(PairSetup **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return EQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_pair_mu);
    PairSetup &d = g_pair[dev];
    if (!d.ready) {
        int rc;
        if ((rc = pair_setup_one<EQ_INT8, kCodecRans>(d)) || (rc = pair_setup_one<EQ_E4M3, kCodecRans>(d)) ||
            (rc = pair_setup_one<EQ_INT8, kCodecHuffman>(d)) || (rc = pair_setup_one<EQ_E4M3, kCodecHuffman>(d)))
            return rc;
        d.ready = true;
    }
    *out = &d;
    return EQ_OK;
}

// True if P can go to the pair kernel on `sms` SMs: the launch gives every
// warp a pair at least once (a launch with less than one round of pairs per
// warp is bound by the latency of each chunk's dependent steps; KB2 spreads it
// over more warps, one chain each, and takes the whole call in one launch) and
// no block's range touches more than kPairTables matrices.
bool pairs_fit(const PairParams &P, uint32_t sms) {
    if (!P.total_pairs || P.total_pairs < sms * (uint32_t)kPairWarps) return false;
    const uint32_t grid = std::min<uint32_t>(sms, P.total_pairs);
    for (uint32_t b = 0; b < grid; ++b) {
        const uint32_t p0 = (uint32_t)((uint64_t)b * P.total_pairs / grid);
        const uint32_t p1 = (uint32_t)((uint64_t)(b + 1) * P.total_pairs / grid);
        if (p0 >= p1) continue;
        uint32_t lo = 0;
        while (lo + 1 < P.n_mats && p0 >= P.mats[lo + 1].first_pair) ++lo;
        uint32_t hi = lo;
        while (hi + 1 < P.n_mats && p1 - 1 >= P.mats[hi + 1].first_pair) ++hi;
        if (hi - lo + 1 > kPairTables) return false;
    }
    return true;
}

}  // namespace

namespace eqw {

bool pair_eligible(const MatrixDesc &d, const void *out) {
    const eq_matrix_info &in = d.info;
    const uint64_t n = (uint64_t)in.rows * in.cols;
    return in.uniform_table && d.n_present0 >= 2 && d.n_present0 <= 32 && in.cols % (2 * kGroupSyms) == 0 &&
           reinterpret_cast<uintptr_t>(out) % 16 == 0 && n >= (uint64_t)kTuple * kChunkSyms;
}

// A launch of the pair kernel: codec, dtype and its parameters.
struct PairLaunch {
    uint32_t codec, dtype;
    PairParams P;
};

// The launches for matrices mats[0..count) written to outs[]: one per (codec,
// dtype) and up to kMaxMatsPerLaunch matrices, each kept only where pairs_fit;
// handled[i] = leading chunks of mats[i] they decode.  Host only.
static void plan_pairs(const eq_model *m, const uint32_t *mats, uint16_t *const *outs, uint32_t count,
                       int32_t *d_status, uint32_t sms, std::vector<PairLaunch> &launches, uint32_t *handled) {
    for (uint32_t i = 0; i < count; ++i) handled[i] = 0;
    for (uint32_t co = 0; co < 2; ++co)
        for (uint32_t dt = 0; dt < 2; ++dt) {
            std::vector<uint32_t> ids;
            for (uint32_t i = 0; i < count; ++i) {
                const MatrixDesc &d = m->mats[mats[i]];
                if (d.codec == co && d.info.dtype == dt + 1 && pair_eligible(d, outs[i])) ids.push_back(i);
            }
            for (size_t base = 0; base < ids.size(); base += kMaxMatsPerLaunch) {
                const size_t cnt = std::min<size_t>(kMaxMatsPerLaunch, ids.size() - base);
                PairParams P{};
                P.blob = m->d_blob;
                P.blob_len = m->len;
                P.status = d_status;
                for (size_t t = 0; t < cnt; ++t) {
                    const MatrixDesc &d = m->mats[mats[ids[base + t]]];
                    PairJob &J = P.mats[P.n_mats++];
                    J.chunk_index = reinterpret_cast<const uint64_t *>(m->d_blob + d.chunk_index_off);
                    J.scales = reinterpret_cast<const float *>(m->d_blob + d.scales_off);
                    J.out = outs[ids[base + t]];
                    J.cols = d.info.cols;
                    J.rows = d.info.rows;
                    J.first_pair = P.total_pairs;
                    J.n_pairs = (uint32_t)((uint64_t)d.info.rows * d.info.cols / ((uint64_t)kTuple * kChunkSyms));
                    P.total_pairs += J.n_pairs;
                }
                if (!pairs_fit(P, sms)) continue;
                for (size_t t = 0; t < cnt; ++t) handled[ids[base + t]] = kTuple * P.mats[t].n_pairs;
                launches.push_back(PairLaunch{co, dt, P});
            }
        }
}

int launch_decode_pairs(const eq_model *m, const uint32_t *mats, uint16_t *const *outs, uint32_t count,
                        int32_t *d_status, cudaStream_t s, int sms, uint32_t *handled) {
    std::vector<PairLaunch> launches;
    plan_pairs(m, mats, outs, count, d_status, (uint32_t)sms, launches, handled);
    if (launches.empty()) return EQ_OK;
    PairSetup *dev = nullptr;
    int rc = pair_setup(&dev);
    if (rc) return rc;
    for (auto &L : launches) {
        const KernelSetup<PairParams> &k = dev->k[L.codec][L.dtype];
        const uint32_t grid = std::min<uint32_t>((uint32_t)sms, L.P.total_pairs);
        k.fn<<<grid, k.warps * 32, k.smem, s>>>(L.P);
        if (cudaGetLastError() != cudaSuccess) return EQ_ERR_CUDA;
    }
    return EQ_OK;
}

int plan_decode_pairs(const eq_model *m, const uint32_t *mats, uint32_t count, uint32_t sms, uint32_t *handled) {
    // outputs as eq_decode_block places them: 256-byte aligned
    std::vector<uint16_t *> outs(count, reinterpret_cast<uint16_t *>(static_cast<uintptr_t>(256)));
    std::vector<PairLaunch> launches;
    plan_pairs(m, mats, outs.data(), count, nullptr, sms, launches, handled);
    return EQ_OK;
}

}  // namespace eqw
