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
// KB2, eq_decode_kernel<WARPS, SHARED> -- one warp per 64 KiB chunk:
//   slot table  4096 entries (f << 20 | (slot - cum) << 8 | sym) in shared
//               memory, so a decoded symbol costs one LDS.  SHARED = true:
//               every chunk of the matrix carries the same frequency table
//               (checked by eq_model_open and again per chunk), so one table
//               per thread block serves all its warps, which work on tiles of
//               consecutive chunks (two per warp; as few warps per tile as
//               keep a small launch on every SM, see assign_tiles);
//               SHARED = false: one table per warp, rebuilt for every chunk.
//   staging     each warp streams its chunk's 16-bit renormalisation words
//               into a private 2 KB shared-memory ring in 512-byte segments
//               with TMA bulk copies (cp.async.bulk, mbarrier completion, no
//               multicast), up to four segments ahead, issued by lane 0.
//   decode      lane l owns interleaved state l; one step of all lanes is
//               slot = x & 4095; x = f * (x >> 12) + (slot - cum);
//               if x < 2^16: x = x << 16 | next word, where the word's position
//               is the warp-wide count of lower lanes that also renormalise
//               (ballot + popcount).
//   dequant     lane l decodes symbols 8l..8l+7 of each 256-symbol group, so
//               every 8 steps it holds 8 consecutive outputs: value * row scale
//               in fp32 (round to nearest even), packed to bf16 (round to
//               nearest even) and stored as one 16-byte vector; a warp's 32
//               stores cover 512 contiguous bytes.  Rank mode (2..32 distinct
//               symbols, cols % 256 == 0): the slot table's low byte is the
//               symbol's rank and lane r holds the fp32 product for rank r of
//               the current row, so a symbol's product is one shuffle.
//   chains      in rank mode with full chunks and cols % 512 == 0 each warp of
//               the shared-table kernel decodes two chunks step by step in
//               lockstep, so two independent state chains hide each other's
//               latency.
// KB3, eq_outlier_scatter_kernel -- out[r * cols + c] = bf16(v) for the super
// weights, after KB2 on the same stream; it also checks that the stream held a
// zero-valued placeholder there (the fused decode + GEMV relies on it).
//
// Every wait on a staged copy is bounded (~1 s of SM clock); on expiry the
// warp records EQ_DEV_TIMEOUT, waits (bounded) for its copies in flight and
// stops decoding.  No tensor cores: nothing here is a dense contraction.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "eqw_device.cuh"
#include "eqw_pairs.h"

#ifndef EQ_USE_PAIRS
#define EQ_USE_PAIRS 1
#endif

namespace {

struct MatJob {
    const uint64_t *chunk_index;  // absolute record offsets, n_chunks + 1 entries
    const float *scales;          // fp32 [rows]
    uint16_t *out;                // bf16 bits, row-major [rows, cols]
    uint64_t n_elems;
    uint32_t cols;
    uint32_t n_chunks;
    uint32_t chunk0;              // first chunk decoded here (the pair kernel took the ones before)
    uint32_t begin;               // first launch-wide work unit (tile or chunk) of this matrix
    uint32_t dtype;
    uint32_t layout;              // kRowUniform: cols % 256 == 0; kLaneRows: cols % 8 == 0; else kGeneric
    uint32_t small_scales;        // all |scale| < 2^8: E4M3 dequant in one multiply
};

struct DecodeParams {
    const uint8_t *blob;
    uint64_t blob_len;
    int32_t *status;
    uint32_t n_mats;
    uint32_t total_units;
    uint32_t tile_warps;          // shared-table kernels: warps that take chunks of a tile (assign_tiles)
    uint32_t tile_chains;         // shared-table kernels: chunks per warp in a tile, 1 or 2 (assign_tiles)
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

// Per-chunk copy of the output-side fields of a matrix, kept in registers.
struct OutCtx {
    uint16_t *out;
    const float *scales;
    uint64_t n_elems;
    uint32_t cols;
    uint32_t rows;
    bool small_scales;
};

__device__ __forceinline__ OutCtx out_ctx(const MatJob &M) {
    return OutCtx{M.out, M.scales, M.n_elems, M.cols, (uint32_t)(M.n_elems / M.cols), M.small_scales != 0};
}

// Element-wise store of `count` outputs starting at linear index idx.
template <int DT>
__device__ __forceinline__ void store_elems(const OutCtx &O, uint64_t idx, uint32_t count, const uint32_t (&e8)[8]) {
#pragma unroll
    for (uint32_t r = 0; r < 8; ++r) {
        if (r < count) {
            const uint64_t i = idx + r;
            O.out[i] = to_bf16(dequant1<DT>(e8[r], __ldg(O.scales + i / O.cols)));
        }
    }
}

// Symbol bytes (layout kSymbolBytes): the low bytes of e8[0..count).
__device__ __forceinline__ void store_symbol_bytes(const OutCtx &O, uint64_t idx, uint32_t count,
                                                   const uint32_t (&e8)[8]) {
    uint8_t *out = reinterpret_cast<uint8_t *>(O.out);
    if (count == 8) {
        const uint32_t lo = (e8[0] & 0xFFu) | (e8[1] & 0xFFu) << 8 | (e8[2] & 0xFFu) << 16 | e8[3] << 24;
        const uint32_t hi = (e8[4] & 0xFFu) | (e8[5] & 0xFFu) << 8 | (e8[6] & 0xFFu) << 16 | e8[7] << 24;
        asm volatile("st.global.v2.b32 [%0], {%1, %2};" ::"l"(out + idx), "r"(lo), "r"(hi) : "memory");
        return;
    }
#pragma unroll
    for (uint32_t r = 0; r < 8; ++r)
        if (r < count) out[idx + r] = (uint8_t)e8[r];
}

// Output bookkeeping for one chunk.  kRowUniform (cols % 256 == 0) keeps the
// warp-uniform row of the current 256-symbol group; kLaneRows keeps each
// lane's own row and column.
struct Cursor {
    uint32_t row, col;
    float scale;
};

template <int DT>
__device__ __forceinline__ float row_scale(const OutCtx &O, uint32_t row) {
    float s = __ldg(O.scales + row);
    if (DT == EQ_E4M3 && O.small_scales) s *= 0x1p120f;  // exact: |s| < 2^8
    return s;
}

template <int DT, uint32_t LAYOUT>
__device__ __forceinline__ void cursor_init(const OutCtx &O, uint64_t first, uint32_t lane, Cursor &c) {
    if constexpr (LAYOUT == kRowUniform || LAYOUT == kLaneRows) {
        const uint64_t e0 = LAYOUT == kRowUniform ? first : first + kGroup * lane;
        c.row = (uint32_t)(e0 / O.cols);
        c.col = (uint32_t)(e0 - (uint64_t)c.row * O.cols);
        c.scale = row_scale<DT>(O, c.row);
    }
}

// Move to the next 256-symbol group (idx: this lane's first output of the
// group just stored).
template <int DT, uint32_t LAYOUT>
__device__ __forceinline__ void cursor_advance(const OutCtx &O, uint64_t idx, Cursor &c) {
    if constexpr (LAYOUT == kRowUniform) {
        c.col += kGroupSyms;
        if (c.col == O.cols) {
            c.col = 0;
            ++c.row;
            if (idx + kGroupSyms < O.n_elems) c.scale = row_scale<DT>(O, c.row);
        }
    } else if constexpr (LAYOUT == kLaneRows) {
        bool moved = false;
        c.col += kGroupSyms;
        while (c.col >= O.cols) {
            c.col -= O.cols;
            ++c.row;
            moved = true;
        }
        if (moved && idx + kGroupSyms < O.n_elems) c.scale = row_scale<DT>(O, c.row);
    }
}

template <int DT, uint32_t LAYOUT>
__device__ __forceinline__ void group_store(const OutCtx &O, uint16_t *dst, uint64_t idx, Cursor &c,
                                            const uint32_t (&e8)[8]) {
    if constexpr (LAYOUT == kGeneric) {
        store_elems<DT>(O, idx, 8, e8);
    } else if constexpr (LAYOUT == kSymbolBytes) {
        store_symbol_bytes(O, idx, 8, e8);
    } else {
        st_global_v4(dst, dequant8<DT>(e8, c.scale, O.small_scales));
        cursor_advance<DT, LAYOUT>(O, idx, c);
    }
}

// One 256-symbol group in a row-uniform layout: 8 steps, dequantised in pairs
// as they are decoded (4 packed registers), one 16-byte store.
template <int DT, uint32_t CODEC>
__device__ __forceinline__ void group_row(uint32_t lut, uint32_t ring, uint32_t &pw, CodecState<CODEC> &x, uint32_t lt,
                                          float2 s2, bool small_scales, uint16_t *dst) {
    const uint32_t rp0 = ring + (pw & (kRingBytes - 1));
    uint32_t rp = rp0;
    uint32_t o[4];
#pragma unroll
    for (int r = 0; r < 8; r += 2) {
        const uint32_t e0 = codec_step<CODEC>(lut, rp, x, lt);
        const uint32_t e1 = codec_step<CODEC>(lut, rp, x, lt);
        float2 v = make_float2(raw_value<DT>(e0), raw_value<DT>(e1));
        if constexpr (DT == EQ_E4M3) {
            if (!small_scales) v = mul2(v, make_float2(0x1p120f, 0x1p120f));
        }
        o[r / 2] = pack_bf16x2(mul2(v, s2));
    }
    st_global_v4(dst, make_uint4(o[0], o[1], o[2], o[3]));
    pw += rp - rp0;
}

// One 256-symbol group in rank mode: 8 steps, 8 shuffles, one 16-byte store.
template <uint32_t CODEC>
__device__ __forceinline__ void group_rank(uint32_t lut, uint32_t ring, uint32_t &pw, CodecState<CODEC> &x, uint32_t lt,
                                           float vr, uint16_t *dst) {
    const uint32_t rp0 = ring + (pw & (kRingBytes - 1));
    uint32_t rp = rp0;
    uint32_t o[4];
#pragma unroll
    for (int r = 0; r < 8; r += 2) {
        const uint32_t e0 = codec_step<CODEC>(lut, rp, x, lt);
        const uint32_t e1 = codec_step<CODEC>(lut, rp, x, lt);
        o[r / 2] = pack_bf16x2(make_float2(__shfl_sync(kFull, vr, e0), __shfl_sync(kFull, vr, e1)));
    }
    st_global_v4(dst, make_uint4(o[0], o[1], o[2], o[3]));
    pw += rp - rp0;
}

// Two chunks per warp in lockstep (rank mode, row-uniform layout, both
// chunks 65536 symbols, cols a multiple of 512): every step of chunk A is
// followed by the same step of chunk B, giving each warp two independent
// state chains whose latencies overlap.  Row changes fall on 512-symbol
// boundaries, i.e. between pairs of groups.
template <uint32_t CODEC>
struct Chain {
    CodecState<CODEC> x;
    uint32_t pw, limit, row, col;
    float vr;
    uint16_t *dst;
};

// One 256-symbol group of each of the C chains in rank mode, interleaved
// step by step (chain 0, 1, ..., C-1 for every step).
template <uint32_t CODEC, uint32_t C>
__device__ __forceinline__ void groupN_rank(uint32_t lut, const uint32_t (&ring)[C], Chain<CODEC> (&ch)[C],
                                            uint32_t lt) {
    uint32_t r0[C], rp[C], o[C][4];
#pragma unroll
    for (uint32_t c = 0; c < C; ++c) rp[c] = r0[c] = ring[c] + (ch[c].pw & (kRingBytes - 1));
#pragma unroll
    for (int r = 0; r < 8; r += 2) {
        uint32_t e0[C], e1[C];
#pragma unroll
        for (uint32_t c = 0; c < C; ++c) e0[c] = codec_step<CODEC>(lut, rp[c], ch[c].x, lt);
#pragma unroll
        for (uint32_t c = 0; c < C; ++c) e1[c] = codec_step<CODEC>(lut, rp[c], ch[c].x, lt);
#pragma unroll
        for (uint32_t c = 0; c < C; ++c)
            o[c][r / 2] = pack_bf16x2(make_float2(__shfl_sync(kFull, ch[c].vr, e0[c]),
                                                  __shfl_sync(kFull, ch[c].vr, e1[c])));
    }
#pragma unroll
    for (uint32_t c = 0; c < C; ++c) {
        st_global_v4(ch[c].dst, make_uint4(o[c][0], o[c][1], o[c][2], o[c][3]));
        ch[c].pw += rp[c] - r0[c];
        ch[c].dst += kGroupSyms;
    }
}

// C full chunks per warp in lockstep (rank mode, row-uniform layout, every
// chunk 65536 symbols, cols a multiple of 512): C independent state chains
// whose latencies overlap.  Row changes fall between pairs of groups.
template <int DT, uint32_t CODEC, uint32_t C>
__device__ __forceinline__ bool decode_multi(int32_t *status, const OutCtx &O, const ChunkHead (&h)[C],
                                             const uint64_t (&first)[C], uint32_t lut, const uint32_t (&ring)[C],
                                             const uint32_t (&mbar)[C], RingCtl *ctl, uint32_t lane, uint32_t lt,
                                             uint32_t lane_sym) {
#pragma unroll
    for (uint32_t c = 0; c < C; ++c) ring_start(ctl + c, h[c]);
    __syncwarp();
    const float vraw = symbol_value<DT>(lane_sym);
    Chain<CODEC> ch[C];
#pragma unroll
    for (uint32_t c = 0; c < C; ++c) {
        ch[c].x = codec_start<CODEC>(h[c].x);
        ch[c].pw = 0;
        ch[c].limit = h[c].n_words ? 0u : kNoLimit;
        ch[c].row = (uint32_t)(first[c] / O.cols);
        ch[c].col = (uint32_t)(first[c] - (uint64_t)ch[c].row * O.cols);
        ch[c].vr = __fmul_rn(vraw, __ldg(O.scales + ch[c].row));
        ch[c].dst = O.out + first[c] + kGroup * lane;
    }
    constexpr uint32_t kPairs = kChunkSyms / (2 * kGroupSyms);
    for (uint32_t q = 0; q < kPairs; ++q) {
        bool dead = false;
#pragma unroll
        for (uint32_t c = 0; c < C; ++c) {
            if (ch[c].pw >= ch[c].limit) ch[c].limit = ring_service(ctl + c, ring[c], mbar[c], ch[c].pw);
            dead = dead || ctl[c].dead;
        }
        if (dead) break;
        groupN_rank<CODEC, C>(lut, ring, ch, lt);
        groupN_rank<CODEC, C>(lut, ring, ch, lt);
#pragma unroll
        for (uint32_t c = 0; c < C; ++c) {
            check_progress(status, ctl + c, ch[c].pw, ch[c].dst, O.out, O.n_elems, lane);
            ch[c].col += 2 * kGroupSyms;
            if (ch[c].col == O.cols) {
                ch[c].col = 0;
                ++ch[c].row;
                if (ch[c].row < O.rows) ch[c].vr = __fmul_rn(vraw, __ldg(O.scales + ch[c].row));
            }
        }
    }
    bool drained = true;
#pragma unroll
    for (uint32_t c = 0; c < C; ++c) drained = ring_drain(ctl + c, mbar[c]) && drained;
    if (!drained) {
        flag(status, EQ_DEV_TIMEOUT);
        return false;
    }
#pragma unroll
    for (uint32_t c = 0; c < C; ++c)
        if (!__all_sync(kFull, codec_done(ch[c].x)) || ch[c].pw != 2u * h[c].n_words) flag(status, EQ_DEV_BAD_END);
    return true;
}

// Symbol bytes (layout kSymbolBytes) of C full chunks per warp in lockstep:
// the same interleaved steps as decode_multi, each lane's 8 low bytes of a
// group packed with byte permutes into one 8-byte store.  Any table (the
// bytes are the stored symbols), any shape (the output is the flat symbol
// array).
__device__ __forceinline__ uint32_t bytes4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    uint32_t ab, cd, r;
    asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(ab) : "r"(a), "r"(b));  // a.b0, b.b0
    asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(cd) : "r"(c), "r"(d));
    asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(r) : "r"(ab), "r"(cd));  // ab.b0 ab.b1 cd.b0 cd.b1
    return r;
}

template <uint32_t CODEC, uint32_t C>
__device__ __forceinline__ void groupN_bytes(uint32_t lut, const uint32_t (&ring)[C], Chain<CODEC> (&ch)[C],
                                             uint32_t lt) {
    uint32_t r0[C], rp[C], o[C][2];
#pragma unroll
    for (uint32_t c = 0; c < C; ++c) rp[c] = r0[c] = ring[c] + (ch[c].pw & (kRingBytes - 1));
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t e[C][4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (uint32_t c = 0; c < C; ++c) e[c][r] = codec_step<CODEC>(lut, rp[c], ch[c].x, lt);
#pragma unroll
        for (uint32_t c = 0; c < C; ++c) o[c][h] = bytes4(e[c][0], e[c][1], e[c][2], e[c][3]);
    }
#pragma unroll
    for (uint32_t c = 0; c < C; ++c) {
        asm volatile("st.global.v2.b32 [%0], {%1, %2};" ::"l"(ch[c].dst), "r"(o[c][0]), "r"(o[c][1]) : "memory");
        ch[c].pw += rp[c] - r0[c];
        ch[c].dst += kGroupSyms / 2;  // 256 bytes, in bf16 units of the output pointer
    }
}

template <uint32_t CODEC, uint32_t C>
__device__ __forceinline__ bool decode_multi_bytes(int32_t *status, const OutCtx &O, const ChunkHead (&h)[C],
                                                   const uint64_t (&first)[C], uint32_t lut,
                                                   const uint32_t (&ring)[C], const uint32_t (&mbar)[C],
                                                   RingCtl *ctl, uint32_t lane, uint32_t lt) {
#pragma unroll
    for (uint32_t c = 0; c < C; ++c) ring_start(ctl + c, h[c]);
    __syncwarp();
    Chain<CODEC> ch[C];
#pragma unroll
    for (uint32_t c = 0; c < C; ++c) {
        ch[c].x = codec_start<CODEC>(h[c].x);
        ch[c].pw = 0;
        ch[c].limit = h[c].n_words ? 0u : kNoLimit;
        // byte address first + 8 lane, carried in a bf16 pointer (always even)
        ch[c].dst = reinterpret_cast<uint16_t *>(reinterpret_cast<uint8_t *>(O.out) + first[c] + kGroup * lane);
    }
    constexpr uint32_t kPairs = kChunkSyms / (2 * kGroupSyms);
    for (uint32_t q = 0; q < kPairs; ++q) {
        bool dead = false;
#pragma unroll
        for (uint32_t c = 0; c < C; ++c) {
            if (ch[c].pw >= ch[c].limit) ch[c].limit = ring_service(ctl + c, ring[c], mbar[c], ch[c].pw);
            dead = dead || ctl[c].dead;
        }
        if (dead) break;
        groupN_bytes<CODEC, C>(lut, ring, ch, lt);
        groupN_bytes<CODEC, C>(lut, ring, ch, lt);
    }
    bool drained = true;
#pragma unroll
    for (uint32_t c = 0; c < C; ++c) drained = ring_drain(ctl + c, mbar[c]) && drained;
    if (!drained) {
        flag(status, EQ_DEV_TIMEOUT);
        return false;
    }
#pragma unroll
    for (uint32_t c = 0; c < C; ++c)
        if (!__all_sync(kFull, codec_done(ch[c].x)) || ch[c].pw != 2u * h[c].n_words) flag(status, EQ_DEV_BAD_END);
    return true;
}

// Decode one chunk whose slot table is ready at `lut` (n_present >= 2) or
// whose single symbol's stored byte is `single` (n_present == 1).  Returns
// false if a bounded wait gave up (the warp must stop).
template <int DT, uint32_t LAYOUT, uint32_t CODEC>
__device__ __forceinline__ bool decode_body(int32_t *status, const OutCtx &O, uint64_t first,
                                            uint32_t n, uint32_t n_words, const uint8_t *payload, bool single_sym,
                                            uint32_t single, uint32_t x0, uint32_t lut, uint32_t ring, uint32_t mbar,
                                            RingCtl *ctl, uint32_t lane, uint32_t lt, bool by_rank,
                                            uint32_t lane_sym) {
    const uint32_t n_full = n / kGroupSyms;
    const uint32_t tail = n % kGroupSyms;
    Cursor cur{0, 0, 0.f};
    cursor_init<DT, LAYOUT>(O, first, lane, cur);
    uint16_t *dst = O.out + first + kGroup * lane;

    if (single_sym) {
        // f = 4096: the states never change and there are no words
        if (n_words != 0 || !__all_sync(kFull, CODEC == kCodecHuffman || x0 == kStateLow)) {
            flag(status, EQ_DEV_BAD_END);
            return true;
        }
        uint32_t e8[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) e8[r] = single;
        for (uint32_t g = 0; g < n_full; ++g, dst += kGroupSyms)
            group_store<DT, LAYOUT>(O, dst, first + (uint64_t)g * kGroupSyms + kGroup * lane, cur, e8);
        if (tail) {
            const uint32_t mine = tail > kGroup * lane ? min(8u, tail - kGroup * lane) : 0u;
            if constexpr (LAYOUT == kSymbolBytes)
                store_symbol_bytes(O, first + (uint64_t)n_full * kGroupSyms + kGroup * lane, mine, e8);
            else
                store_elems<DT>(O, first + (uint64_t)n_full * kGroupSyms + kGroup * lane, mine, e8);
        }
        return true;
    }

    const uint32_t pbytes = (2u * n_words + 15u) & ~15u;
    if (lane == 0) {
        ctl->payload = payload;
        ctl->pbytes = pbytes;
        ctl->n_segs = (pbytes + kSegBytes - 1) / kSegBytes;
        ctl->issued = 0;
        ctl->ready = 0;
    }
    __syncwarp();
    uint32_t limit = pbytes ? 0u : kNoLimit;
    uint32_t pw = 0;
    CodecState<CODEC> x = codec_start<CODEC>(x0);
    bool tail_done = false;
    if constexpr (LAYOUT == kRowUniform) {
      if (by_rank) {
        // runs of groups within one row, two groups per ring check; lane r holds
        // the dequantised value of rank r for the current row
        const float vraw = symbol_value<DT>(lane_sym);
        uint32_t g = 0;
        while (g < n_full && !ctl->dead) {
            const uint32_t run = min((O.cols - cur.col) / kGroupSyms, n_full - g);
            const float vr = __fmul_rn(vraw, __ldg(O.scales + cur.row));
            uint32_t i = 0;
            while (i < run) {
                if (pw >= limit) {
                    limit = ring_service(ctl, ring, mbar, pw);
                    if (ctl->dead) break;
                }
                if (i + 1 < run) {
                    // hot loop: no calls, pairs of groups while the ring guarantees residency
                    do {
                        group_rank(lut, ring, pw, x, lt, vr, dst);
                        group_rank(lut, ring, pw, x, lt, vr, dst + kGroupSyms);
                        i += 2;
                        dst += 2 * kGroupSyms;
                        check_progress(status, ctl, pw, dst, O.out, O.n_elems, lane);
                    } while (i + 1 < run && pw < limit);
                } else {
                    group_rank(lut, ring, pw, x, lt, vr, dst);
                    i += 1;
                    dst += kGroupSyms;
                    check_progress(status, ctl, pw, dst, O.out, O.n_elems, lane);
                }
            }
            g += run;
            cur.col += run * kGroupSyms;
            if (cur.col == O.cols) {
                cur.col = 0;
                ++cur.row;
            }
        }
        if (tail && !ctl->dead) {
            if (pw >= limit) limit = ring_service(ctl, ring, mbar, pw);
            if (!ctl->dead) {
                uint32_t e8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                codec_tail<CODEC>(lut, ring, x, pw, lt, lane, tail, e8);
                const float vr = __fmul_rn(vraw, __ldg(O.scales + cur.row));
                const uint32_t mine = tail > kGroup * lane ? min(8u, tail - kGroup * lane) : 0u;
                const uint64_t idx = first + (uint64_t)n_full * kGroupSyms + kGroup * lane;
#pragma unroll
                for (uint32_t r = 0; r < 8; ++r) {
                    const float v = __shfl_sync(kFull, vr, e8[r]);
                    if (r < mine) O.out[idx + r] = to_bf16(v);
                }
            }
        }
        tail_done = true;
      } else {
        // runs of groups within one row (scale fixed), two groups per ring check
        uint32_t g = 0;
        while (g < n_full && !ctl->dead) {
            const uint32_t run = min((O.cols - cur.col) / kGroupSyms, n_full - g);
            const float2 s2 = make_float2(cur.scale, cur.scale);
            uint32_t i = 0;
            for (; i + 1 < run; i += 2, dst += 2 * kGroupSyms) {
                if (pw >= limit) {
                    limit = ring_service(ctl, ring, mbar, pw);
                    if (ctl->dead) break;
                }
                group_row<DT, CODEC>(lut, ring, pw, x, lt, s2, O.small_scales, dst);
                group_row<DT, CODEC>(lut, ring, pw, x, lt, s2, O.small_scales, dst + kGroupSyms);
                check_progress(status, ctl, pw, dst + 2 * kGroupSyms, O.out, O.n_elems, lane);
            }
            if (i < run && !ctl->dead) {
                if (pw >= limit) limit = ring_service(ctl, ring, mbar, pw);
                if (!ctl->dead) {
                    group_row<DT, CODEC>(lut, ring, pw, x, lt, s2, O.small_scales, dst);
                    dst += kGroupSyms;
                }
            }
            g += run;
            cur.col += run * kGroupSyms;
            if (cur.col == O.cols) {
                cur.col = 0;
                ++cur.row;
                if (g < n_full) cur.scale = row_scale<DT>(O, cur.row);
            }
        }
      }
    } else {
    for (uint32_t g = 0; g < n_full; ++g, dst += kGroupSyms) {
        if (pw >= limit) {
            limit = ring_service(ctl, ring, mbar, pw);
            if (ctl->dead) break;
        }
        const uint32_t rp0 = ring + (pw & (kRingBytes - 1));
        uint32_t rp = rp0;
        if constexpr (LAYOUT == kGeneric || LAYOUT == kSymbolBytes) {
            uint32_t e8[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) e8[r] = codec_step<CODEC>(lut, rp, x, lt);
            if constexpr (LAYOUT == kSymbolBytes)
                store_symbol_bytes(O, first + (uint64_t)g * kGroupSyms + kGroup * lane, 8, e8);
            else
                store_elems<DT>(O, first + (uint64_t)g * kGroupSyms + kGroup * lane, 8, e8);
        } else {
            // dequantise pairs as they are decoded: 4 packed registers instead of 8 entries
            const float2 s2 = make_float2(cur.scale, cur.scale);
            uint32_t o[4];
#pragma unroll
            for (int r = 0; r < 8; r += 2) {
                const uint32_t e0 = codec_step<CODEC>(lut, rp, x, lt);
                const uint32_t e1 = codec_step<CODEC>(lut, rp, x, lt);
                float2 v = make_float2(raw_value<DT>(e0), raw_value<DT>(e1));
                if constexpr (DT == EQ_E4M3) {
                    if (!O.small_scales) v = mul2(v, make_float2(0x1p120f, 0x1p120f));
                }
                o[r / 2] = pack_bf16x2(mul2(v, s2));
            }
            st_global_v4(dst, make_uint4(o[0], o[1], o[2], o[3]));
            cursor_advance<DT, LAYOUT>(O, first + (uint64_t)g * kGroupSyms + kGroup * lane, cur);
        }
        pw += rp - rp0;
        check_progress(status, ctl, pw, dst + kGroupSyms, O.out, O.n_elems, lane);
    }
    }
    if (tail && !tail_done && !ctl->dead) {
        if (pw >= limit) limit = ring_service(ctl, ring, mbar, pw);
        if (!ctl->dead) {
            uint32_t e8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            codec_tail<CODEC>(lut, ring, x, pw, lt, lane, tail, e8);
            const uint32_t mine = tail > kGroup * lane ? min(8u, tail - kGroup * lane) : 0u;
            if constexpr (LAYOUT == kSymbolBytes)
                store_symbol_bytes(O, first + (uint64_t)n_full * kGroupSyms + kGroup * lane, mine, e8);
            else
                store_elems<DT>(O, first + (uint64_t)n_full * kGroupSyms + kGroup * lane, mine, e8);
        }
    }
    if (!ring_drain(ctl, mbar)) {
        flag(status, EQ_DEV_TIMEOUT);
        return false;
    }
    // a valid stream returns every state to 2^16 and consumes exactly n_words
    if (!__all_sync(kFull, codec_done(x)) || pw != 2u * n_words) flag(status, EQ_DEV_BAD_END);
    return true;
}

template <int WARPS, bool SHARED, int DT, uint32_t LAYOUT, uint32_t CODEC>
__global__ void __launch_bounds__(WARPS * 32, SHARED ? kSharedMinCtas : 1)
    eq_decode_kernel(const __grid_constant__ DecodeParams P) {
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
            const MatJob &M = P.mats[mi];
            const uint32_t TW = P.tile_warps, TC = P.tile_chains;
            const uint32_t k0 = M.chunk0 + (unit - M.begin) * TW * TC;
            if (mi != cur_mat) {
                shared_table_rebuild<WARPS, LAYOUT, CODEC>(P, M, k0, lane, warp, S);
                cur_mat = mi;
            }
            const uint32_t np = S.blk[0];
            const uint32_t lane_sym = S.ref_entries[lane < np ? lane : 0] & 0xFFu;
            // this warp's chunks: k0 + warp (+ TW for the second chain); warps >= TW sit the tile out
            ChunkHead hc[C];
            bool have[C];
            for (uint32_t c = 0; c < C; ++c) {
                const uint32_t k = k0 + warp + c * TW;
                have[c] = c < TC && warp < TW && k < M.n_chunks && !ctl[0].dead && !ctl[C - 1].dead;
                if (have[c]) have[c] = shared_chunk_head<CODEC>(P, M, k, lane, np, S, hc[c]);
            }
            const OutCtx O = out_ctx(M);
            if constexpr (C >= 2 && (LAYOUT == kRowUniform || LAYOUT == kSymbolBytes)) {
                bool all_full = LAYOUT == kSymbolBytes ? np >= 2
                                                       : rank_mode<LAYOUT>(np) && O.cols % (2 * kGroupSyms) == 0;
                for (uint32_t c = 0; c < C; ++c) all_full = all_full && have[c] && hc[c].n == kChunkSyms;
                if (all_full) {
                    uint64_t first[C];
                    uint32_t rings[C], mbars[C];
#pragma unroll
                    for (uint32_t c = 0; c < C; ++c) {
                        first[c] = (uint64_t)(k0 + warp + c * TW) * kChunkSyms;
                        rings[c] = S.ring + c * kRingStride;
                        mbars[c] = S.mbar + 8 * kRingSegs * c;
                    }
                    if constexpr (LAYOUT == kSymbolBytes)
                        decode_multi_bytes<CODEC, C>(P.status, O, hc, first, S.lut_addr, rings, mbars, ctl, lane, lt);
                    else
                        decode_multi<DT, CODEC, C>(P.status, O, hc, first, S.lut_addr, rings, mbars, ctl, lane, lt,
                                                   lane_sym);
                    __syncwarp();
                    continue;
                }
            }
            for (uint32_t c = 0; c < C; ++c) {
                if (!have[c] || ctl->dead) continue;
                decode_body<DT, LAYOUT, CODEC>(P.status, O, (uint64_t)(k0 + warp + c * TW) * kChunkSyms, hc[c].n,
                                        hc[c].n_words, hc[c].rec + hc[c].table_bytes, np == 1,
                                        S.ref_entries[0] & 0xFFu, hc[c].x, S.lut_addr, S.ring, S.mbar, ctl, lane,
                                        lt, rank_mode<LAYOUT>(np), lane_sym);
                __syncwarp();
            }
        }
    } else {
        const uint32_t stride = gridDim.x * WARPS;
        for (uint32_t c = blockIdx.x * WARPS + warp; c < P.total_units && !ctl->dead; c += stride) {
            const MatJob &M = P.mats[job_of(P, c)];
            const uint32_t k = M.chunk0 + (c - M.begin);
            ChunkHead h;
            if (!load_head<CODEC>(P, M, k, lane, h)) continue;
            const uint32_t *tab = reinterpret_cast<const uint32_t *>(h.rec + kHeadBytes<CODEC>);
            __syncwarp();  // the previous chunk's reads of the slot table are done
            const bool by_rank = rank_mode<LAYOUT>(h.n_present);
            const bool ok = warp_table<CODEC>(tab, h.n_present, lane, nullptr, nullptr, S.lut, by_rank);
            if (!ok) {
                flag(P.status, EQ_DEV_BAD_TABLE);
                continue;
            }
            __syncwarp();
            if (h.n_present > 1) check_table<CODEC>(P.status, S.lut, lane, 32);
            decode_body<DT, LAYOUT, CODEC>(P.status, out_ctx(M), (uint64_t)k * kChunkSyms, h.n, h.n_words,
                                    h.rec + h.table_bytes, h.n_present == 1, tab[0] & 0xFFu, h.x,
                                    S.lut_addr, S.ring, S.mbar, ctl, lane, lt, by_rank,
                                    tab[lane < h.n_present ? lane : 0] & 0xFFu);
            __syncwarp();
        }
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
    uint16_t *o = J.out + (uint64_t)row * J.cols + col;
    // the stream carries a zero-valued placeholder symbol under every super weight
    if (*o & 0x7FFFu) atomicOr(P.status, EQ_DEV_BAD_OUTLIER);
    *o = to_bf16(v);
}

// Timeout path check: a ring whose only segment counts as issued but was never
// copied, so ring_drain's bounded wait on its mbarrier must give up.
__global__ void eq_wait_timeout_kernel(int32_t *status) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ RingCtl ctl;
    const uint32_t mbar = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(mbar, 1);
        fence_mbar_init();
        ctl.payload = nullptr;
        ctl.pbytes = kSegBytes;
        ctl.n_segs = 1;
        ctl.issued = 1;
        ctl.ready = 0;
        ctl.phase = 0;
        ctl.dead = 0;
    }
    __syncwarp();
    if (!ring_drain(&ctl, mbar)) flag(status, EQ_DEV_TIMEOUT);
}

// ---- host side ---------------------------------------------------------------------

// variants: [codec][shared][dtype - 1][layout]
struct DeviceSetup {
    bool ready = false;
    int sms = 0;
    KernelSetup<DecodeParams> k[2][2][2][4];
};
std::mutex g_setup_mu;
DeviceSetup g_setup[128];

template <int DT, uint32_t LAYOUT, uint32_t CODEC>
int setup_variant(DeviceSetup &d) {
    int rc = setup_kernel(d.k[CODEC][1][DT - 1][LAYOUT], eq_decode_kernel<kSharedWarps, true, DT, LAYOUT, CODEC>,
                          kSharedWarps, Smem<kSharedWarps, true>::kBytes, 1);
    if (rc) return rc;
    return setup_kernel(d.k[CODEC][0][DT - 1][LAYOUT], eq_decode_kernel<kPrivateWarps, false, DT, LAYOUT, CODEC>,
                        kPrivateWarps, Smem<kPrivateWarps, false>::kBytes, kPrivateWarps);
}

template <int DT, uint32_t LAYOUT>
int setup_pair(DeviceSetup &d) {
    int rc = setup_variant<DT, LAYOUT, kCodecRans>(d);
    return rc ? rc : setup_variant<DT, LAYOUT, kCodecHuffman>(d);
}

int device_setup(DeviceSetup **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return EQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    DeviceSetup &d = g_setup[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return EQ_ERR_CUDA;
        int rc;
        if ((rc = setup_pair<EQ_INT8, kRowUniform>(d)) || (rc = setup_pair<EQ_INT8, kLaneRows>(d)) ||
            (rc = setup_pair<EQ_INT8, kGeneric>(d)) || (rc = setup_pair<EQ_INT8, kSymbolBytes>(d)) ||
            (rc = setup_pair<EQ_E4M3, kRowUniform>(d)) || (rc = setup_pair<EQ_E4M3, kLaneRows>(d)) ||
            (rc = setup_pair<EQ_E4M3, kGeneric>(d)) || (rc = setup_pair<EQ_E4M3, kSymbolBytes>(d)))
            return rc;
        d.ready = true;
    }
    *out = &d;
    return EQ_OK;
}

uint32_t layout_of(const eq_matrix_info &in, const uint16_t *out) {
    const bool aligned = reinterpret_cast<uintptr_t>(out) % 16 == 0;
    if (aligned && in.cols % kGroupSyms == 0) return kRowUniform;
    if (aligned && in.cols % kGroup == 0) return kLaneRows;
    return kGeneric;
}

// Decode matrices [first, first + count) of the model into outs[i]: one
// launch per kernel variant (codec x table scope x dtype x layout) present, then one
// scatter launch for the super weights.
int launch_decode(const eq_model *m, uint32_t first, uint32_t count, uint16_t *const *outs, int32_t *d_status,
                  cudaStream_t s, bool symbols = false) {
    DeviceSetup *dev = nullptr;
    int rc = device_setup(&dev);
    if (rc) return rc;
    const int sms = m->sm_limit && m->sm_limit < (uint32_t)dev->sms ? (int)m->sm_limit : dev->sms;
    for (uint32_t base = 0; base < count; base += kMaxMatsPerLaunch) {
        const uint32_t cnt = std::min<uint32_t>(kMaxMatsPerLaunch, count - base);
        DecodeParams P[2][2][2][4];
        for (auto &a : P)
            for (auto &b : a)
                for (auto &c : b)
                    for (auto &v : c) {
                        v = DecodeParams{};
                        v.blob = m->d_blob;
                        v.blob_len = m->len;
                        v.status = d_status;
                    }
        ScatterParams Q{};
        Q.status = d_status;
        uint32_t n_out = 0;
        // leading pairs of full chunks of the common-case matrices: the pair kernel
        uint32_t handled[kMaxMatsPerLaunch] = {};
#if EQ_USE_PAIRS
        if (!symbols) {
            uint32_t ids[kMaxMatsPerLaunch];
            for (uint32_t i = 0; i < cnt; ++i) ids[i] = first + base + i;
            if ((rc = launch_decode_pairs(m, ids, outs + base, cnt, d_status, s, sms, handled))) return rc;
        }
#endif
        for (uint32_t i = 0; i < cnt; ++i) {
            const MatrixDesc &d = m->mats[first + base + i];
            if (d.info.n_chunks == 0) continue;
            const int sh = d.info.uniform_table ? 1 : 0;
            const uint32_t lay = symbols ? kSymbolBytes : layout_of(d.info, outs[base + i]);
            if (handled[i] < d.info.n_chunks) {
                DecodeParams &Pv = P[d.codec][sh][d.info.dtype - 1][lay];
                MatJob &J = Pv.mats[Pv.n_mats++];
                J.chunk_index = reinterpret_cast<const uint64_t *>(m->d_blob + d.chunk_index_off);
                J.scales = reinterpret_cast<const float *>(m->d_blob + d.scales_off);
                J.out = outs[base + i];
                J.n_elems = (uint64_t)d.info.rows * d.info.cols;
                J.cols = d.info.cols;
                J.n_chunks = d.info.n_chunks;
                J.chunk0 = handled[i];
                J.begin = Pv.total_units;
                J.dtype = d.info.dtype;
                J.layout = lay;
                J.small_scales = d.small_scales ? 1u : 0u;
                // per-chunk units; shared-table launches are re-tiled below
                Pv.total_units += d.info.n_chunks - handled[i];
            }
            if (d.info.n_outliers && !symbols) {
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
        Q.total = n_out;
        for (int co = 0; co < 2; ++co)
            for (int dt = 0; dt < 2; ++dt)
                for (int lay = 0; lay < 4; ++lay) {
                    const auto &k = dev->k[co][1][dt][lay];
                    assign_tiles(P[co][1][dt][lay], (uint32_t)(sms * k.ctas_per_sm), kSharedWarps, EQ_CHAINS);
                }
        for (int co = 0; co < 2; ++co)
            for (int sh = 0; sh < 2; ++sh)
                for (int dt = 0; dt < 2; ++dt)
                    for (int lay = 0; lay < 4; ++lay)
                        if ((rc = launch(dev->k[co][sh][dt][lay], sms, P[co][sh][dt][lay], s))) return rc;
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
    const eqw::NvtxScope nvtx_range("eq_decode_matrix");
    if (!m || !d_status || matrix >= m->mats.size()) return EQ_ERR_INVALID_ARG;
    const eq_matrix_info &in = m->mats[matrix].info;
    const uint64_t need = 2ull * in.rows * in.cols;
    if (need && (!d_out || reinterpret_cast<uintptr_t>(d_out) % 2)) return EQ_ERR_INVALID_ARG;
    if (out_bytes < need) return EQ_ERR_NOSPACE;
    uint16_t *out = static_cast<uint16_t *>(d_out);
    return launch_decode(m, matrix, 1, &out, d_status, s);
}

extern "C" EQW_API int eq_decode_symbols(const eq_model *m, uint32_t matrix, void *d_out, size_t out_bytes,
                                         int32_t *d_status, cudaStream_t s) {
    const eqw::NvtxScope nvtx_range("eq_decode_symbols");
    if (!m || !d_status || matrix >= m->mats.size()) return EQ_ERR_INVALID_ARG;
    const eq_matrix_info &in = m->mats[matrix].info;
    const uint64_t need = (uint64_t)in.rows * in.cols;
    if (need && (!d_out || reinterpret_cast<uintptr_t>(d_out) % 16)) return EQ_ERR_INVALID_ARG;
    if (out_bytes < need) return EQ_ERR_NOSPACE;
    uint16_t *out = static_cast<uint16_t *>(d_out);
    return launch_decode(m, matrix, 1, &out, d_status, s, true);
}

extern "C" EQW_API int eq_decode_symbols_block(const eq_model *m, uint32_t layer, void *const *d_outs,
                                               uint32_t count, int32_t *d_status, cudaStream_t s) {
    const eqw::NvtxScope nvtx_range("eq_decode_symbols_block");
    if (!m || !d_status || !d_outs || layer >= m->n_layers || count != m->layer_count[layer])
        return EQ_ERR_INVALID_ARG;
    const uint32_t first = m->layer_first[layer];
    std::vector<uint16_t *> outs(count);
    for (uint32_t i = 0; i < count; ++i) {
        const eq_matrix_info &in = m->mats[first + i].info;
        if ((uint64_t)in.rows * in.cols && (!d_outs[i] || reinterpret_cast<uintptr_t>(d_outs[i]) % 16))
            return EQ_ERR_INVALID_ARG;
        outs[i] = static_cast<uint16_t *>(d_outs[i]);
    }
    return launch_decode(m, first, count, outs.data(), d_status, s, true);
}

extern "C" EQW_API int eq_decode_block(const eq_model *m, uint32_t layer, void *d_out, size_t out_bytes,
                                       int32_t *d_status, cudaStream_t s) {
    const eqw::NvtxScope nvtx_range("eq_decode_block");
    if (!m || !d_status || layer >= m->n_layers) return EQ_ERR_INVALID_ARG;
    const uint32_t first = m->layer_first[layer], count = m->layer_count[layer];
    std::vector<size_t> offs(count);
    size_t total = 0;
    int rc = eq_block_layout(m, layer, offs.data(), count, &total);
    if (rc) return rc;
    if (total && (!d_out || reinterpret_cast<uintptr_t>(d_out) % 16)) return EQ_ERR_INVALID_ARG;
    if (out_bytes < total) return EQ_ERR_NOSPACE;
    std::vector<uint16_t *> outs(count);
    for (uint32_t i = 0; i < count; ++i)
        outs[i] = reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(d_out) + offs[i]);
    return launch_decode(m, first, count, outs.data(), d_status, s);
}

extern "C" EQW_API int eq_decode_model_stream(const eq_model *m, uint32_t layer, void *const d_buf[2],
                                              size_t buf_bytes, int32_t *d_status, cudaStream_t decode_stream,
                                              cudaEvent_t const ev_free[2], cudaEvent_t const ev_ready[2]) {
    const eqw::NvtxScope nvtx_range("eq_decode_model_stream");
    if (!m || !d_buf || !ev_free || !ev_ready || layer >= m->n_layers) return EQ_ERR_INVALID_ARG;
    const uint32_t b = layer & 1u;
    if (!ev_ready[b]) return EQ_ERR_INVALID_ARG;
    if (ev_free[b] && cudaStreamWaitEvent(decode_stream, ev_free[b], 0) != cudaSuccess) return EQ_ERR_CUDA;
    int rc = eq_decode_block(m, layer, d_buf[b], buf_bytes, d_status, decode_stream);
    if (rc) return rc;
    if (cudaEventRecord(ev_ready[b], decode_stream) != cudaSuccess) return EQ_ERR_CUDA;
    return EQ_OK;
}

extern "C" EQW_API int eq_decode_plan(const eq_model *m, uint32_t layer, uint32_t sms, uint32_t *pair_chunks,
                                      uint32_t cap) {
    if (!m || !pair_chunks || !sms || layer >= m->n_layers || cap < m->layer_count[layer]) return EQ_ERR_INVALID_ARG;
    const uint32_t first = m->layer_first[layer], count = m->layer_count[layer];
    const uint32_t eff = m->sm_limit && m->sm_limit < sms ? m->sm_limit : sms;
    for (uint32_t i = 0; i < count; ++i) pair_chunks[i] = 0;
#if EQ_USE_PAIRS
    for (uint32_t base = 0; base < count; base += kMaxMatsPerLaunch) {
        const uint32_t cnt = std::min<uint32_t>(kMaxMatsPerLaunch, count - base);
        uint32_t ids[kMaxMatsPerLaunch];
        for (uint32_t i = 0; i < cnt; ++i) ids[i] = first + base + i;
        plan_decode_pairs(m, ids, cnt, eff, pair_chunks + base);
    }
#endif
    return EQ_OK;
}

extern "C" EQW_API int eq_selftest_wait_timeout(int32_t *d_status, cudaStream_t s) {
    if (!d_status) return EQ_ERR_INVALID_ARG;
    eq_wait_timeout_kernel<<<1, 32, 0, s>>>(d_status);
    return cudaGetLastError() == cudaSuccess ? EQ_OK : EQ_ERR_CUDA;
}

extern "C" EQW_API int eq_build_checked(void) { return EQ_CHECKED; }
