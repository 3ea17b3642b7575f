// Device building blocks shared by the decode kernels (eqw_decode.cu) and the
// fused decode + GEMV kernels (eqw_decode_gemv.cu): word staging ring (TMA
// bulk copies with mbarrier completion, bounded waits), the interleaved rANS
// step, number formats, chunk-record header checks and slot-table expansion.
//
// Container v1 chunk record: n_syms, n_words, n_present, 0 (u32 each), the 32
// lane states, n_present frequency-list entries (symbol | f << 16, ascending
// symbols), padding to 16 bytes, the 16-bit renormalisation words, padding.
// rANS per Duda, "Asymmetric numeral systems" (2013), with 32 interleaved
// states per Giesen, "Interleaved entropy coders" (2014): 12-bit
// frequencies, states in [2^16, 2^32), 16-bit renormalisation.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "eqw_internal.h"

namespace {

using namespace eqw;

constexpr uint32_t kFull = 0xFFFFFFFFu;
#ifndef EQ_RING_BYTES
#define EQ_RING_BYTES 2048
#endif
#ifndef EQ_CHAINS
#define EQ_CHAINS 2
#endif
constexpr uint32_t kRingBytes = EQ_RING_BYTES;  // per chain: 512-byte segments ...
constexpr uint32_t kSegBytes = 512;    // one TMA segment = 256 words
constexpr uint32_t kRingSegs = kRingBytes / kSegBytes;
// ... followed by a 512-byte mirror of segment slot 0, so the up to 512 bytes
// one 256-symbol group reads from any starting offset are contiguous and the
// per-step word address needs no wrap-around mask.
constexpr uint32_t kRingStride = kRingBytes + kSegBytes;
// Words the ring guarantees resident at each service check: two groups.
constexpr uint32_t kSpan = 2 * kSegBytes;
constexpr uint32_t kLutBytes = 4 * kProbTotal;
constexpr long long kWaitCycles = 2000000000LL;
constexpr uint32_t kNoLimit = 0xFFFFFFFFu;

#ifndef EQ_SHARED_WARPS
#define EQ_SHARED_WARPS 24
#endif
#ifndef EQ_SHARED_MIN_CTAS
#define EQ_SHARED_MIN_CTAS 1
#endif
constexpr int kSharedWarps = EQ_SHARED_WARPS;      // warps per block, shared-table kernel
constexpr int kSharedMinCtas = EQ_SHARED_MIN_CTAS; // register budget: blocks of kSharedWarps per SM
constexpr int kPrivateWarps = 4;                   // warps per block, per-warp-table kernel

// Output layouts of the decode kernel: bf16 with warp-uniform rows per group
// (cols % 256 == 0), bf16 with per-lane rows (cols % 8 == 0), bf16 element by
// element, or the raw symbol bytes (no dequant, no super weights).
enum : uint32_t { kRowUniform = 0, kLaneRows = 1, kGeneric = 2, kSymbolBytes = 3 };

// ---- PTX helpers: mbarrier + bulk copy (TMA, 1-D, no multicast) ---------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > kWaitCycles) return false;
    }
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__device__ __forceinline__ void st_global_v4(uint16_t *p, uint4 v) {
    asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// ---- number formats ----------------------------------------------------------------
// Two fp32 products, each rounded to nearest even.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    return make_float2(__fmul_rn(a.x, b.x), __fmul_rn(a.y, b.y));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float2 v) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint16_t to_bf16(float v) {
    __nv_bfloat16 h = __float2bfloat16_rn(v);
    return *reinterpret_cast<uint16_t *>(&h);
}

// Value of the symbol in the low byte of e.  Int8: two's
// complement.  E4M3 (OCP E4M3FN, bias 7): the 7 exponent and mantissa bits
// placed at bit 20 of an fp32 give exactly value * 2^-120 (subnormal codes
// included); the factor 2^120 is applied exactly, on its own or folded into
// a scale below 2^8 (same real product, one rounding).
template <int DT>
__device__ __forceinline__ float raw_value(uint32_t e) {
    if constexpr (DT == EQ_INT8) {
        return static_cast<float>(static_cast<int8_t>(e & 0xFFu));
    } else {
        return __uint_as_float(((e & 0x80u) << 24) | ((e & 0x7Fu) << 20));
    }
}

template <int DT>
__device__ __forceinline__ float dequant1(uint32_t e, float scale) {
    float v = raw_value<DT>(e);
    if constexpr (DT == EQ_E4M3) v = __fmul_rn(v, 0x1p120f);
    return __fmul_rn(v, scale);
}

// 8 symbols (low bytes of e[]) -> 8 bf16 in one 16-byte vector.  For E4M3
// with `folded` the scale already carries the factor 2^120.
template <int DT>
__device__ __forceinline__ uint4 dequant8(const uint32_t (&e)[8], float s, bool folded) {
    const float2 s2 = make_float2(s, s);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 v = make_float2(raw_value<DT>(e[2 * i]), raw_value<DT>(e[2 * i + 1]));
        if constexpr (DT == EQ_E4M3) {
            if (!folded) v = mul2(v, make_float2(0x1p120f, 0x1p120f));
        }
        o[i] = pack_bf16x2(mul2(v, s2));
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ void flag(int32_t *status, int32_t bits) {
    if ((threadIdx.x & 31u) == 0) atomicOr(status, bits);
}

// Checked build (EQ_CHECKED=1): conditions the kernels guarantee by
// construction are tested at run time, per lane; a failure ORs EQ_DEV_CHECK
// into the status word and the kernel carries on.  Compiled out otherwise.
#ifndef EQ_CHECKED
#define EQ_CHECKED 0
#endif
constexpr int32_t kDevCheck = 64;  // EQ_DEV_CHECK

__device__ __forceinline__ void check(int32_t *status, bool cond) {
#if EQ_CHECKED
    if (!cond) atomicOr(status, kDevCheck);
#else
    (void)status;
    (void)cond;
#endif
}

// ---- word staging ring ------------------------------------------------------------
// Per-warp bookkeeping lives in shared memory so that the decode loop keeps a
// single register for it: `limit`, the consumed-byte count at which the next
// group needs service (refill free slots or wait for a segment).
struct RingCtl {
    const uint8_t *payload;
    uint32_t pbytes;   // payload bytes rounded up to 16
    uint32_t n_segs;
    uint32_t issued;
    uint32_t ready;
    uint32_t phase;    // bit k: parity of the next completion of mbar[k]
    uint32_t dead;     // a bounded wait gave up
};

__device__ __forceinline__ uint32_t ring_limit(uint32_t n_segs, uint32_t issued, uint32_t ready) {
    // safe while bytes [pw, pw + kSpan) are resident and no free slot can take a segment
    uint32_t lim = kNoLimit;
    if (ready < n_segs) lim = ready * kSegBytes >= kSpan - 1 ? ready * kSegBytes - (kSpan - 1) : 0u;
    if (issued < n_segs) {
        const uint32_t t = issued >= kRingSegs - 1 ? (issued - (kRingSegs - 1)) * kSegBytes : 0u;
        lim = min(lim, t);
    }
    return lim;
}

#ifndef EQ_RING_INLINE
#define EQ_RING_INLINE __forceinline__
#endif
// Refill free slots, then make payload bytes [pw, pw + kSpan) resident.  Returns
// the new limit; on a wait that gave up sets ctl->dead and returns kNoLimit,
// leaving that segment counted as not ready.
__device__ EQ_RING_INLINE uint32_t ring_service(RingCtl *ctl, uint32_t ring, uint32_t mbar, uint32_t pw) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t n_segs = ctl->n_segs, pbytes = ctl->pbytes;
    uint32_t issued = ctl->issued, ready = ctl->ready, phase = ctl->phase;
    const uint32_t horizon = pw / kSegBytes + kRingSegs;
    if (issued < n_segs && issued < horizon) {
        __syncwarp();
        fence_proxy_async_smem();  // the slots being refilled were read through the generic proxy
        do {
            if (lane == 0) {
                const uint32_t bytes = min(kSegBytes, pbytes - issued * kSegBytes);
                const uint32_t slot = issued % kRingSegs;
                const uint8_t *src = ctl->payload + (size_t)issued * kSegBytes;
                mbar_expect_tx(mbar + 8 * slot, slot == 0 ? 2 * bytes : bytes);
                bulk_load(ring + slot * kSegBytes, src, bytes, mbar + 8 * slot);
                if (slot == 0) bulk_load(ring + kRingBytes, src, bytes, mbar);  // the mirror
            }
            ++issued;
        } while (issued < n_segs && issued < horizon);
    }
    uint32_t need = (pw + kSpan - 1) / kSegBytes;  // last segment touched by bytes [pw, pw + kSpan)
    if (need >= n_segs) need = n_segs - 1;
    bool ok = true;
    while (ready <= need && ready < issued) {
        const uint32_t slot = ready % kRingSegs;
        if (!__all_sync(kFull, mbar_wait_bounded(mbar + 8 * slot, (phase >> slot) & 1u))) {
            ok = false;  // the segment stays not ready: ring_drain waits for its copy again
            break;
        }
        phase ^= 1u << slot;
        ++ready;
    }
    __syncwarp();
    if (lane == 0) {
        ctl->issued = issued;
        ctl->ready = ready;
        ctl->phase = phase;
        if (!ok) ctl->dead = 1;
    }
    __syncwarp();
    return ok ? ring_limit(n_segs, issued, ready) : kNoLimit;
}

// Wait (bounded) for every copy still in flight so the ring can be reused.
__device__ __noinline__ bool ring_drain(RingCtl *ctl, uint32_t mbar) {
    const uint32_t lane = threadIdx.x & 31u;
    uint32_t ready = ctl->ready, phase = ctl->phase;
    const uint32_t issued = ctl->issued;
    bool all_ok = true;
    while (ready < issued) {
        const uint32_t slot = ready % kRingSegs;
        const bool got = mbar_wait_bounded(mbar + 8 * slot, (phase >> slot) & 1u);
        phase ^= 1u << slot;
        ++ready;
        all_ok = __all_sync(kFull, got) && all_ok;
    }
    __syncwarp();
    if (lane == 0) {
        ctl->ready = ready;
        ctl->phase = phase;
        if (!all_ok) ctl->dead = 1;
    }
    __syncwarp();
    return all_ok && !ctl->dead;
}

// Checked build: after a run of groups, the payload bytes consumed so far
// (pw) were all waited for, and the next output position of this lane (dst)
// is still inside the matrix ([out, out + n)).
__device__ __forceinline__ void check_progress(int32_t *status, const RingCtl *ctl, uint32_t pw, const uint16_t *dst,
                                               const uint16_t *out, uint64_t n, uint32_t lane) {
#if EQ_CHECKED
    check(status, pw <= min(ctl->ready * kSegBytes, ctl->pbytes));
    check(status, (uint64_t)(dst - out) <= n + kGroup * lane);
#else
    (void)status;
    (void)ctl;
    (void)pw;
    (void)dst;
    (void)out;
    (void)n;
    (void)lane;
#endif
}

// ---- the rANS step ---------------------------------------------------------------
// Integer helpers that run on the IMAD (FMA) pipe, keeping the ALU pipe free:
// mad.hi gives hi32(a * b) + c, so shifts right and field extraction cost one
// IMAD each.
__device__ __forceinline__ uint32_t mad_hi(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t mad_lo(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// One step of all 32 lanes.  `lut` is the shared-memory address of the slot
// table; `rp` the shared-memory address of the next unread word (inside the
// ring or its mirror), advanced past the words this step consumes.  Returns
// the slot entry (low byte: the stored symbol byte).
//   slot = x & 4095, e = lut[slot] = f << 20 | (slot - cum) << 8 | byte
//   x' = f * (x >> 12) + (slot - cum) = f * ((x >> 12) - 4096) + (e >> 8)
// Every lane reads a word (the ring always holds valid memory) and keeps it
// only if it renormalises (a select, not a branch).  Shifts and field
// extractions are written as IMADs (mad.hi by a power of two) so that they
// run on the FMA pipe next to the busier integer ALU pipe.
__device__ __forceinline__ uint32_t rans_step(uint32_t lut, uint32_t &rp, uint32_t &x, uint32_t lt) {
    const uint32_t addr = mad_hi(mad_lo(x, 1u << 20, 0u), 1u << 14, lut);  // lut + 4 * (x & 4095)
    const uint32_t e = lds_u32(addr);
    const uint32_t t = mad_hi(x, 1u << 20, 0u - kProbTotal);               // (x >> 12) - 4096
    x = mad_lo(mad_hi(e, 1u << 12, 0u), t, mad_hi(e, 1u << 24, 0u));
    const bool need = x < kStateLow;
    const uint32_t b = __ballot_sync(kFull, need);
    const uint32_t w = lds_u16(mad_lo(__popc(b & lt), 2u, rp));
    const uint32_t xr = mad_lo(x, 1u << 16, w);
    x = need ? xr : x;
    rp = mad_lo(__popc(b), 2u, rp);
    return e;
}

// Last, partial group: lane l is active at step r while 8l + r < rem.
__device__ __forceinline__ void rans_tail(uint32_t lut, uint32_t ring, uint32_t &x, uint32_t &pw, uint32_t lt,
                                          uint32_t lane, uint32_t rem, uint32_t (&e8)[8]) {
#pragma unroll
    for (uint32_t r = 0; r < 8; ++r) {
        const bool active = lane * kGroup + r < rem;
        bool need = false;
        if (active) {
            const uint32_t e = lds_u32(lut + 4 * (x & (kProbTotal - 1)));
            x = (e >> 20) * (x >> kProbBits) + ((e >> 8) & 0xFFFu);
            e8[r] = e;
            need = x < kStateLow;
        }
        const uint32_t b = __ballot_sync(kFull, need);
        const uint32_t w = lds_u16(ring + ((pw + 2u * __popc(b & lt)) & (kRingBytes - 1)));
        if (need) x = (x << 16) | w;
        pw += 2u * __popc(b);
    }
}

// ---- the Huffman step (codec 1) --------------------------------------------------
// Each lane holds its unread bits left-aligned in `buf`; `sh` = 16 - (bits
// held), kept as a signed count so that it is directly the shift that places
// a refill word just below the held bits.  A lane holding fewer than 12 bits
// (sh > 4) takes the next word (positions by ballot + popcount, as for rANS);
// then the top 12 bits index the slot table, whose entry gives the code
// length (bits 8..11) and the symbol or its rank (low byte), and the code's
// bits are shifted out.  Shifts by constants and the table address are
// written as IMADs (FMA pipe), leaving the integer ALU pipe the variable
// shifts, the merge and the selects.
__device__ __forceinline__ uint32_t shl_clamped(uint32_t v, uint32_t n) {  // v << n, 0 for n >= 32
    uint32_t r;
    asm("shl.b32 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(n));
    return r;
}

__device__ __forceinline__ uint32_t huff_step(uint32_t lut, uint32_t &rp, uint32_t &buf, uint32_t &sh,
                                              uint32_t lt) {
    const bool need = static_cast<int32_t>(sh) > static_cast<int32_t>(16u - kHuffMaxLen);
    const uint32_t b = __ballot_sync(kFull, need);
    const uint32_t w = lds_u16(mad_lo(__popc(b & lt), 2u, rp));
    const uint32_t filled = buf | shl_clamped(w, sh);
    buf = need ? filled : buf;
    sh = need ? sh - 16u : sh;
    rp = mad_lo(__popc(b), 2u, rp);
    const uint32_t e = lds_u32(mad_lo(mad_hi(buf, 1u << kHuffMaxLen, 0u), 4u, lut));  // lut + 4 * (buf >> 20)
    const uint32_t len = mad_hi(e, 1u << 24, 0u);                                      // e >> 8
    buf = shl_clamped(buf, len);
    sh += len;
    return e;
}

// Last, partial group (lane l active at step r while 8l + r < rem).
__device__ __forceinline__ void huff_tail(uint32_t lut, uint32_t ring, uint32_t &buf, uint32_t &sh, uint32_t &pw,
                                          uint32_t lt, uint32_t lane, uint32_t rem, uint32_t (&e8)[8]) {
#pragma unroll
    for (uint32_t r = 0; r < 8; ++r) {
        const bool active = lane * kGroup + r < rem;
        const bool need = active && static_cast<int32_t>(sh) > static_cast<int32_t>(16u - kHuffMaxLen);
        const uint32_t b = __ballot_sync(kFull, need);
        const uint32_t w = lds_u16(ring + ((pw + 2u * __popc(b & lt)) & (kRingBytes - 1)));
        if (need) {
            buf |= w << sh;
            sh -= 16u;
        }
        pw += 2u * __popc(b);
        if (active) {
            const uint32_t e = lds_u32(lut + 4u * (buf >> (32u - kHuffMaxLen)));
            const uint32_t len = e >> 8;
            buf = shl_clamped(buf, len);
            sh += len;
            e8[r] = e;
        }
    }
}

// Per-lane decoder state of a codec, its step, tail, start and end checks.
template <uint32_t CODEC> struct CodecState;
template <> struct CodecState<kCodecRans> { uint32_t x; };
template <> struct CodecState<kCodecHuffman> { uint32_t buf, sh; };

template <uint32_t CODEC>
__device__ __forceinline__ uint32_t codec_step(uint32_t lut, uint32_t &rp, CodecState<CODEC> &s, uint32_t lt) {
    if constexpr (CODEC == kCodecHuffman) return huff_step(lut, rp, s.buf, s.sh, lt);
    else return rans_step(lut, rp, s.x, lt);
}

template <uint32_t CODEC>
__device__ __forceinline__ void codec_tail(uint32_t lut, uint32_t ring, CodecState<CODEC> &s, uint32_t &pw,
                                           uint32_t lt, uint32_t lane, uint32_t rem, uint32_t (&e8)[8]) {
    if constexpr (CODEC == kCodecHuffman) huff_tail(lut, ring, s.buf, s.sh, pw, lt, lane, rem, e8);
    else rans_tail(lut, ring, s.x, pw, lt, lane, rem, e8);
}

// rANS: the state from the record; Huffman: no bits held.
template <uint32_t CODEC>
__device__ __forceinline__ CodecState<CODEC> codec_start(uint32_t x0) {
    if constexpr (CODEC == kCodecHuffman) return CodecState<CODEC>{0u, 16u};  // no bits held
    else return CodecState<CODEC>{x0};
}

// A valid stream ends with every rANS state back at 2^16 / every Huffman bit
// still held being zero padding.
template <uint32_t CODEC>
__device__ __forceinline__ bool codec_done(const CodecState<CODEC> &s) {
    if constexpr (CODEC == kCodecHuffman) return s.buf == 0;
    else return s.x == kStateLow;
}

// Rank mode: with 2..32 distinct symbols and a warp-uniform row per group, the
// slot table's low byte holds the symbol's rank (index in the ascending
// frequency list) and lane r keeps fp32_rn(value(symbol of rank r) * row
// scale).  A decoded symbol's dequantised value is then one shuffle from the
// lane named by its rank (shfl uses only the low 5 bits of the entry).
template <uint32_t LAYOUT>
__device__ __forceinline__ bool rank_mode(uint32_t n_present) {
    return LAYOUT == kRowUniform && n_present >= 2 && n_present <= 32;
}

// The byte the shared table stores for list entry i (rank mode: the rank).
template <uint32_t LAYOUT>
__device__ __forceinline__ uint32_t table_low_byte(uint32_t n_present, uint32_t i, uint32_t sym) {
    return rank_mode<LAYOUT>(n_present) ? i : sym;
}

// Exact fp32 value of a symbol byte (Int8 or E4M3).
template <int DT>
__device__ __forceinline__ float symbol_value(uint32_t sym) {
    if constexpr (DT == EQ_INT8) {
        return static_cast<float>(static_cast<int8_t>(sym & 0xFFu));
    } else {
        return __fmul_rn(__uint_as_float(((sym & 0x80u) << 24) | ((sym & 0x7Fu) << 20)), 0x1p120f);
    }
}

// A chunk record's header fields and this lane's initial state.
struct ChunkHead {
    const uint8_t *rec;
    uint32_t n, n_words, n_present, table_bytes;
    uint32_t x;
};

// Point a chain's staging ring at a chunk record's payload.
__device__ __forceinline__ bool ring_start(RingCtl *ctl, const ChunkHead &h) {
    if ((threadIdx.x & 31u) == 0) {
        const uint32_t pbytes = (2u * h.n_words + 15u) & ~15u;
        ctl->payload = h.rec + h.table_bytes;
        ctl->pbytes = pbytes;
        ctl->n_segs = (pbytes + kSegBytes - 1) / kSegBytes;
        ctl->issued = 0;
        ctl->ready = 0;
    }
    return true;
}

// Bytes before a record's frequency list / code table: counts, plus the 32
// lane states for rANS (Huffman records carry no states).
template <uint32_t CODEC>
constexpr uint32_t kHeadBytes = CODEC == kCodecHuffman ? kHuffRecordHeadBytes : kRecordHeadBytes;

// Header of chunk k: checks it against the directory; on success fills the
// record pointer, counts and (rANS) this lane's initial state.
template <uint32_t CODEC = kCodecRans, class Params, class Job>
__device__ __forceinline__ bool load_head(const Params &P, const Job &M, uint32_t k, uint32_t lane,
                                          ChunkHead &h) {
    const uint64_t first = (uint64_t)k * kChunkSyms;
    const uint64_t rem = M.n_elems - first;
    const uint32_t n_expect = rem < kChunkSyms ? (uint32_t)rem : kChunkSyms;
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
    if (h.n != n_expect || h.n_present < 1 || h.n_present > 256 ||
        off + h.table_bytes + ((2ull * h.n_words + 15) & ~15ull) != end) {
        flag(P.status, EQ_DEV_BAD_HEADER);
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

// Slots a table entry covers: rANS its frequency f (entry = symbol | f << 16);
// Huffman 2^(12 - length) (entry = symbol | length << 16; the empty code of a
// single-symbol chunk, length 0, covers all 4096), 0 for a length over 12.
template <uint32_t CODEC>
__device__ __forceinline__ uint32_t entry_slots(uint32_t e) {
    if constexpr (CODEC == kCodecHuffman) return (e >> 16) <= kHuffMaxLen ? 1u << (kHuffMaxLen - (e >> 16)) : 0u;
    else return e >> 16;
}

// Order key of a table entry: rANS entries ascend by symbol, Huffman entries
// by (length, symbol), which is the entry itself (bits 8..15 are zero).
template <uint32_t CODEC>
__device__ __forceinline__ int entry_key(uint32_t e) {
    return CODEC == kCodecHuffman ? (int)e : (int)(e & 0xFFu);
}

// Slot-table entry for slot t of a list entry covering f slots: rANS
// f << 20 | t << 8 | low; Huffman length << 8 | low.
template <uint32_t CODEC>
__device__ __forceinline__ uint32_t slot_entry(uint32_t e, uint32_t f, uint32_t t, uint32_t low) {
    if constexpr (CODEC == kCodecHuffman) return ((e >> 16) << 8) | low;
    else return (f << 20) | (t << 8) | low;
}

// Checked build: every slot of a filled table holds a usable entry -- rANS:
// f >= 1 and slot - cum < f; Huffman: a code length of 1..12.  Threads
// `first`, `first + step`, ... check their slots.
template <uint32_t CODEC>
__device__ __forceinline__ void check_table(int32_t *status, const uint32_t *lut, uint32_t first, uint32_t step) {
#if EQ_CHECKED
    for (uint32_t t = first; t < kProbTotal; t += step) {
        const uint32_t e = lut[t];
        if constexpr (CODEC == kCodecHuffman) {
            const uint32_t len = (e >> 8) & 0xFu;
            check(status, len >= 1 && len <= kHuffMaxLen);
        } else {
            check(status, (e >> 20) >= 1 && ((e >> 8) & 0xFFFu) < (e >> 20));
        }
    }
#else
    (void)status;
    (void)lut;
    (void)first;
    (void)step;
#endif
}

// Check a frequency list / code table (n_present entries at `tab`): keys
// ascending, reserved bits zero, every entry covering >= 1 slot, all 4096
// slots covered (rANS: sum of f; Huffman: Kraft equality).  Optionally copies
// the entries and their cumulative slot counts to shared memory, and/or
// expands the list into a warp's slot table.  Returns validity (warp-uniform).
template <uint32_t CODEC = kCodecRans>
__device__ __forceinline__ bool warp_table(const uint32_t *tab, uint32_t n_present, uint32_t lane,
                                           uint32_t *entries_out, uint32_t *cum_out, uint32_t *lut,
                                           bool by_rank) {
    uint32_t run = 0;
    int prev_key = -1;
    bool ok = true;
    for (uint32_t base = 0; base < n_present; base += 32) {
        const uint32_t i = base + lane;
        const bool have = i < n_present;
        const uint32_t e = have ? tab[i] : 0u;
        const uint32_t f = have ? entry_slots<CODEC>(e) : 0u;
        bool good = !have || ((e & 0xFF00u) == 0 && f >= 1 && f <= kProbTotal);
        const int key = entry_key<CODEC>(e);
        const int left = __shfl_up_sync(kFull, key, 1);
        if (have && key <= (lane == 0 ? prev_key : left)) good = false;
        uint32_t inc = f;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t t = __shfl_up_sync(kFull, inc, d);
            if (lane >= (uint32_t)d) inc += t;
        }
        const uint32_t cum = run + inc - f;
        if (have) {
            if (entries_out) entries_out[i] = e;
            if (cum_out) cum_out[i] = cum;
        }
        ok = __all_sync(kFull, good) && ok;
        const uint32_t cnt = min(32u, n_present - base);
        if (lut && n_present > 1) {
            for (uint32_t q = 0; q < cnt; ++q) {
                const uint32_t fq = __shfl_sync(kFull, f, q);
                const uint32_t cq = __shfl_sync(kFull, cum, q);
                const uint32_t eq = __shfl_sync(kFull, e, q);
                const uint32_t low = by_rank ? base + q : (eq & 0xFFu);
                for (uint32_t t = lane; t < fq; t += 32) {
                    const uint32_t slot = cq + t;
                    if (slot < kProbTotal && fq < kProbTotal) lut[slot] = slot_entry<CODEC>(eq, fq, t, low);
                }
            }
        }
        prev_key = __shfl_sync(kFull, key, cnt - 1);
        run += __shfl_sync(kFull, inc, 31);
    }
    return ok && run == kProbTotal;
}

// Shared memory of one block: slot table(s), then per warp a 2.5 KB word ring
// (with its mirror), the ring's mbarriers and bookkeeping, then the block's
// reference frequency list (shared-table kernel only).
template <int WARPS, bool SHARED>
struct Smem {
    static constexpr uint32_t kChains = SHARED ? EQ_CHAINS : 1;          // chunks decoded at once per warp
    static constexpr uint32_t kLuts = SHARED ? 1 : WARPS;
    static constexpr uint32_t kRingOff = kLuts * kLutBytes;             // + runtime pad to 128 B
    static constexpr uint32_t kMbarOff = kRingOff + WARPS * kChains * kRingStride;  // offsets below include the pad
    static constexpr uint32_t kCtlOff = kMbarOff + WARPS * kChains * kRingSegs * 8;
    static constexpr uint32_t kRefOff = kCtlOff + WARPS * kChains * 32;  // 32 bytes of RingCtl per chain
    static constexpr uint32_t kBlockOff = kRefOff + (SHARED ? 2 * 256 * 4 : 0);
    static constexpr uint32_t kBytes = kBlockOff + 16 + 128;            // + worst-case alignment pad
};
static_assert(sizeof(RingCtl) <= 32, "RingCtl slot");

// Per-warp views of a decode block's shared memory (layout Smem<WARPS, SHARED>);
// initialises this warp's ring mbarriers and bookkeeping.
template <int WARPS, bool SHARED>
struct WarpSmem {
    static constexpr uint32_t C = Smem<WARPS, SHARED>::kChains;
    uint32_t ring;              // shared address of chain 0's ring (chain c at + c * kRingStride)
    uint32_t mbar;              // chain 0's mbarriers (chain c at + 8 * kRingSegs * c)
    RingCtl *ctl;               // C entries
    uint32_t *lut;              // the slot table this warp reads
    uint32_t lut_addr;
    uint32_t *ref_entries;      // shared-table kernels: the block's frequency list ...
    uint32_t *ref_cum;          // ... and cumulative frequencies
    volatile uint32_t *blk;     // shared-table kernels: [0] n_present (0 if invalid), [1] valid

    __device__ __forceinline__ WarpSmem(unsigned char *smem_raw, uint32_t warp, uint32_t lane) {
        using L = Smem<WARPS, SHARED>;
        const uint32_t base = smem_u32(smem_raw);
        const uint32_t pad = (128u - ((base + L::kRingOff) & 127u)) & 127u;
        unsigned char *padded = smem_raw + pad;  // offsets from kRingOff on are relative to this
        ring = base + pad + L::kRingOff + warp * C * kRingStride;
        mbar = base + pad + L::kMbarOff + warp * C * kRingSegs * 8;
        ctl = reinterpret_cast<RingCtl *>(padded + L::kCtlOff + warp * C * 32);
        lut = reinterpret_cast<uint32_t *>(smem_raw) + (SHARED ? 0u : warp * kProbTotal);
        lut_addr = smem_u32(lut);
        ref_entries = reinterpret_cast<uint32_t *>(padded + L::kRefOff);
        ref_cum = ref_entries + 256;
        blk = reinterpret_cast<uint32_t *>(padded + L::kBlockOff);
        if (lane == 0) {
            for (uint32_t i = 0; i < C * kRingSegs; ++i) mbar_init(mbar + 8 * i, 1);
            fence_mbar_init();
            for (uint32_t c = 0; c < C; ++c) {
                ctl[c].phase = 0;
                ctl[c].dead = 0;
                ctl[c].issued = ctl[c].ready = 0;
            }
        }
        __syncwarp();
    }
};

// Shared-table kernels, on a change of matrix: rebuild the block's slot table
// from the frequency list of chunk k0 (the first chunk of the block's tile),
// after checking it.  All threads of the block take part.
template <int WARPS, uint32_t LAYOUT, uint32_t CODEC = kCodecRans, class Params, class Job, class WS>
__device__ __forceinline__ void shared_table_rebuild(const Params &P, const Job &M, uint32_t k0, uint32_t lane,
                                                     uint32_t warp, const WS &S) {
    __syncthreads();
    if (warp == 0) {
        ChunkHead h;
        bool ok = load_head<CODEC>(P, M, k0, lane, h);
        if (ok) ok = warp_table<CODEC>(reinterpret_cast<const uint32_t *>(h.rec + kHeadBytes<CODEC>), h.n_present,
                                       lane, S.ref_entries, S.ref_cum, nullptr, false);
        if (lane == 0) {
            S.blk[0] = ok ? h.n_present : 0u;
            S.blk[1] = ok;
        }
    }
    __syncthreads();
    const uint32_t np = S.blk[0];
    if (S.blk[1] && np > 1) {
        for (uint32_t i = 0; i < np; ++i) {
            const uint32_t e = S.ref_entries[i], c = S.ref_cum[i];
            const uint32_t f = entry_slots<CODEC>(e), sy = e & 0xFFu;
            const uint32_t low = table_low_byte<LAYOUT>(np, i, sy);
            for (uint32_t t = threadIdx.x; t < f; t += WARPS * 32)
                if (c + t < kProbTotal && f < kProbTotal) S.lut[c + t] = slot_entry<CODEC>(e, f, t, low);
        }
    }
    __syncthreads();
    if (S.blk[1] && np > 1) check_table<CODEC>(P.status, S.lut, threadIdx.x, WARPS * 32);
}

// Shared-table kernels: chunk k's header, checked, and its frequency list
// compared with the block's (every chunk of a shared-table matrix must carry
// the same list).  False (with a status flag) if either check fails.
template <uint32_t CODEC = kCodecRans, class Params, class Job, class WS>
__device__ __forceinline__ bool shared_chunk_head(const Params &P, const Job &M, uint32_t k, uint32_t lane,
                                                  uint32_t np, const WS &S, ChunkHead &h) {
    if (!load_head<CODEC>(P, M, k, lane, h)) return false;
    bool same = S.blk[1] && h.n_present == np;
    if (same) {
        const uint32_t *tab = reinterpret_cast<const uint32_t *>(h.rec + kHeadBytes<CODEC>);
        for (uint32_t i = lane; i < np; i += 32) same = same && tab[i] == S.ref_entries[i];
    }
    if (!__all_sync(kFull, same)) {
        flag(P.status, EQ_DEV_BAD_TABLE);
        return false;
    }
    return true;
}

// The work item (matrix) that launch-wide unit `unit` belongs to.
template <class Params>
__device__ __forceinline__ uint32_t job_of(const Params &P, uint32_t unit) {
    uint32_t mi = 0;
    while (mi + 1 < P.n_mats && unit >= P.mats[mi + 1].begin) ++mi;
    return mi;
}

// ---- host: kernel variants and launch geometry -----------------------------------------
template <class Params>
struct KernelSetup {
    void (*fn)(Params) = nullptr;
    int warps = 0;
    size_t smem = 0;
    int ctas_per_sm = 0;
    uint32_t units_per_cta = 0;  // work units (tiles or chunks) a block takes per round
};

template <class Params>
int setup_kernel(KernelSetup<Params> &k, void (*fn)(Params), int warps, size_t smem, uint32_t units_per_cta) {
    k.fn = fn;
    k.warps = warps;
    k.smem = smem;
    k.units_per_cta = units_per_cta;
    if (cudaFuncSetAttribute(reinterpret_cast<const void *>(fn), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return EQ_ERR_CUDA;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&k.ctas_per_sm, fn, warps * 32, smem) != cudaSuccess ||
        k.ctas_per_sm < 1)
        return EQ_ERR_CUDA;
    return EQ_OK;
}

// Shared-table kernels take their chunks in tiles: tile t of a matrix holds
// chunks [t * W * C, (t + 1) * W * C), warp w of the block decoding chunks
// w, w + W, ... (C of them, in lockstep when C = 2) of it.  A launch whose
// tiles of max_warps single chunks fit one round of resident blocks runs one
// chain per warp (C = 1: a small launch is bound by the latency of each
// chunk's 2048 dependent steps, and a warp with one chain steps faster than
// one with two); otherwise C = max_chains.  W (P.tile_warps) is the fewest
// warps per tile that still fit the launch into one round, so that a block of
// small matrices spreads over every SM instead of filling a few of them with
// full tiles; when even full tiles need more than one round, W = max_warps.
// Sets the tile shape, every matrix's first unit and the total.
template <class Params>
void assign_tiles(Params &P, uint32_t resident, uint32_t max_warps, uint32_t max_chains) {
    auto units_for = [&](uint32_t w, uint32_t c) {
        uint64_t units = 0;
        for (uint32_t i = 0; i < P.n_mats; ++i) units += (P.mats[i].n_chunks - P.mats[i].chunk0 + w * c - 1) / (w * c);
        return units;
    };
    const uint32_t chains = units_for(max_warps, 1) <= resident ? 1u : max_chains;
    uint32_t tw = max_warps;
    for (uint32_t w = 1; w < max_warps; ++w)
        if (units_for(w, chains) <= resident) {
            tw = w;
            break;
        }
    P.tile_warps = tw;
    P.tile_chains = chains;
    P.total_units = 0;
    for (uint32_t i = 0; i < P.n_mats; ++i) {
        P.mats[i].begin = P.total_units;
        P.total_units += (P.mats[i].n_chunks - P.mats[i].chunk0 + tw * chains - 1) / (tw * chains);
    }
}

// Persistent grid: at most one round of resident blocks, fewer when there is
// less work than that.
template <class Params>
int launch(const KernelSetup<Params> &k, int sms, const Params &P, cudaStream_t s) {
    if (!P.total_units) return EQ_OK;
    const uint32_t resident = (uint32_t)(sms * k.ctas_per_sm);
    const uint32_t want = (P.total_units + k.units_per_cta - 1) / k.units_per_cta;
    const uint32_t grid = want < resident ? want : resident;
    k.fn<<<grid, k.warps * 32, k.smem, s>>>(P);
    return cudaGetLastError() == cudaSuccess ? EQ_OK : EQ_ERR_CUDA;
}

}  // namespace
