// Device encoder for container v1: eq_encode_device, eq_encode_device_workspace.
//
// EntQuant technical summary (gist.science 2601.22787), section 2 "weight
// encoding": the quantised weights are flattened into a symbol stream and
// compressed losslessly by a GPU ANS coder; storage = bitstream + scales +
// metadata.  This is the same encoder as eq_encode_host with the per-symbol
// work on the GPU and the symbols read from device memory:
//   K1 eq_enc_hist_kernel       one warp per chunk: histogram (super-weight
//                               positions count as the placeholder 0), E4M3
//                               NaN-code check; matrix-wide sums by 64-bit
//                               atomics, or the chunk's own histogram;
//   host                        frequency tables by the host encoder's
//                               routine (so both encoders pick the same
//                               table), then the container plan;
//   K2 eq_enc_rans_kernel<0>    one warp per chunk, the 32 interleaved rANS
//                               encoders walking the chunk backwards:
//                               renormalisation word count only;
//   host                        record sizes -> offsets, header, directory,
//                               chunk index, scales, outliers;
//   K2 eq_enc_rans_kernel<1>    the same walk again, now writing states,
//                               table and words into each record.
// Lane l of the encoding warp owns symbols 8l..8l+7 of every 256-symbol group
// (the decoder's lane mapping); within a step the renormalising lanes' words
// are stored in ascending lane order just in front of the words of the
// following steps, at positions given by a ballot and a population count.
// Huffman matrices (EntroLLM technical overview, "Huffman weight encoding")
// take K3 eq_enc_huff_kernel<0/1> in place of K2, with code lengths built on
// the host from the K1 histograms by the host encoder's routine: the
// decoder's refill schedule walked forwards, each lane cutting its own code
// string into the 16-bit words it hands out at its refills.
#include <cuda_runtime.h>

#include <algorithm>
#include <array>
#include <mutex>
#include <vector>

#include "eqw_encode_common.h"

using namespace eqw;

namespace {

constexpr uint32_t kFullMask = 0xFFFFFFFFu;
constexpr int kEncWarps = 8;  // warps per block; one chunk per warp at a time

struct EncMat {
    const uint8_t *symbols;   // device, rows * cols
    const uint32_t *out_row;  // device, n_out (ascending linear index)
    const uint32_t *out_col;
    uint64_t n;               // rows * cols
    uint64_t ci;              // container offset of the chunk index (pass 2)
    uint32_t cols;
    uint32_t n_out;
    uint32_t dtype;
    uint32_t n_chunks;
    uint32_t first_job;       // first chunk in launch-wide job order
    uint32_t per_chunk;       // 1: each chunk has its own table
    uint32_t table0;          // table slot of chunk 0 (per_chunk: + k)
    uint32_t hist0;           // per_chunk: chunk-histogram slot of chunk 0
    uint32_t codec;           // kCodecRans or kCodecHuffman
};

struct EncWork {
    const EncMat *mats;
    uint32_t n_mats;
    uint32_t n_jobs;
    unsigned long long *mat_hist;  // [n_mats][256]
    uint32_t *chunk_hist;          // [per-chunk chunks][256]
    const uint32_t *tables;        // [slots][256] rANS frequencies, or Huffman codes (huff_slot)
    uint32_t *n_words;             // [n_jobs]
    uint32_t *status;              // bit 0: an E4M3 NaN code
    uint8_t *out;                  // container (pass 2)
};

__device__ __forceinline__ uint32_t mat_of(const EncWork &W, uint32_t job) {
    uint32_t lo = 0, hi = W.n_mats;  // last matrix with first_job <= job (empty matrices own no jobs)
    while (hi - lo > 1) {
        const uint32_t mid = (lo + hi) / 2;
        if (W.mats[mid].first_job <= job) lo = mid;
        else hi = mid;
    }
    while (lo + 1 < W.n_mats && W.mats[lo].n_chunks == 0) ++lo;
    return lo;
}

__device__ __forceinline__ uint64_t out_lin(const EncMat &M, uint32_t k) {
    return (uint64_t)M.out_row[k] * M.cols + M.out_col[k];
}

// First outlier with linear index >= lin.
__device__ __forceinline__ uint32_t out_lower_bound(const EncMat &M, uint64_t lin) {
    uint32_t b = 0, e = M.n_out;
    while (b < e) {
        const uint32_t mid = (b + e) / 2;
        if (out_lin(M, mid) < lin) b = mid + 1;
        else e = mid;
    }
    return b;
}

// The 8 symbols lane `lane` owns in group g of a chunk starting at `first`
// (n symbols), as two little-endian words; missing tail bytes are 0.
__device__ __forceinline__ uint2 load8(const EncMat &M, uint64_t first, uint32_t n, uint32_t g, uint32_t lane) {
    const uint32_t j0 = g * kGroupSyms + kGroup * lane;
    const uint8_t *p = M.symbols + first + j0;
    if (j0 + kGroup <= n) return *reinterpret_cast<const uint2 *>(p);
    uint32_t w[2] = {0, 0};
    for (uint32_t r = 0; j0 + r < n && r < kGroup; ++r) w[r / 4] |= (uint32_t)p[r] << (8 * (r % 4));
    return make_uint2(w[0], w[1]);
}

__device__ __forceinline__ uint32_t byte_of(uint2 v, uint32_t r) {
    return ((r < 4 ? v.x : v.y) >> (8 * (r & 3))) & 0xFFu;
}

__global__ void __launch_bounds__(kEncWarps * 32) eq_enc_hist_kernel(const __grid_constant__ EncWork W) {
    __shared__ uint32_t hist_s[kEncWarps][256];
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
    uint32_t *hist = hist_s[warp];
    for (uint32_t job = blockIdx.x * kEncWarps + warp; job < W.n_jobs; job += gridDim.x * kEncWarps) {
        const EncMat &M = W.mats[mat_of(W, job)];
        const uint32_t k = job - M.first_job;
        const uint64_t first = (uint64_t)k * kChunkSyms;
        const uint32_t n = (uint32_t)(M.n - first < kChunkSyms ? M.n - first : kChunkSyms);
        for (uint32_t i = lane; i < 256; i += 32) hist[i] = 0;
        __syncwarp();
        bool nan_code = false;
        const uint32_t groups = (n + kGroupSyms - 1) / kGroupSyms;
        for (uint32_t g = 0; g < groups; ++g) {
            const uint2 v = load8(M, first, n, g, lane);
            const uint32_t j0 = g * kGroupSyms + kGroup * lane;
            for (uint32_t r = 0; r < kGroup; ++r) {
                if (j0 + r >= n) break;
                const uint32_t s = byte_of(v, r);
                nan_code |= M.dtype == EQ_E4M3 && (s & 0x7Fu) == 0x7Fu;
                atomicAdd(&hist[s], 1u);
            }
        }
        __syncwarp();
        if (lane == 0 && M.n_out) {
            // super weights are encoded as the placeholder symbol 0
            for (uint32_t o = out_lower_bound(M, first); o < M.n_out && out_lin(M, o) < first + n; ++o) {
                const uint32_t s = M.symbols[out_lin(M, o)];
                hist[s] -= 1;
                hist[0] += 1;
            }
        }
        __syncwarp();
        if (__any_sync(kFullMask, nan_code) && lane == 0) atomicOr(W.status, 1u);
        if (M.per_chunk) {
            uint32_t *dst = W.chunk_hist + 256ull * (M.hist0 + k);
            for (uint32_t i = lane; i < 256; i += 32) dst[i] = hist[i];
        } else {
            unsigned long long *dst = W.mat_hist + 256ull * (&M - W.mats);
            for (uint32_t i = lane; i < 256; i += 32)
                if (hist[i]) atomicAdd(dst + i, (unsigned long long)hist[i]);
        }
        __syncwarp();
    }
}

// One chunk's rANS encode, walking groups, steps and lanes downwards (the
// reverse of the decoder).  WRITE = 0: count the renormalisation words into
// n_words[job].  WRITE = 1: write the whole record at its offset.
template <int WRITE>
__global__ void __launch_bounds__(kEncWarps * 32) eq_enc_rans_kernel(const __grid_constant__ EncWork W) {
    __shared__ uint32_t freq_s[kEncWarps][256];
    __shared__ uint32_t cum_s[kEncWarps][256];
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
    uint32_t *F = freq_s[warp], *C = cum_s[warp];
    uint32_t lanemask_ge;
    asm("mov.u32 %0, %%lanemask_ge;" : "=r"(lanemask_ge));
    for (uint32_t job = blockIdx.x * kEncWarps + warp; job < W.n_jobs; job += gridDim.x * kEncWarps) {
        const EncMat &M = W.mats[mat_of(W, job)];
        if (M.codec != kCodecRans) continue;
        const uint32_t k = job - M.first_job;
        const uint64_t first = (uint64_t)k * kChunkSyms;
        const uint32_t n = (uint32_t)(M.n - first < kChunkSyms ? M.n - first : kChunkSyms);
        const uint32_t *tab = W.tables + 256ull * (M.table0 + (M.per_chunk ? k : 0u));

        // frequencies, cumulative frequencies (ascending symbols), present count
        uint32_t run = 0, n_present = 0;
        for (uint32_t base = 0; base < 256; base += 32) {
            const uint32_t f = tab[base + lane];
            uint32_t inc = f;
            for (int d = 1; d < 32; d <<= 1) {
                const uint32_t t = __shfl_up_sync(kFullMask, inc, d);
                if (lane >= (uint32_t)d) inc += t;
            }
            F[base + lane] = f;
            C[base + lane] = run + inc - f;
            run += __shfl_sync(kFullMask, inc, 31);
            n_present += __popc(__ballot_sync(kFullMask, f != 0));
        }
        __syncwarp();

        uint8_t *rec = nullptr;
        uint16_t *words = nullptr;
        uint32_t end = 0;  // words still to place below this position (WRITE)
        if (WRITE) {
            const uint64_t off = reinterpret_cast<const uint64_t *>(W.out + M.ci)[k];
            rec = W.out + off;
            words = reinterpret_cast<uint16_t *>(rec + ((kRecordHeadBytes + 4u * n_present + 15u) & ~15u));
            end = W.n_words[job];
        }
        uint32_t count = 0;
        uint32_t x = kStateLow;
        // super weights of this chunk, visited from the last one down
        uint32_t o_lo = 0, o = 0;
        if (M.n_out) {
            o_lo = out_lower_bound(M, first);
            o = out_lower_bound(M, first + n);
        }
        const uint32_t groups = (n + kGroupSyms - 1) / kGroupSyms;
        for (uint32_t g = groups; g-- > 0;) {
            uint2 v = load8(M, first, n, g, lane);
            const uint64_t g_lo = first + (uint64_t)g * kGroupSyms;
            while (o > o_lo && out_lin(M, o - 1) >= g_lo) {
                --o;
                const uint32_t j = (uint32_t)(out_lin(M, o) - g_lo);
                if (lane == j / kGroup) {
                    const uint32_t r = j % kGroup;
                    if (r < 4) v.x &= ~(0xFFu << (8 * r));
                    else v.y &= ~(0xFFu << (8 * (r - 4)));
                }
            }
            const uint32_t j0 = g * kGroupSyms + kGroup * lane;
            for (uint32_t r = kGroup; r-- > 0;) {
                const bool active = j0 + r < n;
                const uint32_t s = byte_of(v, r);
                const uint32_t f = active ? F[s] : 1u;
                const bool need = active && (uint64_t)x >= ((uint64_t)f << (32 - kProbBits));
                const uint32_t b = __ballot_sync(kFullMask, need);
                if (WRITE) {
                    if (need) words[end - __popc(b & lanemask_ge)] = (uint16_t)x;
                    end -= __popc(b);
                }
                count += __popc(b);
                if (need) x >>= 16;
                if (active) {
                    const uint32_t q = x / f;
                    x = q * kProbTotal + (x - q * f) + C[s];
                }
            }
        }
        if (!WRITE) {
            if (lane == 0) W.n_words[job] = count;
        } else {
            uint32_t *head = reinterpret_cast<uint32_t *>(rec);
            if (lane == 0) {
                head[0] = n;
                head[1] = count;
                head[2] = n_present;
                head[3] = 0;
            }
            head[4 + lane] = x;
            uint32_t *entries = head + kRecordHeadBytes / 4;
            uint32_t at = 0;
            for (uint32_t base = 0; base < 256; base += 32) {
                const uint32_t s = base + lane, f = F[s];
                const uint32_t b = __ballot_sync(kFullMask, f != 0);
                if (f) entries[at + __popc(b & ((1u << lane) - 1u))] = s | (f << 16);
                at += __popc(b);
            }
        }
        __syncwarp();
    }
}

// The 8 symbols of load8 with the super weights among them replaced by the
// placeholder symbol 0.
__device__ __forceinline__ uint2 load8_patched(const EncMat &M, uint64_t first, uint32_t n, uint32_t g,
                                               uint32_t lane) {
    uint2 v = load8(M, first, n, g, lane);
    if (M.n_out) {
        const uint64_t lo = first + (uint64_t)g * kGroupSyms + kGroup * lane;
        for (uint32_t o = out_lower_bound(M, lo); o < M.n_out && out_lin(M, o) < lo + kGroup; ++o) {
            const uint32_t r = (uint32_t)(out_lin(M, o) - lo);
            if (r < 4) v.x &= ~(0xFFu << (8 * r));
            else v.y &= ~(0xFFu << (8 * (r - 4)));
        }
    }
    return v;
}

// Huffman table slot entry: code length (0: no code), canonical code, and a
// mark on the one symbol of a table without codes.
__host__ __device__ constexpr uint32_t huff_slot(uint32_t len, uint32_t code, bool single) {
    return len | code << 8 | (single ? 1u << 31 : 0u);
}

// One chunk's Huffman record.  Lane l's code string is the canonical codes
// of its symbols in step order; before each of its symbols the decoder gives
// a lane holding fewer than 12 unread bits its next 16-bit word, the words of
// one step in ascending lane order.  This walks those steps forwards: every
// lane counts the bits it holds and, at a refill, cuts the next 16 bits off
// its string (a producer running ahead over its own symbols; zero padding
// after the last code).  WRITE = 0: word count into n_words[job]; WRITE = 1:
// the whole record at its offset.
template <int WRITE>
__global__ void __launch_bounds__(kEncWarps * 32) eq_enc_huff_kernel(const __grid_constant__ EncWork W) {
    __shared__ uint32_t tab_s[kEncWarps][256];
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
    uint32_t *T = tab_s[warp];
    const uint32_t lt = (1u << lane) - 1u;
    for (uint32_t job = blockIdx.x * kEncWarps + warp; job < W.n_jobs; job += gridDim.x * kEncWarps) {
        const EncMat &M = W.mats[mat_of(W, job)];
        if (M.codec != kCodecHuffman) continue;
        const uint32_t k = job - M.first_job;
        const uint64_t first = (uint64_t)k * kChunkSyms;
        const uint32_t n = (uint32_t)(M.n - first < kChunkSyms ? M.n - first : kChunkSyms);
        const uint32_t *tab = W.tables + 256ull * (M.table0 + (M.per_chunk ? k : 0u));
        uint32_t n_coded = 0, single = 0;
        for (uint32_t base = 0; base < 256; base += 32) {
            const uint32_t e = tab[base + lane];
            T[base + lane] = e;
            n_coded += __popc(__ballot_sync(kFullMask, (e & 0xFFu) != 0));
            const uint32_t m = __ballot_sync(kFullMask, (e >> 31) != 0);
            if (m) single = base + __ffs(m) - 1;
        }
        __syncwarp();
        const uint32_t n_present = n_coded ? n_coded : 1u;

        uint16_t *words = nullptr;
        uint8_t *rec = nullptr;
        if (WRITE) {
            const uint64_t off = reinterpret_cast<const uint64_t *>(W.out + M.ci)[k];
            rec = W.out + off;
            words = reinterpret_cast<uint16_t *>(rec + ((kHuffRecordHeadBytes + 4u * n_present + 15u) & ~15u));
        }
        uint32_t count = 0;  // WRITE = 0: this lane's refills; WRITE = 1: the warp's words so far
        if (n_coded) {
            const uint32_t steps = kGroup * ((n + kGroupSyms - 1) / kGroupSyms);
            uint32_t held = 0;
            uint2 cv = make_uint2(0, 0), pv = make_uint2(0, 0);
            uint32_t cg = ~0u, pg = ~0u;
            uint32_t pt = 0, nacc = 0;  // producer: next step to append, bits pending in acc
            uint64_t acc = 0;
            for (uint32_t t = 0; t < steps; ++t) {
                const uint32_t g = t / kGroup, r = t % kGroup;
                const bool active = g * kGroupSyms + kGroup * lane + r < n;
                if (g != cg) {
                    cv = load8_patched(M, first, n, g, lane);
                    cg = g;
                }
                const bool need = active && held < kHuffMaxLen;
                if (WRITE) {
                    const uint32_t b = __ballot_sync(kFullMask, need);
                    if (need) {
                        for (;;) {
                            if (nacc >= 16) break;
                            const uint32_t pgi = pt / kGroup;
                            if (pgi * kGroupSyms + kGroup * lane + pt % kGroup >= n) break;  // string ends
                            if (pgi != pg) {
                                pv = load8_patched(M, first, n, pgi, lane);
                                pg = pgi;
                            }
                            const uint32_t e = T[byte_of(pv, pt % kGroup)];
                            const uint32_t L = e & 0xFFu;
                            acc = (acc << L) | ((e >> 8) & 0xFFFu);
                            nacc += L;
                            ++pt;
                        }
                        uint32_t w;
                        if (nacc >= 16) {
                            nacc -= 16;
                            w = (uint32_t)(acc >> nacc) & 0xFFFFu;
                            acc &= (1ull << nacc) - 1ull;
                        } else {
                            w = (uint32_t)(acc << (16 - nacc)) & 0xFFFFu;
                            nacc = 0;
                            acc = 0;
                        }
                        words[count + __popc(b & lt)] = (uint16_t)w;
                    }
                    count += __popc(b);
                } else if (need) {
                    ++count;
                }
                if (need) held += 16;
                if (active) held -= T[byte_of(cv, r)] & 0xFFu;
            }
        }
        if (!WRITE) {
            for (int d = 16; d > 0; d >>= 1) count += __shfl_xor_sync(kFullMask, count, d);
            if (lane == 0) W.n_words[job] = count;
        } else {
            uint32_t *head = reinterpret_cast<uint32_t *>(rec);
            if (lane == 0) {
                head[0] = n;
                head[1] = count;
                head[2] = n_present;
                head[3] = 0;
            }
            uint32_t *entries = head + kHuffRecordHeadBytes / 4;
            if (!n_coded) {
                if (lane == 0) entries[0] = single;
            } else {
                uint32_t at = 0;
                for (uint32_t l = 1; l <= kHuffMaxLen; ++l)
                    for (uint32_t base = 0; base < 256; base += 32) {
                        const uint32_t s = base + lane;
                        const bool has = (T[s] & 0xFFu) == l;
                        const uint32_t b = __ballot_sync(kFullMask, has);
                        if (has) entries[at + __popc(b & lt)] = s | (l << 16);
                        at += __popc(b);
                    }
            }
        }
        __syncwarp();
    }
}

struct WorkLayout {
    size_t mats, mat_hist, chunk_hist, tables, n_words, status, total;
    uint32_t n_pc_chunks;
};

WorkLayout work_layout(const eq_matrix_in *mats, uint32_t n_mats, const ContainerPlan &P) {
    WorkLayout L{};
    uint32_t pc = 0;
    for (uint32_t d = 0; d < n_mats; ++d)
        if (mats[P.order[d]].flags & EQ_TABLE_PER_CHUNK) pc += P.n_chunks[d];
    L.n_pc_chunks = pc;
    size_t pos = 0;
    auto take = [&](size_t bytes) {
        const size_t at = pos;
        pos = align_up(pos + bytes, 256);
        return at;
    };
    L.mats = take(sizeof(EncMat) * std::max<uint32_t>(1, n_mats));
    L.mat_hist = take(8ull * 256 * std::max<uint32_t>(1, n_mats));
    L.chunk_hist = take(4ull * 256 * std::max<uint32_t>(1, pc));
    L.tables = take(4ull * 256 * (n_mats + pc + 1));
    L.n_words = take(4ull * std::max<uint32_t>(1, P.n_jobs));
    L.status = take(4);
    L.total = pos;
    return L;
}

int cuda_ok(cudaError_t e) { return e == cudaSuccess ? EQ_OK : EQ_ERR_CUDA; }

}  // namespace

extern "C" EQW_API int eq_encode_bound(const eq_matrix_in *mats, uint32_t n_mats, size_t *out_bytes) {
    if (!out_bytes) return EQ_ERR_INVALID_ARG;
    uint32_t n_layers = 0;
    int rc = validate_shapes(mats, n_mats, &n_layers);
    if (rc) return rc;
    ContainerPlan P;
    plan_order(mats, n_mats, n_layers, P);
    // at most 256 table entries and one word per symbol (a step sheds 16 bits at most once)
    std::vector<uint64_t> rec_size(P.n_jobs);
    for (uint32_t d = 0; d < n_mats; ++d) {
        const uint64_t n = (uint64_t)mats[P.order[d]].rows * mats[P.order[d]].cols;
        for (uint32_t k = 0; k < P.n_chunks[d]; ++k)
            rec_size[P.first_job[d] + k] =
                record_bytes(256, (uint32_t)std::min<uint64_t>(kChunkSyms, n - (uint64_t)k * kChunkSyms));
    }
    plan_offsets(mats, rec_size, P);
    *out_bytes = P.total;
    return EQ_OK;
}

extern "C" EQW_API int eq_encode_device_workspace(const eq_matrix_in *mats, uint32_t n_mats, size_t *work_bytes) {
    if (!work_bytes) return EQ_ERR_INVALID_ARG;
    uint32_t n_layers = 0;
    int rc = validate_shapes(mats, n_mats, &n_layers);
    if (rc) return rc;
    ContainerPlan P;
    plan_order(mats, n_mats, n_layers, P);
    *work_bytes = work_layout(mats, n_mats, P).total;
    return EQ_OK;
}

namespace {

int encode_device(const eq_matrix_in *mats, uint32_t n_mats, void *d_out, size_t out_cap, size_t *out_len,
                  void *d_work, size_t work_bytes, cudaStream_t s) {
    if (!out_len) return EQ_ERR_INVALID_ARG;
    uint32_t n_layers = 0;
    int rc = validate_shapes(mats, n_mats, &n_layers);
    if (rc) return rc;
    for (uint32_t i = 0; i < n_mats; ++i) {
        const eq_matrix_in &m = mats[i];
        if ((uint64_t)m.rows * m.cols && reinterpret_cast<uintptr_t>(m.symbols) % 8) return EQ_ERR_INVALID_ARG;
    }
    ContainerPlan P;
    plan_order(mats, n_mats, n_layers, P);
    const WorkLayout L = work_layout(mats, n_mats, P);
    if (!d_work || work_bytes < L.total) return EQ_ERR_INVALID_ARG;
    uint8_t *wk = static_cast<uint8_t *>(d_work);

    // super weights: copied to the host for the checks and the container records
    std::vector<std::vector<uint32_t>> orow(n_mats), ocol(n_mats);
    std::vector<std::vector<float>> oval(n_mats);
    for (uint32_t d = 0; d < n_mats; ++d) {
        const eq_matrix_in &m = mats[P.order[d]];
        orow[d].resize(m.n_out);
        ocol[d].resize(m.n_out);
        oval[d].resize(m.n_out);
        if (!m.n_out) continue;
        if ((rc = cuda_ok(cudaMemcpyAsync(orow[d].data(), m.out_row, 4ull * m.n_out, cudaMemcpyDeviceToHost, s))) ||
            (rc = cuda_ok(cudaMemcpyAsync(ocol[d].data(), m.out_col, 4ull * m.n_out, cudaMemcpyDeviceToHost, s))) ||
            (rc = cuda_ok(cudaMemcpyAsync(oval[d].data(), m.out_val, 4ull * m.n_out, cudaMemcpyDeviceToHost, s))))
            return rc;
    }
    if ((rc = cuda_ok(cudaStreamSynchronize(s)))) return rc;
    for (uint32_t d = 0; d < n_mats; ++d) {
        const eq_matrix_in &m = mats[P.order[d]];
        if (!outliers_valid(m.rows, m.cols, m.n_out, orow[d].data(), ocol[d].data())) return EQ_ERR_INVALID_ARG;
    }

    // matrix descriptors (directory order)
    std::vector<EncMat> em(n_mats);
    uint32_t pc = 0;
    for (uint32_t d = 0; d < n_mats; ++d) {
        const eq_matrix_in &m = mats[P.order[d]];
        EncMat &e = em[d];
        e.symbols = m.symbols;
        e.out_row = m.out_row;
        e.out_col = m.out_col;
        e.n = (uint64_t)m.rows * m.cols;
        e.ci = 0;
        e.cols = m.cols;
        e.n_out = m.n_out;
        e.dtype = m.dtype;
        e.n_chunks = P.n_chunks[d];
        e.first_job = P.first_job[d];
        e.per_chunk = (m.flags & EQ_TABLE_PER_CHUNK) ? 1u : 0u;
        e.table0 = e.per_chunk ? n_mats + pc : d;
        e.hist0 = pc;
        e.codec = (m.flags & EQ_CODEC_HUFFMAN) ? kCodecHuffman : kCodecRans;
        if (e.per_chunk) pc += P.n_chunks[d];
    }
    EncWork W{};
    W.mats = reinterpret_cast<const EncMat *>(wk + L.mats);
    W.n_mats = n_mats;
    W.n_jobs = P.n_jobs;
    W.mat_hist = reinterpret_cast<unsigned long long *>(wk + L.mat_hist);
    W.chunk_hist = reinterpret_cast<uint32_t *>(wk + L.chunk_hist);
    W.tables = reinterpret_cast<const uint32_t *>(wk + L.tables);
    W.n_words = reinterpret_cast<uint32_t *>(wk + L.n_words);
    W.status = reinterpret_cast<uint32_t *>(wk + L.status);
    W.out = static_cast<uint8_t *>(d_out);
    int sms = 0, dev = 0;
    if ((rc = cuda_ok(cudaGetDevice(&dev))) ||
        (rc = cuda_ok(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev))))
        return rc;
    const uint32_t grid = std::max<uint32_t>(1, std::min<uint32_t>((P.n_jobs + kEncWarps - 1) / kEncWarps,
                                                                   (uint32_t)sms * 8));

    // K1: histograms
    if (n_mats && (rc = cuda_ok(cudaMemcpyAsync(wk + L.mats, em.data(), sizeof(EncMat) * n_mats,
                                                cudaMemcpyHostToDevice, s))))
        return rc;
    if ((rc = cuda_ok(cudaMemsetAsync(wk + L.mat_hist, 0, 8ull * 256 * std::max<uint32_t>(1, n_mats), s))) ||
        (rc = cuda_ok(cudaMemsetAsync(wk + L.status, 0, 4, s))))
        return rc;
    if (P.n_jobs) {
        eq_enc_hist_kernel<<<grid, kEncWarps * 32, 0, s>>>(W);
        if ((rc = cuda_ok(cudaGetLastError()))) return rc;
    }
    std::vector<unsigned long long> mat_hist(256ull * n_mats);
    std::vector<uint32_t> chunk_hist(256ull * pc);
    uint32_t status = 0;
    if ((n_mats && (rc = cuda_ok(cudaMemcpyAsync(mat_hist.data(), wk + L.mat_hist, 8ull * 256 * n_mats,
                                                 cudaMemcpyDeviceToHost, s)))) ||
        (pc && (rc = cuda_ok(cudaMemcpyAsync(chunk_hist.data(), wk + L.chunk_hist, 4ull * 256 * pc,
                                             cudaMemcpyDeviceToHost, s)))) ||
        (rc = cuda_ok(cudaMemcpyAsync(&status, wk + L.status, 4, cudaMemcpyDeviceToHost, s))) ||
        (rc = cuda_ok(cudaStreamSynchronize(s))))
        return rc;
    if (status) return EQ_ERR_INVALID_ARG;  // an E4M3 NaN code

    // tables: slot d for matrix-wide tables, n_mats + chunk for per-chunk
    // ones; rANS: quantised frequencies; Huffman: lengths and canonical codes
    // (huff_slot), both by the host encoder's routines
    std::vector<uint32_t> tables(256ull * (n_mats + pc + 1), 0);
    std::vector<uint32_t> n_present(P.n_jobs, 0);
    for (uint32_t d = 0; d < n_mats; ++d) {
        const EncMat &e = em[d];
        const uint64_t n = e.n;
        uint32_t np_matrix = 0;
        for (uint32_t k = 0; k < e.n_chunks; ++k) {
            uint32_t *f = tables.data() + 256ull * (e.table0 + (e.per_chunk ? k : 0u));
            if (e.per_chunk || k == 0) {
                uint64_t cnt[256];
                for (int t = 0; t < 256; ++t)
                    cnt[t] = e.per_chunk ? chunk_hist[256ull * (e.hist0 + k) + t] : mat_hist[256ull * d + t];
                uint32_t np = 0;
                if (e.codec == kCodecHuffman) {
                    uint8_t len[256];
                    uint16_t code[256];
                    huffman_lengths(cnt, len);
                    huffman_codes(len, code);
                    int first_sym = -1;
                    for (int t = 0; t < 256; ++t) {
                        np += len[t] != 0;
                        if (cnt[t] && first_sym < 0) first_sym = t;
                    }
                    for (int t = 0; t < 256; ++t) f[t] = huff_slot(len[t], code[t], !np && t == first_sym);
                    if (!np) np = 1;  // the empty code: one table entry, no words
                } else {
                    quantize_table(cnt, e.per_chunk ? std::min<uint64_t>(kChunkSyms, n - (uint64_t)k * kChunkSyms)
                                                    : n, f);
                    for (int t = 0; t < 256; ++t) np += f[t] != 0;
                }
                np_matrix = np;
            }
            n_present[e.first_job + k] = np_matrix;
        }
    }
    if ((rc = cuda_ok(cudaMemcpyAsync(wk + L.tables, tables.data(), 4 * tables.size(), cudaMemcpyHostToDevice, s))))
        return rc;

    // K2 / K3, pass 1: word counts
    bool any_rans = false, any_huff = false;
    for (const EncMat &e : em) {
        any_rans |= e.n_chunks && e.codec == kCodecRans;
        any_huff |= e.n_chunks && e.codec == kCodecHuffman;
    }
    std::vector<uint32_t> n_words(P.n_jobs);
    if (P.n_jobs) {
        if (any_rans) eq_enc_rans_kernel<0><<<grid, kEncWarps * 32, 0, s>>>(W);
        if (any_huff) eq_enc_huff_kernel<0><<<grid, kEncWarps * 32, 0, s>>>(W);
        if ((rc = cuda_ok(cudaGetLastError())) ||
            (rc = cuda_ok(cudaMemcpyAsync(n_words.data(), wk + L.n_words, 4ull * P.n_jobs, cudaMemcpyDeviceToHost,
                                          s))))
            return rc;
    }
    if ((rc = cuda_ok(cudaStreamSynchronize(s)))) return rc;

    // the container plan, then everything but the records
    std::vector<uint64_t> rec_size(P.n_jobs);
    for (uint32_t d = 0; d < n_mats; ++d)
        for (uint32_t k = 0; k < em[d].n_chunks; ++k) {
            const uint32_t j = em[d].first_job + k;
            rec_size[j] = record_bytes(n_present[j], n_words[j], em[d].codec);
        }
    plan_offsets(mats, rec_size, P);
    *out_len = P.total;
    if (out_cap < P.total) return EQ_ERR_NOSPACE;
    if (!d_out) return EQ_ERR_INVALID_ARG;
    uint8_t *out = static_cast<uint8_t *>(d_out);
    const size_t meta = kHeaderBytes + (size_t)kDirEntryBytes * n_mats;
    std::vector<uint8_t> head(meta, 0);
    write_header_directory(head.data(), mats, P);
    std::vector<std::vector<uint8_t>> idx(n_mats), outl(n_mats);
    if ((rc = cuda_ok(cudaMemsetAsync(out, 0, P.total, s))) ||
        (rc = cuda_ok(cudaMemcpyAsync(out, head.data(), meta, cudaMemcpyHostToDevice, s))))
        return rc;
    for (uint32_t d = 0; d < n_mats; ++d) {
        const eq_matrix_in &m = mats[P.order[d]];
        const ContainerPlan::Place &pl = P.place[d];
        em[d].ci = pl.ci;
        idx[d].resize(8ull * (P.n_chunks[d] + 1));
        write_chunk_index(idx[d].data(), P, d);
        if ((rc = cuda_ok(cudaMemcpyAsync(out + pl.ci, idx[d].data(), idx[d].size(), cudaMemcpyHostToDevice, s))))
            return rc;
        if (m.rows && (rc = cuda_ok(cudaMemcpyAsync(out + pl.so, m.scales, 4ull * m.rows, cudaMemcpyDeviceToDevice,
                                                     s))))
            return rc;
        if (m.n_out) {
            outl[d].resize(12ull * m.n_out);
            write_outliers(outl[d].data(), m.n_out, orow[d].data(), ocol[d].data(), oval[d].data());
            if ((rc = cuda_ok(cudaMemcpyAsync(out + pl.oo, outl[d].data(), outl[d].size(), cudaMemcpyHostToDevice,
                                              s))))
                return rc;
        }
    }
    if (n_mats && (rc = cuda_ok(cudaMemcpyAsync(wk + L.mats, em.data(), sizeof(EncMat) * n_mats,
                                                cudaMemcpyHostToDevice, s))))
        return rc;

    // K2 / K3, pass 2: the records
    if (P.n_jobs) {
        if (any_rans) eq_enc_rans_kernel<1><<<grid, kEncWarps * 32, 0, s>>>(W);
        if (any_huff) eq_enc_huff_kernel<1><<<grid, kEncWarps * 32, 0, s>>>(W);
        if ((rc = cuda_ok(cudaGetLastError()))) return rc;
    }
    return cuda_ok(cudaStreamSynchronize(s));
}

}  // namespace

extern "C" EQW_API int eq_encode_device(const eq_matrix_in *mats, uint32_t n_mats, void *d_out, size_t out_cap,
                                        size_t *out_len, void *d_work, size_t work_bytes, cudaStream_t s) {
    const eqw::NvtxScope nvtx_range("eq_encode_device");
    return encode_device(mats, n_mats, d_out, out_cap, out_len, d_work, work_bytes, s);
}

namespace {

// Workspace of eq_encode_device_noalloc: a file-scope device array (one per
// device context, reserved when the library's module loads), so that entry
// point allocates nothing; a host mutex serialises its users.  In host code
// the array's name is only a host-side stand-in: its device address comes from
// cudaGetSymbolAddress, looked up once per device (with that device current)
// on the entry point's first call there.
constexpr size_t kStaticScratchBytes = 16u << 20;
static __device__ __align__(256) uint8_t g_encode_scratch[kStaticScratchBytes];
std::mutex g_encode_scratch_mu;
void *g_encode_scratch_ptr[128];  // device address of the array on each device (null: not looked up yet)

}  // namespace

extern "C" EQW_API int eq_encode_device_noalloc(const eq_matrix_in *mats, uint32_t n_mats, void *d_out,
                                                size_t out_cap, size_t *out_len, cudaStream_t s) {
    const eqw::NvtxScope nvtx_range("eq_encode_device_noalloc");
    if (!out_len) return EQ_ERR_INVALID_ARG;
    size_t need = 0;
    int rc = eq_encode_device_workspace(mats, n_mats, &need);
    if (rc) return rc;
    if (need > kStaticScratchBytes) return EQ_ERR_NOSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return EQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_encode_scratch_mu);
    if (!g_encode_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_encode_scratch) != cudaSuccess || !p) return EQ_ERR_CUDA;
        g_encode_scratch_ptr[dev] = p;
    }
    rc = encode_device(mats, n_mats, d_out, out_cap, out_len, g_encode_scratch_ptr[dev], kStaticScratchBytes, s);
    // an error return may come after a kernel launch: let the stream drain before
    // the next caller may reuse the array
    if (rc) cudaStreamSynchronize(s);
    return rc;
}
