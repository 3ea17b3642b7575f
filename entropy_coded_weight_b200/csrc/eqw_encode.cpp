// Host encoder for container v1 (eq_encoder_run / eq_encoded_write /
// eq_encode_host).
//
// EntQuant technical summary (gist.science 2601.22787), section 2 "weight
// encoding": the (already quantised, low-entropy) weights are flattened into a
// symbol stream and compressed losslessly with an ANS coder; storage is the
// bitstream, the scales and metadata.  Here the stream of every matrix is cut
// into independent 65536-symbol chunks (EntroLLM technical overview,
// "parallel decoding strategy": chunks that keep the tensor structure and
// decode independently); each chunk gets its own 12-bit frequency table and
// 32 interleaved rANS states.  Chunks are encoded in parallel on host threads.
#include <algorithm>
#include <array>
#include <atomic>
#include <cmath>
#include <cstring>
#include <memory>
#include <new>
#include <thread>
#include <vector>

#include "eqw_encode_common.h"

using namespace eqw;

namespace {

// ---- one chunk record ----------------------------------------------------------
// Symbol j of the chunk belongs to lane (j % 256) / 8 at step 8 * (j / 256) + j % 8.
// The decoder walks steps upward and lanes upward inside a step, so the encoder
// walks both downward and writes each renormalisation word in front of the
// previous one.
// `table` is the matrix-wide frequency table, or null to quantise this chunk's own histogram.
void encode_record(const uint8_t *sym, uint32_t n, const uint32_t *table, std::vector<uint8_t> &rec,
                   std::vector<uint16_t> &scratch) {
    uint32_t f[256], cum[256];
    if (table) {
        std::memcpy(f, table, sizeof f);
    } else {
        uint64_t cnt[256] = {0};
        for (uint32_t j = 0; j < n; ++j) ++cnt[sym[j]];
        quantize_table(cnt, n, f);
    }
    uint32_t c = 0;
    uint32_t n_present = 0;
    for (int s = 0; s < 256; ++s) {
        cum[s] = c;
        c += f[s];
        n_present += f[s] != 0;
    }

    // x >= limit[s] means the state must shed 16 bits before coding s
    uint64_t limit[256];
    for (int s = 0; s < 256; ++s) limit[s] = (uint64_t)f[s] << (32 - kProbBits);

    if (scratch.size() < n) scratch.resize(n);
    uint16_t *wend = scratch.data() + n;
    uint16_t *w = wend;
    uint32_t x[kLanes];
    for (uint32_t l = 0; l < kLanes; ++l) x[l] = kStateLow;

    const uint32_t groups = (n + kGroupSyms - 1) / kGroupSyms;
    for (uint32_t g = groups; g-- > 0;) {
        const uint32_t base = g * kGroupSyms;
        const bool full = base + kGroupSyms <= n;
        for (uint32_t r = kGroup; r-- > 0;) {
            for (uint32_t l = kLanes; l-- > 0;) {
                const uint32_t j = base + l * kGroup + r;
                if (!full && j >= n) continue;
                const uint32_t s = sym[j];
                uint32_t xv = x[l];
                if (xv >= limit[s]) {
                    *--w = (uint16_t)xv;
                    xv >>= 16;
                }
                const uint32_t q = xv / f[s];
                x[l] = q * kProbTotal + (xv - q * f[s]) + cum[s];
            }
        }
    }
    const uint32_t n_words = (uint32_t)(wend - w);

    const size_t table_end = align_up(kRecordHeadBytes + 4 * (size_t)n_present, 16);
    const size_t total = table_end + align_up(2 * (size_t)n_words, 16);
    rec.assign(total, 0);
    uint8_t *p = rec.data();
    const uint32_t head[4] = {n, n_words, n_present, 0};
    std::memcpy(p, head, 16);
    std::memcpy(p + 16, x, 4 * kLanes);
    uint32_t *tab = reinterpret_cast<uint32_t *>(p + kRecordHeadBytes);
    for (int s = 0, k = 0; s < 256; ++s)
        if (f[s]) tab[k++] = (uint32_t)s | (f[s] << 16);
    std::memcpy(p + table_end, w, 2 * (size_t)n_words);
}

// One Huffman chunk record.  `table_len` holds the matrix-wide lengths, or
// null to build this chunk's own code.  Lane l's bit stream is its symbols'
// canonical codes in step order, most significant bit first, cut into 16-bit
// words; before each of its symbols a lane holding fewer than 12 unread bits
// takes its next word, and the record stores those words in the order they
// are taken (step by step, lanes ascending).
void encode_record_huffman(const uint8_t *sym, uint32_t n, const uint32_t *table_len, std::vector<uint8_t> &rec) {
    uint8_t len[256];
    uint64_t cnt[256] = {0};
    for (uint32_t j = 0; j < n; ++j) ++cnt[sym[j]];
    if (table_len) {
        for (int s = 0; s < 256; ++s) len[s] = (uint8_t)table_len[s];
    } else {
        huffman_lengths(cnt, len);
    }
    // canonical codes; table entries in (length, symbol) order
    uint16_t code[256];
    huffman_codes(len, code);
    std::vector<uint32_t> entries;
    for (uint32_t l = 1; l <= kHuffMaxLen; ++l)
        for (int s = 0; s < 256; ++s)
            if (len[s] == l) entries.push_back((uint32_t)s | (l << 16));
    const bool single = entries.empty();
    std::vector<uint16_t> out;
    if (single) {
        int s0 = 0;
        while (s0 < 255 && !cnt[s0]) ++s0;
        entries.push_back((uint32_t)s0);
    } else {
        // each lane's stream as 16-bit words
        std::vector<uint16_t> stream[kLanes];
        uint32_t acc[kLanes] = {0}, nacc[kLanes] = {0};
        const uint32_t steps = kGroup * ((n + kGroupSyms - 1) / kGroupSyms);
        auto index_of = [](uint32_t t, uint32_t l) { return kGroupSyms * (t / kGroup) + kGroup * l + t % kGroup; };
        for (uint32_t t = 0; t < steps; ++t)
            for (uint32_t l = 0; l < kLanes; ++l) {
                const uint32_t j = index_of(t, l);
                if (j >= n) continue;
                const uint32_t L = len[sym[j]];
                acc[l] = (acc[l] << L) | code[sym[j]];
                nacc[l] += L;
                if (nacc[l] >= 16) {
                    stream[l].push_back((uint16_t)(acc[l] >> (nacc[l] - 16)));
                    nacc[l] -= 16;
                    acc[l] &= (1u << nacc[l]) - 1u;
                }
            }
        for (uint32_t l = 0; l < kLanes; ++l)
            if (nacc[l]) stream[l].push_back((uint16_t)(acc[l] << (16 - nacc[l])));
        // the decoder's refill schedule
        uint32_t held[kLanes] = {0}, taken[kLanes] = {0};
        for (uint32_t t = 0; t < steps; ++t)
            for (uint32_t l = 0; l < kLanes; ++l) {
                const uint32_t j = index_of(t, l);
                if (j >= n) continue;
                if (held[l] < kHuffMaxLen) {
                    out.push_back(taken[l] < stream[l].size() ? stream[l][taken[l]] : (uint16_t)0);
                    ++taken[l];
                    held[l] += 16;
                }
                held[l] -= len[sym[j]];
            }
    }
    const uint32_t n_present = (uint32_t)entries.size();
    const size_t table_end = align_up(kHuffRecordHeadBytes + 4 * (size_t)n_present, 16);
    rec.assign(table_end + align_up(2 * out.size(), 16), 0);
    uint8_t *p = rec.data();
    const uint32_t head[4] = {n, (uint32_t)out.size(), n_present, 0};
    std::memcpy(p, head, 16);
    std::memcpy(p + kHuffRecordHeadBytes, entries.data(), 4 * entries.size());
    if (!out.empty()) std::memcpy(p + table_end, out.data(), 2 * out.size());
}

struct Job {
    uint32_t mat;
    uint32_t chunk;
};

// Shape checks plus the checks that read host data: no E4M3 NaN code, outliers in range and ascending.
int validate(const eq_matrix_in *mats, uint32_t n_mats, uint32_t *n_layers) {
    int rc = validate_shapes(mats, n_mats, n_layers);
    if (rc) return rc;
    for (uint32_t i = 0; i < n_mats; ++i) {
        const eq_matrix_in &m = mats[i];
        const uint64_t n = (uint64_t)m.rows * m.cols;
        if (m.dtype == EQ_E4M3)
            for (uint64_t k = 0; k < n; ++k)
                if ((m.symbols[k] & 0x7F) == 0x7F) return EQ_ERR_INVALID_ARG;
        if (!outliers_valid(m.rows, m.cols, m.n_out, m.out_row, m.out_col)) return EQ_ERR_INVALID_ARG;
    }
    return EQ_OK;
}

}  // namespace

struct eq_encoded {
    std::vector<uint8_t> bytes;
};

extern "C" EQW_API int eq_encoder_run(const eq_matrix_in *mats, uint32_t n_mats, int n_threads,
                                      eq_encoded **h, size_t *size) {
    if (!h || !size) return EQ_ERR_INVALID_ARG;
    *h = nullptr;
    uint32_t n_layers = 0;
    int rc = validate(mats, n_mats, &n_layers);
    if (rc) return rc;

    ContainerPlan P;
    plan_order(mats, n_mats, n_layers, P);
    const std::vector<uint32_t> &order = P.order;
    std::vector<Job> jobs;
    jobs.reserve(P.n_jobs);
    for (uint32_t d = 0; d < n_mats; ++d)
        for (uint32_t k = 0; k < P.n_chunks[d]; ++k) jobs.push_back({d, k});

    // the symbols of chunk i, with super weights replaced by the placeholder 0
    auto chunk_symbols = [&](size_t i, std::vector<uint8_t> &patched, uint32_t *len_out) -> const uint8_t * {
        const eq_matrix_in &m = mats[order[jobs[i].mat]];
        const uint64_t n = (uint64_t)m.rows * m.cols;
        const uint64_t first = (uint64_t)jobs[i].chunk * kChunkSyms;
        const uint32_t len = (uint32_t)std::min<uint64_t>(kChunkSyms, n - first);
        *len_out = len;
        const uint8_t *src = m.symbols + first;
        if (!m.n_out) return src;
        patched.assign(src, src + len);
        for (uint32_t k = 0; k < m.n_out; ++k) {
            const uint64_t lin = (uint64_t)m.out_row[k] * m.cols + m.out_col[k];
            if (lin >= first && lin < first + len) patched[lin - first] = 0;
        }
        return patched.data();
    };
    auto run_parallel = [&](auto &&body) {
        std::atomic<size_t> next{0};
        auto worker = [&]() {
            for (;;) {
                const size_t i = next.fetch_add(1);
                if (i >= jobs.size()) break;
                body(i);
            }
        };
        unsigned nt = n_threads > 0 ? (unsigned)n_threads : std::max(1u, std::thread::hardware_concurrency());
        nt = (unsigned)std::min<size_t>(nt, std::max<size_t>(1, jobs.size()));
        std::vector<std::thread> pool;
        for (unsigned t = 1; t < nt; ++t) pool.emplace_back(worker);
        worker();
        for (auto &t : pool) t.join();
    };

    // pass 1 (matrices with one table): histogram of every chunk, summed per matrix
    std::vector<std::array<uint64_t, 256>> hist(jobs.size());
    bool any_matrix_table = false;
    for (uint32_t d = 0; d < n_mats; ++d) any_matrix_table |= !(mats[order[d]].flags & EQ_TABLE_PER_CHUNK);
    std::vector<std::array<uint32_t, 256>> mat_table(n_mats);
    if (any_matrix_table) {
        run_parallel([&](size_t i) {
            if (mats[order[jobs[i].mat]].flags & EQ_TABLE_PER_CHUNK) return;
            thread_local std::vector<uint8_t> patched;
            uint32_t len = 0;
            const uint8_t *src = chunk_symbols(i, patched, &len);
            hist[i].fill(0);
            for (uint32_t j = 0; j < len; ++j) ++hist[i][src[j]];
        });
        std::vector<std::array<uint64_t, 256>> total(n_mats);
        for (auto &t : total) t.fill(0);
        for (size_t i = 0; i < jobs.size(); ++i)
            if (!(mats[order[jobs[i].mat]].flags & EQ_TABLE_PER_CHUNK))
                for (int s = 0; s < 256; ++s) total[jobs[i].mat][s] += hist[i][s];
        for (uint32_t d = 0; d < n_mats; ++d) {
            uint64_t n = 0;
            for (int s = 0; s < 256; ++s) n += total[d][s];
            if (!n) continue;
            if (mats[order[d]].flags & EQ_CODEC_HUFFMAN) {
                uint8_t len[256];
                huffman_lengths(total[d].data(), len);
                for (int s = 0; s < 256; ++s) mat_table[d][s] = len[s];
            } else {
                quantize_table(total[d].data(), n, mat_table[d].data());
            }
        }
    }
    hist.clear();
    hist.shrink_to_fit();

    // pass 2: encode every chunk
    std::vector<std::vector<uint8_t>> records(jobs.size());
    run_parallel([&](size_t i) {
        thread_local std::vector<uint16_t> scratch;
        thread_local std::vector<uint8_t> patched;
        uint32_t len = 0;
        const uint8_t *src = chunk_symbols(i, patched, &len);
        const uint32_t flags = mats[order[jobs[i].mat]].flags;
        const uint32_t *table = (flags & EQ_TABLE_PER_CHUNK) ? nullptr : mat_table[jobs[i].mat].data();
        if (flags & EQ_CODEC_HUFFMAN) encode_record_huffman(src, len, table, records[i]);
        else encode_record(src, len, table, records[i], scratch);
    });

    std::vector<uint64_t> rec_size(jobs.size());
    for (size_t i = 0; i < jobs.size(); ++i) rec_size[i] = records[i].size();
    plan_offsets(mats, rec_size, P);
    const uint64_t total = P.total;

    auto *enc = new (std::nothrow) eq_encoded;
    if (!enc) return EQ_ERR_NOSPACE;
    try {
        enc->bytes.assign(total, 0);
    } catch (...) {
        delete enc;
        return EQ_ERR_NOSPACE;
    }
    uint8_t *b = enc->bytes.data();
    write_header_directory(b, mats, P);
    for (uint32_t d = 0; d < n_mats; ++d) {
        const eq_matrix_in &m = mats[order[d]];
        const ContainerPlan::Place &pl = P.place[d];
        write_chunk_index(b + pl.ci, P, d);
        if (m.rows) std::memcpy(b + pl.so, m.scales, 4ull * m.rows);
        write_outliers(b + pl.oo, m.n_out, m.out_row, m.out_col, m.out_val);
        for (uint32_t k = 0; k < P.n_chunks[d]; ++k) {
            const uint32_t j = P.first_job[d] + k;
            std::memcpy(b + P.rec_off[j], records[j].data(), records[j].size());
        }
    }
    *h = enc;
    *size = total;
    return EQ_OK;
}

extern "C" EQW_API int eq_encoded_write(const eq_encoded *h, void *out, size_t out_cap) {
    if (!h || (!out && !h->bytes.empty())) return EQ_ERR_INVALID_ARG;
    if (out_cap < h->bytes.size()) return EQ_ERR_NOSPACE;
    std::memcpy(out, h->bytes.data(), h->bytes.size());
    return EQ_OK;
}

extern "C" EQW_API void eq_encoded_free(eq_encoded *h) { delete h; }

extern "C" EQW_API int eq_encode_host(const eq_matrix_in *mats, uint32_t n_mats, int n_threads, void *out,
                                      size_t out_cap, size_t *out_len) {
    const eqw::NvtxScope nvtx_range("eq_encode_host");
    if (!out_len) return EQ_ERR_INVALID_ARG;
    eq_encoded *h = nullptr;
    size_t size = 0;
    int rc = eq_encoder_run(mats, n_mats, n_threads, &h, &size);
    if (rc) return rc;
    *out_len = size;
    rc = eq_encoded_write(h, out, out_cap);
    eq_encoded_free(h);
    return rc;
}
