// Container v1 parsing and validation (eq_model_open and the model queries).
//
// EntQuant technical summary (gist.science 2601.22787), section 2
// "inference-time decoding": the compressed bitstream stays resident in GPU
// memory.  eq_model_open therefore only parses a host copy of the container
// and keeps plain offsets into the caller's device copy; no device memory is
// allocated or copied.  Every field a kernel will rely on for addressing
// (section offsets, chunk record bounds, table sizes) is validated here, so a
// corrupt container is refused before anything is launched.
#include <cstring>
#include <new>

#include "eqw_internal.h"

using namespace eqw;

namespace {

template <class T>
T rd(const uint8_t *p) {
    T v;
    std::memcpy(&v, p, sizeof(T));
    return v;
}

bool in_range(uint64_t off, uint64_t bytes, uint64_t len) { return off <= len && bytes <= len - off; }

// Validate one chunk record [off, end) holding n_expect symbols.
int check_record(const uint8_t *b, uint64_t off, uint64_t end, uint32_t n_expect, uint64_t *n_words_out) {
    if (off % 16 || end % 16 || end < off + kRecordHeadBytes + 16) return EQ_ERR_CORRUPT;
    const uint32_t n = rd<uint32_t>(b + off);
    const uint32_t n_words = rd<uint32_t>(b + off + 4);
    const uint32_t n_present = rd<uint32_t>(b + off + 8);
    if (n != n_expect || n_present < 1 || n_present > 256) return EQ_ERR_CORRUPT;
    const uint64_t table_end = align_up(kRecordHeadBytes + 4ull * n_present, 16);
    if (off + table_end + align_up(2ull * n_words, 16) != end) return EQ_ERR_CORRUPT;
    for (uint32_t l = 0; l < kLanes; ++l)
        if (rd<uint32_t>(b + off + 16 + 4 * l) < kStateLow) return EQ_ERR_CORRUPT;
    uint32_t sum = 0;
    int prev = -1;
    for (uint32_t k = 0; k < n_present; ++k) {
        const uint32_t e = rd<uint32_t>(b + off + kRecordHeadBytes + 4 * k);
        const int sym = (int)(e & 0xFF);
        const uint32_t f = e >> 16;
        if ((e & 0xFF00u) || sym <= prev || f == 0 || f > kProbTotal) return EQ_ERR_CORRUPT;
        prev = sym;
        sum += f;
    }
    if (sum != kProbTotal) return EQ_ERR_CORRUPT;
    // a single-symbol chunk codes nothing: no words, every state at 2^16
    if (n_present == 1) {
        if (n_words) return EQ_ERR_CORRUPT;
        for (uint32_t l = 0; l < kLanes; ++l)
            if (rd<uint32_t>(b + off + 16 + 4 * l) != kStateLow) return EQ_ERR_CORRUPT;
    }
    *n_words_out = n_words;
    return EQ_OK;
}

// Validate one Huffman chunk record [off, end) holding n_expect symbols: table
// sorted by (length, symbol), lengths 1..12 forming a complete prefix code
// (Kraft sum exactly 1), or a single symbol with the empty code and no words.
int check_huffman_record(const uint8_t *b, uint64_t off, uint64_t end, uint32_t n_expect, uint64_t *n_words_out) {
    if (off % 16 || end % 16 || end < off + kHuffRecordHeadBytes + 16) return EQ_ERR_CORRUPT;
    const uint32_t n = rd<uint32_t>(b + off);
    const uint32_t n_words = rd<uint32_t>(b + off + 4);
    const uint32_t n_present = rd<uint32_t>(b + off + 8);
    if (n != n_expect || n_present < 1 || n_present > 256) return EQ_ERR_CORRUPT;
    const uint64_t table_end = align_up(kHuffRecordHeadBytes + 4ull * n_present, 16);
    if (off + table_end + align_up(2ull * n_words, 16) != end) return EQ_ERR_CORRUPT;
    uint32_t kraft = 0;
    uint32_t prev_key = 0;
    for (uint32_t k = 0; k < n_present; ++k) {
        const uint32_t e = rd<uint32_t>(b + off + kHuffRecordHeadBytes + 4 * k);
        const uint32_t len = e >> 16, key = (len << 8) | (e & 0xFFu);
        if (e & 0xFF00u) return EQ_ERR_CORRUPT;
        if (n_present == 1) {
            if (len != 0 || n_words != 0) return EQ_ERR_CORRUPT;
            continue;
        }
        if (len < 1 || len > kHuffMaxLen || (k && key <= prev_key)) return EQ_ERR_CORRUPT;
        prev_key = key;
        kraft += 1u << (kHuffMaxLen - len);
    }
    if (n_present > 1 && kraft != (1u << kHuffMaxLen)) return EQ_ERR_CORRUPT;
    *n_words_out = n_words;
    return EQ_OK;
}

int parse(const uint8_t *b, size_t len, eq_model *m) {
    if (len < kHeaderBytes || std::memcmp(b, "EQW1", 4) != 0) return EQ_ERR_CORRUPT;
    if (rd<uint32_t>(b + 4) != kVersion) return EQ_ERR_UNSUPPORTED;
    if (rd<uint32_t>(b + 8) != kHeaderBytes) return EQ_ERR_CORRUPT;
    if (rd<uint32_t>(b + 12) != kProbBits || rd<uint32_t>(b + 16) != kLanes || rd<uint32_t>(b + 20) != kGroup ||
        rd<uint32_t>(b + 24) != kChunkSyms)
        return EQ_ERR_UNSUPPORTED;
    const uint32_t n_layers = rd<uint32_t>(b + 28);
    const uint32_t n_mats = rd<uint32_t>(b + 32);
    const uint64_t dir = rd<uint64_t>(b + 40);
    if (rd<uint64_t>(b + 48) != len) return EQ_ERR_CORRUPT;
    if (!in_range(dir, (uint64_t)kDirEntryBytes * n_mats, len)) return EQ_ERR_CORRUPT;
    if (n_mats && !n_layers) return EQ_ERR_CORRUPT;

    m->n_layers = n_layers;
    m->mats.resize(n_mats);
    m->layer_first.assign(n_layers, 0);
    m->layer_count.assign(n_layers, 0);
    uint32_t prev_layer = 0, next_index = 0;
    for (uint32_t i = 0; i < n_mats; ++i) {
        const uint8_t *e = b + dir + (uint64_t)kDirEntryBytes * i;
        MatrixDesc &d = m->mats[i];
        eq_matrix_info &in = d.info;
        std::memset(&in, 0, sizeof in);
        in.layer = rd<uint32_t>(e + 0);
        in.index = rd<uint32_t>(e + 4);
        in.dtype = rd<uint32_t>(e + 8);
        in.n_chunks = rd<uint32_t>(e + 12);
        in.rows = rd<uint32_t>(e + 16);
        in.cols = rd<uint32_t>(e + 20);
        in.n_outliers = rd<uint32_t>(e + 24);
        d.chunk_index_off = rd<uint64_t>(e + 32);
        d.scales_off = rd<uint64_t>(e + 40);
        d.outliers_off = rd<uint64_t>(e + 48);
        d.codec = rd<uint32_t>(e + 28);
        in.codec = d.codec;
        if (d.codec != kCodecRans && d.codec != kCodecHuffman) return EQ_ERR_UNSUPPORTED;
        if (in.dtype != EQ_INT8 && in.dtype != EQ_E4M3) return EQ_ERR_CORRUPT;
        if (in.layer >= n_layers || in.layer < prev_layer) return EQ_ERR_CORRUPT;
        if (in.layer != prev_layer || i == 0) next_index = 0;
        if (in.index != next_index++) return EQ_ERR_CORRUPT;
        if (m->layer_count[in.layer] == 0) m->layer_first[in.layer] = i;
        m->layer_count[in.layer]++;
        prev_layer = in.layer;

        const uint64_t n = (uint64_t)in.rows * in.cols;
        if (in.n_chunks != (n + kChunkSyms - 1) / kChunkSyms) return EQ_ERR_CORRUPT;
        if (!in_range(d.chunk_index_off, 8ull * (in.n_chunks + 1), len) || d.chunk_index_off % 8) return EQ_ERR_CORRUPT;
        if (!in_range(d.scales_off, 4ull * in.rows, len) || d.scales_off % 4) return EQ_ERR_CORRUPT;
        if (in.n_outliers) {
            if (!in_range(d.outliers_off, 12ull * in.n_outliers, len) || d.outliers_off % 4) return EQ_ERR_CORRUPT;
            uint64_t prev = 0;
            for (uint32_t k = 0; k < in.n_outliers; ++k) {
                const uint32_t r = rd<uint32_t>(b + d.outliers_off + 12ull * k);
                const uint32_t c = rd<uint32_t>(b + d.outliers_off + 12ull * k + 4);
                if (r >= in.rows || c >= in.cols) return EQ_ERR_CORRUPT;
                const uint64_t lin = (uint64_t)r * in.cols + c;
                if (k && lin <= prev) return EQ_ERR_CORRUPT;
                prev = lin;
            }
        }
        uint64_t words = 0;
        const uint64_t first = rd<uint64_t>(b + d.chunk_index_off);
        in.uniform_table = in.n_chunks > 0;
        uint32_t np0 = 0;
        for (uint32_t k = 0; k < in.n_chunks; ++k) {
            const uint64_t off = rd<uint64_t>(b + d.chunk_index_off + 8ull * k);
            const uint64_t end = rd<uint64_t>(b + d.chunk_index_off + 8ull * (k + 1));
            if (end <= off || end > len) return EQ_ERR_CORRUPT;
            const uint64_t rem = n - (uint64_t)k * kChunkSyms;
            const uint32_t n_expect = (uint32_t)(rem < kChunkSyms ? rem : kChunkSyms);
            uint64_t nw = 0;
            int rc = d.codec == kCodecHuffman ? check_huffman_record(b, off, end, n_expect, &nw)
                                              : check_record(b, off, end, n_expect, &nw);
            if (rc) return rc;
            words += nw;
            // does every chunk carry the first chunk's table?
            const uint32_t np = rd<uint32_t>(b + off + 8);
            if (k == 0) {
                np0 = np;
                d.n_present0 = np;
            } else if (in.uniform_table) {
                const uint64_t off0 = rd<uint64_t>(b + d.chunk_index_off);
                const uint32_t hb = record_head_bytes(d.codec);
                if (np != np0 || std::memcmp(b + off + hb, b + off0 + hb, 4ull * np) != 0)
                    in.uniform_table = 0;
            }
        }
        d.small_scales = true;
        for (uint32_t r = 0; r < in.rows; ++r) {
            const float v = rd<float>(b + d.scales_off + 4ull * r);
            if (!(v > -256.f && v < 256.f)) d.small_scales = false;  // also false for NaN
        }
        in.payload_words = words;
        in.compressed_bytes = rd<uint64_t>(b + d.chunk_index_off + 8ull * in.n_chunks) - first;
    }
    for (uint32_t l = 0; l < n_layers; ++l)
        if (!m->layer_count[l]) return EQ_ERR_CORRUPT;
    return EQ_OK;
}

}  // namespace

extern "C" EQW_API int eq_model_open(const void *d_blob, size_t len, const void *h_blob, eq_model **out) {
    if (!out) return EQ_ERR_INVALID_ARG;
    *out = nullptr;
    if (!d_blob || !h_blob || len < kHeaderBytes) return EQ_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(d_blob) % kSectionAlign) return EQ_ERR_INVALID_ARG;
    auto *m = new (std::nothrow) eq_model;
    if (!m) return EQ_ERR_NOSPACE;
    m->d_blob = static_cast<const uint8_t *>(d_blob);
    m->len = len;
    int rc;
    try {
        rc = parse(static_cast<const uint8_t *>(h_blob), len, m);
    } catch (...) {
        rc = EQ_ERR_NOSPACE;
    }
    if (rc) {
        delete m;
        return rc;
    }
    *out = m;
    return EQ_OK;
}

extern "C" EQW_API void eq_model_close(eq_model *m) { delete m; }

extern "C" EQW_API int eq_model_set_sm_limit(eq_model *m, uint32_t max_sms) {
    if (!m) return EQ_ERR_INVALID_ARG;
    m->sm_limit = max_sms;
    return EQ_OK;
}

extern "C" EQW_API int eq_model_counts(const eq_model *m, uint32_t *n_layers, uint32_t *n_matrices) {
    if (!m) return EQ_ERR_INVALID_ARG;
    if (n_layers) *n_layers = m->n_layers;
    if (n_matrices) *n_matrices = (uint32_t)m->mats.size();
    return EQ_OK;
}

extern "C" EQW_API int eq_matrix_get_info(const eq_model *m, uint32_t matrix, eq_matrix_info *info) {
    if (!m || !info || matrix >= m->mats.size()) return EQ_ERR_INVALID_ARG;
    *info = m->mats[matrix].info;
    return EQ_OK;
}

extern "C" EQW_API int eq_layer_matrices(const eq_model *m, uint32_t layer, uint32_t *first, uint32_t *count) {
    if (!m || !first || !count || layer >= m->n_layers) return EQ_ERR_INVALID_ARG;
    *first = m->layer_first[layer];
    *count = m->layer_count[layer];
    return EQ_OK;
}

extern "C" EQW_API int eq_block_layout(const eq_model *m, uint32_t layer, size_t *offsets, uint32_t cap,
                                       size_t *total_bytes) {
    if (!m || !total_bytes || layer >= m->n_layers || (cap && !offsets)) return EQ_ERR_INVALID_ARG;
    uint64_t pos = 0;
    const uint32_t first = m->layer_first[layer], count = m->layer_count[layer];
    for (uint32_t i = 0; i < count; ++i) {
        if (i < cap) offsets[i] = pos;
        const eq_matrix_info &in = m->mats[first + i].info;
        pos = align_up(pos + 2ull * in.rows * in.cols, kSectionAlign);
    }
    *total_bytes = pos;
    return EQ_OK;
}

extern "C" EQW_API const char *eq_status_string(int status) {
    switch (status) {
        case EQ_OK: return "ok";
        case EQ_ERR_INVALID_ARG: return "invalid argument";
        case EQ_ERR_CORRUPT: return "corrupt container";
        case EQ_ERR_UNSUPPORTED: return "unsupported container version or constants";
        case EQ_ERR_CUDA: return "CUDA runtime error";
        case EQ_ERR_TIMEOUT: return "timed out";
        case EQ_ERR_NOSPACE: return "output buffer too small";
        default: return "unknown status";
    }
}

extern "C" EQW_API int eq_format_version(void) { return (int)kVersion; }
