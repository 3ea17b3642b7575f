// Host-side pieces shared by the two encoders of container v1: eq_encode_host
// (eqw_encode.cpp, symbols in host memory) and eq_encode_device
// (eqw_encode_device.cu, symbols in device memory).  Both quantise frequency
// tables with the same routine and lay out the container with the same plan,
// so for the same inputs they write the same bytes.
//
// EntQuant technical summary (gist.science 2601.22787), section 2 "weight
// encoding": the quantised weights are flattened into a symbol stream and
// compressed losslessly; storage = bitstream + scales + metadata.
#pragma once

#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "eqw_internal.h"

namespace eqw {

// Frequency table from a histogram: the proportional share rounded to nearest
// (at least 1 for every present symbol), then single units moved greedily
// where they cost the fewest expected bits: adding one unit to s saves
// cnt_s * log2((f+1)/f) bits, removing one costs cnt_s * log2(f/(f-1)).
inline void quantize_table(const uint64_t cnt[256], uint64_t n, uint32_t f[256]) {
    int present[256];
    int np = 0;
    int64_t sum = 0;
    for (int s = 0; s < 256; ++s) {
        f[s] = 0;
        if (!cnt[s]) continue;
        present[np++] = s;
        uint64_t q = ((uint64_t)cnt[s] * kProbTotal + n / 2) / n;
        f[s] = q ? (uint32_t)q : 1u;
        sum += f[s];
    }
    while (sum < (int64_t)kProbTotal) {
        int best = -1;
        double gain = -1.0;
        for (int i = 0; i < np; ++i) {
            int s = present[i];
            double g = cnt[s] * std::log2((f[s] + 1.0) / f[s]);
            if (g > gain) { gain = g; best = s; }
        }
        f[best] += 1;
        ++sum;
    }
    while (sum > (int64_t)kProbTotal) {
        int best = -1;
        double loss = 0.0;
        for (int i = 0; i < np; ++i) {
            int s = present[i];
            if (f[s] <= 1) continue;
            double l = cnt[s] * std::log2((double)f[s] / (f[s] - 1.0));
            if (best < 0 || l < loss) { loss = l; best = s; }
        }
        f[best] -= 1;
        --sum;
    }
}

// ---- Huffman codec (EntroLLM technical overview, "Huffman weight encoding") -----
// Code lengths: Huffman's construction (repeatedly merge the two lightest
// nodes; ties by creation order, leaves in symbol order first), then, if a
// code exceeds 12 bits, the length adjustment of the JPEG standard (ITU-T
// T.81 Annex K.3, "Adjust_BITS"): two codes of the longest length i give way
// to one code of length i-1, and one code of the deepest shorter length j
// becomes two codes of length j+1, which keeps the Kraft sum at 1.  The
// lengths are then handed out shortest first to the most frequent symbols.
// One distinct symbol: the empty code (all lengths 0).
inline void huffman_lengths(const uint64_t cnt[256], uint8_t len[256]) {
    std::memset(len, 0, 256);
    struct Node {
        uint64_t w;
        int left, right;
    };
    std::vector<Node> nodes;
    std::vector<int> sym_node(256, -1);
    for (int s = 0; s < 256; ++s)
        if (cnt[s]) {
            sym_node[s] = (int)nodes.size();
            nodes.push_back({cnt[s], -1, -1});
        }
    const int n = (int)nodes.size();
    if (n < 2) return;
    // min-heap on (weight, node index)
    auto heavier = [&](int a, int b) { return nodes[a].w != nodes[b].w ? nodes[a].w > nodes[b].w : a > b; };
    std::vector<int> heap;
    for (int i = 0; i < n; ++i) heap.push_back(i);
    std::make_heap(heap.begin(), heap.end(), heavier);
    while (heap.size() > 1) {
        std::pop_heap(heap.begin(), heap.end(), heavier);
        const int a = heap.back();
        heap.pop_back();
        std::pop_heap(heap.begin(), heap.end(), heavier);
        const int b = heap.back();
        heap.pop_back();
        nodes.push_back({nodes[a].w + nodes[b].w, a, b});
        heap.push_back((int)nodes.size() - 1);
        std::push_heap(heap.begin(), heap.end(), heavier);
    }
    // depth of every leaf
    std::vector<int> depth(nodes.size(), 0);
    for (int i = (int)nodes.size() - 1; i >= n; --i) {
        depth[nodes[i].left] = depth[i] + 1;
        depth[nodes[i].right] = depth[i] + 1;
    }
    std::vector<uint32_t> bits(258, 0);  // bits[l] = number of codes of length l
    int max_len = 0;
    for (int i = 0; i < n; ++i) {
        ++bits[depth[i]];
        max_len = std::max(max_len, depth[i]);
    }
    for (int i = max_len; i > (int)kHuffMaxLen; --i) {
        while (bits[i] > 0) {
            int j = i - 2;
            while (bits[j] == 0) --j;
            bits[i] -= 2;
            bits[i - 1] += 1;
            bits[j + 1] += 2;
            bits[j] -= 1;
        }
    }
    // shortest codes to the most frequent symbols (ties: smaller symbol first)
    std::vector<int> order;
    for (int s = 0; s < 256; ++s)
        if (cnt[s]) order.push_back(s);
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cnt[a] > cnt[b]; });
    size_t k = 0;
    for (uint32_t l = 1; l <= kHuffMaxLen; ++l)
        for (uint32_t c = 0; c < bits[l]; ++c) len[order[k++]] = (uint8_t)l;
}

// Canonical codes from lengths (RFC 1951 section 3.2.2): codes of one length
// are consecutive in symbol order, and each length's first code follows the
// previous length's last code shifted left by the difference in length.
inline void huffman_codes(const uint8_t len[256], uint16_t code[256]) {
    uint32_t c = 0, prev_len = 0;
    for (int s = 0; s < 256; ++s) code[s] = 0;
    for (uint32_t l = 1; l <= kHuffMaxLen; ++l)
        for (int s = 0; s < 256; ++s) {
            if (len[s] != l) continue;
            c = prev_len ? (c + 1) << (l - prev_len) : 0u;
            prev_len = l;
            code[s] = (uint16_t)c;
        }
}

// Byte size of a chunk record with n_present table entries and n_words words.
inline uint64_t record_bytes(uint32_t n_present, uint32_t n_words, uint32_t codec = kCodecRans) {
    return align_up(record_head_bytes(codec) + 4ull * n_present, 16) + align_up(2ull * n_words, 16);
}

// Where everything goes.  Directory order: by layer, input order inside a layer.
struct ContainerPlan {
    struct Place {
        uint64_t ci, so, oo, rec0;  // chunk index, scales, outliers (0 if none), first record
    };
    uint32_t n_layers = 0;
    std::vector<uint32_t> order;     // directory position -> input index
    std::vector<uint32_t> n_chunks;  // per directory position
    std::vector<uint32_t> first_job; // per directory position: its first chunk in job order
    uint32_t n_jobs = 0;             // chunks of all matrices, directory order
    std::vector<Place> place;
    std::vector<uint64_t> rec_off;   // per job; rec_off[n_jobs] unused
    std::vector<uint64_t> rec_end;   // per directory position: end of its last record
    uint64_t total = 0;
};

// Order and chunk counts (needs only shapes and layers; n_layers from the caller's validation).
inline void plan_order(const eq_matrix_in *mats, uint32_t n_mats, uint32_t n_layers, ContainerPlan &P) {
    P.n_layers = n_layers;
    P.order.resize(n_mats);
    for (uint32_t i = 0; i < n_mats; ++i) P.order[i] = i;
    std::stable_sort(P.order.begin(), P.order.end(),
                     [&](uint32_t a, uint32_t b) { return mats[a].layer < mats[b].layer; });
    P.n_chunks.resize(n_mats);
    P.first_job.resize(n_mats);
    P.n_jobs = 0;
    for (uint32_t d = 0; d < n_mats; ++d) {
        const eq_matrix_in &m = mats[P.order[d]];
        const uint64_t n = (uint64_t)m.rows * m.cols;
        P.n_chunks[d] = (uint32_t)((n + kChunkSyms - 1) / kChunkSyms);
        P.first_job[d] = P.n_jobs;
        P.n_jobs += P.n_chunks[d];
    }
}

// Offsets once every record's size is known (rec_size per job, directory order):
// header | directory | per matrix: chunk index, scales, outliers, records.
inline void plan_offsets(const eq_matrix_in *mats, const std::vector<uint64_t> &rec_size, ContainerPlan &P) {
    const uint32_t n_mats = (uint32_t)P.order.size();
    uint64_t pos = align_up(kHeaderBytes + (uint64_t)kDirEntryBytes * n_mats, kSectionAlign);
    P.place.resize(n_mats);
    P.rec_off.assign(P.n_jobs + 1, 0);
    P.rec_end.resize(n_mats);
    uint32_t j = 0;
    for (uint32_t d = 0; d < n_mats; ++d) {
        const eq_matrix_in &m = mats[P.order[d]];
        ContainerPlan::Place &pl = P.place[d];
        pl.ci = pos;
        pos = align_up(pos + 8ull * (P.n_chunks[d] + 1), kSectionAlign);
        pl.so = pos;
        pos = align_up(pos + 4ull * m.rows, kSectionAlign);
        pl.oo = 0;
        if (m.n_out) {
            pl.oo = pos;
            pos = align_up(pos + 12ull * m.n_out, kSectionAlign);
        }
        pl.rec0 = pos;
        for (uint32_t k = 0; k < P.n_chunks[d]; ++k, ++j) {
            P.rec_off[j] = pos;
            pos += rec_size[j];
        }
        P.rec_end[d] = pos;
        pos = align_up(pos, kSectionAlign);
    }
    P.total = pos;
}

inline void put32(uint8_t *p, uint32_t v) { std::memcpy(p, &v, 4); }
inline void put64(uint8_t *p, uint64_t v) { std::memcpy(p, &v, 8); }

// Header and directory: bytes [0, kHeaderBytes + 64 * n_mats) of the container.
inline void write_header_directory(uint8_t *b, const eq_matrix_in *mats, const ContainerPlan &P) {
    const uint32_t n_mats = (uint32_t)P.order.size();
    std::memcpy(b, "EQW1", 4);
    put32(b + 4, kVersion);
    put32(b + 8, kHeaderBytes);
    put32(b + 12, kProbBits);
    put32(b + 16, kLanes);
    put32(b + 20, kGroup);
    put32(b + 24, kChunkSyms);
    put32(b + 28, P.n_layers);
    put32(b + 32, n_mats);
    put64(b + 40, kHeaderBytes);
    put64(b + 48, P.total);
    std::vector<uint32_t> index_in_layer(P.n_layers, 0);
    for (uint32_t d = 0; d < n_mats; ++d) {
        const eq_matrix_in &m = mats[P.order[d]];
        const ContainerPlan::Place &pl = P.place[d];
        uint8_t *e = b + kHeaderBytes + (uint64_t)kDirEntryBytes * d;
        put32(e + 0, m.layer);
        put32(e + 4, index_in_layer[m.layer]++);
        put32(e + 8, m.dtype);
        put32(e + 12, P.n_chunks[d]);
        put32(e + 16, m.rows);
        put32(e + 20, m.cols);
        put32(e + 24, m.n_out);
        put32(e + 28, (m.flags & EQ_CODEC_HUFFMAN) ? kCodecHuffman : kCodecRans);
        put64(e + 32, pl.ci);
        put64(e + 40, pl.so);
        put64(e + 48, pl.oo);
    }
}

// Chunk index of directory position d (8 * (n_chunks + 1) bytes at dst).
inline void write_chunk_index(uint8_t *dst, const ContainerPlan &P, uint32_t d) {
    const uint32_t j0 = P.first_job[d];
    for (uint32_t k = 0; k < P.n_chunks[d]; ++k) put64(dst + 8ull * k, P.rec_off[j0 + k]);
    put64(dst + 8ull * P.n_chunks[d], P.n_chunks[d] ? P.rec_end[d] : P.place[d].rec0);
}

// Outlier records {row, col, value} from host arrays (12 * n_out bytes at dst).
inline void write_outliers(uint8_t *dst, uint32_t n_out, const uint32_t *row, const uint32_t *col, const float *val) {
    for (uint32_t k = 0; k < n_out; ++k) {
        put32(dst + 12ull * k, row[k]);
        put32(dst + 12ull * k + 4, col[k]);
        std::memcpy(dst + 12ull * k + 8, &val[k], 4);
    }
}

// Checks of outliers against the shape: in range, strictly ascending linear index.
inline bool outliers_valid(uint32_t rows, uint32_t cols, uint32_t n_out, const uint32_t *row, const uint32_t *col) {
    uint64_t prev = 0;
    for (uint32_t k = 0; k < n_out; ++k) {
        if (row[k] >= rows || col[k] >= cols) return false;
        const uint64_t lin = (uint64_t)row[k] * cols + col[k];
        if (k && lin <= prev) return false;
        prev = lin;
    }
    return true;
}

// Shape, dtype, flag and layer checks shared by both encoders (no data access).
// On success *n_layers = max layer + 1 (layers must be 0..n-1).
inline int validate_shapes(const eq_matrix_in *mats, uint32_t n_mats, uint32_t *n_layers) {
    if (!mats && n_mats) return EQ_ERR_INVALID_ARG;
    uint32_t max_layer = 0;
    for (uint32_t i = 0; i < n_mats; ++i) {
        const eq_matrix_in &m = mats[i];
        if (m.dtype != EQ_INT8 && m.dtype != EQ_E4M3) return EQ_ERR_INVALID_ARG;
        if (m.flags & ~(EQ_TABLE_PER_CHUNK | EQ_CODEC_HUFFMAN)) return EQ_ERR_INVALID_ARG;
        const uint64_t n = (uint64_t)m.rows * m.cols;
        if (n && (!m.symbols || !m.scales)) return EQ_ERR_INVALID_ARG;
        if ((n + kChunkSyms - 1) / kChunkSyms > 0xFFFFFFFFull) return EQ_ERR_INVALID_ARG;
        if (m.n_out && (!m.out_row || !m.out_col || !m.out_val)) return EQ_ERR_INVALID_ARG;
        max_layer = std::max(max_layer, m.layer);
    }
    if (n_mats) {
        std::vector<char> seen(max_layer + 1, 0);
        for (uint32_t i = 0; i < n_mats; ++i) seen[mats[i].layer] = 1;
        for (char s : seen)
            if (!s) return EQ_ERR_INVALID_ARG;
        *n_layers = max_layer + 1;
    } else {
        *n_layers = 0;
    }
    return EQ_OK;
}

}  // namespace eqw
