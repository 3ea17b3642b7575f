/*
 * CPU oracle, Huffman codec -- TEST INFRASTRUCTURE ONLY (same rules as
 * rans_oracle.c: only the tests, __graft_entry__.smoke() and bench.py's
 * CPU-baseline leg load it; it shares nothing with the product).
 *
 * EntroLLM technical overview (gist.science 2505.02380), "method" items 2 and
 * 3: the quantised weights are Huffman coded (short variable-length codes for
 * frequent values, long ones for rare values) and the coded parameter space
 * is cut into chunks that keep the tensor structure and decode concurrently.
 * The page fixes no code construction, bit order or chunk format; the
 * readings taken here (and by the product) are:
 *
 *   code lengths   optimal lengths under a maximum of 12 bits, computed by
 *                  the package-merge algorithm (Larmore and Hirschberg, "A
 *                  fast algorithm for optimal length-limited Huffman codes",
 *                  1990); a chunk with a single distinct symbol has the empty
 *                  code (length 0, no payload)
 *   codes          canonical: symbols ordered by (length, symbol value) get
 *                  consecutive codes, each code one more than the previous
 *                  and shifted left by the length difference (the canonical
 *                  construction DEFLATE uses, RFC 1951 section 3.2.2)
 *   interleaving   the rANS chunk layout: 32 lanes, symbol j of a chunk in
 *                  lane (j mod 256) div 8 at step 8 (j div 256) + j mod 8; a
 *                  lane's bit stream is the concatenation of its symbols'
 *                  codes in step order, most significant bit first
 *   words          16-bit; before decoding a symbol a lane that holds fewer
 *                  than 12 unread bits takes the next 16 bits of its stream
 *                  (zero-padded past its end); within a step the words are
 *                  stored in ascending lane order, steps in ascending order
 *   end            every word consumed and every bit a lane still holds zero
 *
 * The decoder below reads one bit at a time and matches canonical code
 * ranges length by length (first code and count per length), with no table.
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <stdlib.h>

#define HUF_OK 0
#define HUF_ERR_ARG 1
#define HUF_ERR_CORRUPT 2
#define HUF_ERR_SPACE 3

#define HUF_MAX_LEN 12u
#define HUF_LANES 32u
#define HUF_GROUP 8u
#define HUF_GROUP_SYMS 256u

/* ---- lengths: package-merge -------------------------------------------------
 * Items are (weight, count vector over the 256 symbols).  Level by level, the
 * list is the sorted leaves merged with the pairs ("packages") of the previous
 * level's list; the first 2n - 2 items of the last list give each symbol's
 * length as the number of items it occurs in. */
typedef struct {
    uint64_t w;
    uint16_t cnt[256];
} huf_item;

int orc_huff_lengths(const uint64_t counts[256], uint8_t len[256]) {
    int sym[256];
    int n = 0;
    for (int s = 0; s < 256; ++s) {
        len[s] = 0;
        if (counts[s]) sym[n++] = s;
    }
    if (n == 0) return HUF_ERR_ARG;
    if (n == 1) return HUF_OK; /* empty code */
    huf_item *leaves = calloc((size_t)n, sizeof(huf_item));
    huf_item *list = calloc((size_t)2 * n, sizeof(huf_item));
    huf_item *next = calloc((size_t)2 * n, sizeof(huf_item));
    if (!leaves || !list || !next) {
        free(leaves); free(list); free(next);
        return HUF_ERR_SPACE;
    }
    for (int i = 0; i < n; ++i) {
        leaves[i].w = counts[sym[i]];
        leaves[i].cnt[sym[i]] = 1;
    }
    /* stable order of equal weights: by symbol value (sym[] is ascending) */
    for (int i = 1; i < n; ++i)
        for (int j = i; j > 0 && leaves[j - 1].w > leaves[j].w; --j) {
            huf_item t = leaves[j]; leaves[j] = leaves[j - 1]; leaves[j - 1] = t;
        }
    int m = n;
    memcpy(list, leaves, sizeof(huf_item) * n);
    for (unsigned level = 1; level < HUF_MAX_LEN; ++level) {
        /* packages of adjacent pairs of the current list */
        int p = 0;
        for (int i = 0; i + 1 < m; i += 2, ++p) {
            next[p].w = list[i].w + list[i + 1].w;
            for (int s = 0; s < 256; ++s) next[p].cnt[s] = (uint16_t)(list[i].cnt[s] + list[i + 1].cnt[s]);
        }
        /* merge leaves and packages by weight, leaves first on ties */
        huf_item *merged = calloc((size_t)(n + p), sizeof(huf_item));
        if (!merged) {
            free(leaves); free(list); free(next);
            return HUF_ERR_SPACE;
        }
        int a = 0, b = 0, k = 0;
        while (a < n || b < p) {
            if (b >= p || (a < n && leaves[a].w <= next[b].w)) merged[k++] = leaves[a++];
            else merged[k++] = next[b++];
        }
        m = k < 2 * n ? k : 2 * n;
        memcpy(list, merged, sizeof(huf_item) * m);
        free(merged);
    }
    for (int i = 0; i < 2 * n - 2; ++i)
        for (int s = 0; s < 256; ++s) len[s] = (uint8_t)(len[s] + list[i].cnt[s]);
    free(leaves); free(list); free(next);
    return HUF_OK;
}

/* ---- canonical codes ----------------------------------------------------------- */
/* code[s] for every symbol with len[s] > 0; returns 0 if the lengths are not a
 * complete prefix code of at most 12 bits (or a single length-0 symbol). */
int orc_huff_canonical(const uint8_t len[256], uint16_t code[256]) {
    unsigned n = 0;
    uint64_t kraft = 0; /* sum of 2^(12 - len) */
    for (int s = 0; s < 256; ++s) {
        code[s] = 0;
        if (!len[s]) continue;
        if (len[s] > HUF_MAX_LEN) return 0;
        kraft += 1u << (HUF_MAX_LEN - len[s]);
        ++n;
    }
    if (n == 0) return 1; /* the single-symbol chunk: nothing to assign */
    if (kraft != (1u << HUF_MAX_LEN)) return 0;
    uint32_t c = 0;
    unsigned prev_len = 0;
    for (unsigned L = 1; L <= HUF_MAX_LEN; ++L)
        for (int s = 0; s < 256; ++s) {
            if (len[s] != L) continue;
            if (prev_len) c = (c + 1) << (L - prev_len);
            else c = 0;
            prev_len = L;
            code[s] = (uint16_t)c;
        }
    return 1;
}

static uint32_t huf_symbol_index(uint32_t step, uint32_t lane) {
    return HUF_GROUP_SYMS * (step / HUF_GROUP) + HUF_GROUP * lane + step % HUF_GROUP;
}

/* ---- encode one chunk ---------------------------------------------------------------
 * len[]: the chunk's code lengths (present symbols > 0, or exactly one symbol
 * with the empty code).  Writes n_words words. */
int orc_huff_encode_chunk(const uint8_t *sym, uint32_t n, const uint8_t len[256], int single_symbol,
                          uint16_t *words, uint32_t cap, uint32_t *n_words) {
    uint16_t code[256];
    *n_words = 0;
    if (single_symbol) {
        for (uint32_t j = 0; j < n; ++j)
            if (sym[j] != sym[0]) return HUF_ERR_ARG;
        return HUF_OK;
    }
    if (!orc_huff_canonical(len, code)) return HUF_ERR_ARG;
    for (uint32_t j = 0; j < n; ++j)
        if (!len[sym[j]]) return HUF_ERR_ARG;
    const uint32_t T = HUF_GROUP * ((n + HUF_GROUP_SYMS - 1) / HUF_GROUP_SYMS);
    /* each lane's bit stream, one byte per bit */
    uint8_t *bits[HUF_LANES];
    uint32_t nbits[HUF_LANES], taken[HUF_LANES], held[HUF_LANES];
    for (uint32_t l = 0; l < HUF_LANES; ++l) {
        bits[l] = malloc((size_t)(T + 1) * HUF_MAX_LEN + 32);
        if (!bits[l]) {
            for (uint32_t k = 0; k < l; ++k) free(bits[k]);
            return HUF_ERR_SPACE;
        }
        nbits[l] = taken[l] = held[l] = 0;
    }
    for (uint32_t t = 0; t < T; ++t)
        for (uint32_t l = 0; l < HUF_LANES; ++l) {
            const uint32_t j = huf_symbol_index(t, l);
            if (j >= n) continue;
            const unsigned L = len[sym[j]];
            for (unsigned b = 0; b < L; ++b) bits[l][nbits[l]++] = (uint8_t)((code[sym[j]] >> (L - 1 - b)) & 1u);
        }
    /* walk the decoder's schedule: refills in (step, lane) order */
    int rc = HUF_OK;
    for (uint32_t t = 0; t < T && rc == HUF_OK; ++t)
        for (uint32_t l = 0; l < HUF_LANES; ++l) {
            const uint32_t j = huf_symbol_index(t, l);
            if (j >= n) continue;
            if (held[l] < HUF_MAX_LEN) {
                uint32_t w = 0;
                for (unsigned b = 0; b < 16; ++b) {
                    const uint32_t at = taken[l] + b;
                    w = (w << 1) | (at < nbits[l] ? bits[l][at] : 0u);
                }
                if (*n_words >= cap) {
                    rc = HUF_ERR_SPACE;
                    break;
                }
                words[(*n_words)++] = (uint16_t)w;
                taken[l] += 16;
                held[l] += 16;
            }
            held[l] -= len[sym[j]];
        }
    for (uint32_t l = 0; l < HUF_LANES; ++l) free(bits[l]);
    return rc;
}

/* ---- decode one chunk ------------------------------------------------------------------ */
int orc_huff_decode_chunk(const uint16_t *words, uint32_t n_words, const uint8_t len[256], int single_symbol,
                          uint8_t single, uint32_t n, uint8_t *out) {
    if (single_symbol) {
        if (n_words) return HUF_ERR_CORRUPT;
        for (uint32_t j = 0; j < n; ++j) out[j] = single;
        return HUF_OK;
    }
    uint16_t code[256];
    if (!orc_huff_canonical(len, code)) return HUF_ERR_CORRUPT;
    /* per length: the first canonical code and the symbols in canonical order */
    uint32_t first[HUF_MAX_LEN + 2], count[HUF_MAX_LEN + 2], offset[HUF_MAX_LEN + 2];
    uint8_t order[256];
    unsigned k = 0;
    for (unsigned L = 1; L <= HUF_MAX_LEN; ++L) {
        offset[L] = k;
        count[L] = 0;
        first[L] = 0;
        for (int s = 0; s < 256; ++s)
            if (len[s] == L) {
                if (!count[L]) first[L] = code[s];
                ++count[L];
                order[k++] = (uint8_t)s;
            }
    }
    /* each lane's queue of buffered bits (at most 27 at a time) */
    uint8_t q[HUF_LANES][64];
    uint32_t head[HUF_LANES], held[HUF_LANES];
    for (uint32_t l = 0; l < HUF_LANES; ++l) head[l] = held[l] = 0;
    uint32_t p = 0;
    const uint32_t T = HUF_GROUP * ((n + HUF_GROUP_SYMS - 1) / HUF_GROUP_SYMS);
    for (uint32_t t = 0; t < T; ++t)
        for (uint32_t l = 0; l < HUF_LANES; ++l) {
            const uint32_t j = huf_symbol_index(t, l);
            if (j >= n) continue;
            if (held[l] < HUF_MAX_LEN) {
                if (p >= n_words) return HUF_ERR_CORRUPT;
                const uint32_t w = words[p++];
                for (unsigned b = 0; b < 16; ++b) q[l][(head[l] + held[l] + b) % 64] = (uint8_t)((w >> (15 - b)) & 1u);
                held[l] += 16;
            }
            uint32_t c = 0;
            int found = -1;
            for (unsigned L = 1; L <= HUF_MAX_LEN && found < 0; ++L) {
                if (held[l] < L) return HUF_ERR_CORRUPT;
                c = (c << 1) | q[l][(head[l] + L - 1) % 64];
                if (count[L] && c >= first[L] && c - first[L] < count[L]) {
                    found = order[offset[L] + c - first[L]];
                    head[l] = (head[l] + L) % 64;
                    held[l] -= L;
                }
            }
            if (found < 0) return HUF_ERR_CORRUPT;
            out[j] = (uint8_t)found;
        }
    if (p != n_words) return HUF_ERR_CORRUPT;
    for (uint32_t l = 0; l < HUF_LANES; ++l)
        for (uint32_t b = 0; b < held[l]; ++b)
            if (q[l][(head[l] + b) % 64]) return HUF_ERR_CORRUPT;
    return HUF_OK;
}
