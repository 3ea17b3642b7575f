/*
 * CPU oracle for entropy-coded weight decode -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
 * load this file's library.  The product (the CUDA path and its C-ABI
 * library) never includes, links or calls it, and it includes nothing of the
 * product.  It is written to be read against the method's definition, not to
 * be fast: plain loops, one symbol at a time, exact arithmetic.
 *
 * What it computes (EntQuant technical summary, gist.science 2601.22787,
 * section 2 "weight encoding" and "inference-time decoding"): Int8 / Float8
 * weight symbols are flattened into a symbol stream and compressed losslessly
 * with an ANS coder; at inference a parallel ANS decoder expands them into a
 * weight buffer.  The pages fix neither the ANS variant nor its parameters;
 * this oracle follows the plainest reading, which is the rANS coder of Duda
 * ("Asymmetric numeral systems", 2013) with several interleaved states
 * (Giesen, "Interleaved entropy coders", 2014):
 *
 *   probability precision  M = 2^12 (frequencies f_s sum to 4096)
 *   state                  32-bit, normalised interval [2^16, 2^32)
 *   renormalisation        16-bit words
 *   interleaving           32 states ("lanes") per chunk
 *   chunk                  up to 65536 symbols; chunks are independent, as in
 *                          EntroLLM's parallel decoding (EntroLLM technical
 *                          overview, "parallel decoding strategy")
 *
 * Lane / step assignment inside a chunk of n symbols: symbol j is handled by
 *   lane(j) = (j mod 256) div 8,   step(j) = 8 * (j div 256) + (j mod 8)
 * i.e. within every 256-symbol group each lane owns 8 consecutive symbols.
 * A decoder visits steps t = 0 .. T-1 (T = 8 * ceil(n / 256)) and, inside a
 * step, lanes 0..31 in ascending order; a lane whose symbol index is >= n is
 * idle at that step.  The encoder visits the same positions in exactly the
 * reverse order.
 *
 * Dequantisation (EntQuant: per-channel scales S, Int8 / Float8 base formats):
 *   out[i] = bf16_rne( fp32_rn( value(sym[i]) * scale[row(i)] ) )
 * followed by the super-weight scatter out[r*cols+c] = bf16_rne(v).
 *
 * Parity pins for every function here live in tests/ (round trip, brute
 * force on tiny alphabets, the rANS ideal-code-length identity, the Shannon
 * size bound, library routines for the number formats).
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <stdlib.h>
#include <math.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_CORRUPT 2
#define ORC_ERR_SPACE 3

#define PROB_BITS 12
#define PROB_TOTAL 4096u          /* M */
#define STATE_LOW 65536u          /* L = 2^16, lower end of the state interval */
#define LANES 32u
#define GROUP 8u                  /* consecutive symbols a lane owns per group */
#define GROUP_SYMS (LANES * GROUP) /* 256 */

/* Symbol index handled by lane `lane` at step `step` (see header). */
static uint32_t symbol_index(uint32_t step, uint32_t lane)
{
    return GROUP_SYMS * (step / GROUP) + GROUP * lane + (step % GROUP);
}

static uint32_t n_steps(uint32_t n)
{
    return GROUP * ((n + GROUP_SYMS - 1) / GROUP_SYMS);
}

/* ------------------------------------------------------------------------ */
/* frequency table                                                          */
/* ------------------------------------------------------------------------ */

/*
 * Quantise a byte histogram to frequencies summing to M = 4096.
 * f_s = max(1, floor(c_s * 4096 / n + 1/2)) for every present symbol, 0
 * otherwise; the difference to 4096 goes to the symbol with the largest f
 * (smallest byte on ties); if that would leave it below 1, take 1 at a time
 * from the largest f > 1 instead.  Any table with sum 4096 and f_s >= 1 for
 * every present symbol decodes correctly; only the compressed size depends
 * on this choice.
 */
int orc_quantize_freqs(const uint64_t counts[256], uint32_t f[256])
{
    uint64_t n = 0;
    for (int s = 0; s < 256; s++) n += counts[s];
    if (n == 0) return ORC_ERR_ARG;
    int64_t sum = 0;
    for (int s = 0; s < 256; s++) {
        if (counts[s] == 0) { f[s] = 0; continue; }
        /* floor(c * 4096 / n + 1/2) == floor((2 * c * 4096 + n) / (2 n)) */
        uint64_t q = (2u * counts[s] * PROB_TOTAL + n) / (2u * n);
        f[s] = q < 1 ? 1u : (uint32_t)q;
        sum += f[s];
    }
    int64_t d = (int64_t)PROB_TOTAL - sum;
    int best = 0;
    for (int s = 1; s < 256; s++)
        if (f[s] > f[best]) best = s;
    if ((int64_t)f[best] + d >= 1) {
        f[best] = (uint32_t)((int64_t)f[best] + d);
    } else {
        while (sum > (int64_t)PROB_TOTAL) {
            int big = -1;
            for (int s = 0; s < 256; s++)
                if (f[s] > 1 && (big < 0 || f[s] > f[big])) big = s;
            if (big < 0) return ORC_ERR_ARG; /* more than 4096 distinct symbols: impossible */
            f[big] -= 1;
            sum -= 1;
        }
    }
    return ORC_OK;
}

static int table_ok(const uint32_t f[256], uint32_t cum[256])
{
    uint32_t c = 0;
    for (int s = 0; s < 256; s++) {
        cum[s] = c;
        if (f[s] > PROB_TOTAL) return 0;
        c += f[s];
    }
    return c == PROB_TOTAL;
}

/* ------------------------------------------------------------------------ */
/* rANS encode of one chunk                                                  */
/* ------------------------------------------------------------------------ */

/*
 * Encode n (1..65536) symbols with table f.  Writes the 32 final encoder
 * states (= the decoder's initial states) and the renormalisation words in
 * decode order.  Encoding one symbol s from state x (Duda's rANS):
 *   if x >= f_s * 2^20 (the bound that keeps the result below 2^32):
 *       emit the low 16 bits of x, x = x >> 16       (at most once)
 *   x = floor(x / f_s) * 4096 + (x mod f_s) + cum_s
 * Positions are visited in reverse decode order, so each emitted word is
 * prepended; the decoder then reads words front to back.
 */
int orc_encode_chunk(const uint8_t *sym, uint32_t n, const uint32_t f[256],
                     uint32_t states[32], uint16_t *words, uint32_t words_cap,
                     uint32_t *n_words)
{
    uint32_t cum[256];
    if (n == 0 || n > 65536u || !table_ok(f, cum)) return ORC_ERR_ARG;
    for (uint32_t j = 0; j < n; j++)
        if (f[sym[j]] == 0) return ORC_ERR_ARG;

    uint64_t x[32];
    for (uint32_t l = 0; l < LANES; l++) x[l] = STATE_LOW;

    /* emitted words are collected back to front at the end of `words` */
    uint32_t w = 0;
    const uint32_t T = n_steps(n);
    for (uint32_t t = T; t-- > 0;) {
        for (uint32_t l = LANES; l-- > 0;) {
            uint32_t j = symbol_index(t, l);
            if (j >= n) continue;
            uint32_t s = sym[j];
            uint64_t fs = f[s];
            if (x[l] >= (fs << 20)) {
                if (w >= words_cap) return ORC_ERR_SPACE;
                words[words_cap - 1 - w] = (uint16_t)(x[l] & 0xFFFFu);
                w++;
                x[l] >>= 16;
            }
            x[l] = (x[l] / fs) * PROB_TOTAL + (x[l] % fs) + cum[s];
        }
    }
    memmove(words, words + (words_cap - w), (size_t)w * sizeof(uint16_t));
    for (uint32_t l = 0; l < LANES; l++) states[l] = (uint32_t)x[l];
    *n_words = w;
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* rANS decode of one chunk                                                  */
/* ------------------------------------------------------------------------ */

/*
 * Decode n symbols.  For each position in decode order:
 *   slot = x mod 4096
 *   s    = the symbol with cum_s <= slot < cum_s + f_s
 *   x    = f_s * (x div 4096) + slot - cum_s
 *   if x < 2^16: x = x * 2^16 + next word
 * A well-formed chunk starts with every state in [2^16, 2^32), ends with
 * every state equal to 2^16 and has consumed exactly n_words words; anything
 * else is reported as ORC_ERR_CORRUPT.  If `check_each` is non-zero the
 * state is also checked to lie in [2^16, 2^32) after every symbol.
 * `final_states` (may be NULL) receives the states at the end.
 */
int orc_decode_chunk(const uint32_t states[32], const uint16_t *words, uint32_t n_words,
                     const uint32_t f[256], uint32_t n, uint8_t *out,
                     int check_each, uint32_t *final_states)
{
    uint32_t cum[256];
    if (n == 0 || n > 65536u) return ORC_ERR_ARG;
    if (!table_ok(f, cum)) return ORC_ERR_CORRUPT;

    /* present symbols in ascending byte order (the order of cum) */
    int present[256], n_present = 0;
    for (int c = 0; c < 256; c++)
        if (f[c] != 0) present[n_present++] = c;

    uint64_t x[32];
    for (uint32_t l = 0; l < LANES; l++) {
        x[l] = states[l];
        if (x[l] < STATE_LOW) return ORC_ERR_CORRUPT;
    }
    uint32_t p = 0;
    const uint32_t T = n_steps(n);
    for (uint32_t t = 0; t < T; t++) {
        for (uint32_t l = 0; l < LANES; l++) {
            uint32_t j = symbol_index(t, l);
            if (j >= n) continue;
            uint32_t slot = (uint32_t)(x[l] % PROB_TOTAL);
            int s = -1;
            for (int k = 0; k < n_present; k++) {
                int c = present[k];
                if (cum[c] <= slot && slot < cum[c] + f[c]) { s = c; break; }
            }
            if (s < 0) return ORC_ERR_CORRUPT; /* cannot happen for a valid table */
            out[j] = (uint8_t)s;
            x[l] = (uint64_t)f[s] * (x[l] / PROB_TOTAL) + slot - cum[s];
            if (x[l] < STATE_LOW) {
                if (p >= n_words) return ORC_ERR_CORRUPT;
                x[l] = (x[l] << 16) | words[p];
                p++;
            }
            if (check_each && (x[l] < STATE_LOW || x[l] > 0xFFFFFFFFull)) return ORC_ERR_CORRUPT;
        }
    }
    if (final_states)
        for (uint32_t l = 0; l < LANES; l++) final_states[l] = (uint32_t)x[l];
    for (uint32_t l = 0; l < LANES; l++)
        if (x[l] != STATE_LOW) return ORC_ERR_CORRUPT;
    if (p != n_words) return ORC_ERR_CORRUPT;
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* number formats and dequantisation                                         */
/* ------------------------------------------------------------------------ */

/* Int8 symbol: the two's-complement value of the byte. */
double orc_int8_value(uint8_t b)
{
    return b < 128 ? (double)b : (double)b - 256.0;
}

/*
 * Float8 E4M3 (OCP "E4M3FN"): bit 7 sign, bits 6..3 exponent e, bits 2..0
 * mantissa m, bias 7; e = 0 is subnormal (m / 8) * 2^-6, otherwise
 * (1 + m / 8) * 2^(e - 7); 0x7F / 0xFF are NaN; 0x80 is -0.
 */
double orc_e4m3_value(uint8_t b)
{
    int sign = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp(m / 8.0, -6);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

/*
 * fp32 product with round-to-nearest-even: the exact product of two fp32
 * numbers needs at most 48 significant bits, so it is exact in fp64, and one
 * conversion to fp32 rounds it once, to nearest even (subnormals kept).
 */
float orc_fp32_mul_rn(float a, float b)
{
    volatile double p = (double)a * (double)b;
    return (float)p;
}

/* fp32 -> bf16 bits, round to nearest even: (b + 0x7FFF + bit16) >> 16. */
uint16_t orc_bf16_rne(float v)
{
    uint32_t b;
    memcpy(&b, &v, 4);
    return (uint16_t)((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
}

/* bf16_rne over an array */
void orc_bf16_rne_n(const float *v, uint64_t n, uint16_t *out)
{
    for (uint64_t k = 0; k < n; k++) out[k] = orc_bf16_rne(v[k]);
}

/* value of one symbol of the given dtype (1 = Int8, 2 = E4M3) */
static double symbol_value(int dtype, uint8_t b)
{
    return dtype == 1 ? orc_int8_value(b) : orc_e4m3_value(b);
}

/* bf16 output of one symbol with its row scale */
uint16_t orc_dequant_one(int dtype, uint8_t sym, float scale)
{
    float v = (float)symbol_value(dtype, sym); /* exact: Int8 and E4M3 values are fp32 numbers */
    return orc_bf16_rne(orc_fp32_mul_rn(v, scale));
}

/*
 * Dequantise a row-major [rows, cols] symbol matrix (or `count` symbols
 * starting at linear index `first`): out[i] = bf16_rne(fp32(value * scale[row])).
 */
int orc_dequant(int dtype, const uint8_t *sym, uint64_t first, uint64_t count, uint64_t cols,
                const float *scales, uint16_t *out)
{
    if ((dtype != 1 && dtype != 2) || cols == 0) return ORC_ERR_ARG;
    for (uint64_t k = 0; k < count; k++) {
        uint64_t i = first + k;
        out[k] = orc_dequant_one(dtype, sym[k], scales[i / cols]);
    }
    return ORC_OK;
}

/*
 * Dequantise arbitrary (symbol, scale) pairs one by one (used to check
 * sampled outputs of very large matrices).
 */
void orc_dequant_pairs(int dtype, const uint8_t *sym, const float *scale, uint64_t count, uint16_t *out)
{
    for (uint64_t k = 0; k < count; k++) out[k] = orc_dequant_one(dtype, sym[k], scale[k]);
}

/*
 * Super-weight scatter (EntQuant: super weights are excluded from the
 * entropy-optimised stream and kept at full precision): for each outlier,
 * out[row * cols + col] = bf16_rne(value).  Outliers must be in range,
 * unique and sorted by linear index.
 */
int orc_scatter(uint64_t rows, uint64_t cols, uint32_t n_out, const uint32_t *out_row,
                const uint32_t *out_col, const float *out_val, uint16_t *out)
{
    uint64_t prev = 0;
    for (uint32_t k = 0; k < n_out; k++) {
        if (out_row[k] >= rows || out_col[k] >= cols) return ORC_ERR_CORRUPT;
        uint64_t lin = (uint64_t)out_row[k] * cols + out_col[k];
        if (k > 0 && lin <= prev) return ORC_ERR_CORRUPT;
        prev = lin;
        out[lin] = orc_bf16_rne(out_val[k]);
    }
    return ORC_OK;
}
