/*
 * eqw.h -- C ABI of libeqw, B200 (sm_100a) decoder for entropy-coded weights.
 *
 * The method (EntQuant technical summary, gist.science paper 2601.22787,
 * section 2 "weight encoding" and "inference-time decoding"): weights keep an
 * Int8 or Float8 base format, are flattened into a symbol stream and
 * compressed losslessly with an ANS coder; storage is the bitstream plus the
 * per-channel scales plus metadata.  The bitstream stays resident in GPU
 * memory and, just before a transformer block runs, a parallel ANS decoder
 * expands that block's weights into a buffer; decoding and the forward
 * kernels are interleaved.  Super weights (extreme Int8 outliers, section 2
 * "super weights") are kept outside the entropy-coded stream.  Chunks are
 * independent so that they decode in parallel (EntroLLM technical overview,
 * "parallel decoding strategy").
 *
 * Coding used here: rANS, 12-bit frequencies (M = 4096), 32-bit states in
 * [2^16, 2^32), 16-bit renormalisation words, 32 interleaved states per chunk
 * of up to 65536 symbols, per-chunk frequency tables, fp32 per-row scales,
 * fp32 COO outliers; or, per matrix, canonical Huffman codes on the same
 * chunk and lane layout (EQ_CODEC_HUFFMAN below).  Byte layout ("container v1", little-endian, sections
 * 256-byte aligned):
 *   header (64 B): "EQW1", version 1, format constants, counts, total length;
 *   directory (64 B per matrix): layer, index, dtype, rows, cols, chunk
 *     count, outlier count, offsets of the chunk index, scales, outliers;
 *   per matrix: chunk index u64[n_chunks + 1] (record offsets, the last one
 *     the end), scales f32[rows], outliers {u32 row, u32 col, f32 value}
 *     sorted by linear index (the symbol stream holds symbol 0 under each);
 *   chunk records (16-byte aligned): u32 n_syms, n_words, n_present, 0;
 *     u32 states[32]; u32 table[n_present] = symbol | f << 16 in ascending
 *     symbol order; padding to 16 B; u16 words[n_words]; padding to 16 B.
 *   Symbol j of a chunk belongs to lane (j mod 256) div 8 at step
 *   8 (j div 256) + j mod 8; words are consumed step by step, lanes in
 *   ascending order within a step.
 *
 * Conventions for every function below:
 *   - Return value: EQ_OK (0) or one of the EQ_ERR_* codes; nothing throws.
 *   - The caller owns all memory, streams and events.  The library never
 *     allocates device memory, never frees caller memory and never
 *     synchronises a stream or the device, except the device encoders
 *     (eq_encode_device, eq_encode_device_noalloc), which synchronise their
 *     stream.  The only allocations it makes are host-side
 *     descriptors and staging (eq_model, eq_encoded, encoder plans).
 *   - Device pointers are plain addresses in the current CUDA device's
 *     memory (from PyTorch: tensor.data_ptr()); streams/events are raw
 *     cudaStream_t / cudaEvent_t handles (torch.cuda.Stream().cuda_stream).
 *     Every decode call launches on the stream it is given, in the device
 *     that is current when it is called.
 *   - Problems found by a kernel are OR-ed asynchronously into *d_status, a
 *     caller-provided device int32 the caller zeroes beforehand and reads
 *     after its own synchronisation (EQ_DEV_* bits below).  A chunk with a
 *     problem leaves its output range unspecified; all others are exact.
 *   - Decoded values are bit-exact: out = bf16_rne(fp32_rn(value * scale))
 *     with round-to-nearest-even in both steps, no FMA, no flush-to-zero;
 *     outliers are written as bf16_rne(value).
 */
#ifndef EQW_H
#define EQW_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define EQW_API __attribute__((visibility("default")))

/* ---- status codes --------------------------------------------------------- */
enum {
    EQ_OK = 0,
    EQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad dtype, unsorted outliers ... */
    EQ_ERR_CORRUPT = 2,      /* container fails validation */
    EQ_ERR_UNSUPPORTED = 3,  /* format constant or version this build does not decode */
    EQ_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, event, attribute) */
    EQ_ERR_TIMEOUT = 5,      /* reserved for host-side bounded waits */
    EQ_ERR_NOSPACE = 6       /* output buffer too small; required size is reported */
};

/* bits OR-ed into *d_status by the kernels */
enum {
    EQ_DEV_BAD_HEADER = 1,   /* chunk record header inconsistent with the directory */
    EQ_DEV_BAD_TABLE = 2,    /* frequency table not ascending / f = 0 / sum != 4096 */
    EQ_DEV_BAD_STATE = 4,    /* an initial state outside [2^16, 2^32) */
    EQ_DEV_BAD_END = 8,      /* final states != 2^16 or words consumed != n_words */
    EQ_DEV_TIMEOUT = 16,     /* a bounded wait for a staged copy gave up */
    EQ_DEV_BAD_OUTLIER = 32, /* outlier position outside its matrix, or a non-zero stream value under it */
    EQ_DEV_CHECK = 64        /* checked build only (EQ_CHECKED=1): an invariant the kernels rely on failed --
                                a staging-ring word read outside the ring or before its copy was waited for,
                                an unfilled slot-table entry, a store outside the matrix, or a bulk copy
                                outside the chunk's payload; never set by a release build */
};

/* symbol formats */
enum { EQ_INT8 = 1, EQ_E4M3 = 2 };

/* ---- host encoder ------------------------------------------------------------
 * One weight matrix to encode.  `symbols` is row-major [rows, cols] (Int8 as
 * two's-complement bytes, or E4M3 bytes; the E4M3 NaN codes 0x7F / 0xFF are
 * rejected).  `scales` holds one fp32 scale per row.  Outliers (super
 * weights) are given as parallel arrays, sorted by row * cols + col, unique
 * and in range; their positions are coded as symbol 0 in the stream and
 * overwritten by the scatter after decoding.  `layer` groups matrices into
 * blocks: layers must be 0..n_layers-1; matrices of one layer keep their
 * order in the input array (that order is their index within the layer).
 * All pointers are host pointers and are only read.
 */
typedef struct eq_matrix_in {
    uint32_t layer;
    uint32_t dtype;          /* EQ_INT8 or EQ_E4M3 */
    uint32_t rows;
    uint32_t cols;
    const uint8_t *symbols;  /* rows * cols bytes */
    const float *scales;     /* rows floats */
    uint32_t n_out;
    const uint32_t *out_row; /* n_out entries (may be NULL if n_out == 0) */
    const uint32_t *out_col;
    const float *out_val;
    uint32_t flags;          /* EQ_TABLE_* below; 0 = default */
} eq_matrix_in;

/*
 * Frequency-table scope (eq_matrix_in.flags).  Every chunk record always
 * carries its own 12-bit table.  By default the encoder quantises one table
 * from the whole matrix's histogram and writes it into every chunk, which
 * lets the decoder keep a single slot table per thread block for the matrix;
 * EQ_TABLE_PER_CHUNK quantises each chunk's own histogram instead (adapts to
 * local statistics; the decoder then builds one slot table per warp).
 */
#define EQ_TABLE_PER_CHUNK 1u

/*
 * Codec (eq_matrix_in.flags; directory entry word 7 = 0 rANS, 1 Huffman).
 * Default rANS.  EQ_CODEC_HUFFMAN codes the matrix with canonical Huffman
 * codes of at most 12 bits (EntroLLM technical overview, "Huffman weight
 * encoding"), on the same chunk and lane layout: a lane's bit stream is its
 * symbols' codes in step order, most significant bit first; before decoding a
 * symbol a lane holding fewer than 12 unread bits takes the next 16-bit word
 * (words ordered by step, then lane); a chunk with one distinct symbol has
 * the empty code.  Huffman chunk record: u32 n_syms, n_words, n_present, 0;
 * u32 table[n_present] = symbol | length << 16 sorted by (length, symbol);
 * padding to 16 B; u16 words; padding to 16 B (no states).  Both encoders
 * write it (the same bytes for the same inputs).
 */
#define EQ_CODEC_HUFFMAN 2u

typedef struct eq_encoded eq_encoded;  /* host-side result of eq_encoder_run */

/*
 * Encode `n_mats` matrices into a container with `n_threads` host threads
 * (<= 0: all online cores).  On success *h holds the encoded container in
 * library-owned host memory and *size its exact byte length.  Errors:
 * EQ_ERR_INVALID_ARG for bad inputs.
 */
EQW_API int eq_encoder_run(const eq_matrix_in *mats, uint32_t n_mats, int n_threads,
                           eq_encoded **h, size_t *size);

/* Copy the encoded container to `out` (host, >= size bytes). EQ_ERR_NOSPACE if out_cap < size. */
EQW_API int eq_encoded_write(const eq_encoded *h, void *out, size_t out_cap);

/* Release the result of eq_encoder_run (NULL is ignored). */
EQW_API void eq_encoded_free(eq_encoded *h);

/*
 * One-call encoder: eq_encoder_run + eq_encoded_write + eq_encoded_free.
 * *out_len receives the container size; if out_cap is smaller the call
 * returns EQ_ERR_NOSPACE and leaves `out` untouched.
 */
EQW_API int eq_encode_host(const eq_matrix_in *mats, uint32_t n_mats, int n_threads,
                           void *out, size_t out_cap, size_t *out_len);

/* ---- device encoder ----------------------------------------------------------------
 * eq_encode_device writes the same container bytes as eq_encode_host for the
 * same inputs (same tables, same layout), with the per-symbol work on the GPU
 * (EntQuant section 2 "weight encoding": a GPU ANS coder).  Here every
 * pointer inside eq_matrix_in is a DEVICE address: symbols (8-byte aligned),
 * scales, out_row, out_col, out_val.  Steps, all on stream `s`: per-chunk
 * histograms on the GPU (super-weight positions count as symbol 0; an E4M3
 * NaN code is an error), frequency tables (rANS) or code lengths and
 * canonical codes (Huffman) on the host with the host encoder's routines, a
 * GPU pass that counts each chunk's words, the container plan on the host,
 * and a GPU pass that writes the records.  Unlike every other entry point it synchronises `s` (the plan
 * needs the counts on the host).
 *   d_out    device, out_cap bytes (eq_encode_bound gives a sufficient size);
 *            *out_len receives the exact container size; EQ_ERR_NOSPACE
 *            (d_out untouched) if out_cap is smaller.
 *   d_work   device workspace of eq_encode_device_workspace() bytes,
 *            caller-owned; contents undefined afterwards.
 * Errors: EQ_ERR_INVALID_ARG (shapes, flags, alignment, layers not 0..n-1,
 * an E4M3 NaN code, super weights out of range or not ascending),
 * EQ_ERR_NOSPACE, EQ_ERR_CUDA.
 */
EQW_API int eq_encode_device(const eq_matrix_in *mats, uint32_t n_mats, void *d_out, size_t out_cap,
                             size_t *out_len, void *d_work, size_t work_bytes, cudaStream_t s);

/* eq_encode_device with a workspace the library keeps in a file-scope device
 * array (16 MiB per device, reserved when the library loads): no device
 * memory is allocated and no workspace is passed, for callers that cannot
 * allocate device memory themselves.  The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress) with that device current;
 * make that first call before any stream capture.  Every call shares the
 * array: the library serialises its own callers with a host lock and
 * synchronises `s` before returning (also on errors), so its calls never
 * overlap on the GPU.  EQ_ERR_NOSPACE if the matrices need more workspace than
 * the array holds (eq_encode_device_workspace tells).  The pages have no
 * counterpart of this entry point. */
EQW_API int eq_encode_device_noalloc(const eq_matrix_in *mats, uint32_t n_mats, void *d_out, size_t out_cap,
                                     size_t *out_len, cudaStream_t s);

/* Workspace bytes eq_encode_device needs for these matrices (shapes only). */
EQW_API int eq_encode_device_workspace(const eq_matrix_in *mats, uint32_t n_mats, size_t *work_bytes);

/* An upper bound of the container size for these matrices (shapes only):
 * every chunk with a 256-entry table and one word per symbol. */
EQW_API int eq_encode_bound(const eq_matrix_in *mats, uint32_t n_mats, size_t *out_bytes);

/* ---- model (a container resident in device memory) ---------------------------- */
typedef struct eq_model eq_model;

typedef struct eq_matrix_info {
    uint32_t layer, index, dtype, rows, cols, n_chunks, n_outliers;
    uint32_t uniform_table;     /* 1 if every chunk carries the same frequency table */
    uint32_t codec;             /* 0 rANS, 1 Huffman */
    uint32_t reserved;
    uint64_t compressed_bytes;  /* bytes of its chunk records (tables, states, words) */
    uint64_t payload_words;     /* total 16-bit renormalisation words */
} eq_matrix_info;

/*
 * Open a container that the caller has copied to device memory at `d_blob`
 * (`len` bytes, 256-byte aligned).  `h_blob` must point to a host copy of the
 * same `len` bytes; it is read only during this call, to parse and validate
 * the header, the directory, every chunk index entry and every chunk
 * record's header and frequency table.  The model keeps `d_blob` (not a
 * copy): the device bytes must outlive the model and must not change.
 * Errors: EQ_ERR_INVALID_ARG, EQ_ERR_CORRUPT, EQ_ERR_UNSUPPORTED.
 */
EQW_API int eq_model_open(const void *d_blob, size_t len, const void *h_blob, eq_model **m);

/* Free the host descriptor (NULL is ignored).  Device memory is the caller's. */
EQW_API void eq_model_close(eq_model *m);

/*
 * Let this model's decode launches (eq_decode_*, eq_decode_gemv_*) and its
 * prefill GEMMs (eq_gemm_symbols*) use at most `max_sms` SMs (0: all, the
 * default).  The decode kernels keep one
 * block per SM for the whole launch, so a kernel that must run beside them
 * -- the consumer of the previous block in a streamed forward pass -- only
 * gets SMs they leave free.  Host-side setting; takes effect for launches
 * enqueued after the call.  Errors: EQ_ERR_INVALID_ARG (m NULL).
 */
EQW_API int eq_model_set_sm_limit(eq_model *m, uint32_t max_sms);

EQW_API int eq_model_counts(const eq_model *m, uint32_t *n_layers, uint32_t *n_matrices);
EQW_API int eq_matrix_get_info(const eq_model *m, uint32_t matrix, eq_matrix_info *info);

/* Matrices of `layer` are [*first, *first + *count) in directory order. */
EQW_API int eq_layer_matrices(const eq_model *m, uint32_t layer, uint32_t *first, uint32_t *count);

/*
 * Where eq_decode_block puts each matrix of `layer`: the bf16 matrices are
 * packed in index order, each starting at a 256-byte-aligned byte offset.
 * `offsets` (host, `cap` entries, may be NULL when cap == 0) receives the
 * byte offsets; *total_bytes the buffer size a block decode needs.
 */
EQW_API int eq_block_layout(const eq_model *m, uint32_t layer, size_t *offsets, uint32_t cap,
                            size_t *total_bytes);

/*
 * How a decode of `layer` (eq_decode_block, eq_decode_model_stream) divides
 * the layer's chunks between the two decode kernels on a GPU with `sms` SMs
 * (or the model's SM limit, if that is lower): pair_chunks[i] (host, `cap` >=
 * the layer's matrix count) receives how many leading chunks of the layer's
 * i-th matrix go to the kernel that decodes two full chunks per warp in
 * lockstep; the general kernel takes the rest.  A matrix qualifies when all
 * its chunks share one frequency table of 2..32 symbols and its rows are a
 * multiple of 512 symbols; a launch qualifies when it gives every warp of every
 * SM at least one pair.  Host only, no CUDA call: the decision is a pure
 * function of the container and `sms`.  The pages describe no such split
 * (EntroLLM technical overview, "parallel decoding strategy", only has chunks
 * decode independently).  Errors: EQ_ERR_INVALID_ARG (m or pair_chunks NULL,
 * layer out of range, cap too small, sms == 0).
 */
EQW_API int eq_decode_plan(const eq_model *m, uint32_t layer, uint32_t sms, uint32_t *pair_chunks, uint32_t cap);

/* ---- decode (hot path) ------------------------------------------------------
 * Decode one matrix into `d_out` (device, 2-byte aligned; 16-byte aligned and
 * cols % 8 == 0 take the vectorised stores; >= 2*rows*cols bytes, row-major
 * bf16): rANS or Huffman decode + dequant of every chunk (one warp per chunk,
 * two chunks per warp in lockstep where they fill whole tiles), then the
 * outlier scatter, both enqueued on `s`.
 */
EQW_API int eq_decode_matrix(const eq_model *m, uint32_t matrix, void *d_out, size_t out_bytes,
                             int32_t *d_status, cudaStream_t s);

/*
 * Decode every matrix of `layer` into `d_out` (device, 16-byte aligned,
 * >= eq_block_layout total): one decode launch per kernel variant the layer
 * needs (codec x table scope x dtype x output layout; one for a uniform
 * layer) plus one scatter launch when the layer has outliers.
 * EQ_ERR_NOSPACE if out_bytes is too small.
 */
EQW_API int eq_decode_block(const eq_model *m, uint32_t layer, void *d_out, size_t out_bytes,
                            int32_t *d_status, cudaStream_t s);

/*
 * Ping-pong streaming step for block-wise decode interleaved with a consumer
 * (EntQuant section 2 "inference-time decoding").  With b = layer & 1 it
 * enqueues on `decode_stream`: wait for ev_free[b] (skipped if NULL), decode
 * the block into d_buf[b] (eq_decode_block), record ev_ready[b].  The
 * consumer, on its own stream, waits for ev_ready[b], reads d_buf[b] and
 * records ev_free[b] when done.  Both buffers hold `buf_bytes` bytes.
 */
EQW_API int eq_decode_model_stream(const eq_model *m, uint32_t layer, void *const d_buf[2],
                                   size_t buf_bytes, int32_t *d_status, cudaStream_t decode_stream,
                                   cudaEvent_t const ev_free[2], cudaEvent_t const ev_ready[2]);

/*
 * Batch-1 consumer: y[r] = sum_c W[r, c] * x[c] with W bf16 [rows, cols]
 * row-major (16-byte aligned rows: cols % 8 == 0), x bf16 [cols], y fp32
 * [rows]; products and sums in fp32.  Enqueued on `s`.
 */
EQW_API int eq_gemv_bf16(const void *d_w, const void *d_x, float *d_y, uint32_t rows, uint32_t cols,
                         cudaStream_t s);

/* ---- fused decode + batch-1 GEMV --------------------------------------------------
 * y = W x for an entropy-coded matrix W without materialising W: each chunk
 * is decoded in registers (same decoder as eq_decode_block) and multiplied by
 * x as it is decoded (EntQuant section 2 "inference-time decoding"; its
 * section 5 expects large speed-ups from dedicated fused kernels).
 *   W[r, c] = bf16(fp32(value(sym) * scale[r])) with both roundings to nearest
 *             even, and bf16(v) at the super weights -- exactly the matrix
 *             eq_decode_block writes;
 *   y[r]    = sum_c W[r, c] * x[c], products exact in fp32, sums in fp32 in
 *             an order fixed by the chunk and lane layout (per lane, then a
 *             warp butterfly, then at most two chunk partials per row when
 *             cols <= 65536, so the result is deterministic).  Error bound:
 *             |y - exact| <= gamma_h * sum_c |W[r, c] x[c]| with
 *             h = cols / 64 + 8 + (super weights in the row), gamma_h =
 *             h u / (1 - h u), u = 2^-24.
 * The stream must hold a zero-valued symbol at every super-weight position
 * (both encoders write symbol 0 there; eq_decode_* check it, see
 * EQ_DEV_BAD_OUTLIER).
 * Arguments: x (device, bf16 [cols], 16-byte aligned), y (device, fp32 [rows],
 * overwritten: zeroed on `s` first, then accumulated by the kernel), d_status
 * as for the decoders.  Every matrix with rows * cols > 0 needs
 * cols % 256 == 0 (EQ_ERR_UNSUPPORTED otherwise); rANS and Huffman matrices
 * alike.  Enqueued on `s`.
 */
EQW_API int eq_decode_gemv_matrix(const eq_model *m, uint32_t matrix, const void *d_x, float *d_y,
                                  int32_t *d_status, cudaStream_t s);

/*
 * The same for every matrix of `layer`: d_x[i], d_y[i] (host arrays of
 * `count` device pointers, count = the layer's matrix count) belong to
 * matrix i of the layer in directory order.  One launch per kernel variant.
 */
EQW_API int eq_decode_gemv_block(const eq_model *m, uint32_t layer, const void *const *d_x, float *const *d_y,
                                 uint32_t count, int32_t *d_status, cudaStream_t s);

/* ---- prefill path: symbol bytes + tensor-core GEMM ------------------------------
 * EntQuant section 4: the decode cost is amortised at long sequences, where a
 * linear layer's forward pass is a GEMM over many tokens.
 *
 * eq_decode_symbols: decode one matrix's symbols, without dequantisation, into
 * `d_out` (device, 16-byte aligned, >= rows * cols bytes, row-major): Int8 or
 * E4M3 codes, half the bytes of bf16.  Super-weight positions hold the
 * stream's placeholder symbol 0 (their values stay in the container).
 */
EQW_API int eq_decode_symbols(const eq_model *m, uint32_t matrix, void *d_out, size_t out_bytes, int32_t *d_status,
                              cudaStream_t s);

/* The same for every matrix of `layer` in one launch: d_outs[i] (host array of
 * `count` device pointers, count = the layer's matrix count, each 16-byte
 * aligned with rows * cols bytes) receives matrix i of the layer. */
EQW_API int eq_decode_symbols_block(const eq_model *m, uint32_t layer, void *const *d_outs, uint32_t count,
                                    int32_t *d_status, cudaStream_t s);

/*
 * eq_gemm_symbols: Y = X W^T for a matrix whose symbols eq_decode_symbols
 * wrote to `d_sym`, on the tensor cores (tcgen05.mma, bf16 inputs, fp32
 * accumulation in tensor memory):
 *   Y[t, r] = scale[r] * sum_c X[t, c] * value(sym[r, c])
 *             + sum over super weights (r, c, v) of bf16(v) * X[t, c]
 * value() is exact in bf16; the scale multiplies the fp32 sum once per output
 * (round to nearest even).  X: device bf16 [tokens, cols] row-major, Y:
 * device fp32 [tokens, rows] row-major, both 16-byte aligned.  Needs
 * rows % 128 == 0, rows <= 128 * 65535 and cols % 64 == 0
 * (EQ_ERR_UNSUPPORTED otherwise).
 * Enqueued on `s`.
 */
EQW_API int eq_gemm_symbols(const eq_model *m, uint32_t matrix, const void *d_sym, const void *d_x, uint32_t tokens,
                            float *d_y, int32_t *d_status, cudaStream_t s);

/* The same for every matrix of `layer`, one persistent launch per weight type
 * (the tiles of all the layer's matrices shared out over the SMs, so that a
 * small matrix does not leave SMs idle; 256-token tiles of matrices with a
 * multiple of 256 rows run on pairs of SMs with tcgen05.mma.cta_group::2, and
 * inputs of at most 128 tokens take 128-token tiles): d_syms[i], d_xs[i], d_ys[i] (host
 * arrays of `count` device pointers, count = the layer's matrix count) belong
 * to matrix i of the layer in directory order; all take `tokens` tokens.  Each
 * matrix has the requirements of eq_gemm_symbols; nothing is launched when one
 * fails them (EQ_ERR_UNSUPPORTED / EQ_ERR_INVALID_ARG). */
EQW_API int eq_gemm_symbols_block(const eq_model *m, uint32_t layer, const void *const *d_syms,
                                  const void *const *d_xs, uint32_t tokens, float *const *d_ys, uint32_t count,
                                  int32_t *d_status, cudaStream_t s);

/* ---- failure detection ----------------------------------------------------------
 * Check of the decode kernels' timeout path: one warp runs the decoder's own
 * staging-ring drain on a ring slot marked as issued whose copy was never
 * started (its mbarrier is never completed), so the bounded wait gives up
 * after its limit (~2e9 SM cycles, about one second) and the warp ORs
 * EQ_DEV_TIMEOUT into *d_status and returns; nothing faults or hangs and
 * the context stays usable.  Enqueued on `s`; d_status as for the decoders.
 */
EQW_API int eq_selftest_wait_timeout(int32_t *d_status, cudaStream_t s);

/* 1 if this library was built with EQ_CHECKED=1 (libeqw_checked.so: the decode
 * kernels test their invariants at run time and report EQ_DEV_CHECK), else 0.
 * The checked build's outputs are those of the release build, bit for bit. */
EQW_API int eq_build_checked(void);

/*
 * The same check for the prefill GEMM's waits (eq_gemm_symbols): one block
 * with the GEMM's TMEM allocation and mbarrier ring, whose MMA lane waits on a
 * "full" barrier no producer arrives on; after the bounded wait gives up (~1
 * s) the block ORs EQ_DEV_TIMEOUT into *d_status, frees its TMEM and returns.
 * No fault, trap or hang.  Errors: EQ_ERR_INVALID_ARG, EQ_ERR_CUDA.
 */
EQW_API int eq_selftest_gemm_wait_timeout(int32_t *d_status, cudaStream_t s);

/* ---- misc ----------------------------------------------------------------------- */
EQW_API const char *eq_status_string(int status);

/* Container version this build decodes (1). */
EQW_API int eq_format_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EQW_H */
