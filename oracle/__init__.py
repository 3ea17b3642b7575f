"""CPU oracle for entropy-coded weight decode -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  The product
(``entropy_coded_weight_b200``) never imports it and shares no code with it:
the scalar rANS coder, the container writer and parser, the number formats
and the dequantiser here are written independently of the CUDA path.

Two ways to obtain the decoded bf16 weights of a matrix:

* **O-direct** (:func:`dequant_direct`): straight from the generator's
  symbols.  The coding is lossless (EntQuant technical summary, section 2:
  the low-entropy weights are compressed losslessly by an ANS coder), so the
  decode result is unique and equals the input symbols, dequantised.
* **O-decode** (:func:`decode_container`): this package's own scalar rANS
  decode of a container, followed by the same dequantiser and scatter.

The scalar coder lives in ``rans_oracle.c`` (plain C, built by :func:`build`);
this module holds the container format v1 (magic "EQW1": header, matrix
directory, chunk index, scales, outliers, 16-byte aligned chunk records) and
thin ctypes wrappers.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
(round trip, brute force over tiny alphabets, the rANS ideal-code-length
identity, the Shannon size bound, hand-derived fixtures in ``tests/golden``,
and torch / numpy library routines for Int8, E4M3, fp32 and bf16).
"""
from __future__ import annotations

import ctypes
import os
import struct
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rans_oracle.c")
_SRC_HUFF = os.path.join(_HERE, "huffman_oracle.c")
_LIB = os.path.join(_HERE, "_oracle.so")

OK, ERR_ARG, ERR_CORRUPT, ERR_SPACE = 0, 1, 2, 3

INT8, E4M3 = 1, 2
CODEC_RANS, CODEC_HUFFMAN = 0, 1  # directory entry word 7
PROB_TOTAL = 4096
STATE_LOW = 1 << 16
LANES = 32
GROUP = 8
CHUNK_SYMS = 65536
HEADER_BYTES = 64
DIR_ENTRY_BYTES = 64
SECTION_ALIGN = 256
MAGIC = b"EQW1"
VERSION = 1


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: oracle error {code}")
        self.code = code


# ---------------------------------------------------------------------------
# build / load the C part
# ---------------------------------------------------------------------------

def build(force: bool = False) -> str:
    """Compile rans_oracle.c and huffman_oracle.c into _oracle.so (gcc -O2, IEEE arithmetic, no contraction)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_SRC_HUFF))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fno-fast-math", "-ffp-contract=off",
            "-shared", "-fPIC", "-o", tmp, _SRC, _SRC_HUFF, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if _LIB_PATH[0] == _LIB:
            build()
        L = ctypes.CDLL(_LIB_PATH[0])
        vp, u32, u64, i32 = ctypes.c_void_p, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int
        L.orc_quantize_freqs.argtypes = [vp, vp]
        L.orc_encode_chunk.argtypes = [vp, u32, vp, vp, vp, u32, vp]
        L.orc_decode_chunk.argtypes = [vp, vp, u32, vp, u32, vp, i32, vp]
        L.orc_int8_value.argtypes = [ctypes.c_uint8]
        L.orc_int8_value.restype = ctypes.c_double
        L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_value.restype = ctypes.c_double
        L.orc_fp32_mul_rn.argtypes = [ctypes.c_float, ctypes.c_float]
        L.orc_fp32_mul_rn.restype = ctypes.c_float
        L.orc_bf16_rne.argtypes = [ctypes.c_float]
        L.orc_bf16_rne.restype = ctypes.c_uint16
        L.orc_dequant_one.argtypes = [i32, ctypes.c_uint8, ctypes.c_float]
        L.orc_dequant_one.restype = ctypes.c_uint16
        L.orc_dequant.argtypes = [i32, vp, u64, u64, u64, vp, vp]
        L.orc_dequant_pairs.argtypes = [i32, vp, vp, u64, vp]
        L.orc_dequant_pairs.restype = None
        L.orc_scatter.argtypes = [u64, u64, u32, vp, vp, vp, vp]
        L.orc_bf16_rne_n.argtypes = [vp, u64, vp]
        L.orc_bf16_rne_n.restype = None
        L.orc_huff_lengths.argtypes = [vp, vp]
        L.orc_huff_canonical.argtypes = [vp, vp]
        L.orc_huff_encode_chunk.argtypes = [vp, u32, vp, i32, vp, u32, vp]
        L.orc_huff_decode_chunk.argtypes = [vp, u32, vp, i32, ctypes.c_uint8, u32, vp]
        _lib = L
    return _lib


def _use_library(path: str | None) -> None:
    """Test hook: load the C part from ``path`` (a deliberately broken build in
    the mutation tests) or, with None, go back to the real one."""
    global _lib
    _lib = None
    if path is not None:
        real = _LIB_PATH[0]
        _LIB_PATH[0] = path
        try:
            lib()
        finally:
            _LIB_PATH[0] = real


_LIB_PATH = [_LIB]


def _p(a: np.ndarray) -> int:
    return a.ctypes.data


def _threads(threads: int | None) -> int:
    if threads:
        return threads
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------
# one chunk
# ---------------------------------------------------------------------------

def quantize_freqs(symbols: np.ndarray) -> np.ndarray:
    """12-bit frequency table (uint32[256], sum 4096) of a chunk's byte histogram."""
    counts = np.bincount(np.asarray(symbols, np.uint8).reshape(-1), minlength=256).astype(np.uint64)
    f = np.zeros(256, np.uint32)
    rc = lib().orc_quantize_freqs(_p(counts), _p(f))
    if rc:
        raise OracleError(rc, "quantize_freqs")
    return f


def encode_chunk(symbols: np.ndarray, f: np.ndarray | None = None):
    """rANS-encode one chunk.  Returns (states uint32[32], words uint16[W], f uint32[256])."""
    sym = np.ascontiguousarray(symbols, dtype=np.uint8).reshape(-1)
    if f is None:
        f = quantize_freqs(sym)
    f = np.ascontiguousarray(f, dtype=np.uint32)
    states = np.zeros(32, np.uint32)
    cap = max(1, sym.size)
    words = np.zeros(cap, np.uint16)
    nw = np.zeros(1, np.uint32)
    rc = lib().orc_encode_chunk(_p(sym), sym.size, _p(f), _p(states), _p(words), cap, _p(nw))
    if rc:
        raise OracleError(rc, "encode_chunk")
    return states, words[: int(nw[0])].copy(), f


def decode_chunk(states: np.ndarray, words: np.ndarray, f: np.ndarray, n: int,
                 check_each: bool = False, return_final: bool = False):
    """rANS-decode one chunk of ``n`` symbols.  Raises OracleError on corrupt data."""
    states = np.ascontiguousarray(states, dtype=np.uint32)
    words = np.ascontiguousarray(words, dtype=np.uint16)
    f = np.ascontiguousarray(f, dtype=np.uint32)
    out = np.zeros(max(n, 1), np.uint8)
    fin = np.zeros(32, np.uint32)
    rc = lib().orc_decode_chunk(_p(states), _p(words) if words.size else None, words.size, _p(f), n,
                                _p(out), int(check_each), _p(fin))
    if return_final:
        return rc, out[:n], fin
    if rc:
        raise OracleError(rc, "decode_chunk")
    return out[:n]


# ---------------------------------------------------------------------------
# one chunk, Huffman codec (EntroLLM technical overview, "Huffman weight
# encoding"; readings in huffman_oracle.c)
# ---------------------------------------------------------------------------

HUFF_MAX_LEN = 12


def huff_lengths(symbols=None, counts=None) -> np.ndarray:
    """Optimal code lengths (uint8[256], <= 12 bits; all 0 for a single distinct symbol)."""
    if counts is None:
        counts = np.bincount(np.asarray(symbols, np.uint8).reshape(-1), minlength=256)
    counts = np.ascontiguousarray(counts, np.uint64)
    ln = np.zeros(256, np.uint8)
    rc = lib().orc_huff_lengths(_p(counts), _p(ln))
    if rc:
        raise OracleError(rc, "huff_lengths")
    return ln


def huff_canonical(lengths) -> np.ndarray | None:
    """Canonical codes (uint16[256]) for the lengths, or None if they are not a complete code."""
    ln = np.ascontiguousarray(lengths, np.uint8)
    code = np.zeros(256, np.uint16)
    return code if lib().orc_huff_canonical(_p(ln), _p(code)) else None


def huff_encode_chunk(symbols: np.ndarray, lengths: np.ndarray | None = None):
    """Huffman-encode one chunk.  Returns (words uint16[W], lengths uint8[256], single)."""
    sym = np.ascontiguousarray(symbols, dtype=np.uint8).reshape(-1)
    if lengths is None:
        lengths = huff_lengths(sym)
    ln = np.ascontiguousarray(lengths, np.uint8)
    single = int(sym.size > 0 and not ln.any())
    cap = max(1, sym.size)
    words = np.zeros(cap, np.uint16)
    nw = np.zeros(1, np.uint32)
    rc = lib().orc_huff_encode_chunk(_p(sym), sym.size, _p(ln), single, _p(words), cap, _p(nw))
    if rc:
        raise OracleError(rc, "huff_encode_chunk")
    return words[: int(nw[0])].copy(), ln, bool(single)


def huff_decode_chunk(words: np.ndarray, lengths: np.ndarray, n: int, single_symbol: int | None = None):
    """Huffman-decode one chunk of ``n`` symbols (``single_symbol``: the symbol of an empty code)."""
    words = np.ascontiguousarray(words, dtype=np.uint16)
    ln = np.ascontiguousarray(lengths, np.uint8)
    out = np.zeros(max(n, 1), np.uint8)
    rc = lib().orc_huff_decode_chunk(_p(words) if words.size else None, words.size, _p(ln),
                                     int(single_symbol is not None), single_symbol or 0, n, _p(out))
    if rc:
        raise OracleError(rc, "huff_decode_chunk")
    return out[:n]


def symbol_position(j: int) -> tuple[int, int]:
    """(lane, step) that handles symbol j of a chunk."""
    return (j % 256) // 8, 8 * (j // 256) + (j % 8)


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------

def int8_value(b: int) -> float:
    return lib().orc_int8_value(b)


def e4m3_value(b: int) -> float:
    return lib().orc_e4m3_value(b)


def fp32_mul_rn(a: float, b: float) -> float:
    return lib().orc_fp32_mul_rn(a, b)


def bf16_rne_scalar(v: float) -> int:
    return lib().orc_bf16_rne(v)


def bf16_rne(v: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bits, round to nearest even (the C oracle's routine, element by element)."""
    v = np.ascontiguousarray(v, dtype=np.float32).reshape(-1)
    out = np.zeros(v.size, np.uint16)
    lib().orc_bf16_rne_n(_p(v), v.size, _p(out))
    return out


def dequant_pairs(dtype: int, sym: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """bf16 bits of value(sym[k]) * scale[k], one pair at a time."""
    sym = np.ascontiguousarray(sym, dtype=np.uint8).reshape(-1)
    scale = np.ascontiguousarray(scale, dtype=np.float32).reshape(-1)
    assert sym.size == scale.size
    out = np.zeros(sym.size, np.uint16)
    lib().orc_dequant_pairs(dtype, _p(sym), _p(scale), sym.size, _p(out))
    return out


def dequant(dtype: int, symbols: np.ndarray, scales: np.ndarray, threads: int | None = None) -> np.ndarray:
    """[rows, cols] bf16 bits: bf16_rne(fp32_rn(value(sym) * scale[row]))."""
    sym = np.ascontiguousarray(symbols, dtype=np.uint8)
    rows, cols = sym.shape
    sc = np.ascontiguousarray(scales, dtype=np.float32)
    out = np.zeros((rows, cols), np.uint16)
    n = rows * cols
    if n == 0:
        return out
    flat_s, flat_o = sym.reshape(-1), out.reshape(-1)
    step = max(cols, ((1 << 22) // cols) * cols)
    L = lib()

    def part(first):
        cnt = min(step, n - first)
        rc = L.orc_dequant(dtype, _p(flat_s) + first, first, cnt, cols, _p(sc), _p(flat_o) + 2 * first)
        if rc:
            raise OracleError(rc, "dequant")

    with ThreadPoolExecutor(_threads(threads)) as ex:
        list(ex.map(part, range(0, n, step)))
    return out


def scatter(out: np.ndarray, out_row, out_col, out_val) -> None:
    """In place: out[r, c] = bf16_rne(v) for every outlier (sorted, unique, in range)."""
    rows, cols = out.shape
    r = np.ascontiguousarray(out_row, np.uint32)
    c = np.ascontiguousarray(out_col, np.uint32)
    v = np.ascontiguousarray(out_val, np.float32)
    if r.size == 0:
        return
    assert out.flags.c_contiguous and out.dtype == np.uint16
    rc = lib().orc_scatter(rows, cols, r.size, _p(r), _p(c), _p(v), _p(out))
    if rc:
        raise OracleError(rc, "scatter")


def dequant_direct(m, threads: int | None = None) -> np.ndarray:
    """O-direct: the decoded bf16 bits of matrix ``m`` computed from its symbols."""
    out = dequant(m.dtype, m.symbols, m.scales, threads)
    scatter(out, m.out_row, m.out_col, m.out_val)
    return out


def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns -> their exact values as float64 (bf16 is the top half of an fp32)."""
    b = np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def gemv_exact(w_bits: np.ndarray, x_bits: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Batch-1 forward of a decoded matrix: y[r] = sum_c W[r, c] * x[c], and sum_c |W[r, c] * x[c]|.

    EntQuant technical summary, section 2 "inference-time decoding": the
    decoded block's weights feed its forward pass, which at batch 1 is a
    matrix-vector product per linear layer.  W (bf16 bits, [rows, cols]) and
    x (bf16 bits, [cols]) are widened exactly to float64; every product of two
    bf16 values is exact there (at most 16 significant bits), and the float64
    sums are within cols * 2^-53 of exact relative to the second result,
    far below any fp32 bound a test applies.
    """
    w = bf16_to_f64(w_bits).reshape(np.shape(w_bits))
    x = bf16_to_f64(x_bits).reshape(-1)
    return w @ x, np.abs(w) @ np.abs(x)


def symbol_values(dtype: int) -> np.ndarray:
    """Exact value of every symbol byte (float64[256]; NaN codes of E4M3 are NaN)."""
    f = int8_value if dtype == INT8 else e4m3_value
    return np.array([f(b) for b in range(256)], np.float64)


def stream_symbols(m) -> np.ndarray:
    """The symbols a container stores for matrix ``m``: its symbols with the
    placeholder 0 at every super-weight position."""
    sym = np.ascontiguousarray(m.symbols, np.uint8).copy()
    if len(m.out_row):
        sym[np.asarray(m.out_row, np.int64), np.asarray(m.out_col, np.int64)] = 0
    return sym


def gemm_symbols_exact(m, x_bits: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Prefill forward of matrix ``m`` on tokens ``x`` (bf16 bits [tokens, cols]), in float64:
    Y[t, r] = scale[r] * sum_c X[t, c] * value(sym[r, c]) + sum over super weights (r, c, v)
    of bf16(v) * X[t, c]; and the matching sum of absolute terms (for error bounds).

    EntQuant technical summary, section 4: at long sequences the decode cost is
    amortised over a GEMM per linear layer.  The scale multiplies the row's sum
    (it is the same real number as multiplying every product); super weights
    enter with their bf16 value, as the decode path writes them.
    """
    vals = symbol_values(m.dtype)
    w = vals[stream_symbols(m)]                       # [rows, cols], exact
    x = bf16_to_f64(x_bits).reshape(np.shape(x_bits))  # [tokens, cols], exact
    sc = np.asarray(m.scales, np.float64)
    y = (x @ w.T) * sc[None, :]
    mag = (np.abs(x) @ np.abs(w).T) * np.abs(sc)[None, :]
    if len(m.out_row):
        ov = bf16_to_f64(bf16_rne(np.asarray(m.out_val, np.float32)))
        for r, c, v in zip(np.asarray(m.out_row, np.int64), np.asarray(m.out_col, np.int64), ov):
            y[:, r] += v * x[:, c]
            mag[:, r] += abs(v) * np.abs(x[:, c])
    return y, mag


# ---------------------------------------------------------------------------
# container format v1 (writer)
# ---------------------------------------------------------------------------

def _align(x: int, a: int) -> int:
    return (x + a - 1) // a * a


def _huffman_record(sym: np.ndarray) -> bytes:
    """Huffman chunk record: n_syms, n_words, n_present, 0; entries symbol | length << 16
    sorted by (length, symbol) (one entry of length 0 for a single-symbol chunk); words."""
    words, ln, single = huff_encode_chunk(sym)
    if single:
        table = np.array([int(sym[0])], np.uint32)
    else:
        present = np.nonzero(ln)[0]
        present = present[np.lexsort((present, ln[present]))]
        table = (present.astype(np.uint32) | (ln[present].astype(np.uint32) << 16)).astype(np.uint32)
    body = struct.pack("<4I", sym.size, words.size, table.size, 0) + table.astype("<u4").tobytes()
    body += b"\0" * (_align(len(body), 16) - len(body))
    wb = words.astype("<u2").tobytes()
    wb += b"\0" * (_align(len(wb), 16) - len(wb))
    return body + wb


def _chunk_record(sym: np.ndarray, codec: int = CODEC_RANS) -> bytes:
    if codec == CODEC_HUFFMAN:
        return _huffman_record(sym)
    states, words, f = encode_chunk(sym)
    present = np.nonzero(f)[0]
    table = (present.astype(np.uint32) | (f[present].astype(np.uint32) << 16)).astype(np.uint32)
    head = struct.pack("<4I", sym.size, words.size, present.size, 0)
    body = head + states.astype("<u4").tobytes() + table.astype("<u4").tobytes()
    body += b"\0" * (_align(len(body), 16) - len(body))
    wb = words.astype("<u2").tobytes()
    wb += b"\0" * (_align(len(wb), 16) - len(wb))
    return body + wb


def _check_matrix(m) -> None:
    if m.dtype not in (INT8, E4M3):
        raise OracleError(ERR_ARG, "dtype")
    if m.dtype == E4M3 and m.n and np.any((m.symbols & 0x7F) == 0x7F):
        raise OracleError(ERR_ARG, "E4M3 NaN code")
    r = np.asarray(m.out_row, np.int64)
    c = np.asarray(m.out_col, np.int64)
    if r.size:
        if np.any(r >= m.rows) or np.any(c >= m.cols):
            raise OracleError(ERR_ARG, "outlier out of range")
        lin = r * m.cols + c
        if np.any(np.diff(lin) <= 0):
            raise OracleError(ERR_ARG, "outliers not sorted/unique")


def encode_container(mats, threads: int | None = None, codec: str = "rans") -> np.ndarray:
    """Write matrices (objects with layer, index, dtype, symbols, scales, out_*) into a v1 blob.

    Layers must be numbered 0..n_layers-1; within a layer the matrices are
    ordered by ``index``.  The symbol at each outlier position is replaced by
    the placeholder 0 before encoding (its value is overwritten by the scatter).
    ``codec``: "rans" or "huffman" for every matrix (a matrix's own ``codec``
    attribute, if present, wins).
    """
    mats = sorted(mats, key=lambda m: (m.layer, m.index))
    layers = sorted({m.layer for m in mats})
    if layers != list(range(len(layers))):
        raise OracleError(ERR_ARG, "layers must be 0..n-1")
    for m in mats:
        _check_matrix(m)

    codecs = [{"rans": CODEC_RANS, "huffman": CODEC_HUFFMAN}[getattr(m, "codec", codec)] for m in mats]
    jobs = []
    for mi, m in enumerate(mats):
        flat = np.ascontiguousarray(m.symbols, np.uint8).reshape(-1)
        if len(m.out_row):
            flat = flat.copy()
            flat[np.asarray(m.out_row, np.int64) * m.cols + np.asarray(m.out_col, np.int64)] = 0
        for k in range(0, m.n, CHUNK_SYMS):
            jobs.append((mi, flat[k:k + CHUNK_SYMS]))
    with ThreadPoolExecutor(_threads(threads)) as ex:
        records = list(ex.map(lambda j: _chunk_record(j[1], codecs[j[0]]), jobs))
    per_mat: list[list[bytes]] = [[] for _ in mats]
    for (mi, _), rec in zip(jobs, records):
        per_mat[mi].append(rec)

    # layout: header | directory | per matrix: chunk index, scales, outliers, chunk records
    pos = _align(HEADER_BYTES + DIR_ENTRY_BYTES * len(mats), SECTION_ALIGN)
    dir_off = HEADER_BYTES
    places = []
    for mi, m in enumerate(mats):
        nch = len(per_mat[mi])
        ci = pos
        pos = _align(pos + 8 * (nch + 1), SECTION_ALIGN)
        so = pos
        pos = _align(pos + 4 * m.rows, SECTION_ALIGN)
        oo = 0
        if len(m.out_row):
            oo = pos
            pos = _align(pos + 12 * len(m.out_row), SECTION_ALIGN)
        rec0 = pos
        offs = [rec0]
        for rec in per_mat[mi]:
            offs.append(offs[-1] + len(rec))
        pos = _align(offs[-1], SECTION_ALIGN)
        places.append((ci, so, oo, offs))
    total = pos

    blob = np.zeros(total, np.uint8)
    mv = memoryview(blob)
    mv[0:HEADER_BYTES] = struct.pack("<4s9I3Q", MAGIC, VERSION, HEADER_BYTES, 12, LANES, GROUP, CHUNK_SYMS,
                                     len(layers), len(mats), 0, dir_off, total, 0)
    for mi, m in enumerate(mats):
        ci, so, oo, offs = places[mi]
        nch = len(per_mat[mi])
        e = dir_off + DIR_ENTRY_BYTES * mi
        mv[e:e + DIR_ENTRY_BYTES] = struct.pack("<8I4Q", m.layer, m.index, m.dtype, nch, m.rows, m.cols,
                                                len(m.out_row), codecs[mi], ci, so, oo, 0)
        mv[ci:ci + 8 * (nch + 1)] = np.asarray(offs, "<u8").tobytes()
        mv[so:so + 4 * m.rows] = np.ascontiguousarray(m.scales, "<f4").tobytes()
        if len(m.out_row):
            rec = np.zeros((len(m.out_row), 3), "<u4")
            rec[:, 0] = m.out_row
            rec[:, 1] = m.out_col
            rec[:, 2] = np.asarray(m.out_val, "<f4").view("<u4")
            mv[oo:oo + rec.nbytes] = rec.tobytes()
        for k, rec in enumerate(per_mat[mi]):
            mv[offs[k]:offs[k] + len(rec)] = rec
    return blob


# ---------------------------------------------------------------------------
# container format v1 (parser + O-decode)
# ---------------------------------------------------------------------------

def parse_container(blob) -> dict:
    """Parse and validate the header, directory and chunk indices of a v1 blob."""
    b = np.frombuffer(blob, np.uint8) if not isinstance(blob, np.ndarray) else blob
    if b.size < HEADER_BYTES:
        raise OracleError(ERR_CORRUPT, "short blob")
    (magic, ver, hbytes, pbits, lanes, group, csyms, n_layers, n_mats, _r0,
     dir_off, total, _r1) = struct.unpack("<4s9I3Q", bytes(b[:HEADER_BYTES]))
    if magic != MAGIC or ver != VERSION or hbytes != HEADER_BYTES:
        raise OracleError(ERR_CORRUPT, "bad magic/version")
    if (pbits, lanes, group, csyms) != (12, LANES, GROUP, CHUNK_SYMS):
        raise OracleError(ERR_CORRUPT, "unsupported format constants")
    if total != b.size or dir_off + DIR_ENTRY_BYTES * n_mats > total:
        raise OracleError(ERR_CORRUPT, "bad sizes")
    mats = []
    for mi in range(n_mats):
        e = dir_off + DIR_ENTRY_BYTES * mi
        (layer, index, dtype, nch, rows, cols, n_out, codec, ci, so, oo, _q) = struct.unpack(
            "<8I4Q", bytes(b[e:e + DIR_ENTRY_BYTES]))
        n = rows * cols
        if dtype not in (INT8, E4M3) or layer >= n_layers or codec not in (CODEC_RANS, CODEC_HUFFMAN):
            raise OracleError(ERR_CORRUPT, "bad directory entry")
        if nch != (n + CHUNK_SYMS - 1) // CHUNK_SYMS:
            raise OracleError(ERR_CORRUPT, "chunk count")
        if ci + 8 * (nch + 1) > total or so + 4 * rows > total or (n_out and oo + 12 * n_out > total):
            raise OracleError(ERR_CORRUPT, "section out of range")
        offs = np.frombuffer(bytes(b[ci:ci + 8 * (nch + 1)]), "<u8").astype(np.int64)
        min_rec = 144 if codec == CODEC_RANS else 32
        if np.any(np.diff(offs) < min_rec) or offs[-1] > total or np.any(offs % 16):
            raise OracleError(ERR_CORRUPT, "chunk index")
        scales = np.frombuffer(bytes(b[so:so + 4 * rows]), "<f4").copy()
        if n_out:
            o = np.frombuffer(bytes(b[oo:oo + 12 * n_out]), "<u4").reshape(n_out, 3)
            orow, ocol, oval = o[:, 0].copy(), o[:, 1].copy(), o[:, 2].copy().view(np.float32)
        else:
            orow = ocol = np.zeros(0, np.uint32)
            oval = np.zeros(0, np.float32)
        mats.append(dict(layer=layer, index=index, dtype=dtype, codec=codec, rows=rows, cols=cols, n_chunks=nch,
                         chunk_offsets=offs, scales=scales, out_row=orow, out_col=ocol, out_val=oval))
    return dict(n_layers=n_layers, matrices=mats, blob=b)


def _decode_huffman_record(b: np.ndarray, off: int, end: int, n: int, nw: int, npres: int) -> np.ndarray:
    table = np.frombuffer(bytes(b[off + 16:off + 16 + 4 * npres]), "<u4")
    wo = off + _align(16 + 4 * npres, 16)
    if wo + 2 * nw > end:
        raise OracleError(ERR_CORRUPT, "chunk record overflows")
    words = np.frombuffer(bytes(b[wo:wo + 2 * nw]), "<u2")
    syms, lens = (table & 0xFF).astype(np.int64), (table >> 16).astype(np.int64)
    if np.any((table >> 8) & 0xFF):
        raise OracleError(ERR_CORRUPT, "table entry")
    if npres == 1:
        if lens[0] != 0:
            raise OracleError(ERR_CORRUPT, "single-symbol code")
        return huff_decode_chunk(words, np.zeros(256, np.uint8), n, single_symbol=int(syms[0]))
    key = lens * 256 + syms
    if np.any(np.diff(key) <= 0) or np.any(lens < 1) or np.any(lens > HUFF_MAX_LEN):
        raise OracleError(ERR_CORRUPT, "table order")
    ln = np.zeros(256, np.uint8)
    ln[syms] = lens
    return huff_decode_chunk(words, ln, n)


def _decode_record(b: np.ndarray, off: int, end: int, n_expected: int, codec: int = CODEC_RANS) -> np.ndarray:
    head = np.frombuffer(bytes(b[off:off + 16]), "<u4")
    n, nw, npres = int(head[0]), int(head[1]), int(head[2])
    if n != n_expected or not (1 <= npres <= 256):
        raise OracleError(ERR_CORRUPT, "chunk header")
    if codec == CODEC_HUFFMAN:
        return _decode_huffman_record(b, off, end, n, nw, npres)
    states = np.frombuffer(bytes(b[off + 16:off + 144]), "<u4")
    table = np.frombuffer(bytes(b[off + 144:off + 144 + 4 * npres]), "<u4")
    wo = off + _align(144 + 4 * npres, 16)
    if wo + 2 * nw > end:
        raise OracleError(ERR_CORRUPT, "chunk record overflows")
    words = np.frombuffer(bytes(b[wo:wo + 2 * nw]), "<u2")
    f = np.zeros(256, np.uint32)
    syms = table & 0xFF
    if np.any(np.diff(syms.astype(np.int64)) <= 0) or np.any((table >> 8) & 0xFF):
        raise OracleError(ERR_CORRUPT, "table order")
    f[syms] = table >> 16
    return decode_chunk(states, words, f, n)


def decode_matrix_symbols(parsed: dict, mi: int, threads: int | None = None) -> np.ndarray:
    """O-decode of one matrix's symbols ([rows, cols] uint8)."""
    m = parsed["matrices"][mi]
    b = parsed["blob"]
    n = m["rows"] * m["cols"]
    out = np.zeros(n, np.uint8)
    offs = m["chunk_offsets"]

    def one(k):
        lo = k * CHUNK_SYMS
        cnt = min(CHUNK_SYMS, n - lo)
        out[lo:lo + cnt] = _decode_record(b, int(offs[k]), int(offs[k + 1]), cnt, m["codec"])

    with ThreadPoolExecutor(_threads(threads)) as ex:
        list(ex.map(one, range(m["n_chunks"])))
    return out.reshape(m["rows"], m["cols"])


def decode_container(blob, layer: int | None = None, threads: int | None = None) -> list[np.ndarray]:
    """O-decode: bf16 bits of every matrix (of ``layer``, if given), in directory order."""
    parsed = parse_container(blob)
    res = []
    for mi, m in enumerate(parsed["matrices"]):
        if layer is not None and m["layer"] != layer:
            continue
        sym = decode_matrix_symbols(parsed, mi, threads)
        out = dequant(m["dtype"], sym, m["scales"], threads)
        scatter(out, m["out_row"], m["out_col"], m["out_val"])
        res.append(out)
    return res
