"""Seeded synthetic weight workloads for the entropy-coded weight decoder.

This module is shared by the tests, ``bench.py`` and ``__graft_entry__.smoke``.
It only *draws inputs*: Int8 / Float8-E4M3 weight symbols, fp32 per-row
scales, super-weight outlier lists and GEMV activations.  It contains none of
the method's arithmetic (no entropy coder, no container, no dequantisation to
bf16), so the CPU oracle and the CUDA path can both consume its output
without sharing any code with each other.

The pages measure on real checkpoints (LLaMA, Qwen3, Mistral, phi3) and public
evaluation suites; none of those are available here, so these generators stand
in for the *shapes* and *entropy levels* of the weights only:

* Int8 symbols: a discretised Laplace law on [-127, 127] whose scale ``b`` is
  chosen by bisection so that the symbol entropy hits a target (2.1, 2.5 or
  3.0 bits).  EntQuant keeps Int8 / Float8 symbols but drives their entropy
  down (EntQuant technical summary, section 2 "core concept" and
  "entropy-constrained optimisation"); a peaked, two-sided-geometric histogram
  is the shape that optimisation produces.
* Float8 E4M3 symbols: W = N(0, (0.02 * sigma_r)^2) with sigma_r lognormal,
  row scale = absmax_r * alpha / 448 (the AbsMax initialisation the EntQuant
  summary names), alpha chosen per matrix by bisection for the target entropy.
* Super-weight outliers in the down projection (EntQuant technical summary,
  section 2 "super weights"): unique seeded positions, magnitude 50-200x the
  row's standard deviation, random sign.

Every draw comes from ``numpy.random.Generator(PCG64(SeedSequence([...])))``
keyed by (workload id, layer, matrix index, 20260101).
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

SEED_TAG = 20260101

# dtype codes, as stored in the container directory (int8 = 1, e4m3 = 2)
INT8 = 1
E4M3 = 2

MATRIX_NAMES = ("q", "k", "v", "o", "gate", "up", "down")

# [out, in] shapes of one transformer block, row-major
LLAMA7B_BLOCK = (
    (4096, 4096), (4096, 4096), (4096, 4096), (4096, 4096),
    (11008, 4096), (11008, 4096), (4096, 11008),
)
LLAMA70B_BLOCK = (
    (8192, 8192), (1024, 8192), (1024, 8192), (8192, 8192),
    (28672, 8192), (28672, 8192), (8192, 28672),
)

# resolution of the inverse-CDF table used to draw Laplace symbols
_LAPLACE_TABLE_BITS = 16


def rng_for(workload_id: int, layer: int, matrix_idx: int, stream: int = 0) -> np.random.Generator:
    """The seeded generator for one matrix of one layer of one workload."""
    return np.random.Generator(np.random.PCG64(
        np.random.SeedSequence([workload_id, layer, matrix_idx, SEED_TAG, stream])))


# ---------------------------------------------------------------------------
# discretised Laplace Int8 symbols
# ---------------------------------------------------------------------------

def _entropy_bits(p: np.ndarray) -> float:
    p = p[p > 0]
    return float(-(p * np.log2(p)).sum())


def _laplace_counts(b: float, total: int) -> np.ndarray:
    """Integer counts (summing to ``total``) of a Laplace law on k = -127..127.

    p(k) is proportional to exp(-|k| / b); counts are the largest-remainder
    rounding of total * p(k), so the table is an exact discretisation at
    2^-16 resolution.
    """
    k = np.arange(-127, 128, dtype=np.float64)
    p = np.exp(-np.abs(k) / b)
    p /= p.sum()
    raw = p * total
    cnt = np.floor(raw).astype(np.int64)
    rem = total - int(cnt.sum())
    order = np.argsort(-(raw - cnt), kind="stable")
    cnt[order[:rem]] += 1
    return cnt


def laplace_b_for_entropy(h_bits: float) -> float:
    """Bisection for the Laplace scale whose 2^-16-resolution table has entropy ``h_bits``."""
    total = 1 << _LAPLACE_TABLE_BITS
    lo, hi = 0.05, 60.0
    for _ in range(80):
        mid = 0.5 * (lo + hi)
        h = _entropy_bits(_laplace_counts(mid, total) / total)
        if h < h_bits:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def laplace_table(h_bits: float) -> np.ndarray:
    """uint8 table of 2^16 entries: uniform index -> Int8 symbol byte (two's complement)."""
    total = 1 << _LAPLACE_TABLE_BITS
    cnt = _laplace_counts(laplace_b_for_entropy(h_bits), total)
    vals = (np.arange(-127, 128, dtype=np.int64) & 0xFF).astype(np.uint8)
    return np.repeat(vals, cnt)


_TABLE_CACHE: dict[float, np.ndarray] = {}


def _cached_table(h_bits: float) -> np.ndarray:
    key = round(float(h_bits), 6)
    if key not in _TABLE_CACHE:
        _TABLE_CACHE[key] = laplace_table(h_bits)
    return _TABLE_CACHE[key]


def laplace_int8_symbols(rng: np.random.Generator, rows: int, cols: int, h_bits: float) -> np.ndarray:
    """[rows, cols] uint8 array of Int8 symbols (two's complement bytes)."""
    table = _cached_table(h_bits)
    n = rows * cols
    out = np.empty(n, dtype=np.uint8)
    step = 1 << 26
    for s in range(0, n, step):
        u = rng.random(min(step, n - s), dtype=np.float32)
        u *= np.float32(1 << _LAPLACE_TABLE_BITS)
        out[s:s + u.size] = table[u.astype(np.uint16)]
    return out.reshape(rows, cols)


def lognormal_scales(rng: np.random.Generator, rows: int) -> np.ndarray:
    """fp32 per-row scales exp(ln(1e-3) + 0.3 z), z ~ N(0, 1)."""
    z = rng.standard_normal(rows)
    return np.exp(math.log(1e-3) + 0.3 * z).astype(np.float32)


def empirical_entropy_bits(symbols: np.ndarray) -> float:
    """Entropy (bits/symbol) of the byte histogram of ``symbols``."""
    c = np.bincount(np.asarray(symbols).reshape(-1), minlength=256).astype(np.float64)
    n = c.sum()
    return _entropy_bits(c / n) if n else 0.0


# ---------------------------------------------------------------------------
# Float8 E4M3 symbols (AbsMax-scaled Gaussian rows)
# ---------------------------------------------------------------------------

def _to_e4m3_bytes(v: np.ndarray) -> np.ndarray:
    """Saturate to +-448 then round-to-nearest-even into E4M3 (torch's cast).

    torch maps finite values above 448 to the NaN code 0x7F, so the
    saturation must happen first.
    """
    import torch
    t = torch.from_numpy(np.clip(v, -448.0, 448.0).astype(np.float32, copy=False))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _gaussian_rows(rng: np.random.Generator, rows: int, cols: int) -> tuple[np.ndarray, np.ndarray]:
    sigma = np.exp(0.25 * rng.standard_normal(rows)).astype(np.float32)
    w = rng.standard_normal((rows, cols), dtype=np.float32)
    w *= (0.02 * sigma)[:, None]
    return w, np.abs(w).max(axis=1)


def e4m3_matrix(rng: np.random.Generator, rows: int, cols: int, h_bits: float = 2.1,
                alpha: float | None = None) -> tuple[np.ndarray, np.ndarray, float]:
    """E4M3 symbols + fp32 row scales for a Gaussian weight matrix.

    scale_r = absmax_r * alpha / 448; symbols = E4M3(W / scale_r).  If
    ``alpha`` is None it is found by bisection (on up to 256 rows) so that the
    matrix's E4M3 symbol entropy is ``h_bits`` (+-0.02 checked on the full
    matrix).  Returns (symbols uint8 [rows, cols], scales fp32 [rows], alpha).
    """
    w, absmax = _gaussian_rows(rng, rows, cols)
    absmax = np.where(absmax > 0, absmax, np.float32(1.0)).astype(np.float32)

    def symbols_for(a: float, sl: slice) -> np.ndarray:
        sc = (absmax[sl] * np.float32(a / 448.0)).astype(np.float32)
        return _to_e4m3_bytes(w[sl] / sc[:, None])

    if alpha is None:
        sample = slice(0, min(rows, 256))
        lo, hi = 0.0, 25.0  # log2(alpha)
        for _ in range(40):
            mid = 0.5 * (lo + hi)
            h = empirical_entropy_bits(symbols_for(2.0 ** mid, sample))
            if h > h_bits:
                lo = mid
            else:
                hi = mid
        alpha = float(2.0 ** (0.5 * (lo + hi)))
    scales = (absmax * np.float32(alpha / 448.0)).astype(np.float32)
    sym = np.empty((rows, cols), dtype=np.uint8)
    step = max(1, (1 << 24) // max(cols, 1))
    for r in range(0, rows, step):
        sym[r:r + step] = _to_e4m3_bytes(w[r:r + step] / scales[r:r + step, None])
    return sym, scales, alpha


# ---------------------------------------------------------------------------
# super-weight outliers
# ---------------------------------------------------------------------------

def outliers_for(rng: np.random.Generator, symbols: np.ndarray, scales: np.ndarray, n_out: int,
                 dtype: int = INT8) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """``n_out`` unique positions sorted by linear index, |v| in U(50, 200) * row std.

    The row std is that of the row's real-valued weights symbol * scale
    (computed in float64: it only sizes the outliers).  Returns
    (row u32, col u32, value f32).
    """
    rows, cols = symbols.shape
    lin = np.sort(rng.choice(rows * cols, size=n_out, replace=False)).astype(np.int64)
    r = (lin // cols).astype(np.uint32)
    c = (lin % cols).astype(np.uint32)
    if dtype == INT8:
        vals = symbols[r].view(np.int8).astype(np.float64)
    else:
        import torch
        vals = torch.from_numpy(np.ascontiguousarray(symbols[r])).view(torch.float8_e4m3fn).double().numpy()
    rowstd = (vals * scales[r].astype(np.float64)[:, None]).std(axis=1)
    mag = rng.uniform(50.0, 200.0, size=n_out) * rowstd
    sign = np.where(rng.integers(0, 2, size=n_out) == 1, 1.0, -1.0)
    return r, c, (sign * mag).astype(np.float32)


# ---------------------------------------------------------------------------
# matrices and blocks
# ---------------------------------------------------------------------------

@dataclass
class Matrix:
    """One weight matrix: [rows, cols] symbols, fp32 row scales, outlier COO."""
    layer: int
    index: int
    name: str
    dtype: int
    symbols: np.ndarray          # uint8 [rows, cols], row-major
    scales: np.ndarray           # float32 [rows]
    out_row: np.ndarray = field(default_factory=lambda: np.zeros(0, np.uint32))
    out_col: np.ndarray = field(default_factory=lambda: np.zeros(0, np.uint32))
    out_val: np.ndarray = field(default_factory=lambda: np.zeros(0, np.float32))

    @property
    def rows(self) -> int:
        return int(self.symbols.shape[0])

    @property
    def cols(self) -> int:
        return int(self.symbols.shape[1])

    @property
    def n(self) -> int:
        return self.rows * self.cols


def _int8_matrix(wid: int, layer: int, i: int, shape, h_bits: float, n_out: int = 0) -> Matrix:
    rng = rng_for(wid, layer, i)
    rows, cols = shape
    sym = laplace_int8_symbols(rng, rows, cols, h_bits)
    sc = lognormal_scales(rng, rows)
    m = Matrix(layer, i, MATRIX_NAMES[i % 7], INT8, sym, sc)
    if n_out:
        m.out_row, m.out_col, m.out_val = outliers_for(rng, sym, sc, n_out, INT8)
    return m


def _parallel(fn, items, threads: int | None = None):
    threads = threads or min(len(items), os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        return list(ex.map(fn, items))


def single_matrix(h_bits: float = 2.1) -> list[Matrix]:
    """Workload 1: one 1024x1024 Int8 matrix, Laplace symbols at ~2.1 bits."""
    return [_int8_matrix(1, 0, 0, (1024, 1024), h_bits)]


def llama7b_int8_block(h_bits: float = 2.1, workload_id: int = 2, threads: int | None = None) -> list[Matrix]:
    """Workload 2: a 7B-shape block (q,k,v,o,gate,up,down) of Int8 symbols at ``h_bits``."""
    wid = workload_id * 100 + int(round(h_bits * 10))
    return _parallel(lambda i: _int8_matrix(wid, 0, i, LLAMA7B_BLOCK[i], h_bits), range(7), threads)


def llama70b_e4m3_block(h_bits: float = 2.1, threads: int | None = None) -> list[Matrix]:
    """Workload 3: a 70B-shape block of E4M3 symbols at ``h_bits``."""
    def one(i):
        rows, cols = LLAMA70B_BLOCK[i]
        sym, sc, _ = e4m3_matrix(rng_for(3, 0, i), rows, cols, h_bits)
        return Matrix(0, i, MATRIX_NAMES[i], E4M3, sym, sc)
    return _parallel(one, range(7), threads)


def llama7b_int8_block_with_outliers(h_bits: float = 2.5, n_out: int = 16,
                                     threads: int | None = None) -> list[Matrix]:
    """Workload 4: the 7B-shape Int8 block at ~2.5 bits plus ``n_out`` outliers in ``down``."""
    return _parallel(lambda i: _int8_matrix(4, 0, i, LLAMA7B_BLOCK[i], h_bits, n_out if i == 6 else 0),
                     range(7), threads)


def llama70b_int8_layer(layer: int, h_bits: float = 2.1, threads: int | None = None) -> list[Matrix]:
    """Workload 5: one layer of the streamed 80-layer 70B-shape model, Int8 at ~2.1 bits."""
    return _parallel(lambda i: _int8_matrix(5, layer, i, LLAMA70B_BLOCK[i], h_bits), range(7), threads)


def gemv_activation(layer: int, matrix_idx: int, n: int):
    """bf16 activation x ~ N(0, 1) of length ``n`` for the batch-1 GEMV consumer (torch CPU tensor)."""
    import torch
    z = rng_for(5, layer, matrix_idx, stream=1).standard_normal(n).astype(np.float32)
    return torch.from_numpy(z).to(torch.bfloat16)


def random_int8_matrix(seed: int, rows: int, cols: int, h_bits: float = 2.1,
                       n_out: int = 0, layer: int = 0, index: int = 0) -> Matrix:
    """A small seeded Int8 matrix of any shape (ragged sizes for edge-case tests)."""
    rng = rng_for(900 + seed, layer, index)
    sym = laplace_int8_symbols(rng, rows, cols, h_bits)
    sc = lognormal_scales(rng, rows)
    m = Matrix(layer, index, f"m{index}", INT8, sym, sc)
    if n_out:
        m.out_row, m.out_col, m.out_val = outliers_for(rng, sym, sc, n_out, INT8)
    return m


def random_e4m3_matrix(seed: int, rows: int, cols: int, alpha: float = 1.0,
                       layer: int = 0, index: int = 0) -> Matrix:
    """A small seeded E4M3 matrix; alpha = 1 exercises the normal E4M3 range (~250 codes)."""
    sym, sc, _ = e4m3_matrix(rng_for(950 + seed, layer, index), rows, cols, alpha=alpha)
    return Matrix(layer, index, f"m{index}", E4M3, sym, sc)
