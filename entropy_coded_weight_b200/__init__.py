"""entropy_coded_weight_b200 -- B200 decoder for entropy-coded LLM weights.

Thin Python layer over libeqw.so (C ABI in include/eqw.h).  Every function
marshals arguments and calls the C entry point of the same name; all decoding
runs in the library's CUDA kernels.  PyTorch provides device memory, streams
and events.

Typical use (EntQuant technical summary, gist.science 2601.22787, section 2:
weights stored as a compressed bitstream in GPU memory and expanded block by
block just before each block's forward pass)::

    blob = encode_host(matrices)                 # host, threads over chunks
    d_blob = upload(blob)                        # one copy into HBM
    model = Model(d_blob, blob)                  # parse + validate
    out = torch.empty(model.block_bytes(layer), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    model.decode_block(layer, out, status)       # rANS decode + dequant + scatter
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _lib
from ._lib import (EQ_DEV_BAD_END, EQ_DEV_BAD_HEADER, EQ_DEV_BAD_OUTLIER, EQ_DEV_BAD_STATE, EQ_DEV_BAD_TABLE,
                   EQ_CODEC_HUFFMAN, EQ_DEV_TIMEOUT, EQ_E4M3, EQ_INT8, EQ_TABLE_PER_CHUNK, EqError, check, eq_matrix_in,
                   eq_matrix_info, load)

__all__ = [
    "EQ_INT8", "EQ_E4M3", "EqError", "Model", "encode_host", "upload", "gemv_bf16", "eq_status_string",
    "eq_format_version", "EQ_DEV_BAD_HEADER", "EQ_DEV_BAD_TABLE", "EQ_DEV_BAD_STATE", "EQ_DEV_BAD_END",
    "EQ_DEV_TIMEOUT", "EQ_DEV_BAD_OUTLIER",
]


def _ptr(a) -> int | None:
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        return a.ctypes.data
    return a.data_ptr()


def _stream_handle(stream) -> int | None:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def eq_status_string(code: int) -> str:
    return load().eq_status_string(code).decode()


def eq_format_version() -> int:
    return load().eq_format_version()


def _matrix_in_array(matrices, table_scope: str = "matrix", codec: str = "rans"):
    """eq_matrix_in[] for objects with layer, dtype, symbols, scales, out_row/out_col/out_val."""
    keep = []
    arr = (eq_matrix_in * max(1, len(matrices)))()
    for i, m in enumerate(matrices):
        sym = np.ascontiguousarray(m.symbols, dtype=np.uint8)
        if sym.ndim != 2:
            raise ValueError("symbols must be [rows, cols]")
        sc = np.ascontiguousarray(m.scales, dtype=np.float32)
        orow = np.ascontiguousarray(getattr(m, "out_row", np.zeros(0)), dtype=np.uint32)
        ocol = np.ascontiguousarray(getattr(m, "out_col", np.zeros(0)), dtype=np.uint32)
        oval = np.ascontiguousarray(getattr(m, "out_val", np.zeros(0)), dtype=np.float32)
        keep += [sym, sc, orow, ocol, oval]
        e = arr[i]
        e.layer = int(m.layer)
        e.dtype = int(m.dtype)
        e.rows, e.cols = sym.shape
        e.symbols = sym.ctypes.data if sym.size else None
        e.scales = sc.ctypes.data if sc.size else None
        e.n_out = orow.size
        e.out_row = orow.ctypes.data if orow.size else None
        e.out_col = ocol.ctypes.data if ocol.size else None
        e.out_val = oval.ctypes.data if oval.size else None
        e.flags = _flags(m, table_scope, codec)
    return arr, keep


def _flags(m, table_scope: str, codec: str) -> int:
    if table_scope not in ("matrix", "chunk") or codec not in ("rans", "huffman"):
        raise ValueError("table_scope must be 'matrix' or 'chunk', codec 'rans' or 'huffman'")
    return (int(getattr(m, "flags", 0)) | (EQ_TABLE_PER_CHUNK if table_scope == "chunk" else 0)
            | (EQ_CODEC_HUFFMAN if getattr(m, "codec", codec) == "huffman" else 0))


def encode_host(matrices, n_threads: int = 0, table_scope: str = "matrix", codec: str = "rans") -> np.ndarray:
    """Encode matrices into a container v1 blob (uint8 numpy array) with eq_encoder_run.

    ``table_scope``: "matrix" (one table from the whole matrix's histogram,
    written into every chunk) or "chunk" (each chunk's own histogram).
    ``codec``: "rans" (12-bit rANS) or "huffman" (canonical Huffman codes of
    at most 12 bits); a matrix's own ``codec`` attribute wins.
    """
    L = load()
    arr, keep = _matrix_in_array(matrices, table_scope, codec)
    h = ctypes.c_void_p()
    size = ctypes.c_size_t()
    check(L.eq_encoder_run(arr, len(matrices), n_threads, ctypes.byref(h), ctypes.byref(size)), "eq_encoder_run")
    try:
        out = np.empty(size.value, np.uint8)
        check(L.eq_encoded_write(h, out.ctypes.data, out.size), "eq_encoded_write")
    finally:
        L.eq_encoded_free(h)
    del keep
    return out


def _device_matrix_in_array(matrices, table_scope: str, codec: str = "rans"):
    """eq_matrix_in[] whose pointers are device addresses (CUDA tensors on one device)."""
    import torch
    keep = []
    arr = (eq_matrix_in * max(1, len(matrices)))()
    for i, m in enumerate(matrices):
        sym = m.symbols
        if not (isinstance(sym, torch.Tensor) and sym.is_cuda and sym.dtype == torch.uint8 and sym.dim() == 2):
            raise ValueError("symbols must be a uint8 CUDA tensor [rows, cols]")
        sym = sym.contiguous()
        sc = m.scales.to(torch.float32).contiguous()
        n_out = 0 if getattr(m, "out_row", None) is None else int(m.out_row.numel())
        orow = ocol = oval = None
        if n_out:
            orow = m.out_row.to(torch.int32).contiguous()  # the library reads them as uint32
            ocol = m.out_col.to(torch.int32).contiguous()
            oval = m.out_val.to(torch.float32).contiguous()
        keep += [sym, sc, orow, ocol, oval]
        e = arr[i]
        e.layer = int(m.layer)
        e.dtype = int(m.dtype)
        e.rows, e.cols = sym.shape
        e.symbols = sym.data_ptr() if sym.numel() else None
        e.scales = sc.data_ptr() if sc.numel() else None
        e.n_out = n_out
        e.out_row = orow.data_ptr() if n_out else None
        e.out_col = ocol.data_ptr() if n_out else None
        e.out_val = oval.data_ptr() if n_out else None
        e.flags = _flags(m, table_scope, codec)
    return arr, keep


def encode_device(matrices, table_scope: str = "matrix", stream=None, codec: str = "rans"):
    """eq_encode_device: encode matrices whose symbols, scales and super weights
    are CUDA tensors; returns the container as a uint8 CUDA tensor (the same
    bytes eq_encode_host writes).  Each matrix needs ``layer``, ``dtype``,
    ``symbols`` (uint8 [rows, cols]), ``scales`` (float32 [rows]) and optionally
    ``out_row``, ``out_col`` (integer), ``out_val`` (float32).  ``table_scope``
    and ``codec`` as for encode_host.  Synchronises the stream."""
    import torch
    arr, keep = _device_matrix_in_array(matrices, table_scope, codec)
    n = len(matrices)
    L = load()
    wb, ob, ln = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    check(L.eq_encode_device_workspace(arr, n, ctypes.byref(wb)), "eq_encode_device_workspace")
    check(L.eq_encode_bound(arr, n, ctypes.byref(ob)), "eq_encode_bound")
    dev = keep[0].device if keep else torch.device("cuda")
    work = torch.empty(max(1, wb.value), dtype=torch.uint8, device=dev)
    out = torch.empty(max(1, ob.value), dtype=torch.uint8, device=dev)
    check(L.eq_encode_device(arr, n, out.data_ptr(), ob.value, ctypes.byref(ln), work.data_ptr(), wb.value,
                             _stream_handle(stream)), "eq_encode_device")
    return out[:ln.value]


def upload(blob: np.ndarray, device=None):
    """Copy a host container into a fresh device tensor (uint8; the allocator aligns it to >= 256 B)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(blob, dtype=np.uint8))
    return t.to(device or "cuda", non_blocking=False)


class Model:
    """A container resident in device memory (eq_model_open / eq_model_close)."""

    def __init__(self, d_blob, h_blob):
        self._L = load()
        self.d_blob = d_blob  # keep the device bytes alive
        self._h = np.ascontiguousarray(h_blob, dtype=np.uint8)
        if d_blob.numel() != self._h.size:
            raise ValueError("device and host copies differ in length")
        handle = ctypes.c_void_p()
        check(self._L.eq_model_open(d_blob.data_ptr(), self._h.size, self._h.ctypes.data, ctypes.byref(handle)),
              "eq_model_open")
        self._m = handle
        nl, nm = ctypes.c_uint32(), ctypes.c_uint32()
        check(self._L.eq_model_counts(self._m, ctypes.byref(nl), ctypes.byref(nm)), "eq_model_counts")
        self.n_layers, self.n_matrices = nl.value, nm.value
        self._h = None  # only needed while opening

    def close(self) -> None:
        if getattr(self, "_m", None):
            self._L.eq_model_close(self._m)
            self._m = None

    def set_sm_limit(self, max_sms: int) -> None:
        """eq_model_set_sm_limit: decode launches of this model use at most
        ``max_sms`` SMs (0: all), leaving the rest to a kernel that runs beside
        them, e.g. the consumer of the previous block."""
        check(self._L.eq_model_set_sm_limit(self._m, int(max_sms)), "eq_model_set_sm_limit")

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self) -> int:
        return self._m.value

    def info(self, matrix: int) -> eq_matrix_info:
        inf = eq_matrix_info()
        check(self._L.eq_matrix_get_info(self._m, matrix, ctypes.byref(inf)), "eq_matrix_get_info")
        return inf

    def layer_matrices(self, layer: int) -> range:
        f, c = ctypes.c_uint32(), ctypes.c_uint32()
        check(self._L.eq_layer_matrices(self._m, layer, ctypes.byref(f), ctypes.byref(c)), "eq_layer_matrices")
        return range(f.value, f.value + c.value)

    def block_layout(self, layer: int) -> tuple[list[int], int]:
        n = len(self.layer_matrices(layer))
        offs = (ctypes.c_size_t * max(1, n))()
        total = ctypes.c_size_t()
        check(self._L.eq_block_layout(self._m, layer, offs, n, ctypes.byref(total)), "eq_block_layout")
        return [offs[i] for i in range(n)], total.value

    def block_bytes(self, layer: int) -> int:
        return self.block_layout(layer)[1]

    def decode_plan(self, layer: int, sms: int) -> list[int]:
        """eq_decode_plan: per matrix of ``layer``, the leading chunks the
        two-chunks-per-warp kernel decodes on a GPU with ``sms`` SMs."""
        n = len(self.layer_matrices(layer))
        out = (ctypes.c_uint32 * max(1, n))()
        check(self._L.eq_decode_plan(self._m, layer, sms, out, n), "eq_decode_plan")
        return [out[i] for i in range(n)]

    def decode_matrix(self, matrix: int, out, status, stream=None) -> None:
        """eq_decode_matrix into ``out`` (device tensor, >= 2*rows*cols bytes)."""
        nbytes = out.numel() * out.element_size()
        check(self._L.eq_decode_matrix(self._m, matrix, out.data_ptr(), nbytes, status.data_ptr(),
                                       _stream_handle(stream)), "eq_decode_matrix")

    def decode_block(self, layer: int, out, status, stream=None) -> None:
        """eq_decode_block into ``out`` (device tensor, >= block_bytes(layer) bytes)."""
        nbytes = out.numel() * out.element_size()
        check(self._L.eq_decode_block(self._m, layer, out.data_ptr(), nbytes, status.data_ptr(),
                                      _stream_handle(stream)), "eq_decode_block")

    def decode_model_stream(self, layer: int, bufs, status, decode_stream, ev_free, ev_ready) -> None:
        """eq_decode_model_stream: wait ev_free[b], decode into bufs[b], record ev_ready[b] (b = layer & 1)."""
        nbytes = min(b.numel() * b.element_size() for b in bufs)
        pbuf = (ctypes.c_void_p * 2)(bufs[0].data_ptr(), bufs[1].data_ptr())
        pfree = (ctypes.c_void_p * 2)(*(e.cuda_event if e is not None else None for e in ev_free))
        pready = (ctypes.c_void_p * 2)(*(e.cuda_event for e in ev_ready))
        check(self._L.eq_decode_model_stream(self._m, layer, pbuf, nbytes, status.data_ptr(),
                                             _stream_handle(decode_stream), pfree, pready),
              "eq_decode_model_stream")

    def decode_symbols(self, matrix: int, out, status, stream=None) -> None:
        """eq_decode_symbols: the matrix's raw symbol bytes into ``out`` (uint8 CUDA tensor, >= rows*cols)."""
        nbytes = out.numel() * out.element_size()
        check(self._L.eq_decode_symbols(self._m, matrix, out.data_ptr(), nbytes, status.data_ptr(),
                                        _stream_handle(stream)), "eq_decode_symbols")

    def decode_symbols_block(self, layer: int, outs, status, stream=None) -> None:
        """eq_decode_symbols_block: raw symbol bytes of every matrix of ``layer`` into ``outs[i]``."""
        n = len(outs)
        po = (ctypes.c_void_p * max(1, n))(*(o.data_ptr() for o in outs))
        check(self._L.eq_decode_symbols_block(self._m, layer, po, n, status.data_ptr(), _stream_handle(stream)),
              "eq_decode_symbols_block")

    def gemm_symbols(self, matrix: int, sym, x, y, status, stream=None) -> None:
        """eq_gemm_symbols: y[t, r] = scale[r] * sum_c x[t, c] * value(sym[r, c]) (+ super weights), on the
        tensor cores; x bf16 [tokens, cols], y fp32 [tokens, rows] (CUDA tensors)."""
        check(self._L.eq_gemm_symbols(self._m, matrix, sym.data_ptr(), x.data_ptr(), x.shape[0], y.data_ptr(),
                                      status.data_ptr(), _stream_handle(stream)), "eq_gemm_symbols")

    def gemm_symbols_block(self, layer: int, syms, xs, ys, status, stream=None) -> None:
        """eq_gemm_symbols_block: ``gemm_symbols`` for every matrix of ``layer`` (``syms[i]``, ``xs[i]``,
        ``ys[i]`` belong to matrix i of the layer), one persistent tensor-core launch per weight type."""
        n = len(syms)
        if len(xs) != n or len(ys) != n:
            raise ValueError("syms, xs and ys must have one entry per matrix of the layer")
        tokens = xs[0].shape[0] if n else 0
        if any(x.shape[0] != tokens for x in xs):
            raise ValueError("every input of a block GEMM takes the same number of tokens")
        ps = (ctypes.c_void_p * max(1, n))(*(t.data_ptr() for t in syms))
        px = (ctypes.c_void_p * max(1, n))(*(t.data_ptr() for t in xs))
        py = (ctypes.c_void_p * max(1, n))(*(t.data_ptr() for t in ys))
        check(self._L.eq_gemm_symbols_block(self._m, layer, ps, px, tokens, py, n, status.data_ptr(),
                                            _stream_handle(stream)), "eq_gemm_symbols_block")

    def decode_gemv_matrix(self, matrix: int, x, y, status, stream=None) -> None:
        """eq_decode_gemv_matrix: y = W x without materialising W (x bf16 [cols], y fp32 [rows], device)."""
        check(self._L.eq_decode_gemv_matrix(self._m, matrix, x.data_ptr(), y.data_ptr(), status.data_ptr(),
                                            _stream_handle(stream)), "eq_decode_gemv_matrix")

    def decode_gemv_block(self, layer: int, xs, ys, status, stream=None) -> None:
        """eq_decode_gemv_block: ys[i] = W_i xs[i] for matrix i of ``layer`` (directory order)."""
        n = len(xs)
        px = (ctypes.c_void_p * max(1, n))(*(x.data_ptr() for x in xs))
        py = (ctypes.c_void_p * max(1, n))(*(y.data_ptr() for y in ys))
        check(self._L.eq_decode_gemv_block(self._m, layer, px, py, n, status.data_ptr(), _stream_handle(stream)),
              "eq_decode_gemv_block")


def gemv_bf16(w, x, y, stream=None) -> None:
    """eq_gemv_bf16: y[r] = sum_c w[r, c] * x[c] (w bf16 [rows, cols], x bf16 [cols], y fp32 [rows])."""
    rows, cols = w.shape
    check(load().eq_gemv_bf16(w.data_ptr(), x.data_ptr(), y.data_ptr(), rows, cols, _stream_handle(stream)),
          "eq_gemv_bf16")


def selftest_wait_timeout(status, stream=None) -> None:
    """eq_selftest_wait_timeout: make one bounded staging wait run out (about a
    second); the kernel ORs EQ_DEV_TIMEOUT into ``status`` (device int32)."""
    check(load().eq_selftest_wait_timeout(status.data_ptr(), _stream_handle(stream)), "eq_selftest_wait_timeout")


def selftest_gemm_wait_timeout(status, stream=None) -> None:
    """eq_selftest_gemm_wait_timeout: the prefill GEMM's MMA lane waits on a
    "full" barrier nothing arrives on until its bounded wait runs out (about a
    second); the block ORs EQ_DEV_TIMEOUT into ``status`` and frees its TMEM."""
    check(load().eq_selftest_gemm_wait_timeout(status.data_ptr(), _stream_handle(stream)),
          "eq_selftest_gemm_wait_timeout")
