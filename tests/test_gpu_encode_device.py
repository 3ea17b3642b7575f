"""GPU encoder (eq_encode_device): its containers decoded by the CPU oracle,
and its bytes against the host encoder's.

The first check is independent of the product: the oracle's own scalar
decoder (O-decode, which shares no code with either encoder) must turn every
container the GPU wrote back into exactly the oracle's direct dequantisation
of the input symbols (EntQuant technical summary, section 2 "weight
encoding": the ANS coding is lossless).  The second pins the two product
encoders to each other: they quantise the same tables and lay out the same
container, so for the same inputs their bytes must be equal.
"""
import ctypes
from dataclasses import dataclass

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def eqw():
    from entropy_coded_weight_b200 import build
    build.build()
    import entropy_coded_weight_b200 as E
    E.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return E


@dataclass
class DevMatrix:
    layer: int
    dtype: int
    symbols: torch.Tensor
    scales: torch.Tensor
    out_row: torch.Tensor | None
    out_col: torch.Tensor | None
    out_val: torch.Tensor | None


def _dev(m):
    has = len(m.out_row) > 0
    d = DevMatrix(m.layer, m.dtype, torch.from_numpy(np.ascontiguousarray(m.symbols)).cuda(),
                  torch.from_numpy(np.ascontiguousarray(m.scales)).cuda(),
                  torch.from_numpy(m.out_row.astype(np.int32)).cuda() if has else None,
                  torch.from_numpy(m.out_col.astype(np.int32)).cuda() if has else None,
                  torch.from_numpy(m.out_val.astype(np.float32)).cuda() if has else None)
    if hasattr(m, "codec"):
        d.codec = m.codec  # a matrix's own codec wins over the call's
    return d


def _oracle_decodes(orc, blob, mats):
    """The oracle decodes the container exactly to O-direct, matrix by matrix."""
    got = orc.decode_container(blob)
    assert len(got) == len(mats)
    for g, m in zip(got, mats):
        want = orc.dequant_direct(m)
        assert g.shape == want.shape
        if not np.array_equal(g, want):
            raise AssertionError(f"matrix {m.layer}/{m.index}: {int(np.count_nonzero(g != want))} of {m.n} "
                                 f"outputs differ after the oracle's decode")


def _ragged():
    mats = [
        W.random_int8_matrix(1, 300, 229, layer=0, index=0),                 # tail chunk, cols % 8 != 0
        W.random_int8_matrix(2, 1, 1, layer=0, index=1),
        W.random_e4m3_matrix(3, 77, 1000, alpha=1.0, layer=0, index=2),      # ~250 codes
        W.random_int8_matrix(4, 512, 256, n_out=16, layer=1, index=0),
        W.random_int8_matrix(5, 3, 7, h_bits=1.0, layer=1, index=1),
        W.random_int8_matrix(6, 0, 64, layer=1, index=2),                    # empty
        W.random_int8_matrix(7, 700, 1300, h_bits=3.0, n_out=5, layer=2, index=0),
        W.random_e4m3_matrix(8, 96, 2048, alpha=9.1e4, layer=2, index=1),
    ]
    single = W.random_int8_matrix(9, 64, 1100, layer=2, index=2)
    single.symbols[:] = 0x03                                                # f = 4096 in every chunk
    mats.append(single)
    return mats


@pytest.mark.parametrize("codec", ["rans", "huffman"])
@pytest.mark.parametrize("scope", ["matrix", "chunk"])
def test_ragged_bytes_equal_host_encoder(eqw, orc, scope, codec):
    mats = _ragged()
    host = eqw.encode_host(mats, table_scope=scope, codec=codec)
    dev = eqw.encode_device([_dev(m) for m in mats], table_scope=scope, codec=codec).cpu().numpy()
    _oracle_decodes(orc, dev, mats)
    assert dev.size == host.size
    assert np.array_equal(dev, host)


def test_mixed_codecs_bytes_equal_host_encoder(eqw, orc):
    mats = _ragged()
    for i, m in enumerate(mats):
        m.codec = "huffman" if i % 2 else "rans"
    host = eqw.encode_host(mats)
    dev = eqw.encode_device([_dev(m) for m in mats]).cpu().numpy()
    _oracle_decodes(orc, dev, mats)
    assert np.array_equal(dev, host)


def test_huffman_long_codes_bytes_equal_host_encoder(eqw, orc):
    """Skewed counts over 254 E4M3 codes: many codes at the 12-bit limit, long refill look-ahead."""
    rng = np.random.default_rng(5)
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    p = 0.5 ** np.arange(codes.size) + 1e-6
    sym = rng.choice(codes, size=(64, 4096), p=p / p.sum()).astype(np.uint8)
    sym[0, :len(codes)] = codes
    m = W.Matrix(0, 0, "all", W.E4M3, sym, np.ones(64, np.float32))
    for scope in ("matrix", "chunk"):
        host = eqw.encode_host([m], table_scope=scope, codec="huffman")
        dev = eqw.encode_device([_dev(m)], table_scope=scope, codec="huffman").cpu().numpy()
        _oracle_decodes(orc, dev, [m])
        assert np.array_equal(dev, host), scope


@pytest.mark.parametrize("codec", ["rans", "huffman"])
@pytest.mark.parametrize("which", ["llama70b_int8_layer", "llama70b_e4m3_block", "llama7b_int8_block_with_outliers"])
def test_full_size_bytes_equal_host_encoder(eqw, orc, which, codec):
    mats = W.llama70b_int8_layer(0) if which == "llama70b_int8_layer" else getattr(W, which)()
    host = eqw.encode_host(mats, codec=codec)
    dev = eqw.encode_device([_dev(m) for m in mats], codec=codec).cpu().numpy()
    _oracle_decodes(orc, dev, mats)
    assert np.array_equal(dev, host)


def test_rejects_bad_inputs(eqw):
    m = W.random_e4m3_matrix(10, 8, 64)
    m.symbols[3, 3] = 0xFF                                               # E4M3 NaN code
    with pytest.raises(eqw.EqError) as e:
        eqw.encode_device([_dev(m)])
    assert e.value.code == 1
    m = W.random_int8_matrix(11, 8, 64, n_out=3)
    m.out_row, m.out_col = m.out_row[::-1].copy(), m.out_col[::-1].copy()  # not ascending
    with pytest.raises(eqw.EqError) as e:
        eqw.encode_device([_dev(m)])
    assert e.value.code == 1
    d = _dev(W.random_int8_matrix(12, 8, 64))
    buf = torch.zeros(8 * 64 + 8, dtype=torch.uint8, device="cuda")
    d.symbols = buf[1:1 + 8 * 64].view(8, 64)                              # not 8-byte aligned
    with pytest.raises(eqw.EqError) as e:
        eqw.encode_device([d])
    assert e.value.code == 1


def test_reports_required_size(eqw):
    m = W.random_int8_matrix(13, 64, 512)
    arr, keep = eqw._device_matrix_in_array([_dev(m)], "matrix")
    L = eqw.load()
    wb, ln = ctypes.c_size_t(), ctypes.c_size_t()
    assert L.eq_encode_device_workspace(arr, 1, ctypes.byref(wb)) == 0
    work = torch.empty(wb.value, dtype=torch.uint8, device="cuda")
    out = torch.zeros(16, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    rc = L.eq_encode_device(arr, 1, out.data_ptr(), 16, ctypes.byref(ln), work.data_ptr(), wb.value, s)
    assert rc == 6 and ln.value == eqw.encode_host([m]).size
    assert not out.any()
