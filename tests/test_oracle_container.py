"""Pins for the oracle's container writer / parser and its O-decode path.

Container v1 stores, per matrix, the chunked rANS bitstream, the fp32 row
scales, the outlier COO list and the metadata needed to decode (EntQuant
technical summary, section 2 "weight encoding": bitstream + scaling
parameters + metadata, scale overhead below 1 %).  O-decode must reproduce
O-direct exactly because the coding is lossless.
"""
import struct

import numpy as np
import pytest

from conftest import read_golden
import workloads as W


def _ragged_model():
    """Two layers of awkward shapes: tail chunks, partial 256-groups, cols not
    a multiple of 8, a 1x1 matrix, a single-symbol matrix, an empty matrix,
    E4M3 in the normal range, outliers."""
    mats = [
        W.random_int8_matrix(10, 300, 229, layer=0, index=0),          # 68700: 2 chunks, ragged tail
        W.random_int8_matrix(11, 1, 1, layer=0, index=1),              # one symbol
        W.random_e4m3_matrix(12, 77, 1000, alpha=1.0, layer=0, index=2),
        W.random_int8_matrix(13, 512, 256, n_out=16, layer=1, index=0),  # exactly 2 chunks
        W.random_int8_matrix(14, 3, 7, h_bits=1.0, layer=1, index=1),
    ]
    single = W.random_int8_matrix(15, 64, 1100, layer=1, index=2)
    single.symbols[:] = 0xFE
    mats.append(single)
    empty = W.random_int8_matrix(16, 0, 64, layer=1, index=3)
    mats.append(empty)
    return mats


def test_container_roundtrip_ragged(orc):
    mats = _ragged_model()
    blob = orc.encode_container(mats)
    parsed = orc.parse_container(blob)
    assert parsed["n_layers"] == 2 and len(parsed["matrices"]) == len(mats)
    dec = orc.decode_container(blob)
    for m, got, pm in zip(mats, dec, parsed["matrices"]):
        assert (pm["rows"], pm["cols"], pm["dtype"]) == (m.rows, m.cols, m.dtype)
        assert np.array_equal(pm["scales"], m.scales)
        assert np.array_equal(got, orc.dequant_direct(m))


def test_container_layer_filter(orc):
    mats = _ragged_model()
    blob = orc.encode_container(mats)
    l1 = orc.decode_container(blob, layer=1)
    assert len(l1) == 4
    for m, got in zip([m for m in mats if m.layer == 1], l1):
        assert np.array_equal(got, orc.dequant_direct(m))


def test_header_and_alignment(orc):
    mats = _ragged_model()
    blob = orc.encode_container(mats)
    magic, ver, hb, pb, lanes, group, cs, nl, nm = struct.unpack("<4s8I", bytes(blob[:36]))
    assert (magic, ver, hb, pb, lanes, group, cs, nl, nm) == (b"EQW1", 1, 64, 12, 32, 8, 65536, 2, 7)
    parsed = orc.parse_container(blob)
    for m in parsed["matrices"]:
        assert np.all(m["chunk_offsets"] % 16 == 0)
        assert m["chunk_offsets"][0] % 256 == 0


def test_single_symbol_matrix_has_empty_payload(orc):
    mats = _ragged_model()
    blob = orc.encode_container(mats)
    parsed = orc.parse_container(blob)
    m = [p for p in parsed["matrices"] if p["layer"] == 1 and p["index"] == 2][0]
    off = int(m["chunk_offsets"][0])
    n, nw, npres = struct.unpack("<3I", bytes(blob[off:off + 12]))
    assert (n, nw, npres) == (65536, 0, 1)  # first of two chunks (70400 symbols)


def test_outlier_placeholder_does_not_matter(orc):
    m = W.random_int8_matrix(20, 256, 256, n_out=16)
    blob = orc.encode_container([m])
    # the stream carries 0 at outlier positions; the decoded symbols show it
    parsed = orc.parse_container(blob)
    sym = orc.decode_matrix_symbols(parsed, 0)
    assert np.all(sym[m.out_row, m.out_col] == 0)
    assert np.array_equal(orc.decode_container(blob)[0], orc.dequant_direct(m))


def test_scale_overhead_below_page_bound(orc):
    """Page figure: scales cost < 1 % of the compressed weights (7B block, 2.1 bits)."""
    bound = float([r for r in read_golden("page_figures.txt") if r.startswith("scale_overhead")][0]
                  .split("=")[1])
    mats = W.llama7b_int8_block(2.1)
    blob = orc.encode_container(mats)
    scale_bytes = sum(4 * m.rows for m in mats)
    assert scale_bytes / blob.size < bound
    n = sum(m.n for m in mats)
    bits = 8.0 * blob.size / n
    assert 2.1 < bits < 2.2  # payload at the entropy plus < 5 % metadata

    # size bound per chunk: payload <= 1.01 x sum(n_c * H_c) / 8
    parsed = orc.parse_container(blob)
    payload = 0
    shannon = 0.0
    for pm, m in zip(parsed["matrices"], mats):
        flat = m.symbols.reshape(-1)
        offs = pm["chunk_offsets"]
        for k in range(pm["n_chunks"]):
            off = int(offs[k])
            n_k, nw = struct.unpack("<2I", bytes(blob[off:off + 8]))
            payload += 2 * nw
            c = np.bincount(flat[k * 65536:k * 65536 + n_k], minlength=256).astype(np.float64)
            p = c[c > 0] / n_k
            shannon += n_k * float(-(p * np.log2(p)).sum()) / 8.0
    assert payload <= 1.01 * shannon


def test_rejects_bad_inputs(orc):
    m = W.random_e4m3_matrix(30, 8, 64)
    m.symbols[0, 0] = 0x7F
    with pytest.raises(orc.OracleError):
        orc.encode_container([m])
    m = W.random_int8_matrix(31, 8, 64, n_out=4)
    m.out_row = m.out_row[::-1].copy()
    m.out_col = m.out_col[::-1].copy()
    with pytest.raises(orc.OracleError):
        orc.encode_container([m])
    m = W.random_int8_matrix(32, 8, 64, n_out=2)
    m.out_col[0] = 64
    with pytest.raises(orc.OracleError):
        orc.encode_container([m])


@pytest.mark.parametrize("what", ["magic", "version", "total", "table_sum", "payload", "chunk_index"])
def test_corrupt_container_detected(orc, what):
    m = W.random_int8_matrix(40, 256, 600)
    blob = orc.encode_container([m]).copy()
    parsed = orc.parse_container(blob)
    off0 = int(parsed["matrices"][0]["chunk_offsets"][0])
    if what == "magic":
        blob[0] ^= 1
    elif what == "version":
        blob[4] = 9
    elif what == "total":
        blob[48] ^= 0x10
    elif what == "table_sum":
        blob[off0 + 144 + 2] ^= 1      # f of the first table entry
    elif what == "payload":
        npres = struct.unpack("<I", bytes(blob[off0 + 8:off0 + 12]))[0]
        wo = off0 + ((144 + 4 * npres + 15) // 16) * 16
        blob[wo + 40] ^= 0x5A
    elif what == "chunk_index":
        ci = struct.unpack("<Q", bytes(blob[64 + 32:64 + 40]))[0]
        blob[ci + 8] ^= 0x20           # second chunk offset
    with pytest.raises(orc.OracleError):
        orc.decode_container(blob)
