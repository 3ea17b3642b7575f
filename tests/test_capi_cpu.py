"""Host-side checks of the C-ABI library libeqw.so (no GPU, no kernel launches).

* the library loads and exports every function include/eqw.h declares;
* its host encoder (eq_encoder_run) writes containers that the oracle's
  independent parser and scalar decoder turn back into exactly the input
  (lossless: EntQuant technical summary, section 2 "weight encoding");
* its parser (eq_model_open) accepts the oracle's containers and rejects
  corrupt ones -- it only reads the host copy, the device address given here
  is never dereferenced on the host.
"""
import ctypes
import os
import re
import struct

import numpy as np
import pytest

import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE_DEVICE_PTR = 0x7F0000000000  # 256-byte aligned; parsing never touches it


@pytest.fixture(scope="module")
def eqw():
    from entropy_coded_weight_b200 import build
    build.build()
    import entropy_coded_weight_b200 as E
    E.load()
    return E


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "eqw.h")).read()
    return re.findall(r"EQW_API\s+[\w\s\*]+?\b(eq_\w+)\s*\(", src)


def test_exports_every_declared_symbol(eqw):
    names = _declared_functions()
    assert len(names) >= 15
    lib = eqw.load()
    for n in names:
        assert hasattr(lib, n), n
    # and the binding covers all of them
    from entropy_coded_weight_b200._lib import SIGNATURES
    assert set(names) == set(SIGNATURES)


def test_version_and_status_strings(eqw):
    assert eqw.eq_format_version() == 1
    assert eqw.eq_status_string(0) == "ok"
    assert "corrupt" in eqw.eq_status_string(2)


def _ragged(seed=0):
    return [
        W.random_int8_matrix(seed + 1, 300, 229, layer=0, index=0),
        W.random_int8_matrix(seed + 2, 1, 1, layer=0, index=1),
        W.random_e4m3_matrix(seed + 3, 77, 1000, alpha=1.0, layer=0, index=2),
        W.random_int8_matrix(seed + 4, 512, 256, n_out=16, layer=1, index=0),
        W.random_int8_matrix(seed + 5, 3, 7, h_bits=1.0, layer=1, index=1),
        W.random_int8_matrix(seed + 6, 0, 64, layer=1, index=2),
    ]


def test_product_encoder_decodes_with_oracle(eqw, orc):
    mats = _ragged()
    single = W.random_int8_matrix(9, 64, 1100, layer=1, index=3)
    single.symbols[:] = 0x03
    mats.append(single)
    blob = eqw.encode_host(mats)
    parsed = orc.parse_container(blob)
    assert len(parsed["matrices"]) == len(mats)
    for m, got in zip(mats, orc.decode_container(blob)):
        assert np.array_equal(got, orc.dequant_direct(m))


def test_product_encoder_thread_count_does_not_change_bytes(eqw):
    mats = _ragged(20)
    a = eqw.encode_host(mats, n_threads=1)
    b = eqw.encode_host(mats, n_threads=8)
    assert np.array_equal(a, b)


def test_product_encoder_size_near_entropy(eqw, orc):
    """Payload within 1 % of the per-chunk Shannon bound (2.1 / 3.0 bits)."""
    for h in (2.1, 3.0):
        m = W.random_int8_matrix(30 + int(h * 10), 1024, 1024, h_bits=h)
        blob = eqw.encode_host([m])
        parsed = orc.parse_container(blob)
        pm = parsed["matrices"][0]
        flat = m.symbols.reshape(-1)
        payload, shannon = 0, 0.0
        for k in range(pm["n_chunks"]):
            off = int(pm["chunk_offsets"][k])
            n_k, nw = struct.unpack("<2I", bytes(blob[off:off + 8]))
            payload += 2 * nw
            c = np.bincount(flat[k * 65536:k * 65536 + n_k], minlength=256).astype(np.float64)
            p = c[c > 0] / n_k
            shannon += n_k * float(-(p * np.log2(p)).sum()) / 8
        assert payload <= 1.01 * shannon


def _open(eqw, blob):
    h = ctypes.c_void_p()
    rc = eqw.load().eq_model_open(FAKE_DEVICE_PTR, blob.size, blob.ctypes.data, ctypes.byref(h))
    return rc, h


def test_parser_accepts_oracle_containers(eqw, orc):
    mats = _ragged(40)
    blob = orc.encode_container(mats)
    rc, h = _open(eqw, blob)
    assert rc == 0
    L = eqw.load()
    nl, nm = ctypes.c_uint32(), ctypes.c_uint32()
    assert L.eq_model_counts(h, ctypes.byref(nl), ctypes.byref(nm)) == 0
    assert (nl.value, nm.value) == (2, 6)
    info = eqw.eq_matrix_info()
    assert L.eq_matrix_get_info(h, 3, ctypes.byref(info)) == 0
    assert (info.layer, info.index, info.rows, info.cols, info.n_outliers, info.dtype) == (1, 0, 512, 256, 16, 1)
    offs = (ctypes.c_size_t * 3)()
    total = ctypes.c_size_t()
    assert L.eq_block_layout(h, 1, offs, 3, ctypes.byref(total)) == 0
    assert list(offs) == [0, 512 * 256 * 2, 512 * 256 * 2 + 256]
    assert total.value == 512 * 256 * 2 + 256  # 3x7 bf16 rounded up to 256 B, empty matrix 0
    L.eq_model_close(h)


def test_parser_rejects_misaligned_device_pointer(eqw, orc):
    blob = orc.encode_container([W.random_int8_matrix(50, 16, 16)])
    h = ctypes.c_void_p()
    assert eqw.load().eq_model_open(FAKE_DEVICE_PTR + 8, blob.size, blob.ctypes.data, ctypes.byref(h)) == 1


@pytest.mark.parametrize("what", ["magic", "version", "constants", "total", "dtype", "n_chunks",
                                  "chunk_index", "n_syms", "table_sum", "table_order", "state", "outlier"])
def test_parser_rejects_corruption(eqw, orc, what):
    m = W.random_int8_matrix(60, 256, 600, n_out=4)
    blob = orc.encode_container([m]).copy()
    parsed = orc.parse_container(blob)
    pm = parsed["matrices"][0]
    off0 = int(pm["chunk_offsets"][0])
    d = 64  # directory entry 0
    ci, so, oo = struct.unpack("<3Q", bytes(blob[d + 32:d + 56]))
    if what == "magic":
        blob[1] ^= 0xFF
    elif what == "version":
        blob[4] = 2
    elif what == "constants":
        blob[12] = 11
    elif what == "total":
        blob[48] ^= 1
    elif what == "dtype":
        blob[d + 8] = 7
    elif what == "n_chunks":
        blob[d + 12] += 1
    elif what == "chunk_index":
        blob[ci + 8] ^= 0x10
    elif what == "n_syms":
        blob[off0] ^= 1
    elif what == "table_sum":
        blob[off0 + 144 + 2] ^= 1
    elif what == "table_order":
        t0 = bytes(blob[off0 + 144:off0 + 148])
        t1 = bytes(blob[off0 + 148:off0 + 152])
        blob[off0 + 144:off0 + 148] = np.frombuffer(t1, np.uint8)
        blob[off0 + 148:off0 + 152] = np.frombuffer(t0, np.uint8)
    elif what == "state":
        blob[off0 + 16:off0 + 20] = np.frombuffer(struct.pack("<I", 1000), np.uint8)
    elif what == "outlier":
        blob[oo:oo + 4] = np.frombuffer(struct.pack("<I", 256), np.uint8)
    rc, _ = _open(eqw, blob)
    assert rc in (2, 3)


def test_encoder_rejects_bad_inputs(eqw):
    m = W.random_e4m3_matrix(70, 8, 64)
    m.symbols[3, 3] = 0xFF
    with pytest.raises(eqw.EqError):
        eqw.encode_host([m])
    m = W.random_int8_matrix(71, 8, 64, n_out=3)
    m.out_row, m.out_col = m.out_row[::-1].copy(), m.out_col[::-1].copy()
    with pytest.raises(eqw.EqError):
        eqw.encode_host([m])
    a = W.random_int8_matrix(72, 8, 64, layer=0)
    b = W.random_int8_matrix(73, 8, 64, layer=2)  # layer 1 missing
    with pytest.raises(eqw.EqError):
        eqw.encode_host([a, b])


def test_encoder_reports_required_size(eqw):
    m = W.random_int8_matrix(80, 64, 64)
    arr, keep = eqw._matrix_in_array([m])
    out = np.zeros(16, np.uint8)
    need = ctypes.c_size_t()
    rc = eqw.load().eq_encode_host(arr, 1, 1, out.ctypes.data, out.size, ctypes.byref(need))
    assert rc == 6 and need.value > 16 and not out.any()
    out = np.zeros(need.value, np.uint8)
    assert eqw.load().eq_encode_host(arr, 1, 1, out.ctypes.data, out.size, ctypes.byref(need)) == 0
    assert np.array_equal(out, eqw.encode_host([m]))


def test_table_scope_matrix_vs_chunk(eqw, orc):
    """Default: one table per matrix (identical in every chunk); per-chunk on request.
    Both decode exactly with the oracle; the parser flags uniform tables."""
    m = W.random_int8_matrix(90, 700, 300, h_bits=2.4)  # 4 chunks
    L = eqw.load()
    for scope, uniform in (("matrix", 1), ("chunk", 0)):
        blob = eqw.encode_host([m], table_scope=scope)
        assert np.array_equal(orc.decode_container(blob)[0], orc.dequant_direct(m))
        rc, h = _open(eqw, blob)
        assert rc == 0
        info = eqw.eq_matrix_info()
        assert L.eq_matrix_get_info(h, 0, ctypes.byref(info)) == 0
        assert info.uniform_table == uniform
        L.eq_model_close(h)
    # the oracle's own containers use per-chunk tables
    rc, h = _open(eqw, orc.encode_container([m]))
    info = eqw.eq_matrix_info()
    assert rc == 0 and L.eq_matrix_get_info(h, 0, ctypes.byref(info)) == 0 and info.uniform_table == 0
    L.eq_model_close(h)


def test_matrix_table_costs_little(eqw):
    """A shared table adds well under 0.5 % to the payload on stationary data."""
    m = W.random_int8_matrix(91, 2048, 2048, h_bits=2.1)
    a = eqw.encode_host([m], table_scope="matrix").size
    b = eqw.encode_host([m], table_scope="chunk").size
    assert a <= b * 1.005


# ---- Huffman codec (EntroLLM technical overview, "Huffman weight encoding") ----

def _ragged_consistent(seed=0):
    mats = [
        W.random_int8_matrix(seed + 1, 300, 229, layer=0, index=0),
        W.random_int8_matrix(seed + 2, 1, 1, layer=0, index=1),
        W.random_e4m3_matrix(seed + 3, 77, 1000, alpha=1.0, layer=0, index=2),
        W.random_int8_matrix(seed + 4, 512, 256, n_out=16, layer=1, index=0),
        W.random_int8_matrix(seed + 5, 0, 64, layer=1, index=1),
        W.random_int8_matrix(seed + 6, 700, 1300, h_bits=3.0, n_out=5, layer=1, index=2),
    ]
    single = W.random_int8_matrix(seed + 7, 64, 1100, layer=1, index=3)
    single.symbols[:] = 0x03
    mats.append(single)
    return mats


@pytest.mark.parametrize("scope", ["matrix", "chunk"])
def test_product_huffman_encoder_decodes_with_oracle(eqw, orc, scope):
    mats = _ragged_consistent(100)
    blob = eqw.encode_host(mats, table_scope=scope, codec="huffman")
    for m, got in zip(mats, orc.decode_container(blob)):
        assert np.array_equal(got, orc.dequant_direct(m))
    rc, h = _open(eqw, blob)
    assert rc == 0
    info = eqw.eq_matrix_info()
    assert eqw.load().eq_matrix_get_info(h, 0, ctypes.byref(info)) == 0 and info.codec == 1
    eqw.load().eq_model_close(h)


def test_parser_accepts_oracle_huffman_containers(eqw, orc):
    blob = orc.encode_container(_ragged_consistent(200), codec="huffman")
    rc, h = _open(eqw, blob)
    assert rc == 0
    eqw.load().eq_model_close(h)


def test_mixed_codecs_in_one_container(eqw, orc):
    mats = _ragged_consistent(300)
    for i, m in enumerate(mats):
        m.codec = "huffman" if i % 2 else "rans"
    blob = eqw.encode_host(mats)
    parsed = orc.parse_container(blob)
    assert [pm["codec"] for pm in parsed["matrices"]] == [i % 2 for i in range(len(mats))]
    for m, got in zip(mats, orc.decode_container(blob)):
        assert np.array_equal(got, orc.dequant_direct(m))


@pytest.mark.parametrize("what", ["kraft", "order", "long_code", "single_with_words", "codec"])
def test_parser_rejects_huffman_corruption(eqw, orc, what):
    m = W.random_int8_matrix(400, 256, 600)
    blob = eqw.encode_host([m], codec="huffman").copy()
    off0 = int(orc.parse_container(blob)["matrices"][0]["chunk_offsets"][0])
    t0 = off0 + 16
    if what == "kraft":
        blob[t0 + 2] += 1  # first (shortest) code one bit longer: Kraft sum < 1
    elif what == "order":
        a, b = bytes(blob[t0:t0 + 4]), bytes(blob[t0 + 4:t0 + 8])
        blob[t0:t0 + 4] = np.frombuffer(b, np.uint8)
        blob[t0 + 4:t0 + 8] = np.frombuffer(a, np.uint8)
    elif what == "long_code":
        npres = int(np.frombuffer(bytes(blob[off0 + 8:off0 + 12]), "<u4")[0])
        blob[t0 + 4 * (npres - 1) + 2] = 13
    elif what == "single_with_words":
        s = W.random_int8_matrix(401, 64, 64)
        s.symbols[:] = 1
        blob = eqw.encode_host([s], codec="huffman").copy()
        o = int(orc.parse_container(blob)["matrices"][0]["chunk_offsets"][0])
        blob[o + 4] = 1  # claims a word it does not have
    elif what == "codec":
        blob[64 + 28] = 7
    rc, _ = _open(eqw, blob)
    assert rc in (2, 3)


def test_huffman_size_near_entropy(eqw, orc):
    """Huffman payload within one bit per symbol of the per-chunk Shannon bound
    (integer code lengths) and never below it."""
    m = W.random_int8_matrix(402, 1024, 1024, h_bits=2.1)
    blob = eqw.encode_host([m], codec="huffman", table_scope="chunk")
    pm = orc.parse_container(blob)["matrices"][0]
    flat = m.symbols.reshape(-1)
    payload, shannon = 0, 0.0
    for k in range(pm["n_chunks"]):
        off = int(pm["chunk_offsets"][k])
        n_k, nw = struct.unpack("<2I", bytes(blob[off:off + 8]))
        payload += 2 * nw
        c = np.bincount(flat[k * 65536:k * 65536 + n_k], minlength=256).astype(np.float64)
        p = c[c > 0] / n_k
        shannon += n_k * float(-(p * np.log2(p)).sum()) / 8
    assert shannon <= payload <= shannon + flat.size / 8


def test_sm_limit_is_a_host_setting(eqw, orc):
    blob = orc.encode_container(_ragged(41))
    rc, h = _open(eqw, blob)
    assert rc == 0
    L = eqw.load()
    assert L.eq_model_set_sm_limit(h, 17) == 0
    assert L.eq_model_set_sm_limit(h, 0) == 0
    assert L.eq_model_set_sm_limit(None, 4) == 1  # EQ_ERR_INVALID_ARG
    L.eq_model_close(h)
