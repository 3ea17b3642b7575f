"""GPU parity of the Huffman codec (EntroLLM technical overview, "Huffman
weight encoding" and "parallel decoding strategy"): containers written by the
product's host encoder or by the oracle, decoded by eq_decode_kernel's
Huffman instances, compared bit for bit with the oracle's O-direct weights.
"""
import numpy as np
import pytest
import torch

import workloads as W
from test_gpu_parity import _assert_parity, _decode_matrices, _ragged

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def eqw():
    from entropy_coded_weight_b200 import build
    build.build()
    import entropy_coded_weight_b200 as E
    E.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return E


@pytest.mark.parametrize("encoder", ["product", "product-chunk-tables", "oracle"])
@pytest.mark.parametrize("per_matrix", [True, False])
def test_ragged_shapes_bit_exact(eqw, orc, encoder, per_matrix):
    mats = _ragged()
    if encoder == "oracle":
        blob = orc.encode_container(mats, codec="huffman")
    else:
        blob = eqw.encode_host(mats, table_scope="chunk" if encoder.endswith("tables") else "matrix",
                               codec="huffman")
    got, st = _decode_matrices(eqw, blob, per_matrix)
    assert st == 0
    _assert_parity(got, mats, orc)


def test_every_tail_length(eqw, orc):
    mats = [W.random_int8_matrix(100 + n, 1, n, h_bits=2.5, layer=0, index=i) for i, n in
            enumerate(list(range(1, 300)) + [511, 512, 513, 700])]
    for scope in ("matrix", "chunk"):
        got, st = _decode_matrices(eqw, eqw.encode_host(mats, table_scope=scope, codec="huffman"), False)
        assert st == 0
        _assert_parity(got, mats, orc)


def test_e4m3_all_codes_long_codes(eqw, orc):
    """254 codes with skewed counts: many codes at the 12-bit limit."""
    rng = np.random.default_rng(5)
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    p = 0.5 ** np.arange(codes.size) + 1e-6
    sym = rng.choice(codes, size=(64, 4096), p=p / p.sum()).astype(np.uint8)
    sym[0, :len(codes)] = codes
    sc = np.exp(rng.uniform(-90, 80, size=64)).astype(np.float32)
    m = W.Matrix(0, 0, "all", W.E4M3, sym, sc)
    for scope in ("matrix", "chunk"):
        blob = eqw.encode_host([m], table_scope=scope, codec="huffman")
        got, st = _decode_matrices(eqw, blob)
        assert st == 0
        _assert_parity(got, [m], orc)


def test_mixed_codecs_in_one_block(eqw, orc):
    mats = _ragged()
    for i, m in enumerate(mats):
        m.codec = "huffman" if i % 2 else "rans"
    got, st = _decode_matrices(eqw, eqw.encode_host(mats), per_matrix=False)
    assert st == 0
    _assert_parity(got, mats, orc)


@pytest.mark.parametrize("which", ["single_matrix", "llama7b_int8_block", "llama70b_e4m3_block",
                                   "llama7b_int8_block_with_outliers", "llama70b_int8_layer"])
def test_workloads_full_size(eqw, orc, which):
    mats = W.llama70b_int8_layer(0) if which == "llama70b_int8_layer" else getattr(W, which)()
    got, st = _decode_matrices(eqw, eqw.encode_host(mats, codec="huffman"), per_matrix=False)
    assert st == 0
    _assert_parity(got, mats, orc)


def _corrupt_and_decode(E, blob, mutate):
    d_blob = E.upload(blob)
    model = E.Model(d_blob, blob)
    mutate(d_blob)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    offs, total = model.block_layout(0)
    out = torch.empty(total, dtype=torch.uint8, device="cuda")
    model.decode_block(0, out, status)
    torch.cuda.synchronize()
    model.close()
    return int(status.item())


@pytest.mark.parametrize("scope", ["matrix", "chunk"])
def test_device_detects_corruption(eqw, orc, scope):
    m = W.random_int8_matrix(200, 512, 512, n_out=4)
    blob = eqw.encode_host([m], table_scope=scope, codec="huffman")
    off0 = int(orc.parse_container(blob)["matrices"][0]["chunk_offsets"][0])
    npres = int(np.frombuffer(bytes(blob[off0 + 8:off0 + 12]), "<u4")[0])
    n_words = int(np.frombuffer(bytes(blob[off0 + 4:off0 + 8]), "<u4")[0])
    words = off0 + ((16 + 4 * npres + 15) // 16) * 16

    def table(d):
        d[off0 + 16 + 2] += 1               # shortest code one bit longer: not a complete code

    def n_syms(d):
        d[off0] ^= 0x01

    def payload(d):
        d[words:words + 2 * n_words] ^= 0xFF  # every bit of the chunk's words

    assert _corrupt_and_decode(eqw, blob, table) & eqw.EQ_DEV_BAD_TABLE
    assert _corrupt_and_decode(eqw, blob, n_syms) & eqw.EQ_DEV_BAD_HEADER
    assert _corrupt_and_decode(eqw, blob, payload) & eqw.EQ_DEV_BAD_END


@pytest.mark.parametrize("scope", ["matrix", "chunk"])
def test_fused_gemv_within_bound(eqw, orc, scope):
    """Fused decode + GEMV on Huffman matrices: the bound of test_gpu_fused_gemv."""
    from test_gpu_fused_gemv import _bits, _bound_ok, _n_out_rows, _run_matrices, _x_for
    mats = [W.random_int8_matrix(300, 64, 512, layer=0, index=0),
            W.random_int8_matrix(301, 300, 1024, n_out=7, layer=0, index=1),
            W.random_e4m3_matrix(302, 96, 4096, alpha=1.0, layer=0, index=2),
            W.random_int8_matrix(303, 1024, 8192, layer=0, index=3)]
    single = W.random_int8_matrix(304, 40, 2048, layer=0, index=4)
    single.symbols[:] = 0x05
    mats.append(single)
    blob = eqw.encode_host(mats, table_scope=scope, codec="huffman")
    for per_matrix in (True, False):
        st, ys = _run_matrices(eqw, blob, mats, per_matrix=per_matrix)
        assert st == 0
        for m, y in zip(mats, ys):
            ref, mag = orc.gemv_exact(orc.dequant_direct(m), _bits(_x_for(m)))
            ok, info = _bound_ok(y, ref, mag, m.cols, _n_out_rows(m))
            assert ok, (scope, per_matrix, m.index, info)


def test_fused_gemv_needs_cols_multiple_of_256(eqw):
    m = W.random_int8_matrix(305, 64, 500)
    blob = eqw.encode_host([m], codec="huffman")
    model = eqw.Model(eqw.upload(blob), blob)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(eqw.EqError) as e:
        model.decode_gemv_matrix(0, torch.zeros(512, dtype=torch.bfloat16, device="cuda"),
                                 torch.zeros(64, dtype=torch.float32, device="cuda"), status)
    assert e.value.code == 3
    model.close()
