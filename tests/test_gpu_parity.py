"""GPU parity: the CUDA decode path vs the CPU oracle, bit for bit (0 ULP).

All calls go through the C ABI (libeqw.so via the ctypes binding).  Expected
values come only from the oracle: O-direct (dequantised generator symbols,
unique because the coding is lossless -- EntQuant technical summary,
section 2) and, for containers written by the oracle's own encoder, the
decode must match the same O-direct.
"""
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


def _decode_matrices(E, blob, per_matrix=True):
    """Upload, open, decode every matrix; returns ([uint16 arrays], status)."""
    d_blob = E.upload(blob)
    model = E.Model(d_blob, blob)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    if per_matrix:
        for i in range(model.n_matrices):
            inf = model.info(i)
            out = torch.empty(max(1, inf.rows * inf.cols), dtype=torch.int16, device="cuda")
            model.decode_matrix(i, out, status)
            outs.append((out, inf.rows, inf.cols))
    else:
        for layer in range(model.n_layers):
            offs, total = model.block_layout(layer)
            buf = torch.empty(max(total, 16), dtype=torch.uint8, device="cuda")
            model.decode_block(layer, buf, status)
            for i, off in zip(model.layer_matrices(layer), offs):
                inf = model.info(i)
                outs.append((buf[off:off + 2 * inf.rows * inf.cols].view(torch.int16), inf.rows, inf.cols))
    torch.cuda.synchronize()
    res = [o[: r * c].cpu().numpy().view(np.uint16).reshape(r, c) for o, r, c in outs]
    st = int(status.item())
    model.close()
    return res, st


def _assert_parity(got, mats, orc):
    for g, m in zip(got, mats):
        want = orc.dequant_direct(m)
        if not np.array_equal(g, want):
            bad = np.argwhere(g != want)
            raise AssertionError(f"matrix {m.layer}/{m.index} {m.rows}x{m.cols}: {len(bad)} mismatches, "
                                 f"first at {bad[0].tolist()}: got {g[tuple(bad[0])]:#06x} "
                                 f"want {want[tuple(bad[0])]:#06x}")


def _ragged():
    mats = [
        W.random_int8_matrix(1, 300, 229, layer=0, index=0),            # cols % 8 != 0, ragged tail
        W.random_int8_matrix(2, 1, 1, layer=0, index=1),                # one symbol
        W.random_e4m3_matrix(3, 77, 1000, alpha=1.0, layer=0, index=2),  # E4M3 normal range, tail
        W.random_int8_matrix(4, 512, 256, n_out=16, layer=0, index=3),  # exactly two chunks + outliers
        W.random_int8_matrix(5, 3, 7, h_bits=1.0, layer=1, index=0),
        W.random_int8_matrix(6, 0, 64, layer=1, index=1),               # empty
        W.random_int8_matrix(7, 129, 1032, h_bits=7.9, layer=1, index=2),  # near-uniform: ~8 bits/sym
        W.random_int8_matrix(8, 1000, 264, h_bits=0.05, layer=1, index=3),  # very low entropy
    ]
    single = W.random_int8_matrix(9, 64, 1100, layer=1, index=4)
    single.symbols[:] = 0x81                                             # f = 4096 chunks
    mats.append(single)
    mostly = W.random_int8_matrix(10, 64, 1024, layer=1, index=5)
    mostly.symbols[:] = 0
    mostly.symbols[5, 7] = 0x7F                                           # one rare symbol (f = 1)
    mats.append(mostly)
    return mats


@pytest.mark.parametrize("encoder", ["product", "product-chunk-tables", "oracle"])
@pytest.mark.parametrize("per_matrix", [True, False])
def test_ragged_shapes_bit_exact(eqw, orc, encoder, per_matrix):
    mats = _ragged()
    if encoder == "oracle":
        blob = orc.encode_container(mats)
    else:
        blob = eqw.encode_host(mats, table_scope="chunk" if encoder.endswith("tables") else "matrix")
    got, st = _decode_matrices(eqw, blob, per_matrix)
    assert st == 0
    _assert_parity(got, mats, orc)


def test_every_tail_length(eqw, orc):
    """n = 1..700 symbols in one chunk: every partial group / lane mask."""
    mats = [W.random_int8_matrix(100 + n, 1, n, h_bits=2.5, layer=0, index=i) for i, n in
            enumerate(list(range(1, 300)) + [511, 512, 513, 700])]
    blob = eqw.encode_host(mats)
    got, st = _decode_matrices(eqw, blob, per_matrix=False)
    assert st == 0
    _assert_parity(got, mats, orc)


def test_e4m3_all_codes_and_signed_zero(eqw, orc):
    rng = np.random.default_rng(5)
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    sym = rng.choice(codes, size=(64, 4096)).astype(np.uint8)
    sym[0, :len(codes)] = codes
    sc = np.exp(rng.uniform(-90, 80, size=64)).astype(np.float32)
    sc[1] = np.float32(1e-40)  # subnormal scale: products land on bf16 subnormals
    m = W.Matrix(0, 0, "all", W.E4M3, sym, sc)
    got, st = _decode_matrices(eqw, eqw.encode_host([m]))
    assert st == 0
    _assert_parity(got, [m], orc)


@pytest.mark.parametrize("cols", [4096, 1000, 1001])
def test_e4m3_large_scales_each_layout(eqw, orc, cols):
    """Scales >= 2^8 take the two-multiply E4M3 path; cols picks the output layout
    (multiple of 256: warp-uniform rows; of 8: per-lane rows; else element-wise)."""
    rng = np.random.default_rng(cols)
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    sym = rng.choice(codes, size=(40, cols)).astype(np.uint8)
    sc = np.exp(rng.uniform(-20, 70, size=40)).astype(np.float32)
    sc[0] = np.float32(300.0)
    m = W.Matrix(0, 0, "big", W.E4M3, sym, sc)
    for scope in ("matrix", "chunk"):
        got, st = _decode_matrices(eqw, eqw.encode_host([m], table_scope=scope))
        assert st == 0
        _assert_parity(got, [m], orc)


def test_int8_all_codes_extreme_scales(eqw, orc):
    rng = np.random.default_rng(6)
    sym = rng.integers(0, 256, size=(32, 2048)).astype(np.uint8)
    sc = np.exp(rng.uniform(-100, 85, size=32)).astype(np.float32)
    sc[3] = np.float32(3e38)  # overflows to inf after the fp32 multiply
    m = W.Matrix(0, 0, "all", W.INT8, sym, sc)
    got, st = _decode_matrices(eqw, eqw.encode_host([m]))
    assert st == 0
    _assert_parity(got, [m], orc)


def test_workload1_single_matrix(eqw, orc):
    mats = W.single_matrix()
    for blob in (eqw.encode_host(mats), orc.encode_container(mats)):
        got, st = _decode_matrices(eqw, blob, per_matrix=False)
        assert st == 0
        _assert_parity(got, mats, orc)


@pytest.mark.parametrize("h,scope", [(2.1, "matrix"), (3.0, "matrix"), (2.1, "chunk")])
def test_workload2_llama7b_block(eqw, orc, h, scope):
    mats = W.llama7b_int8_block(h)
    got, st = _decode_matrices(eqw, eqw.encode_host(mats, table_scope=scope), per_matrix=False)
    assert st == 0
    _assert_parity(got, mats, orc)


@pytest.mark.parametrize("scope", ["matrix", "chunk"])
def test_workload3_llama70b_e4m3_block(eqw, orc, scope):
    mats = W.llama70b_e4m3_block(2.1)
    for m in mats:
        assert abs(W.empirical_entropy_bits(m.symbols) - 2.1) < 0.02
    got, st = _decode_matrices(eqw, eqw.encode_host(mats, table_scope=scope), per_matrix=False)
    assert st == 0
    _assert_parity(got, mats, orc)


def test_workload4_outliers(eqw, orc):
    mats = W.llama7b_int8_block_with_outliers()
    assert len(mats[6].out_row) == 16
    got, st = _decode_matrices(eqw, eqw.encode_host(mats), per_matrix=False)
    assert st == 0
    _assert_parity(got, mats, orc)
    # the 16 positions carry bf16(v), not the placeholder's dequantised value
    d = mats[6]
    vals = torch.from_numpy(d.out_val).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got[6][d.out_row, d.out_col], vals)


# ---- device-side validation (corrupt device bytes; every access stays in bounds) ----

def _corrupt_and_decode(E, blob, mutate):
    d_blob = E.upload(blob)
    model = E.Model(d_blob, blob)     # validated on the clean host copy
    mutate(d_blob)                    # then the device copy is damaged
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    offs, total = model.block_layout(0)
    out = torch.empty(total, dtype=torch.uint8, device="cuda")
    model.decode_block(0, out, status)
    torch.cuda.synchronize()
    model.close()
    return int(status.item())


@pytest.mark.parametrize("what,bit", [("payload", "EQ_DEV_BAD_END"), ("table", "EQ_DEV_BAD_TABLE"),
                                      ("n_syms", "EQ_DEV_BAD_HEADER"), ("state_low", "EQ_DEV_BAD_STATE"),
                                      ("state", "EQ_DEV_BAD_END"), ("outlier", "EQ_DEV_BAD_OUTLIER")])
def test_device_detects_corruption(eqw, orc, what, bit):
    m = W.random_int8_matrix(200, 512, 512, n_out=4)
    blob = eqw.encode_host([m])
    parsed = orc.parse_container(blob)
    off0 = int(parsed["matrices"][0]["chunk_offsets"][0])
    npres = int(np.frombuffer(bytes(blob[off0 + 8:off0 + 12]), "<u4")[0])
    words = off0 + ((144 + 4 * npres + 15) // 16) * 16
    oo = int(np.frombuffer(bytes(blob[64 + 48:64 + 56]), "<u8")[0])

    def mutate(d):
        if what == "payload":
            d[words + 100] ^= 0x40
        elif what == "table":
            d[off0 + 144 + 2] ^= 0x01
        elif what == "n_syms":
            d[off0] ^= 0x01
        elif what == "state_low":
            d[off0 + 16 + 4 * 5 + 2] = 0
            d[off0 + 16 + 4 * 5 + 3] = 0
        elif what == "state":
            d[off0 + 16 + 4 * 9 + 3] ^= 0x10
        elif what == "outlier":
            d[oo + 3] = 0x7F  # row far out of range
    st = _corrupt_and_decode(eqw, blob, mutate)
    assert st & getattr(eqw, bit), (what, st)


def test_api_argument_errors(eqw):
    m = W.random_int8_matrix(300, 64, 64)
    blob = eqw.encode_host([m])
    d_blob = eqw.upload(blob)
    model = eqw.Model(d_blob, blob)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    small = torch.empty(100, dtype=torch.uint8, device="cuda")
    with pytest.raises(eqw.EqError) as e:
        model.decode_block(0, small, status)
    assert e.value.code == 6
    with pytest.raises(eqw.EqError) as e:
        model.decode_matrix(5, small, status)
    assert e.value.code == 1
    model.close()
