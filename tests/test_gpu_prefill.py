"""GPU tests of the prefill path: eq_decode_symbols + eq_gemm_symbols (tcgen05).

Expected values come from the oracle only (oracle.stream_symbols,
oracle.gemm_symbols_exact).  One-hot token rows make every output a single
product, value(sym) * x rounded once by the row scale, so those cases are
compared bit for bit; random tokens are compared with an fp32 accumulation
bound: the products are exact, the tensor core sums K = 16 per instruction
and the accumulator adds one instruction's partial sum per step, so the sum
has depth at most cols / 16 + 4; the test allows
(cols / 16 + 32) * 2^-22 * sum |terms| (four times the unit roundoff, for the
tensor core's internal alignment) plus one rounding for the scale.
"""
import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

EQ_ERR_UNSUPPORTED = 3


@pytest.fixture(scope="module")
def eqw():
    from entropy_coded_weight_b200 import build
    build.build()
    import entropy_coded_weight_b200 as E
    E.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return E


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _open(eqw, mats, **kw):
    blob = eqw.encode_host(mats, **kw)
    return eqw.Model(eqw.upload(blob), blob)


def test_one_cta_one_hot_bit_exact(eqw, orc):
    """Smallest case first: one 128 x 128 tile, one K slab."""
    m = W.random_int8_matrix(1, 128, 64, h_bits=3.0)
    model = _open(eqw, [m])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sym = torch.empty(128 * 64, dtype=torch.uint8, device="cuda")
    model.decode_symbols(0, sym, status)
    x = torch.zeros(64, 64, dtype=torch.bfloat16)
    for t in range(64):
        x[t, t] = float(1 + t % 5)
    y = torch.full((64, 128), float("nan"), dtype=torch.float32, device="cuda")
    model.gemm_symbols(0, sym, x.cuda(), y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert np.array_equal(sym.cpu().numpy().reshape(128, 64), orc.stream_symbols(m))
    ref, _ = orc.gemm_symbols_exact(m, _bits(x))
    assert np.array_equal(y.cpu().numpy().view(np.uint32), ref.astype(np.float32).view(np.uint32))
    model.close()


@pytest.mark.parametrize("codec", ["rans", "huffman"])
@pytest.mark.parametrize("scope", ["matrix", "chunk"])
def test_decode_symbols_bit_exact(eqw, orc, codec, scope):
    mats = [W.random_int8_matrix(2, 300, 229, layer=0, index=0),
            W.random_e4m3_matrix(3, 77, 1000, alpha=1.0, layer=0, index=1),
            W.random_int8_matrix(4, 512, 256, n_out=16, layer=0, index=2),
            W.random_int8_matrix(5, 256, 8192, layer=0, index=3)]
    model = _open(eqw, mats, codec=codec, table_scope=scope)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for i, m in enumerate(mats):
        out = torch.empty(max(1, m.rows * m.cols), dtype=torch.uint8, device="cuda")
        model.decode_symbols(i, out, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert np.array_equal(out[:m.rows * m.cols].cpu().numpy().reshape(m.rows, m.cols), orc.stream_symbols(m)), i
    model.close()


@pytest.mark.parametrize("dtype", ["int8", "e4m3"])
def test_one_hot_tokens_bit_exact_multi_tile(eqw, orc, dtype):
    m = (W.random_int8_matrix(6, 256, 512, h_bits=4.0) if dtype == "int8"
         else W.random_e4m3_matrix(6, 256, 512, alpha=1.0))
    tokens = 130
    rng = np.random.default_rng(7)
    cols = rng.integers(0, 512, size=tokens)
    x = torch.zeros(tokens, 512, dtype=torch.bfloat16)
    x[torch.arange(tokens), torch.from_numpy(cols)] = torch.from_numpy(
        rng.choice([-2.0, -0.5, 1.0, 3.0], size=tokens).astype(np.float32)).to(torch.bfloat16)
    model = _open(eqw, [m])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sym = torch.empty(256 * 512, dtype=torch.uint8, device="cuda")
    model.decode_symbols(0, sym, status)
    y = torch.empty(tokens, 256, dtype=torch.float32, device="cuda")
    model.gemm_symbols(0, sym, x.cuda(), y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, _ = orc.gemm_symbols_exact(m, _bits(x))
    assert np.array_equal(y.cpu().numpy().view(np.uint32), ref.astype(np.float32).view(np.uint32))
    model.close()


def _check_bound(y, ref, mag, cols):
    u = 2.0 ** -22
    h = cols / 16 + 32
    err = np.abs(y.astype(np.float64) - ref)
    tol = h * u * mag + 2.0 ** -24 * np.abs(ref) + 1e-30
    bad = err > tol
    assert not bad.any(), (np.argwhere(bad)[:3], err[bad][:3], tol[bad][:3])


@pytest.mark.parametrize("shape,tokens,kind", [((128, 64), 1, "int8"), ((256, 1024), 7, "e4m3"),
                                               ((1024, 8192), 128, "int8"), ((384, 2048), 300, "int8-outliers")])
def test_random_tokens_within_bound(eqw, orc, shape, tokens, kind):
    rows, cols = shape
    if kind == "e4m3":
        m = W.random_e4m3_matrix(10, rows, cols, alpha=1.0)
    else:
        m = W.random_int8_matrix(11, rows, cols, h_bits=2.1, n_out=12 if kind.endswith("outliers") else 0)
    x = W.gemv_activation(3, 1, tokens * cols).reshape(tokens, cols)
    model = _open(eqw, [m])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sym = torch.empty(rows * cols, dtype=torch.uint8, device="cuda")
    model.decode_symbols(0, sym, status)
    y = torch.empty(tokens, rows, dtype=torch.float32, device="cuda")
    model.gemm_symbols(0, sym, x.cuda(), y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, mag = orc.gemm_symbols_exact(m, _bits(x))
    _check_bound(y.cpu().numpy(), ref, mag, cols)
    model.close()


@pytest.mark.parametrize("which", [0, 4, 6])
def test_llama70b_matrices_256_tokens(eqw, orc, which):
    """Full-size q (8192 x 8192), gate (28672 x 8192) and down (8192 x 28672) of a 70B layer."""
    rows, cols = W.LLAMA70B_BLOCK[which]
    m = W._int8_matrix(5, 0, which, (rows, cols), 2.1)
    tokens = 256
    x = W.gemv_activation(4, which, tokens * cols).reshape(tokens, cols)
    model = _open(eqw, [m])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sym = torch.empty(rows * cols, dtype=torch.uint8, device="cuda")
    model.decode_symbols(0, sym, status)
    y = torch.empty(tokens, rows, dtype=torch.float32, device="cuda")
    model.gemm_symbols(0, sym, x.cuda(), y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, mag = orc.gemm_symbols_exact(m, _bits(x))
    _check_bound(y.cpu().numpy(), ref, mag, cols)
    model.close()


def test_unsupported_shapes(eqw):
    m = W.random_int8_matrix(12, 100, 64)
    model = _open(eqw, [m])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sym = torch.empty(100 * 64, dtype=torch.uint8, device="cuda")
    with pytest.raises(eqw.EqError) as e:
        model.gemm_symbols(0, sym, torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda"),
                           torch.zeros(4, 100, dtype=torch.float32, device="cuda"), status)
    assert e.value.code == EQ_ERR_UNSUPPORTED
    model.close()


def test_decode_symbols_block_bit_exact(eqw, orc):
    mats = W.llama70b_int8_layer(0)
    model = _open(eqw, mats)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = [torch.empty(m.rows * m.cols, dtype=torch.uint8, device="cuda") for m in mats]
    model.decode_symbols_block(0, outs, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for m, o in zip(mats, outs):
        assert np.array_equal(o.cpu().numpy().reshape(m.rows, m.cols), orc.stream_symbols(m))
    model.close()
