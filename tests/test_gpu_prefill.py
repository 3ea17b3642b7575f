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


def _one_hot(seed, tokens, cols):
    rng = np.random.default_rng(seed)
    x = torch.zeros(tokens, cols, dtype=torch.bfloat16)
    x[torch.arange(tokens), torch.from_numpy(rng.integers(0, cols, size=tokens))] = torch.from_numpy(
        rng.choice([-2.0, -0.5, 1.0, 3.0], size=tokens).astype(np.float32)).to(torch.bfloat16)
    return x


def _block_mats():
    """Both weight types, K from 64 to 1024, super weights, in one layer."""
    return [W.random_int8_matrix(30, 256, 512, n_out=8, layer=0, index=0),
            W.random_e4m3_matrix(31, 128, 192, alpha=1.0, layer=0, index=1),
            W.random_int8_matrix(32, 384, 64, layer=0, index=2),
            W.random_int8_matrix(33, 128, 1024, h_bits=4.0, layer=0, index=3),
            W.random_e4m3_matrix(34, 256, 256, alpha=1.0, layer=0, index=4)]


@pytest.mark.parametrize("tokens", [700, 100])
@pytest.mark.parametrize("sms", [0, 1, 3])
def test_gemm_block_one_hot_bit_exact(eqw, orc, sms, tokens):
    """One persistent launch per weight type over every tile of the layer; sms = 1 or 3 makes each
    CTA run many tiles of different matrices (stage ring and barrier phases carried across tiles).
    700 tokens: three 256-token tiles, the last one ragged; 100: one ragged 128-token tile."""
    mats = _block_mats()
    model = _open(eqw, mats)
    model.set_sm_limit(sms)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    syms = [torch.empty(m.rows * m.cols, dtype=torch.uint8, device="cuda") for m in mats]
    model.decode_symbols_block(0, syms, status)
    xs = [_one_hot(40 + i, tokens, m.cols) for i, m in enumerate(mats)]
    ys = [torch.full((tokens, m.rows), float("nan"), dtype=torch.float32, device="cuda") for m in mats]
    model.gemm_symbols_block(0, syms, [x.cuda() for x in xs], ys, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for i, (m, x, y) in enumerate(zip(mats, xs, ys)):
        ref, _ = orc.gemm_symbols_exact(m, _bits(x))
        assert np.array_equal(y.cpu().numpy().view(np.uint32), ref.astype(np.float32).view(np.uint32)), i
    model.close()


@pytest.mark.parametrize("tokens", [300, 128])
def test_gemm_block_random_tokens_within_bound(eqw, orc, tokens):
    mats = _block_mats()
    model = _open(eqw, mats)
    model.set_sm_limit(2)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    syms = [torch.empty(m.rows * m.cols, dtype=torch.uint8, device="cuda") for m in mats]
    model.decode_symbols_block(0, syms, status)
    xs = [W.gemv_activation(9, i, tokens * m.cols).reshape(tokens, m.cols) for i, m in enumerate(mats)]
    ys = [torch.empty(tokens, m.rows, dtype=torch.float32, device="cuda") for m in mats]
    model.gemm_symbols_block(0, syms, [x.cuda() for x in xs], ys, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for m, x, y in zip(mats, xs, ys):
        ref, mag = orc.gemm_symbols_exact(m, _bits(x))
        _check_bound(y.cpu().numpy(), ref, mag, m.cols)
    model.close()


@pytest.mark.parametrize("tokens", [512, 96])
def test_gemm_block_llama70b_layer_sampled_rows(eqw, orc, tokens):
    """A full 70B-shape layer (7 matrices: 1312 tiles of 256 tokens at 512 tokens, 448 tiles of 128
    tokens at 96) in one launch: every output equals the single-matrix launch's bit for bit (same tile
    arithmetic), and sampled weight rows of every matrix are within the fp32 bound of the oracle."""
    mats = W.llama70b_int8_layer(0)
    model = _open(eqw, mats)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    syms = [torch.empty(m.rows * m.cols, dtype=torch.uint8, device="cuda") for m in mats]
    model.decode_symbols_block(0, syms, status)
    xs = [W.gemv_activation(11, i, tokens * m.cols).reshape(tokens, m.cols) for i, m in enumerate(mats)]
    xd = [x.cuda() for x in xs]
    ys = [torch.empty(tokens, m.rows, dtype=torch.float32, device="cuda") for m in mats]
    model.gemm_symbols_block(0, syms, xd, ys, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rng = np.random.default_rng(12)
    for i, (m, x, y) in enumerate(zip(mats, xs, ys)):
        y1 = torch.empty_like(y)
        model.gemm_symbols(i, syms[i], xd[i], y1, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(y.view(torch.int32), y1.view(torch.int32)), i
        rows = np.sort(rng.choice(m.rows, size=64, replace=False))
        sub = W.Matrix(m.layer, m.index, m.name, m.dtype, m.symbols[rows], m.scales[rows])
        ref, mag = orc.gemm_symbols_exact(sub, _bits(x))
        _check_bound(y.cpu().numpy()[:, rows], ref, mag, m.cols)
    model.close()


def test_gemm_block_argument_errors(eqw):
    mats = _block_mats()
    model = _open(eqw, mats)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    syms = [torch.empty(m.rows * m.cols, dtype=torch.uint8, device="cuda") for m in mats]
    xs = [torch.zeros(4, m.cols, dtype=torch.bfloat16, device="cuda") for m in mats]
    ys = [torch.zeros(4, m.rows, dtype=torch.float32, device="cuda") for m in mats]
    with pytest.raises(ValueError):
        model.gemm_symbols_block(0, syms[:-1], xs, ys, status)
    with pytest.raises(eqw.EqError):                 # count != the layer's matrix count
        model.gemm_symbols_block(0, syms[:-1], xs[:-1], ys[:-1], status)
    bad = list(ys)
    bad[2] = torch.zeros(4 * mats[2].rows + 1, dtype=torch.float32, device="cuda")[1:].view(4, mats[2].rows)
    with pytest.raises(eqw.EqError):                 # y not 16-byte aligned: nothing launched
        model.gemm_symbols_block(0, syms, xs, bad, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    model.close()


def _pair_mats():
    """Every matrix a whole number of 256-row tiles: the layer takes the 2-SM (cta_group::2) kernel."""
    return [W.random_int8_matrix(50, 256, 512, n_out=6, layer=0, index=0),
            W.random_int8_matrix(51, 512, 64, layer=0, index=1),
            W.random_int8_matrix(52, 256, 1024, h_bits=4.0, layer=0, index=2),
            W.random_e4m3_matrix(53, 256, 192, alpha=1.0, layer=0, index=3),
            W.random_e4m3_matrix(54, 512, 256, alpha=1.0, layer=0, index=4)]


@pytest.mark.parametrize("sms", [0, 2, 5])
def test_gemm_block_pair_kernel_one_hot_bit_exact(eqw, orc, sms):
    """The 2-SM kernel: 700 tokens (three 256-token tiles, the last ragged), both weight types, K from 64
    to 1024, super weights; sms = 2 or 5 leaves one or two CTA pairs, each running many tiles."""
    mats = _pair_mats()
    tokens = 700
    model = _open(eqw, mats)
    model.set_sm_limit(sms)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    syms = [torch.empty(m.rows * m.cols, dtype=torch.uint8, device="cuda") for m in mats]
    model.decode_symbols_block(0, syms, status)
    xs = [_one_hot(60 + i, tokens, m.cols) for i, m in enumerate(mats)]
    ys = [torch.full((tokens, m.rows), float("nan"), dtype=torch.float32, device="cuda") for m in mats]
    model.gemm_symbols_block(0, syms, [x.cuda() for x in xs], ys, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for i, (m, x, y) in enumerate(zip(mats, xs, ys)):
        ref, _ = orc.gemm_symbols_exact(m, _bits(x))
        assert np.array_equal(y.cpu().numpy().view(np.uint32), ref.astype(np.float32).view(np.uint32)), i
    model.close()


def test_gemm_block_pair_kernel_random_tokens_within_bound(eqw, orc):
    mats = _pair_mats()
    tokens = 300
    model = _open(eqw, mats)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    syms = [torch.empty(m.rows * m.cols, dtype=torch.uint8, device="cuda") for m in mats]
    model.decode_symbols_block(0, syms, status)
    xs = [W.gemv_activation(13, i, tokens * m.cols).reshape(tokens, m.cols) for i, m in enumerate(mats)]
    ys = [torch.empty(tokens, m.rows, dtype=torch.float32, device="cuda") for m in mats]
    model.gemm_symbols_block(0, syms, [x.cuda() for x in xs], ys, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for m, x, y in zip(mats, xs, ys):
        ref, mag = orc.gemm_symbols_exact(m, _bits(x))
        _check_bound(y.cpu().numpy(), ref, mag, m.cols)
    model.close()
