"""Host-side argument checks of the prefill GEMM entry points (no GPU, no kernel
launch): eq_gemm_symbols and eq_gemm_symbols_block validate every request --
matrix index, shape (rows % 128, cols % 64), null and misaligned pointers, the
layer's matrix count -- before any CUDA call, and launch nothing when one
request fails.  With zero tokens and valid requests they return EQ_OK without
touching the device, so the pointers given here (never dereferenced on the
host) are never used.
"""
import ctypes

import pytest

import workloads as W

FAKE = 0x7F0000000000  # 256-byte aligned device-looking address; never dereferenced
EQ_OK, EQ_ERR_INVALID_ARG, EQ_ERR_UNSUPPORTED = 0, 1, 3


@pytest.fixture(scope="module")
def eqw():
    from entropy_coded_weight_b200 import build
    build.build()
    import entropy_coded_weight_b200 as E
    E.load()
    return E


@pytest.fixture()
def model(eqw, orc):
    """A two-layer container: layer 0 GEMM-shaped, layer 1 with a 100-row matrix."""
    mats = [W.random_int8_matrix(1, 256, 512, layer=0, index=0),
            W.random_e4m3_matrix(2, 128, 192, layer=0, index=1),
            W.random_int8_matrix(3, 100, 64, layer=1, index=0),
            W.random_int8_matrix(4, 128, 64, layer=1, index=1)]
    blob = orc.encode_container(mats)
    h = ctypes.c_void_p()
    L = eqw.load()
    assert L.eq_model_open(FAKE, blob.size, blob.ctypes.data, ctypes.byref(h)) == 0
    yield L, h
    L.eq_model_close(h)


def _gemm(L, h, matrix, sym=FAKE, x=FAKE, tokens=0, y=FAKE, status=FAKE):
    return L.eq_gemm_symbols(h, matrix, sym, x, tokens, y, status, None)


def _block(L, h, layer, n, tokens=0, syms=None, xs=None, ys=None, count=None, status=FAKE):
    arr = ctypes.c_void_p * max(1, n)
    ps = arr(*(syms or [FAKE] * n))
    px = arr(*(xs or [FAKE] * n))
    py = arr(*(ys or [FAKE] * n))
    return L.eq_gemm_symbols_block(h, layer, ps, px, tokens, py, n if count is None else count, status, None)


def test_single_matrix_checks(model):
    L, h = model
    assert _gemm(L, h, 0) == EQ_OK                       # valid, zero tokens: nothing to launch
    assert _gemm(L, h, 1) == EQ_OK
    assert _gemm(L, h, 4) == EQ_ERR_INVALID_ARG          # no such matrix
    assert _gemm(L, h, 2) == EQ_ERR_UNSUPPORTED          # 100 rows: not a multiple of 128
    assert _gemm(L, h, 0, sym=0) == EQ_ERR_INVALID_ARG
    assert _gemm(L, h, 0, x=0) == EQ_ERR_INVALID_ARG
    assert _gemm(L, h, 0, y=0) == EQ_ERR_INVALID_ARG
    assert _gemm(L, h, 0, status=0) == EQ_ERR_INVALID_ARG
    for field in ("sym", "x", "y"):                       # TMA and vector accesses need 16-byte alignment
        assert _gemm(L, h, 0, **{field: FAKE + 8}) == EQ_ERR_INVALID_ARG
    assert L.eq_gemm_symbols(None, 0, FAKE, FAKE, 0, FAKE, FAKE, None) == EQ_ERR_INVALID_ARG


def test_block_checks(model):
    L, h = model
    assert _block(L, h, 0, 2) == EQ_OK
    assert _block(L, h, 0, 2, count=1) == EQ_ERR_INVALID_ARG   # count must be the layer's matrix count
    assert _block(L, h, 2, 2) == EQ_ERR_INVALID_ARG            # no such layer
    assert _block(L, h, 1, 2) == EQ_ERR_UNSUPPORTED            # one matrix of the layer is unsupported
    assert _block(L, h, 0, 2, ys=[FAKE, FAKE + 8]) == EQ_ERR_INVALID_ARG
    assert _block(L, h, 0, 2, syms=[FAKE, 0]) == EQ_ERR_INVALID_ARG
    assert L.eq_gemm_symbols_block(h, 0, None, None, 0, None, 2, FAKE, None) == EQ_ERR_INVALID_ARG
    assert _block(L, h, 0, 2, status=0) == EQ_ERR_INVALID_ARG


def test_block_rejects_before_any_launch_even_with_tokens(model):
    """A failing request stops the call before CUDA: with real token counts the invalid layer-1 block
    still returns the argument error (a launch would need a device and fail differently)."""
    L, h = model
    assert _block(L, h, 1, 2, tokens=512) == EQ_ERR_UNSUPPORTED
    assert _block(L, h, 0, 2, tokens=512, xs=[FAKE + 4, FAKE]) == EQ_ERR_INVALID_ARG
