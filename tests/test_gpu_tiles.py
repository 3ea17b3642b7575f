"""Shared-table launches at every tile shape.

The shared-table kernels take a matrix's chunks in tiles of (warps per tile) x
(chunks per warp): one chunk per warp when tiles of 24 single chunks fit one
round of resident blocks (one per SM), else two in lockstep; as few warps per
tile as keep the launch within one round.  The cases below are sized so that
the chosen shape runs from 1 warp to the full block with one and with two
chains per warp, with ragged last tiles, and decode and fused decode + GEMV
are compared with the oracle: decode bit for bit, GEMV within the bound of
test_gpu_fused_gemv.  `tile_shape` mirrors the host rule so each case states
which shape it exercises.
"""
import numpy as np
import pytest
import torch

import workloads as W
from test_gpu_fused_gemv import _bound_ok, _n_out_rows, _run_matrices, _x_for

pytestmark = pytest.mark.gpu

FULL_WARPS = 24
CHAINS = 2


@pytest.fixture(scope="module")
def eqw():
    from entropy_coded_weight_b200 import build
    build.build()
    import entropy_coded_weight_b200 as E
    E.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return E


def tile_shape(n_chunks: list[int], resident: int) -> tuple[int, int]:
    def units(w, c):
        return sum(-(-n // (w * c)) for n in n_chunks)
    chains = 1 if units(FULL_WARPS, 1) <= resident else CHAINS
    for w in range(1, FULL_WARPS):
        if units(w, chains) <= resident:
            return w, chains
    return FULL_WARPS, chains


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _matrix(seed, n_chunks, cols=4096, layer=0, index=0, n_out=0):
    rows = n_chunks * 65536 // cols
    return W.random_int8_matrix(seed, rows, cols, h_bits=2.1, n_out=n_out, layer=layer, index=index)


CASES = {
    "one_chunk": [1],
    "one_tile_ragged": [3],
    "width_2_many_tiles": [290],
    "width_3": [300],
    "width_14_ragged": [2000],
    "block_mixed": [16, 64, 700, 700, 1100],
    "two_chains_width_17": [5000],
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_decode_block_bit_exact(eqw, orc, name):
    counts = CASES[name]
    mats = [_matrix(500 + i, n, index=i, n_out=4 if i == 0 else 0) for i, n in enumerate(counts)]
    tw, tc = tile_shape(counts, _sms())
    assert 1 <= tw <= FULL_WARPS and tc in (1, 2)
    blob = eqw.encode_host(mats)
    model = eqw.Model(eqw.upload(blob), blob)
    offs, total = model.block_layout(0)
    out = torch.empty(total, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    model.decode_block(0, out, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    host = out.cpu().numpy()
    for m, o in zip(mats, offs):
        got = host[o:o + 2 * m.n].view(np.uint16).reshape(m.rows, m.cols)
        assert np.array_equal(got, orc.dequant_direct(m)), (name, tw, tc, m.index)
    model.close()


def test_shape_range_is_covered():
    """On a 148-SM B200 the cases above span one-chain widths 1 to 18 and a
    two-chain width of 17; 7B- and 70B-shape blocks get (22, 1) and (24, 2)."""
    shapes = {name: tile_shape(c, 148) for name, c in CASES.items()}
    assert shapes["one_chunk"] == (1, 1) and shapes["one_tile_ragged"] == (1, 1)
    assert shapes["width_2_many_tiles"] == (2, 1)
    assert shapes["width_3"] == (3, 1)
    assert shapes["width_14_ragged"] == (14, 1)
    assert shapes["block_mixed"] == (18, 1)
    assert shapes["two_chains_width_17"] == (17, 2)
    assert tile_shape([256] * 4 + [688] * 3, 148) == (22, 1)     # Llama-7B-shape block
    assert tile_shape([1024, 128, 128, 1024, 3584, 3584, 3584], 148) == (FULL_WARPS, 2)  # Llama-70B shape


@pytest.mark.parametrize("name", ["one_tile_ragged", "width_3", "width_14_ragged", "block_mixed", "two_chains_width_17"])
def test_fused_gemv_within_bound(eqw, orc, name):
    counts = CASES[name]
    mats = [_matrix(600 + i, n, cols=8192, index=i) for i, n in enumerate(counts)]
    blob = eqw.encode_host(mats)
    st, ys = _run_matrices(eqw, blob, mats, per_matrix=False)
    assert st == 0
    for m, y in zip(mats, ys):
        ref, mag = orc.gemv_exact(orc.dequant_direct(m), _bits(_x_for(m)))
        ok, info = _bound_ok(y, ref, mag, m.cols, _n_out_rows(m))
        assert ok, (name, m.index, info)


@pytest.mark.parametrize("limit", [1, 7, 100])
def test_sm_limit_keeps_results(eqw, orc, limit):
    """eq_model_set_sm_limit: fewer resident blocks, more rounds per block; the
    decoded block and the fused GEMV stay exact / within bound."""
    counts = [700, 1100]
    mats = [_matrix(700 + i, n, cols=8192, index=i) for i, n in enumerate(counts)]
    blob = eqw.encode_host(mats)
    model = eqw.Model(eqw.upload(blob), blob)
    model.set_sm_limit(limit)
    offs, total = model.block_layout(0)
    out = torch.empty(total, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    model.decode_block(0, out, status)
    xs = [_x_for(m).cuda() for m in mats]
    ys = [torch.empty(m.rows, dtype=torch.float32, device="cuda") for m in mats]
    model.decode_gemv_block(0, xs, ys, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    host = out.cpu().numpy()
    for m, o, y in zip(mats, offs, ys):
        w = orc.dequant_direct(m)
        assert np.array_equal(host[o:o + 2 * m.n].view(np.uint16).reshape(m.rows, m.cols), w)
        ref, mag = orc.gemv_exact(w, _bits(_x_for(m)))
        ok, info = _bound_ok(y.cpu().numpy(), ref, mag, m.cols, _n_out_rows(m))
        assert ok, (limit, m.index, info)
    model.close()
