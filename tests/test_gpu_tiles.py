"""Shared-table launches at every tile width.

The shared-table kernels take a matrix's chunks in tiles of (warps per tile) x
2 chunks, using as few warps per tile as keep the launch within one block per
SM.  The cases below are sized so that the chosen width runs from 1 to the
full block, with ragged last tiles, and decode and fused decode + GEMV are
compared with the oracle: decode bit for bit, GEMV within the bound of
test_gpu_fused_gemv.  `tile_warps` mirrors the host rule so each case states
which width it exercises.
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


def tile_warps(n_chunks: list[int], resident: int) -> int:
    for w in range(1, FULL_WARPS):
        if sum(-(-n // (w * CHAINS)) for n in n_chunks) <= resident:
            return w
    return FULL_WARPS


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
    "width_1_many_tiles": [290],
    "width_2": [300],
    "width_7_ragged": [2000],
    "block_mixed": [16, 64, 700, 700, 1100],
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_decode_block_bit_exact(eqw, orc, name):
    counts = CASES[name]
    mats = [_matrix(500 + i, n, index=i, n_out=4 if i == 0 else 0) for i, n in enumerate(counts)]
    tw = tile_warps(counts, _sms())
    assert 1 <= tw <= FULL_WARPS
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
        assert np.array_equal(got, orc.dequant_direct(m)), (name, tw, m.index)
    model.close()


def test_width_range_is_covered():
    """On a 148-SM B200 the cases above span widths 1, 2, 7 and a mixed block."""
    widths = {name: tile_warps(c, 148) for name, c in CASES.items()}
    assert widths["one_chunk"] == 1 and widths["width_1_many_tiles"] == 1
    assert widths["width_2"] == 2
    assert widths["width_7_ragged"] == 7
    assert tile_warps([13056], 148) == FULL_WARPS  # a Llama-70B-shape block keeps full tiles


@pytest.mark.parametrize("name", ["one_tile_ragged", "width_2", "width_7_ragged", "block_mixed"])
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
