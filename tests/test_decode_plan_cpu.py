"""Host-side split of a block decode between the two decode kernels
(eq_decode_plan), checked on CPU: which matrices qualify for the kernel that
decodes two full chunks per warp, how many leading chunks it takes, and when a
launch falls back to the general kernel.  No GPU is needed: the plan is a pure
function of the container and the SM count.
"""
import types

import numpy as np
import pytest

import workloads as W

FAKE_DEVICE_PTR = 0x7F0000000000  # 256-byte aligned; the plan never touches device memory
CHUNK = 65536


@pytest.fixture(scope="module")
def eqw():
    from entropy_coded_weight_b200 import build
    build.build()
    import entropy_coded_weight_b200 as E
    E.load()
    return E


def _model(E, blob):
    fake = types.SimpleNamespace(data_ptr=lambda: FAKE_DEVICE_PTR, numel=lambda: blob.size)
    return E.Model(fake, blob)


def _chunks(m):
    return -(-m.rows * m.cols // CHUNK)


def test_single_matrix_needs_a_full_round(eqw):
    # 768 x 4096 = 48 full chunks = 24 pairs: exactly one pair per warp of one SM
    full = W.random_int8_matrix(1, 768, 4096)
    model = _model(eqw, eqw.encode_host([full]))
    assert model.decode_plan(0, 1) == [48]
    assert model.decode_plan(0, 2) == [0]       # 24 pairs cannot fill 48 warps
    model.close()
    short = W.random_int8_matrix(2, 767, 4096)  # 47 full chunks + a tail: 23 pairs
    model = _model(eqw, eqw.encode_host([short]))
    assert model.decode_plan(0, 1) == [0]
    model.close()


def test_odd_and_partial_chunks_stay_with_the_general_kernel(eqw):
    m = W.random_int8_matrix(3, 784 + 5, 4096)  # 49 full chunks + a partial one
    assert _chunks(m) == 50
    model = _model(eqw, eqw.encode_host([m]))
    assert model.decode_plan(0, 1) == [48]
    model.close()


def test_ineligible_matrices(eqw):
    mats = [
        W.random_e4m3_matrix(4, 768, 4096, alpha=1.0, layer=0, index=0),    # ~250 codes: no rank mode
        W.random_int8_matrix(5, 1536, 2304, layer=0, index=1),              # rows not a multiple of 512
        W.random_int8_matrix(6, 768, 4096, layer=0, index=2),               # eligible
        W.random_e4m3_matrix(7, 768, 4096, alpha=9e4, layer=0, index=3),    # few codes: eligible (E4M3 launch)
    ]
    model = _model(eqw, eqw.encode_host(mats))
    assert model.decode_plan(0, 1) == [0, 0, 48, 48]
    model.close()
    # per-chunk tables: no matrix-wide slot table, so no pair kernel
    model = _model(eqw, eqw.encode_host(mats[2:3], table_scope="chunk"))
    assert model.decode_plan(0, 1) == [0]
    model.close()


def test_huffman_codec_qualifies(eqw):
    m = W.random_int8_matrix(8, 768, 4096)
    model = _model(eqw, eqw.encode_host([m], codec="huffman"))
    assert model.decode_plan(0, 1) == [48]
    model.close()


def test_block_ranges_touch_at_most_three_matrices(eqw):
    # five matrices of 16 pairs: one block would span all five (refused), two
    # blocks span three each (accepted)
    mats = [W.random_int8_matrix(10 + i, 512, 4096, layer=0, index=i) for i in range(5)]
    model = _model(eqw, eqw.encode_host(mats))
    assert model.decode_plan(0, 1) == [0] * 5
    assert model.decode_plan(0, 2) == [32] * 5
    assert model.decode_plan(0, 4) == [0] * 5   # 80 pairs < 4 SMs x 24 warps
    model.close()


def test_sm_limit_caps_the_plan(eqw):
    m = W.random_int8_matrix(20, 768, 4096)
    model = _model(eqw, eqw.encode_host([m]))
    assert model.decode_plan(0, 148) == [0]
    model.set_sm_limit(1)
    assert model.decode_plan(0, 148) == [48]
    model.close()


def test_llama70b_shapes_go_to_the_pair_kernel(eqw):
    """The 70B-shape block's matrices (q, o 8192x8192; k, v 1024x8192; gate, up
    28672x8192; down 8192x28672): every chunk count is even, every block range
    of 6528 / 148 pairs touches at most two matrices and the launch fills all
    148 SMs, so the whole block takes the pair kernel.  The plan depends only
    on shapes and tables, so near-constant symbols (two per chunk) stand in for
    the Laplace workload and keep the encode cheap."""
    mats = []
    for i, (r, c) in enumerate(W.LLAMA70B_BLOCK):
        sym = np.zeros((r, c), dtype=np.uint8)
        sym.reshape(-1)[::CHUNK] = 1
        mats.append(W.Matrix(0, i, f"m{i}", W.INT8, sym, np.ones(r, dtype=np.float32)))
    model = _model(eqw, eqw.encode_host(mats))
    assert model.decode_plan(0, 148) == [_chunks(m) for m in mats]
    assert sum(model.decode_plan(0, 148)) == 13056
    # with fewer SMs the same block still qualifies; a single SM's range would span all seven
    assert model.decode_plan(0, 64) == [_chunks(m) for m in mats]
    assert model.decode_plan(0, 1) == [0] * 7
    model.close()


def test_plan_arguments_checked(eqw):
    m = W.random_int8_matrix(40, 16, 4096)
    model = _model(eqw, eqw.encode_host([m]))
    L = eqw.load()
    import ctypes
    buf = (ctypes.c_uint32 * 4)()
    assert L.eq_decode_plan(model._m, 0, 0, buf, 4) == 1     # sms == 0
    assert L.eq_decode_plan(model._m, 1, 8, buf, 4) == 1     # no such layer
    assert L.eq_decode_plan(model._m, 0, 8, buf, 0) == 1     # cap too small
    assert L.eq_decode_plan(model._m, 0, 8, None, 4) == 1
    assert L.eq_decode_plan(model._m, 0, 8, buf, 4) == 0
    model.close()
