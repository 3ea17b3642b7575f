"""GPU parity of the fused decode + batch-1 GEMV (eq_decode_gemv_matrix / eq_decode_gemv_block).

Expected values come from the oracle only: oracle.gemv_exact (fp64) on the
O-direct weights (oracle.dequant_direct, or oracle.dequant_pairs for sampled
rows) and the seeded bf16 activation.  The kernel's products are exact in
fp32 and its sums form a tree of height at most
h = cols / 64 + 8 + (super weights in the row) + (chunks the row spans)
(per lane two accumulators over cols / 64 terms each, one add to join them,
five butterfly levels, the row's super weights, one add per chunk partial),
so |y - exact| <= gamma_h * sum_c |W[r, c] x[c]| with gamma_h = h u / (1 - h u),
u = 2^-24 (Higham, "Accuracy and Stability of Numerical Algorithms", 4.2).
The test allows h + 8.  A single dropped or doubled product of typical size
exceeds this bound by an order of magnitude.
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


def _x_for(m, seed=0):
    return W.gemv_activation(1000 + seed + m.layer, m.index, m.cols)


def _bound_ok(y, ref, mag, cols, n_out_row):
    u = 2.0 ** -24
    h = cols / 64 + 16 + n_out_row + (cols + 65535) // 65536 + 1
    g = h * u / (1 - h * u)
    err = np.abs(y.astype(np.float64) - ref)
    bad = err > g * mag
    return not bad.any(), (np.flatnonzero(bad)[:5], err[bad][:5], (g * mag)[bad][:5])


def _n_out_rows(m):
    return np.bincount(np.asarray(m.out_row, np.int64), minlength=m.rows)


def _run_matrices(E, blob, mats, per_matrix=True):
    """Fused y for every matrix (layer by layer), as numpy float32 arrays."""
    model = E.Model(E.upload(blob), blob)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xs = [_x_for(m).cuda() for m in mats]
    ys = [torch.full((m.rows,), float("nan"), dtype=torch.float32, device="cuda") for m in mats]
    order = sorted(range(len(mats)), key=lambda i: (mats[i].layer, mats[i].index))
    if per_matrix:
        for mi, i in enumerate(order):
            model.decode_gemv_matrix(mi, xs[i], ys[i], status)
    else:
        layers = sorted({m.layer for m in mats})
        for L in layers:
            idx = [i for i in order if mats[i].layer == L]
            model.decode_gemv_block(L, [xs[i] for i in idx], [ys[i] for i in idx], status)
    torch.cuda.synchronize()
    st = int(status.item())
    model.close()
    return st, [y.cpu().numpy() for y in ys]


def _ragged():
    mats = [
        W.random_int8_matrix(1, 300, 1024, h_bits=2.1, layer=0, index=0),
        W.random_int8_matrix(2, 77, 256, h_bits=3.0, layer=0, index=1),
        W.random_e4m3_matrix(3, 5, 512, alpha=1.0, layer=0, index=2),          # ~250 codes: no rank mode
        W.random_int8_matrix(4, 1, 65536, layer=0, index=3),                   # one row = one chunk
        W.random_int8_matrix(5, 3, 131072, layer=1, index=0),                  # rows span two chunks
        W.random_int8_matrix(6, 513, 768, n_out=12, layer=1, index=1),         # cols % 512 != 0, outliers
        W.random_int8_matrix(7, 256, 8192, n_out=8, layer=1, index=2),         # 32 chunks: two-chain path
        W.random_int8_matrix(8, 0, 256, layer=1, index=3),                     # empty
        W.random_e4m3_matrix(9, 96, 2048, alpha=9.1e4, layer=1, index=4),     # few subnormal codes
    ]
    single = W.random_int8_matrix(10, 40, 4096, layer=1, index=5)
    single.symbols[:] = 0x05                                                    # one symbol: f = 4096
    mats.append(single)
    return mats


@pytest.mark.parametrize("encoder", ["matrix", "chunk", "oracle"])
@pytest.mark.parametrize("per_matrix", [True, False])
def test_ragged_shapes_within_fp32_bound(eqw, orc, encoder, per_matrix):
    mats = _ragged()
    blob = orc.encode_container(mats) if encoder == "oracle" else eqw.encode_host(mats, table_scope=encoder)
    st, ys = _run_matrices(eqw, blob, mats, per_matrix)
    assert st == 0
    for m, y in zip(mats, ys):
        assert y.shape == (m.rows,)
        ref, mag = orc.gemv_exact(orc.dequant_direct(m), _bits(_x_for(m)))
        ok, info = _bound_ok(y, ref, mag, m.cols, _n_out_rows(m))
        assert ok, (m.rows, m.cols, info)


def test_deterministic_and_block_equals_matrix(eqw, orc):
    mats = [m for m in _ragged() if m.cols <= 65536]
    blob = eqw.encode_host(mats)
    _, a = _run_matrices(eqw, blob, mats, True)
    _, b = _run_matrices(eqw, blob, mats, True)
    _, c = _run_matrices(eqw, blob, mats, False)
    for ya, yb, yc in zip(a, b, c):
        assert np.array_equal(ya.view(np.uint32), yb.view(np.uint32))
        assert np.array_equal(ya.view(np.uint32), yc.view(np.uint32))


def test_unsupported_and_argument_errors(eqw):
    m = W.random_int8_matrix(20, 16, 1000)
    blob = eqw.encode_host([m])
    model = eqw.Model(eqw.upload(blob), blob)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = torch.zeros(1000, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(eqw.EqError) as e:
        model.decode_gemv_matrix(0, x, y, status)
    assert e.value.code == EQ_ERR_UNSUPPORTED
    with pytest.raises(eqw.EqError) as e:
        model.decode_gemv_block(0, [x, x], [y, y], status)  # the layer has one matrix
    assert e.value.code == 1
    model.close()


def _sampled_rows_check(orc, m, y, rows):
    cols = m.cols
    sym = m.symbols[rows].reshape(-1)
    w = orc.dequant_pairs(m.dtype, sym, np.repeat(m.scales[rows], cols)).reshape(len(rows), cols)
    if len(m.out_row):
        for r, c, v in zip(m.out_row, m.out_col, m.out_val):
            hit = np.flatnonzero(rows == r)
            if hit.size:
                w[hit[0], c] = orc.bf16_rne(np.array([v], np.float32))[0]
    ref, mag = orc.gemv_exact(w, _bits(_x_for(m)))
    ok, info = _bound_ok(y[rows], ref, mag, cols, _n_out_rows(m)[rows])
    assert ok, (m.rows, m.cols, info)


@pytest.mark.parametrize("which", ["llama70b_int8_layer", "llama70b_e4m3_block", "llama7b_int8_block_with_outliers"])
def test_full_size_workloads_sampled_rows(eqw, orc, which):
    """Full-size blocks in one fused launch; 96 seeded rows per matrix (plus
    every row holding a super weight) recomputed by the oracle."""
    if which == "llama70b_int8_layer":
        mats = W.llama70b_int8_layer(0)
    else:
        mats = getattr(W, which)()
    blob = eqw.encode_host(mats)
    st, ys = _run_matrices(eqw, blob, mats, per_matrix=False)
    assert st == 0
    rng = np.random.default_rng(77)
    for m, y in zip(mats, ys):
        assert not np.isnan(y).any()
        rows = np.unique(np.concatenate([rng.choice(m.rows, size=96, replace=False),
                                         np.asarray(m.out_row, np.int64)])).astype(np.int64)
        _sampled_rows_check(orc, m, y, rows)


def test_device_corruption_flags_in_fused_path(eqw, orc):
    m = W.random_int8_matrix(200, 512, 512, n_out=4)
    blob = eqw.encode_host([m])
    parsed = orc.parse_container(blob)
    off0 = int(parsed["matrices"][0]["chunk_offsets"][0])
    npres = int(np.frombuffer(bytes(blob[off0 + 8:off0 + 12]), "<u4")[0])
    words = off0 + ((144 + 4 * npres + 15) // 16) * 16
    for what, bit in (("payload", eqw.EQ_DEV_BAD_END), ("table", eqw.EQ_DEV_BAD_TABLE)):
        d_blob = eqw.upload(blob)
        model = eqw.Model(d_blob, blob)
        if what == "payload":
            d_blob[words + 100] ^= 0x40
        else:
            d_blob[off0 + 144 + 2] ^= 0x01
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        y = torch.empty(512, dtype=torch.float32, device="cuda")
        model.decode_gemv_matrix(0, _x_for(m).cuda(), y, status)
        torch.cuda.synchronize()
        assert int(status.item()) & bit, what
        model.close()


def test_scatter_checks_zero_placeholder(eqw):
    """The decode path flags a super weight whose stream value is not zero
    (the fused path relies on that placeholder)."""
    m = W.random_int8_matrix(201, 64, 512, n_out=3)
    taken = set(zip(m.out_row.tolist(), m.out_col.tolist()))
    k = next(k for k in range(3) if int(m.out_col[k]) % 256 != 255 and
             (int(m.out_row[k]), int(m.out_col[k]) + 1) not in taken)
    r, c = int(m.out_row[k]), int(m.out_col[k])
    m.symbols[r, c + 1] = 0x07
    blob = eqw.encode_host([m])
    d_blob = eqw.upload(blob)
    model = eqw.Model(d_blob, blob)
    oo = int(np.frombuffer(bytes(blob[64 + 48:64 + 56]), "<u8")[0])
    d_blob[oo + 12 * k + 4] += 1  # device copy: outlier k now sits on column c + 1
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(64 * 512, dtype=torch.bfloat16, device="cuda")
    model.decode_matrix(0, out, status)
    torch.cuda.synchronize()
    assert int(status.item()) & eqw.EQ_DEV_BAD_OUTLIER
    model.close()
