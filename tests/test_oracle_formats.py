"""Pins for the oracle's number formats and dequantiser.

Dequantisation (EntQuant technical summary, section 2: Int8 / Float8 symbols
with per-channel scales S) is defined here as
out = bf16_rne(fp32_rn(value(sym) * scale[row])).  Every step is checked
against an independent library routine (torch / numpy), against the format's
defining landmark values, or exhaustively.
"""
import numpy as np
import pytest
import torch

from conftest import read_golden


def test_int8_values_all_codes(orc):
    for b in range(256):
        assert orc.int8_value(b) == float(np.array([b], np.uint8).view(np.int8)[0])


def test_e4m3_values_match_torch_all_codes(orc):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).double().numpy()
    for b in range(256):
        v = orc.e4m3_value(b)
        if (b & 0x7F) == 0x7F:
            assert np.isnan(v) and np.isnan(ref[b])
            continue
        assert v == ref[b], hex(b)
        assert np.signbit(v) == np.signbit(ref[b]), hex(b)


def test_e4m3_landmarks(orc):
    for row in read_golden("e4m3_reference_values.txt"):
        code, val = [c.strip() for c in row.split("|")]
        v = orc.e4m3_value(int(code, 16))
        assert v == float(val) and np.signbit(v) == val.startswith("-"), code


def _bf16_bits_torch(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_bf16_rne_all_high_halves_against_torch(orc):
    """Every fp32 exponent/sign/high-mantissa pattern with the low halves that
    decide rounding (0, ties, just above/below ties, max) plus random lows."""
    hi = np.arange(65536, dtype=np.uint32) << 16
    lows = [0x0000, 0x0001, 0x7FFF, 0x8000, 0x8001, 0xFFFF, 0x4000, 0xC000]
    rng = np.random.default_rng(1)
    lows += rng.integers(0, 65536, size=24).tolist()
    for lo in lows:
        bits = hi | np.uint32(lo)
        f = bits.view(np.float32)
        keep = ~np.isnan(f)
        got = orc.bf16_rne(f[keep])
        want = _bf16_bits_torch(f[keep])
        assert np.array_equal(got, want), hex(lo)


def test_bf16_rne_scalar_matches_array(orc):
    rng = np.random.default_rng(2)
    vals = rng.standard_normal(2000).astype(np.float32) * np.float32(1e-3)
    vals = np.concatenate([vals, np.array([0.0, -0.0, np.inf, -np.inf, 1e-40, -1e-40], np.float32)])
    vec = orc.bf16_rne(vals)
    for v, b in zip(vals, vec):
        assert orc.bf16_rne_scalar(float(v)) == b


def test_fp32_mul_rn_against_numpy(orc):
    """fp32 products, including ones that land on subnormals (no flush to zero)."""
    rng = np.random.default_rng(3)
    a = (rng.standard_normal(3000) * 100).astype(np.float32)
    b = np.exp(rng.uniform(-95, -1, size=3000)).astype(np.float32)
    b[:50] = np.float32(1.5e-39)  # subnormal scale
    for x, y in zip(a, b):
        want = np.float32(x) * np.float32(y)
        got = np.float32(orc.fp32_mul_rn(float(x), float(y)))
        assert got.view(np.uint32) == want.view(np.uint32)


def test_dequant_int8_matches_torch(orc):
    import workloads as W
    m = W.random_int8_matrix(1, 333, 517, h_bits=6.0)
    got = orc.dequant(W.INT8, m.symbols, m.scales)
    ref = (torch.from_numpy(m.symbols.view(np.int8)).float() * torch.from_numpy(m.scales)[:, None])
    assert np.array_equal(got, ref.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


def test_dequant_e4m3_matches_torch(orc):
    import workloads as W
    m = W.random_e4m3_matrix(2, 129, 640, alpha=1.0)
    assert len(np.unique(m.symbols)) > 200  # normal range exercised
    got = orc.dequant(W.E4M3, m.symbols, m.scales)
    v = torch.from_numpy(m.symbols).view(torch.float8_e4m3fn).float()
    ref = (v * torch.from_numpy(m.scales)[:, None]).to(torch.bfloat16)
    assert np.array_equal(got, ref.view(torch.int16).numpy().view(np.uint16))


def test_dequant_keeps_negative_zero_and_subnormals(orc):
    sym = np.array([[0x80, 0x00, 0x01, 0x81]], np.uint8)
    got = orc.dequant(2, sym, np.array([1e-37], np.float32))
    v = torch.from_numpy(sym).view(torch.float8_e4m3fn).float() * torch.tensor(1e-37, dtype=torch.float32)
    assert np.array_equal(got, v.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    assert got[0, 0] == 0x8000 and got[0, 1] == 0x0000
    assert got[0, 2] != 0 and (got[0, 2] & 0x7F80) == 0  # a bf16 subnormal, not flushed


def test_dequant_pairs_matches_matrix_dequant(orc):
    import workloads as W
    m = W.random_int8_matrix(3, 40, 96)
    full = orc.dequant(W.INT8, m.symbols, m.scales)
    rows = np.repeat(np.arange(40), 96)
    pairs = orc.dequant_pairs(W.INT8, m.symbols.reshape(-1), m.scales[rows])
    assert np.array_equal(full.reshape(-1), pairs)


def test_scatter_closed_form(orc):
    import workloads as W
    m = W.random_int8_matrix(4, 64, 200, n_out=16)
    base = orc.dequant(W.INT8, m.symbols, m.scales)
    out = base.copy()
    orc.scatter(out, m.out_row, m.out_col, m.out_val)
    mask = np.zeros(base.shape, bool)
    mask[m.out_row, m.out_col] = True
    assert np.array_equal(out[~mask], base[~mask])
    want = torch.from_numpy(m.out_val).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(out[m.out_row, m.out_col], want)
    # outliers are 50-200x the row std: far outside the Int8 * scale range
    assert np.all(np.abs(m.out_val) > 10 * m.scales[m.out_row])


def test_scatter_rejects_unsorted_or_out_of_range(orc):
    out = np.zeros((4, 4), np.uint16)
    with pytest.raises(orc.OracleError):
        orc.scatter(out, [1, 0], [0, 0], [1.0, 2.0])
    with pytest.raises(orc.OracleError):
        orc.scatter(out, [0, 0], [1, 1], [1.0, 2.0])
    with pytest.raises(orc.OracleError):
        orc.scatter(out, [4], [0], [1.0])
