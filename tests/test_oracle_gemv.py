"""Pins of the oracle's batch-1 GEMV (oracle.gemv_exact) and bf16 widening.

The fused decode + GEMV path is checked against y = W x computed by the
oracle from the O-direct weights; these tests pin that computation to facts
that do not come from it: torch's own bf16 -> fp32 conversion, a closed-form
sum, the operand orientation, and exact rational arithmetic.
"""
from fractions import Fraction

import numpy as np
import torch


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_bf16_widening_matches_torch_for_every_pattern(orc):
    pats = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = orc.bf16_to_f64(pats)
    ref = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16).float().double().numpy()
    assert np.array_equal(ours, ref, equal_nan=True)
    # signed zero survives
    assert np.signbit(orc.bf16_to_f64(np.array([0x8000], np.uint16)))[0]


def test_orientation_rows_times_x():
    import oracle
    w = _bits(torch.tensor([[1.0, 2.0], [3.0, 4.0]], dtype=torch.bfloat16))
    x = _bits(torch.tensor([1.0, 0.0], dtype=torch.bfloat16))
    y, mag = oracle.gemv_exact(w, x)
    assert list(y) == [1.0, 3.0]  # W^T x would give [1, 2]
    assert list(mag) == [1.0, 3.0]


def test_closed_form_triangular_sum(orc):
    n = 256  # 1..256 are exact in bf16
    w = _bits(torch.ones(3, n, dtype=torch.bfloat16))
    x = _bits(torch.arange(1, n + 1, dtype=torch.float32).to(torch.bfloat16))
    w[1] = _bits(torch.full((n,), -2.0, dtype=torch.bfloat16))
    y, mag = orc.gemv_exact(w, x)
    assert list(y) == [n * (n + 1) / 2, -n * (n + 1), n * (n + 1) / 2]
    assert list(mag) == [n * (n + 1) / 2, n * (n + 1), n * (n + 1) / 2]


def test_against_exact_rationals(orc):
    rng = np.random.default_rng(5)
    w = _bits(torch.from_numpy(rng.standard_normal((7, 13)).astype(np.float32) * 3).to(torch.bfloat16))
    x = _bits(torch.from_numpy(rng.standard_normal(13).astype(np.float32)).to(torch.bfloat16))
    y, mag = orc.gemv_exact(w, x)
    wf, xf = orc.bf16_to_f64(w).reshape(7, 13), orc.bf16_to_f64(x)
    for r in range(7):
        exact = sum(Fraction(float(wf[r, c])) * Fraction(float(xf[c])) for c in range(13))
        absum = sum(abs(Fraction(float(wf[r, c])) * Fraction(float(xf[c]))) for c in range(13))
        assert abs(Fraction(float(y[r])) - exact) <= Fraction(13, 2 ** 53) * absum
        assert float(absum) == mag[r]


# ---- prefill GEMM on symbols (oracle.gemm_symbols_exact) ----

def test_gemm_symbols_orientation_and_scale(orc):
    import workloads as W
    m = W.random_int8_matrix(3, 2, 3)
    m.symbols[:] = np.array([[1, 2, 3], [0xFF, 0, 5]], np.uint8)  # values 1 2 3 / -1 0 5
    m.scales[:] = np.array([0.5, 2.0], np.float32)
    x = _bits(torch.tensor([[1.0, 0.0, 0.0], [0.0, 1.0, 1.0]], dtype=torch.bfloat16))
    y, mag = orc.gemm_symbols_exact(m, x)
    # token 0 selects column 0: [0.5 * 1, 2 * -1]; token 1 sums columns 1, 2: [0.5 * 5, 2 * 5]
    assert y.tolist() == [[0.5, -2.0], [2.5, 10.0]]
    assert mag.tolist() == [[0.5, 2.0], [2.5, 10.0]]


def test_gemm_symbols_e4m3_values_and_outliers(orc):
    import workloads as W
    m = W.random_e4m3_matrix(4, 2, 4)
    m.symbols[:] = np.array([[0x38, 0xB8, 0x01, 0x7E], [0x00, 0x80, 0x40, 0x08]], np.uint8)
    m.scales[:] = 1.0
    m.out_row = np.array([1], np.uint32)
    m.out_col = np.array([3], np.uint32)
    m.out_val = np.array([100.0], np.float32)
    x = _bits(torch.ones(1, 4, dtype=torch.bfloat16))
    y, _ = orc.gemm_symbols_exact(m, x)
    # 0x38 = 1, 0xB8 = -1, 0x01 = 2^-9, 0x7E = 448; row 1: 0, -0, 0x40 = 2, 0x08 = 2^-6 replaced by
    # the placeholder 0 under the super weight, which adds 100
    assert y.tolist() == [[1.0 - 1.0 + 2.0 ** -9 + 448.0, 2.0 + 100.0]]
