"""Pins for the oracle's scalar rANS coder (oracle/rans_oracle.c).

The pages (EntQuant technical summary, section 2 "weight encoding" and
"inference-time decoding") only say that the weights are compressed
losslessly with an ANS coder and decoded in parallel; they print no worked
example.  The oracle is pinned here by facts that do not depend on its own
code: hand-derived encodings (tests/golden/rans_hand_examples.txt), brute
force over every short sequence on tiny alphabets, the closed-form end state
of a valid rANS stream, the rANS ideal-code-length identity, and the Shannon
bound on the compressed size.
"""
import itertools
import math

import numpy as np
import pytest

from conftest import read_golden


def _table(spec):
    f = np.zeros(256, np.uint32)
    for item in spec.split(","):
        s, v = item.split(":")
        f[int(s, 16)] = int(v)
    return f


def _symbols(spec):
    out = []
    for tok in spec.split():
        if "*" in tok:
            s, k = tok.split("*")
            out += [int(s, 16)] * int(k)
        else:
            out.append(int(tok, 16))
    return np.array(out, np.uint8)


def test_hand_derived_examples(orc):
    rows = read_golden("rans_hand_examples.txt")
    assert len(rows) == 4
    for row in rows:
        name, table, syms, states, words = [c.strip() for c in row.split("|")]
        f = _table(table)
        sym = _symbols(syms)
        st, w, _ = orc.encode_chunk(sym, f)
        want = np.full(32, 65536, np.uint32)
        if states != "-":
            for item in states.split(","):
                lane, val = item.split(":")
                want[int(lane)] = int(val)
        assert st.tolist() == want.tolist(), name
        want_w = [] if words == "-" else [int(x, 16) for x in words.split()]
        assert w.tolist() == want_w, name
        assert orc.decode_chunk(st, w, f, sym.size).tolist() == sym.tolist(), name


def test_lane_step_assignment(orc):
    # within a 256-symbol group, lane l owns symbols 8l .. 8l+7, one per step
    assert orc.symbol_position(0) == (0, 0)
    assert orc.symbol_position(7) == (0, 7)
    assert orc.symbol_position(8) == (1, 0)
    assert orc.symbol_position(255) == (31, 7)
    assert orc.symbol_position(256) == (0, 8)
    seen = {orc.symbol_position(j) for j in range(65536)}
    assert len(seen) == 65536  # a bijection onto (lane, step) pairs


def _all_sequences(k, length):
    return itertools.product(range(k), repeat=length)


@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_brute_force_tiny_alphabets(orc, k):
    """Every sequence of length 1..8 over k symbols round-trips with every state
    in [2^16, 2^32) after each step, under the sequence's own table and under a
    fixed table that gives rare symbols f = 1 (so renormalisation happens)."""
    skewed = np.zeros(256, np.uint32)
    skewed[:k] = 1
    skewed[k - 1] = 4096 - (k - 1)
    tables = [None, skewed]
    n_checked = 0
    for length in range(1, 9):
        for seq in _all_sequences(k, length):
            sym = np.array(seq, np.uint8)
            for tab in tables:
                st, w, f = orc.encode_chunk(sym, tab)
                rc, dec, fin = orc.decode_chunk(st, w, f, sym.size, check_each=True, return_final=True)
                assert rc == 0 and dec.tolist() == list(seq)
                assert fin.tolist() == [65536] * 32
                n_checked += 1
    assert n_checked == 2 * sum(k ** L for L in range(1, 9))


def test_every_tail_shape(orc):
    """n = 1..600 covers every partial 256-symbol group (all 32-lane x 8-step masks)."""
    rng = np.random.default_rng(7)
    for n in range(1, 601):
        sym = rng.integers(0, 5, size=n).astype(np.uint8)
        sym[rng.random(n) < 0.02] = 200  # a rare symbol: frequent renormalisation
        st, w, f = orc.encode_chunk(sym)
        rc, dec, fin = orc.decode_chunk(st, w, f, n, check_each=True, return_final=True)
        assert rc == 0 and np.array_equal(dec, sym), n
        assert fin.tolist() == [65536] * 32


def test_single_symbol_chunk_has_no_payload(orc):
    sym = np.full(65536, 0x80, np.uint8)
    st, w, f = orc.encode_chunk(sym)
    assert f[0x80] == 4096 and w.size == 0 and st.tolist() == [65536] * 32
    assert np.array_equal(orc.decode_chunk(st, w, f, 65536), sym)


def test_full_alphabet_uniform(orc):
    rng = np.random.default_rng(3)
    sym = rng.integers(0, 256, size=65536).astype(np.uint8)
    st, w, f = orc.encode_chunk(sym)
    assert f.sum() == 4096 and np.all(f[np.unique(sym)] >= 1)
    assert np.array_equal(orc.decode_chunk(st, w, f, sym.size), sym)
    # ~8 bits/symbol: 16-bit words ~= n / 2
    assert abs(w.size - 32768) < 400


def _laplace_chunk(h, seed):
    import workloads as W
    return W.laplace_int8_symbols(W.rng_for(77, seed, 0), 1, 65536, h).reshape(-1)


@pytest.mark.parametrize("h", [2.1, 2.5, 3.0])
def test_ideal_code_length_identity(orc, h):
    """rANS coding cost: 16 W + sum_l (log2 x_l - 16) equals sum_j -log2(f_sj / 4096).

    Each encoder step maps x to x * 4096 / f_s up to an additive error below
    4096 on a state of at least 2^16, so the two sides agree to a small
    relative error (measured ~1e-5); a wrong cum, a swapped f or a dropped
    renormalisation breaks it by far more.
    """
    sym = _laplace_chunk(h, int(h * 10))
    st, w, f = orc.encode_chunk(sym)
    cost = 16.0 * w.size + sum(math.log2(int(x)) - 16.0 for x in st)
    info = float(-np.log2(f[sym].astype(np.float64) / 4096.0).sum())
    assert abs(cost - info) <= 1e-4 * info + 64


@pytest.mark.parametrize("h", [2.1, 2.5, 3.0])
def test_size_within_one_percent_of_shannon(orc, h):
    """Payload <= 1.01 x n * H_emp / 8 for a full Laplace chunk (the 32 flushed
    states are counted as header overhead, like the table)."""
    sym = _laplace_chunk(h, 100 + int(h * 10))
    st, w, f = orc.encode_chunk(sym)
    c = np.bincount(sym, minlength=256).astype(np.float64)
    p = c[c > 0] / sym.size
    shannon_bytes = sym.size * float(-(p * np.log2(p)).sum()) / 8.0
    assert 2 * w.size <= 1.01 * shannon_bytes
    assert 2 * w.size + 128 <= 1.02 * shannon_bytes


def test_quantized_table_properties(orc):
    rng = np.random.default_rng(11)
    for trial in range(300):
        k = int(rng.integers(1, 257))
        alphabet = rng.choice(256, size=k, replace=False)
        n = int(rng.integers(1, 65537))
        probs = rng.dirichlet(np.full(k, 0.3))
        sym = rng.choice(alphabet, size=n, p=probs).astype(np.uint8)
        f = orc.quantize_freqs(sym)
        present = np.unique(sym)
        assert f.sum() == 4096
        assert np.all(f[present] >= 1)
        assert np.all(np.delete(f, present) == 0)


def test_quantized_table_rounds_to_nearest(orc):
    # exact halves round up: counts 1 and 3 out of 4 -> 1024 and 3072
    sym = np.array([0, 1, 1, 1], np.uint8)
    f = orc.quantize_freqs(sym)
    assert (f[0], f[1]) == (1024, 3072)
    # 4096/6 = 682.67 -> 683 three times, 3*4096/6 = 2048; the sum 4097 is
    # fixed on the largest f (symbol 3)
    f = orc.quantize_freqs(np.array([0, 1, 2, 3, 3, 3], np.uint8))
    assert f[:4].tolist() == [683, 683, 683, 2047]
    # ties for the largest f go to the smallest byte: 1638.4 -> 1638 twice,
    # 819.2 -> 819, sum 4095, +1 on byte 5 (not byte 9)
    f = orc.quantize_freqs(np.array([5, 5, 9, 9, 1], np.uint8))
    assert (f[1], f[5], f[9]) == (819, 1639, 1638)
    # a symbol seen once in 65536 still gets f = 1; the mode pays for it
    sym = np.zeros(65536, np.uint8)
    sym[5] = 9
    f = orc.quantize_freqs(sym)
    assert (f[0], f[9]) == (4095, 1)


@pytest.mark.parametrize("what", ["word", "state", "table", "extra_word", "missing_word"])
def test_corruption_is_detected(orc, what):
    sym = _laplace_chunk(2.1, 5)
    st, w, f = orc.encode_chunk(sym)
    st, w, f = st.copy(), w.copy(), f.copy()
    if what == "word":
        w[w.size // 2] ^= 0x0100
    elif what == "state":
        st[3] ^= 0x00010000
    elif what == "table":
        f[0] -= 1
    elif what == "extra_word":
        w = np.append(w, np.uint16(7))
    elif what == "missing_word":
        w = w[:-1]
    rc, _, _ = orc.decode_chunk(st, w, f, sym.size, return_final=True)
    assert rc == orc.ERR_CORRUPT


def test_state_below_lower_bound_is_corrupt(orc):
    sym = np.array([1, 0], np.uint8)
    st, w, f = orc.encode_chunk(sym)
    st = st.copy()
    st[7] = 65535
    rc, _, _ = orc.decode_chunk(st, w, f, 2, return_final=True)
    assert rc == orc.ERR_CORRUPT
