"""Pins of the oracle's Huffman codec (oracle/huffman_oracle.c).

EntroLLM technical overview (gist.science 2505.02380), "method" item 2: the
quantised weights are Huffman coded; item 3: chunks decode in parallel.  The
code construction and the chunk format are readings (length limit 12,
canonical codes, the rANS lane layout, 16-bit refills); these tests tie the
oracle to facts from outside it: textbook and RFC worked examples, a
hand-derived interleaving, an independent dynamic program for optimal
length-limited codes, the Kraft equality, Huffman's H <= L < H + 1 bound, and
exhaustive round trips on tiny inputs.
"""
import functools
import itertools

import numpy as np
import pytest

from conftest import read_golden


def _golden():
    rows = {}
    for line in read_golden("huffman_examples.txt"):
        name, inp, exp = (part.strip() for part in line.split("|"))
        rows[name] = (inp.split(), exp.split())
    return rows


def test_textbook_lengths(orc):
    inp, exp = _golden()["lengths_textbook"]
    counts = np.zeros(256, np.uint64)
    counts[:6] = [int(v) for v in inp]
    ln = orc.huff_lengths(counts=counts)
    assert list(ln[:6]) == [int(v) for v in exp]
    assert not ln[6:].any()


def test_rfc1951_canonical_codes(orc):
    inp, exp = _golden()["canonical_rfc1951"]
    ln = np.zeros(256, np.uint8)
    ln[:8] = [int(v) for v in inp]
    code = orc.huff_canonical(ln)
    assert [format(int(code[i]), f"0{ln[i]}b") for i in range(8)] == exp


def test_hand_derived_interleaving(orc):
    inp, exp = _golden()["interleave_two_lanes"]
    sym = np.array([int(v) for v in inp], np.uint8)
    ln = np.zeros(256, np.uint8)
    ln[:2] = 1
    words, _, single = orc.huff_encode_chunk(sym, ln)
    assert not single
    assert [format(int(w), "04x") for w in words] == exp
    assert np.array_equal(orc.huff_decode_chunk(words, ln, sym.size), sym)


def test_hand_derived_interleaving_multibit_codes(orc):
    inp, exp = _golden()["interleave_rfc_codes"]
    split = inp.index(";")
    ln = np.zeros(256, np.uint8)
    ln[:8] = [int(v) for v in inp[:split]]
    sym = np.array([int(v) for v in inp[split + 1:]], np.uint8)
    words, _, _ = orc.huff_encode_chunk(sym, ln)
    assert [format(int(w), "04x") for w in words] == exp
    assert np.array_equal(orc.huff_decode_chunk(words, ln, sym.size), sym)


def _optimal_cost(weights, limit):
    """Minimum of sum w_i l_i over complete prefix codes with lengths <= limit
    (weights sorted descending => lengths ascending): a dynamic program over
    (symbol, its length, Kraft units used so far)."""
    w = sorted(weights, reverse=True)
    n, full = len(w), 1 << limit

    @functools.lru_cache(maxsize=None)
    def best(i, min_len, used):
        if i == n:
            return 0 if used == full else None
        out = None
        for L in range(max(1, min_len), limit + 1):
            u = used + (1 << (limit - L))
            if u > full:
                continue
            rest = best(i + 1, L, u)
            if rest is not None and (out is None or w[i] * L + rest < out):
                out = w[i] * L + rest
        return out

    return best(0, 1, 0)


@pytest.mark.parametrize("seed", range(6))
def test_lengths_optimal_against_dynamic_program(orc, seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(2, 9))
    counts = np.zeros(256, np.uint64)
    syms = rng.choice(256, size=n, replace=False)
    counts[syms] = rng.integers(1, 1000, size=n)
    ln = orc.huff_lengths(counts=counts)
    cost = int(sum(int(counts[s]) * int(ln[s]) for s in syms))
    assert cost == _optimal_cost([int(counts[s]) for s in syms], 12)


def test_length_limit_binds_and_stays_optimal(orc):
    """Fibonacci weights need depth n - 1 without a limit; with 15 symbols the
    12-bit limit binds, and the cost must still be the constrained optimum."""
    fib = [1, 1]
    while len(fib) < 15:
        fib.append(fib[-1] + fib[-2])
    counts = np.zeros(256, np.uint64)
    counts[10:25] = fib
    ln = orc.huff_lengths(counts=counts)
    assert ln.max() == 12
    cost = int(sum(int(counts[s]) * int(ln[s]) for s in range(10, 25)))
    assert cost == _optimal_cost(fib, 12)


@pytest.mark.parametrize("seed", range(20))
def test_kraft_equality_and_entropy_bound(orc, seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(2, 256))
    counts = np.zeros(256, np.uint64)
    counts[rng.choice(256, size=n, replace=False)] = (rng.pareto(0.7, size=n) * 10 + 1).astype(np.uint64)
    ln = orc.huff_lengths(counts=counts)
    present = counts > 0
    assert np.all(ln[present] >= 1) and np.all(ln[present] <= 12) and not ln[~present].any()
    assert sum(2.0 ** -int(v) for v in ln[present]) == 1.0
    assert orc.huff_canonical(ln) is not None
    p = counts[present] / counts.sum()
    H = float(-(p * np.log2(p)).sum())
    avg = float((counts[present] * ln[present]).sum() / counts.sum())
    if ln.max() < 12:  # unconstrained Huffman: H <= average length < H + 1
        assert H - 1e-12 <= avg < H + 1


def test_single_symbol_chunk_is_empty(orc):
    sym = np.full(1000, 7, np.uint8)
    words, ln, single = orc.huff_encode_chunk(sym)
    assert single and words.size == 0 and not ln.any()
    assert np.array_equal(orc.huff_decode_chunk(words, ln, 1000, single_symbol=7), sym)


def test_exhaustive_round_trip_tiny(orc):
    for alphabet in (2, 3):
        ln = orc.huff_lengths(counts=np.array([1] * alphabet + [0] * (256 - alphabet), np.uint64))
        for n in range(1, 7):
            for seq in itertools.product(range(alphabet), repeat=n):
                sym = np.array(seq, np.uint8)
                words, _, _ = orc.huff_encode_chunk(sym, ln)
                assert np.array_equal(orc.huff_decode_chunk(words, ln, n), sym)


@pytest.mark.parametrize("n", [1, 7, 8, 9, 255, 256, 257, 300, 511, 600, 4097, 65536])
def test_round_trip_tails_and_full_chunk(orc, n):
    import workloads as W
    m = W.random_int8_matrix(7, 1, n, h_bits=2.1)
    sym = m.symbols.reshape(-1)
    words, ln, single = orc.huff_encode_chunk(sym)
    got = orc.huff_decode_chunk(words, ln, n, single_symbol=int(sym[0]) if single else None)
    assert np.array_equal(got, sym)


def test_corruption_detected(orc):
    import workloads as W
    sym = W.random_int8_matrix(8, 1, 5000, h_bits=2.5).symbols.reshape(-1)
    words, ln, _ = orc.huff_encode_chunk(sym)
    for bad in (words[:-1], np.concatenate([words, np.zeros(1, np.uint16)])):
        with pytest.raises(orc.OracleError):
            orc.huff_decode_chunk(bad, ln, sym.size)
    tail = words.copy()
    tail[-1] ^= 1  # the last word's low bit is padding
    with pytest.raises(orc.OracleError):
        orc.huff_decode_chunk(tail, ln, sym.size)
    with pytest.raises(orc.OracleError):  # not a complete code
        bad_ln = ln.copy()
        bad_ln[np.argmax(ln)] += 1
        orc.huff_decode_chunk(words, bad_ln, sym.size)


def test_payload_close_to_entropy(orc):
    """The payload is the codes plus end padding: a lane holds fewer than 12
    unread bits before its last refill, so it leaves at most 11 + 16 bits
    unused.  Integer code lengths cost at most one bit per symbol over H."""
    import workloads as W
    sym = W.random_int8_matrix(9, 1, 65536, h_bits=2.1).symbols.reshape(-1)
    words, ln, _ = orc.huff_encode_chunk(sym)
    c = np.bincount(sym, minlength=256).astype(np.float64)
    p = c[c > 0] / sym.size
    H = float(-(p * np.log2(p)).sum())
    bits_used = float((c * ln).sum())
    assert bits_used <= 16 * words.size <= bits_used + 32 * 27
    assert bits_used <= 1.10 * sym.size * H + sym.size
