"""Host-side pieces of bench.py, on CPU.

The per-workload stream check compares checksums that the GPU computes with
torch on each decoded block against checksums that numpy computes on the
oracle's weights; both must give the same numbers for the same bits and must
change when values move between positions.  The oracle's rate sampler must
decode whole chunks and stop after its time bound.
"""
import numpy as np
import torch

import bench
import oracle
import workloads as W


def test_checksums_agree_between_numpy_and_torch():
    rng = np.random.default_rng(3)
    for shape in [(1, 1), (7, 513), (64, 1024)]:
        bits = rng.integers(0, 1 << 16, size=shape).astype(np.uint16)
        host = bench._checksums_host(bits)
        dev = bench._checksums_device(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)).numpy()
        assert np.array_equal(host, dev)


def test_checksums_see_moved_values():
    bits = np.arange(12, dtype=np.uint16).reshape(3, 4) * 1000 + 7
    base = bench._checksums_host(bits)
    assert not np.array_equal(base, bench._checksums_host(bits.T.copy().reshape(3, 4)))
    swapped = bits.copy()
    swapped[0, 0], swapped[2, 3] = bits[2, 3], bits[0, 0]
    assert not np.array_equal(base, bench._checksums_host(swapped))
    swapped = bits.copy()
    swapped[0, 1], swapped[1, 0] = bits[1, 0], bits[0, 1]
    assert not np.array_equal(base, bench._checksums_host(swapped))


def test_oracle_rate_counts_whole_chunks():
    m = W.random_int8_matrix(40, 96, 2048)  # 3 chunks
    blob = oracle.encode_container([m])
    done, n_sample, dt, n_chunks = bench.oracle_rate(blob, 2, 0.05)
    assert n_chunks == 3
    assert n_sample % 8 == 0 and n_sample >= 8
    # 96 x 2048 = three full chunks of 64 Ki symbols
    assert done == n_sample * 65536
    assert dt >= 0.05


def test_oracle_rate_decodes_huffman_containers():
    m = W.random_int8_matrix(41, 64, 1024)  # one full chunk
    blob = oracle.encode_container([m], codec="huffman")
    done, n_sample, dt, n_chunks = bench.oracle_rate(blob, 1, 0.01)
    assert n_chunks == 1 and done == n_sample * 65536
