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


def test_configs_table_row_formats_a_result_line():
    row = {"config": "2a", "workload": "Llama-7B-shape block, Int8 ~2.1 bits/sym", "symbols": 202375168,
           "bits_per_sym_records": 2.1251, "bits_per_sym_container": 2.133, "bit_exact": True,
           "l2_flushed": {"launch_ms": 0.231, "decoded_gb_s": 1751.8, "gsym_s": 875.92, "hbm_frac": 0.3078},
           "oracle": {"gsym_s_1core": 0.04253, "gsym_s_all": 0.42649, "cores": 16}}
    line = bench.configs_table_row(row)
    assert line.startswith("| 2a: Llama-7B-shape block") and line.endswith("|")
    cells = [c.strip() for c in line.strip("|").split("|")]
    assert cells[1] == "202,375,168" and cells[2] == "2.125 / 2.133" and cells[3] == "1752"
    assert cells[5] == "30.8 %" and cells[6] == "yes" and cells[8] == "0.43"
    hot = dict(row, hot={"decoded_gb_s": 11.4, "gsym_s": 5.68, "hbm_frac": 0.002})
    assert "11.4 / 1751.8" in bench.configs_table_row(hot)


def test_device_encoder_check_accepts_matching_container_and_catches_a_wrong_one():
    """The bench's gate on the device-encoded model (run before any timing): the oracle decodes the
    first, last and one random chunk of every matrix and compares them with the generated symbols."""
    import entropy_coded_weight_b200 as E
    from entropy_coded_weight_b200 import build
    build.build()
    mats = [W.random_int8_matrix(1, 300, 700, layer=0, index=0),
            W.random_int8_matrix(2, 64, 64, layer=0, index=1),
            W.random_e4m3_matrix(3, 200, 1000, alpha=1.0, layer=1, index=0)]
    blob = E.encode_host(mats)
    # first, last and one seeded random chunk of the 4-chunk matrix (3 distinct here), 1 of each other
    assert bench.oracle_check_sampled_chunks(blob, mats, 2) == 3 + 1 + 1
    wrong = list(mats)
    wrong[1] = W.random_int8_matrix(9, 64, 64, layer=0, index=1)  # other symbols, same shape
    try:
        bench.oracle_check_sampled_chunks(blob, wrong, 2)
    except RuntimeError as e:
        assert "(1, 0)" in str(e)
    else:
        raise AssertionError("a container that does not decode to the generated symbols was accepted")
