"""GPU parity of the two-chunks-per-warp decode kernel against the CPU oracle,
bit for bit, and its device-side checks.

The kernel only takes launches that give every warp of every SM a pair of
full chunks, so these tests cap the model's decode at one or two SMs
(eq_model_set_sm_limit) to route small matrices through it; eq_decode_plan
confirms the route before each decode.  Leftover chunks (an odd last chunk, a
short tail) go to the general kernel in the same call, so every case also
checks the seam between the two.  Expected values come only from the oracle's
direct dequantisation (EntQuant technical summary, section 2: the coding is
lossless, so the decoded block is unique).
"""
import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu
CHUNK = 65536


@pytest.fixture(scope="module")
def eqw():
    from entropy_coded_weight_b200 import build
    build.build()
    import entropy_coded_weight_b200 as E
    E.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return E


def _decode_block(E, model, layer):
    offs, total = model.block_layout(layer)
    buf = torch.empty(max(total, 16), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    model.decode_block(layer, buf, status)
    torch.cuda.synchronize()
    host = buf.cpu().numpy()
    out = []
    for i, off in zip(model.layer_matrices(layer), offs):
        inf = model.info(i)
        out.append(host[off:off + 2 * inf.rows * inf.cols].view(np.uint16).reshape(inf.rows, inf.cols))
    return out, int(status.item())


def _check(got, mats, orc):
    for g, m in zip(got, mats):
        want = orc.dequant_direct(m)
        if not np.array_equal(g, want):
            bad = np.argwhere(g != want)
            raise AssertionError(f"matrix {m.index} {m.rows}x{m.cols}: {len(bad)} mismatches, first at "
                                 f"{bad[0].tolist()} (chunk {(bad[0][0] * m.cols + bad[0][1]) // CHUNK})")


def _cases():
    # every eligible matrix has >= 96 full chunks (48 pairs: one round of 24 warps on 2 SMs)
    return {
        "int8_exact_round": [W.random_int8_matrix(1, 1536, 4096)],
        "int8_odd_and_tail": [W.random_int8_matrix(2, 1557, 4096, n_out=16)],
        "int8_2p5bit_wide_rows": [W.random_int8_matrix(3, 192, 32768, h_bits=2.5)],
        "e4m3_few_codes": [W.random_e4m3_matrix(4, 1600, 4096, alpha=9e4)],
        "mixed_with_ineligible": [
            W.random_e4m3_matrix(5, 300, 4096, alpha=1.0, layer=0, index=0),
            W.random_int8_matrix(6, 1600, 4096, layer=0, index=1),
            W.random_int8_matrix(7, 100, 2304, layer=0, index=2),
        ],
        "five_matrices_three_per_block": [W.random_int8_matrix(10 + i, 512, 4096, layer=0, index=i)
                                          for i in range(5)],
    }


@pytest.mark.parametrize("sms", [1, 2])
@pytest.mark.parametrize("codec", ["rans", "huffman"])
@pytest.mark.parametrize("case", list(_cases()))
def test_pair_kernel_bit_exact(eqw, orc, case, codec, sms):
    mats = _cases()[case]
    blob = eqw.encode_host(mats, codec=codec)
    model = eqw.Model(eqw.upload(blob), blob)
    model.set_sm_limit(sms)
    plan = model.decode_plan(0, 148)
    if not (case == "five_matrices_three_per_block" and sms == 1):  # one block would span five matrices
        # routed through the pair kernel (whole pairs of full chunks only)
        assert any(plan) and all(p % 2 == 0 for p in plan), plan
    got, st = _decode_block(eqw, model, 0)
    assert st == 0
    _check(got, mats, orc)
    # the per-matrix entry point takes the same route
    for i, m in enumerate(mats):
        out = torch.empty(m.rows * m.cols, dtype=torch.int16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        model.decode_matrix(i, out, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert np.array_equal(out.cpu().numpy().view(np.uint16).reshape(m.rows, m.cols), orc.dequant_direct(m))
    model.close()


def test_pair_kernel_repeatable(eqw, orc):
    """Two decodes into the same buffer give the same bytes (no state leaks
    between launches: ring counters and mbarrier phases restart per launch)."""
    mats = [W.random_int8_matrix(20, 1024, 4096)]
    blob = eqw.encode_host(mats)
    model = eqw.Model(eqw.upload(blob), blob)
    model.set_sm_limit(1)
    a, st_a = _decode_block(eqw, model, 0)
    b, st_b = _decode_block(eqw, model, 0)
    assert st_a == st_b == 0
    assert np.array_equal(a[0], b[0])
    _check(a, mats, orc)
    model.close()


def _corrupt_and_decode(eqw, orc, edit):
    """Upload a 48-chunk Int8 matrix, open the model on the intact bytes, then
    change the device copy with edit(device_bytes, chunk_offsets) and decode
    through the pair kernel; returns the status word."""
    m = W.random_int8_matrix(30, 768, 4096)
    blob = eqw.encode_host([m])
    d_blob = eqw.upload(blob)
    model = eqw.Model(d_blob, blob)
    model.set_sm_limit(1)
    assert model.decode_plan(0, 148) == [48]
    offs = orc.parse_container(blob)["matrices"][0]["chunk_offsets"]
    edit(d_blob, offs)
    _, st = _decode_block(eqw, model, 0)
    model.close()
    return st


def test_pair_kernel_flags_a_changed_table(eqw, orc):
    def edit(d, offs):
        rec = int(offs[10])
        entry = d[rec + 144: rec + 148].clone()
        entry[2] ^= 1                                    # frequency of the first entry, chunk 10
        d[rec + 144: rec + 148] = entry
    st = _corrupt_and_decode(eqw, orc, edit)
    assert st & eqw.EQ_DEV_BAD_TABLE


def test_pair_kernel_flags_a_bad_state(eqw, orc):
    def edit(d, offs):
        rec = int(offs[7])
        d[rec + 16 + 4 * 3: rec + 16 + 4 * 4] = torch.tensor([5, 0, 0, 0], dtype=torch.uint8, device=d.device)
    st = _corrupt_and_decode(eqw, orc, edit)
    assert st & eqw.EQ_DEV_BAD_STATE


def test_pair_kernel_flags_a_changed_word(eqw, orc):
    def edit(d, offs):
        rec = int(offs[9])
        nw_pos = rec + 144 + 4 * int(np.frombuffer(d[rec + 8: rec + 12].cpu().numpy().tobytes(), np.uint32)[0])
        nw_pos = (nw_pos + 15) // 16 * 16 + 40           # a word well inside the payload
        d[nw_pos] ^= 0x5A
    st = _corrupt_and_decode(eqw, orc, edit)
    assert st & eqw.EQ_DEV_BAD_END
