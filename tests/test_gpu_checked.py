"""The checked build (libeqw_checked.so, EQ_CHECKED=1) against the release
build: its kernels test their invariants at run time (staging-ring words read
only inside the ring and after their copy was waited for, every slot-table
entry filled, every store inside its matrix, every bulk copy inside its
chunk), report a failure as EQ_DEV_CHECK, and must produce the release
build's bytes.  Each build runs in its own process (the library is chosen at
load time through EQW_LIBRARY); both outputs are also compared with the
oracle's direct dequantisation.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_CHILD = r"""
import json, os, sys
import numpy as np, torch
sys.path.insert(0, os.environ["EQW_ROOT"])
import entropy_coded_weight_b200 as E
L = E.load()
blob = np.load(os.environ["EQW_BLOB"])
model = E.Model(E.upload(blob), blob)
model.set_sm_limit(int(os.environ["EQW_SMS"]))
offs, total = model.block_layout(0)
out = torch.empty(max(total, 16), dtype=torch.uint8, device="cuda")
status = torch.zeros(1, dtype=torch.int32, device="cuda")
model.decode_block(0, out, status)
torch.cuda.synchronize()
np.save(os.environ["EQW_OUT"], out.cpu().numpy()[:total])
print(json.dumps({"checked": int(L.eq_build_checked()), "status": int(status.item())}))
"""


@pytest.fixture(scope="module")
def libs():
    from entropy_coded_weight_b200 import build
    return build.build(), build.build(checked=True)


def _run(lib, blob_path, out_path, sms):
    env = dict(os.environ, EQW_LIBRARY=lib, EQW_ROOT=ROOT, EQW_BLOB=blob_path, EQW_OUT=out_path, EQW_SMS=str(sms))
    r = subprocess.run([sys.executable, "-c", _CHILD], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1]), np.load(out_path)


def _ragged():
    mats = [
        W.random_int8_matrix(1, 300, 229, layer=0, index=0),
        W.random_int8_matrix(2, 1, 1, layer=0, index=1),
        W.random_e4m3_matrix(3, 77, 1000, alpha=1.0, layer=0, index=2),
        W.random_int8_matrix(4, 512, 256, n_out=16, layer=0, index=3),
        W.random_int8_matrix(5, 1000, 264, h_bits=0.05, layer=0, index=4),
        W.random_int8_matrix(6, 129, 1032, h_bits=7.9, layer=0, index=5),
    ]
    single = W.random_int8_matrix(9, 64, 1100, layer=0, index=6)
    single.symbols[:] = 0x81
    mats.append(single)
    return mats


CASES = {
    "ragged_matrix_tables": (_ragged, "rans", "matrix", 0),
    "ragged_chunk_tables": (_ragged, "rans", "chunk", 0),
    "ragged_huffman": (_ragged, "huffman", "matrix", 0),
    "workload1_single_matrix": (lambda: W.single_matrix(2.1), "rans", "matrix", 0),
    "pair_kernel_int8": (lambda: [W.random_int8_matrix(20, 1557, 4096, n_out=8)], "rans", "matrix", 1),
    "pair_kernel_huffman_e4m3": (lambda: [W.random_e4m3_matrix(21, 1600, 4096, alpha=9e4)], "huffman", "matrix", 2),
}


@pytest.mark.parametrize("case", list(CASES))
def test_checked_build_matches_release_and_oracle(libs, orc, tmp_path, case):
    release, checked = libs
    make, codec, scope, sms = CASES[case]
    mats = make()
    import entropy_coded_weight_b200 as E
    blob = E.encode_host(mats, codec=codec, table_scope=scope)
    blob_path = str(tmp_path / "blob.npy")
    np.save(blob_path, blob)
    info_r, out_r = _run(release, blob_path, str(tmp_path / "rel.npy"), sms)
    info_c, out_c = _run(checked, blob_path, str(tmp_path / "chk.npy"), sms)
    assert info_r == {"checked": 0, "status": 0}
    assert info_c == {"checked": 1, "status": 0}      # no invariant failed (EQ_DEV_CHECK clear)
    assert np.array_equal(out_r, out_c)
    # and both are the oracle's direct dequantisation
    model_offsets = []
    off = 0
    for m in mats:
        off = (off + 255) // 256 * 256
        model_offsets.append(off)
        off += 2 * m.n
    for m, o in zip(mats, model_offsets):
        got = out_c[o:o + 2 * m.n].view(np.uint16).reshape(m.rows, m.cols)
        assert np.array_equal(got, orc.dequant_direct(m)), m.index
    assert torch.cuda.is_available()
