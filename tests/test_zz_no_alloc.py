"""eq_encode_device_noalloc: the GPU encoder with its workspace in a file-scope
device array instead of caller memory.

Same bytes as the host encoder; no device memory allocated by the call (free
device memory is unchanged across a call once the library's module is
loaded); EQ_ERR_NOSPACE when the matrices need more workspace than the
array holds.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def eqw():
    from entropy_coded_weight_b200 import build
    build.build()
    import entropy_coded_weight_b200 as E
    E.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return E


class _Dev:
    def __init__(self, m):
        self.layer, self.dtype = m.layer, m.dtype
        self.symbols = torch.from_numpy(np.ascontiguousarray(m.symbols)).cuda()
        self.scales = torch.from_numpy(np.ascontiguousarray(m.scales)).cuda()
        has = len(m.out_row) > 0
        self.out_row = torch.from_numpy(m.out_row.astype(np.int32)).cuda() if has else None
        self.out_col = torch.from_numpy(m.out_col.astype(np.int32)).cuda() if has else None
        self.out_val = torch.from_numpy(m.out_val.astype(np.float32)).cuda() if has else None


def _encode_noalloc(E, dev_mats, scope="matrix"):
    arr, keep = E._device_matrix_in_array(dev_mats, scope)
    L = E.load()
    bound, ln = ctypes.c_size_t(), ctypes.c_size_t()
    assert L.eq_encode_bound(arr, len(dev_mats), ctypes.byref(bound)) == 0
    out = torch.empty(bound.value, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    rc = L.eq_encode_device_noalloc(arr, len(dev_mats), out.data_ptr(), bound.value, ctypes.byref(ln),
                                    torch.cuda.current_stream().cuda_stream)
    free1 = torch.cuda.mem_get_info()[0]
    return rc, out[:ln.value].cpu().numpy(), free0 - free1


@pytest.mark.parametrize("scope", ["matrix", "chunk"])
def test_bytes_equal_host_and_nothing_allocated(eqw, orc, scope):
    mats = [W.random_int8_matrix(1, 300, 1229, n_out=6, layer=0, index=0),
            W.random_e4m3_matrix(2, 77, 1000, alpha=1.0, layer=0, index=1),
            W.random_int8_matrix(3, 512, 2048, h_bits=3.0, layer=1, index=0)]
    dev = [_Dev(m) for m in mats]
    rc, first, _ = _encode_noalloc(eqw, dev, scope)    # loads the module and its scratch array
    assert rc == 0
    rc, got, allocated = _encode_noalloc(eqw, dev, scope)
    assert rc == 0
    assert allocated == 0
    # two calls in a row give the same bytes as the entry point with a caller workspace ...
    with_workspace = eqw.encode_device(dev, table_scope=scope).cpu().numpy()
    assert np.array_equal(first, with_workspace)
    assert np.array_equal(got, with_workspace)
    assert np.array_equal(got, eqw.encode_host(mats, table_scope=scope))
    # ... and the CPU oracle decodes them exactly to its direct dequantisation
    for g, m in zip(orc.decode_container(got), mats):
        assert np.array_equal(g, orc.dequant_direct(m))


def test_reports_nospace_beyond_static_workspace(eqw):
    big = type("M", (), {})()
    big.layer, big.dtype = 0, eqw.EQ_INT8
    big.symbols = torch.zeros((8192, 65536), dtype=torch.uint8, device="cuda")  # 8192 chunks
    big.scales = torch.ones(8192, dtype=torch.float32, device="cuda")
    big.out_row = big.out_col = big.out_val = None
    arr, keep = eqw._device_matrix_in_array([big], "chunk")   # one table per chunk: > 16 MiB of workspace
    L = eqw.load()
    ln = ctypes.c_size_t()
    out = torch.empty(16, dtype=torch.uint8, device="cuda")
    rc = L.eq_encode_device_noalloc(arr, 1, out.data_ptr(), 16, ctypes.byref(ln),
                                    torch.cuda.current_stream().cuda_stream)
    assert rc == 6
