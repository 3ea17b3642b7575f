"""GPU failure detection without a fault: a bounded wait that runs out.

The decode kernels wait on staged copies with a limit of about 2e9 SM cycles.
eq_selftest_wait_timeout drives the decoder's own ring drain on a ring slot
whose copy never started (a completion nothing signals), so the wait must give
up, report EQ_DEV_TIMEOUT through the status word and return.  The context
must stay usable: a decode on the same stream afterwards is still exact.
eq_selftest_gemm_wait_timeout does the same for the prefill GEMM's mbarrier
ring (a "full" barrier nothing arrives on); its tensor memory must be freed on
that path, so a real GEMM afterwards still runs and is exact.
"""
import time

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

EQ_DEV_TIMEOUT = 16


@pytest.fixture(scope="module")
def eqw():
    from entropy_coded_weight_b200 import build
    build.build()
    import entropy_coded_weight_b200 as E
    E.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return E


def test_bounded_wait_reports_timeout_and_context_survives(eqw, orc):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    eqw.selftest_wait_timeout(status)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(status.item()) == EQ_DEV_TIMEOUT
    # the limit is 2e9 cycles: between ~0.5 s (above the max clock) and a few seconds
    assert 0.5 < dt < 10.0, dt

    m = W.random_int8_matrix(7, 96, 1024, layer=0, index=0)
    blob = eqw.encode_host([m])
    model = eqw.Model(eqw.upload(blob), blob)
    out = torch.empty(96 * 1024, dtype=torch.bfloat16, device="cuda")
    status.zero_()
    model.decode_matrix(0, out, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = out.view(torch.int16).cpu().numpy().view(np.uint16).reshape(96, 1024)
    assert np.array_equal(got, orc.dequant_direct(m))
    model.close()


def test_gemm_bounded_wait_reports_timeout_and_frees_tmem(eqw, orc):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    eqw.selftest_gemm_wait_timeout(status)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(status.item()) == EQ_DEV_TIMEOUT
    assert 0.5 < dt < 10.0, dt

    # the same context: a prefill GEMM (which allocates tensor memory again) runs and is exact
    m = W.random_int8_matrix(8, 256, 1024, layer=0, index=0)
    blob = eqw.encode_host([m])
    model = eqw.Model(eqw.upload(blob), blob)
    sym = torch.empty(m.n, dtype=torch.uint8, device="cuda")
    status.zero_()
    model.decode_symbols(0, sym, status)
    tokens = 64
    xt = torch.zeros(tokens, m.cols, dtype=torch.bfloat16)
    xt[torch.arange(tokens), torch.arange(tokens) * 7 % m.cols] = 1.0
    yt = torch.empty(tokens, m.rows, dtype=torch.float32, device="cuda")
    model.gemm_symbols(0, sym, xt.cuda(), yt, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    want, _ = orc.gemm_symbols_exact(m, xt.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(yt.cpu().numpy().view(np.uint32), want.astype(np.float32).view(np.uint32))
    model.close()
