"""GPU tests of block streaming (ping-pong buffers) and its GEMV consumer.

EntQuant technical summary (gist.science 2601.22787), section 2
"inference-time decoding": a block's weights are decoded into a buffer just
before its forward pass, interleaved with the forward kernels.  Expected
values come from the CPU oracle only.
"""
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


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def test_ping_pong_every_block_bit_exact(eqw, orc):
    """Six blocks of three ragged matrices, streamed through two buffers; the
    consumer copies each block out on its own stream, so any ordering slip
    between decode and consumer shows up as a mismatch."""
    from entropy_coded_weight_b200.streamer import PingPongStreamer, Step
    mats = []
    for layer in range(6):
        mats += [W.random_int8_matrix(500 + 10 * layer, 512, 1024, h_bits=2.1, layer=layer, index=0),
                 W.random_int8_matrix(501 + 10 * layer, 256, 520, h_bits=3.0, layer=layer, index=1, n_out=5),
                 W.random_e4m3_matrix(502 + 10 * layer, 300, 2048, alpha=1.0, layer=layer, index=2)]
    blob = eqw.encode_host(mats)
    d_blob = eqw.upload(blob)
    model = eqw.Model(d_blob, blob)
    steps = [Step(model, layer) for layer in range(6)]
    streamer = PingPongStreamer(steps)
    copies = {}

    def consumer(i, step, views, stream):
        copies[i] = [v.clone() for v in views]

    for _ in range(2):
        streamer.run(consumer)
    torch.cuda.synchronize()
    assert int(streamer.status.item()) == 0
    for i in range(6):
        for j, v in enumerate(copies[i]):
            m = mats[3 * i + j]
            assert np.array_equal(_bits(v), orc.dequant_direct(m)), (i, j)
    model.close()


def test_blocks_decode_after_their_copy_lands(eqw, orc):
    """ready_events: every block of two resident copies waits for the host-to-
    device copy of its own container copy, issued on a side stream from pinned
    memory into freshly zeroed device buffers; any decode that ran before its
    copy landed would read zeros and fail the end check or the comparison."""
    from entropy_coded_weight_b200.streamer import PingPongStreamer, Step
    mats = []
    for layer in range(4):
        mats += [W.random_int8_matrix(600 + layer, 1024, 1024, layer=layer, index=0),
                 W.random_int8_matrix(610 + layer, 256, 2048, layer=layer, index=1, n_out=3)]
    blob = eqw.encode_host(mats)
    pinned = torch.from_numpy(blob).pin_memory()
    d_blobs = [torch.zeros(blob.size, dtype=torch.uint8, device="cuda") for _ in range(2)]
    torch.cuda.synchronize()
    models = [eqw.Model(d, blob) for d in d_blobs]
    steps = [Step(models[i // 4], i % 4) for i in range(8)]
    streamer = PingPongStreamer(steps)
    side = torch.cuda.Stream()
    landed = []
    with torch.cuda.stream(side):
        for d in d_blobs:
            torch.cuda._sleep(2_000_000)  # hold the copy back so an unordered decode would overtake it
            d.copy_(pinned, non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(side)
            landed.append(ev)
    copies = {}

    def consumer(i, step, views, stream):
        copies[i] = [v.clone() for v in views]

    streamer.run(consumer, None, [landed[i // 4] for i in range(8)])
    torch.cuda.synchronize()
    assert int(streamer.status.item()) == 0
    for i in range(8):
        for j, v in enumerate(copies[i]):
            assert np.array_equal(_bits(v), orc.dequant_direct(mats[2 * (i % 4) + j])), (i, j)
    for m in models:
        m.close()


def test_gemv_consumer_against_fp64(eqw):
    torch.manual_seed(0)
    for rows, cols in ((1024, 8192), (8192, 28672), (7, 16)):
        w = torch.randn(rows, cols, dtype=torch.float32).to(torch.bfloat16).cuda()
        x = torch.randn(cols, dtype=torch.float32).to(torch.bfloat16).cuda()
        y = torch.empty(rows, dtype=torch.float32, device="cuda")
        eqw.gemv_bf16(w, x, y)
        torch.cuda.synchronize()
        ref = (w.double() @ x.double()).cpu()
        mag = (w.double().abs() @ x.double().abs()).cpu()
        err = (y.double().cpu() - ref).abs()
        # fp32 products are exact for bf16 inputs; the sum rounds at most
        # cols times by 2^-24 relative to the partial sums' magnitude
        assert torch.all(err <= mag * cols * 2.0 ** -24 + 1e-30), float((err / mag).max())


def test_workload5_streamed_80_layers_bench_configuration(eqw, orc):
    """The bench's resident 80-layer stack (8 distinct layers x 10 HBM copies),
    decoded through the ping-pong streamer with the bench's stream setup.
    Full compare of layers 0, 1, 40 and 79; 2^18 seeded sampled positions of
    every matrix of every layer against the oracle one by one."""
    import bench
    from entropy_coded_weight_b200.streamer import PingPongStreamer
    distinct = 8
    layers = [W.llama70b_int8_layer(layer, 2.1) for layer in range(distinct)]
    blob = eqw.encode_host([m for L in layers for m in L])
    dev = torch.device("cuda", torch.cuda.current_device())
    stack = bench.ResidentStack(blob, distinct, dev, bench.N_LAYERS)
    streamer = PingPongStreamer(stack.steps, dev)
    full = {0, 1, 40, 79}
    rng = np.random.default_rng(2026)
    samples = []
    for rows, cols in W.LLAMA70B_BLOCK:
        idx = np.sort(rng.choice(rows * cols, size=1 << 18, replace=False))
        samples.append(torch.from_numpy(idx).to(dev))
    got_full, got_samples = {}, {}

    def consumer(i, step, views, stream):
        got_samples[i] = [v.reshape(-1)[s] for v, s in zip(views, samples)]
        if i in full:
            got_full[i] = [v.clone() for v in views]

    streamer.run(consumer)
    torch.cuda.synchronize()
    assert int(streamer.status.item()) == 0
    for i in range(bench.N_LAYERS):
        src = layers[i % distinct]
        for j, m in enumerate(src):
            s = samples[j].cpu().numpy()
            rows = s // m.cols
            want = orc.dequant_pairs(m.dtype, m.symbols.reshape(-1)[s], m.scales[rows])
            assert np.array_equal(_bits(got_samples[i][j]), want), (i, j)
    for i in sorted(full):
        for j, m in enumerate(layers[i % distinct]):
            assert np.array_equal(_bits(got_full[i][j]), orc.dequant_direct(m)), (i, j)
    stack.close()
