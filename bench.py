"""Benchmark: decoded bf16 weight throughput of the entropy-coded weight decoder on B200.

Default workload (N = 1): the streamed 80-layer 70B-shape model -- every
layer's seven matrices (q, o 8192x8192; k, v 1024x8192; gate, up 28672x8192;
down 8192x28672) as Int8 symbols at ~2.1 bits/symbol, rANS-coded in 64 KiB
chunks and resident in HBM (~17 GB), decoded block by block into a bf16
ping-pong buffer pair (EntQuant technical summary, gist.science 2601.22787,
section 2 "inference-time decoding").  Eight distinct seeded layers are
encoded once and placed ten times at distinct HBM addresses; every layer is
far larger than L2, so nothing is served from cache across layers.

One "step" = one pass over all 80 blocks (decode + dequant + ping-pong
events, no-op consumer).  The line also reports the same loop with the
batch-1 bf16 GEMV consumer overlapped, the fused decode + GEMV kernel over
the same blocks, the dominant kernel's roofline, the CPU oracle on the host
cores, an end-to-end number through the public API with the compressed
weights copied from pinned host memory every step, and the GPU encoder's
throughput (it builds the resident model; one layer is cross-checked against
the host encoder byte for byte).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {eqw,reference}]

Multi-GPU (torchrun, one process per GPU): independent replicas, no
collective on the data path (the decode does not shard any exchange);
``value`` is the sum over ranks of decoded bytes divided by the slowest
rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decoded bf16 weight GB/s per B200 (and Gsym/s); % of HBM roofline"
UNIT = "GB/s"

# DRAM bytes (read + write) of one eq_decode_pairs_kernel launch on a
# 70B-shape block, from an ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum) of the same launch configuration, and the SHA-256 of
# the decode sources it was taken on: the figure is reported only while the
# sources are unchanged.
DECODE_TRAFFIC_BYTES = 232_944_384 + 1_652_174_848
DECODE_TRAFFIC_SOURCES_SHA256 = "c666edbb4fc0b5da6aa116bb08ab7b245bdc780b8d4385492f4f919781f9e6c5"
DECODE_SOURCES = ("entropy_coded_weight_b200/csrc/eqw_decode.cu", "entropy_coded_weight_b200/csrc/eqw_device.cuh",
                  "entropy_coded_weight_b200/csrc/eqw_decode_pairs.cu")


def decode_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    root = os.path.dirname(os.path.abspath(__file__))
    for rel in DECODE_SOURCES:
        with open(os.path.join(root, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def decode_traffic() -> int | None:
    if DECODE_TRAFFIC_BYTES is None or decode_sources_sha256() != DECODE_TRAFFIC_SOURCES_SHA256:
        return None
    return DECODE_TRAFFIC_BYTES


FALLBACK_HBM_GBS = 6650.0


# ---------------------------------------------------------------------------
# ranks (plumbing only: NCCL broadcast of the encoded blob, barrier, max/sum)
# ---------------------------------------------------------------------------

class Dist:
    def __init__(self, backend: str | None = None):
        import torch
        import torch.distributed as dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.dist = dist if self.world > 1 else None
        if self.dist is not None and not dist.is_initialized():
            import datetime
            backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
            if backend == "nccl":
                torch.cuda.set_device(self.local_rank)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
        self.backend = dist.get_backend() if self.dist is not None else None

    def _dev(self):
        import torch
        return torch.device("cuda", torch.cuda.current_device()) if self.backend == "nccl" else torch.device("cpu")

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def reduce(self, values: list[float], op: str) -> list[float]:
        if self.dist is None:
            return list(values)
        import torch
        t = torch.tensor(values, dtype=torch.float64, device=self._dev())
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX if op == "max" else self.dist.ReduceOp.SUM)
        return t.cpu().tolist()

    def broadcast_bytes(self, arr: np.ndarray | None) -> np.ndarray:
        """Rank 0's uint8 array on every rank."""
        if self.dist is None:
            return arr
        import torch
        n = torch.tensor([arr.size if self.rank == 0 else 0], dtype=torch.int64, device=self._dev())
        self.dist.broadcast(n, 0)
        if self.rank == 0:
            t = torch.from_numpy(arr).to(self._dev())
        else:
            t = torch.empty(int(n.item()), dtype=torch.uint8, device=self._dev())
        self.dist.broadcast(t, 0)
        return arr if self.rank == 0 else t.cpu().numpy()

    def close(self):
        if self.dist is not None and self.dist.is_initialized():
            self.dist.destroy_process_group()


def combine(local_ms: float, local_units: float, d: Dist) -> tuple[float, float]:
    """(max over ranks of the timed milliseconds, sum over ranks of units)."""
    ms = d.reduce([local_ms], "max")[0]
    units = d.reduce([local_units], "sum")[0]
    return ms, units


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import torch
        self.proc = None
        self.lines: list[str] = []
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", uuid], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for name, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons)}


def measured_bf16_peak() -> float:
    """Dense bf16 TFLOP/s: the measured burst figure, else the recipe's fallback (1590)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


def measured_hbm_peak() -> tuple[float, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            return float(json.load(fh)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# workload: streamed 80-layer 70B-shape model
# ---------------------------------------------------------------------------

N_LAYERS = 80


class DeviceMatrix:
    """A matrix whose symbols and scales live on the GPU (input of eq_encode_device)."""

    def __init__(self, m, device):
        import torch
        self.layer, self.dtype = m.layer, m.dtype
        self.symbols = torch.from_numpy(np.ascontiguousarray(m.symbols)).to(device)
        self.scales = torch.from_numpy(np.ascontiguousarray(m.scales)).to(device)
        self.out_row = self.out_col = self.out_val = None


def oracle_check_sampled_chunks(blob: np.ndarray, mats, threads: int) -> int:
    """Check of the device-encoded container, outside any timed region: the
    oracle decodes the first, the last and one seeded random chunk of every
    matrix of every layer, and each must give the generated symbols back.
    Returns the number of chunks checked; raises on any mismatch."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    parsed = oracle.parse_container(blob)
    if len(parsed["matrices"]) != len(mats):
        raise RuntimeError("device-encoded container: wrong matrix count")
    rng = np.random.default_rng(11)
    jobs = []
    for mi, pm in enumerate(parsed["matrices"]):
        nc = int(pm["n_chunks"])
        for k in sorted({0, nc - 1, int(rng.integers(nc))}):
            jobs.append((mi, k))

    def one(job):
        mi, k = job
        pm, m = parsed["matrices"][mi], mats[mi]
        first = k * oracle.CHUNK_SYMS
        cnt = min(oracle.CHUNK_SYMS, m.n - first)
        sym = oracle._decode_record(parsed["blob"], int(pm["chunk_offsets"][k]), int(pm["chunk_offsets"][k + 1]),
                                    cnt, pm.get("codec", oracle.CODEC_RANS))
        return bool(np.array_equal(sym, np.ascontiguousarray(m.symbols).reshape(-1)[first:first + cnt]))

    with ThreadPoolExecutor(threads) as ex:
        ok = list(ex.map(one, jobs))
    if not all(ok):
        bad = [jobs[i] for i, v in enumerate(ok) if not v][:4]
        raise RuntimeError(f"device-encoded container: the oracle's decode differs at (matrix, chunk) {bad}")
    return len(jobs)


def build_blob(distinct: int, threads: int, device) -> tuple[np.ndarray, dict]:
    """Generate `distinct` seeded 70B-shape Int8 layers (host) and encode them on
    the GPU with eq_encode_device; layer 0 is also encoded on the host, timed,
    and must give the same bytes."""
    import torch

    import entropy_coded_weight_b200 as E
    import workloads as W
    t0 = time.time()
    mats = []
    for layer in range(distinct):
        mats += W.llama70b_int8_layer(layer, 2.1, threads=threads)
    t1 = time.time()
    dmats = [DeviceMatrix(m, device) for m in mats]
    torch.cuda.synchronize(device)
    t2 = time.time()
    d_blob = E.encode_device(dmats)
    t3 = time.time()
    blob = d_blob.cpu().numpy()
    del d_blob, dmats
    n_checked = oracle_check_sampled_chunks(blob, mats, threads)
    n_syms = sum(m.n for m in mats)
    layer0 = [m for m in mats if m.layer == 0]
    t4 = time.time()
    host0 = E.encode_host(layer0, n_threads=threads)
    t5 = time.time()
    same = bool(np.array_equal(host0, E.encode_device([DeviceMatrix(m, device) for m in layer0]).cpu().numpy()))
    n0 = sum(m.n for m in layer0)
    del mats, layer0
    torch.cuda.empty_cache()
    print(f"[bench] generated {distinct} layers in {t1 - t0:.1f}s, device-encoded in {t3 - t2:.1f}s "
          f"({8.0 * blob.size / n_syms:.3f} bits/sym incl. metadata); host encode of one layer {t5 - t4:.1f}s",
          file=sys.stderr, flush=True)
    enc = {"device_gsym_s": round(n_syms / (t3 - t2) / 1e9, 3), "device_s": round(t3 - t2, 2),
           "symbols": n_syms, "host_gsym_s": round(n0 / (t5 - t4) / 1e9, 3), "host_threads": threads,
           "bytes_equal_host": same, "oracle_checked_chunks": n_checked,
           "note": "eq_encode_device on symbols already in HBM (wall clock, it synchronises); host = eq_encode_host "
                   "of layer 0 on all cores; oracle_checked_chunks: first, last and one random chunk of every "
                   "matrix of every layer decoded by the oracle and equal to the generated symbols"}
    if not same:
        raise RuntimeError("device and host encoders disagree")
    return blob, enc


class ResidentStack:
    """`copies` device copies of an encoded `distinct`-layer blob = `n_layers` resident blocks."""

    def __init__(self, blob: np.ndarray, distinct: int, device, n_layers: int = N_LAYERS):
        import torch

        import entropy_coded_weight_b200 as E
        from entropy_coded_weight_b200.streamer import Step
        self.copies = (n_layers + distinct - 1) // distinct
        self.d_blobs = [E.upload(blob, device) for _ in range(self.copies)]
        self.models = [E.Model(d, blob) for d in self.d_blobs]
        self.steps = [Step(self.models[i // distinct], i % distinct) for i in range(n_layers)]
        torch.cuda.synchronize(device)

    def layer_bytes(self, step) -> dict:
        """Algorithmic bytes of one block decode (read compressed + index + scales, write bf16)."""
        m = step.model
        comp = idx = sc = n = 0
        for i in m.layer_matrices(step.layer):
            inf = m.info(i)
            comp += inf.compressed_bytes
            idx += 8 * (inf.n_chunks + 1)
            sc += 4 * inf.rows
            n += inf.rows * inf.cols
        return {"read": comp + idx + sc, "write": 2 * n, "symbols": n}

    def close(self):
        for m in self.models:
            m.close()


def run_pass(streamer, consumer=None, decode_events=None):
    streamer.run(consumer, decode_events)


def timed_passes(streamer, k: int, consumer=None):
    """Time k passes of the ping-pong loop on the device (ms)."""
    import torch
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(streamer.consumer_stream)
    streamer.begin(start)
    for _ in range(k):
        run_pass(streamer, consumer)
    streamer.join()
    end.record(streamer.consumer_stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end)


def isolated_launches(stack, n: int, dev) -> list[float]:
    """Durations (ms) of n block decodes issued back to back on one stream, each
    bracketed by CUDA events on that stream: the dominant kernel on its own."""
    import torch
    s = torch.cuda.Stream(device=dev)
    buf = torch.empty(max(st.model.block_bytes(st.layer) for st in stack.steps), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    pairs = []
    torch.cuda.synchronize()
    for i in range(n):
        st = stack.steps[i % len(stack.steps)]
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(s)
        st.model.decode_block(st.layer, buf, status, s)
        b.record(s)
        pairs.append((a, b))
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"decode status {int(status.item())}")
    return [a.elapsed_time(b) for a, b in pairs]


def oracle_rate(blob: np.ndarray, threads: int, target_s: float, layer: int = 0) -> tuple[int, int, float, int]:
    """The CPU oracle (scalar rANS or Huffman decode + dequant) on chunks of one
    layer, in a seeded random order, ``threads`` at a time, until at least
    ``target_s`` of wall time has passed.  Returns (symbols, chunks, seconds,
    chunks in the layer)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    parsed = oracle.parse_container(blob)
    chunks = [(mi, k) for mi, m in enumerate(parsed["matrices"]) if m["layer"] == layer
              for k in range(m["n_chunks"])]
    chunks = [chunks[i] for i in np.random.default_rng(0).permutation(len(chunks))]

    def one(job):
        mi, k = job
        m = parsed["matrices"][mi]
        n = m["rows"] * m["cols"]
        cnt = min(oracle.CHUNK_SYMS, n - k * oracle.CHUNK_SYMS)
        sym = oracle._decode_record(parsed["blob"], int(m["chunk_offsets"][k]), int(m["chunk_offsets"][k + 1]), cnt,
                                    m.get("codec", oracle.CODEC_RANS))
        first = k * oracle.CHUNK_SYMS
        rows = np.arange(first, first + cnt) // m["cols"]
        oracle.dequant_pairs(m["dtype"], sym, m["scales"][rows])
        return cnt

    # batches of 4 chunks per thread until at least target_s of wall time has passed
    batch = 4 * threads
    done, n_sample, pos = 0, 0, 0
    with ThreadPoolExecutor(threads) as ex:
        t0 = time.perf_counter()
        while True:
            sample = [chunks[(pos + i) % len(chunks)] for i in range(batch)]
            pos += batch
            done += sum(ex.map(one, sample))
            n_sample += batch
            dt = time.perf_counter() - t0
            if dt >= target_s:
                break
    return done, n_sample, dt, len(chunks)


def cpu_oracle_sample(blob: np.ndarray, target_s: float = 12.0) -> dict:
    """The CPU oracle (scalar rANS decode + dequant) on a bounded sample of chunks, all host cores."""
    cores = len(os.sched_getaffinity(0))
    done, n_sample, dt, n_chunks = oracle_rate(blob, cores, target_s)
    return {"value": round(2.0 * done / dt / 1e9, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n_sample} chunks ({done} symbols, cycling over the {n_chunks} chunks of layer 0 "
                      f"in a seeded order), scalar rANS decode + dequant, {cores} threads, {dt:.1f}s",
            "gsym_s": round(done / dt / 1e9, 5)}


def workload_config(layers: int, distinct: int, world: int) -> dict:
    """The bench line's `config`: the streamed 70B-shape model as decoded here."""
    import workloads as W
    per_layer = sum(r * c for r, c in W.LLAMA70B_BLOCK)
    return {"workload": f"streamed {layers}-layer Llama-70B-shape model, Int8 ~2.1 bits/sym, "
                        f"{distinct} distinct layers x {(layers + distinct - 1) // distinct} HBM copies, "
                        "ping-pong bf16 buffers, no-op consumer",
            "layers": layers, "symbols_per_step": layers * per_layer,
            "l2": "inputs larger than L2 (each layer ~0.23 GB compressed, 1.7 GB decoded)",
            "parallelism": f"replicas x{world}"}


def bench_eqw(args, d: Dist) -> dict | None:
    import torch

    from entropy_coded_weight_b200.streamer import GemvConsumer, PingPongStreamer
    import workloads as W

    dev = torch.device("cuda", torch.cuda.current_device())
    threads = len(os.sched_getaffinity(0))
    blob, enc = None, None
    if d.rank == 0:
        blob, enc = build_blob(args.distinct_layers, threads, dev)
    blob = d.broadcast_bytes(blob)
    stack = ResidentStack(blob, args.distinct_layers, dev, args.layers)
    streamer = PingPongStreamer(stack.steps, dev)
    layer_bytes = [stack.layer_bytes(s) for s in stack.steps]
    n_syms_pass = sum(b["symbols"] for b in layer_bytes)
    dec_bytes_pass = 2.0 * n_syms_pass
    alg_bytes_pass = sum(b["read"] + b["write"] for b in layer_bytes)

    # ---- A: no-op consumer ----
    for _ in range(args.warmup):
        run_pass(streamer)
    torch.cuda.synchronize()
    if int(streamer.status.item()) != 0:
        raise RuntimeError(f"decode status {int(streamer.status.item())}")
    d.barrier()
    clocks = ClockSampler(dev.index)
    ms = timed_passes(streamer, args.steps)
    clk = clocks.stop()
    d.barrier()
    ms_max, dec_bytes_all = combine(ms, dec_bytes_pass * args.steps, d)
    value = dec_bytes_all / (ms_max / 1e3) / 1e9
    gsym = value / 2.0

    # dominant kernel: one block decode launch, timed on its own stream
    per_launch = isolated_launches(stack, max(len(stack.steps), 3 * args.distinct_layers), dev)
    launch_ms = statistics.mean(per_launch[len(per_launch) // 4:])
    alg_per_launch = alg_bytes_pass / len(stack.steps)
    peak, peak_kind = measured_hbm_peak()
    achieved = alg_per_launch / (launch_ms / 1e3) / 1e9

    # ---- B: GEMV consumer overlapped ----
    xs, ys = [], []
    for j, (rows, cols) in enumerate(W.LLAMA70B_BLOCK):
        xs.append(W.gemv_activation(0, j, cols).to(dev))
        ys.append(torch.empty(rows, dtype=torch.float32, device=dev))
    gemv = GemvConsumer(xs, ys)
    # the decode blocks leave SMs to the consumer kernels that run beside them
    for m in stack.models:
        m.set_sm_limit(args.consumer_sm_limit)
    for _ in range(max(1, args.warmup)):
        run_pass(streamer, gemv)
    ms_b = timed_passes(streamer, args.steps, gemv)
    for m in stack.models:
        m.set_sm_limit(0)
    ms_b_max, _ = combine(ms_b, 0.0, d)
    value_b = dec_bytes_all / (ms_b_max / 1e3) / 1e9

    # ---- D: the Huffman codec on layer 0 (host-encoded), one block decode at a time ----
    huff = None
    if d.rank == 0:
        import entropy_coded_weight_b200 as E
        layer0 = W.llama70b_int8_layer(0, 2.1, threads=threads)
        hblob = E.encode_host(layer0, n_threads=threads, codec="huffman")
        n0 = sum(m.n for m in layer0)
        del layer0
        hstack = ResidentStack(hblob, 1, dev, 12)
        hb = hstack.layer_bytes(hstack.steps[0])
        per_h = isolated_launches(hstack, 36, dev)
        h_ms = statistics.mean(per_h[len(per_h) // 4:])
        rstep = stack.steps[0]
        r_read = stack.layer_bytes(rstep)["read"]
        huff = {"value": round(2.0 * n0 / (h_ms / 1e3) / 1e9, 2), "unit": UNIT, "launch_ms": round(h_ms, 4),
                "bits_per_sym": round(8.0 * hb["read"] / n0, 4), "rans_bits_per_sym": round(8.0 * r_read / n0, 4),
                "rans_launch_ms": round(launch_ms, 4),
                "note": "layer 0 Huffman-coded (canonical codes <= 12 bits) and decoded by the pair kernel's "
                        "Huffman instance, launches timed alone; bits/sym incl. tables and chunk index"}
        if not args.no_cpu_baseline and d.world == 1:
            # the multi-threaded CPU decode of the same chunks (the oracle's bit-serial Huffman decoder)
            hs, hn, ht, _ = oracle_rate(hblob, threads, 4.0)
            huff["cpu_oracle"] = {"value": round(2.0 * hs / ht / 1e9, 4), "unit": UNIT, "cores": threads,
                                  "sample": f"{hn} chunks of layer 0, {ht:.1f}s"}
        hstack.close()
        del hblob

    # ---- E: prefill on tensor cores: symbols of layer 0 decoded once, the layer's 7 GEMMs in one ----
    # ---- persistent launch over 128, 1024 and 4096 tokens                                        ----
    prefill = None
    if d.rank == 0:
        pstep = stack.steps[0]
        pm = pstep.model
        idx = list(pm.layer_matrices(pstep.layer))
        infos = [pm.info(i) for i in idx]
        syms = [torch.empty(inf.rows * inf.cols, dtype=torch.uint8, device=dev) for inf in infos]
        pst = torch.zeros(1, dtype=torch.int32, device=dev)
        ps = torch.cuda.Stream(device=dev)
        bf16_peak = measured_bf16_peak()

        def p_time(fn, n=5):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(ps)
            for _ in range(n):
                fn()
            b.record(ps)
            torch.cuda.synchronize()
            return a.elapsed_time(b) / n

        dec_ms = p_time(lambda: pm.decode_symbols_block(pstep.layer, syms, pst, ps))
        # comparison path: the same layer decoded to bf16 by eq_decode_block, then one library
        # (torch / cuBLAS) bf16 matmul per matrix; context for the symbol-buffer path, not the product
        offs, total = pm.block_layout(pstep.layer)
        wbuf = torch.empty(total, dtype=torch.uint8, device=dev)
        dec_bf16_ms = p_time(lambda: pm.decode_block(pstep.layer, wbuf, pst, ps))
        wmats = [wbuf[o:o + 2 * inf.rows * inf.cols].view(torch.bfloat16).view(inf.rows, inf.cols)
                 for o, inf in zip(offs, infos)]
        by_tokens = {}
        for tokens in (128, 1024, 4096):
            xs_p = [W.gemv_activation(7, j, tokens * inf.cols).reshape(tokens, inf.cols).to(dev)
                    for j, inf in enumerate(infos)]
            ys_p = [torch.empty(tokens, inf.rows, dtype=torch.float32, device=dev) for inf in infos]
            gemm_ms = p_time(lambda: pm.gemm_symbols_block(pstep.layer, syms, xs_p, ys_p, pst, ps))
            flops = sum(2.0 * tokens * inf.rows * inf.cols for inf in infos)
            tflops = flops / (gemm_ms / 1e3) / 1e12
            row = {"gemm_ms": round(gemm_ms, 4), "tflops": round(tflops, 1), "frac": round(tflops / bf16_peak, 4),
                   "layer_ms": round(dec_ms + gemm_ms, 4)}
            if tokens <= 1024:
                def lib_gemm():
                    with torch.cuda.stream(ps):
                        for x, w in zip(xs_p, wmats):
                            torch.matmul(x, w.t())
                lib_ms = p_time(lib_gemm)
                row["bf16_path"] = {"decode_ms": round(dec_bf16_ms, 4), "library_gemm_ms": round(lib_ms, 4),
                                    "layer_ms": round(dec_bf16_ms + lib_ms, 4)}
            by_tokens[tokens] = row
            del xs_p, ys_p
        if int(pst.item()) != 0:
            raise RuntimeError(f"prefill status {int(pst.item())}")
        prefill = {"tokens": 1024, "decode_symbols_ms": round(dec_ms, 4), **by_tokens[1024],
                   "unit": "TFLOP/s", "bf16_peak": bf16_peak, "tokens_128": by_tokens[128],
                   "tokens_4096": by_tokens[4096],
                   "kernel": "eq_gemm_symbols_pair_kernel (tcgen05.mma.cta_group::2) at 1024 and 4096 tokens, "
                             "eq_gemm_symbols_kernel (cta_group::1, 128-token tiles) at 128",
                   "note": "layer 0: the 7 matrices' symbols decoded to bytes in one launch, then the 7 "
                           "tcgen05 GEMMs in one persistent launch (eq_gemm_symbols_block; 256-row x 256-token "
                           "tiles over CTA pairs, 128-token tiles up to 128 tokens), bf16 tokens, fp32 out; "
                           "frac of the measured "
                           "cuBLAS bf16 burst peak.  bf16_path: the same layer decoded to bf16 by "
                           "eq_decode_block, then one torch (cuBLAS) bf16 matmul per matrix, for comparison"}
        del syms, wbuf, wmats

    # ---- C: fused decode + GEMV, no bf16 buffers; blocks in sequence on one stream ----
    fstream = torch.cuda.Stream(device=dev)
    fys = [torch.empty_like(y) for y in ys]

    def fused_pass():
        for st in stack.steps:
            st.model.decode_gemv_block(st.layer, xs, fys, streamer.status, fstream)

    for _ in range(args.warmup):
        fused_pass()
    torch.cuda.synchronize()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(fstream)
    for _ in range(args.steps):
        fused_pass()
    f1.record(fstream)
    torch.cuda.synchronize()
    if int(streamer.status.item()) != 0:
        raise RuntimeError(f"fused decode status {int(streamer.status.item())}")
    ms_c_max, _ = combine(f0.elapsed_time(f1), 0.0, d)
    value_c = dec_bytes_all / (ms_c_max / 1e3) / 1e9
    fused_read = statistics.mean(b["read"] for b in layer_bytes) + \
        sum(2 * c + 4 * r for r, c in W.LLAMA70B_BLOCK)

    # ---- e2e: compressed weights copied from pinned host memory every step ----
    pinned = torch.from_numpy(blob).pin_memory()
    copy_stream = torch.cuda.Stream(device=dev)
    status_host = torch.zeros(1, dtype=torch.int32).pin_memory()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(copy_stream)
    for _ in range(args.steps):
        # one copy per resident blob; the blocks of a blob decode as soon as it has landed
        landed = []
        with torch.cuda.stream(copy_stream):
            for db in stack.d_blobs:
                db.copy_(pinned, non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(copy_stream)
                landed.append(ev)
        streamer.begin(landed[0])
        streamer.run(None, None, [landed[i // args.distinct_layers] for i in range(len(stack.steps))])
        streamer.join()
        with torch.cuda.stream(streamer.consumer_stream):
            status_host.copy_(streamer.status, non_blocking=True)
        copy_stream.wait_stream(streamer.consumer_stream)
    e1.record(copy_stream)
    torch.cuda.synchronize()
    ms_e = e0.elapsed_time(e1)
    ms_e_max, _ = combine(ms_e, 0.0, d)
    value_e = dec_bytes_all / (ms_e_max / 1e3) / 1e9
    if int(status_host.item()) != 0 or int(streamer.status.item()) != 0:
        raise RuntimeError("decode status nonzero after the e2e loop")

    cpu = cpu_oracle_sample(blob) if (d.rank == 0 and d.world == 1 and not args.no_cpu_baseline) else None
    stack.close()
    if d.rank != 0:
        return None
    # workloads 1-4, one block per launch, each checked against the oracle outside its timing
    per_config = None
    if not args.no_per_config:
        del streamer, pinned
        torch.cuda.empty_cache()
        per_config = per_config_summary(dev, threads, 3, 10, peak)
    launches = len(stack.steps) * args.steps  # one decode kernel per block (no outliers in this workload)
    return {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": d.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u32 rANS state, f32 dequant -> bf16",
        "data": "synthetic (seeded Laplace Int8 symbols at 2.1 bits; no checkpoint)",
        "config": workload_config(args.layers, args.distinct_layers, d.world),
        "gsym_s": round(gsym, 2),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": decode_traffic(),
                     "peak_kind": f"{peak_kind} copy bandwidth", "kernel": "eq_decode_pairs_kernel",
                     "alg_bytes_per_launch": int(alg_per_launch), "launch_ms": round(launch_ms, 4)},
        "with_gemv_consumer": {"value": round(value_b, 2), "unit": UNIT, "ms_per_step": round(ms_b_max / args.steps, 3),
                               "decode_sm_limit": args.consumer_sm_limit,
                               "loop_bytes_frac": round((alg_bytes_pass + dec_bytes_pass) * args.steps
                                                        / (ms_b_max / 1e3) / 1e9 / peak, 4)},
        "with_fused_gemv": {"value": round(value_c, 2), "unit": UNIT,
                            "ms_per_step": round(ms_c_max / args.steps, 3),
                            "ms_per_layer": round(ms_c_max / args.steps / len(stack.steps), 4),
                            "hbm_frac": round(fused_read * len(stack.steps) * args.steps
                                              / (ms_c_max / 1e3) / 1e9 / peak, 4),
                            "kernel": "eq_decode_gemv_kernel",
                            "note": "y = W x per matrix with W decoded in registers; value = bf16 weight bytes "
                                    "consumed per second (2 x symbols / time), one block after another"},
        "huffman": huff,
        "prefill": prefill,
        "e2e": {"value": round(value_e, 2), "unit": UNIT, "h2d_bytes_per_step": int(blob.size * stack.copies),
                "d2h_bytes_per_step": 4, "ms_per_step": round(ms_e_max / args.steps, 3)},
        "cpu_baseline": cpu,
        "per_config": per_config,
        "encode": enc,
        "clocks": clk,
        "gpu_launches": launches,
    }


# ---------------------------------------------------------------------------
# per-workload table: workloads 1-4 one block at a time, workload 5's stream parity
# ---------------------------------------------------------------------------

def _config_rows():
    import workloads as W
    return (
        ("1", "single 1024x1024 Int8 matrix, ~2.1 bits/sym", lambda t: W.single_matrix(2.1)),
        ("2a", "Llama-7B-shape block, Int8 ~2.1 bits/sym", lambda t: W.llama7b_int8_block(2.1, threads=t)),
        ("2b", "Llama-7B-shape block, Int8 ~3.0 bits/sym", lambda t: W.llama7b_int8_block(3.0, threads=t)),
        ("3", "Llama-70B-shape block, E4M3 ~2.1 bits/sym", lambda t: W.llama70b_e4m3_block(2.1, threads=t)),
        ("4", "Llama-7B-shape block, Int8 ~2.5 bits/sym, 16 outliers in down",
         lambda t: W.llama7b_int8_block_with_outliers(threads=t)),
    )


def _block_launches(model, layer: int, n: int, dev, flush=None) -> list[float]:
    """n decodes of one block, each bracketed by CUDA events on its stream; with
    ``flush`` (a buffer larger than L2) rewritten before each, outside the bracket."""
    import torch
    s = torch.cuda.Stream(device=dev)
    buf = torch.empty(model.block_bytes(layer), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    pairs = []
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        for i in range(n):
            if flush is not None:
                flush.fill_(i & 0xFF)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(s)
            model.decode_block(layer, buf, status, s)
            b.record(s)
            pairs.append((a, b))
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"decode status {int(status.item())}")
    return [a.elapsed_time(b) for a, b in pairs]


def _checksums_host(bits: np.ndarray) -> np.ndarray:
    """(sum, row-weighted sum, column-weighted sum) of a uint16 [rows, cols] matrix, exact in int64."""
    v = bits.astype(np.int64)
    rows, cols = v.shape
    return np.array([v.sum(), (v.sum(1) * np.arange(1, rows + 1)).sum(), (v.sum(0) * np.arange(1, cols + 1)).sum()],
                    np.int64)


def _checksums_device(w):
    import torch
    v = w.view(torch.int16).to(torch.int64) & 0xFFFF
    rows, cols = v.shape
    r = torch.arange(1, rows + 1, device=v.device, dtype=torch.int64)
    c = torch.arange(1, cols + 1, device=v.device, dtype=torch.int64)
    return torch.stack([v.sum(), (v.sum(1) * r).sum(), (v.sum(0) * c).sum()])


def configs_table_row(row: dict) -> str:
    """One markdown row of the per-workload results table from a `--configs` JSON line."""
    fl = row["l2_flushed"]
    if "hot" in row:
        gbs = f"{row['hot']['decoded_gb_s']:.1f} / {fl['decoded_gb_s']:.1f}"
        gsym = f"{row['hot']['gsym_s']:.2f} / {fl['gsym_s']:.2f}"
    else:
        gbs, gsym = f"{fl['decoded_gb_s']:.0f}", f"{fl['gsym_s']:.0f}"
    o = row["oracle"]
    return (f"| {row['config']}: {row['workload']} | {row['symbols']:,} | {row['bits_per_sym_records']:.3f} / "
            f"{row['bits_per_sym_container']:.3f} | {gbs} | {gsym} | {100 * fl['hbm_frac']:.1f} % | "
            f"{'yes' if row['bit_exact'] else 'NO'} | {o['gsym_s_1core']:.3f} | {o['gsym_s_all']:.2f} |")


def measure_config(key: str, name: str, mats, blob: np.ndarray, dev, cores: int, flush, warmup: int, steps: int,
                   peak: float) -> dict:
    """One workload block: bit-exactness of the whole decoded block against the
    oracle's direct dequantisation (outside any timed region), then `steps`
    block decodes after `warmup`, each timed with CUDA events on its stream and
    L2 rewritten before it (config 1, which fits in L2, is also timed hot)."""
    import torch

    import entropy_coded_weight_b200 as E
    import oracle
    import workloads as W
    n = sum(m.n for m in mats)
    model = E.Model(E.upload(blob, dev), blob)
    infos = [model.info(i) for i in model.layer_matrices(0)]
    records = sum(i.compressed_bytes for i in infos)
    read = records + sum(8 * (i.n_chunks + 1) + 4 * i.rows + 12 * i.n_outliers for i in infos)
    write = 2 * n + sum(2 * i.n_outliers for i in infos)
    offs, total = model.block_layout(0)
    out = torch.empty(total, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    model.decode_block(0, out, status)
    torch.cuda.synchronize()
    host = out.cpu().numpy()
    exact = int(status.item()) == 0
    for m, o in zip(mats, offs):
        got = host[o:o + 2 * m.n].view(np.uint16).reshape(m.rows, m.cols)
        exact = exact and bool(np.array_equal(got, oracle.dequant_direct(m, threads=cores)))
    del host, out
    lines = {"l2_flushed": statistics.mean(_block_launches(model, 0, warmup + steps, dev, flush)[warmup:])}
    if key == "1":
        lines["hot"] = statistics.mean(_block_launches(model, 0, warmup + 10 * steps, dev)[warmup:])
    row = {"config": key, "workload": name, "symbols": n, "matrices": len(mats),
           "bits_per_sym_records": round(8.0 * records / n, 4),
           "bits_per_sym_container": round(8.0 * blob.size / n, 4),
           "empirical_entropy_bits": round(float(np.mean([W.empirical_entropy_bits(m.symbols) for m in mats])), 4),
           "bit_exact": exact}
    for kind, ms in lines.items():
        row[kind] = {"launch_ms": round(ms, 5), "decoded_gb_s": round(2.0 * n / (ms / 1e3) / 1e9, 1),
                     "gsym_s": round(n / (ms / 1e3) / 1e9, 2),
                     "hbm_frac": round((read + write) / (ms / 1e3) / 1e9 / peak, 4)}
    model.close()
    return row


def per_config_summary(dev, cores: int, warmup: int, steps: int, peak: float) -> dict:
    """Workloads 1-4 one block per launch, compactly, for the bench line."""
    import torch

    import entropy_coded_weight_b200 as E
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # 2 x L2
    res = {}
    for key, name, make in _config_rows():
        mats = make(cores)
        blob = E.encode_host(mats, n_threads=cores)
        row = measure_config(key, name, mats, blob, dev, cores, flush, warmup, steps, peak)
        ent = {"symbols": row["symbols"], "bit_exact": row["bit_exact"],
               "bits_per_sym": row["bits_per_sym_records"]}
        for kind in ("l2_flushed", "hot"):
            if kind in row:
                ent[kind] = {k: row[kind][k] for k in ("launch_ms", "decoded_gb_s", "gsym_s", "hbm_frac")}
        res[key] = ent
        del mats, blob
    del flush
    torch.cuda.empty_cache()
    return res


def bench_configs(args) -> None:
    """One JSON line per workload: decode throughput of one block per launch
    (inputs in HBM, L2 rewritten between launches), compression, bit-exactness
    of the whole block against the oracle, and the oracle's own rate on 1 and
    on all host cores (bounded samples).  Then the streamed 80-layer model's
    parity: every block that the ping-pong loop hands its consumer is
    checksummed on the device and compared with the oracle's, and four layers
    are compared element by element."""
    import torch

    import entropy_coded_weight_b200 as E
    import oracle
    from entropy_coded_weight_b200.streamer import PingPongStreamer
    import workloads as W
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cores = len(os.sched_getaffinity(0))
    peak, peak_kind = measured_hbm_peak()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # 2 x L2
    for key, name, make in _config_rows():
        mats = make(cores)
        blob = E.encode_host(mats, n_threads=cores)
        row = measure_config(key, name, mats, blob, dev, cores, flush, args.warmup, args.steps, peak)
        s1, _, t1, _ = oracle_rate(blob, 1, 3.0)
        sa, _, ta, _ = oracle_rate(blob, cores, 3.0)
        row["oracle"] = {"gsym_s_1core": round(s1 / t1 / 1e9, 5), "gsym_s_all": round(sa / ta / 1e9, 5),
                         "cores": cores, "sample_s": [round(t1, 1), round(ta, 1)]}
        row["peak"] = {"hbm_gbs": peak, "kind": peak_kind}
        print(json.dumps(row), flush=True)
        print(configs_table_row(row), file=sys.stderr, flush=True)
        del mats, blob

    # workload 5: the streamed model; every block checksummed as the consumer sees it
    distinct = args.distinct_layers
    blob, _ = build_blob(distinct, cores, dev)
    stack = ResidentStack(blob, distinct, dev, args.layers)
    streamer = PingPongStreamer(stack.steps, dev)
    sums = torch.zeros(len(stack.steps), 7, 3, dtype=torch.int64, device=dev)

    def consumer(i, step, views, stream):
        for j, w in enumerate(views):
            sums[i, j] = _checksums_device(w)

    run_pass(streamer, consumer)
    streamer.join()
    torch.cuda.synchronize()
    ok_status = int(streamer.status.item()) == 0
    got = sums.cpu().numpy()
    want = np.zeros((distinct, 7, 3), np.int64)
    full = []
    for layer in range(distinct):
        mats = W.llama70b_int8_layer(layer, 2.1, threads=cores)
        direct = [oracle.dequant_direct(m, threads=cores) for m in mats]
        for j, w in enumerate(direct):
            want[layer, j] = _checksums_host(w)
        if layer < 4:  # element by element: block decoded on its own, copied back
            st = next(s for s in stack.steps if s.layer == layer)
            offs, total = st.model.block_layout(layer)
            out = torch.empty(total, dtype=torch.uint8, device=dev)
            status = torch.zeros(1, dtype=torch.int32, device=dev)
            st.model.decode_block(layer, out, status)
            torch.cuda.synchronize()
            host = out.cpu().numpy()
            full.append(int(status.item()) == 0 and all(
                np.array_equal(host[o:o + 2 * m.n].view(np.uint16).reshape(m.rows, m.cols), w)
                for m, o, w in zip(mats, offs, direct)))
            del out, host
        del mats, direct
    match = [bool(np.array_equal(got[i], want[i % distinct])) for i in range(len(stack.steps))]
    print(json.dumps({"config": "5", "workload": f"streamed {args.layers}-layer Llama-70B-shape model, Int8 ~2.1 bits/sym "
                                                  f"({distinct} distinct layers)",
                      "stream_status_ok": ok_status, "blocks_checksum_equal": f"{sum(match)}/{len(match)}",
                      "layers_compared_in_full": len(full), "full_compare_equal": all(full)}), flush=True)
    stack.close()


def bench_reference(args) -> dict:
    """The CPU oracle, as it stands, on host cores: the same metric, unit and
    config as the GPU arm, each step a bounded sample of layer 0's 13,056 chunks
    (the same seeded layer the GPU arm decodes, here encoded by the oracle's own
    encoder)."""
    import oracle
    import workloads as W
    cores = len(os.sched_getaffinity(0))
    mats = W.llama70b_int8_layer(0, 2.1, threads=cores)
    blob = oracle.encode_container(mats, threads=cores)
    del mats
    res = []
    for _ in range(args.warmup + args.steps):
        res.append(cpu_oracle_sample(blob, target_s=max(2.0, 60.0 / max(1, args.warmup + args.steps))))
    timed = res[args.warmup:]
    v = statistics.mean(r["value"] for r in timed)
    cpu = dict(timed[-1])
    cpu["value"] = round(v, 4)
    return {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": UNIT, "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "u32 rANS state, f32 dequant -> bf16",
            "data": "synthetic (seeded Laplace Int8 symbols at 2.1 bits; no checkpoint)",
            "config": workload_config(args.layers, args.distinct_layers, 1),
            "cpu_baseline": cpu, "e2e": {"value": round(v, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                                         "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["eqw", "reference"], default="eqw")
    ap.add_argument("--distinct-layers", type=int, default=8)
    ap.add_argument("--layers", type=int, default=N_LAYERS, help="blocks per pass (80 = the 70B model)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the one-block-per-launch table of workloads 1-4 in the bench line")
    ap.add_argument("--consumer-sm-limit", type=int, default=112,
                    help="SMs the decode launches may use while the GEMV consumer runs beside them (0: all)")
    ap.add_argument("--configs", action="store_true",
                    help="per-workload table (workloads 1-4, stream parity of 5) instead of the bench line")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        print(json.dumps(bench_reference(args)), flush=True)
        return 0

    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    if args.configs:
        bench_configs(args)
        return 0
    d = Dist()
    if d.world == 1:
        torch.cuda.set_device(0)
    try:
        line = bench_eqw(args, d)
    finally:
        d.close()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
