"""Block streaming through a ping-pong buffer pair (host orchestration of eq_decode_model_stream).

EntQuant technical summary (gist.science 2601.22787), section 2
"inference-time decoding": just before each transformer block's forward pass,
a parallel ANS decoder expands that block's weights into a buffer, and
decoding is densely interleaved with the forward kernels.  Here block i+1 is
decoded into buffer (i+1) & 1 on a decode stream while the consumer reads
buffer i & 1 on its own stream; per-buffer "ready" / "free" events order the
two (the waits and records happen inside eq_decode_model_stream on the decode
side and below on the consumer side).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import Model, gemv_bf16


@dataclass
class Step:
    """One block of the stream: layer ``layer`` of ``model``."""
    model: Model
    layer: int


class PingPongStreamer:
    """Decode a sequence of blocks into two alternating bf16 buffers.

    ``steps`` lists the blocks in execution order.  The buffer of step i is
    ``layer & 1`` (eq_decode_model_stream's rule), so consecutive steps must
    alternate layer parity for decode and consumer to overlap (they stay
    correct either way: the events serialise them).
    """

    def __init__(self, steps: list[Step], device=None, decode_priority: int = 0, overlap_decodes: bool = True):
        self.steps = steps
        self.device = torch.device(device or "cuda")
        self.buf_bytes = max(s.model.block_bytes(s.layer) for s in steps)
        self.bufs = [torch.empty(self.buf_bytes, dtype=torch.uint8, device=self.device) for _ in range(2)]
        # One decode stream per buffer lets the decode of block i+1 start while
        # the last chunks of block i are still decoding; the per-buffer events
        # keep each buffer's writer and reader ordered.
        first = torch.cuda.Stream(device=self.device, priority=decode_priority)
        second = torch.cuda.Stream(device=self.device, priority=decode_priority) if overlap_decodes else first
        self.decode_streams = [first, second]
        self.decode_stream = first
        self.consumer_stream = torch.cuda.Stream(device=self.device)
        self.ev_free = [torch.cuda.Event(), torch.cuda.Event()]
        self.ev_ready = [torch.cuda.Event(), torch.cuda.Event()]
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        # events must exist (be recorded once) before the library waits on them
        for e in self.ev_free + self.ev_ready:
            e.record(self.consumer_stream)
        self._layouts = {}

    def layout(self, step: Step):
        key = (id(step.model), step.layer)
        if key not in self._layouts:
            offs, _ = step.model.block_layout(step.layer)
            infos = [step.model.info(m) for m in step.model.layer_matrices(step.layer)]
            self._layouts[key] = [(o, i.rows, i.cols) for o, i in zip(offs, infos)]
        return self._layouts[key]

    def matrix_views(self, buf: torch.Tensor, step: Step) -> list[torch.Tensor]:
        """bf16 [rows, cols] views of one decoded block inside ``buf``."""
        out = []
        for off, rows, cols in self.layout(step):
            out.append(buf[off:off + 2 * rows * cols].view(torch.bfloat16).view(rows, cols))
        return out

    def begin(self, event) -> None:
        """Make both decode streams wait for ``event`` (e.g. the start of a timed region)."""
        for ds in set(self.decode_streams):
            ds.wait_event(event)

    def join(self) -> None:
        """Make the consumer stream wait for all decode work enqueued so far."""
        for ds in set(self.decode_streams):
            self.consumer_stream.wait_stream(ds)

    def run(self, consumer=None, decode_events: list | None = None, ready_events: list | None = None) -> None:
        """Enqueue one pass over all steps.

        ``consumer(i, step, views, stream)`` is called for step i after its
        buffer is ready, with bf16 matrix views, and must only enqueue work on
        ``stream``.  ``decode_events`` (optional) receives (start, end) CUDA
        events recorded on the decode stream around each block decode.
        ``ready_events`` (optional, one per step, entries may be None): the
        decode of step i waits for ``ready_events[i]`` first, e.g. the end of
        the copy that brings its compressed block into device memory, so the
        copies of later blocks overlap the decode of earlier ones.
        """
        for i, step in enumerate(self.steps):
            b = step.layer & 1
            ds = self.decode_streams[b]
            if ready_events is not None and ready_events[i] is not None:
                ds.wait_event(ready_events[i])
            ev0 = ev1 = None
            if decode_events is not None:
                # start after the buffer is free so the pair brackets the kernels only
                ds.wait_event(self.ev_free[b])
                ev0 = torch.cuda.Event(enable_timing=True)
                ev0.record(ds)
            step.model.decode_model_stream(step.layer, self.bufs, self.status, ds, self.ev_free, self.ev_ready)
            if decode_events is not None:
                ev1 = torch.cuda.Event(enable_timing=True)
                ev1.record(ds)
                decode_events.append((ev0, ev1))
            self.consumer_stream.wait_event(self.ev_ready[b])
            if consumer is not None:
                with torch.cuda.stream(self.consumer_stream):
                    consumer(i, step, self.matrix_views(self.bufs[b], step), self.consumer_stream)
            self.ev_free[b].record(self.consumer_stream)


class GemvConsumer:
    """Batch-1 bf16 GEMV of every matrix of a block with a fixed activation per matrix slot."""

    def __init__(self, xs: list[torch.Tensor], ys: list[torch.Tensor]):
        self.xs, self.ys = xs, ys

    def __call__(self, i, step, views, stream):
        for j, w in enumerate(views):
            gemv_bf16(w, self.xs[j], self.ys[j], stream)
