"""Device scratch and streams for the host-memory entry points
(``host_rms_norm``, ``host_fused_add_rms_norm``, ``host_fused_add_rms_norm_fp8``
in this package; C ABI ``rn_host_pipeline``).

The C entry points cut the rows into chunks and send chunk c to stream
c % n and scratch slot c % n: copy in, kernel, copy out. Slot s is therefore
only ever used by stream s, and consecutive calls through one pipeline may
overlap as long as their slots are laid out alike (same op, H and chunk
rows). A HostPipeline fixes the chunk rows when it is made; when a call's
layout differs from the previous call's, it first orders every stream after
the work already queued on all the others, so that slots of different
layouts are never in use at the same time.
"""
from __future__ import annotations

import ctypes

import torch

from . import HOST_MAX_STREAMS, RnHostPipeline, host_plan_chunks

__all__ = ["HostPipeline"]

_UNBOUNDED = 1 << 50  # scratch size that never limits the automatic chunking


class HostPipeline:
    """A device scratch buffer and `n_streams` CUDA streams on one device."""

    def __init__(self, device, scratch_bytes: int, n_streams: int = 3, chunk_rows: int = 0):
        if not 1 <= n_streams <= HOST_MAX_STREAMS:
            raise ValueError(f"n_streams must be 1..{HOST_MAX_STREAMS}")
        dev = torch.device(device)
        if dev.type != "cuda":
            raise ValueError("the pipeline's scratch and streams live on a CUDA device")
        self.device = dev.index if dev.index is not None else torch.cuda.current_device()
        self.chunk_rows = int(chunk_rows)
        self.scratch = torch.empty(max(int(scratch_bytes), 1), dtype=torch.uint8,
                                   device=torch.device("cuda", self.device))
        self.streams = [torch.cuda.Stream(device=self.device) for _ in range(n_streams)]
        self._handles = (ctypes.c_void_p * n_streams)(*[s.cuda_stream for s in self.streams])
        d = RnHostPipeline()
        d.scratch = self.scratch.data_ptr()
        d.scratch_bytes = int(scratch_bytes)
        d.streams = ctypes.cast(self._handles, ctypes.POINTER(ctypes.c_void_p))
        d.n_streams = n_streams
        d.reserved = 0
        d.chunk_rows = self.chunk_rows
        self._desc = d
        self._ref = ctypes.byref(d)
        self._layout = None

    @classmethod
    def for_problem(cls, ops, T: int, H: int, device, n_streams: int = 3) -> "HostPipeline":
        """A pipeline for calls of the ops in `ops` (a name or a list) on up to
        T rows of width H: the automatic chunk rows of the first op at T are
        fixed, and the scratch holds the slots of the largest op."""
        ops = [ops] if isinstance(ops, str) else list(ops)
        rows = host_plan_chunks(ops[0], T, H, _UNBOUNDED, n_streams)["chunk_rows"]
        need = 0
        for op in ops:
            p = host_plan_chunks(op, T, H, _UNBOUNDED, n_streams, rows)
            need = max(need, p["slots"] * p["slot_bytes"])
        return cls(device, need, n_streams, rows)

    def descriptor_ref(self):
        """By-reference rn_host_pipeline for the C calls."""
        return self._ref

    def begin(self, layout, join: bool) -> None:
        """Orders the streams before a call whose slots are laid out by
        `layout` = (op, H). With automatic chunk rows the layout also depends
        on T, so every call counts as a change."""
        cur = torch.cuda.current_stream(self.device)
        if join:
            for s in self.streams:
                s.wait_stream(cur)
        changed = self.chunk_rows <= 0 or layout != self._layout
        if self._layout is not None and changed:
            events = [s.record_event() for s in self.streams]
            for s in self.streams:
                for e in events:
                    s.wait_event(e)
        self._layout = layout

    def end(self, join: bool) -> None:
        if join:
            self.join_into()

    def join_into(self, stream=None) -> None:
        """Makes `stream` (default: the current stream) wait for all the work
        queued on the pipeline's streams."""
        stream = torch.cuda.current_stream(self.device) if stream is None else stream
        for s in self.streams:
            stream.wait_stream(s)

    def wait_for(self, stream=None) -> None:
        """Makes every pipeline stream wait for the work queued on `stream`
        (default: the current stream)."""
        stream = torch.cuda.current_stream(self.device) if stream is None else stream
        for s in self.streams:
            s.wait_stream(stream)

    def synchronize(self) -> None:
        for s in self.streams:
            s.synchronize()
