"""Group state for the tensor-parallel all-reduce fused with the residual add
and RMSNorm (``allreduce_fused_add_rms_norm(_fp8)`` in this package; C ABI
``rn_allreduce_comm``).

An ``AllReduceComm`` holds, as seen from this process, every rank's exchange
buffer and signal pad. The kernels number the calls themselves, with a
counter kept in each rank's signal pad (so CUDA-graph replays stay
numbered). Two ways to build one:

* ``AllReduceComm.single_device(world, max_rows, hidden, device)``: the whole
  group on one device (all buffers local; one call computes every rank, with
  operands stacked on a leading rank dimension). This runs the kernel's full
  exchange protocol inside one launch.
* ``AllReduceComm.from_process_group(max_rows, hidden, device, group)``: one
  rank per process and GPU; each process allocates its buffer and pad, and
  the processes exchange CUDA IPC handles over ``torch.distributed``
  (``all_gather_object``), then map their peers' buffers.

Buffers are sized for at most ``max_rows`` rows of ``hidden`` 16-bit values
per call (two halves, alternated by call parity), with room for the two-shot
algorithm unless ``algorithm="one_shot"``. Pads start zero-filled. Every rank
of a group must make the same sequence of calls with the same algorithm.
"""
from __future__ import annotations

import ctypes
import itertools
import weakref
from typing import Optional, Sequence

import torch

from . import ALLREDUCE_ALGORITHMS, ALLREDUCE_MAX_WORLD, ALLREDUCE_SIGNAL_BYTES, RnAllreduceComm

__all__ = ["AllReduceComm", "buffer_bytes_for", "exchange_records", "lookup"]

# Live communicators by integer handle (the torch custom ops take the handle:
# their schemas admit tensors and scalars only).
_LIVE: "weakref.WeakValueDictionary[int, AllReduceComm]" = weakref.WeakValueDictionary()
_HANDLES = itertools.count(1)


def lookup(handle: int) -> "AllReduceComm":
    """The live AllReduceComm with this handle (KeyError when gone)."""
    return _LIVE[handle]


def buffer_bytes_for(max_rows: int, hidden: int, two_shot: bool = True) -> int:
    """Exchange-buffer size for calls of up to max_rows x hidden 16-bit values:
    two halves of T*H values (one-shot) or of 3*T*H values (two-shot too)."""
    return (12 if two_shot else 4) * max_rows * hidden + 32


def exchange_records(record: dict, group=None) -> list[dict]:
    """Gathers one record per rank (ordered by rank) and checks that the
    ranks agree on the buffer geometry; raises ValueError naming the field
    otherwise (on every rank, since every rank sees every record)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    gathered: list = [None] * world
    dist.all_gather_object(gathered, record, group=group)
    for p, rec in enumerate(gathered):
        if rec.get("rank") != p:
            raise ValueError(f"record {p} comes from rank {rec.get('rank')}")
        for key in ("buffer_bytes", "max_rows", "hidden", "world", "algorithm"):
            if rec.get(key) != gathered[0].get(key):
                raise ValueError(f"ranks disagree on {key}: rank 0 has {gathered[0].get(key)}, "
                                 f"rank {p} has {rec.get(key)}")
    return gathered


class AllReduceComm:
    """Exchange buffers and signal pads of one tensor-parallel group, as
    addressed from this process."""

    def __init__(self, world: int, rank: int, local_ranks: int, buffers: Sequence[int],
                 signals: Sequence[int], buffer_bytes: int, timeout_s: float = 1.0,
                 keepalive: Sequence = (), local_pads: Sequence[torch.Tensor] = (),
                 algorithm: str = "auto"):
        if not 1 <= world <= ALLREDUCE_MAX_WORLD:
            raise ValueError(f"world must be 1..{ALLREDUCE_MAX_WORLD}")
        if len(buffers) != world or len(signals) != world:
            raise ValueError("one buffer and one signal pad per rank")
        self.world, self.rank, self.local_ranks = world, rank, local_ranks
        self.buffers, self.signals = list(buffers), list(signals)
        self.buffer_bytes = int(buffer_bytes)
        self.timeout_ns = int(timeout_s * 1e9)
        self.algorithm = algorithm
        self._keepalive = list(keepalive)
        self._local_pads = list(local_pads)
        d = RnAllreduceComm()
        d.world, d.rank, d.local_ranks = world, rank, local_ranks
        d.algorithm = ALLREDUCE_ALGORITHMS[algorithm]
        for p in range(world):
            d.buffers[p] = self.buffers[p]
            d.signals[p] = self.signals[p]
        d.buffer_bytes = self.buffer_bytes
        d.timeout_ns = self.timeout_ns
        self._desc = d
        self._ref = ctypes.byref(d)
        self.handle = next(_HANDLES)
        _LIVE[self.handle] = self

    @property
    def max_elements(self) -> int:
        """Largest T * H one one-shot call may carry (a third of it two-shot)."""
        return ((self.buffer_bytes // 2) & ~15) // 2

    def descriptor(self) -> RnAllreduceComm:
        return self._desc

    def descriptor_ref(self):
        """By-reference rn_allreduce_comm for the C calls."""
        return self._ref

    def call_counters(self) -> list[int]:
        """The call counter of each rank whose pad this process allocated
        (reads device memory; synchronises)."""
        return [int(p[:4].view(torch.int32).item()) & 0xFFFFFFFF for p in self._local_pads]

    @classmethod
    def single_device(cls, world: int, max_rows: int, hidden: int, device,
                      timeout_s: float = 1.0, algorithm: str = "auto") -> "AllReduceComm":
        nbytes = buffer_bytes_for(max_rows, hidden, algorithm != "one_shot")
        bufs = [torch.zeros(nbytes, dtype=torch.uint8, device=device) for _ in range(world)]
        pads = [torch.zeros(ALLREDUCE_SIGNAL_BYTES, dtype=torch.uint8, device=device)
                for _ in range(world)]
        return cls(world, 0, world, [b.data_ptr() for b in bufs], [p.data_ptr() for p in pads],
                   nbytes, timeout_s, keepalive=bufs + pads, local_pads=pads,
                   algorithm=algorithm)

    @classmethod
    def from_process_group(cls, max_rows: int, hidden: int, device, group=None,
                           timeout_s: float = 1.0, algorithm: str = "auto") -> "AllReduceComm":
        import torch.distributed as dist
        world, rank = dist.get_world_size(group), dist.get_rank(group)
        nbytes = buffer_bytes_for(max_rows, hidden, algorithm != "one_shot")
        buf = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        pad = torch.zeros(ALLREDUCE_SIGNAL_BYTES, dtype=torch.uint8, device=device)
        torch.cuda.synchronize(device)  # zeros in place before any peer maps them
        mine = {"rank": rank, "world": world, "buffer_bytes": nbytes, "max_rows": max_rows,
                "hidden": hidden, "algorithm": algorithm, "buffer": _export(buf),
                "signal": _export(pad)}
        records = exchange_records(mine, group)
        keep = [buf, pad]
        bufs, pads = [], []
        for p, rec in enumerate(records):
            if p == rank:
                bufs.append(buf.data_ptr())
                pads.append(pad.data_ptr())
                continue
            b, s = _import(rec["buffer"]), _import(rec["signal"])
            keep += [b, s]
            bufs.append(b.data_ptr())
            pads.append(s.data_ptr())
        dist.barrier(group)  # every rank has mapped every buffer
        return cls(world, rank, 1, bufs, pads, nbytes, timeout_s, keepalive=keep, local_pads=[pad],
                   algorithm=algorithm)


def _export(t: torch.Tensor) -> tuple:
    """CUDA IPC description of a tensor's storage (torch's own sharing path)."""
    return tuple(t.untyped_storage()._share_cuda_())


def _import(handle: Optional[tuple]):
    """Maps a peer's storage from its IPC description."""
    return torch.UntypedStorage._new_shared_cuda(*handle)
