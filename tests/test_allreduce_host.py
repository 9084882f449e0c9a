"""Host-side logic of the tensor-parallel fused all-reduce, on CPU only:
the C ABI's validation of rn_allreduce_comm and of the operands (every
refusal returns before any CUDA call, so host pointers serve as stand-ins),
the epoch sequence of AllReduceComm, and the rank-ordered exchange of buffer
records over torch.distributed (gloo, two processes)."""
import ctypes
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import residual_add_rmsnorm_rms_b200 as rn
from residual_add_rmsnorm_rms_b200.allreduce import (AllReduceComm, buffer_bytes_for,
                                                     exchange_records)


def _comm(world=2, rank=0, local=2, nbytes=None, T=8, H=512, bufs=None, pads=None):
    keep = []
    if bufs is None:
        bufs = []
        for _ in range(world):
            b = torch.zeros(buffer_bytes_for(T, H, False) // 8 + 8, dtype=torch.int64)
            keep.append(b)
            bufs.append(b.data_ptr())
    if pads is None:
        pads = []
        for _ in range(world):
            p = torch.zeros(rn.ALLREDUCE_SIGNAL_BYTES // 8, dtype=torch.int64)
            keep.append(p)
            pads.append(p.data_ptr())
    c = rn.RnAllreduceComm()
    c.world, c.rank, c.local_ranks = world, rank, local
    for i in range(world):
        c.buffers[i], c.signals[i] = bufs[i], pads[i]
    c.buffer_bytes = buffer_bytes_for(T, H, False) if nbytes is None else nbytes
    c.timeout_ns = 0
    return c, keep


def _call(out, x, r, w, comm, fp8=False, scale=None):
    ds = [rn.describe(t) for t in (out, scale, x, r, w)]
    ref = [None if d is None else ctypes.byref(d) for d, _ in ds]
    cref = None if comm is None else ctypes.byref(comm)
    if fp8:
        st = rn.lib.rn_allreduce_fused_add_rms_norm_fp8(ref[0], ref[1], ref[2], ref[3], ref[4],
                                                        1e-6, cref, None)
    else:
        st = rn.lib.rn_allreduce_fused_add_rms_norm(ref[0], ref[2], ref[3], ref[4], 1e-6,
                                                    cref, None)
    return rn.STATUS[st]


def _ops(L=2, T=8, H=512, dt=torch.bfloat16):
    x = torch.zeros(L, T, H, dtype=dt)
    return torch.zeros_like(x), x, torch.zeros_like(x), torch.ones(H, dtype=dt)


def test_comm_validation():
    out, x, r, w = _ops()
    assert _call(out, x, r, w, None) == "RN_ERR_NULL"
    bad = [("world", 0), ("world", 9), ("rank", 2), ("rank", -1), ("rank", 1),  # rank 1 with 2 local
           ("local_ranks", 3), ("local_ranks", 0), ("algorithm", 3), ("algorithm", -1),
           ("algorithm", 2),  # two-shot needs 3 ranks and buffers of 12*T*H + 32
           ("buffer_bytes", buffer_bytes_for(8, 512, False) - 64), ("buffer_bytes", -1)]
    for field, value in bad:
        c, keep = _comm()
        setattr(c, field, value)
        assert _call(out, x, r, w, c) == "RN_ERR_COMM", (field, value)
    o4, x4, r4, _ = _ops(L=4, T=8, H=512)
    c4, keep4 = _comm(world=4, local=4)  # buffers sized for one-shot only
    c4.algorithm = 2
    assert _call(o4, x4, r4, w, c4) == "RN_ERR_COMM"
    c, keep = _comm()
    c.buffers[1] = None
    assert _call(out, x, r, w, c) == "RN_ERR_COMM"
    c, keep = _comm()
    c.signals[0] = c.signals[0] + 4  # misaligned pad
    assert _call(out, x, r, w, c) == "RN_ERR_COMM"
    c, keep = _comm()
    c.buffers[0] = c.buffers[0] + 8  # misaligned buffer
    assert _call(out, x, r, w, c) == "RN_ERR_COMM"


def test_operand_validation():
    c, keep = _comm()
    out, x, r, w = _ops()
    assert _call(out, x.float(), r, w, c) == "RN_ERR_DTYPE"
    assert _call(out, x, r, w.half(), c) == "RN_ERR_WEIGHT_DTYPE"
    o3, x3, r3, _ = _ops(L=3, T=5)  # 15 rows over 2 ranks
    c3, keep3 = _comm(T=16)
    assert _call(o3, x3, r3, w, c3) == "RN_ERR_SHAPE"
    o, xx, rr, ww = _ops(H=1004)  # H % 8 != 0
    c2, keep2 = _comm(H=1004)
    assert _call(o, xx, rr, ww, c2) == "RN_ERR_LAYOUT"
    o, xx, rr, ww = _ops(L=2, T=1, H=32768 + 8)
    c2, keep2 = _comm(T=1, H=32768 + 8)
    assert _call(o, xx, rr, ww, c2) == "RN_ERR_SHAPE"
    # a 16-bit-misaligned view (offset by one element) of a dense buffer
    big = torch.zeros(2 * 8 * 512 + 8, dtype=torch.bfloat16)
    xm = big[1:1 + 2 * 8 * 512].view(2, 8, 512)
    assert _call(out, xm, r, w, c) == "RN_ERR_LAYOUT"
    # residual aliasing x, and an operand inside a local exchange buffer
    assert _call(out, x, x, w, c) == "RN_ERR_ALIAS"
    buf = torch.zeros(buffer_bytes_for(8, 512, False) // 2, dtype=torch.bfloat16)
    cb, keepb = _comm(bufs=[buf.data_ptr(), keep[1].data_ptr()])
    inside = buf[: 2 * 8 * 512].view(2, 8, 512)
    assert _call(inside, x, r, w, cb) == "RN_ERR_ALIAS"
    # fp8 op: q / scale dtypes and sizes (every call here must be refused before
    # any CUDA call: the stand-in pointers are host memory)
    q = torch.zeros(2, 8, 512, dtype=torch.uint8)
    assert _call(q, x, r, w, c, fp8=True, scale=torch.zeros(2, 8, dtype=torch.float64)) == \
        "RN_ERR_DTYPE"
    assert _call(q, x, r, w, c, fp8=True, scale=torch.zeros(2, 7)) == "RN_ERR_SHAPE"
    assert _call(q, x, r, w, c, fp8=True, scale=None) == "RN_ERR_NULL"


def test_comm_descriptor():
    comm = AllReduceComm(2, 0, 2, [16, 32], [48, 64], 4096, timeout_s=0.25)
    d = comm.descriptor()
    assert (d.world, d.rank, d.local_ranks, d.algorithm) == (2, 0, 2, 0)
    assert AllReduceComm(3, 0, 3, [0] * 3, [0] * 3, 64, algorithm="two_shot").descriptor().algorithm == 2
    assert buffer_bytes_for(8, 512) == 12 * 8 * 512 + 32
    assert buffer_bytes_for(8, 512, two_shot=False) == 4 * 8 * 512 + 32
    assert [d.buffers[0], d.buffers[1], d.signals[0], d.signals[1]] == [16, 32, 48, 64]
    assert (d.buffer_bytes, d.timeout_ns) == (4096, 250_000_000)
    assert comm.max_elements == 1024
    assert ctypes.sizeof(rn.RnAllreduceComm) == 3 * 4 + 4 + 2 * 8 * 8 + 2 * 8  # C layout
    with pytest.raises(ValueError):
        AllReduceComm(9, 0, 1, [0] * 9, [0] * 9, 64)
    with pytest.raises(ValueError):
        AllReduceComm(2, 0, 1, [0], [0, 0], 64)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _exchange_worker(rank, world, port, hidden, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rec = {"rank": rank, "world": world, "buffer_bytes": 4096, "max_rows": 2,
               "hidden": hidden[rank], "buffer": ("handle", rank)}
        try:
            got = exchange_records(rec, None)
            q.put((rank, [g["buffer"] for g in got]))
        except ValueError as e:
            q.put((rank, "error: " + str(e)))
    finally:
        dist.destroy_process_group()


def _run_exchange(hidden):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_exchange_worker, args=(r, 2, port, hidden, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def test_exchange_records_orders_by_rank():
    res = _run_exchange([512, 512])
    assert res[0] == res[1] == [("handle", 0), ("handle", 1)]


def test_exchange_records_detects_disagreement():
    res = _run_exchange([512, 1024])
    assert all(isinstance(v, str) and "hidden" in v for v in res.values())


def test_no_alloc_entry_point_validation():
    """Refusals of rn_allreduce_fused_add_rms_norm_local that come before any
    CUDA call (host stand-in pointers are never dereferenced)."""
    def call(out, x, r, w, world):
        ds = [rn.describe(t) for t in (out, x, r, w)]
        ref = [None if d is None else ctypes.byref(d) for d, _ in ds]
        return rn.STATUS[rn.lib.rn_allreduce_fused_add_rms_norm_local(*ref, 1e-6, world, None)]
    out, x, r, w = _ops(L=2, T=8, H=512)
    for world in (0, 9, -1):
        assert call(out, x, r, w, world) == "RN_ERR_COMM"
    assert call(out, x, r, w.half(), 2) == "RN_ERR_WEIGHT_DTYPE"
    o3, x3, r3, _ = _ops(L=3, T=5)
    assert call(o3, x3, r3, w, 2) == "RN_ERR_SHAPE"
    big = torch.zeros(8, 257, 4096, dtype=torch.bfloat16)  # 8 ranks x 257 rows: > 32 MiB
    assert call(torch.zeros_like(big), big, torch.zeros_like(big), None, 8) == "RN_ERR_CAPACITY"
