"""CUDA IPC plumbing of AllReduceComm.from_process_group: two processes on
one GPU (gloo for the host-side record exchange) allocate their exchange
buffers and signal pads, exchange the IPC handles and map each other's.
Each process then writes a pattern into its own buffer and pad and reads the
peer's through the mapping. No kernel waits on another process here (the
fused kernels' multi-rank path needs one GPU per rank)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import residual_add_rmsnorm_rms_b200 as rn
        from residual_add_rmsnorm_rms_b200.allreduce import AllReduceComm
        torch.cuda.set_device(0)
        comm = AllReduceComm.from_process_group(4, 512, "cuda:0")
        buf, pad = comm._keepalive[0], comm._keepalive[1]
        assert comm.buffers[rank] == buf.data_ptr() and comm.signals[rank] == pad.data_ptr()
        assert comm.local_ranks == 1 and comm.world == world and comm.rank == rank
        assert comm.call_counters() == [0]  # pads start zero-filled
        buf.fill_(17 + rank)
        pad[:64].fill_(100 + rank)
        torch.cuda.synchronize()
        dist.barrier()
        peer = 1 - rank
        stor_b, stor_s = comm._keepalive[2], comm._keepalive[3]
        assert comm.buffers[peer] == stor_b.data_ptr() and comm.signals[peer] == stor_s.data_ptr()
        tb = torch.empty(0, dtype=torch.uint8, device="cuda:0").set_(stor_b)
        ts = torch.empty(0, dtype=torch.uint8, device="cuda:0").set_(stor_s)
        ok_b = bool((tb[: comm.buffer_bytes] == 17 + peer).all())
        ok_s = bool((ts[:64] == 100 + peer).all()) and bool((ts[64:rn.ALLREDUCE_SIGNAL_BYTES] == 0).all())
        dist.barrier()  # the peer's mapping stays valid until both have read
        q.put((rank, ok_b, ok_s))
        del comm, tb, ts, stor_b, stor_s
        torch.cuda.synchronize()
        dist.barrier()
    except Exception as e:  # report, so the parent fails with the reason
        q.put((rank, "error", repr(e)))
    finally:
        dist.destroy_process_group()


def test_from_process_group_maps_peer_buffers():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=120)
    assert sorted(res) == [(0, True, True), (1, True, True)], res
    assert all(p.exitcode == 0 for p in procs)
