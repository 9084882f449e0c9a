"""GPU parity of the tensor-parallel all-reduce fused with the residual add
and RMSNorm (+ FP8), against the oracle's exact all-reduce followed by its
fused ops.

The whole group runs on one device (``AllReduceComm.single_device``): one
cooperative launch computes every rank, and the blocks of different ranks
exchange partials through the same buffers, signal pads and epoch protocol a
multi-GPU group uses, so the protocol is exercised without kernels of
different launches waiting on one another.

Tolerances: the all-reduce sum is exact on these inputs (binary64 holds the
sum of the partials exactly whenever their exponents span at most 42
binades, asserted below from the inputs), so the written-back residual must
be bit-exact, and out / q / scale follow the fused ops' tolerances
(tests/gpu_util.py). Every rank must produce bit-identical results.
"""
import numpy as np
import pytest
import torch

import oracle
import residual_add_rmsnorm_rms_b200 as rn
import synth
from residual_add_rmsnorm_rms_b200 import torch_ops  # noqa: F401  (registers the ops)
from residual_add_rmsnorm_rms_b200.allreduce import AllReduceComm
from tests.cmp_util import bits16
from tests.gpu_util import CORES, compare, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    yield
    assert rn.device_errors() == 0


def _span_ok(parts_bits: np.ndarray, dtype: str) -> bool:
    """Every element's non-zero partials span at most 42 binades (bf16)."""
    if dtype == "fp16":
        return True
    e = ((parts_bits >> 7) & 0xFF).astype(np.int32)
    nz = (parts_bits & 0x7FFF) != 0
    hi = np.where(nz, e, -1).max(axis=0)
    lo = np.where(nz, np.maximum(e, 1), 1000).min(axis=0)
    return bool(((hi < 0) | (hi - lo <= 42)).all())


def _run(fp8, comm, parts, residual, weight, eps, out=None):
    """parts [W, T, H] on the device; residual [T, H] replicated into a
    [W, T, H] stack (updated in place). Returns per-rank outputs."""
    W, T, H = parts.shape
    res = residual.unsqueeze(0).repeat(W, 1, 1).contiguous()
    if fp8:
        q = torch.empty(W, T, H, dtype=torch.float8_e4m3fn, device=parts.device)
        sc = torch.empty(W, T, dtype=torch.float32, device=parts.device)
        rn.allreduce_fused_add_rms_norm_fp8(q, sc, parts, res, weight, eps, comm)
        torch.cuda.synchronize()
        return {"residual": res, "q": q, "scale": sc}
    out = torch.empty_like(parts) if out is None else out
    rn.allreduce_fused_add_rms_norm(out, parts, res, weight, eps, comm)
    torch.cuda.synchronize()
    return {"residual": res, "out": out}


def _check(fp8, got, wl, dtype, rows=None):
    """Rank 0 against the oracle (on `rows`), every other rank against rank 0."""
    parts = bits16(wl.x)
    r_bits, w_bits = bits16(wl.residual), bits16(wl.weight)
    if rows is not None:
        parts, r_bits = parts[:, rows], r_bits[rows]
    assert _span_ok(parts, dtype)
    W = parts.shape[0]
    if fp8:
        _, r2, q, sc = oracle.allreduce_fused_add_rms_norm_fp8(parts, r_bits, w_bits, dtype,
                                                              wl.eps, threads=CORES)
        want = {"residual": r2, "q": q, "scale": sc}
        g0 = {"residual": got["residual"][0], "q": got["q"][0], "scale": got["scale"][0]}
    else:
        _, r2, out = oracle.allreduce_fused_add_rms_norm(parts, r_bits, w_bits, dtype, wl.eps,
                                                        threads=CORES)
        want = {"residual": r2, "out": out}
        g0 = {"residual": got["residual"][0], "out": got["out"][0]}
    stats = compare("fp8" if fp8 else "fused", g0, want, dtype, rows=rows)
    for key, t in got.items():
        a = t.view(torch.uint8) if t.dtype == torch.float8_e4m3fn else t
        for p in range(1, W):
            assert torch.equal(a[p], a[0]), f"rank {p} differs from rank 0 in {key}"
    return stats


# (4, 2048, 1024) and (8, 256, 3840) run the 80-register kernels of groups of
# 4-8 ranks on many rows (two-shot from 2048 rows, one-shot from 256).
CASES = [(1, 1, 512), (2, 7, 512), (2, 300, 3840), (4, 64, 4096), (8, 1, 3840),
         (8, 256, 3840), (3, 33, 1032), (8, 5, 32768), (5, 129, 24), (4, 2048, 1024)]


@pytest.mark.parametrize("W,T,H", CASES)
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("fp8", [False, True], ids=["bf16out", "fp8"])
@pytest.mark.parametrize("algorithm", ["one_shot", "two_shot"])
def test_allreduce_parity(algorithm, fp8, dtype, W, T, H):
    if algorithm == "two_shot" and W < 3:
        pytest.skip("two-shot needs three or more ranks")
    wl = synth.make_tp_inputs(dtype, W, T, H)
    comm = AllReduceComm.single_device(W, T, H, "cuda", algorithm=algorithm)
    got = _run(fp8, comm, wl.x.cuda(), wl.residual.cuda(), wl.weight.cuda(), wl.eps)
    print(_check(fp8, got, wl, dtype))


@pytest.mark.parametrize("W", synth.TP_W)
@pytest.mark.parametrize("fp8", [False, True], ids=["bf16out", "fp8"])
@pytest.mark.parametrize("algorithm", ["one_shot", "auto"])
def test_allreduce_prefill_size(algorithm, fp8, W):
    """Full prefill size [8192 x 3840] bf16, sampled rows against the oracle
    (the automatic choice is two-shot here from four ranks on)."""
    T, H = 8192, 3840
    wl = synth.make_tp_inputs("bf16", W, T, H, device="cuda")
    comm = AllReduceComm.single_device(W, T, H, "cuda", algorithm=algorithm)
    got = _run(fp8, comm, wl.x, wl.residual, wl.weight, wl.eps)
    rows = sample_rows(T, k=96)
    wl.x, wl.residual, wl.weight = wl.x.cpu(), wl.residual.cpu(), wl.weight.cpu()
    print(_check(fp8, got, wl, "bf16", rows=rows))


@pytest.mark.parametrize("algorithm", ["one_shot", "two_shot"])
def test_allreduce_consecutive_calls(algorithm):
    """Calls 1..8 on the same buffers with changing row counts (both buffer
    halves and both flag parities, grids of different sizes, a call with no
    rows in between), each call checked in full; the device call counters
    advance once per call."""
    W, H = 4, 3840
    comm = AllReduceComm.single_device(W, 300, H, "cuda", algorithm=algorithm)
    for i, T in enumerate([5, 300, 1, 0, 64, 300, 2, 17]):
        wl = synth.make_tp_inputs("bf16", W, T, H, seed=100 + i)
        fp8 = i % 2 == 1
        got = _run(fp8, comm, wl.x.cuda(), wl.residual.cuda(), wl.weight.cuda(), wl.eps)
        assert comm.call_counters() == [i + 1] * W
        if T:
            _check(fp8, got, wl, "bf16")


def test_allreduce_in_place_and_no_weight():
    W, T, H = 2, 40, 4096
    wl = synth.make_tp_inputs("fp16", W, T, H)
    comm = AllReduceComm.single_device(W, T, H, "cuda")
    parts = wl.x.cuda()
    got = _run(False, comm, parts, wl.residual.cuda(), None, wl.eps, out=parts)
    assert got["out"].data_ptr() == parts.data_ptr()
    _, r2, out = oracle.allreduce_fused_add_rms_norm(bits16(wl.x), bits16(wl.residual), None,
                                                    "fp16", wl.eps)
    compare("fused", {"residual": got["residual"][1], "out": got["out"][1]},
            {"residual": r2, "out": out}, "fp16")


def test_allreduce_exact_sum_edge_values():
    """Signed zeros, cancellation, subnormals and overflow in the sum (fp16:
    binary64 holds every fp16 sum exactly, so the residual is bit-exact)."""
    W, T, H = 2, 1, 8
    vals = np.array([[0.0, -0.0, 65504.0, -65504.0, 6e-8, 1.0, 1000.0, 0.5],
                     [-0.0, -0.0, 16.0, -8.0, -6e-8, 2.0 ** -11, -1000.0, 0.25]])
    parts = torch.from_numpy(vals.astype(np.float16)).view(W, T, H)
    res = torch.full((T, H), -0.0, dtype=torch.float16)  # x + (-0) == x, signed zeros included
    comm = AllReduceComm.single_device(W, T, H, "cuda")
    got = _run(False, comm, parts.cuda(), res.cuda(), None, 1e-6)
    x, r2, _ = oracle.allreduce_fused_add_rms_norm(bits16(parts), bits16(res), None, "fp16", 1e-6)
    np.testing.assert_array_equal(bits16(got["residual"][0]).reshape(-1), r2.reshape(-1))
    np.testing.assert_array_equal(r2.reshape(-1), x.reshape(-1))  # residual -0: r' = x
    assert r2.reshape(-1)[2] == 0x7C00 and r2.reshape(-1)[1] == 0x8000


def test_allreduce_capacity_and_comm_checks():
    W, T, H = 2, 16, 512
    wl = synth.make_tp_inputs("bf16", W, T, H, device="cuda")
    comm = AllReduceComm.single_device(W, T // 2, H, "cuda", algorithm="one_shot")  # 8 rows
    with pytest.raises(rn.RmsNormError) as e:
        _run(False, comm, wl.x, wl.residual, wl.weight, wl.eps)
    assert e.value.name == "RN_ERR_COMM"
    assert comm.call_counters() == [0, 0]  # a refused call launches nothing
    with pytest.raises(rn.RmsNormError) as e:  # rows not divisible by the ranks
        rn.allreduce_fused_add_rms_norm(torch.empty(3, 5, H, dtype=torch.bfloat16, device="cuda"),
                                        torch.empty(3, 5, H, dtype=torch.bfloat16, device="cuda"),
                                        torch.empty(3, 5, H, dtype=torch.bfloat16, device="cuda"),
                                        None, 1e-6, AllReduceComm.single_device(2, 8, H, "cuda"))
    assert e.value.name == "RN_ERR_SHAPE"
    # two-shot forced on buffers sized for one-shot, and with two ranks
    wl4 = synth.make_tp_inputs("bf16", 4, 8, H, device="cuda")
    small = AllReduceComm.single_device(4, 8, H, "cuda", algorithm="one_shot")
    forced = AllReduceComm(4, 0, 4, small.buffers, small.signals, small.buffer_bytes,
                           keepalive=[small], algorithm="two_shot")
    with pytest.raises(rn.RmsNormError) as e:
        _run(False, forced, wl4.x, wl4.residual, wl4.weight, wl4.eps)
    assert e.value.name == "RN_ERR_COMM"
    with pytest.raises(rn.RmsNormError) as e:
        _run(False, AllReduceComm.single_device(2, T, H, "cuda", algorithm="two_shot"), wl.x,
             wl.residual, wl.weight, wl.eps)
    assert e.value.name == "RN_ERR_COMM"


def test_allreduce_peer_timeout_is_reported():
    """A group of two driven from one rank: the other rank never publishes,
    so every block's bounded wait runs out (50 ms), the blocks leave their
    rows unwritten and the device error flag reports it; the device stays
    usable. (The peer buffer and pad are local allocations nothing writes.)"""
    T, H = 4, 512
    buf = [torch.zeros(4 * T * H + 32, dtype=torch.uint8, device="cuda") for _ in range(2)]
    pad = [torch.zeros(rn.ALLREDUCE_SIGNAL_BYTES, dtype=torch.uint8, device="cuda")
           for _ in range(2)]
    comm = AllReduceComm(2, 0, 1, [b.data_ptr() for b in buf], [p.data_ptr() for p in pad],
                         4 * T * H + 32, timeout_s=0.05, keepalive=buf + pad)
    x = torch.ones(T, H, dtype=torch.bfloat16, device="cuda")
    r = torch.full((T, H), 3.0, dtype=torch.bfloat16, device="cuda")
    out = torch.full((T, H), 7.0, dtype=torch.bfloat16, device="cuda")
    rn.allreduce_fused_add_rms_norm(out, x, r, None, 1e-6, comm)
    torch.cuda.synchronize()
    assert rn.device_errors() == 2
    assert (out == 7.0).all() and (r == 3.0).all()
    # the context still works
    wl = synth.make_tp_inputs("bf16", 2, 3, 512)
    good = AllReduceComm.single_device(2, 3, 512, "cuda")
    _check(False, _run(False, good, wl.x.cuda(), wl.residual.cuda(), wl.weight.cuda(), wl.eps),
           wl, "bf16")


@pytest.mark.parametrize("algorithm", ["one_shot", "two_shot"])
def test_allreduce_cuda_graph_replay(algorithm):
    """Calls captured in a CUDA graph take fresh call numbers on every replay
    (the counter lives in the signal pads), so replays with new data in the
    captured tensors stay correct."""
    W, T, H = 4, 48, 3840
    comm = AllReduceComm.single_device(W, T, H, "cuda", algorithm=algorithm)
    parts = torch.empty(W, T, H, dtype=torch.bfloat16, device="cuda")
    res = torch.empty(W, T, H, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(W, T, H, dtype=torch.bfloat16, device="cuda")
    wl0 = synth.make_tp_inputs("bf16", W, T, H, seed=500)
    weight = wl0.weight.cuda()
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            for _ in range(3):  # three calls per replay, chained through the residual
                rn.allreduce_fused_add_rms_norm(out, parts, res, weight, wl0.eps, comm)
    torch.cuda.synchronize()
    assert comm.call_counters() == [0] * W  # capture launches nothing
    for rep in range(3):
        wl = synth.make_tp_inputs("bf16", W, T, H, seed=501 + rep)
        parts.copy_(wl.x.cuda())
        res.copy_(wl.residual.cuda().unsqueeze(0).expand(W, T, H))
        g.replay()
        torch.cuda.synchronize()
        assert comm.call_counters() == [3 * (rep + 1)] * W
        # expected: the same partials added three times into the residual
        r_bits, w_bits, p_bits = bits16(wl.residual), bits16(wl0.weight), bits16(wl.x)
        for _ in range(3):
            _, r_bits, out_bits = oracle.allreduce_fused_add_rms_norm(p_bits, r_bits, w_bits,
                                                                     "bf16", wl0.eps)
        got = {"residual": res[rep % W], "out": out[rep % W]}
        compare("fused", got, {"residual": r_bits, "out": out_bits}, "bf16")
    del g


def test_allreduce_torch_ops_equal_direct_calls():
    """The torch custom ops (communicator passed by handle) against the
    direct binding, bit for bit, and through torch.compile."""
    W, T, H = 2, 16, 3840
    wl = synth.make_tp_inputs("bf16", W, T, H, seed=77)
    x, w = wl.x.cuda(), wl.weight.cuda()
    res = wl.residual.cuda().unsqueeze(0).repeat(W, 1, 1).contiguous()
    comm = AllReduceComm.single_device(W, T, H, "cuda")
    ra, rb = res.clone(), res.clone()
    out_a = torch.ops.rmsnorm_b200.allreduce_fused_add_rms_norm(x, ra, w, wl.eps, comm.handle)
    out_b = torch.empty_like(x)
    rn.allreduce_fused_add_rms_norm(out_b, x, rb, w, wl.eps, comm)
    torch.cuda.synchronize()
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
    assert torch.equal(ra.view(torch.int16), rb.view(torch.int16))

    def layer(x, r, w):
        return torch.ops.rmsnorm_b200.allreduce_fused_add_rms_norm_fp8(x, r, w, wl.eps,
                                                                       comm.handle)

    rc, re_ = res.clone(), res.clone()
    qc, sc = torch.compile(layer, backend="aot_eager", fullgraph=True)(x, rc, w)
    qe, se = layer(x, re_, w)
    torch.cuda.synchronize()
    assert sc.shape == (W, T, 1)
    assert torch.equal(qc.view(torch.uint8), qe.view(torch.uint8)) and torch.equal(sc, se)
    assert torch.equal(rc.view(torch.int16), re_.view(torch.int16))


@pytest.mark.parametrize("W,T", [(3, 1), (4, 2), (8, 5), (8, 7), (5, 3)])
def test_allreduce_two_shot_fewer_rows_than_ranks(W, T):
    """Two-shot slices of ceil(T / W) rows leave some ranks without rows."""
    H = 512
    for fp8 in (False, True):
        wl = synth.make_tp_inputs("bf16", W, T, H, seed=W * 10 + T)
        comm = AllReduceComm.single_device(W, T, H, "cuda", algorithm="two_shot")
        got = _run(fp8, comm, wl.x.cuda(), wl.residual.cuda(), wl.weight.cuda(), wl.eps)
        _check(fp8, got, wl, "bf16")
