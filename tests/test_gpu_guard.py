"""Guard regions around every buffer a kernel or entry point writes: each
written buffer sits inside a larger allocation whose bytes before and after it
(GUARD bytes each side) hold a sentinel pattern; after the call the sentinels
must be untouched and the in-bounds results must match the CPU oracle (or,
for the exchange memory, the entry point with unguarded memory, bit for bit).

This stands in for a memory checker (none is available on the GPU machines): it
shows that the predicated vector loads and stores (idle vector slots of a row
group, sub-warp rows, 32-byte vector pairs, 16-byte fallbacks), the scalar
tail on ragged rows and misaligned bases, the staged kernel, the SwiGLU
kernels, the fp8 GEMM's output tiles, the host-memory pipeline's scratch slots
and host outputs, and the all-reduce exchange buffers and signal pads stay
inside their buffers. Small cases only."""
import math

import numpy as np
import pytest
import torch

import oracle
import residual_add_rmsnorm_rms_b200 as rn
import synth
from residual_add_rmsnorm_rms_b200.allreduce import AllReduceComm, buffer_bytes_for
from residual_add_rmsnorm_rms_b200.host import HostPipeline
from tests.cmp_util import bits16, code_dist8, codes8
from tests.gpu_util import CORES, compare, oracle_run
from tests.test_gpu_fp8_gemm import _check as gemm_check

pytestmark = pytest.mark.gpu

GUARD = 256        # sentinel bytes before and after each written buffer
SENTINEL = 0xA5
OPS = ("rms_norm", "fused_add_rms_norm", "fused_add_rms_norm_fp8")


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    rn.force_plan(0, 0)
    rn.force_staged(0, 0, 0)
    rn.set_launch_options(-1, 0)
    yield
    rn.force_plan(0, 0)
    rn.force_staged(0, 0, 0)
    rn.set_launch_options(-1, 0)
    assert rn.device_errors() == 0


class Guarded:
    """A view of `shape` x `dtype` at byte offset GUARD + `shift` of a byte
    buffer filled with SENTINEL (device, or page-locked host memory). Device
    and pinned allocations are at least 512-byte aligned, so `shift` sets the
    view's alignment: 0 gives 256-byte aligned rows' base, 16 a base that is
    16- but not 32-byte aligned, 2 one that is only element aligned."""

    def __init__(self, shape, dtype, shift=0, init=None, device="cuda", pinned=False):
        esize = torch.empty((), dtype=dtype).element_size()
        self.n = math.prod(shape) * esize
        self.off = GUARD + shift
        raw = torch.full((self.off + self.n + GUARD,), SENTINEL, dtype=torch.uint8,
                         device=device)
        self.raw = raw.pin_memory() if pinned else raw
        self.t = self.raw[self.off:self.off + self.n].view(dtype).view(shape)
        if init is not None:
            self.t.copy_(init)

    def assert_intact(self, what=""):
        raw = self.raw.cpu()
        head, tail = raw[:self.off], raw[self.off + self.n:]
        bad_head = int((head != SENTINEL).sum())
        bad_tail = int((tail != SENTINEL).sum())
        assert bad_head == 0 and bad_tail == 0, \
            f"{what}: {bad_head} guard bytes changed before the buffer, {bad_tail} after"


def _inputs(T, H, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    dt = synth.to_dtype(dtype)
    x = synth.normal((T, H), 1.0, g, "cpu").to(dt)
    r = synth.normal((T, H), 4.0, g, "cpu").to(dt)
    w = synth.weight(H, dt, g, "cpu")
    return x, r, w


def _norm_guarded(op, T, H, dtype="bf16", shift=0, seed=0, expect_kernel=None):
    """One call of `op` with x, residual, out, q and scale all guarded."""
    x, r, w = _inputs(T, H, dtype, seed)
    dt = synth.to_dtype(dtype)
    if expect_kernel is not None:
        plan = rn.plan_launch(op, dt, T, H, vector_ok=shift % 16 == 0)
        assert plan["kernel"] == expect_kernel, plan
    gx = Guarded((T, H), dt, shift, x)
    gr = Guarded((T, H), dt, shift, r) if op != "rms_norm" else None
    wd = w.cuda()
    bufs = {"x": gx}
    if op == "fused_add_rms_norm_fp8":
        gq = Guarded((T, H), torch.float8_e4m3fn, shift)
        gs = Guarded((T,), torch.float32, shift & ~3)
        rn.fused_add_rms_norm_fp8(gq.t, gs.t, gx.t, gr.t, wd, 1e-6)
        got = {"q": gq.t, "scale": gs.t, "residual": gr.t}
        bufs.update(q=gq, scale=gs, residual=gr)
    else:
        go = Guarded((T, H), dt, shift)
        if op == "rms_norm":
            rn.rms_norm(go.t, gx.t, wd, 1e-6)
            got = {"out": go.t}
        else:
            rn.fused_add_rms_norm(go.t, gx.t, gr.t, wd, 1e-6)
            got = {"out": go.t, "residual": gr.t}
            bufs["residual"] = gr
        bufs["out"] = go
    torch.cuda.synchronize()
    for name, b in bufs.items():
        b.assert_intact(f"{op} [{T} x {H}] {name}")
    compare(op, got, oracle_run(op, x, r if op != "rms_norm" else None, w, 1e-6, dtype), dtype)


# ---------------------------------------------------------------- vector kernel

@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("T,H", [
    (37, 3840),     # 32-byte vector pairs, four vectors per thread
    (9, 2056),      # idle vector slots in the row group (257 vectors)
    (13, 64),       # sub-warp rows (8 vectors per row)
    (33, 8),        # one vector per row
    (5, 16384),     # wide rows, several warps per row
    (300, 2048),    # many rows per block, ragged last block
])
def test_vector_kernel_stays_in_bounds(op, T, H):
    _norm_guarded(op, T, H, seed=T * 31 + H, expect_kernel=0)


@pytest.mark.parametrize("op", OPS)
def test_vector_kernel_16_byte_accesses_stay_in_bounds(op):
    # base 16- but not 32-byte aligned: the kernel falls back to 16-byte vectors
    _norm_guarded(op, 21, 3840, shift=16, seed=5, expect_kernel=0)


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("tpr,vpt,rpc", [(64, 5, 3), (32, 10, 2), (16, 2, 8), (128, 3, 1)])
def test_forced_shapes_with_idle_slots_stay_in_bounds(op, tpr, vpt, rpc):
    H = 2048 if tpr * vpt * 8 >= 2048 else tpr * vpt * 8 - 8
    rn.force_plan(tpr, vpt, rpc)
    _norm_guarded(op, 19, H, seed=tpr + vpt, expect_kernel=0)


@pytest.mark.parametrize("op", OPS)
def test_capped_grid_strides_stay_in_bounds(op):
    rn.set_launch_options(-1, 3)  # three blocks stride over every row
    _norm_guarded(op, 50, 3840, seed=11, expect_kernel=0)


@pytest.mark.parametrize("op", OPS)
def test_prefetch_stays_in_bounds(op):
    rn.set_prefetch(1)
    try:
        _norm_guarded(op, 41, 3840, seed=12, expect_kernel=0)
    finally:
        rn.set_prefetch(-1)


# ---------------------------------------------------------------- scalar kernel

@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("H,shift", [(100, 0), (1004, 0), (3840, 2), (7, 2)])
def test_scalar_kernel_stays_in_bounds(op, H, shift):
    _norm_guarded(op, 9, H, shift=shift, seed=H + shift, expect_kernel=1)


# ---------------------------------------------------------------- staged kernel

@pytest.mark.parametrize("op", OPS)
def test_staged_kernel_stays_in_bounds(op):
    rn.force_staged(1, 2, 256)
    _norm_guarded(op, 20, 3840, seed=13, expect_kernel=2)


# ---------------------------------------------------------------- SwiGLU + FP8

@pytest.mark.parametrize("T,I,shift", [(5, 2048, 0), (3, 15360, 0), (7, 100, 0), (4, 2048, 2)])
def test_swiglu_stays_in_bounds(T, I, shift):
    g = torch.Generator().manual_seed(T * I)
    x = synth.normal((T, 2 * I), 1.0, g, "cpu").to(torch.bfloat16)
    gx = Guarded((T, 2 * I), torch.bfloat16, shift, x)
    gq = Guarded((T, I), torch.float8_e4m3fn, shift)
    gs = Guarded((T,), torch.float32)
    rn.silu_and_mul_fp8(gq.t, gs.t, gx.t)
    torch.cuda.synchronize()
    for name, b in (("x", gx), ("q", gq), ("scale", gs)):
        b.assert_intact(f"silu_and_mul_fp8 [{T} x {I}] {name}")
    want_q, want_s = oracle.silu_and_mul_fp8(bits16(x), "bf16", threads=CORES)
    assert code_dist8(codes8(gq.t), want_q).max() <= 1
    err = np.abs(gs.t.cpu().numpy().astype(np.float64) - want_s) / np.where(want_s == 0, 1, want_s)
    assert err.max() <= 2e-6


# ---------------------------------------------------------------- fp8 GEMM output

@pytest.mark.parametrize("M,N,K", [(1, 200, 128), (37, 264, 256), (130, 136, 64)])
def test_fp8_gemm_output_stays_in_bounds(M, N, K):
    g = torch.Generator().manual_seed(M + N + K)
    a = (torch.randn(M, K, generator=g) * 40).clamp_(-448, 448).to(torch.float8_e4m3fn)
    b = (torch.randn(N, K, generator=g) * 40).clamp_(-448, 448).to(torch.float8_e4m3fn)
    sa = torch.rand(M, generator=g) * 0.02 + 1e-3
    sb = torch.rand(N, generator=g) * 0.02 + 1e-3
    gd = Guarded((M, N), torch.bfloat16)
    ref = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    args = (a.cuda(), b.cuda(), sa.cuda(), sb.cuda())
    rn.fp8_rowwise_gemm(gd.t, *args)
    rn.fp8_rowwise_gemm(ref, *args)
    torch.cuda.synchronize()
    gd.assert_intact(f"fp8_rowwise_gemm [{M} x {N} x {K}] d")
    assert torch.equal(gd.t.view(torch.int16), ref.view(torch.int16))
    gemm_check(gd.t, codes8(a), codes8(b), sa.numpy(), sb.numpy())


# ---------------------------------------------------------------- host-memory pipeline

@pytest.mark.parametrize("op", OPS)
def test_host_pipeline_scratch_and_host_outputs_stay_in_bounds(op):
    T, H, n, chunk = 29, 3840, 2, 8   # four chunks, ragged last one, over two slots
    x, r, w = _inputs(T, H, "bf16", 17)
    plan = rn.host_plan_chunks(op, T, H, 1 << 50, n, chunk)
    scratch_bytes = plan["slots"] * plan["slot_bytes"]
    pipe = HostPipeline("cuda", scratch_bytes, n, chunk)
    gscr = Guarded((scratch_bytes,), torch.uint8)
    pipe.scratch = gscr.t                      # the pipeline now uses guarded scratch
    pipe._desc.scratch = gscr.t.data_ptr()
    hx = Guarded((T, H), torch.bfloat16, 0, x, device="cpu", pinned=True)
    hr = Guarded((T, H), torch.bfloat16, 0, r, device="cpu", pinned=True)
    wd = w.cuda()
    if op == "fused_add_rms_norm_fp8":
        hq = Guarded((T, H), torch.float8_e4m3fn, 0, device="cpu", pinned=True)
        hs = Guarded((T,), torch.float32, 0, device="cpu", pinned=True)
        rn.host_fused_add_rms_norm_fp8(hq.t, hs.t, hx.t, hr.t, wd, 1e-6, pipe)
        got, outs = {"q": hq.t, "scale": hs.t, "residual": hr.t}, {"q": hq, "scale": hs}
    else:
        ho = Guarded((T, H), torch.bfloat16, 0, device="cpu", pinned=True)
        if op == "rms_norm":
            rn.host_rms_norm(ho.t, hx.t, wd, 1e-6, pipe)
            got = {"out": ho.t}
        else:
            rn.host_fused_add_rms_norm(ho.t, hx.t, hr.t, wd, 1e-6, pipe)
            got = {"out": ho.t, "residual": hr.t}
        outs = {"out": ho}
    pipe.synchronize()
    torch.cuda.synchronize()
    gscr.assert_intact(f"{op} host pipeline scratch")
    for name, b in dict(outs, x=hx, residual=hr).items():
        b.assert_intact(f"{op} host {name}")
    compare(op, got, oracle_run(op, x, r if op != "rms_norm" else None, w, 1e-6, "bf16"), "bf16")


# ---------------------------------------------------------------- all-reduce exchange memory

@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("W,T,algorithm", [(2, 5, "one_shot"), (4, 13, "one_shot"),
                                           (4, 13, "two_shot"), (8, 40, "two_shot")])
def test_allreduce_exchange_memory_stays_in_bounds(W, T, algorithm, fp8):
    H = 3840
    wl = synth.make_tp_inputs("bf16", W, T, H, seed=W * 100 + T, device="cuda")
    res = wl.residual.unsqueeze(0).repeat(W, 1, 1).contiguous()
    nbytes = buffer_bytes_for(T, H, algorithm != "one_shot")
    gbuf = [Guarded((nbytes,), torch.uint8, 0, torch.zeros(nbytes, dtype=torch.uint8))
            for _ in range(W)]
    gpad = [Guarded((rn.ALLREDUCE_SIGNAL_BYTES,), torch.uint8, 0,
                    torch.zeros(rn.ALLREDUCE_SIGNAL_BYTES, dtype=torch.uint8))
            for _ in range(W)]
    comm = AllReduceComm(W, 0, W, [b.t.data_ptr() for b in gbuf], [p.t.data_ptr() for p in gpad],
                         nbytes, keepalive=[b.raw for b in gbuf + gpad],
                         local_pads=[p.t for p in gpad], algorithm=algorithm)
    ref = AllReduceComm.single_device(W, T, H, "cuda", algorithm=algorithm)
    for call in range(3):       # both buffer halves, and a reuse of the first
        gr = Guarded((W, T, H), torch.bfloat16, 0, res)
        rr = res.clone()
        if fp8:
            gq = Guarded((W, T, H), torch.float8_e4m3fn)
            gs = Guarded((W, T), torch.float32)
            qr = torch.empty(W, T, H, dtype=torch.float8_e4m3fn, device="cuda")
            sr = torch.empty(W, T, dtype=torch.float32, device="cuda")
            rn.allreduce_fused_add_rms_norm_fp8(gq.t, gs.t, wl.x, gr.t, wl.weight, wl.eps, comm)
            rn.allreduce_fused_add_rms_norm_fp8(qr, sr, wl.x, rr, wl.weight, wl.eps, ref)
            torch.cuda.synchronize()
            outs = {"q": gq, "scale": gs}
            assert torch.equal(gq.t.view(torch.uint8), qr.view(torch.uint8))
            assert torch.equal(gs.t, sr)
        else:
            go = Guarded((W, T, H), torch.bfloat16)
            orf = torch.empty(W, T, H, dtype=torch.bfloat16, device="cuda")
            rn.allreduce_fused_add_rms_norm(go.t, wl.x, gr.t, wl.weight, wl.eps, comm)
            rn.allreduce_fused_add_rms_norm(orf, wl.x, rr, wl.weight, wl.eps, ref)
            torch.cuda.synchronize()
            outs = {"out": go}
            assert torch.equal(go.t.view(torch.int16), orf.view(torch.int16))
        assert torch.equal(gr.t.view(torch.int16), rr.view(torch.int16))
        for name, b in dict(outs, residual=gr).items():
            b.assert_intact(f"allreduce W={W} T={T} {algorithm} call {call} {name}")
        for p in range(W):
            gbuf[p].assert_intact(f"allreduce W={W} exchange buffer {p} call {call}")
            gpad[p].assert_intact(f"allreduce W={W} signal pad {p} call {call}")
    # the last call's rank-0 rows against the oracle
    xs = bits16(wl.x.cpu())
    if fp8:
        _, r2, q, s = oracle.allreduce_fused_add_rms_norm_fp8(
            xs, bits16(wl.residual.cpu()), bits16(wl.weight.cpu()), "bf16", wl.eps)
        compare("fused_add_rms_norm_fp8", {"q": gq.t[0], "scale": gs.t[0], "residual": gr.t[0]},
                {"q": q, "scale": s, "residual": r2}, "bf16")
    else:
        _, r2, out = oracle.allreduce_fused_add_rms_norm(
            xs, bits16(wl.residual.cpu()), bits16(wl.weight.cpu()), "bf16", wl.eps)
        compare("fused_add_rms_norm", {"out": go.t[0], "residual": gr.t[0]},
                {"out": out, "residual": r2}, "bf16")
