"""Host logic of the host-memory entry points, on CPU only: the chunking rule
of rn_host_plan_chunks restated from its documentation, and the refusals of
rn_host_* (every one returns before any CUDA call, so host buffers stand in
for the device scratch). The refusal test is skipped where a GPU is present:
a call that wrongly got past validation would copy and launch there."""
import ctypes

import pytest
import torch

import residual_add_rmsnorm_rms_b200 as rn

OPS = ("rms_norm", "fused_add_rms_norm", "fused_add_rms_norm_fp8")
BIG = 1 << 50


def _ru(v, m=256):
    return (v + m - 1) // m * m


def _slot(op, rows, H):
    b = _ru(2 * rows * H)
    if op != "rms_norm":
        b += _ru(2 * rows * H)
    if op == "fused_add_rms_norm_fp8":
        b += _ru(rows * H) + _ru(4 * rows)
    return b


def _auto_rows(op, T, H, scratch, n):
    rows = min(T, max(-(-T // (4 * n)), -(-(8 << 20) // (2 * H))))
    fit = 0
    while _slot(op, fit + 1, H) * n <= scratch and fit < rows:  # brute force, small cases
        fit += 1
    return min(rows, fit)


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("T,H,n", [(8192, 3840, 3), (1000, 512, 2), (5, 16384, 4), (1, 8, 1),
                                   (300, 1004, 8)])
def test_plan_chunks_rule(op, T, H, n):
    p = rn.host_plan_chunks(op, T, H, BIG, n)
    rows = min(T, max(-(-T // (4 * n)), -(-(8 << 20) // (2 * H))))
    chunks = -(-T // rows)
    assert p == {"chunk_rows": rows, "chunks": chunks, "slot_bytes": _slot(op, rows, H),
                 "slots": min(n, chunks)}
    # a requested chunk size, and the exact capacity edge
    want = max(1, rows // 3)
    need = min(n, -(-T // want)) * _slot(op, want, H)
    q = rn.host_plan_chunks(op, T, H, need, n, want)
    assert (q["chunk_rows"], q["slot_bytes"]) == (want, _slot(op, want, H))
    with pytest.raises(rn.RmsNormError) as e:
        rn.host_plan_chunks(op, T, H, need - 1, n, want)
    assert e.value.name == "RN_ERR_CAPACITY"


@pytest.mark.parametrize("op", OPS)
def test_plan_chunks_shrinks_to_scratch(op):
    T, H, n = 4000, 512, 2
    for scratch in (_slot(op, 1, H) * n, _slot(op, 7, H) * n + 100, 3_000_000):
        p = rn.host_plan_chunks(op, T, H, scratch, n)
        assert p["chunk_rows"] == _auto_rows(op, T, H, scratch, n)
        assert p["slots"] * p["slot_bytes"] <= scratch
    with pytest.raises(rn.RmsNormError) as e:
        rn.host_plan_chunks(op, T, H, _slot(op, 1, H) * n - 1, n)
    assert e.value.name == "RN_ERR_CAPACITY"


def test_plan_chunks_errors():
    def status(*a):
        p = rn.RnHostPlan()
        return rn.STATUS[rn.lib.rn_host_plan_chunks(*a, ctypes.byref(p))], p
    assert status(3, 10, 512, BIG, 2, 0)[0] == "RN_ERR_CONFIG"   # SwiGLU has no host form
    assert status(0, 10, 512, BIG, 0, 0)[0] == "RN_ERR_CONFIG"
    assert status(0, 10, 512, BIG, 9, 0)[0] == "RN_ERR_CONFIG"
    assert status(0, -1, 512, BIG, 2, 0)[0] == "RN_ERR_SHAPE"
    assert status(0, 10, 0, BIG, 2, 0)[0] == "RN_ERR_SHAPE"
    assert status(0, 1 << 40, 1 << 20, BIG, 2, 0)[0] == "RN_ERR_SHAPE"
    st, p = status(1, 0, 512, 0, 2, 0)
    assert st == "RN_OK" and (p.chunk_rows, p.chunks, p.slots) == (0, 0, 0)
    assert rn.lib.rn_host_plan_chunks(0, 10, 512, BIG, 2, 0, None) == 1  # RN_ERR_NULL
    # the largest scratch size plans like any ample one (no overflow)
    for op in OPS:
        assert rn.host_plan_chunks(op, 8192, 3840, (1 << 63) - 1, 8) == \
            rn.host_plan_chunks(op, 8192, 3840, BIG, 8)
    assert ctypes.sizeof(rn.RnHostPipeline) == 8 + 8 + 8 + 4 + 4 + 8  # C layout
    assert ctypes.sizeof(rn.RnHostPlan) == 8 * 3 + 4 + 4


@pytest.mark.skipif(torch.cuda.is_available(), reason="host stand-ins must not reach a GPU")
def test_host_entry_refusals():
    T, H = 64, 512
    x = torch.zeros(T, H, dtype=torch.bfloat16)
    r, out = torch.zeros_like(x), torch.zeros_like(x)
    w = torch.ones(H, dtype=torch.bfloat16)
    q = torch.zeros(T, H, dtype=torch.uint8)
    sc = torch.zeros(T)
    arena = torch.zeros(1 << 21, dtype=torch.uint8)
    base = arena.data_ptr()
    aligned = base + (-base) % 256
    streams = (ctypes.c_void_p * 2)(None, None)

    def pipe(scratch=aligned, nbytes=1 << 20, n=2, reserved=0, chunk=16, strm=True):
        d = rn.RnHostPipeline()
        d.scratch, d.scratch_bytes, d.n_streams, d.reserved, d.chunk_rows = \
            scratch, nbytes, n, reserved, chunk
        d.streams = ctypes.cast(streams, ctypes.POINTER(ctypes.c_void_p)) if strm else None
        return d

    def call(op, d, xx=x, rr=r, oo=out, dt_w=w):
        keep = [rn.describe(t) for t in (oo, xx, rr, dt_w, q, sc)]
        o, xd, rd, wd, qd, sd = [ctypes.byref(k[0]) for k in keep]
        ref = None if d is None else ctypes.byref(d)
        if op == "rms_norm":
            st = rn.lib.rn_host_rms_norm(o, xd, wd, 1e-6, -1, ref)
        elif op == "fused_add_rms_norm":
            st = rn.lib.rn_host_fused_add_rms_norm(o, xd, rd, wd, 1e-6, -1, ref)
        else:
            st = rn.lib.rn_host_fused_add_rms_norm_fp8(qd, sd, xd, rd, wd, 1e-6, -1, ref)
        return rn.STATUS[st]

    for op in OPS:
        assert call(op, None) == "RN_ERR_NULL"
        assert call(op, pipe(n=0)) == "RN_ERR_CONFIG"
        assert call(op, pipe(n=9)) == "RN_ERR_CONFIG"
        assert call(op, pipe(reserved=1)) == "RN_ERR_CONFIG"
        assert call(op, pipe(strm=False)) == "RN_ERR_NULL"
        assert call(op, pipe(scratch=None)) == "RN_ERR_NULL"
        assert call(op, pipe(scratch=aligned + 128)) == "RN_ERR_LAYOUT"
        assert call(op, pipe(nbytes=1000)) == "RN_ERR_CAPACITY"
        assert call(op, pipe(chunk=0, nbytes=1000)) == "RN_ERR_CAPACITY"
        # scratch overlapping a host operand or the weight
        xs = arena[aligned - base:aligned - base + 2 * T * H].view(torch.bfloat16).view(T, H)
        assert call(op, pipe(), xx=xs) == "RN_ERR_ALIAS"
        ws = arena[aligned - base:aligned - base + 2 * H].view(torch.bfloat16)
        assert call(op, pipe(), dt_w=ws) == "RN_ERR_ALIAS"
        # operand checks come first, whatever the pipeline
        assert call(op, pipe(n=0), xx=x.float()) == "RN_ERR_DTYPE"
        assert call(op, pipe(n=0), dt_w=w.half()) == "RN_ERR_WEIGHT_DTYPE"
        # T == 0 is a no-op before the scratch is looked at
        e = torch.zeros(0, H, dtype=torch.bfloat16)
        if op != "fused_add_rms_norm_fp8":
            assert call(op, pipe(scratch=None), xx=e, rr=e.clone(), oo=e.clone()) == "RN_OK"
    # host aliasing rules as for the device ops
    assert call("fused_add_rms_norm", pipe(), rr=x) == "RN_ERR_ALIAS"
    assert call("fused_add_rms_norm", pipe(), oo=r) == "RN_ERR_ALIAS"
