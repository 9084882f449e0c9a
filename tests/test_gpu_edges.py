"""GPU edge cases and kernel-variant coverage, each against the CPU oracle.

Ragged hidden sizes (scalar kernel), idle vector slots, every compiled
vectors-per-thread width and threads-per-row shape (forced), misaligned bases,
rows aligned for 16-byte but not 32-byte accesses,
T == 0, tensors of more than 2^31 elements, in-place out == x, no weight,
N-D views, zero rows, fp16 subnormal
inputs, determinism, the structural identity fused(x, r).out ==
rms_norm(r'), non-default streams and validation errors on real tensors.
"""
import numpy as np
import pytest
import torch

import synth
import residual_add_rmsnorm_rms_b200 as rn
from tests.cmp_util import bits16
from tests.gpu_util import compare, gpu_run, oracle_run, sample_rows

pytestmark = pytest.mark.gpu
OPS = ["rms_norm", "fused_add_rms_norm", "fused_add_rms_norm_fp8"]


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    rn.force_plan(0, 0)
    rn.force_staged(0, 0, 0)
    yield
    rn.force_plan(0, 0)
    rn.force_staged(0, 0, 0)
    assert rn.device_errors() == 0, "a kernel recorded a device-side error"


def _inputs(T, H, dtype, seed, var_r=4.0):
    g = torch.Generator().manual_seed(seed)
    dt = synth.to_dtype(dtype)
    x = synth.normal((T, H), 1.0, g, "cpu").to(dt)
    r = synth.normal((T, H), var_r, g, "cpu").to(dt)
    w = synth.weight(H, dt, g, "cpu")
    return x, r, w


def _check(op, x, r, w, eps, dtype, expect_kernel=None):
    if expect_kernel is not None:
        T = x.numel() // x.shape[-1]
        plan = rn.plan_launch(op, x.dtype, T, x.shape[-1])
        assert plan["kernel"] == expect_kernel, plan
    got = gpu_run(op, x.cuda(), None if r is None else r.cuda().clone(),
                  None if w is None else w.cuda(), eps)
    torch.cuda.synchronize()
    want = oracle_run(op, x, r, w, eps, dtype)
    return compare(op, got, want, dtype)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("H", [1, 7, 100, 1004, 4100])
def test_ragged_hidden_sizes_scalar_kernel(op, dtype, H):
    for T in (1, 5, 33):
        x, r, w = _inputs(T, H, dtype, seed=H * 7 + T)
        _check(op, x, r, w, 1e-6, dtype, expect_kernel=1)


@pytest.mark.parametrize("op", OPS)
def test_large_hidden_sizes(op):
    for H in (32768, 40000, 131072 + 8):
        x, r, w = _inputs(3, H, "bf16", seed=H)
        _check(op, x, r, w, 1e-6, "bf16")


# More than 2^31 elements per tensor: element indices and byte offsets past
# 32 bits. 4.6 GB per 16-bit tensor.
BIG_T = 139264


@pytest.mark.parametrize("H", [16384, 16383], ids=["vector", "scalar"])
@pytest.mark.parametrize("op", OPS)
def test_more_than_2_31_elements(op, H):
    """The automatic plan on [139264 x H] bf16 (H = 16383 takes the scalar
    kernel); the oracle checks a row sample that includes the rows around
    element 2^31 and the last rows."""
    wl = synth.make_inputs("sweep", op, "bf16", BIG_T, H, device="cuda")
    edge = (1 << 31) // H
    rows = np.unique(np.concatenate([sample_rows(BIG_T, k=64),
                                     [edge - 1, edge, edge + 1, BIG_T - 2, BIG_T - 1]]))
    ridx = torch.from_numpy(rows).cuda()
    x_s = wl.x.index_select(0, ridx).cpu()
    r_s = None if wl.residual is None else wl.residual.index_select(0, ridx).cpu()
    got = gpu_run(op, wl.x, wl.residual, wl.weight, wl.eps)
    got = {k: (v.index_select(0, ridx) if v.dim() and v.shape[0] == BIG_T else v)
           for k, v in got.items()}
    torch.cuda.synchronize()
    want = oracle_run(op, x_s, r_s, wl.weight.cpu(), wl.eps, "bf16")
    compare(op, got, want, "bf16")
    del wl, got
    torch.cuda.empty_cache()


def _tpr_for(nvec, vpt):
    need = -(-nvec // vpt)
    if need <= 32:
        t = 1
        while t < need:
            t <<= 1
        return t
    return -(-need // 32) * 32


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("op", OPS)
def test_every_compiled_width_forced(op, dtype):
    """Each vectors-per-thread width at H = 4096 (and its natural
    threads-per-row), with T = 37 so the last CTA holds a partial set of rows."""
    H, T = 4096, 37
    x, r, w = _inputs(T, H, dtype, seed=11)
    for vpt in rn.supported_vectors_per_thread():
        tpr = _tpr_for(H // 8, vpt)
        if tpr > (1024 if vpt <= 4 else 512 if vpt <= 8 else 256):
            continue
        rn.force_plan(tpr, vpt)
        p = rn.plan_launch(op, x.dtype, T, H)
        assert p["kernel"] == 0 and p["vectors_per_thread"] == vpt
        _check(op, x, r, w, 1e-5, dtype)
    rn.force_plan(0, 0)


@pytest.mark.parametrize("op", OPS)
def test_sub_warp_and_idle_slot_shapes(op):
    """Rows narrower than a warp (several rows per warp), and shapes that
    leave idle vector slots (H = 3840 on 64 x 8 = 512 slots for 480 vectors)."""
    cases = [(512, 4, 16), (512, 8, 8), (512, 16, 4), (512, 32, 2), (512, 64, 1),
             (3840, 64, 8), (3840, 32, 15), (3840, 96, 5), (3840, 160, 3), (3840, 480, 1),
             (2048 + 8, 32, 10), (8, 1, 1)]
    for H, tpr, vpt in cases:
        rn.force_plan(tpr, vpt)
        for T in (1, 3, 67):
            x, r, w = _inputs(T, H, "bf16", seed=H + tpr + T)
            _check(op, x, r, w, 1e-6, "bf16", expect_kernel=0)
    rn.force_plan(0, 0)


STAGED_SHAPES = [  # (H, ctas per SM, stages, threads, T)
    (3840, 4, 3, 256, 1000), (3840, 1, 2, 96, 7), (4096, 2, 6, 256, 333), (512, 4, 8, 64, 777),
    (16384, 1, 2, 1024, 150), (2048, 4, 5, 32, 1), (7168, 2, 3, 448, 300), (8, 4, 4, 32, 50),
    (5120, 2, 5, 320, 597),
]


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("op", OPS)
def test_staged_kernel_forced_shapes(op, dtype):
    """The shared-memory-ring kernel on rings of 2..8 stages, 1..4 CTAs per SM,
    threads from 1 to 5 vectors per pass, and row counts that leave CTAs with
    unequal numbers of rows."""
    for H, c, S, thr, T in STAGED_SHAPES:
        rn.force_staged(c, S, thr)
        x, r, w = _inputs(T, H, dtype, seed=H + S + T)
        _check(op, x, r, w, 1e-6, dtype, expect_kernel=2)
        _check(op, x, r, None, 1e-6, dtype, expect_kernel=2)
    rn.force_staged(0, 0, 0)


@pytest.mark.parametrize("op", ["rms_norm", "fused_add_rms_norm"])
def test_staged_in_place_out_is_x(op):
    rn.force_staged(2, 4, 128)
    T, H = 500, 2048
    x, r, w = _inputs(T, H, "bf16", seed=21)
    xd, rd = x.cuda().clone(), r.cuda().clone()
    if op == "rms_norm":
        rn.rms_norm(xd, xd, w.cuda(), 1e-6)
        got = {"out": xd}
    else:
        rn.fused_add_rms_norm(xd, xd, rd, w.cuda(), 1e-6)
        got = {"out": xd, "residual": rd}
    torch.cuda.synchronize()
    compare(op, got, oracle_run(op, x, r, w, 1e-6, "bf16"), "bf16")


@pytest.mark.parametrize("op", OPS)
def test_misaligned_base_uses_scalar_kernel(op):
    T, H = 9, 4096
    x, r, w = _inputs(T, H, "bf16", seed=5)
    xb = torch.empty(T * H + 1, dtype=torch.bfloat16, device="cuda")
    xm = xb[1:].view(T, H)
    xm.copy_(x.cuda())
    st, plan = rn.validate(op, torch.empty(T, H, dtype=torch.bfloat16) if op != "fused_add_rms_norm_fp8"
                           else torch.empty(T, H, dtype=torch.uint8),
                           xm, None if op == "rms_norm" else r.cuda(), w.cuda(),
                           scale=torch.empty(T, dtype=torch.float32, device="cuda"))
    got = gpu_run(op, xm, None if r is None else r.cuda().clone(), w.cuda(), 1e-6)
    torch.cuda.synchronize()
    want = oracle_run(op, x, r, w, 1e-6, "bf16")
    compare(op, got, want, "bf16")


def _offset_view(t, elems):
    """A copy of `t` on the device whose data starts `elems` elements past a
    fresh allocation (which is at least 256-byte aligned)."""
    buf = torch.empty(t.numel() + elems, dtype=t.dtype, device="cuda")
    v = buf[elems:].view(t.shape)
    v.copy_(t.cuda() if not t.is_cuda else t)
    return v


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("offset", [8, 16])
def test_16_byte_but_not_32_byte_aligned_rows(op, offset):
    """Rows 16-byte but not 32-byte aligned (offset 8 elements: x, residual,
    out; offset 16 keeps them 32-byte aligned) with an even vector count per
    thread: the vector kernel with single 16-byte accesses, or with 32-byte
    pairs, both checked in full against the oracle."""
    T, H = 67, 3840
    x, r, w = _inputs(T, H, "bf16", seed=31 + offset)
    assert rn.plan_launch(op, torch.bfloat16, T, H)["vectors_per_thread"] % 2 == 0
    xs = _offset_view(x, offset)
    rs = None if op == "rms_norm" else _offset_view(r, offset)
    out = None
    if op != "fused_add_rms_norm_fp8":
        out = _offset_view(torch.zeros(T, H, dtype=torch.bfloat16), offset)
    got = gpu_run(op, xs, rs, w.cuda(), 1e-6, out=out)
    torch.cuda.synchronize()
    compare(op, got, oracle_run(op, x, r, w, 1e-6, "bf16"), "bf16")


@pytest.mark.parametrize("op", ["fused_add_rms_norm_fp8"])
def test_fp8_codes_8_byte_aligned(op):
    """Codes 8-byte but not 16-byte aligned: the fp8 op stores them 8 bytes
    at a time even when x and the residual allow 32-byte pairs."""
    T, H = 40, 4096
    x, r, w = _inputs(T, H, "bf16", seed=41)
    qb = torch.empty(T * H + 8, dtype=torch.float8_e4m3fn, device="cuda")
    q = qb[8:].view(T, H)
    scale = torch.empty(T, dtype=torch.float32, device="cuda")
    rr = r.cuda().clone()
    rn.fused_add_rms_norm_fp8(q, scale, x.cuda(), rr, w.cuda(), 1e-6)
    torch.cuda.synchronize()
    compare(op, {"q": q, "scale": scale, "residual": rr}, oracle_run(op, x, r, w, 1e-6, "bf16"),
            "bf16")


@pytest.mark.parametrize("op", OPS)
def test_empty_batch_is_a_noop(op):
    x = torch.empty(0, 4096, dtype=torch.bfloat16, device="cuda")
    r = torch.empty_like(x)
    gpu_run(op, x, r, None, 1e-6)
    torch.cuda.synchronize()


@pytest.mark.parametrize("op", ["rms_norm", "fused_add_rms_norm"])
def test_in_place_out_is_x(op):
    T, H = 64, 3840
    x, r, w = _inputs(T, H, "bf16", seed=9)
    xd = x.cuda().clone()
    rd = r.cuda().clone()
    if op == "rms_norm":
        rn.rms_norm(xd, xd, w.cuda(), 1e-6)
        got = {"out": xd}
    else:
        rn.fused_add_rms_norm(xd, xd, rd, w.cuda(), 1e-6)
        got = {"out": xd, "residual": rd}
    torch.cuda.synchronize()
    compare(op, got, oracle_run(op, x, r, w, 1e-6, "bf16"), "bf16")


@pytest.mark.parametrize("op", OPS)
def test_no_weight_and_nd_views(op):
    T, H = 24, 2048
    x, r, w = _inputs(T, H, "fp16", seed=3)
    _check(op, x, r, None, 1e-6, "fp16")
    # a 3-D view flattens for free and gives the 2-D result
    x3, r3 = x.view(4, 6, H), r.view(4, 6, H)
    got = gpu_run(op, x3.cuda(), r3.cuda().clone(), w.cuda(), 1e-6)
    torch.cuda.synchronize()
    compare(op, {k: v.reshape(T, -1) if v.dim() > 1 else v for k, v in got.items()},
            oracle_run(op, x, r, w, 1e-6, "fp16"), "fp16")


def test_zero_rows_and_fp16_subnormals():
    T, H = 6, 1024
    x = torch.zeros(T, H, dtype=torch.float16)
    r = torch.zeros(T, H, dtype=torch.float16)
    # rows 3..5: fp16 subnormal inputs (|v| < 2^-14), normalised with eps = 0
    g = torch.Generator().manual_seed(1)
    x[3:] = (torch.randn(3, H, generator=g) * 2e-6).half()
    r[3:] = (torch.randn(3, H, generator=g) * 2e-6).half()
    assert (x[3:].abs() < 2 ** -14).all()
    for op in OPS:
        got = gpu_run(op, x.cuda(), r.cuda().clone(), None, 0.0 if op != "rms_norm" else 1e-30)
        torch.cuda.synchronize()
        want = oracle_run(op, x, r, None, 0.0 if op != "rms_norm" else 1e-30, "fp16")
        if op == "fused_add_rms_norm_fp8":
            assert (want["scale"][:3] == 0).all() and (want["q"][:3] == 0).all()
            # rows 0..2 are all zero: scale 0, codes 0 (eps = 0 would make y NaN there)
            assert (got["scale"][:3].cpu() == 0).all()
            assert (got["q"][:3].view(torch.uint8).cpu() == 0).all()
            got = {k: v[3:] for k, v in got.items()}
            want = {k: v[3:] for k, v in want.items()}
            compare(op, got, want, "fp16")
        elif op == "rms_norm":
            compare(op, got, want, "fp16")
        else:
            got = {k: v[3:] for k, v in got.items()}
            want = {k: v[3:] for k, v in want.items()}
            compare(op, got, want, "fp16")


@pytest.mark.parametrize("op", OPS)
def test_deterministic(op):
    wl = synth.make_inputs("prefill", op, "bf16", 1024, 3840)
    outs = []
    for _ in range(2):
        r = None if wl.residual is None else wl.residual.cuda().clone()
        got = gpu_run(op, wl.x.cuda(), r, wl.weight.cuda(), wl.eps)
        torch.cuda.synchronize()
        outs.append({k: bits16(v) if v.dtype in (torch.bfloat16, torch.float16)
                     else v.view(torch.uint8).cpu().numpy() if v.dtype == torch.float8_e4m3fn
                     else v.cpu().numpy() for k, v in got.items()})
    for k in outs[0]:
        assert np.array_equal(outs[0][k], outs[1][k]), k


def test_fused_equals_rms_norm_of_written_back_residual_on_gpu():
    for dtype in ("bf16", "fp16"):
        wl = synth.make_inputs("decode", "fused_add_rms_norm", dtype, 256, 4096)
        x, r, w = wl.x.cuda(), wl.residual.cuda().clone(), wl.weight.cuda()
        out = torch.empty_like(x)
        rn.fused_add_rms_norm(out, x, r, w, wl.eps)
        out2 = torch.empty_like(x)
        rn.rms_norm(out2, r, w, wl.eps)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


def test_bf16_rms_norm_equals_fused_on_subnormals_and_extremes():
    """bf16 rms_norm squares and weights its inputs with the mixed-precision
    fma (16-bit operands, fp32 result); the fused op widens them first.
    rms_norm of the written-back residual must equal the fused op's output
    bit for bit, here on rows mixing normal values, bf16 subnormals and
    values near 1e15 (squares stay inside fp32, the supported range), with and
    without a weight. (With x = 0 the written-back residual is r itself
    except that -0 becomes +0.)"""
    g = torch.Generator().manual_seed(17)
    T, H = 64, 4096
    r = torch.randn(T, H, generator=g)
    sub = torch.rand(T, H, generator=g) < 0.1
    r[sub] = torch.randn(int(sub.sum()), generator=g) * 1e-39   # bf16 subnormals
    big = torch.rand(T, H, generator=g) < 0.01
    r[big] = torch.randn(int(big.sum()), generator=g) * 1e15
    r[7] = torch.randn(H, generator=g) * 1e-39                   # a row of subnormals only
    r = r.bfloat16()
    assert ((r.abs() < 2 ** -126) & (r != 0)).sum() > 1000
    w = synth.weight(H, torch.bfloat16, g, "cpu")
    for weight in (w, None):
        x = torch.zeros(T, H, dtype=torch.bfloat16, device="cuda")
        rr = r.cuda().clone()
        out = torch.empty_like(x)
        rn.fused_add_rms_norm(out, x, rr, None if weight is None else weight.cuda(), 1e-30)
        out2 = torch.empty_like(x)
        rn.rms_norm(out2, rr, None if weight is None else weight.cuda(), 1e-30)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
        want = oracle_run("fused_add_rms_norm", x.cpu(), r, weight, 1e-30, "bf16")
        compare("fused_add_rms_norm", {"out": out, "residual": rr}, want, "bf16")
        compare("rms_norm", {"out": out2},
                oracle_run("rms_norm", rr.cpu(), None, weight, 1e-30, "bf16"), "bf16")


def test_non_default_stream():
    wl = synth.make_inputs("decode", "fused_add_rms_norm", "bf16", 64, 4096)
    s = torch.cuda.Stream()
    x, r, w = wl.x.cuda(), wl.residual.cuda().clone(), wl.weight.cuda()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        out = torch.empty_like(x)
        rn.fused_add_rms_norm(out, x, r, w, wl.eps)
    s.synchronize()
    compare("fused_add_rms_norm", {"out": out, "residual": r},
            oracle_run("fused_add_rms_norm", wl.x, wl.residual, wl.weight, wl.eps, "bf16"), "bf16")


def test_errors_on_real_tensors_launch_nothing():
    x = torch.randn(4, 256, device="cuda").bfloat16()
    r = torch.randn(4, 256, device="cuda").bfloat16()
    r0 = r.clone()
    with pytest.raises(rn.RmsNormError) as e:
        rn.fused_add_rms_norm(torch.empty_like(x), x, x, None, 1e-6)
    assert e.value.name == "RN_ERR_ALIAS"
    with pytest.raises(rn.RmsNormError) as e:
        rn.fused_add_rms_norm(torch.empty_like(x), x, r, None, 1e-6, variance_size=128)
    assert e.value.name == "RN_ERR_VARIANCE_SIZE"
    with pytest.raises(rn.RmsNormError) as e:
        rn.rms_norm(torch.empty_like(x), x.t(), None, 1e-6)
    assert e.value.name in ("RN_ERR_LAYOUT", "RN_ERR_SHAPE")
    with pytest.raises(rn.RmsNormError) as e:
        rn.fused_add_rms_norm(torch.empty_like(x), x, r, x[0].half(), 1e-6)
    assert e.value.name == "RN_ERR_WEIGHT_DTYPE"
    torch.cuda.synchronize()
    assert torch.equal(r, r0)  # nothing ran


def test_loaded_device_code_is_sm100a():
    """The device code the library loaded was compiled for compute
    capability 10.0 (sm_100a is the only target the build emits)."""
    assert rn.kernel_binary_version() == 100
