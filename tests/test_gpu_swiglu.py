"""GPU parity of the fused SwiGLU + per-token FP8 cast (silu_and_mul_fp8)
against the fp64 oracle.

Tolerance (the pages state none for this kernel; derived from the
arithmetic): silu(g) = g / (1 + e^-g) with e^-g = 2^p, p = -g log2(e)
carried in two floats (the exact rounding error of the product by an fma
plus the low part of log2(e)), so the multi-function unit's base-2
exponential (a few ulp) and one fma rounding are its only errors whatever
|g|; 1 + e^-g rounds once (half an ulp), the fast division adds at most 2
ulp, the up product half an ulp: y is within about 6 ulp (3.6e-7) of the
exact value, and the scale max|y| / 448 (one more rounding) within 1e-6
relative, the per-token scale tolerance of the norm's fp8 op, for any gate.
The heavy-tailed test feeds gates up to 1e3 in magnitude and rows whose
maximum comes from gates between -80 and -5, where an exponential whose
argument were rounded to one float would be off by up to ~100 ulp. e4m3
codes: distance <= 1 everywhere, non-zero on at most 0.1 % of elements (as
for the norm's fp8 op)."""
import numpy as np
import pytest
import torch

import oracle
import residual_add_rmsnorm_rms_b200 as rn
import synth
from residual_add_rmsnorm_rms_b200 import torch_ops  # noqa: F401  (registers the ops)
from tests.cmp_util import bits16, code_dist8, codes8
from tests.gpu_util import CORES, sample_rows

pytestmark = pytest.mark.gpu
SCALE_RTOL = 1e-6


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    rn.force_plan(0, 0)
    yield
    rn.force_plan(0, 0)
    assert rn.device_errors() == 0


def _gpu(x):
    T, I = x.shape[0], x.shape[1] // 2
    q = torch.empty(T, I, dtype=torch.float8_e4m3fn, device="cuda")
    s = torch.empty(T, dtype=torch.float32, device="cuda")
    rn.silu_and_mul_fp8(q, s, x)
    torch.cuda.synchronize()
    return q, s


def _check(x_host, q, s, dtype, rows=None):
    want_q, want_s = oracle.silu_and_mul_fp8(bits16(x_host), dtype, threads=CORES)
    gq, gs = codes8(q), s.cpu().numpy()
    if rows is not None:
        gq, gs = gq[rows], gs[rows]
    assert not ((gq & 0x7F) == 0x7F).any()
    d = code_dist8(gq, want_q)
    assert d.max() <= 1, d.max()
    frac = np.count_nonzero(d) / d.size
    assert frac <= 1e-3, frac
    err = np.abs(gs.astype(np.float64) - want_s) / np.where(want_s == 0, 1, want_s)
    assert err.max() <= SCALE_RTOL, err.max()
    return frac, err.max()


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("T", synth.SWIGLU_T)
def test_swiglu_workload(T, dtype):
    """x = [gate | up], I = 15360, gate, up ~ N(0,1); the 8192-row case on
    GPU-drawn inputs with a row sample."""
    if T <= 256:
        wl = synth.make_inputs("swiglu", "silu_and_mul_fp8", dtype, T, synth.SWIGLU_I)
        q, s = _gpu(wl.x.cuda())
        print(_check(wl.x, q, s, dtype))
    else:
        wl = synth.make_inputs("swiglu", "silu_and_mul_fp8", dtype, T, synth.SWIGLU_I,
                               device="cuda")
        rows = sample_rows(T)
        q, s = _gpu(wl.x)
        xs = wl.x.index_select(0, torch.from_numpy(rows).cuda()).cpu()
        print(_check(xs, q, s, dtype, rows=rows))


def test_swiglu_more_than_2_31_elements():
    """x of [69632 x 2 * 16384] bf16 (2.3e9 elements; row 65536 starts at
    element 2^31): a row sample including the rows around that element and
    the last row."""
    T, I = 69632, 16384
    wl = synth.make_inputs("swiglu", "silu_and_mul_fp8", "bf16", T, I, device="cuda")
    edge = (1 << 31) // (2 * I)
    rows = np.unique(np.concatenate([sample_rows(T, k=64), [edge - 1, edge, edge + 1, T - 1]]))
    q, s = _gpu(wl.x)
    xs = wl.x.index_select(0, torch.from_numpy(rows).cuda()).cpu()
    print(_check(xs, q, s, "bf16", rows=rows))
    del wl, q, s
    torch.cuda.empty_cache()


@pytest.mark.parametrize("I", [8, 1000, 1004, 4096, 15360, 40000])
def test_swiglu_shapes_and_scalar_path(I):
    """Ragged I (scalar kernel), narrow and wide rows."""
    g = torch.Generator().manual_seed(I)
    x = synth.normal((7, 2 * I), 1.0, g, "cpu").bfloat16()
    q, s = _gpu(x.cuda())
    _check(x, q, s, "bf16")


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_swiglu_heavy_tailed_and_large_gates(dtype):
    """Gates ~ 10 x Student-t(3) clipped to +-1e3, ups ~ N(0,1) with 1 % of
    the columns x50; in the first 16 rows every gate lies in [-80, -5] (the
    row maximum then comes from a negative gate, where e^-g is large)."""
    g = torch.Generator().manual_seed(21)
    T, I = 64, 4096
    gate = synth.student_t3((T, I), 100.0, g, "cpu") * 10
    up = synth.normal((T, I), 1.0, g, "cpu")
    up[:, synth.outlier_columns(I, 0.01, g, "cpu")] *= 50
    gate[:16] = -(torch.rand(16, I, generator=g) * 75 + 5)
    up[:16] = torch.rand(16, I, generator=g) + 0.5
    x = torch.cat([gate, up], 1).to(synth.to_dtype(dtype))
    q, s = _gpu(x.cuda())
    frac, err = _check(x, q, s, dtype)
    print(dtype, "code mismatch fraction", frac, "max scale rel err", err)


def test_swiglu_zero_and_extreme_rows():
    I = 1024
    x = torch.zeros(4, 2 * I)
    x[1, :I] = -60.0      # silu underflows towards 0 (y tiny but non-zero)
    x[1, I:] = 1.0
    x[2, :I] = 30.0       # silu(a) ~ a
    x[2, I:] = torch.linspace(-2, 2, I)
    x[3] = torch.randn(2 * I, generator=torch.Generator().manual_seed(3)) * 3
    xb = x.bfloat16()
    q, s = _gpu(xb.cuda())
    assert s[0].item() == 0 and (q[0].view(torch.uint8) == 0).all()
    _check(xb[2:], q[2:], s[2:], "bf16")


def test_swiglu_torch_op_and_forced_shapes():
    g = torch.Generator().manual_seed(11)
    x = synth.normal((3, 5, 2 * 4096), 1.0, g, "cpu").bfloat16()
    q, s = torch.ops.rmsnorm_b200.silu_and_mul_fp8(x.cuda())
    torch.cuda.synchronize()
    assert q.shape == (3, 5, 4096) and s.shape == (3, 5, 1)
    _check(x.reshape(15, -1), q.reshape(15, -1), s.reshape(15), "bf16")
    for tpr, vpt in [(128, 4), (64, 8), (512, 1), (32, 16)]:
        rn.force_plan(tpr, vpt)
        q2, s2 = _gpu(x.reshape(15, -1).cuda())
        _check(x.reshape(15, -1), q2, s2, "bf16")
    rn.force_plan(0, 0)


def test_swiglu_validation():
    x = torch.zeros(4, 2 * 64, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(4, 64, dtype=torch.float8_e4m3fn, device="cuda")
    s = torch.empty(4, dtype=torch.float32, device="cuda")
    with pytest.raises(rn.RmsNormError) as e:
        rn.silu_and_mul_fp8(q, s, torch.zeros(4, 127, dtype=torch.bfloat16, device="cuda"))
    assert e.value.name == "RN_ERR_SHAPE"
    with pytest.raises(rn.RmsNormError) as e:
        rn.silu_and_mul_fp8(torch.empty(4, 65, dtype=torch.float8_e4m3fn, device="cuda"), s, x)
    assert e.value.name == "RN_ERR_SHAPE"
    with pytest.raises(rn.RmsNormError) as e:
        rn.silu_and_mul_fp8(q, s, x.float())
    assert e.value.name == "RN_ERR_DTYPE"
    q_in_x = x.view(torch.uint8).view(-1)[: 4 * 64].view(4, 64)  # dense, inside x
    with pytest.raises(rn.RmsNormError) as e:
        rn.silu_and_mul_fp8(q_in_x, s, x)
    assert e.value.name == "RN_ERR_ALIAS"
    with pytest.raises(rn.RmsNormError) as e:
        rn.silu_and_mul_fp8(x.view(torch.uint8)[:, :64], s, x)  # padded rows
    assert e.value.name == "RN_ERR_LAYOUT"
