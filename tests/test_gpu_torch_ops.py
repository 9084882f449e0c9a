"""torch custom ops on the GPU: same bits as the direct C-ABI calls and the
oracle on N-D inputs, opcheck of schemas and fake implementations, and a
torch.compile trace (aot_eager, fullgraph) through the mutating ops."""
import pytest
import torch

import residual_add_rmsnorm_rms_b200 as rn
import synth
from residual_add_rmsnorm_rms_b200 import torch_ops as ops
from tests.gpu_util import compare, oracle_run

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    rn.force_plan(0, 0)
    yield
    assert rn.device_errors() == 0


def _inputs(shape, dtype="bf16", seed=0):
    g = torch.Generator().manual_seed(seed)
    dt = synth.to_dtype(dtype)
    x = synth.normal(shape, 1.0, g, "cpu").to(dt)
    r = synth.normal(shape, 4.0, g, "cpu").to(dt)
    w = synth.weight(shape[-1], dt, g, "cpu")
    return x, r, w


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_ops_match_oracle_on_nd_inputs(dtype):
    shape = (3, 5, 2048)
    x, r, w = _inputs(shape, dtype, 1)
    T = 15
    # rms_norm
    out = ops.rms_norm(x.cuda(), w.cuda(), 1e-6)
    torch.cuda.synchronize()
    compare("rms_norm", {"out": out.reshape(T, -1)},
            oracle_run("rms_norm", x.reshape(T, -1), None, w, 1e-6, dtype), dtype)
    # fused, in place on x
    xd, rd = x.cuda().clone(), r.cuda().clone()
    assert ops.fused_add_rms_norm(xd, rd, w.cuda(), 1e-6) is None
    torch.cuda.synchronize()
    compare("fused_add_rms_norm", {"out": xd.reshape(T, -1), "residual": rd.reshape(T, -1)},
            oracle_run("fused_add_rms_norm", x.reshape(T, -1), r.reshape(T, -1), w, 1e-6, dtype),
            dtype)
    # fp8
    rd = r.cuda().clone()
    q, s = ops.fused_add_rms_norm_fp8(x.cuda(), rd, w.cuda(), 1e-6)
    torch.cuda.synchronize()
    assert q.shape == shape and s.shape == (3, 5, 1)
    compare("fused_add_rms_norm_fp8",
            {"q": q.reshape(T, -1), "scale": s.reshape(T), "residual": rd.reshape(T, -1)},
            oracle_run("fused_add_rms_norm_fp8", x.reshape(T, -1), r.reshape(T, -1), w, 1e-6,
                       dtype), dtype)


def test_ops_equal_direct_calls_bitwise():
    x, r, w = _inputs((64, 3840), "bf16", 2)
    x, r, w = x.cuda(), r.cuda(), w.cuda()
    out_a = ops.rms_norm(x, w, 1e-6)
    out_b = torch.empty_like(x)
    rn.rms_norm(out_b, x, w, 1e-6)
    xa, ra = x.clone(), r.clone()
    ops.fused_add_rms_norm(xa, ra, w, 1e-6)
    ob, rb = torch.empty_like(x), r.clone()
    rn.fused_add_rms_norm(ob, x, rb, w, 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
    assert torch.equal(xa.view(torch.int16), ob.view(torch.int16))
    assert torch.equal(ra.view(torch.int16), rb.view(torch.int16))


def test_opcheck_schema_and_fake():
    x, r, w = _inputs((8, 1024), "bf16", 3)
    x, r, w = x.cuda(), r.cuda(), w.cuda()
    utils = ("test_schema", "test_faketensor")
    torch.library.opcheck(torch.ops.rmsnorm_b200.rms_norm.default, (x, w, 1e-6), test_utils=utils)
    torch.library.opcheck(torch.ops.rmsnorm_b200.fused_add_rms_norm.default,
                          (x.clone(), r.clone(), w, 1e-6), test_utils=utils)
    torch.library.opcheck(torch.ops.rmsnorm_b200.fused_add_rms_norm_fp8.default,
                          (x, r.clone(), w, 1e-6), test_utils=utils)


def test_torch_compile_traces_through_the_ops():
    x, r, w = _inputs((32, 4096), "bf16", 4)
    x, r, w = x.cuda(), r.cuda(), w.cuda()

    def layer(x, r, w):
        torch.ops.rmsnorm_b200.fused_add_rms_norm(x, r, w, 1e-6)
        return torch.ops.rmsnorm_b200.fused_add_rms_norm_fp8(x, r, w, 1e-6)

    compiled = torch.compile(layer, backend="aot_eager", fullgraph=True)
    xe, re_ = x.clone(), r.clone()
    qe, se = layer(xe, re_, w)
    xc, rc = x.clone(), r.clone()
    qc, sc = compiled(xc, rc, w)
    torch.cuda.synchronize()
    assert torch.equal(xe.view(torch.int16), xc.view(torch.int16))
    assert torch.equal(re_.view(torch.int16), rc.view(torch.int16))
    assert torch.equal(qe.view(torch.uint8), qc.view(torch.uint8))
    assert torch.equal(se, sc)
