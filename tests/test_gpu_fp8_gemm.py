"""GPU parity of the row-wise scaled fp8 GEMM (tcgen05 tensor cores) against
the fp64 oracle, whose dot products are exact.

Tolerance, derived from the arithmetic: every e4m3 x e4m3 product is exact
in fp32 (4-bit significands); the tensor cores accumulate K of them in fp32,
so the accumulated sum is within gamma_K * sum_k |a_k b_k| of the exact sum,
gamma_K = K * 2^-24 (the worst case of any fp32 summation order); the two
scale products add 2 * 2^-24 relative, and the result is rounded once to
bf16 (half an ulp). The test requires, per element,
    |D - y| <= 1 ulp_bf16(|y|) + (K + 2) * 2^-24 * a_scale * b_scale * sum_k |a_k b_k|
with y the oracle's unrounded value, and reports how many elements equal
the correctly rounded value."""
import numpy as np
import pytest
import torch

import oracle
import residual_add_rmsnorm_rms_b200 as rn
import synth
from residual_add_rmsnorm_rms_b200 import torch_ops  # noqa: F401  (registers the ops)
from tests.cmp_util import bits16, codes8, ulp16
from tests.gpu_util import CORES, oracle_run, sample_rows

pytestmark = pytest.mark.gpu

# (N, K) weight shapes of Gemma 4 12B's fp8 linear layers, from the
# weight-shape table of "VLLM_ROCM_USE_AITER=1 slows Gemma 4 on an AMD MI300X"
GEMMA_NK = [(8192, 3840), (9216, 3840), (30720, 3840), (3840, 4096), (3840, 8192), (3840, 15360)]
DEC = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    yield
    assert rn.device_errors() == 0


def _operands(M, N, K, seed, device="cpu"):
    g = torch.Generator(device=device).manual_seed(seed)
    a = (torch.randn(M, K, generator=g, device=device) * 40).clamp_(-448, 448)
    b = (torch.randn(N, K, generator=g, device=device) * 40).clamp_(-448, 448)
    sa = torch.rand(M, generator=g, device=device) * 0.02 + 1e-3
    sb = torch.rand(N, generator=g, device=device) * 0.02 + 1e-3
    return a.to(torch.float8_e4m3fn), b.to(torch.float8_e4m3fn), sa, sb


def _gemm(a, b, sa, sb):
    d = torch.empty(a.shape[0], b.shape[0], dtype=torch.bfloat16, device="cuda")
    rn.fp8_rowwise_gemm(d, a, b, sa, sb)
    torch.cuda.synchronize()
    return d


def _check(d_gpu, a_codes, b_codes, sa, sb, rows=None):
    """d_gpu holds the rows `rows` (or all); returns the fraction equal to RNE(y)."""
    want, y = oracle.fp8_rowwise_gemm(a_codes, b_codes, sa, sb, rows=rows, want_y=True,
                                      threads=CORES)
    A = a_codes if rows is None else a_codes[rows]
    sa_r = sa if rows is None else sa[rows]
    K = A.shape[1]
    absdot = np.abs(DEC[A]) @ np.abs(DEC[b_codes]).T
    bound = (K + 2) * 2.0 ** -24 * absdot * sa_r.astype(np.float64)[:, None] \
        * sb.astype(np.float64)[None, :]
    got = torch.from_numpy(d_gpu.astype(np.int16) if isinstance(d_gpu, np.ndarray) else
                           bits16(d_gpu).view(np.int16)).view(torch.bfloat16).double().numpy()
    ay = np.abs(y)
    ulp = np.where(ay > 0, 2.0 ** (np.floor(np.log2(np.maximum(ay, 1e-300))) - 7), 2.0 ** -133)
    err = np.abs(got - y)
    assert (err <= ulp + bound).all(), float(np.max((err - ulp) / np.maximum(bound, 1e-300)))
    gbits = bits16(d_gpu) if not isinstance(d_gpu, np.ndarray) else d_gpu
    return float(np.mean(ulp16(gbits, want) == 0))


@pytest.mark.parametrize("M,N,K", [(1, 8, 16), (7, 128, 128), (128, 128, 128), (300, 264, 400),
                                   (129, 3840, 4096), (64, 8, 15360)])
def test_gemm_small_shapes_full(M, N, K):
    a, b, sa, sb = _operands(M, N, K, seed=M + N + K)
    d = _gemm(a.cuda(), b.cuda(), sa.cuda(), sb.cuda())
    exact_frac = _check(d, codes8(a), codes8(b), sa.numpy(), sb.numpy())
    print(M, N, K, "correctly rounded fraction", exact_frac)


# Shapes that leave ragged tiles in every configuration: M below, at and
# above the token widths 16/32/64, N not a multiple of 64 or 128.
CONFIG_SHAPES = [(1, 8, 16), (5, 264, 400), (16, 128, 128), (33, 520, 272), (64, 3840, 4096),
                 (130, 200, 144)]


@pytest.mark.parametrize("M,N,K", CONFIG_SHAPES)
@pytest.mark.parametrize("config", list(rn.GEMM_CONFIGS))
def test_gemm_every_config(config, M, N, K):
    """Each tile configuration (token-major, and channel-major D^T tiles)
    forced on shapes that are ragged for it, checked in full."""
    a, b, sa, sb = _operands(M, N, K, seed=7 * M + N + K)
    rn.fp8_gemm_force_config(config)
    try:
        d = _gemm(a.cuda(), b.cuda(), sa.cuda(), sb.cuda())
    finally:
        rn.fp8_gemm_force_config(None)
    exact_frac = _check(d, codes8(a), codes8(b), sa.numpy(), sb.numpy())
    print(config, M, N, K, "correctly rounded fraction", exact_frac)


@pytest.mark.parametrize("N,K", GEMMA_NK)
@pytest.mark.parametrize("M", [1, 16, 33, 64, 256, 8192])
def test_gemm_gemma_shapes(M, N, K):
    a, b, sa, sb = _operands(M, N, K, seed=N + K + M, device="cuda")
    d = _gemm(a, b, sa, sb)
    rows = sample_rows(M, k=32)
    exact_frac = _check(bits16(d)[rows], codes8(a), codes8(b), sa.cpu().numpy(),
                        sb.cpu().numpy(), rows=rows)
    print(M, N, K, "correctly rounded fraction", exact_frac)


def test_norm_then_gemm_chain():
    """The decode chain through the torch ops: fused_add_rms_norm_fp8's codes
    and [T, 1] per-token scales feed fp8_rowwise_gemm directly. The GEMM's
    parity is judged on the oracle's own codes and scales for the same
    synthetic inputs (no GPU output becomes an oracle input); the GPU chain
    must then give the same D on every row whose GPU codes and scale equal
    the oracle's (and both stages are checked against the oracle elsewhere)."""
    wl = synth.make_inputs("prefill", "fused_add_rms_norm_fp8", "bf16", 256, 3840)
    want = oracle_run("fused_add_rms_norm_fp8", wl.x, wl.residual, wl.weight, wl.eps, "bf16")
    _, b, _, sb = _operands(1, 8192, 3840, seed=77)
    b, sb = b.cuda(), sb.cuda()

    q_o = torch.from_numpy(want["q"].reshape(256, 3840)).cuda().view(torch.float8_e4m3fn)
    s_o = torch.from_numpy(want["scale"].astype(np.float32)).cuda().view(256, 1)
    d_o = torch.ops.rmsnorm_b200.fp8_rowwise_gemm(q_o, b, s_o, sb)
    torch.cuda.synchronize()
    assert d_o.shape == (256, 8192) and d_o.dtype == torch.bfloat16
    _check(d_o, want["q"].reshape(256, 3840), codes8(b), want["scale"].astype(np.float32),
           sb.cpu().numpy())

    q, s = torch.ops.rmsnorm_b200.fused_add_rms_norm_fp8(
        wl.x.cuda(), wl.residual.cuda().clone(), wl.weight.cuda(), wl.eps)
    d = torch.ops.rmsnorm_b200.fp8_rowwise_gemm(q, b, s, sb)
    torch.cuda.synchronize()
    same = ((codes8(q) == want["q"].reshape(256, 3840)).all(axis=1)
            & (s.view(-1).cpu().numpy() == want["scale"].astype(np.float32)))
    # scales agree to 1e-6 relative, not always bit for bit: compare the rows
    # whose every code and scale bit match (about 40 % of them)
    assert same.mean() > 0.1
    assert (bits16(d)[same] == bits16(d_o)[same]).all()


def test_gemm_validation():
    a = torch.zeros(4, 32, dtype=torch.float8_e4m3fn, device="cuda")
    b = torch.zeros(16, 32, dtype=torch.float8_e4m3fn, device="cuda")
    sa = torch.ones(4, device="cuda")
    sb = torch.ones(16, device="cuda")
    d = torch.empty(4, 16, dtype=torch.bfloat16, device="cuda")
    rn.fp8_rowwise_gemm(d, a, b, sa, sb)
    torch.cuda.synchronize()
    assert (d.float() == 0).all()
    cases = [
        ((d, a[:, :24], b[:, :24], sa, sb), "RN_ERR_LAYOUT"),       # padded rows
        ((d, torch.zeros(4, 24, dtype=torch.float8_e4m3fn, device="cuda"),
          torch.zeros(16, 24, dtype=torch.float8_e4m3fn, device="cuda"), sa, sb), "RN_ERR_SHAPE"),
        ((torch.empty(4, 12, dtype=torch.bfloat16, device="cuda"), a, b[:12], sa, sb[:12]),
         "RN_ERR_SHAPE"),                                          # N % 8
        ((d, a, b, sa[:3], sb), "RN_ERR_SHAPE"),
        ((d.float(), a, b, sa, sb), "RN_ERR_DTYPE"),
        ((d, a.view(torch.uint8).to(torch.bfloat16), b, sa, sb), "RN_ERR_DTYPE"),
    ]
    for args, name in cases:
        with pytest.raises(rn.RmsNormError) as e:
            rn.fp8_rowwise_gemm(*args)
        assert e.value.name == name, (name, e.value.name)
    empty = torch.empty(0, 32, dtype=torch.float8_e4m3fn, device="cuda")
    rn.fp8_rowwise_gemm(torch.empty(0, 16, dtype=torch.bfloat16, device="cuda"), empty, b,
                        torch.empty(0, device="cuda"), sb)


_CAPTURE_FIRST = r"""
import torch, residual_add_rmsnorm_rms_b200 as rn
torch.cuda.init()
g = torch.Generator(device="cuda").manual_seed(3)
M, N, K = 16, 3840, 4096
a = (torch.randn(M, K, generator=g, device="cuda") * 40).clamp_(-448, 448).to(torch.float8_e4m3fn)
b = (torch.randn(N, K, generator=g, device="cuda") * 40).clamp_(-448, 448).to(torch.float8_e4m3fn)
sa = torch.rand(M, generator=g, device="cuda") * 0.01 + 1e-3
sb = torch.rand(N, generator=g, device="cuda") * 0.01 + 1e-3
d_graph = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
st = torch.cuda.Stream()
graph = torch.cuda.CUDAGraph()
with torch.cuda.stream(st):
    with torch.cuda.graph(graph, stream=st):  # the process's first GEMM call
        rn.fp8_rowwise_gemm(d_graph, a, b, sa, sb)
graph.replay()
torch.cuda.synchronize()
d = torch.empty_like(d_graph)
rn.fp8_rowwise_gemm(d, a, b, sa, sb)
torch.cuda.synchronize()
assert torch.equal(d.view(torch.int16), d_graph.view(torch.int16))
assert rn.device_errors() == 0
print("ok")
"""


def test_gemm_first_call_inside_graph_capture():
    """A process whose first GEMM call is recorded into a CUDA graph (the
    kernel's shared-memory limit is then set during the capture) replays it
    to the same bits as an eager call."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", _CAPTURE_FIRST], cwd=root, capture_output=True,
                         text=True, timeout=300, env=dict(os.environ, PYTHONPATH=root))
    assert out.returncode == 0 and out.stdout.strip().endswith("ok"), out.stderr[-2000:]
