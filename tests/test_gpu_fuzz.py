"""Seeded random shapes and layouts against the oracle: T from 1 to 400, H
from 1 to 9000 (multiples of 8 on the vector kernels, any H on the scalar
one), bf16 and fp16, with and without weight, rows scaled by powers of two
over a wide range, bases offset by one element (the scalar kernel) or by 16
bytes (16- but not 32-byte aligned rows), and out == x in place. Each case
meets the oracle tolerances (residual bit-exact, outputs within 1 ulp, codes
within 1, scales within 1e-6); the fraction of e4m3 codes that differ is
bounded over all the fp8 cases together (<= 0.1 %), as for one workload.
The fused SwiGLU + FP8 op gets the same treatment on random [T x 2I] rows,
and the fp8 GEMM on random M x N x K with its automatic tile choice."""
import numpy as np
import pytest
import torch

import residual_add_rmsnorm_rms_b200 as rn
import synth
from tests.cmp_util import bits16, code_dist8, codes8
from tests.gpu_util import FP8_MAX_MISMATCH_FRAC, SCALE_RTOL, compare, oracle_run

pytestmark = pytest.mark.gpu
CASES = 60


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    rn.force_plan(0, 0)
    yield
    assert rn.device_errors() == 0


def _case(rng):
    T = int(rng.integers(1, 401))
    if rng.random() < 0.7:
        H = 8 * int(rng.integers(1, 1126))
    else:
        H = int(rng.integers(1, 5001))
    dtype = "bf16" if rng.random() < 0.6 else "fp16"
    with_w = rng.random() < 0.8
    offset = int(rng.choice([0, 0, 0, 1, 8]))  # elements: none, 2 bytes, 16 bytes
    return T, H, dtype, with_w, offset


def _tensor(host, offset):
    """`host` [T, H] on the GPU at `offset` elements into a larger buffer."""
    flat = torch.empty(host.numel() + offset + 8, dtype=host.dtype, device="cuda")
    view = flat[offset:offset + host.numel()].view(host.shape)
    view.copy_(host.cuda())
    return view


def _inputs(T, H, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    dt = synth.to_dtype(dtype)
    # per-row powers of two: rows from 2^-12 to 2^12 times N(0, 1) (fp16: 2^-6..2^6)
    span = 12 if dtype == "bf16" else 6
    k = torch.randint(-span, span + 1, (T, 1), generator=g).double()
    x = (synth.normal((T, H), 1.0, g, "cpu").double() * torch.pow(2.0, k)).to(dt)
    r = (synth.normal((T, H), 4.0, g, "cpu").double() * torch.pow(2.0, k)).to(dt)
    w = synth.weight(H, dt, g, "cpu")
    return x, r, w


@pytest.mark.parametrize("op", ["rms_norm", "fused_add_rms_norm"])
def test_fuzz_16bit_ops(op):
    rng = np.random.default_rng(1234 if op == "rms_norm" else 4321)
    for c in range(CASES):
        T, H, dtype, with_w, offset = _case(rng)
        x, r, w = _inputs(T, H, dtype, seed=c)
        xd = _tensor(x, offset)
        rd = _tensor(r, offset)
        wd = w.cuda() if with_w else None
        in_place = rng.random() < 0.25
        out = xd if in_place else _tensor(torch.zeros_like(x), offset)
        if op == "rms_norm":
            rn.rms_norm(out, xd, wd, 1e-6)
            got = {"out": out}
        else:
            rn.fused_add_rms_norm(out, xd, rd, wd, 1e-6)
            got = {"out": out, "residual": rd}
        torch.cuda.synchronize()
        want = oracle_run(op, x, None if op == "rms_norm" else r, w if with_w else None, 1e-6,
                          dtype)
        compare(op, got, want, dtype)


def test_fuzz_fp8_op():
    rng = np.random.default_rng(777)
    diff, total = 0, 0
    for c in range(CASES):
        T, H, dtype, with_w, offset = _case(rng)
        x, r, w = _inputs(T, H, dtype, seed=100 + c)
        xd, rd = _tensor(x, offset), _tensor(r, offset)
        qbuf = torch.empty(T * H + 16, dtype=torch.uint8, device="cuda")
        q = qbuf[offset:offset + T * H].view(T, H).view(torch.float8_e4m3fn)
        scale = torch.empty(T, dtype=torch.float32, device="cuda")
        rn.fused_add_rms_norm_fp8(q, scale, xd, rd, w.cuda() if with_w else None, 1e-6)
        torch.cuda.synchronize()
        want = oracle_run("fused_add_rms_norm_fp8", x, r, w if with_w else None, 1e-6, dtype)
        assert np.array_equal(bits16(rd).reshape(T, H), want["residual"].reshape(T, H))
        d = code_dist8(codes8(q).reshape(T, H), want["q"].reshape(T, H))
        assert d.max() <= 1, (c, T, H, dtype)
        diff += int(np.count_nonzero(d))
        total += d.size
        ws = want["scale"].astype(np.float64)
        gs = scale.cpu().numpy().astype(np.float64)
        assert (np.abs(gs - ws) <= SCALE_RTOL * np.abs(ws)).all(), (c, T, H, dtype)
    assert diff / total <= FP8_MAX_MISMATCH_FRAC, diff / total


def test_fuzz_swiglu():
    """silu_and_mul_fp8 on random [T x 2I] (I any width; the vector kernel
    where I % 8 == 0 and the pointers allow), rows scaled by 2^-4..2^4."""
    import oracle
    from tests.gpu_util import CORES
    rng = np.random.default_rng(99)
    diff, total = 0, 0
    for c in range(CASES):
        T = int(rng.integers(1, 301))
        I = 8 * int(rng.integers(1, 1201)) if rng.random() < 0.7 else int(rng.integers(1, 3001))
        dtype = "bf16" if rng.random() < 0.6 else "fp16"
        offset = int(rng.choice([0, 0, 1, 8]))
        g = torch.Generator().manual_seed(500 + c)
        k = torch.randint(-4, 5, (T, 1), generator=g).double()
        x = (synth.normal((T, 2 * I), 1.0, g, "cpu").double() * torch.pow(2.0, k)).to(
            synth.to_dtype(dtype))
        xd = _tensor(x, offset)
        qbuf = torch.empty(T * I + 16, dtype=torch.uint8, device="cuda")
        q = qbuf[offset:offset + T * I].view(T, I).view(torch.float8_e4m3fn)
        s = torch.empty(T, dtype=torch.float32, device="cuda")
        rn.silu_and_mul_fp8(q, s, xd)
        torch.cuda.synchronize()
        want_q, want_s = oracle.silu_and_mul_fp8(bits16(x), dtype, threads=CORES)
        d = code_dist8(codes8(q).reshape(T, I), want_q.reshape(T, I))
        assert d.max() <= 1, (c, T, I, dtype)
        diff += int(np.count_nonzero(d))
        total += d.size
        ws = want_s.astype(np.float64)
        gs = s.cpu().numpy().astype(np.float64)
        assert (np.abs(gs - ws) <= SCALE_RTOL * np.abs(ws)).all(), (c, T, I, dtype)
    assert diff / total <= FP8_MAX_MISMATCH_FRAC, diff / total


def test_fuzz_fp8_gemm():
    """fp8_rowwise_gemm with the automatic tile configuration on random M x N x
    K (N a multiple of 8, K of 16), checked in full against the oracle with
    the derived per-element bound of the GEMM tests."""
    from tests.test_gpu_fp8_gemm import _check, _operands
    rng = np.random.default_rng(2024)
    for c in range(30):
        M = int(rng.integers(1, 301))
        N = 8 * int(rng.integers(1, 257))
        K = 16 * int(rng.integers(1, 129))
        a, b, sa, sb = _operands(M, N, K, seed=900 + c)
        d = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        rn.fp8_rowwise_gemm(d, a.cuda(), b.cuda(), sa.cuda(), sb.cuda())
        torch.cuda.synchronize()
        _check(d, codes8(a), codes8(b), sa.numpy(), sb.numpy())
