"""Chains of dependent calls on one stream, as a decoder layer issues them: each
launch reads rows the previous launch has just written (its 16-bit output, and
the residual it updated in place). Under programmatic dependent launch each
launch asks L2 for its first rows before the previous launch has finished
writing them (here: the residual every step updates in place, and the
output of the last 16-bit step); L2 is the device's point of coherence, so every load after
`griddepcontrol.wait` must still see the previous launch's writes. These tests
check that every step of such chains, eager and replayed from a CUDA graph,
matches the oracle applied to that step's own inputs (the residual bit for
bit, outputs within 1 ulp, codes within one step), at a prefill size whose
launches overlap the previous one's tail and at a decode size."""
import numpy as np
import pytest
import torch

import residual_add_rmsnorm_rms_b200 as rn
import synth
from tests.cmp_util import bits16
from tests.gpu_util import compare, oracle_run

pytestmark = pytest.mark.gpu
STEPS = 6


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    rn.set_prefetch(-1)
    yield
    rn.set_prefetch(-1)
    assert rn.device_errors() == 0


def _ops(fp8):
    """The op of each step: fused_add_rms_norm, alternating with
    fused_add_rms_norm_fp8 when `fp8`."""
    return ["fused_add_rms_norm_fp8" if fp8 and k % 2 == 1 else "fused_add_rms_norm"
            for k in range(STEPS)]


def _fused_chain(T, H, dtype, fp8=False, graph=False):
    """Every step reads the residual the previous step updated in place, and
    x = the output of the last fused_add_rms_norm step (the input x for the
    first). Only this library's kernels run between the launches. Returns
    the inputs, the starting residual, the residual after the chain and
    every step's outputs."""
    wl = synth.make_inputs("prefill", "fused_add_rms_norm", dtype, T, H, device="cuda")
    r = wl.residual.clone()
    r0 = r.clone()
    outs = [torch.empty(T, H, dtype=wl.dtype, device="cuda") for _ in range(STEPS)]
    qs = [torch.empty(T, H, dtype=torch.float8_e4m3fn, device="cuda") for _ in range(STEPS)]
    scales = [torch.empty(T, dtype=torch.float32, device="cuda") for _ in range(STEPS)]
    ops = _ops(fp8)

    def run():
        x = wl.x
        for k, op in enumerate(ops):
            if op == "fused_add_rms_norm":
                rn.fused_add_rms_norm(outs[k], x, r, wl.weight, wl.eps)
                x = outs[k]
            else:
                rn.fused_add_rms_norm_fp8(qs[k], scales[k], x, r, wl.weight, wl.eps)

    if graph:
        st = torch.cuda.Stream()
        with torch.cuda.stream(st):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=st):
                run()
        r.copy_(r0)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        del g
    else:
        run()
        torch.cuda.synchronize()
    return wl, r0, r, outs, qs, scales


def _check_fused_chain(T, H, dtype, fp8=False, graph=False, rows=None):
    wl, r0, r_end, outs, qs, scales = _fused_chain(T, H, dtype, fp8, graph)
    sel = (lambda t: t.cpu()) if rows is None else (lambda t: t[rows].cpu())
    r = sel(r0)
    x = sel(wl.x)
    w = wl.weight.cpu()
    for k, op in enumerate(_ops(fp8)):
        want = oracle_run(op, x, r, w, wl.eps, dtype)
        if op == "fused_add_rms_norm":
            compare(op, {"out": sel(outs[k])}, {"out": want["out"]}, dtype)
            x = sel(outs[k])  # the next steps read this step's GPU output
        else:
            compare(op, {"q": sel(qs[k]), "scale": sel(scales[k])},
                    {"q": want["q"], "scale": want["scale"]}, dtype)
        # the residual after each step is exact: carry the oracle's forward
        r = torch.from_numpy(want["residual"].astype(np.int16)).view(synth.to_dtype(dtype))
    assert np.array_equal(bits16(sel(r_end)), bits16(r)), "residual after the chain differs"


@pytest.mark.parametrize("graph", [False, True], ids=["eager", "graph"])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_dependent_fused_chain_prefill(dtype, graph):
    """[8192 x 3840]: every launch overlaps the tail of the previous one;
    a sample of rows (first, last, spread) is checked at every step."""
    rows = torch.from_numpy(np.unique(np.concatenate(
        [[0, 8191], np.linspace(0, 8191, 61).astype(np.int64),
         np.random.default_rng(5).integers(0, 8192, 64)]))).cuda()
    _check_fused_chain(8192, 3840, dtype, fp8=True, graph=graph, rows=rows)


@pytest.mark.parametrize("graph", [False, True], ids=["eager", "graph"])
def test_dependent_fused_chain_decode(graph):
    _check_fused_chain(64, 4096, "bf16", fp8=True, graph=graph)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_dependent_rms_norm_chain(dtype):
    """y_{k+1} = rms_norm(y_k), every step in its own buffer: each launch
    normalises the rows the previous one has just written."""
    T, H = 4096, 8192
    wl = synth.make_inputs("sweep", "rms_norm", dtype, T, H, device="cuda")
    ys = [wl.x] + [torch.empty_like(wl.x) for _ in range(STEPS)]
    for k in range(STEPS):
        rn.rms_norm(ys[k + 1], ys[k], wl.weight, wl.eps)
    torch.cuda.synchronize()
    rows = torch.arange(0, T, 97, device="cuda")
    w = wl.weight.cpu()
    for k in range(STEPS):
        want = oracle_run("rms_norm", ys[k][rows].cpu(), None, w, wl.eps, dtype)
        compare("rms_norm", {"out": ys[k + 1][rows].cpu()}, want, dtype)


@pytest.mark.parametrize("prefetch", [0, 1])
def test_chain_results_do_not_depend_on_the_prefetch(prefetch):
    """The same chain with the prefetch off and on gives identical bits."""
    rn.set_prefetch(prefetch)
    _, _, r_end, outs, qs, scales = _fused_chain(2048, 3840, "bf16", fp8=True)
    rn.set_prefetch(1 - prefetch)
    _, _, r_end2, outs2, qs2, scales2 = _fused_chain(2048, 3840, "bf16", fp8=True)
    assert torch.equal(r_end.view(torch.int16), r_end2.view(torch.int16))
    for k, op in enumerate(_ops(True)):
        if op == "fused_add_rms_norm":
            assert torch.equal(outs[k].view(torch.int16), outs2[k].view(torch.int16))
        else:
            assert torch.equal(qs[k].view(torch.uint8), qs2[k].view(torch.uint8))
            assert torch.equal(scales[k], scales2[k])
