"""The host-memory entry points (rn_host_rms_norm, rn_host_fused_add_rms_norm,
rn_host_fused_add_rms_norm_fp8): activations in host memory, cut into chunks
that are copied in, normalised on the device and copied back over one to
four streams. Every result is checked against the CPU oracle on the same
input bits: ragged last chunks, one-row chunks, one chunk, the scalar
kernel's rows (H % 8 != 0), pageable and page-locked host memory, in-place
output, the prefill batch with the automatic chunking, calls of different
ops queued back to back through one pipeline, and a call captured in a CUDA
graph and replayed."""
import pytest
import torch

import residual_add_rmsnorm_rms_b200 as rn
import synth
from residual_add_rmsnorm_rms_b200.host import HostPipeline
from tests.gpu_util import compare, oracle_run, sample_rows

pytestmark = pytest.mark.gpu

OPS = ("rms_norm", "fused_add_rms_norm", "fused_add_rms_norm_fp8")


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    yield
    assert rn.device_errors() == 0


def _pipeline(op, T, H, n, chunk):
    if chunk <= 0:
        return HostPipeline.for_problem(op, T, H, "cuda", n_streams=n)
    p = rn.host_plan_chunks(op, T, H, 1 << 50, n, chunk)
    return HostPipeline("cuda", p["slots"] * p["slot_bytes"], n, chunk)


def _host(t, pinned):
    t = t.clone()
    return t.pin_memory() if pinned else t


def _run_host(op, x, r, w, eps, pipe, pinned=True, join=True, in_place=False):
    """Host copies of the inputs through `pipe`; returns the host results."""
    hx = _host(x, pinned)
    hr = None if r is None else _host(r, pinned)
    wd = None if w is None else w.cuda()
    if op == "fused_add_rms_norm_fp8":
        T = x.numel() // x.shape[-1]
        q = torch.empty(x.shape, dtype=torch.float8_e4m3fn)
        scale = torch.empty(T, dtype=torch.float32)
        if pinned:
            q, scale = q.pin_memory(), scale.pin_memory()
        rn.host_fused_add_rms_norm_fp8(q, scale, hx, hr, wd, eps, pipe, join=join)
        return {"q": q, "scale": scale, "residual": hr}
    out = hx if in_place else _host(torch.empty_like(x), pinned)
    if op == "rms_norm":
        rn.host_rms_norm(out, hx, wd, eps, pipe, join=join)
        return {"out": out}
    rn.host_fused_add_rms_norm(out, hx, hr, wd, eps, pipe, join=join)
    return {"out": out, "residual": hr}


# (workload, T, H, chunk rows (0: automatic), streams, page-locked)
CASES = [
    ("small", 1000, 512, 77, 3, True),    # 13 chunks, ragged last one
    ("decode", 130, 4096, 0, 2, True),    # automatic: one chunk
    ("outlier", 64, 16384, 10, 4, False),  # pageable host memory
    ("small", 33, 1004, 5, 1, True),      # H % 8 != 0: scalar kernel
    ("small", 9, 2048, 1, 3, True),       # one row per chunk
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-{c[1]}x{c[2]}-c{c[3]}-s{c[4]}")
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("op", OPS)
def test_host_pipeline_parity(op, dtype, case):
    name, T, H, chunk, n, pinned = case
    wl = synth.make_inputs(name, op, dtype, T, H)
    pipe = _pipeline(op, T, H, n, chunk)
    got = _run_host(op, wl.x, wl.residual, wl.weight, wl.eps, pipe, pinned=pinned)
    torch.cuda.synchronize()
    compare(op, got, oracle_run(op, wl.x, wl.residual, wl.weight, wl.eps, dtype), dtype)


@pytest.mark.parametrize("op", ["rms_norm", "fused_add_rms_norm"])
def test_host_pipeline_in_place(op):
    T, H = 500, 3840
    wl = synth.make_inputs("small", op, "bf16", T, H)
    pipe = _pipeline(op, T, H, 3, 64)
    got = _run_host(op, wl.x, wl.residual, wl.weight, wl.eps, pipe, in_place=True)
    torch.cuda.synchronize()
    compare(op, got, oracle_run(op, wl.x, wl.residual, wl.weight, wl.eps, "bf16"), "bf16")


def test_host_pipeline_no_weight():
    T, H = 200, 2048
    wl = synth.make_inputs("small", "fused_add_rms_norm_fp8", "bf16", T, H)
    pipe = _pipeline("fused_add_rms_norm_fp8", T, H, 2, 30)
    got = _run_host("fused_add_rms_norm_fp8", wl.x, wl.residual, None, wl.eps, pipe)
    torch.cuda.synchronize()
    compare("fused_add_rms_norm_fp8", got,
            oracle_run("fused_add_rms_norm_fp8", wl.x, wl.residual, None, wl.eps, "bf16"), "bf16")


@pytest.mark.parametrize("op", ["fused_add_rms_norm", "fused_add_rms_norm_fp8"])
def test_host_pipeline_prefill_sampled(op):
    """The prefill batch [8192 x 3840] with the automatic chunking over three
    streams; the oracle checks a sample of rows."""
    T, H = 8192, 3840
    wl = synth.make_inputs("prefill", op, "bf16", T, H)
    pipe = HostPipeline.for_problem(op, T, H, "cuda", n_streams=3)
    assert rn.host_plan_chunks(op, T, H, 1 << 50, 3)["chunks"] >= 6
    got = _run_host(op, wl.x, wl.residual, wl.weight, wl.eps, pipe)
    torch.cuda.synchronize()
    rows = sample_rows(T)
    want = oracle_run(op, wl.x[rows], wl.residual[rows], wl.weight, wl.eps, "bf16")
    compare(op, got, want, "bf16", rows=rows)


def test_host_pipeline_back_to_back_ops():
    """fused, fp8, fused, rms_norm queued through one pipeline without joining
    in between (the slot layout changes at each call), then one join."""
    T, H = 700, 4096
    seq = ["fused_add_rms_norm", "fused_add_rms_norm_fp8", "fused_add_rms_norm", "rms_norm"]
    pipe = HostPipeline.for_problem(["fused_add_rms_norm_fp8", "fused_add_rms_norm"], T, H,
                                    "cuda", n_streams=3)
    runs = []
    for i, op in enumerate(seq):
        wl = synth.make_inputs("small", op, "bf16", T, H, seed=4100 + i)
        runs.append((op, wl, _run_host(op, wl.x, wl.residual, wl.weight, wl.eps, pipe,
                                       join=False)))
    pipe.join_into()
    torch.cuda.synchronize()
    for op, wl, got in runs:
        compare(op, got, oracle_run(op, wl.x, wl.residual, wl.weight, wl.eps, "bf16"), "bf16")


def test_host_pipeline_empty_and_plan():
    pipe = HostPipeline("cuda", 1 << 20, 2, 16)
    x = torch.empty(0, 512, dtype=torch.bfloat16)
    rn.host_rms_norm(torch.empty_like(x), x, None, 1e-6, pipe)
    p = rn.host_plan_chunks("fused_add_rms_norm", 100, 512, 1 << 20, 2, 16)
    assert (p["chunk_rows"], p["chunks"], p["slots"]) == (16, 7, 2)
    # scratch smaller than the slots in use is refused before any copy
    small = HostPipeline("cuda", p["slot_bytes"], 2, 16)
    wl = synth.make_inputs("small", "fused_add_rms_norm", "bf16", 100, 512)
    with pytest.raises(rn.RmsNormError) as e:
        _run_host("fused_add_rms_norm", wl.x, wl.residual, wl.weight, wl.eps, small)
    assert e.value.name == "RN_ERR_CAPACITY"


def test_host_pipeline_refuses_host_weight():
    """The weight must be device memory: a page-locked host weight is refused
    before any copy or launch (page-locked, so that even a launch could only
    read mapped host memory), by the binding and by the C ABI itself."""
    T, H = 64, 512
    wl = synth.make_inputs("small", "fused_add_rms_norm", "bf16", T, H)
    pipe = _pipeline("fused_add_rms_norm", T, H, 2, 16)
    hx, hr, out = wl.x.clone(), wl.residual.clone(), torch.empty_like(wl.x)
    w_host = wl.weight.clone().pin_memory()
    with pytest.raises(ValueError):
        rn.host_fused_add_rms_norm(out, hx, hr, w_host, wl.eps, pipe)
    st = rn.lib.rn_host_fused_add_rms_norm(rn._desc(out, 0), rn._desc(hx, 1), rn._desc(hr, 2),
                                           rn._desc(w_host, 3), wl.eps, -1,
                                           pipe.descriptor_ref())
    torch.cuda.synchronize()
    assert rn.STATUS[st] == "RN_ERR_LAYOUT"
    assert torch.equal(hr.view(torch.int16), wl.residual.view(torch.int16))


def test_host_pipeline_in_a_cuda_graph():
    """A host-memory call captured in a CUDA graph (the pipeline's streams fork
    from and join back into the capturing stream): each replay copies the
    page-locked rows in, normalises them and copies them back, so two replays
    apply the fused op twice."""
    T, H = 600, 4096
    wl = synth.make_inputs("small", "fused_add_rms_norm", "bf16", T, H)
    pipe = _pipeline("fused_add_rms_norm", T, H, 2, 128)
    hx = wl.x.clone().pin_memory()
    hr = wl.residual.clone().pin_memory()
    out = torch.empty_like(wl.x).pin_memory()
    w = wl.weight.cuda()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side, capture_error_mode="relaxed"):
            rn.host_fused_add_rms_norm(out, hx, hr, w, wl.eps, pipe)
    torch.cuda.synchronize()
    assert torch.equal(hr.view(torch.int16), wl.residual.view(torch.int16))  # nothing ran yet
    graph.replay()
    torch.cuda.synchronize()
    want = oracle_run("fused_add_rms_norm", wl.x, wl.residual, wl.weight, wl.eps, "bf16")
    compare("fused_add_rms_norm", {"out": out.clone(), "residual": hr.clone()}, want, "bf16")
    r1 = torch.from_numpy(want["residual"].view("int16").copy()).view(torch.bfloat16).view(T, H)
    graph.replay()
    torch.cuda.synchronize()
    want2 = oracle_run("fused_add_rms_norm", wl.x, r1, wl.weight, wl.eps, "bf16")
    compare("fused_add_rms_norm", {"out": out, "residual": hr}, want2, "bf16")
    del graph
