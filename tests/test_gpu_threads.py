"""Several host threads driving the library at once, each on its own CUDA
stream and buffers (ctypes releases the GIL during the C calls, so the calls
really overlap): every thread's results equal, bit for bit, those of the
same calls made one after another on one thread (the kernels are
deterministic), and no call fails. Covers the per-thread descriptor caches of
the binding and the library's thread-local error text."""
import threading

import pytest
import torch

import residual_add_rmsnorm_rms_b200 as rn
import synth

pytestmark = pytest.mark.gpu

# (op, T, H) per thread: different shapes, so every thread fills its own
# descriptor cache entries
WORK = [("fused_add_rms_norm", 512, 3840), ("fused_add_rms_norm_fp8", 300, 4096),
        ("rms_norm", 1024, 2048), ("silu_and_mul_fp8", 256, 1536),
        ("fp8_rowwise_gemm", 16, 3840), ("fused_add_rms_norm", 77, 5120)]
ROUNDS = 40


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    yield
    assert rn.device_errors() == 0


def _inputs(op, T, H, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    dt = torch.bfloat16
    if op == "silu_and_mul_fp8":
        return {"x": torch.randn(T, 2 * H, generator=g, device="cuda").to(dt)}
    if op == "fp8_rowwise_gemm":
        a = (torch.randn(T, H, generator=g, device="cuda") * 40).clamp_(-448, 448)
        b = (torch.randn(2048, H, generator=g, device="cuda") * 40).clamp_(-448, 448)
        return {"a": a.to(torch.float8_e4m3fn), "b": b.to(torch.float8_e4m3fn),
                "sa": torch.rand(T, generator=g, device="cuda") * 0.01 + 1e-3,
                "sb": torch.rand(2048, generator=g, device="cuda") * 0.01 + 1e-3}
    return {"x": torch.randn(T, H, generator=g, device="cuda").to(dt),
            "r": (torch.randn(T, H, generator=g, device="cuda") * 2).to(dt),
            "w": (1 + 0.3 * torch.randn(H, generator=g, device="cuda")).to(dt)}


def _run(op, inp, rounds, stream=None):
    """`rounds` dependent calls (the fused ops update the residual in place);
    returns the final outputs."""
    if op == "fp8_rowwise_gemm":
        d = torch.empty(inp["a"].shape[0], inp["b"].shape[0], dtype=torch.bfloat16,
                        device="cuda")
        for _ in range(rounds):
            rn.fp8_rowwise_gemm(d, inp["a"], inp["b"], inp["sa"], inp["sb"], stream=stream)
        return [d]
    if op == "silu_and_mul_fp8":
        T, I = inp["x"].shape[0], inp["x"].shape[1] // 2
        q = torch.empty(T, I, dtype=torch.float8_e4m3fn, device="cuda")
        s = torch.empty(T, dtype=torch.float32, device="cuda")
        for _ in range(rounds):
            rn.silu_and_mul_fp8(q, s, inp["x"], stream=stream)
        return [q.view(torch.uint8), s]
    x, r, w = inp["x"], inp["r"].clone(), inp["w"]
    if op == "rms_norm":
        out = torch.empty_like(x)
        for _ in range(rounds):
            rn.rms_norm(out, x, w, 1e-6, stream=stream)
        return [out.view(torch.int16)]
    if op == "fused_add_rms_norm":
        out = torch.empty_like(x)
        for _ in range(rounds):
            rn.fused_add_rms_norm(out, x, r, w, 1e-6, stream=stream)
        return [out.view(torch.int16), r.view(torch.int16)]
    q = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device="cuda")
    s = torch.empty(x.shape[0], dtype=torch.float32, device="cuda")
    for _ in range(rounds):
        rn.fused_add_rms_norm_fp8(q, s, x, r, w, 1e-6, stream=stream)
    return [q.view(torch.uint8), s, r.view(torch.int16)]


def test_threads_each_on_its_own_stream():
    inputs = [_inputs(op, T, H, seed=i) for i, (op, T, H) in enumerate(WORK)]
    want = [_run(op, inp, ROUNDS) for (op, _, _), inp in zip(WORK, inputs)]
    torch.cuda.synchronize()
    got, errors = [None] * len(WORK), []
    start = threading.Barrier(len(WORK))

    def worker(i):
        try:
            torch.cuda.set_device(0)
            st = torch.cuda.Stream()
            with torch.cuda.stream(st):
                start.wait()
                got[i] = _run(WORK[i][0], inputs[i], ROUNDS, stream=st)
            st.synchronize()
        except Exception as e:  # noqa: BLE001 (reported below)
            errors.append((i, repr(e)))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(WORK))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not any(t.is_alive() for t in threads)
    assert not errors, errors
    for i, (w, g) in enumerate(zip(want, got)):
        for a, b in zip(w, g):
            assert torch.equal(a, b), (WORK[i], "differs from the one-thread result")


def test_error_text_is_per_thread():
    """A failing call on one thread does not leave its error text on another
    (rn_last_cuda_error is thread-local): a validation error carries no CUDA
    text at all, and a thread that made no failing call reads ''."""
    seen = {}

    def fail():
        x = torch.empty(4, 6, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(rn.RmsNormError) as e:  # odd 2I: RN_ERR_SHAPE, before any CUDA call
            rn.silu_and_mul_fp8(torch.empty(4, 3, dtype=torch.float8_e4m3fn, device="cuda"),
                                torch.empty(4, device="cuda"), x[:, :5])
        seen["fail"] = e.value.name

    def clean():
        seen["clean"] = rn.lib.rn_last_cuda_error().decode()

    for f in (fail, clean):
        t = threading.Thread(target=f)
        t.start()
        t.join()
    assert seen["fail"] in ("RN_ERR_SHAPE", "RN_ERR_LAYOUT")
    assert seen["clean"] == ""
