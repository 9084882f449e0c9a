"""Host-side tests of the C ABI (CPU only: nothing here launches a kernel).

* the shared library loads and exports every function include/rmsnorm_b200.h
  declares;
* argument validation (rn_validate, the dry run that performs exactly the
  checks of the real entry points) accepts and rejects the layouts of
  flatten_to_2d_is_free ("vllm.kernels.aiter_ops") and the dtype /
  variance-size rules of rms_no_var_16bit_only and rms_add_no_var_16bit_only;
* the launch planner's invariants.
The real entry points are also called, but only with arguments that fail
validation (so they return before any CUDA call).
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

import residual_add_rmsnorm_rms_b200 as rn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rmsnorm_b200.h")
BF, F16 = torch.bfloat16, torch.float16


def header_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^RN_API\s+[\w\s\*]+?\b(rn_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_three_operators():
    names = header_functions()
    for op in ("rn_rms_norm", "rn_fused_add_rms_norm", "rn_fused_add_rms_norm_fp8"):
        assert op in names


def test_library_exports_every_declared_symbol():
    names = header_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(rn.lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", rn.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)$", out, flags=re.M))
    assert set(names) <= exported
    # nothing else leaks out of the library under the rn_ prefix
    assert {e for e in exported if e.startswith("rn_")} == set(names)


def test_build_targets_sm100a_only():
    """The build compiles and links device code for sm_100a and nothing else
    (the loaded code's version is checked on the GPU through
    rn_kernel_binary_version)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_rn_build_flags", os.path.join(ROOT, "residual_add_rmsnorm_rms_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    assert b.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    for flags in (b.NVCC_FLAGS, b.CUTLASS_FLAGS):
        for f in flags:
            assert not re.search(r"(sm|compute)_(?!100a)\d+", f), f
            assert f not in ("-arch", "--gpu-architecture", "--generate-code"), f


def test_python_constants_match_the_header():
    src = open(HEADER).read()
    define = lambda n: int(re.search(rf"#define {n} (\d+)", src).group(1))  # noqa: E731
    assert rn.ALLREDUCE_MAX_WORLD == define("RN_ALLREDUCE_MAX_WORLD")
    assert rn.ALLREDUCE_SIGNAL_BYTES == define("RN_ALLREDUCE_SIGNAL_BYTES")
    assert rn.HOST_MAX_STREAMS == define("RN_HOST_MAX_STREAMS")
    assert rn.LOCAL_EXCHANGE_BYTES == define("RN_LOCAL_EXCHANGE_BYTES")
    assert rn.MAX_DIMS == define("RN_MAX_DIMS")


def V(op, *args, **kw):
    return rn.validate(op, *args, **kw)[0]


def VR(out, x, weight=None, **kw):
    """rms_norm dry run (it takes no residual)."""
    return rn.validate("rms_norm", out, x, None, weight, **kw)[0]


def t(shape, dtype=BF, **kw):
    return torch.empty(shape, dtype=dtype, **kw)


H = 256


@pytest.mark.parametrize("op", ["rms_norm", "fused_add_rms_norm"])
def test_flatten_to_2d_is_free_cases(op):
    def call(x):
        out = torch.empty_like(x, memory_format=torch.contiguous_format) if x.is_contiguous() \
            else torch.empty(x.shape, dtype=x.dtype)
        res = torch.empty(x.shape, dtype=x.dtype) if op != "rms_norm" else None
        return V(op, out, x, res)

    # contiguous N-D: accepted
    assert call(t((2, 3, H))) == "RN_OK"
    assert call(t((H,))) == "RN_OK"  # 1-D: a single row
    # transposed leading dims: reshape would copy -> rejected
    assert call(t((3, 2, H)).transpose(0, 1)) == "RN_ERR_LAYOUT"
    # size-1 dims may carry any stride
    x = t((4 * H,)).as_strided((4, 1, H), (H, 7, 1))
    assert call(x) == "RN_OK"
    # strided last dim: flattens without a copy but not densely -> rejected
    assert call(t((4, 2 * H))[:, ::2]) == "RN_ERR_LAYOUT"
    # padded rows: rejected for > 2-D and (this library's reading) for 2-D
    assert call(t((2, 4, H + 8))[:, :, :H]) == "RN_ERR_LAYOUT"
    assert call(t((4, H + 8))[:, :H]) == "RN_ERR_LAYOUT"
    # degenerate shapes
    assert call(t((0, H))) == "RN_OK"  # T == 0: a no-op
    assert call(t((4, 0))) == "RN_ERR_SHAPE"  # H == 0
    assert call(torch.tensor(1.0, dtype=BF)) == "RN_ERR_SHAPE"  # 0-d


def test_dtype_and_weight_rules():
    x = t((4, H))
    assert VR(t((4, H)), x, None) == "RN_OK"
    assert VR(t((4, H), F16), t((4, H), F16), t((H,), F16)) == "RN_OK"
    assert VR(t((4, H), torch.float32), t((4, H), torch.float32), None) == "RN_ERR_DTYPE"
    assert VR(t((4, H), F16), x, None) == "RN_ERR_DTYPE"  # out dtype != x
    assert VR(t((4, H)), x, t((H,), F16)) == "RN_ERR_WEIGHT_DTYPE"
    assert VR(t((4, H)), x, t((H,), torch.float32)) == "RN_ERR_WEIGHT_DTYPE"
    assert VR(t((4, H)), x, t((H + 1,))) == "RN_ERR_SHAPE"
    assert VR(t((4, H)), x, t((1, H))) == "RN_ERR_SHAPE"
    assert VR(t((4, H)), x, t((2 * H,))[::2]) == "RN_ERR_LAYOUT"
    assert V("fused_add_rms_norm", t((4, H)), x, t((4, H), F16), None) == "RN_ERR_DTYPE"
    assert V("fused_add_rms_norm", t((4, H)), x, t((4, H + 8)), None) == "RN_ERR_SHAPE"
    assert V("fused_add_rms_norm", t((4, H)), x, t((5, H)), None) == "RN_ERR_SHAPE"
    # N-D views of matching [T x H] flatten alike
    assert V("fused_add_rms_norm", t((2, 2, H)), x, t((4, 1, H)), None) == "RN_OK"


def test_variance_size_and_eps():
    x = t((4, H))
    for op, res in (("rms_norm", None), ("fused_add_rms_norm", t((4, H)))):
        assert V(op, t((4, H)), x, res, variance_size=H) == "RN_ERR_VARIANCE_SIZE"
        assert V(op, t((4, H)), x, res, variance_size=0) == "RN_ERR_VARIANCE_SIZE"
        assert V(op, t((4, H)), x, res, variance_size=None) == "RN_OK"
        for eps in (-1e-6, float("nan"), float("inf")):
            assert V(op, t((4, H)), x, res, eps=eps) == "RN_ERR_EPS"
        assert V(op, t((4, H)), x, res, eps=0.0) == "RN_OK"


def test_fp8_operands():
    x, r = t((4, H)), t((4, H))
    q, s = t((4, H), torch.float8_e4m3fn), t((4,), torch.float32)
    assert V("fused_add_rms_norm_fp8", q, x, r, None, scale=s) == "RN_OK"
    assert V("fused_add_rms_norm_fp8", t((4, H), torch.uint8), x, r, None, scale=s) == "RN_OK"
    assert V("fused_add_rms_norm_fp8", q, x, r, None, scale=t((4, 1), torch.float32)) == "RN_OK"
    assert V("fused_add_rms_norm_fp8", t((4, H)), x, r, None, scale=s) == "RN_ERR_DTYPE"
    assert V("fused_add_rms_norm_fp8", q, x, r, None, scale=t((4,), BF)) == "RN_ERR_DTYPE"
    assert V("fused_add_rms_norm_fp8", q, x, r, None, scale=t((5,), torch.float32)) == "RN_ERR_SHAPE"
    assert V("fused_add_rms_norm_fp8", q, x, r, None, scale=t((8,), torch.float32)[::2]) == "RN_ERR_LAYOUT"
    assert V("fused_add_rms_norm_fp8", q, x, r, None, scale=None) == "RN_ERR_NULL"
    assert V("fused_add_rms_norm_fp8", t((4, H + 8), torch.float8_e4m3fn)[:, :H], x, r, None,
             scale=s) == "RN_ERR_LAYOUT"


def test_aliasing_rules():
    buf = t((8, H))
    x = buf[:4]
    # out == x exactly: in place, allowed
    assert VR(x, x, None) == "RN_OK"
    assert V("fused_add_rms_norm", x, x, t((4, H)), None) == "RN_OK"
    # out overlapping x partially
    assert VR(buf[2:6], x, None) == "RN_ERR_ALIAS"
    # residual aliasing x, or out aliasing residual
    r = t((4, H))
    assert V("fused_add_rms_norm", t((4, H)), x, x, None) == "RN_ERR_ALIAS"
    assert V("fused_add_rms_norm", r, x, r, None) == "RN_ERR_ALIAS"
    # weight inside a written buffer
    out = t((4, H))
    assert VR(out, x, out[0]) == "RN_ERR_ALIAS"
    # weight inside x is read-only data: allowed when x is not written
    assert VR(t((4, H)), x, x[0]) == "RN_OK"
    # fp8: q/scale overlapping inputs or each other
    big = t((16, H))
    q8 = big.view(torch.uint8)[:2].reshape(4, H)  # the bytes of bf16 rows 0-1
    assert V("fused_add_rms_norm_fp8", q8, big[8:12], big[12:16], None,
             scale=t((4,), torch.float32)) == "RN_OK"
    qx = big.view(torch.uint8)[4:6].reshape(4, H)  # inside x = rows 4-7
    assert V("fused_add_rms_norm_fp8", qx, big[4:8], big[12:16], None,
             scale=t((4,), torch.float32)) == "RN_ERR_ALIAS"
    sc = big[12].view(torch.float32)[:4]
    assert V("fused_add_rms_norm_fp8", q8, big[8:12], big[12:16], None, scale=sc) == "RN_ERR_ALIAS"


def _raw_desc(ptr, shape, strides, dtype=1):
    n = len(shape)
    sizes = (ctypes.c_int64 * n)(*shape)
    strd = (ctypes.c_int64 * n)(*strides)
    return rn.RnTensor(ptr, dtype, n, sizes, strd), (sizes, strd)


def test_null_and_misaligned_pointers_never_launch():
    # data NULL with T > 0
    d0, k0 = _raw_desc(0, (4, H), (H, 1))
    d1, k1 = _raw_desc(0x10000, (4, H), (H, 1))
    plan = rn.RnPlan()
    assert rn.lib.rn_validate(0, ctypes.byref(d1), None, ctypes.byref(d0), None, None, 1e-6, -1,
                              ctypes.byref(plan)) == 1
    # misaligned (odd byte address) 16-bit data
    dm, km = _raw_desc(0x10001, (4, H), (H, 1))
    assert rn.lib.rn_validate(0, ctypes.byref(d1), None, ctypes.byref(dm), None, None, 1e-6, -1,
                              None) == 5
    # NULL descriptors on the real entry points return before any CUDA call
    assert rn.lib.rn_rms_norm(None, ctypes.byref(d1), None, 1e-6, -1, None) == 1
    assert rn.lib.rn_fused_add_rms_norm(ctypes.byref(d1), ctypes.byref(d1), None, None, 1e-6, -1,
                                        None) == 1
    assert rn.lib.rn_fused_add_rms_norm_fp8(None, None, ctypes.byref(d1), ctypes.byref(d1), None,
                                            1e-6, -1, None) == 1
    # and so do the other validation failures
    assert rn.lib.rn_rms_norm(ctypes.byref(d1), ctypes.byref(d1), None, 1e-6, 3, None) == 7
    assert rn.lib.rn_rms_norm(ctypes.byref(d1), ctypes.byref(d1), None, -1.0, -1, None) == 8


def test_binding_rejects_cpu_tensors():
    x = t((4, H))
    with pytest.raises(ValueError):
        rn.rms_norm(torch.empty_like(x), x, None, 1e-6)


def test_alignment_selects_kernel():
    x = t((4, 4096 + 16))
    xs = x[:, 1:4097]  # not a dense view -> layout error
    assert VR(t((4, 4096)), xs, None) == "RN_ERR_LAYOUT"
    flat = t((4 * 4096 + 1,))
    xo = flat[1:].view(4, 4096)  # dense but 2-byte (not 16-byte) aligned
    st, plan = rn.validate("rms_norm", t((4, 4096)), xo)
    assert st == "RN_OK" and plan["kernel"] == 1  # scalar kernel
    st, plan = rn.validate("rms_norm", t((4, 4096)), t((4, 4096)))
    assert st == "RN_OK" and plan["kernel"] == 0
    st, plan = rn.validate("rms_norm", t((4, 1004)), t((4, 1004)))  # H % 8 != 0
    assert st == "RN_OK" and plan["kernel"] == 1


SWEEP_T = (1, 8, 16, 64, 256, 4096, 8192, 32768, 65536)
SWEEP_H = (512, 2048, 3840, 4096, 5120, 7168, 8192, 16384)


@pytest.mark.parametrize("op", list(rn.OPS))
def test_planner_invariants(op):
    for T in SWEEP_T:
        for Hh in SWEEP_H:
            p = rn.plan_launch(op, BF, T, Hh)
            assert p["kernel"] == 0, (T, Hh)
            if p["kernel"] == 2:
                # staged: persistent grid, ring of >= 2 stages within 227 KB
                nin = 1 if op == "rms_norm" else 2
                slot = -(-2 * Hh // 128) * 128
                assert p["stages"] >= 2
                assert p["smem_bytes"] == p["stages"] * (nin * slot + 8) + 4 * Hh + 256
                assert p["smem_bytes"] <= 227 * 1024
                assert p["ctas_per_sm"] * (p["smem_bytes"] + 1024) <= 228 * 1024
                assert p["ctas_per_sm"] * p["block_threads"] <= 1024
                assert p["block_threads"] % 32 == 0
                assert p["grid"] == min(T, p["ctas_per_sm"] * 148)
                assert T >= 4 * 148
                continue
            tpr, vpt, rpc = p["threads_per_row"], p["vectors_per_thread"], p["rows_per_cta"]
            assert tpr * vpt * 8 >= Hh
            assert tpr * vpt * 8 - Hh < Hh  # at most one idle slot per used slot
            assert p["block_threads"] == tpr * rpc
            assert p["block_threads"] % 32 == 0 and p["block_threads"] <= 1024
            if tpr > 32:
                assert tpr % 32 == 0 and rpc <= 15
            else:
                assert 32 % tpr == 0
            # grid: one block per rpc rows, capped at 16 blocks per SM (148
            # SMs) except for the fused ops on 8192 rows or more
            blocks = -(-T // rpc)
            uncapped = op != "rms_norm" and T >= 8192
            assert p["grid"] == (blocks if uncapped else min(blocks, 16 * 148))
            assert vpt in rn.supported_vectors_per_thread()
    # the scalar kernel beyond the vector kernel's reach
    assert rn.plan_launch(op, BF, 4, 1 << 17)["kernel"] == 1


def test_planner_measured_choices():
    """The launch shapes the forced-shape grids on B200 chose: four vectors
    per thread at H = 3840 (they move as two 32-byte pairs); blocks of about
    256 threads for rms_norm, about 512 for fused_add_rms_norm, about 256
    then 512 (from 16384 rows) for the fp8 op, which takes eight vectors per
    thread on wide rows below 8192 rows; no grid cap for the fused ops from
    8192 rows on."""
    def shape(op, T, H):
        p = rn.plan_launch(op, BF, T, H)
        return p["threads_per_row"], p["vectors_per_thread"], p["rows_per_cta"]
    fused, fp8 = "fused_add_rms_norm", "fused_add_rms_norm_fp8"
    assert shape(fused, 8192, 3840) == (128, 4, 4)
    assert shape(fused, 4096, 2048) == (64, 4, 8)
    assert shape(fused, 4096, 5120) == (160, 4, 3)
    assert shape(fused, 32768, 8192) == (256, 4, 2)
    assert shape(fp8, 8192, 3840) == (128, 4, 2)
    assert shape(fp8, 16384, 3840) == (128, 4, 4)
    assert shape(fp8, 4096, 3840) == (128, 4, 2)
    assert shape(fp8, 4096, 5120) == (160, 4, 2)
    assert shape(fp8, 4096, 7168) == (128, 8, 1)
    assert shape(fp8, 8192, 7168) == (224, 4, 2)
    assert shape(fp8, 32768, 5120) == (160, 4, 3)
    assert rn.plan_launch(fp8, BF, 8192, 3840)["grid"] == 4096  # uncapped
    for op in (fused, fp8):
        assert shape(op, 32768, 4096) == (128, 4, 4)
        assert rn.plan_launch(op, BF, 65536, 4096)["grid"] == 65536 // 4
        assert rn.plan_launch(op, BF, 4096, 4096)["grid"] <= 16 * 148
    assert rn.plan_launch("rms_norm", BF, 65536, 4096)["grid"] == 16 * 148
    # rows that would take 512 threads at four vectors: eight, one row per block
    for T in (4096, 65536):
        assert shape("rms_norm", T, 16384) == (256, 8, 1)
        assert shape(fp8, T, 16384) == (256, 8, 1)
        assert shape(fused, T, 16384) == (512, 4, 1)
    # fp16: the fp8 op keeps four vectors per thread (its widening costs more)
    def shape16(op, T, H):
        p = rn.plan_launch(op, F16, T, H)
        return p["threads_per_row"], p["vectors_per_thread"], p["rows_per_cta"]
    assert shape16(fp8, 4096, 7168) == (224, 4, 2)
    assert shape16(fp8, 4096, 16384) == (512, 4, 1)
    assert shape16(fp8, 65536, 16384) == (512, 4, 1)
    assert shape16("rms_norm", 4096, 16384) == (256, 8, 1)
    assert shape16(fused, 8192, 3840) == shape(fused, 8192, 3840)
    assert shape("rms_norm", 8192, 3840) == (128, 4, 2)
    assert shape("rms_norm", 32768, 4096) == (128, 4, 2)
    assert shape("rms_norm", 32768, 2048) == (64, 4, 4)
    assert shape("rms_norm", 4096, 5120) == (160, 4, 2)  # 160-thread rows: two per block
    assert shape("rms_norm", 4096, 7168) == (224, 4, 1)
    assert shape("rms_norm", 32768, 8192) == (256, 4, 1)


def test_force_plan_hook():
    with pytest.raises(rn.RmsNormError):
        rn.force_plan(48, 4)  # not a power of two <= 32 nor a multiple of 32
    with pytest.raises(rn.RmsNormError):
        rn.force_plan(64, 9)  # width not compiled
    try:
        rn.force_plan(32, 16)
        p = rn.plan_launch("fused_add_rms_norm", BF, 100, 4096)
        assert (p["threads_per_row"], p["vectors_per_thread"]) == (32, 16)
        # a forced shape too small for the row falls back to the scalar kernel
        assert rn.plan_launch("fused_add_rms_norm", BF, 100, 8192)["kernel"] == 1
    finally:
        rn.force_plan(0, 0)
    assert rn.plan_launch("fused_add_rms_norm", BF, 100, 4096)["kernel"] == 0


def test_force_staged_hook():
    with pytest.raises(rn.RmsNormError):
        rn.force_staged(3, 4, 256)
    with pytest.raises(rn.RmsNormError):
        rn.force_staged(2, 1, 256)
    with pytest.raises(rn.RmsNormError):
        rn.force_staged(2, 4, 100)
    try:
        rn.force_staged(1, 5, 384)
        p = rn.plan_launch("fused_add_rms_norm", BF, 50, 3840)
        assert (p["kernel"], p["ctas_per_sm"], p["stages"], p["block_threads"]) == (2, 1, 5, 384)
        assert p["grid"] == 50
        # a forced ring that does not fit in shared memory is not used
        p = rn.plan_launch("fused_add_rms_norm", BF, 50, 16384 * 4)
        assert p["kernel"] != 2
    finally:
        rn.force_staged(0, 0, 0)
    assert rn.plan_launch("fused_add_rms_norm", BF, 50, 3840)["kernel"] == 0


CH_SHAPES = {"ch64_tok16": (64, 16), "ch64_tok32": (64, 32), "ch64_tok64": (64, 64),
             "ch128_tok16": (128, 16), "ch128_tok32": (128, 32), "ch128_tok64": (128, 64)}


def _tiles(name, M, N):
    ch, tok = CH_SHAPES[name]
    return -(-N // ch) * -(-M // tok)


def test_gemm_config_choice():
    """Channel-major tiles maximising the tiles of one wave; the Gemma 4 12B
    decode shapes get the configurations measured fastest."""
    cfg = rn.fp8_gemm_config
    assert cfg(1, 8192, 3840, 148) == "ch64_tok16"      # 128 tiles
    assert cfg(16, 8192, 3840, 148) == "ch64_tok16"
    assert cfg(32, 8192, 3840, 148) == "ch64_tok32"     # 128 tiles (tok16 would be 256)
    assert cfg(64, 8192, 3840, 148) == "ch64_tok64"
    assert cfg(32, 3840, 4096, 148) == "ch64_tok16"     # 120 tiles
    assert cfg(64, 3840, 15360, 148) == "ch64_tok32"    # 120 tiles
    assert cfg(1, 30720, 3840, 148) == "ch128_tok16"    # nothing fits one wave
    assert cfg(33, 30720, 3840, 148) == "ch128_tok64"
    assert cfg(256, 3840, 8192, 148) == "ch128_tok64"   # 120 tiles
    assert cfg(256, 8192, 3840, 148) == "tok128_ch128"   # 64 tiles of 128 x 256: < 1 wave
    assert cfg(8192, 8192, 3840, 148) == "tok128_ch256"
    assert cfg(256, 30720, 3840, 148) == "tok128_ch256"  # 240 tiles of 128 x 256
    assert cfg(0, 8, 16) in rn.GEMM_CONFIGS               # empty problem: any valid config
    for bad in ((-1, 8, 16), (1, 0, 16), (1, 8, 0)):
        with pytest.raises(rn.RmsNormError) as e:
            cfg(*bad)
        assert e.value.name == "RN_ERR_SHAPE"


@pytest.mark.parametrize("seed", range(3))
def test_gemm_config_choice_is_the_fullest_wave(seed):
    """Brute force over the rule's candidates on random shapes."""
    rng = np.random.default_rng(seed)
    for _ in range(300):
        M = int(rng.integers(1, 600))
        N = 8 * int(rng.integers(1, 5000))
        sms = int(rng.integers(1, 200))
        got = rn.fp8_gemm_config(M, N, 16, sms)
        fits = {c: _tiles(c, M, N) for c in CH_SHAPES if _tiles(c, M, N) <= sms}
        if fits:
            assert got in fits and fits[got] == max(fits.values()), (M, N, sms, got)
            order = list(CH_SHAPES)
            assert got == next(c for c in order if fits.get(c) == max(fits.values()))
        elif M <= 64:
            assert got == min((c for c in CH_SHAPES if c.startswith("ch128") and
                               CH_SHAPES[c][1] >= M), key=lambda c: CH_SHAPES[c][1])
        else:
            t256 = -(-M // 128) * -(-N // 256)
            assert got == ("tok128_ch256" if t256 >= sms else "tok128_ch128")


def test_gemm_force_config_hook():
    for bad in (-2, 8, 100):
        with pytest.raises(rn.RmsNormError) as e:
            rn.fp8_gemm_force_config(bad)
        assert e.value.name == "RN_ERR_CONFIG"
    try:
        for name in rn.GEMM_CONFIGS:
            rn.fp8_gemm_force_config(name)
            assert rn.fp8_gemm_config(8192, 8192, 3840) == name
            assert rn.fp8_gemm_config(1, 8, 16) == name
    finally:
        rn.fp8_gemm_force_config(None)
    assert rn.fp8_gemm_config(8192, 8192, 3840) == "tok128_ch256"


def test_status_strings():
    for code, name in rn.STATUS.items():
        assert rn.status_string(code)
    assert rn.status_string(999) == "unknown status"


def test_host_logic_from_many_threads():
    """rn_validate and rn_plan_launch from eight threads at once give the
    results of the same calls made serially (pure host logic, per-thread
    descriptor caches in the binding)."""
    import threading
    shapes = [(op, T, H) for op in ("rms_norm", "fused_add_rms_norm", "fused_add_rms_norm_fp8")
              for T in (1, 7, 4096) for H in (8, 3840, 16384, 4100)]

    def run_all():
        out = []
        for op, T, H in shapes:
            x = torch.empty(T, H, dtype=torch.bfloat16)
            o = (torch.empty(T, H, dtype=torch.float8_e4m3fn) if op.endswith("fp8")
                 else torch.empty_like(x))
            sc = torch.empty(T, dtype=torch.float32) if op.endswith("fp8") else None
            r = None if op == "rms_norm" else torch.empty_like(x)
            st, plan = rn.validate(op, o, x, residual=r, weight=torch.empty(H, dtype=torch.bfloat16),
                                   scale=sc)
            out.append((st, tuple(sorted(plan.items())),
                        tuple(sorted(rn.plan_launch(op, torch.bfloat16, T, H).items()))))
        return out

    want = run_all()
    got, errors = [None] * 8, []

    def worker(i):
        try:
            got[i] = [run_all() for _ in range(3)]
        except Exception as e:  # noqa: BLE001
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(8)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    for g in got:
        assert all(r == want for r in g)
