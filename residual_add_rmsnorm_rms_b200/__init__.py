"""B200 (sm_100a) RMSNorm library: rms_norm, fused_add_rms_norm and
fused_add_rms_norm_fp8 over dense 16-bit activations.

This module is a thin ctypes binding over the C ABI declared in
``include/rmsnorm_b200.h`` (``librmsnorm_b200.so``, built in-tree by
``python residual_add_rmsnorm_rms_b200/build.py``). It only marshals torch
tensors into ``rn_tensor`` descriptors and passes the current CUDA stream;
every step of the computation runs in the library's CUDA kernels. There is no
CPU or PyTorch fallback: if the shared library is missing, importing this
package raises.

Operators as wrapped in "vllm.kernels.aiter_ops" (rms_no_var_16bit_only,
rms_add_no_var_16bit_only, flatten_to_2d_is_free); the fp8 variant is the
residual + RMSNorm + FP8 single pass of "Custom CUDA kernels juice Llama 3.1
405B on AMD MI300X, skipping Nvidia lock-in".
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "RmsNormError", "rms_norm", "fused_add_rms_norm", "fused_add_rms_norm_fp8",
    "silu_and_mul_fp8", "fp8_rowwise_gemm", "fp8_gemm_config", "fp8_gemm_force_config",
    "GEMM_CONFIGS", "allreduce_fused_add_rms_norm", "allreduce_fused_add_rms_norm_fp8",
    "allreduce_fused_add_rms_norm_local",
    "host_rms_norm", "host_fused_add_rms_norm", "host_fused_add_rms_norm_fp8",
    "host_plan_chunks", "RnHostPipeline", "RnHostPlan", "HOST_MAX_STREAMS",
    "RnAllreduceComm", "ALLREDUCE_MAX_WORLD", "ALLREDUCE_SIGNAL_BYTES", "ALLREDUCE_ALGORITHMS",
    "plan_launch", "validate", "force_plan", "force_staged",
    "set_launch_options", "set_prefetch", "device_errors", "supported_vectors_per_thread",
    "status_string", "kernel_binary_version", "MAX_DIMS", "LOCAL_EXCHANGE_BYTES",
    "LIB_PATH", "lib", "RnTensor", "RnPlan", "STATUS", "OPS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librmsnorm_b200.so")

STATUS = {
    0: "RN_OK", 1: "RN_ERR_NULL", 2: "RN_ERR_DTYPE", 3: "RN_ERR_WEIGHT_DTYPE", 4: "RN_ERR_SHAPE",
    5: "RN_ERR_LAYOUT", 6: "RN_ERR_ALIAS", 7: "RN_ERR_VARIANCE_SIZE", 8: "RN_ERR_EPS",
    9: "RN_ERR_CUDA", 10: "RN_ERR_CONFIG", 11: "RN_ERR_COMM", 12: "RN_ERR_CAPACITY",
}
HOST_MAX_STREAMS = 8
OPS = {"rms_norm": 0, "fused_add_rms_norm": 1, "fused_add_rms_norm_fp8": 2}
PLAN_OPS = dict(OPS, silu_and_mul_fp8=3)
_DTYPES = {torch.float16: 0, torch.bfloat16: 1, torch.float8_e4m3fn: 2, torch.float32: 3,
           torch.uint8: 2}


# Restated from include/rmsnorm_b200.h (a CPU test checks they agree).
MAX_DIMS = 8
LOCAL_EXCHANGE_BYTES = 33554432
ALLREDUCE_MAX_WORLD = 8
ALLREDUCE_SIGNAL_BYTES = 131136
ALLREDUCE_ALGORITHMS = {"auto": 0, "one_shot": 1, "two_shot": 2}


class RnAllreduceComm(ctypes.Structure):
    """rn_allreduce_comm (include/rmsnorm_b200.h)."""
    _fields_ = [
        ("world", ctypes.c_int32),
        ("rank", ctypes.c_int32),
        ("local_ranks", ctypes.c_int32),
        ("algorithm", ctypes.c_int32),
        ("buffers", ctypes.c_void_p * ALLREDUCE_MAX_WORLD),
        ("signals", ctypes.c_void_p * ALLREDUCE_MAX_WORLD),
        ("buffer_bytes", ctypes.c_int64),
        ("timeout_ns", ctypes.c_int64),
    ]


class RnHostPipeline(ctypes.Structure):
    """rn_host_pipeline (include/rmsnorm_b200.h)."""
    _fields_ = [
        ("scratch", ctypes.c_void_p),
        ("scratch_bytes", ctypes.c_int64),
        ("streams", ctypes.POINTER(ctypes.c_void_p)),
        ("n_streams", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("chunk_rows", ctypes.c_int64),
    ]


class RnHostPlan(ctypes.Structure):
    """rn_host_plan (include/rmsnorm_b200.h)."""
    _fields_ = [
        ("chunk_rows", ctypes.c_int64),
        ("chunks", ctypes.c_int64),
        ("slot_bytes", ctypes.c_int64),
        ("slots", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_ if k != "reserved"}


class RnTensor(ctypes.Structure):
    _fields_ = [
        ("data", ctypes.c_void_p),
        ("dtype", ctypes.c_int32),
        ("ndim", ctypes.c_int32),
        ("sizes", ctypes.POINTER(ctypes.c_int64)),
        ("strides", ctypes.POINTER(ctypes.c_int64)),
    ]


class RnPlan(ctypes.Structure):
    _fields_ = [
        ("kernel", ctypes.c_int32),
        ("threads_per_row", ctypes.c_int32),
        ("vectors_per_thread", ctypes.c_int32),
        ("rows_per_cta", ctypes.c_int32),
        ("block_threads", ctypes.c_int32),
        ("smem_bytes", ctypes.c_int32),
        ("stages", ctypes.c_int32),
        ("ctas_per_sm", ctypes.c_int32),
        ("grid", ctypes.c_int64),
    ]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


class RmsNormError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"{what}: {self.name} ({status_string(status)})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python residual_add_rmsnorm_rms_b200/build.py` "
            "(this package has no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(RnTensor)
    F, I64, VP = ctypes.c_float, ctypes.c_int64, ctypes.c_void_p
    L.rn_rms_norm.argtypes = [P, P, P, F, I64, VP]
    L.rn_fused_add_rms_norm.argtypes = [P, P, P, P, F, I64, VP]
    L.rn_fused_add_rms_norm_fp8.argtypes = [P, P, P, P, P, F, I64, VP]
    for f in (L.rn_rms_norm, L.rn_fused_add_rms_norm, L.rn_fused_add_rms_norm_fp8):
        f.restype = ctypes.c_int
    L.rn_silu_and_mul_fp8.argtypes = [P, P, P, VP]
    L.rn_silu_and_mul_fp8.restype = ctypes.c_int
    L.rn_fp8_rowwise_gemm.argtypes = [P, P, P, P, P, VP]
    L.rn_fp8_rowwise_gemm.restype = ctypes.c_int
    C = ctypes.POINTER(RnAllreduceComm)
    L.rn_allreduce_fused_add_rms_norm.argtypes = [P, P, P, P, F, C, VP]
    L.rn_allreduce_fused_add_rms_norm_fp8.argtypes = [P, P, P, P, P, F, C, VP]
    L.rn_allreduce_fused_add_rms_norm.restype = ctypes.c_int
    L.rn_allreduce_fused_add_rms_norm_local.argtypes = [P, P, P, P, F, ctypes.c_int32, VP]
    L.rn_allreduce_fused_add_rms_norm_local.restype = ctypes.c_int
    L.rn_allreduce_fused_add_rms_norm_fp8.restype = ctypes.c_int
    HP = ctypes.POINTER(RnHostPipeline)
    L.rn_host_rms_norm.argtypes = [P, P, P, F, I64, HP]
    L.rn_host_fused_add_rms_norm.argtypes = [P, P, P, P, F, I64, HP]
    L.rn_host_fused_add_rms_norm_fp8.argtypes = [P, P, P, P, P, F, I64, HP]
    for f in (L.rn_host_rms_norm, L.rn_host_fused_add_rms_norm, L.rn_host_fused_add_rms_norm_fp8):
        f.restype = ctypes.c_int
    L.rn_host_plan_chunks.argtypes = [ctypes.c_int32, I64, I64, I64, ctypes.c_int32, I64,
                                      ctypes.POINTER(RnHostPlan)]
    L.rn_host_plan_chunks.restype = ctypes.c_int
    L.rn_fp8_gemm_config.argtypes = [I64, I64, I64, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)]
    L.rn_fp8_gemm_config.restype = ctypes.c_int
    L.rn_fp8_gemm_force_config.argtypes = [ctypes.c_int32]
    L.rn_fp8_gemm_force_config.restype = ctypes.c_int
    L.rn_status_string.argtypes = [ctypes.c_int]
    L.rn_status_string.restype = ctypes.c_char_p
    L.rn_last_cuda_error.argtypes = []
    L.rn_last_cuda_error.restype = ctypes.c_char_p
    L.rn_plan_launch.argtypes = [ctypes.c_int32, ctypes.c_int32, I64, I64, ctypes.c_int32,
                                 ctypes.POINTER(RnPlan)]
    L.rn_plan_launch.restype = ctypes.c_int
    L.rn_validate.argtypes = [ctypes.c_int32, P, P, P, P, P, F, I64, ctypes.POINTER(RnPlan)]
    L.rn_validate.restype = ctypes.c_int
    L.rn_force_plan.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
    L.rn_force_plan.restype = ctypes.c_int
    L.rn_force_staged.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
    L.rn_force_staged.restype = ctypes.c_int
    L.rn_set_launch_options.argtypes = [ctypes.c_int32, ctypes.c_int64]
    L.rn_set_launch_options.restype = ctypes.c_int
    L.rn_kernel_binary_version.argtypes = [ctypes.POINTER(ctypes.c_int32)]
    L.rn_kernel_binary_version.restype = ctypes.c_int
    L.rn_set_prefetch.argtypes = [ctypes.c_int32]
    L.rn_set_prefetch.restype = ctypes.c_int
    L.rn_device_errors.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
    L.rn_device_errors.restype = ctypes.c_int
    L.rn_supported_vectors_per_thread.argtypes = [ctypes.POINTER(ctypes.c_int32), ctypes.c_int32]
    L.rn_supported_vectors_per_thread.restype = ctypes.c_int32
    L.rn_version.argtypes = []
    L.rn_version.restype = ctypes.c_char_p
    return L


lib = _load()


def status_string(status: int) -> str:
    return lib.rn_status_string(int(status)).decode()


def describe(t: torch.Tensor | None):
    """(RnTensor, keepalive) for a tensor; (None, None) for None. Builds fresh
    ctypes arrays (used by validate(); the operator calls use _desc)."""
    if t is None:
        return None, None
    n = t.dim()
    sizes = (ctypes.c_int64 * max(n, 1))(*t.shape)
    strides = (ctypes.c_int64 * max(n, 1))(*t.stride())
    dt = _DTYPES.get(t.dtype, -1)
    d = RnTensor(t.data_ptr() if t.numel() else 0, dt, n, sizes, strides)
    return d, (sizes, strides)


_tls = threading.local()
_CACHE_MAX = 256


def _desc(t: torch.Tensor, slot: int):
    """A by-reference rn_tensor for `t`. Descriptors are cached per thread,
    argument slot and (dtype, shape, strides), and only the data pointer is
    rewritten per call: marshalling stays cheap next to a kernel launch."""
    cache = getattr(_tls, "cache", None)
    if cache is None:
        cache = _tls.cache = {}
    key = (slot, t.dtype, t.shape, t.stride())
    ent = cache.get(key)
    if ent is None:
        if len(cache) >= _CACHE_MAX:
            cache.clear()
        d, keep = describe(t)
        ent = cache[key] = (d, keep, ctypes.byref(d))
    ent[0].data = t.data_ptr() if t.numel() else 0
    return ent[2]


def _ref(d):
    return None if d is None else ctypes.byref(d)


def _vs(variance_size) -> int:
    return -1 if variance_size is None else int(variance_size)


# The raw handle of torch's current stream and the current device index,
# without building Python stream objects (about 1 us a call less); the public
# calls where this torch lacks them.
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)
_cur_device = getattr(torch._C, "_cuda_getDevice", None)


def _stream_for(tensors, stream):
    """The device index shared by all tensors and the raw stream handle."""
    dev = -2
    for t in tensors:
        if t is None:
            continue
        d = t.get_device()
        if d < 0:
            raise ValueError("all operands must be CUDA tensors (the library takes device pointers)")
        if dev == -2:
            dev = d
        elif d != dev:
            raise ValueError("operands are on different devices")
    if stream is None:
        if _raw_stream is not None:
            return dev, _raw_stream(dev)
        stream = torch.cuda.current_stream(dev)
    return dev, (stream.cuda_stream if hasattr(stream, "cuda_stream") else stream)


def _call(fn, dev: int, *args):
    if (_cur_device() if _cur_device is not None else torch.cuda.current_device()) == dev:
        return fn(*args)
    with torch.cuda.device(dev):
        return fn(*args)


def _check(status: int, what: str):
    if status != 0:
        err = RmsNormError(status, what)
        if status == 9:
            err.args = (err.args[0] + ": " + lib.rn_last_cuda_error().decode(),)
        raise err


def rms_norm(out: torch.Tensor, x: torch.Tensor, weight: torch.Tensor | None, eps: float,
             variance_size=None, stream=None) -> None:
    """out = x / sqrt(mean(x^2) + eps) * weight over the last dim (C ABI rn_rms_norm)."""
    dev, s = _stream_for((out, x, weight), stream)
    st = _call(lib.rn_rms_norm, dev, _desc(out, 0), _desc(x, 1),
               None if weight is None else _desc(weight, 2), eps, _vs(variance_size), s)
    _check(st, "rn_rms_norm")


def fused_add_rms_norm(out: torch.Tensor, x: torch.Tensor, residual: torch.Tensor,
                       weight: torch.Tensor | None, eps: float, variance_size=None,
                       stream=None) -> None:
    """residual += x (rounded, in place); out = rms_norm(residual) (C ABI rn_fused_add_rms_norm)."""
    dev, s = _stream_for((out, x, residual, weight), stream)
    st = _call(lib.rn_fused_add_rms_norm, dev, _desc(out, 0), _desc(x, 1), _desc(residual, 2),
               None if weight is None else _desc(weight, 3), eps, _vs(variance_size), s)
    _check(st, "rn_fused_add_rms_norm")


def fused_add_rms_norm_fp8(q: torch.Tensor, scale: torch.Tensor, x: torch.Tensor,
                           residual: torch.Tensor, weight: torch.Tensor | None, eps: float,
                           variance_size=None, stream=None) -> None:
    """residual += x (in place); q, scale = per-token e4m3 cast of rms_norm(residual)
    (C ABI rn_fused_add_rms_norm_fp8). q: float8_e4m3fn (or uint8) [T, H]; scale: float32 [T]."""
    dev, s = _stream_for((q, scale, x, residual, weight), stream)
    st = _call(lib.rn_fused_add_rms_norm_fp8, dev, _desc(q, 0), _desc(scale, 1), _desc(x, 2),
               _desc(residual, 3), None if weight is None else _desc(weight, 4), eps,
               _vs(variance_size), s)
    _check(st, "rn_fused_add_rms_norm_fp8")


def silu_and_mul_fp8(q: torch.Tensor, scale: torch.Tensor, x: torch.Tensor, stream=None) -> None:
    """Fused SwiGLU + per-token e4m3 cast (C ABI rn_silu_and_mul_fp8): x = [gate | up]
    ([..., 2I]); q (float8_e4m3fn or uint8, [..., I]); scale (float32, T values)."""
    dev, s = _stream_for((q, scale, x), stream)
    st = _call(lib.rn_silu_and_mul_fp8, dev, _desc(q, 0), _desc(scale, 1), _desc(x, 2), s)
    _check(st, "rn_silu_and_mul_fp8")


def fp8_rowwise_gemm(d: torch.Tensor, a: torch.Tensor, b: torch.Tensor, a_scale: torch.Tensor,
                     b_scale: torch.Tensor, stream=None) -> None:
    """D = bf16(b_scale[n] * a_scale[m] * (A @ B^T)) on the tensor cores (C ABI
    rn_fp8_rowwise_gemm). a: [M, K] e4m3, b: [N, K] e4m3, scales fp32, d: [M, N] bf16."""
    dev, s = _stream_for((d, a, b, a_scale, b_scale), stream)
    st = _call(lib.rn_fp8_rowwise_gemm, dev, _desc(d, 0), _desc(a, 1), _desc(b, 2),
               _desc(a_scale, 3), _desc(b_scale, 4), s)
    _check(st, "rn_fp8_rowwise_gemm")


def allreduce_fused_add_rms_norm(out: torch.Tensor, x: torch.Tensor, residual: torch.Tensor,
                                 weight: torch.Tensor | None, eps: float, comm,
                                 stream=None) -> None:
    """Tensor-parallel all-reduce of the partials x across the group of
    `comm` (an ``allreduce.AllReduceComm``), then the fused residual add and
    RMSNorm (C ABI rn_allreduce_fused_add_rms_norm). With comm.local_ranks > 1
    the operands carry a leading rank dimension."""
    dev, s = _stream_for((out, x, residual, weight), stream)
    st = _call(lib.rn_allreduce_fused_add_rms_norm, dev, _desc(out, 0), _desc(x, 1),
               _desc(residual, 2), None if weight is None else _desc(weight, 3), eps,
               comm.descriptor_ref(), s)
    _check(st, "rn_allreduce_fused_add_rms_norm")


def allreduce_fused_add_rms_norm_fp8(q: torch.Tensor, scale: torch.Tensor, x: torch.Tensor,
                                     residual: torch.Tensor, weight: torch.Tensor | None,
                                     eps: float, comm, stream=None) -> None:
    """As allreduce_fused_add_rms_norm, with the per-token e4m3 output of
    fused_add_rms_norm_fp8 (C ABI rn_allreduce_fused_add_rms_norm_fp8)."""
    dev, s = _stream_for((q, scale, x, residual, weight), stream)
    st = _call(lib.rn_allreduce_fused_add_rms_norm_fp8, dev, _desc(q, 0), _desc(scale, 1),
               _desc(x, 2), _desc(residual, 3), None if weight is None else _desc(weight, 4),
               eps, comm.descriptor_ref(), s)
    _check(st, "rn_allreduce_fused_add_rms_norm_fp8")


def allreduce_fused_add_rms_norm_local(out: torch.Tensor, x: torch.Tensor,
                                       residual: torch.Tensor, weight: torch.Tensor | None,
                                       eps: float, world: int, stream=None) -> None:
    """A whole group of `world` ranks on one device (operands [world, T, H])
    with the library's own static exchange memory: allocates nothing (C ABI
    rn_allreduce_fused_add_rms_norm_local). Calls sharing a device must not
    overlap in time; the first call, and the first after a change of
    `world`, must be made outside CUDA-graph capture."""
    dev, s = _stream_for((out, x, residual, weight), stream)
    st = _call(lib.rn_allreduce_fused_add_rms_norm_local, dev, _desc(out, 0), _desc(x, 1),
               _desc(residual, 2), None if weight is None else _desc(weight, 3), eps,
               int(world), s)
    _check(st, "rn_allreduce_fused_add_rms_norm_local")


def host_plan_chunks(op: str, T: int, H: int, scratch_bytes: int, n_streams: int,
                     chunk_rows: int = 0) -> dict:
    """The chunking of a host-memory call (C ABI rn_host_plan_chunks; host logic)."""
    p = RnHostPlan()
    _check(lib.rn_host_plan_chunks(OPS[op], T, H, scratch_bytes, n_streams, chunk_rows,
                                   ctypes.byref(p)), "rn_host_plan_chunks")
    return p.as_dict()


def _host_call(fn, name, pipeline, tensors, weight, args, join):
    """Validates that the activations are CPU tensors and the weight lives on
    the pipeline's device, then enqueues through the pipeline's streams."""
    for t in tensors:
        if t.is_cuda:
            raise ValueError(f"{name}: activations must be host (CPU) tensors")
    if weight is not None and weight.get_device() != pipeline.device:
        raise ValueError(f"{name}: the weight must be on the pipeline's device")
    with torch.cuda.device(pipeline.device):
        pipeline.begin(args[0], join)
        st = fn(*args[1:], pipeline.descriptor_ref())
        pipeline.end(join)
    _check(st, name)


def host_rms_norm(out: torch.Tensor, x: torch.Tensor, weight: torch.Tensor | None, eps: float,
                  pipeline, variance_size=None, join: bool = True) -> None:
    """rms_norm on host-memory activations through `pipeline` (a
    ``host.HostPipeline``): chunked copy in, kernel, copy out (C ABI
    rn_host_rms_norm). With join, the pipeline's streams start after the
    current stream's work and the current stream waits for them."""
    _host_call(lib.rn_host_rms_norm, "rn_host_rms_norm", pipeline, (out, x), weight,
               (("rms_norm", x.shape[-1] if x.dim() else 0), _desc(out, 0), _desc(x, 1),
                None if weight is None else _desc(weight, 2), eps, _vs(variance_size)), join)


def host_fused_add_rms_norm(out: torch.Tensor, x: torch.Tensor, residual: torch.Tensor,
                            weight: torch.Tensor | None, eps: float, pipeline,
                            variance_size=None, join: bool = True) -> None:
    """fused_add_rms_norm on host-memory activations (C ABI
    rn_host_fused_add_rms_norm); residual is updated in host memory."""
    _host_call(lib.rn_host_fused_add_rms_norm, "rn_host_fused_add_rms_norm", pipeline,
               (out, x, residual), weight,
               (("fused_add_rms_norm", x.shape[-1] if x.dim() else 0), _desc(out, 0),
                _desc(x, 1), _desc(residual, 2), None if weight is None else _desc(weight, 3),
                eps, _vs(variance_size)), join)


def host_fused_add_rms_norm_fp8(q: torch.Tensor, scale: torch.Tensor, x: torch.Tensor,
                                residual: torch.Tensor, weight: torch.Tensor | None, eps: float,
                                pipeline, variance_size=None, join: bool = True) -> None:
    """fused_add_rms_norm_fp8 on host-memory activations (C ABI
    rn_host_fused_add_rms_norm_fp8); q and scale are written in host memory."""
    _host_call(lib.rn_host_fused_add_rms_norm_fp8, "rn_host_fused_add_rms_norm_fp8", pipeline,
               (q, scale, x, residual), weight,
               (("fused_add_rms_norm_fp8", x.shape[-1] if x.dim() else 0), _desc(q, 0),
                _desc(scale, 1), _desc(x, 2), _desc(residual, 3),
                None if weight is None else _desc(weight, 4), eps, _vs(variance_size)), join)


# rn_gemm_config values: TOK = token-major (tokens x channels) tiles, CH =
# channel-major (channels x tokens) tiles computing D^T.
GEMM_CONFIGS = {"tok128_ch128": 0, "ch128_tok16": 1, "ch128_tok32": 2, "ch128_tok64": 3,
                "ch64_tok16": 4, "ch64_tok32": 5, "ch64_tok64": 6, "tok128_ch256": 7}


def fp8_gemm_config(M: int, N: int, K: int, num_sms: int = 0) -> str:
    """Name of the tile configuration rn_fp8_rowwise_gemm uses (host logic)."""
    c = ctypes.c_int32(-1)
    _check(lib.rn_fp8_gemm_config(M, N, K, num_sms, ctypes.byref(c)), "rn_fp8_gemm_config")
    return {v: k for k, v in GEMM_CONFIGS.items()}[c.value]


def fp8_gemm_force_config(config) -> None:
    """Test/tuning hook: force a GEMM tile configuration (name or id); None or
    -1 restores the automatic choice."""
    cid = -1 if config is None else (GEMM_CONFIGS[config] if isinstance(config, str) else config)
    _check(lib.rn_fp8_gemm_force_config(cid), "rn_fp8_gemm_force_config")


def plan_launch(op: str, dtype: torch.dtype, T: int, H: int, vector_ok: bool = True) -> dict:
    """The launch shape the library picks (pure host logic; no GPU needed)."""
    p = RnPlan()
    st = lib.rn_plan_launch(PLAN_OPS[op], _DTYPES[dtype], T, H, int(vector_ok), ctypes.byref(p))
    _check(st, "rn_plan_launch")
    return p.as_dict()


def validate(op: str, out_or_q, x, residual=None, weight=None, eps: float = 1e-6,
             variance_size=None, scale=None):
    """Dry run of an entry point on tensor METADATA (no memory is touched, no
    CUDA call): returns (status_name, plan dict). Works for CPU tensors too."""
    keep = []
    descs = []
    for t in (out_or_q, scale, x, residual, weight):
        d, k = describe(t)
        keep.append(k)
        descs.append(d)
    p = RnPlan()
    st = lib.rn_validate(OPS[op], *[_ref(d) for d in descs], eps, _vs(variance_size),
                         ctypes.byref(p))
    return STATUS.get(st, str(st)), p.as_dict()


def force_plan(threads_per_row: int, vectors_per_thread: int, rows_per_cta: int = 0) -> None:
    """Test/tuning hook: force the vector kernel's shape; (0, 0) restores auto."""
    _check(lib.rn_force_plan(threads_per_row, vectors_per_thread, rows_per_cta), "rn_force_plan")


def force_staged(ctas_per_sm: int, stages: int, threads: int) -> None:
    """Test/tuning hook: force the staged kernel's shape; (0, 0, 0) restores auto."""
    _check(lib.rn_force_staged(ctas_per_sm, stages, threads), "rn_force_staged")


def set_launch_options(pdl: int = -1, max_grid: int = 0) -> None:
    """Tuning hook: pdl 1/0/-1 (on/off/default) and a cap on blocks launched
    (0 = the library's default cap)."""
    _check(lib.rn_set_launch_options(pdl, max_grid), "rn_set_launch_options")


def set_prefetch(mode: int = -1) -> None:
    """Tuning hook: L2 prefetch of the first rows before waiting for the
    previous kernel (1 on, 0 off, -1 library default)."""
    _check(lib.rn_set_prefetch(mode), "rn_set_prefetch")


def kernel_binary_version() -> int:
    """Compute capability the loaded device code was built for (100 = sm_100a)."""
    v = ctypes.c_int32(0)
    _check(lib.rn_kernel_binary_version(ctypes.byref(v)), "rn_kernel_binary_version")
    return int(v.value)


def device_errors() -> int:
    """Reads and clears the current device's kernel error flags (0 = none)."""
    v = ctypes.c_uint32(0)
    _check(lib.rn_device_errors(ctypes.byref(v)), "rn_device_errors")
    return int(v.value)


def supported_vectors_per_thread() -> list[int]:
    buf = (ctypes.c_int32 * 64)()
    n = lib.rn_supported_vectors_per_thread(buf, 64)
    return list(buf[:n])
