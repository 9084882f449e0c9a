"""torch custom ops over the C ABI, eligibility predicates and a priority
dispatcher, in the manner of the AITER wrappers of "vllm.kernels.aiter_ops"
(``aiter_lib`` / ``direct_register_aiter_op``: ops kept opaque to
torch.compile; ``rms_no_var_16bit_only`` / ``rms_add_no_var_16bit_only``:
16-bit activations, weight of the same dtype or None, no variance-size
override, inputs whose flattening to 2-D is free; and the priority list that
tries each backend whose predicate holds).

Ops (namespace ``rmsnorm_b200``; CUDA only, N-D inputs flattened to
[T x H] over the last dimension, no copies):

* ``rms_norm(x, weight, epsilon) -> out``
* ``fused_add_rms_norm(x!, residual!, weight, epsilon) -> ()``: in place, as
  vLLM's fused op is used: residual := x + residual, x := rms_norm(residual)
* ``silu_and_mul_fp8(x) -> (q, scale)``: x = [gate | up] over the last dim;
  q (float8_e4m3fn, last dim halved), scale (float32, last dim 1): the fused
  SwiGLU + per-token FP8 cast
* ``fp8_rowwise_gemm(a, b, a_scale, b_scale) -> d``: bf16 [..., N] from
  e4m3 a [..., K] with per-row a_scale and an e4m3 weight b [N, K] with
  per-channel b_scale (tcgen05 tensor cores)
* ``fused_add_rms_norm_fp8(x, residual!, weight, epsilon) -> (q, scale)``:
  residual := x + residual; q (float8_e4m3fn, shape of x) and scale
  (float32, shape of x with the last dim 1) the per-token dynamic cast of
  rms_norm(residual)
* ``allreduce_fused_add_rms_norm(x, residual!, weight, epsilon, comm) -> out``
  and ``allreduce_fused_add_rms_norm_fp8(...) -> (q, scale)``: the
  tensor-parallel forms, x the local partial sum, all-reduced across the
  group of the AllReduceComm whose ``handle`` is ``comm`` before the fused op
  (with a whole group on one device, the operands carry the leading rank
  dimension)

Each has a fake (meta) implementation, so torch.compile traces through it.

The dispatcher (``rms_norm`` / ``fused_add_rms_norm`` /
``fused_add_rms_norm_fp8`` below) walks the backends registered for the
operator in priority order and runs the first whose predicate accepts the
arguments. This package registers exactly one backend, "b200" (the CUDA
kernels); inputs it does not accept raise ``IneligibleInput`` naming the
failed condition. A caller that wants another path for such inputs registers
it with ``register_backend``; this package ships none.
"""
from __future__ import annotations

from typing import Callable, NamedTuple, Optional

import torch

from . import fused_add_rms_norm as _fused
from . import fused_add_rms_norm_fp8 as _fused_fp8
from . import rms_norm as _rms
from . import fp8_rowwise_gemm as _gemm
from . import silu_and_mul_fp8 as _silu_fp8
from . import allreduce_fused_add_rms_norm as _ar
from . import allreduce_fused_add_rms_norm_fp8 as _ar_fp8
from .allreduce import lookup as _comm_lookup

__all__ = [
    "flatten_to_2d_is_free", "rms_no_var_16bit_only", "rms_add_no_var_16bit_only",
    "IneligibleInput", "register_backend", "backends", "rms_norm", "fused_add_rms_norm",
    "fused_add_rms_norm_fp8", "LIB",
]

LIB = "rmsnorm_b200"
_16BIT = (torch.float16, torch.bfloat16)


# --------------------------------------------------------------------------- predicates

def flatten_to_2d_is_free(x: torch.Tensor) -> bool:
    """Whether ``x.reshape(-1, x.shape[-1])`` is a view with dense, unit-stride
    rows: the last stride is 1 and every leading dim of size != 1 has the
    stride of a dense layout (size-1 dims may carry any stride). The rule of
    "vllm.kernels.aiter_ops" ``flatten_to_2d_is_free``, applied to 1-D and
    2-D tensors too (the kernels take dense rows only; padded 2-D rows fail)."""
    if x.dim() < 1 or x.shape[-1] == 0:
        return False
    if x.numel() == 0:
        return True
    if x.stride(-1) != 1:
        return False
    expected = x.shape[-1]
    for i in range(x.dim() - 2, -1, -1):
        if x.shape[i] != 1 and x.stride(i) != expected:
            return False
        expected *= x.shape[i]
    return True


def rms_no_var_16bit_only(x, weight, epsilon, variance_size=None) -> bool:
    """Eligibility of rms_norm ("vllm.kernels.aiter_ops", rms_no_var_16bit_only)."""
    return (variance_size is None and x.dtype in _16BIT
            and (weight is None or weight.dtype == x.dtype) and flatten_to_2d_is_free(x))


def rms_add_no_var_16bit_only(x, x_residual, weight, epsilon, variance_size=None) -> bool:
    """Eligibility of fused_add_rms_norm ("vllm.kernels.aiter_ops",
    rms_add_no_var_16bit_only)."""
    return (variance_size is None and x.dtype in _16BIT
            and (weight is None or weight.dtype == x.dtype)
            and flatten_to_2d_is_free(x) and flatten_to_2d_is_free(x_residual))


def _b200_common(x, residual, weight) -> Optional[str]:
    """Conditions the CUDA backend adds to the predicates; None if all hold."""
    ts = [t for t in (x, residual, weight) if t is not None]
    if not all(t.is_cuda for t in ts):
        return "operands must be CUDA tensors"
    if len({t.device for t in ts}) != 1:
        return "operands on different devices"
    if residual is not None and (residual.shape != x.shape or residual.dtype != x.dtype):
        return "residual must match x in shape and dtype"
    if weight is not None and (weight.dim() != 1 or weight.shape[0] != x.shape[-1]
                               or weight.stride(0) != 1):
        return "weight must be a dense [H] vector"
    return None


# --------------------------------------------------------------------------- custom ops

def _dense_like(x: torch.Tensor, dtype=None) -> torch.Tensor:
    return torch.empty(x.shape, dtype=dtype or x.dtype, device=x.device)


@torch.library.custom_op(f"{LIB}::rms_norm", mutates_args=(), device_types="cuda")
def _rms_norm_op(x: torch.Tensor, weight: Optional[torch.Tensor], epsilon: float) -> torch.Tensor:
    out = _dense_like(x)
    _rms(out, x, weight, epsilon)
    return out


@_rms_norm_op.register_fake
def _(x, weight, epsilon):
    return _dense_like(x)


@torch.library.custom_op(f"{LIB}::fused_add_rms_norm", mutates_args=("x", "residual"),
                         device_types="cuda")
def _fused_add_rms_norm_op(x: torch.Tensor, residual: torch.Tensor,
                           weight: Optional[torch.Tensor], epsilon: float) -> None:
    _fused(x, x, residual, weight, epsilon)


@_fused_add_rms_norm_op.register_fake
def _(x, residual, weight, epsilon):
    return None


@torch.library.custom_op(f"{LIB}::fused_add_rms_norm_fp8", mutates_args=("residual",),
                         device_types="cuda")
def _fused_add_rms_norm_fp8_op(x: torch.Tensor, residual: torch.Tensor,
                               weight: Optional[torch.Tensor],
                               epsilon: float) -> tuple[torch.Tensor, torch.Tensor]:
    q = _dense_like(x, torch.float8_e4m3fn)
    scale = torch.empty(x.shape[:-1] + (1,), dtype=torch.float32, device=x.device)
    _fused_fp8(q, scale, x, residual, weight, epsilon)
    return q, scale


@_fused_add_rms_norm_fp8_op.register_fake
def _(x, residual, weight, epsilon):
    return (_dense_like(x, torch.float8_e4m3fn),
            torch.empty(x.shape[:-1] + (1,), dtype=torch.float32, device=x.device))


@torch.library.custom_op(f"{LIB}::silu_and_mul_fp8", mutates_args=(), device_types="cuda")
def _silu_and_mul_fp8_op(x: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    shape = x.shape[:-1] + (x.shape[-1] // 2,)
    q = torch.empty(shape, dtype=torch.float8_e4m3fn, device=x.device)
    scale = torch.empty(x.shape[:-1] + (1,), dtype=torch.float32, device=x.device)
    _silu_fp8(q, scale, x)
    return q, scale


@_silu_and_mul_fp8_op.register_fake
def _(x):
    shape = x.shape[:-1] + (x.shape[-1] // 2,)
    return (torch.empty(shape, dtype=torch.float8_e4m3fn, device=x.device),
            torch.empty(x.shape[:-1] + (1,), dtype=torch.float32, device=x.device))


@torch.library.custom_op(f"{LIB}::fp8_rowwise_gemm", mutates_args=(), device_types="cuda")
def _fp8_rowwise_gemm_op(a: torch.Tensor, b: torch.Tensor, a_scale: torch.Tensor,
                         b_scale: torch.Tensor) -> torch.Tensor:
    d = torch.empty(a.shape[:-1] + (b.shape[0],), dtype=torch.bfloat16, device=a.device)
    _gemm(d, a, b, a_scale, b_scale)
    return d


@_fp8_rowwise_gemm_op.register_fake
def _(a, b, a_scale, b_scale):
    return torch.empty(a.shape[:-1] + (b.shape[0],), dtype=torch.bfloat16, device=a.device)


@torch.library.custom_op(f"{LIB}::allreduce_fused_add_rms_norm", mutates_args=("residual",),
                         device_types="cuda")
def _allreduce_fused_add_rms_norm_op(x: torch.Tensor, residual: torch.Tensor,
                                     weight: Optional[torch.Tensor], epsilon: float,
                                     comm: int) -> torch.Tensor:
    out = _dense_like(x)
    _ar(out, x, residual, weight, epsilon, _comm_lookup(comm))
    return out


@_allreduce_fused_add_rms_norm_op.register_fake
def _(x, residual, weight, epsilon, comm):
    return _dense_like(x)


@torch.library.custom_op(f"{LIB}::allreduce_fused_add_rms_norm_fp8", mutates_args=("residual",),
                         device_types="cuda")
def _allreduce_fused_add_rms_norm_fp8_op(x: torch.Tensor, residual: torch.Tensor,
                                         weight: Optional[torch.Tensor], epsilon: float,
                                         comm: int) -> tuple[torch.Tensor, torch.Tensor]:
    q = _dense_like(x, torch.float8_e4m3fn)
    scale = torch.empty(x.shape[:-1] + (1,), dtype=torch.float32, device=x.device)
    _ar_fp8(q, scale, x, residual, weight, epsilon, _comm_lookup(comm))
    return q, scale


@_allreduce_fused_add_rms_norm_fp8_op.register_fake
def _(x, residual, weight, epsilon, comm):
    return (_dense_like(x, torch.float8_e4m3fn),
            torch.empty(x.shape[:-1] + (1,), dtype=torch.float32, device=x.device))


# --------------------------------------------------------------------------- dispatch

class IneligibleInput(ValueError):
    """No registered backend accepts the arguments."""


class Backend(NamedTuple):
    name: str
    predicate: Callable[..., Optional[str]]  # None = accepted, else the reason
    impl: Callable


def _pred_rms(x, weight, epsilon, variance_size=None):
    if not rms_no_var_16bit_only(x, weight, epsilon, variance_size):
        return "rms_no_var_16bit_only is false"
    return _b200_common(x, None, weight)


def _pred_add(x, residual, weight, epsilon, variance_size=None):
    if not rms_add_no_var_16bit_only(x, residual, weight, epsilon, variance_size):
        return "rms_add_no_var_16bit_only is false"
    return _b200_common(x, residual, weight)


_REGISTRY: dict[str, list[Backend]] = {
    "rms_norm": [Backend("b200", _pred_rms,
                         lambda x, w, e, v=None: torch.ops.rmsnorm_b200.rms_norm(x, w, e))],
    "fused_add_rms_norm": [Backend(
        "b200", _pred_add,
        lambda x, r, w, e, v=None: torch.ops.rmsnorm_b200.fused_add_rms_norm(x, r, w, e))],
    "fused_add_rms_norm_fp8": [Backend(
        "b200", _pred_add,
        lambda x, r, w, e, v=None: torch.ops.rmsnorm_b200.fused_add_rms_norm_fp8(x, r, w, e))],
}


def register_backend(op: str, name: str, predicate: Callable[..., Optional[str]],
                     impl: Callable, priority: Optional[int] = None) -> None:
    """Adds a backend for `op` at position `priority` (default: last).
    `predicate(*args)` returns None to accept the call, else a reason."""
    lst = _REGISTRY[op]
    if any(b.name == name for b in lst):
        raise ValueError(f"backend {name!r} already registered for {op}")
    lst.insert(len(lst) if priority is None else priority, Backend(name, predicate, impl))


def unregister_backend(op: str, name: str) -> None:
    if name == "b200":
        raise ValueError("the CUDA backend cannot be removed")
    _REGISTRY[op][:] = [b for b in _REGISTRY[op] if b.name != name]


def backends(op: str) -> list[str]:
    """Backend names for `op`, highest priority first."""
    return [b.name for b in _REGISTRY[op]]


def _dispatch(op: str, *args):
    reasons = []
    for b in _REGISTRY[op]:
        why = b.predicate(*args)
        if why is None:
            return b.impl(*args)
        reasons.append(f"{b.name}: {why}")
    raise IneligibleInput(f"{op}: no backend accepts these arguments ({'; '.join(reasons)})")


def rms_norm(x, weight, epsilon, variance_size=None):
    """out = rms_norm(x) over the last dim, by the first backend that accepts it."""
    return _dispatch("rms_norm", x, weight, epsilon, variance_size)


def fused_add_rms_norm(x, residual, weight, epsilon, variance_size=None):
    """In place: residual := x + residual, x := rms_norm(residual)."""
    return _dispatch("fused_add_rms_norm", x, residual, weight, epsilon, variance_size)


def fused_add_rms_norm_fp8(x, residual, weight, epsilon, variance_size=None):
    """residual := x + residual; returns (q, scale) of rms_norm(residual)."""
    return _dispatch("fused_add_rms_norm_fp8", x, residual, weight, epsilon, variance_size)
