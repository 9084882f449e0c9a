"""Seeded synthetic inputs for the RMSNorm operators.

This module only draws random numbers and casts them to the 16-bit storage
type; it performs none of the normalisation arithmetic. Both the CPU oracle and
the CUDA library consume the very same 16-bit bit patterns produced here, so the
two sides always see identical inputs.

Distribution notation: ``N(mu, v)`` names a normal distribution with mean ``mu``
and VARIANCE ``v`` (so ``N(0, 4)`` has standard deviation 2).

Workloads (activation shapes follow the dense 2-D ``[tokens x hidden]`` layout the
AITER norm wrappers accept, "vllm.kernels.aiter_ops", ``flatten_to_2d_is_free``;
hidden 3840 is the Gemma 4 12B model width printed in the weight shapes of
"VLLM_ROCM_USE_AITER=1 slows Gemma 4 on an AMD MI300X", section "Why the fp8
Multiplies Run Slower"):

* ``small``    rms_norm, bf16, x [8 x 512] ~ N(0,1), eps 1e-6, seed 0.
* ``decode``   fused_add_rms_norm, bf16 and fp16, [T x 4096], T in {1,8,64,256},
               x ~ N(0,1), residual ~ N(0,4), eps 1e-5.
* ``outlier``  fused_add_rms_norm_fp8, bf16, [64 x 16384], x and residual ~ N(0,1)
               with the same 1 % of channels (ceil(0.01 * H) columns) scaled by 50
               in both, eps 1e-6.
* ``prefill``  fused_add_rms_norm and fused_add_rms_norm_fp8, bf16, [8192 x 3840],
               x ~ Student-t(3) clipped to +-1e3, residual ~ N(0,16), eps 1e-6.
* ``swiglu``   silu_and_mul_fp8, bf16 and fp16, x = [gate | up] of [T x 2I]
               with I = 15360 (the Gemma 4 12B intermediate size: the
               30720 x 3840 gate-up and 3840 x 15360 down projections in the
               weight-shape table of "VLLM_ROCM_USE_AITER=1 slows Gemma 4 on an
               AMD MI300X"), T in {1, 8, 64, 256, 8192}, gate, up ~ N(0,1).
* ``sweep``    all three ops, bf16 and fp16, T in {1,16,256,4096,32768,65536} x
               H in {2048,4096,5120,7168,8192,16384}, x ~ N(0,1),
               residual ~ N(0,4), eps 1e-6.
* ``tp``       the tensor-parallel fused ops (``make_tp_inputs``): W ranks'
               partial sums [W x T x H], each ~ N(0, 1/W) (their sum has the
               decode workload's N(0,1)), one residual [T x H] ~ N(0,4)
               replicated on every rank, eps 1e-5; W in {2, 4, 8}, T in
               {1, 8, 64, 256, 8192}, H 3840 (Gemma 4 12B) and 4096.

Every workload uses weight = 1 + N(0, 0.1) in the activation dtype.
"""
from __future__ import annotations

import dataclasses
import math
import zlib

import torch

__all__ = [
    "Workload",
    "cell_seed",
    "normal",
    "student_t3",
    "weight",
    "outlier_columns",
    "make_inputs",
    "DECODE_T",
    "SWEEP_T",
    "SWEEP_H",
    "SWIGLU_I",
    "SWIGLU_T",
    "TP_W",
    "TP_T",
    "to_dtype",
    "make_tp_inputs",
]

DECODE_T = (1, 8, 64, 256)
SWEEP_T = (1, 16, 256, 4096, 32768, 65536)
SWEEP_H = (2048, 4096, 5120, 7168, 8192, 16384)
SWIGLU_I = 15360
SWIGLU_T = (1, 8, 64, 256, 8192)
TP_W = (2, 4, 8)
TP_T = (1, 8, 64, 256, 8192)


def to_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp16": torch.float16}[name]


def cell_seed(*parts) -> int:
    """A stable 31-bit seed for one workload cell (CRC32 of its description)."""
    return zlib.crc32("|".join(str(p) for p in parts).encode()) & 0x7FFFFFFF


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, var: float, gen: torch.Generator, device) -> torch.Tensor:
    """fp32 samples of N(0, var) (var is the variance)."""
    z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if var != 1.0:
        z.mul_(math.sqrt(var))
    return z


def student_t3(shape, clip: float, gen: torch.Generator, device) -> torch.Tensor:
    """fp32 samples of Student-t with 3 degrees of freedom, clipped to +-clip.

    Drawn as Z / sqrt(V / 3) with Z ~ N(0,1) and V a chi-square with three
    degrees of freedom (the sum of three squared standard normals)."""
    z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    v = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(3):
        n = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        v.addcmul_(n, n)
    t = z.div_(torch.sqrt(v.div_(3.0)))
    return t.clamp_(-clip, clip)


def weight(h: int, dtype: torch.dtype, gen: torch.Generator, device) -> torch.Tensor:
    """weight = 1 + N(0, 0.1), cast to the activation dtype."""
    return (1.0 + normal((h,), 0.1, gen, device)).to(dtype)


def outlier_columns(h: int, frac: float, gen: torch.Generator, device) -> torch.Tensor:
    """ceil(frac * h) distinct column indices, drawn once per seed."""
    k = int(math.ceil(frac * h))
    return torch.randperm(h, generator=gen, device=device)[:k].sort().values


@dataclasses.dataclass
class Workload:
    """One seeded input set: x, residual (None for rms_norm) and weight."""

    name: str
    op: str
    dtype: torch.dtype
    T: int
    H: int
    eps: float
    seed: int
    x: torch.Tensor
    residual: torch.Tensor | None
    weight: torch.Tensor
    outliers: torch.Tensor | None = None


def make_inputs(name: str, op: str, dtype: str, T: int, H: int, device="cpu",
                seed: int | None = None) -> Workload:
    """Draws the inputs of one cell of a named workload on ``device``.

    The same (name, op, dtype, T, H, seed) always gives the same bits on the
    same device type. CPU and CUDA generators differ, so a test that needs the
    oracle's view of GPU-drawn inputs copies them to the host."""
    dt = to_dtype(dtype)
    device = torch.device(device)
    if seed is None:
        seed = 0 if name == "small" else cell_seed(name, op, dtype, T, H)
    g = _gen(seed, device)
    outl = None
    needs_res = op not in ("rms_norm", "silu_and_mul_fp8")
    if name == "small":
        eps = 1e-6
        x = normal((T, H), 1.0, g, device)
        r = normal((T, H), 4.0, g, device) if needs_res else None
    elif name == "decode":
        eps = 1e-5
        x = normal((T, H), 1.0, g, device)
        r = normal((T, H), 4.0, g, device) if needs_res else None
    elif name == "outlier":
        eps = 1e-6
        x = normal((T, H), 1.0, g, device)
        r = normal((T, H), 1.0, g, device) if needs_res else None
        outl = outlier_columns(H, 0.01, g, device)
        x[:, outl] *= 50.0
        if r is not None:
            r[:, outl] *= 50.0
    elif name == "prefill":
        eps = 1e-6
        x = student_t3((T, H), 1e3, g, device)
        r = normal((T, H), 16.0, g, device) if needs_res else None
    elif name == "swiglu":
        # x = [gate | up] rows of 2 * H (H is the intermediate size I);
        # gate, up ~ N(0, 1); no residual or weight
        eps = 0.0
        x = normal((T, 2 * H), 1.0, g, device)
        r = None
    elif name == "sweep":
        eps = 1e-6
        x = normal((T, H), 1.0, g, device)
        r = normal((T, H), 4.0, g, device) if needs_res else None
    else:
        raise ValueError(f"unknown workload {name!r}")
    w = weight(H, dt, g, device)
    return Workload(
        name=name, op=op, dtype=dt, T=T, H=H, eps=eps, seed=seed,
        x=x.to(dt), residual=None if r is None else r.to(dt), weight=w,
        outliers=outl,
    )


def make_tp_inputs(dtype: str, W: int, T: int, H: int, device="cpu",
                   seed: int | None = None) -> Workload:
    """Inputs of one tensor-parallel cell: ``x`` holds the W partial sums
    [W x T x H] (each ~ N(0, 1/W)), ``residual`` the replicated residual
    [T x H] ~ N(0, 4); weight 1 + N(0, 0.1); eps 1e-5."""
    dt = to_dtype(dtype)
    device = torch.device(device)
    if seed is None:
        seed = cell_seed("tp", dtype, W, T, H)
    g = _gen(seed, device)
    x = normal((W, T, H), 1.0 / W, g, device)
    r = normal((T, H), 4.0, g, device)
    w = weight(H, dt, g, device)
    return Workload(name="tp", op="allreduce_fused_add_rms_norm", dtype=dt, T=T, H=H,
                    eps=1e-5, seed=seed, x=x.to(dt), residual=r.to(dt), weight=w)
