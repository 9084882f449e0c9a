"""Helpers for the GPU parity tests: run one operator through the C ABI and
through the CPU oracle on the same bits, and compare with the tolerances
below.

Tolerances:
* residual write-back: bit-exact (a single addition rounded once; fp32 holds
  at least 2p+2 bits of either 16-bit format, so fp32-then-round equals the
  correctly rounded sum);
* 16-bit outputs: within 1 ulp of the oracle's RNE16(y) (ordered-integer
  distance <= 1, i.e. relative 2^-8 for bf16 and 2^-11 for fp16);
* e4m3 codes: ordered code distance <= 1 everywhere and != 0 on at most 0.1 %
  of the elements; per-token scales within relative 1e-6.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import residual_add_rmsnorm_rms_b200 as rn
from tests.cmp_util import bits16, code_dist8, codes8, ulp16

FP8_MAX_MISMATCH_FRAC = 1e-3
SCALE_RTOL = 1e-6
DT = {torch.bfloat16: "bf16", torch.float16: "fp16"}
CORES = oracle.usable_cores()


def gpu_run(op, x, residual, weight, eps, out=None):
    """Runs `op` on CUDA tensors (residual is updated in place). Returns dict."""
    if op == "rms_norm":
        out = torch.empty_like(x) if out is None else out
        rn.rms_norm(out, x, weight, eps)
        return {"out": out}
    if op == "fused_add_rms_norm":
        out = torch.empty_like(x) if out is None else out
        rn.fused_add_rms_norm(out, x, residual, weight, eps)
        return {"out": out, "residual": residual}
    T = x.numel() // x.shape[-1]
    q = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    scale = torch.empty(T, dtype=torch.float32, device=x.device)
    rn.fused_add_rms_norm_fp8(q, scale, x, residual, weight, eps)
    return {"q": q, "scale": scale, "residual": residual}


def oracle_run(op, x, residual, weight, eps, dtype: str):
    """Oracle on CPU copies (any device in). Returns dict of numpy arrays."""
    H = x.shape[-1]
    xb = bits16(x).reshape(-1, H)
    wb = None if weight is None else bits16(weight)
    if op == "rms_norm":
        return {"out": oracle.rms_norm(xb, wb, dtype, eps, threads=CORES)}
    rb = bits16(residual).reshape(-1, H)
    if op == "fused_add_rms_norm":
        r_out, out = oracle.fused_add_rms_norm(xb, rb, wb, dtype, eps, threads=CORES)
        return {"out": out, "residual": r_out}
    r_out, q, scale = oracle.fused_add_rms_norm_fp8(xb, rb, wb, dtype, eps, threads=CORES)
    return {"q": q, "scale": scale, "residual": r_out}


def _nan16(b, dtype):
    if dtype == "bf16":
        return ((b & 0x7F80) == 0x7F80) & ((b & 0x7F) != 0)
    return ((b & 0x7C00) == 0x7C00) & ((b & 0x3FF) != 0)


def compare(op, got: dict, want: dict, dtype: str, rows=None) -> dict:
    """Asserts the tolerances; `rows` selects the oracle-computed rows of a
    sampled comparison (got holds all rows). Returns summary statistics."""
    stats = {}

    def sel(a):
        a = a.reshape(-1, a.shape[-1]) if a.ndim > 1 else a
        return a if rows is None else a[rows]

    if "residual" in want:
        g = sel(bits16(got["residual"]).reshape(-1, want["residual"].shape[-1]))
        w = want["residual"]
        bad = np.count_nonzero(g != w)
        assert bad == 0, f"residual write-back differs in {bad} elements"
        stats["residual_mismatch"] = 0
    if "out" in want:
        g = sel(bits16(got["out"]).reshape(-1, want["out"].shape[-1]))
        w = want["out"]
        nan_g, nan_w = _nan16(g, dtype), _nan16(w, dtype)
        assert np.array_equal(nan_g, nan_w), "NaN positions differ"
        d = ulp16(g[~nan_w], w[~nan_w])
        stats["out_max_ulp"] = int(d.max()) if d.size else 0
        stats["out_frac_1ulp"] = float(np.count_nonzero(d)) / max(d.size, 1)
        assert stats["out_max_ulp"] <= 1, f"16-bit output off by {stats['out_max_ulp']} ulp"
    if "q" in want:
        g = sel(codes8(got["q"]).reshape(-1, want["q"].shape[-1]))
        w = want["q"]
        assert not ((g & 0x7F) == 0x7F).any(), "NaN code produced"
        d = code_dist8(g, w)
        stats["q_max_code"] = int(d.max()) if d.size else 0
        stats["q_frac_diff"] = float(np.count_nonzero(d)) / max(d.size, 1)
        assert stats["q_max_code"] <= 1, f"fp8 code off by {stats['q_max_code']}"
        assert stats["q_frac_diff"] <= FP8_MAX_MISMATCH_FRAC, f"fp8 mismatch {stats['q_frac_diff']}"
        gs = got["scale"].detach().cpu().numpy().reshape(-1)
        gs = gs if rows is None else gs[rows]
        ws = want["scale"].astype(np.float64)
        err = np.abs(gs.astype(np.float64) - ws)
        ok = err <= SCALE_RTOL * np.abs(ws)
        stats["scale_max_rel"] = float(np.max(err / np.where(ws == 0, 1, np.abs(ws)))) if ws.size else 0.0
        assert ok.all(), f"scale off: max rel {stats['scale_max_rel']}"
    return stats


def sample_rows(T: int, k: int = 256, seed: int = 0) -> np.ndarray:
    """All rows when T <= k, else the first, last, evenly spaced and random rows."""
    if T <= k:
        return np.arange(T)
    rng = np.random.default_rng(seed)
    picks = np.concatenate([[0, T - 1], np.linspace(0, T - 1, k // 2).astype(np.int64),
                            rng.integers(0, T, k // 2 - 2)])
    return np.unique(picks)
