"""Pins that tie the CPU oracle to something other than itself.

Each ``pin_*`` takes an oracle module ``orc`` (the real one, or a deliberately
mutated copy in ``test_oracle_mutants.py``) and raises AssertionError when the
oracle disagrees with:

* closed-form hand cases (``tests/golden/hand_cases.json``);
* the exact RMS invariant of a normalised row, mean(y^2) = ms / (ms + eps);
* power-of-two scaling of the input (exact in 16-bit);
* ``torch.nn.functional.rms_norm`` in float64 (an independent library routine);
* torch's bf16 and numpy's float16 addition (the residual write-back);
* torch's / numpy's format conversions, the e4m3 -> fp16 bit reinterpretation
  from "MI210 LLM Stack - Optimizing 310B MoE Inference on 2x AMD MI210
  (gfx90a)" (insight 4), and brute-force nearest-value search (the codecs);
* properties every per-token e4m3 row must have.

Operators: "vllm.kernels.aiter_ops" (rms_no_var_16bit_only,
rms_add_no_var_16bit_only) and the fused residual + RMSNorm + FP8 pass of
"Custom CUDA kernels juice Llama 3.1 405B on AMD MI300X, skipping Nvidia
lock-in".
"""
from __future__ import annotations

import bisect
import math
from decimal import Decimal
from fractions import Fraction

import numpy as np
import torch

import synth
from tests.cmp_util import bits16, ulp16

ALL16 = np.arange(65536, dtype=np.uint32).astype(np.uint16)


def _nan16(b, dtype):
    if dtype == "bf16":
        return ((b & 0x7F80) == 0x7F80) & ((b & 0x7F) != 0)
    return ((b & 0x7C00) == 0x7C00) & ((b & 0x3FF) != 0)


def _close(got, want_strs, rel=4e-16):
    for g, w in zip(got, want_strs):
        w = float(Decimal(w))
        assert abs(g - w) <= rel * abs(w) + 1e-300, (g, w)


def _nearest_even(sorted_vals, sorted_codes, v):
    """Brute force: nearest representable value; a tie goes to the code whose
    last bit (the significand's last bit) is 0."""
    i = bisect.bisect_left(sorted_vals, v)
    cands = [j for j in (i - 1, i) if 0 <= j < len(sorted_vals)]
    best = min(abs(sorted_vals[j] - v) for j in cands)
    ties = [j for j in cands if abs(sorted_vals[j] - v) == best]
    if len(ties) == 1:
        return sorted_codes[ties[0]]
    even = [j for j in ties if (sorted_codes[j] & 1) == 0]
    assert len(even) == 1
    return sorted_codes[even[0]]


def _bits(orc, values, dtype):
    return orc.encode16(np.asarray(values, dtype=np.float64), dtype)


# ---------------------------------------------------------------- codecs

def pin_bf16_decode(orc, golden=None):
    got = orc.decode16(ALL16, "bf16")
    ref = torch.from_numpy(ALL16.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    nan = _nan16(ALL16, "bf16")
    assert np.isnan(got[nan]).all()
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def pin_f16_decode(orc, golden=None):
    got = orc.decode16(ALL16, "fp16")
    ref = ALL16.view(np.float16).astype(np.float64)
    nan = _nan16(ALL16, "fp16")
    assert np.isnan(got[nan]).all()
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def pin_e4m3_decode_bit_trick(orc, golden=None):
    # h = ((u & 0x80) << 8) | ((u & 0x7f) << 7) is an fp16 holding exactly
    # 2^-8 times the e4m3 value, for normals and subnormals alike.
    u = np.arange(256, dtype=np.uint16)
    h = ((u & 0x80) << 8) | ((u & 0x7F) << 7)
    trick = h.astype(np.uint16).view(np.float16).astype(np.float64) * 256.0
    got = orc.decode_e4m3(u.astype(np.uint8))
    nan_codes = (u & 0x7F) == 0x7F
    assert np.isnan(got[nan_codes]).all()
    np.testing.assert_array_equal(got[~nan_codes], trick[~nan_codes])
    assert np.array_equal(np.signbit(got[~nan_codes]), np.signbit(trick[~nan_codes]))
    ref = torch.from_numpy(u.astype(np.uint8)).view(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(got[~nan_codes], ref[~nan_codes])


def pin_e4m3_encode(orc, golden=None):
    u = np.arange(256, dtype=np.uint8)
    finite = (u & 0x7F) != 0x7F
    np.testing.assert_array_equal(orc.encode_e4m3(orc.decode_e4m3(u[finite])), u[finite])
    pos = u[u < 0x7F]
    pv = torch.from_numpy(pos.copy()).view(torch.float8_e4m3fn).double().numpy()
    order = np.argsort(pv)
    sv, sc = list(pv[order]), [int(c) for c in pos[order]]
    rng = np.random.default_rng(7)
    mids = [(sv[k] + sv[k + 1]) / 2 for k in range(len(sv) - 1)]
    vals = np.concatenate([rng.uniform(0, 448, 2000), 2.0 ** rng.uniform(-12, 9, 2000),
                           np.array(mids)])
    got = orc.encode_e4m3(vals)
    for v, g in zip(vals, got):
        assert int(g) == _nearest_even(sv, sc, float(v)), v
    np.testing.assert_array_equal(orc.encode_e4m3(-vals), got | 0x80)
    big = np.array([448.0, 449.0, 463.9, 464.0, 480.0, 1e6, math.inf])
    np.testing.assert_array_equal(orc.encode_e4m3(big), np.full(7, 0x7E))
    np.testing.assert_array_equal(orc.encode_e4m3(-big), np.full(7, 0xFE))
    assert orc.encode_e4m3(np.array([336.0]))[0] == 0x7A  # tie 320|352 -> 320
    assert orc.encode_e4m3(np.array([math.nan]))[0] == 0x7F
    # against torch's own cast on float32-exact, in-range values
    v = np.clip(np.concatenate([rng.normal(0, 50, 5000), rng.normal(0, 0.01, 2000)]),
                -448, 448).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(orc.encode_e4m3(v.astype(np.float64)), ref)


def pin_f16_encode(orc, golden=None):
    rng = np.random.default_rng(3)
    v = np.concatenate([
        rng.normal(0, 1, 20000), rng.normal(0, 1e-5, 5000), rng.uniform(6e4, 7e4, 2000),
        np.array([65519.99, 65520.0, 65520.01, 2.0 ** -25, 2.0 ** -25 * 1.0000001,
                  3 * 2.0 ** -26, 0.0]),
    ])
    v = np.concatenate([v, -v])
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)  # numpy rounds binary64 -> fp16 directly
    np.testing.assert_array_equal(orc.encode16(v, "fp16"), ref)
    h = orc.encode16(np.array([1 + 2 ** -11, 1 + 3 * 2 ** -11, 2.0 ** -25, 3 * 2.0 ** -25,
                               65520.0, 65519.0, -1e300]), "fp16")
    assert list(h) == [0x3C00, 0x3C02, 0x0000, 0x0002, 0x7C00, 0x7BFF, 0xFC00]


def pin_bf16_encode(orc, golden=None):
    rng = np.random.default_rng(5)
    v32 = np.concatenate([
        rng.normal(0, 1, 20000), rng.normal(0, 1e-39, 3000),
        np.array([3.3895313892515355e38, 3.39e38, 3.4028234e38]),
    ]).astype(np.float32)
    v32 = np.concatenate([v32, -v32])
    ref = torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(orc.encode16(v32.astype(np.float64), "bf16"), ref)
    b = orc.encode16(np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -30]), "bf16")
    assert list(b) == [0x3F80, 0x3F82, 0x3F81]


def pin_encode16_brute_force(orc, golden=None):
    """Doubles that are not float32-exact, against a brute-force nearest search."""
    for dtype in ("bf16", "fp16"):
        if dtype == "bf16":
            allv = torch.from_numpy(ALL16.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
        else:
            allv = ALL16.view(np.float16).astype(np.float64)
        finite = np.isfinite(allv) & (ALL16 < 0x8000)
        idx = np.argsort(allv[finite])
        sv = list(allv[finite][idx])
        sc = [int(c) for c in ALL16[finite][idx]]
        rng = np.random.default_rng(13)
        hi = 3.3e38 if dtype == "bf16" else 65000.0
        v = np.concatenate([np.exp(rng.uniform(-30, math.log(hi), 1500)),
                            rng.uniform(0.5, 4, 1000) + rng.uniform(-1e-12, 1e-12, 1000)])
        k = rng.integers(0, len(sv) - 1, 500)
        v = np.concatenate([v, (np.array(sv)[k] + np.array(sv)[k + 1]) / 2])
        got = orc.encode16(v, dtype)
        for x, g in zip(v, got):
            assert int(g) == _nearest_even(sv, sc, float(x)), (dtype, x, hex(g))


# ---------------------------------------------------------------- operators

def pin_rms_norm_hand_cases(orc, golden):
    for dtype in ("bf16", "fp16"):
        for case in golden["rms_norm"]:
            x = _bits(orc, [case["x"]], dtype)
            w = None if case["w"] is None else _bits(orc, case["w"], dtype)
            out, y = orc.rms_norm(x, w, dtype, case["eps"], want_y=True)
            _close(y[0], case["y"])
            if dtype == "bf16" and "bf16_out" in case:
                assert [int(v) for v in out[0]] == [int(s, 16) for s in case["bf16_out"]]


def pin_fused_hand_cases(orc, golden):
    for dtype in ("bf16", "fp16"):
        for case in golden["fused_add_rms_norm"]:
            if "x_bits" in case:
                if case["dtype"] != dtype:
                    continue
                x = np.array([[int(s, 16) for s in case["x_bits"]]], np.uint16)
                r = np.array([[int(s, 16) for s in case["r_bits"]]], np.uint16)
                r_out, _ = orc.fused_add_rms_norm(x, r, None, dtype, 1e-6)
                assert [int(v) for v in r_out[0]] == [int(s, 16) for s in case["r_out_bits"]]
                continue
            x = _bits(orc, [case["x"]], dtype)
            r = _bits(orc, [case["r"]], dtype)
            r_out, out, y = orc.fused_add_rms_norm(x, r, None, dtype, case["eps"], want_y=True)
            np.testing.assert_array_equal(orc.decode16(r_out, dtype)[0], case["r_out"])
            _close(y[0], case["y"])


def pin_fp8_hand_cases(orc, golden):
    for dtype in ("bf16", "fp16"):
        for case in golden["fused_add_rms_norm_fp8"]:
            x = _bits(orc, [case["x"]], dtype)
            r = _bits(orc, [case["r"]], dtype)
            w = None if case["w"] is None else _bits(orc, case["w"], dtype)
            _, q, scale = orc.fused_add_rms_norm_fp8(x, r, w, dtype, case["eps"])
            assert [int(c) for c in q[0]] == [int(s, 16) for s in case["q_bits"]]
            assert scale[0] == np.float32(float(case["scale"]))


def _rows(T, H, dtype, seed, var=1.0):
    g = torch.Generator().manual_seed(seed)
    return bits16(synth.normal((T, H), var, g, "cpu").to(synth.to_dtype(dtype)))


def pin_rms_invariant(orc, golden=None):
    """With w = 1: mean(y^2) = ms / (ms + eps), exactly in closed form."""
    for dtype in ("bf16", "fp16"):
        for eps in (0.0, 1e-6, 0.5):
            x = _rows(16, 1000, dtype, 1)
            _, y = orc.rms_norm(x, None, dtype, eps, want_y=True)
            xv = torch.from_numpy(x.view(np.int16).copy()).view(synth.to_dtype(dtype)).double().numpy()
            ms = (xv * xv).mean(axis=1)
            lhs = np.sqrt((y * y).mean(axis=1))
            rhs = np.sqrt(ms / (ms + np.float64(np.float32(eps))))
            np.testing.assert_allclose(lhs, rhs, rtol=1e-14)


def pin_power_of_two_scaling(orc, golden=None):
    for dtype in ("bf16", "fp16"):
        tdt = synth.to_dtype(dtype)
        g = torch.Generator().manual_seed(2)
        xf = synth.normal((8, 512), 1.0, g, "cpu")
        xf = torch.sign(xf) * xf.abs().clamp_min(0.01)  # keep 2^-3 x a normal number
        x = bits16(xf.to(tdt))
        w = _rows(1, 512, dtype, 3)[0]
        xv = torch.from_numpy(x.view(np.int16).copy()).view(tdt).double()
        wv = torch.from_numpy(w.view(np.int16).copy()).view(tdt).double().numpy()
        for k in (-3, 4):
            a = 2.0 ** k
            xs = bits16((xv * a).to(tdt))  # exact: power-of-two scaling of normals
            assert np.array_equal(orc.decode16(xs, dtype), xv.numpy() * a)
            np.testing.assert_array_equal(orc.rms_norm(xs, w, dtype, 0.0),
                                          orc.rms_norm(x, w, dtype, 0.0))
            eps = 1e-2
            _, y1 = orc.rms_norm(xs, w, dtype, eps, want_y=True)
            xn = xv.numpy()
            ms = (xn * xn).mean(axis=1, keepdims=True)
            expect = a * xn / np.sqrt(a * a * ms + np.float64(np.float32(eps))) * wv
            np.testing.assert_allclose(y1, expect, rtol=1e-14, atol=0)


def pin_torch_rms_norm_float64(orc, golden=None):
    for dtype in ("bf16", "fp16"):
        for with_w in (True, False):
            wl = synth.make_inputs("sweep", "rms_norm", dtype, 33, 2048)
            w = wl.weight if with_w else None
            _, y = orc.rms_norm(bits16(wl.x), None if w is None else bits16(w), dtype,
                                wl.eps, want_y=True)
            ref = torch.nn.functional.rms_norm(
                wl.x.double(), (2048,), None if w is None else w.double(),
                eps=float(np.float32(wl.eps))).numpy()
            np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-300)


def pin_residual_library_addition(orc, golden=None):
    """r' = RNE16(x + r) against torch's bf16 and numpy's float16 addition over
    bit patterns that include subnormals, ties and large exponent gaps."""
    rng = np.random.default_rng(17)
    pats = np.concatenate([rng.integers(0, 65536, 3000),
                           np.array([0x0001, 0x8001, 0x3F80, 0x3B80, 0x3F81, 0x0400, 0x7BFF])])
    pats = pats.astype(np.uint16)
    xs = np.repeat(pats, 32)
    rs = rng.choice(pats, xs.size).astype(np.uint16)
    for dtype in ("bf16", "fp16"):
        if dtype == "bf16":
            tx = torch.from_numpy(xs.view(np.int16).copy()).view(torch.bfloat16)
            tr = torch.from_numpy(rs.view(np.int16).copy()).view(torch.bfloat16)
            ok = (torch.isfinite(tx) & torch.isfinite(tr)).numpy()
            ref = (tx + tr).view(torch.int16).numpy().view(np.uint16)[ok]
        else:
            fx, fr = xs.view(np.float16), rs.view(np.float16)
            ok = np.isfinite(fx) & np.isfinite(fr)
            with np.errstate(over="ignore"):
                ref = (fx[ok] + fr[ok]).view(np.uint16)
        x2, r2 = xs[ok].reshape(1, -1), rs[ok].reshape(1, -1)
        r_out, _ = orc.fused_add_rms_norm(x2, r2, None, dtype, 1e-6)
        got = r_out[0]
        nan_ref = _nan16(ref, dtype)
        assert (_nan16(got, dtype) == nan_ref).all()
        np.testing.assert_array_equal(got[~nan_ref], ref[~nan_ref])


def pin_fused_equals_norm_of_written_back(orc, golden=None):
    for dtype in ("bf16", "fp16"):
        wl = synth.make_inputs("decode", "fused_add_rms_norm", dtype, 64, 4096)
        x, r, w = bits16(wl.x), bits16(wl.residual), bits16(wl.weight)
        r_out, out = orc.fused_add_rms_norm(x, r, w, dtype, wl.eps)
        np.testing.assert_array_equal(out, orc.rms_norm(r_out, w, dtype, wl.eps))
        # the same output computed from torch's own rounded sum
        rs = bits16(wl.x + wl.residual)
        np.testing.assert_array_equal(out, orc.rms_norm(rs, w, dtype, wl.eps))


def pin_fp8_row_properties(orc, golden=None):
    for dtype in ("bf16", "fp16"):
        wl = synth.make_inputs("outlier", "fused_add_rms_norm_fp8", dtype, 64, 16384)
        x, r, w = bits16(wl.x), bits16(wl.residual), bits16(wl.weight)
        r_out, q, scale, y = orc.fused_add_rms_norm_fp8(x, r, w, dtype, wl.eps, want_y=True)
        r2, out16 = orc.fused_add_rms_norm(x, r, w, dtype, wl.eps)
        np.testing.assert_array_equal(r_out, r2)
        # y agrees with float64 torch on the written-back residual
        tdt = synth.to_dtype(dtype)
        rt = torch.from_numpy(r_out.view(np.int16).copy()).view(tdt).double()
        yt = torch.nn.functional.rms_norm(rt, (16384,), wl.weight.double(),
                                          eps=float(np.float32(wl.eps))).numpy()
        np.testing.assert_allclose(y, yt, rtol=1e-13, atol=1e-300)
        # every non-zero row reaches the largest code and never a NaN code
        assert ((q == 0x7E) | (q == 0xFE)).any(axis=1).all()
        assert not ((q & 0x7F) == 0x7F).any()
        amax = np.abs(yt).max(axis=1)
        np.testing.assert_allclose(scale, amax / 448.0, rtol=2 ** -24)
        # dequantised codes lie within half an e4m3 step of y
        deq = torch.from_numpy(q.copy()).view(torch.float8_e4m3fn).double().numpy() \
            * (amax / 448.0)[:, None]
        half_step = np.maximum(np.abs(yt) * 2.0 ** -4, 2.0 ** -10 * (amax / 448.0)[:, None])
        assert (np.abs(deq - yt) <= half_step * (1 + 1e-9)).all()
        # the codes depend only on x*w / max|x*w|, not on eps or the rms
        _, q_eps, _ = orc.fused_add_rms_norm_fp8(x, r, w, dtype, 0.5)
        np.testing.assert_array_equal(q_eps, q)
        # the 16-bit output of the same row is RNE16(y), per torch's rounding of y
        assert ulp16(out16, bits16(torch.from_numpy(yt).to(tdt))).max() <= 1


def pin_zero_rows(orc, golden=None):
    x = np.zeros((3, 64), np.uint16)
    r_out, q, scale = orc.fused_add_rms_norm_fp8(x, x, None, "bf16", 1e-6)
    assert (q == 0).all() and (scale == 0).all() and (r_out == 0).all()
    assert (orc.rms_norm(x, None, "fp16", 1e-6) == 0).all()
    _, y = orc.rms_norm(x, None, "bf16", 0.0, want_y=True)
    assert np.isnan(y).all()  # 0/0 with eps = 0


# ---------------------------------------------------------------- SwiGLU + FP8

def _swiglu_inputs(dtype, T=16, I=512, seed=21):
    wl = synth.make_inputs("swiglu", "silu_and_mul_fp8", dtype, T, I, seed=seed)
    return wl.x


def pin_swiglu_matches_torch_silu_float64(orc, golden=None):
    """y = silu(gate) * up with gate the first half (torch.nn.functional.silu
    in float64 as the library routine)."""
    for dtype in ("bf16", "fp16"):
        x = _swiglu_inputs(dtype)
        q, scale, y = orc.silu_and_mul_fp8(bits16(x), dtype, want_y=True)
        xd = x.double()
        I = x.shape[1] // 2
        ref = (torch.nn.functional.silu(xd[:, :I]) * xd[:, I:]).numpy()
        np.testing.assert_allclose(y, ref, rtol=1e-14, atol=1e-300)
        amax = np.abs(ref).max(axis=1)
        np.testing.assert_allclose(scale, amax / 448.0, rtol=2 ** -24)


def pin_swiglu_silu_identity(orc, golden=None):
    """silu(a) - silu(-a) = a exactly in real arithmetic (sigma(-a) = 1 - sigma(a));
    with up = 1 the oracle's y must satisfy it to binary64 rounding."""
    for dtype in ("bf16", "fp16"):
        g = torch.Generator().manual_seed(5)
        a = synth.normal((4, 256), 4.0, g, "cpu").to(synth.to_dtype(dtype))
        one = torch.ones_like(a)
        xp = torch.cat([a, one], dim=1)
        xn = torch.cat([-a, one], dim=1)
        _, _, yp = orc.silu_and_mul_fp8(bits16(xp), dtype, want_y=True)
        _, _, yn = orc.silu_and_mul_fp8(bits16(xn), dtype, want_y=True)
        av = a.double().numpy()
        np.testing.assert_allclose(yp - yn, av, rtol=1e-14, atol=1e-15)
        # silu(0) = 0 and silu is positive for positive gates
        x0 = torch.cat([torch.zeros(1, 8), torch.ones(1, 8)], dim=1).to(synth.to_dtype(dtype))
        q0, s0, y0 = orc.silu_and_mul_fp8(bits16(x0), dtype, want_y=True)
        assert (y0 == 0).all() and (s0 == 0).all() and (q0 == 0).all()
        assert (yp[av > 0] > 0).all()


def pin_swiglu_fp8_row_properties(orc, golden=None):
    for dtype in ("bf16", "fp16"):
        x = _swiglu_inputs(dtype, T=32, I=1024, seed=9)
        q, scale, y = orc.silu_and_mul_fp8(bits16(x), dtype, want_y=True)
        assert ((q == 0x7E) | (q == 0xFE)).any(axis=1).all()
        assert not ((q & 0x7F) == 0x7F).any()
        deq = torch.from_numpy(q.copy()).view(torch.float8_e4m3fn).double().numpy() \
            * scale.astype(np.float64)[:, None]
        amax = np.abs(y).max(axis=1)
        half_step = np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10 * (amax / 448.0)[:, None])
        assert (np.abs(deq - y) <= half_step * (1 + 1e-6)).all()


# ---------------------------------------------------------------- fp8 row-wise GEMM

def _e4m3_codes(shape, seed, spread=4.0):
    g = torch.Generator().manual_seed(seed)
    v = synth.normal(shape, spread, g, "cpu").clamp_(-448, 448)
    return v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def pin_gemm_exact_rationals(orc, golden=None):
    """A tiny GEMM against exact rational arithmetic (brute force)."""
    from fractions import Fraction
    A = _e4m3_codes((3, 16), 1)
    B = _e4m3_codes((4, 16), 2)
    rng = np.random.default_rng(3)
    sa = rng.uniform(0.01, 2.0, 3).astype(np.float32)
    sb = rng.uniform(0.01, 2.0, 4).astype(np.float32)
    D, y = orc.fp8_rowwise_gemm(A, B, sa, sb, want_y=True)
    dec = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for m in range(3):
        for n in range(4):
            acc = sum(Fraction(dec[A[m, k]]) * Fraction(dec[B[n, k]]) for k in range(16))
            exact = acc * Fraction(float(sa[m])) * Fraction(float(sb[n]))
            assert abs(Fraction(y[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 51)
            assert D[m, n] == orc.encode16(np.array([float(exact)]), "bf16")[0]


def pin_gemm_matches_float64_matmul(orc, golden=None):
    """Library pin: numpy float64 matmul of the decoded codes (exact here)."""
    A = _e4m3_codes((24, 256), 4)
    B = _e4m3_codes((40, 256), 5)
    rng = np.random.default_rng(6)
    sa = rng.uniform(0.001, 1.0, 24).astype(np.float32)
    sb = rng.uniform(0.001, 1.0, 40).astype(np.float32)
    dec = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    ref = (dec[A] @ dec[B].T) * sa.astype(np.float64)[:, None] * sb.astype(np.float64)[None, :]
    D, y = orc.fp8_rowwise_gemm(A, B, sa, sb, want_y=True)
    np.testing.assert_array_equal(y, ref)
    np.testing.assert_array_equal(D, bits16(torch.from_numpy(ref).to(torch.bfloat16)))
    rows = np.array([0, 5, 23])
    D2, y2 = orc.fp8_rowwise_gemm(A, B, sa, sb, rows=rows, want_y=True)
    np.testing.assert_array_equal(y2, ref[rows])


# --------------------------------------------------------------------------
# All-reduce sum of tensor-parallel partials (the all-reduce that precedes the
# residual add and RMSNorm in a tensor-parallel layer; "AITER: AMD's operator
# library for ROCm", ecosystem section: all-reduce and RMSNorm for SGLang).

_FMT16 = {"bf16": (8, -126, 127), "fp16": (11, -14, 15)}  # p, emin, emax


def _exact16(q: Fraction, dtype: str) -> float:
    """Round-to-nearest-even of an exact rational onto the 16-bit format,
    from the format definition (p significand bits, gradual underflow,
    overflow to infinity past the largest finite value); returns the value."""
    p, emin, emax = _FMT16[dtype]
    if q == 0:
        return 0.0
    a = abs(q)
    E = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** E > a:
        E -= 1
    while Fraction(2) ** (E + 1) <= a:
        E += 1
    quantum = Fraction(2) ** (max(E, emin) - (p - 1))
    n = a / quantum
    fl = n.numerator // n.denominator
    frac = n - fl
    r = fl + 1 if frac > Fraction(1, 2) else fl if frac < Fraction(1, 2) else fl + (fl % 2)
    v = r * quantum
    if v > (2 - Fraction(2) ** (1 - p)) * Fraction(2) ** emax:
        return math.copysign(math.inf, q)
    return math.copysign(float(v), q)


def _lib16(values, dtype: str) -> np.ndarray:
    """Bits of exactly representable values, by numpy / torch conversion."""
    v = np.asarray(values, dtype=np.float64)
    if dtype == "fp16":
        return v.astype(np.float16).view(np.uint16)
    return bits16(torch.from_numpy(v).to(torch.bfloat16))


def _finite_codes(rng, n, dtype, lo_exp=None, hi_exp=None):
    """Random finite 16-bit codes whose exponent field spans [lo_exp, hi_exp]."""
    if dtype == "bf16":
        lo, hi = (lo_exp or 0), (hi_exp or 254)
        e = rng.integers(lo, hi + 1, n)
        m = rng.integers(0, 128, n)
        return ((rng.integers(0, 2, n) << 15) | (e << 7) | m).astype(np.uint16)
    lo, hi = (lo_exp or 0), (hi_exp or 30)
    e = rng.integers(lo, hi + 1, n)
    m = rng.integers(0, 1024, n)
    return ((rng.integers(0, 2, n) << 15) | (e << 10) | m).astype(np.uint16)


def pin_allreduce_single_rank_identity(orc, golden=None):
    """One rank: the sum is the partial itself, for every 16-bit pattern."""
    for dtype in ("bf16", "fp16"):
        got = orc.allreduce_sum16(ALL16.reshape(1, -1), dtype)
        nan = _nan16(ALL16, dtype)
        assert (_nan16(got, dtype) == nan).all()
        np.testing.assert_array_equal(got[~nan], ALL16[~nan])


def pin_allreduce_two_ranks_library_addition(orc, golden=None):
    """Two ranks: torch's bf16 and numpy's float16 addition (one operation,
    computed wider and rounded once: correctly rounded), over random patterns
    and every pairing of the special values (zeros, infinities, NaN,
    subnormal extremes, the largest finite values)."""
    rng = np.random.default_rng(71)
    for dtype in ("bf16", "fp16"):
        special = ([0x0000, 0x8000, 0x7F80, 0xFF80, 0x7FC0, 0x0001, 0x8001, 0x7F7F, 0xFF7F,
                    0x3F80, 0xBF80, 0x3B80] if dtype == "bf16" else
                   [0x0000, 0x8000, 0x7C00, 0xFC00, 0x7E00, 0x0001, 0x8001, 0x7BFF, 0xFBFF,
                    0x3C00, 0xBC00, 0x1400])
        sp = np.array(special, dtype=np.uint16)
        a = np.concatenate([rng.integers(0, 65536, 100000).astype(np.uint16), np.repeat(sp, sp.size)])
        b = np.concatenate([rng.integers(0, 65536, 100000).astype(np.uint16), np.tile(sp, sp.size)])
        if dtype == "bf16":
            ta = torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16)
            tb = torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16)
            ref = bits16(ta + tb)
        else:
            with np.errstate(over="ignore", invalid="ignore"):
                ref = (a.view(np.float16) + b.view(np.float16)).view(np.uint16)
        got = orc.allreduce_sum16(np.stack([a, b]), dtype)
        nan = _nan16(ref, dtype)
        assert (_nan16(got, dtype) == nan).all()
        np.testing.assert_array_equal(got[~nan], ref[~nan])


def pin_allreduce_exact_rationals(orc, golden=None):
    """3 to 8 ranks: the exact rational sum rounded by the format definition,
    on values spanning the whole exponent range (where binary64 summation is
    not exact) and on built rounding ties broken only by a far smaller term."""
    rng = np.random.default_rng(72)
    for dtype in ("bf16", "fp16"):
        for W in (3, 5, 8):
            parts = np.stack([_finite_codes(rng, 400, dtype) for _ in range(W)])
            vals = orc.decode16(parts, dtype)
            want = [_exact16(sum(Fraction(float(v)) for v in vals[:, i]), dtype)
                    for i in range(parts.shape[1])]
            got = orc.decode16(orc.allreduce_sum16(parts, dtype), dtype)
            nz = np.array(want) != 0
            np.testing.assert_array_equal(got[nz], np.array(want)[nz])
            np.testing.assert_array_equal(got[~nz], 0.0)
        tiny = 2.0 ** -133 if dtype == "bf16" else 2.0 ** -24
        step = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -11  # half an ulp of 1
        cases = [([1.0, step, 0.0], 1.0), ([1.0, step, tiny], 1.0 + 2 * step),
                 ([1.0, step, -tiny], 1.0), ([1.0 + 2 * step, step, 0.0], 1.0 + 4 * step),
                 ([1.0 + 2 * step, step, -tiny], 1.0 + 2 * step),
                 ([-1.0, -step, -tiny], -(1.0 + 2 * step)), ([tiny, -tiny, tiny], tiny),
                 ([4.0, -4.0, tiny], tiny)]
        parts = np.stack([_lib16([c[0][r] for c in cases], dtype) for r in range(3)])
        want = _lib16([c[1] for c in cases], dtype)
        np.testing.assert_array_equal(orc.allreduce_sum16(parts, dtype), want)


def pin_allreduce_signed_zero_and_overflow(orc, golden=None):
    for dtype in ("bf16", "fp16"):
        z, nz = 0x0000, 0x8000
        parts = np.array([[nz, nz, z, nz], [nz, z, nz, nz], [nz, nz, nz, z]], dtype=np.uint16)
        np.testing.assert_array_equal(orc.allreduce_sum16(parts, dtype), [nz, z, z, z])
        big = 0x7F7F if dtype == "bf16" else 0x7BFF
        inf = 0x7F80 if dtype == "bf16" else 0x7C00
        parts = np.array([[big, big | 0x8000], [big, big | 0x8000]], dtype=np.uint16)
        np.testing.assert_array_equal(orc.allreduce_sum16(parts, dtype), [inf, inf | 0x8000])
    # fp16: 65504 + 16 = 65520 is the midpoint to 2^16: ties to even overflow
    parts = _lib16([[65504.0, 65504.0], [16.0, 15.0]], "fp16").reshape(2, 2)
    np.testing.assert_array_equal(orc.allreduce_sum16(parts, "fp16"), [0x7C00, 0x7BFF])


def pin_allreduce_rank_order_invariance(orc, golden=None):
    """The exact sum does not depend on the order of the ranks."""
    rng = np.random.default_rng(73)
    for dtype in ("bf16", "fp16"):
        parts = np.stack([_finite_codes(rng, 20000, dtype) for _ in range(8)])
        ref = orc.allreduce_sum16(parts, dtype)
        for _ in range(3):
            perm = rng.permutation(8)
            np.testing.assert_array_equal(orc.allreduce_sum16(parts[perm], dtype), ref)


def pin_allreduce_fused_composition(orc, golden=None):
    """The tensor-parallel fused ops are the all-reduce followed by the plain
    fused ops: with one rank holding x and the others zeros, and with x split
    exactly into two halves, they reduce to fused_add_rms_norm(x, r)."""
    for dtype in ("bf16", "fp16"):
        wl = synth.make_inputs("decode", "fused_add_rms_norm", dtype, 16, 4096)
        x, r, w = bits16(wl.x), bits16(wl.residual), bits16(wl.weight)
        r_ref, out_ref = orc.fused_add_rms_norm(x, r, w, dtype, wl.eps)
        zeros = np.zeros_like(x)
        half = bits16(wl.x / 2)  # exact: scaling by a power of two (normal range)
        assert (orc.decode16(half, dtype) * 2 == orc.decode16(x, dtype)).all()
        for parts in (np.stack([zeros, x, zeros, zeros]), np.stack([half, half])):
            xs, r2, out = orc.allreduce_fused_add_rms_norm(parts, r, w, dtype, wl.eps)
            np.testing.assert_array_equal(xs, x)
            np.testing.assert_array_equal(r2, r_ref)
            np.testing.assert_array_equal(out, out_ref)
            xs, r3, q, sc = orc.allreduce_fused_add_rms_norm_fp8(parts, r, w, dtype, wl.eps)
            r4, q4, sc4 = orc.fused_add_rms_norm_fp8(x, r, w, dtype, wl.eps)
            np.testing.assert_array_equal(r3, r4)
            np.testing.assert_array_equal(q, q4)
            np.testing.assert_array_equal(sc, sc4)


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
