"""Python handle on the fp64 CPU oracle (``rmsnorm_oracle.c``).

TEST INFRASTRUCTURE ONLY. The tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg are the only users. The CUDA library
and its binding never import this package, and this package imports nothing
from them.

The oracle is a plain C loop in IEEE binary64, compiled with
``-O2 -ffp-contract=off`` (no FMA contraction, no fast-math). Inputs and outputs
are raw 16-bit bit patterns (uint16), e4m3fn codes (uint8) and fp32 scales, so
the oracle never depends on how a library rounds. What each function computes
is stated in the C file's header.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
(closed-form hand cases, invariants, independent library codecs and
``torch.nn.functional.rms_norm`` in float64); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rmsnorm_oracle.c")
_LIB = os.path.join(_HERE, "librmsnorm_oracle.so")
_lock = threading.Lock()
_lib = None

DTYPES = {"fp16": 0, "bf16": 1}
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    """Compiles the oracle with gcc (rebuilds when the source is newer)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        F = ctypes.c_float
        lib.oracle_rms_norm.argtypes = [P, P, I, I64, I64, F, P, P, P, P]
        lib.oracle_fused_add_rms_norm.argtypes = [P, P, P, I, I64, I64, F, P, P, P, P, P]
        lib.oracle_fused_add_rms_norm_fp8.argtypes = [P, P, P, I, I64, I64, F, P, P, P, P, P, P]
        for f in (lib.oracle_rms_norm, lib.oracle_fused_add_rms_norm,
                  lib.oracle_fused_add_rms_norm_fp8):
            f.restype = I
        lib.oracle_silu_and_mul_fp8.argtypes = [P, I, I64, I64, P, P, P, P]
        lib.oracle_silu_and_mul_fp8.restype = I
        lib.oracle_fp8_rowwise_gemm.argtypes = [P, P, P, P, I64, I64, I64, I64, I64, P, P]
        lib.oracle_fp8_rowwise_gemm.restype = I
        lib.oracle_allreduce_sum16.argtypes = [P, I, I64, I, P]
        lib.oracle_allreduce_sum16.restype = I
        lib.oracle_decode16_array.argtypes = [P, I, I64, P]
        lib.oracle_encode16_array.argtypes = [P, I, I64, P]
        lib.oracle_decode_e4m3_array.argtypes = [P, I64, P]
        lib.oracle_encode_e4m3_array.argtypes = [P, I64, P]
        _lib = lib
        return lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _bits16(a) -> np.ndarray:
    """uint16 view of a 16-bit numpy array or CPU torch tensor."""
    if hasattr(a, "numpy"):  # torch tensor
        import torch
        a = a.detach().cpu().contiguous().view(torch.int16).numpy()
    a = np.ascontiguousarray(a)
    if a.dtype.itemsize != 2:
        raise TypeError(f"expected 16-bit data, got {a.dtype}")
    return a.view(np.uint16)


# --------------------------------------------------------------------------
# codecs

def decode16(bits, dtype: str) -> np.ndarray:
    b = _bits16(bits)
    out = np.empty(b.shape, np.float64)
    _load().oracle_decode16_array(_ptr(b), DTYPES[dtype], b.size, _ptr(out))
    return out


def encode16(values, dtype: str) -> np.ndarray:
    v = np.ascontiguousarray(values, dtype=np.float64)
    out = np.empty(v.shape, np.uint16)
    _load().oracle_encode16_array(_ptr(v), DTYPES[dtype], v.size, _ptr(out))
    return out


def decode_e4m3(codes) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    _load().oracle_decode_e4m3_array(_ptr(c), c.size, _ptr(out))
    return out


def encode_e4m3(values) -> np.ndarray:
    v = np.ascontiguousarray(values, dtype=np.float64)
    out = np.empty(v.shape, np.uint8)
    _load().oracle_encode_e4m3_array(_ptr(v), v.size, _ptr(out))
    return out


# --------------------------------------------------------------------------
# operators

def _shape2d(x):
    if x.ndim != 2:
        raise ValueError("oracle takes [T x H] arrays")
    return x.shape


def _blocks(T: int, threads: int):
    threads = max(1, min(threads, T)) if T else 1
    step = (T + threads - 1) // threads if T else 0
    return [(s, min(T, s + step)) for s in range(0, T, step)] if T else []


def _run(fn, T: int, H: int, threads: int):
    """Runs fn(t0, t1, row, yrow) over row blocks; ctypes drops the GIL."""
    blocks = _blocks(T, threads)
    if len(blocks) <= 1:
        for t0, t1 in blocks:
            fn(t0, t1, np.empty(H), np.empty(H))
        return
    with ThreadPoolExecutor(len(blocks)) as ex:
        list(ex.map(lambda b: fn(b[0], b[1], np.empty(H), np.empty(H)), blocks))


def rms_norm(x, weight, dtype: str, eps: float, want_y: bool = False, threads: int = 1):
    """out = RNE16(x / sqrt(mean(x^2) + eps) * w) per row; optional fp64 y."""
    lib = _load()
    xb = _bits16(x)
    T, H = _shape2d(xb)
    wb = None if weight is None else _bits16(weight).reshape(-1)
    if wb is not None and wb.size != H:
        raise ValueError("weight size")
    out = np.empty((T, H), np.uint16)
    y = np.empty((T, H), np.float64) if want_y else None
    dt = DTYPES[dtype]

    def blk(t0, t1, row, yrow):
        rc = lib.oracle_rms_norm(_ptr(xb[t0:t1]), _ptr(wb), dt, t1 - t0, H, eps,
                                 _ptr(out[t0:t1]), None if y is None else _ptr(y[t0:t1]),
                                 _ptr(row), _ptr(yrow))
        assert rc == 0

    _run(blk, T, H, threads)
    return (out, y) if want_y else out


def fused_add_rms_norm(x, residual, weight, dtype: str, eps: float, want_y: bool = False,
                       threads: int = 1):
    """Returns (r', out[, y]): r' = RNE16(x + residual); out = rms_norm(r')."""
    lib = _load()
    xb, rb = _bits16(x), _bits16(residual)
    T, H = _shape2d(xb)
    if rb.shape != (T, H):
        raise ValueError("residual shape")
    wb = None if weight is None else _bits16(weight).reshape(-1)
    r_out = np.empty((T, H), np.uint16)
    out = np.empty((T, H), np.uint16)
    y = np.empty((T, H), np.float64) if want_y else None
    dt = DTYPES[dtype]

    def blk(t0, t1, row, yrow):
        rc = lib.oracle_fused_add_rms_norm(
            _ptr(xb[t0:t1]), _ptr(rb[t0:t1]), _ptr(wb), dt, t1 - t0, H, eps,
            _ptr(r_out[t0:t1]), _ptr(out[t0:t1]), None if y is None else _ptr(y[t0:t1]),
            _ptr(row), _ptr(yrow))
        assert rc == 0

    _run(blk, T, H, threads)
    return (r_out, out, y) if want_y else (r_out, out)


def fused_add_rms_norm_fp8(x, residual, weight, dtype: str, eps: float,
                           want_y: bool = False, threads: int = 1):
    """Returns (r', q, scale[, y]) of the fused pass with a per-token e4m3 cast."""
    lib = _load()
    xb, rb = _bits16(x), _bits16(residual)
    T, H = _shape2d(xb)
    if rb.shape != (T, H):
        raise ValueError("residual shape")
    wb = None if weight is None else _bits16(weight).reshape(-1)
    r_out = np.empty((T, H), np.uint16)
    q = np.empty((T, H), np.uint8)
    scale = np.empty((T,), np.float32)
    y = np.empty((T, H), np.float64) if want_y else None
    dt = DTYPES[dtype]

    def blk(t0, t1, row, yrow):
        rc = lib.oracle_fused_add_rms_norm_fp8(
            _ptr(xb[t0:t1]), _ptr(rb[t0:t1]), _ptr(wb), dt, t1 - t0, H, eps,
            _ptr(r_out[t0:t1]), _ptr(q[t0:t1]), _ptr(scale[t0:t1]),
            None if y is None else _ptr(y[t0:t1]), _ptr(row), _ptr(yrow))
        assert rc == 0

    _run(blk, T, H, threads)
    return (r_out, q, scale, y) if want_y else (r_out, q, scale)


def silu_and_mul_fp8(x, dtype: str, want_y: bool = False, threads: int = 1):
    """x: [T x 2I] 16-bit bits, gate first. Returns (q [T x I], scale [T][, y])."""
    lib = _load()
    xb = _bits16(x)
    T, H2 = _shape2d(xb)
    if H2 % 2:
        raise ValueError("x must have an even last dimension")
    I = H2 // 2
    q = np.empty((T, I), np.uint8)
    scale = np.empty((T,), np.float32)
    y = np.empty((T, I), np.float64) if want_y else None
    dt = DTYPES[dtype]

    def blk(t0, t1, row, yrow):
        rc = lib.oracle_silu_and_mul_fp8(_ptr(xb[t0:t1]), dt, t1 - t0, I, _ptr(q[t0:t1]),
                                         _ptr(scale[t0:t1]), None if y is None else _ptr(y[t0:t1]),
                                         _ptr(yrow))
        assert rc == 0

    _run(blk, T, I, threads)
    return (q, scale, y) if want_y else (q, scale)


def fp8_rowwise_gemm(a_codes, b_codes, a_scale, b_scale, rows=None, want_y: bool = False,
                     threads: int = 1):
    """D = bf16((A @ B^T) * a_scale[:, None] * b_scale[None, :]) from e4m3 codes
    (uint8, A [M x K], B [N x K]). `rows` (sorted indices) restricts the rows
    computed; the result then holds those rows only. Returns D bits [, y]."""
    lib = _load()
    A = np.ascontiguousarray(a_codes, dtype=np.uint8)
    B = np.ascontiguousarray(b_codes, dtype=np.uint8)
    sa = np.ascontiguousarray(a_scale, dtype=np.float32).reshape(-1)
    sb = np.ascontiguousarray(b_scale, dtype=np.float32).reshape(-1)
    M, K = A.shape
    N = B.shape[0]
    if B.shape[1] != K or sa.size != M or sb.size != N:
        raise ValueError("shape mismatch")
    if rows is not None:
        rows = np.asarray(rows, dtype=np.int64)
        A, sa = np.ascontiguousarray(A[rows]), np.ascontiguousarray(sa[rows])
        M = A.shape[0]
    D = np.empty((M, N), np.uint16)
    y = np.empty((M, N), np.float64) if want_y else None

    def blk(t0, t1, row, yrow):
        rc = lib.oracle_fp8_rowwise_gemm(_ptr(A), _ptr(B), _ptr(sa), _ptr(sb), M, N, K, t0, t1,
                                         _ptr(D), None if y is None else _ptr(y))
        assert rc == 0

    _run(blk, M, 1, threads)
    return (D, y) if want_y else D


def allreduce_sum16(parts, dtype: str, threads: int = 1) -> np.ndarray:
    """x = RNE16(exact sum over ranks) of W partial arrays (16-bit bits,
    stacked on a leading rank axis: [W, ...]). Returns bits of shape [...]."""
    lib = _load()
    pb = _bits16(parts)
    W = pb.shape[0]
    flat = pb.reshape(W, -1)
    n = flat.shape[1]
    x = np.empty(n, np.uint16)
    dt = DTYPES[dtype]
    chunks = _blocks(n, threads)

    def blk(c):
        i0, i1 = c
        part = np.ascontiguousarray(flat[:, i0:i1])
        rc = lib.oracle_allreduce_sum16(_ptr(part), W, i1 - i0, dt, _ptr(x[i0:i1]))
        assert rc == 0

    if len(chunks) <= 1:
        for c in chunks:
            blk(c)
    else:
        with ThreadPoolExecutor(len(chunks)) as ex:
            list(ex.map(blk, chunks))
    return x.reshape(pb.shape[1:])


def allreduce_fused_add_rms_norm(parts, residual, weight, dtype: str, eps: float,
                                 want_y: bool = False, threads: int = 1):
    """Tensor-parallel form: x = allreduce_sum16(parts) ([W, T, H] partials),
    then fused_add_rms_norm(x, residual). Returns (x, r', out[, y])."""
    x = allreduce_sum16(parts, dtype, threads)
    return (x, *fused_add_rms_norm(x, residual, weight, dtype, eps, want_y, threads))


def allreduce_fused_add_rms_norm_fp8(parts, residual, weight, dtype: str, eps: float,
                                     want_y: bool = False, threads: int = 1):
    """x = allreduce_sum16(parts), then fused_add_rms_norm_fp8(x, residual).
    Returns (x, r', q, scale[, y])."""
    x = allreduce_sum16(parts, dtype, threads)
    return (x, *fused_add_rms_norm_fp8(x, residual, weight, dtype, eps, want_y, threads))


def usable_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1
