"""Property test of the oracle's exact all-reduce sum (CPU only): for random
groups of 1 to 8 finite 16-bit partials, drawn from the whole exponent range
and from a few clustered binades (where cancellations and rounding ties are
frequent), the result equals the exact rational sum rounded to nearest even
by the format definition (tests/oracle_pins.py `_exact16`), independently of
the order of the ranks. "AITER: AMD's operator library for ROCm", ecosystem
section: the all-reduce before RMSNorm."""
from fractions import Fraction

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from tests.oracle_pins import _exact16, _nan16

_EXP_BITS = {"bf16": (7, 0xFF), "fp16": (10, 0x1F)}


def _code(dtype, sign, exp, mant):
    shift, emax = _EXP_BITS[dtype]
    return (sign << 15) | (min(exp, emax - 1) << shift) | (mant & ((1 << shift) - 1))


@st.composite
def groups(draw):
    dtype = draw(st.sampled_from(["bf16", "fp16"]))
    W = draw(st.integers(1, 8))
    _, emax = _EXP_BITS[dtype]
    clustered = draw(st.booleans())
    base = draw(st.integers(0, emax - 4))
    codes = []
    for _ in range(W):
        exp = draw(st.integers(base, base + 3) if clustered else st.integers(0, emax - 1))
        mant = draw(st.integers(0, 1023))
        codes.append(_code(dtype, draw(st.integers(0, 1)), exp, mant))
    perm = draw(st.permutations(list(range(W))))
    return dtype, np.array(codes, dtype=np.uint16), perm


@settings(max_examples=400, deadline=None)
@given(groups())
def test_allreduce_sum_is_the_exact_sum_rounded_once(g):
    dtype, codes, perm = g
    parts = codes.reshape(-1, 1)
    got = oracle.allreduce_sum16(parts, dtype)[0]
    assert not _nan16(np.array([got]), dtype)[0]
    vals = oracle.decode16(codes, dtype)
    exact = sum((Fraction(float(v)) for v in vals), Fraction(0))
    want = _exact16(exact, dtype)
    got_v = float(oracle.decode16(np.array([got]), dtype)[0])
    if want == 0:
        assert got_v == 0
    else:
        assert got_v == want, (codes, got_v, want)
    assert oracle.allreduce_sum16(codes[perm].reshape(-1, 1), dtype)[0] == got
