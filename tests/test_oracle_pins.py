"""The CPU oracle against its pins (see tests/oracle_pins.py). CPU only."""
import pytest

import oracle
from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin, golden):
    pin(oracle, golden)


def test_threads_do_not_change_results():
    import numpy as np
    import synth
    from tests.cmp_util import bits16
    wl = synth.make_inputs("prefill", "fused_add_rms_norm", "bf16", 96, 3840)
    x, r, w = bits16(wl.x), bits16(wl.residual), bits16(wl.weight)
    a = oracle.fused_add_rms_norm_fp8(x, r, w, "bf16", wl.eps, threads=1)
    b = oracle.fused_add_rms_norm_fp8(x, r, w, "bf16", wl.eps, threads=5)
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)
