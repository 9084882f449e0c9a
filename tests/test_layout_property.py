"""Property test (CPU): for random strided views, the C ABI's layout check
(rn_validate) accepts exactly the views the eligibility predicate
flatten_to_2d_is_free accepts, and never accepts a view whose flattening to
2-D would copy or leave gaps."""
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import residual_add_rmsnorm_rms_b200 as rn
from residual_add_rmsnorm_rms_b200 import torch_ops as ops


@st.composite
def views(draw):
    ndim = draw(st.integers(1, 4))
    sizes = [draw(st.integers(1, 5)) for _ in range(ndim - 1)] + [draw(st.sampled_from([8, 16, 24]))]
    dense = draw(st.booleans())
    strides = []
    expected = 1
    for s in reversed(sizes):
        if dense:
            strides.append(expected)
        else:
            strides.append(draw(st.integers(1, 3)) * expected + draw(st.sampled_from([0, 0, 8])))
        expected *= s
    strides = list(reversed(strides))
    if draw(st.booleans()) and ndim > 1:  # permute the leading dims
        perm = draw(st.permutations(list(range(ndim - 1)))) + [ndim - 1]
        sizes = [sizes[p] for p in perm]
        strides = [strides[p] for p in perm]
    need = 1 + sum((s - 1) * t for s, t in zip(sizes, strides))
    base = torch.empty(need, dtype=torch.bfloat16)
    return base.as_strided(sizes, strides)


@settings(max_examples=400, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(views())
def test_c_abi_layout_check_matches_predicate(v):
    st_, _ = rn.validate("rms_norm", torch.empty(v.shape, dtype=v.dtype), v)
    free = ops.flatten_to_2d_is_free(v)
    assert (st_ == "RN_OK") == free, (v.shape, v.stride(), st_)
    if free:
        # accepted views are exactly dense: reshape is a view with unit-stride rows
        flat = v.reshape(-1, v.shape[-1])
        assert flat.data_ptr() == v.data_ptr()
        assert flat.stride() == (v.shape[-1], 1) or flat.shape[0] == 1
