"""torch custom ops, eligibility predicates and the priority dispatcher, on the
CPU (no kernel runs): predicate semantics against "vllm.kernels.aiter_ops"
(rms_no_var_16bit_only, rms_add_no_var_16bit_only, flatten_to_2d_is_free),
agreement with the C ABI's layout check, fake (meta) shape inference for
torch.compile, and dispatch order with a caller-registered backend."""
import pytest
import torch

import residual_add_rmsnorm_rms_b200 as rn
from residual_add_rmsnorm_rms_b200 import torch_ops as ops

BF = torch.bfloat16
H = 64


def t(shape, dtype=BF):
    return torch.empty(shape, dtype=dtype)


def test_flatten_to_2d_is_free_cases():
    f = ops.flatten_to_2d_is_free
    assert f(t((2, 3, H)))
    assert f(t((H,)))
    assert f(t((4 * H,)).as_strided((4, 1, H), (H, 7, 1)))  # size-1 dim, any stride
    assert not f(t((3, 2, H)).transpose(0, 1))  # reshape would copy
    assert not f(t((4, 2 * H))[:, ::2])  # strided last dim
    assert not f(t((2, 4, H + 8))[:, :, :H])  # padded rows
    assert not f(t((4, H + 8))[:, :H])  # padded 2-D rows (this library's reading)
    assert f(t((0, H)))
    assert not f(t((4, 0)))


def test_predicate_matches_c_abi_layout_check():
    views = [t((2, 3, H)), t((H,)), t((3, 2, H)).transpose(0, 1), t((4, 2 * H))[:, ::2],
             t((2, 4, H + 8))[:, :, :H], t((4, H + 8))[:, :H],
             t((4 * H,)).as_strided((4, 1, H), (H, 7, 1)), t((1, 1, 5, H)),
             t((5, 1, H)).as_strided((5, 1, H), (H, 1, 1))]
    for v in views:
        st, _ = rn.validate("rms_norm", t(v.shape), v)
        assert ops.flatten_to_2d_is_free(v) == (st == "RN_OK"), (v.shape, v.stride(), st)


def test_eligibility_predicates():
    x, w = t((4, H)), t((H,))
    assert ops.rms_no_var_16bit_only(x, w, 1e-6)
    assert ops.rms_no_var_16bit_only(x, None, 1e-6)
    assert not ops.rms_no_var_16bit_only(x, w, 1e-6, variance_size=H)
    assert not ops.rms_no_var_16bit_only(t((4, H), torch.float32), None, 1e-6)
    assert not ops.rms_no_var_16bit_only(x, t((H,), torch.float16), 1e-6)
    assert ops.rms_add_no_var_16bit_only(x, t((4, H)), w, 1e-6)
    assert not ops.rms_add_no_var_16bit_only(x, t((4, 2 * H))[:, ::2], w, 1e-6)


def test_ops_are_registered_with_schemas():
    for name in ("rms_norm", "fused_add_rms_norm", "fused_add_rms_norm_fp8"):
        assert hasattr(torch.ops.rmsnorm_b200, name)
    schema = str(torch.ops.rmsnorm_b200.fused_add_rms_norm.default._schema)
    import re
    assert re.search(r"Tensor\(a\d*!\) x", schema) and re.search(r"Tensor\(a\d*!\) residual", schema)
    assert "Tensor? weight" in schema


def test_fake_implementations_infer_shapes():
    from torch._subclasses.fake_tensor import FakeTensorMode
    with FakeTensorMode():
        x = torch.empty(2, 3, H, dtype=BF, device="cuda")
        r = torch.empty(2, 3, H, dtype=BF, device="cuda")
        w = torch.empty(H, dtype=BF, device="cuda")
        out = torch.ops.rmsnorm_b200.rms_norm(x, w, 1e-6)
        assert out.shape == x.shape and out.dtype == BF
        q, s = torch.ops.rmsnorm_b200.fused_add_rms_norm_fp8(x, r, w, 1e-6)
        assert q.shape == x.shape and q.dtype == torch.float8_e4m3fn
        assert s.shape == (2, 3, 1) and s.dtype == torch.float32
        assert torch.ops.rmsnorm_b200.fused_add_rms_norm(x, r, w, 1e-6) is None
        out = torch.ops.rmsnorm_b200.allreduce_fused_add_rms_norm(x, r, w, 1e-6, 7)
        assert out.shape == x.shape and out.dtype == BF
        q, s = torch.ops.rmsnorm_b200.allreduce_fused_add_rms_norm_fp8(x, r, w, 1e-6, 7)
        assert q.shape == x.shape and s.shape == (2, 3, 1)


def test_allreduce_ops_schemas_and_comm_handles():
    import re
    for name in ("allreduce_fused_add_rms_norm", "allreduce_fused_add_rms_norm_fp8"):
        schema = str(getattr(torch.ops.rmsnorm_b200, name).default._schema)
        assert re.search(r"Tensor\(a\d*!\) residual", schema) and "Int comm" in schema, schema
    from residual_add_rmsnorm_rms_b200.allreduce import AllReduceComm, lookup
    a = AllReduceComm(2, 0, 2, [16, 32], [48, 64], 4096)
    b = AllReduceComm(1, 0, 1, [16], [48], 4096)
    assert a.handle != b.handle and lookup(a.handle) is a and lookup(b.handle) is b
    h = b.handle
    del b
    import gc
    gc.collect()
    with pytest.raises(KeyError):
        lookup(h)


def test_dispatch_rejects_ineligible_inputs_loudly():
    x = t((4, H))
    with pytest.raises(ops.IneligibleInput, match="rms_no_var_16bit_only"):
        ops.rms_norm(t((4, H), torch.float32), None, 1e-6)
    with pytest.raises(ops.IneligibleInput, match="rms_no_var_16bit_only"):
        ops.rms_norm(x, None, 1e-6, variance_size=32)
    with pytest.raises(ops.IneligibleInput, match="CUDA"):
        ops.rms_norm(x, None, 1e-6)  # CPU tensors: no CPU path in this package
    with pytest.raises(ops.IneligibleInput, match="rms_add_no_var_16bit_only"):
        ops.fused_add_rms_norm(x, t((4, 2 * H))[:, ::2], None, 1e-6)


def test_caller_registered_backend_takes_what_b200_declines():
    calls = []

    def pred(x, w, e, v=None):
        return None if x.dtype == torch.float32 else "only fp32"

    def impl(x, w, e, v=None):
        calls.append(x.dtype)
        return "caller-backend"

    assert ops.backends("rms_norm") == ["b200"]
    ops.register_backend("rms_norm", "caller", pred, impl)
    try:
        assert ops.backends("rms_norm") == ["b200", "caller"]
        assert ops.rms_norm(t((4, H), torch.float32), None, 1e-6) == "caller-backend"
        assert calls == [torch.float32]
        with pytest.raises(ValueError):
            ops.register_backend("rms_norm", "caller", pred, impl)
    finally:
        ops.unregister_backend("rms_norm", "caller")
    assert ops.backends("rms_norm") == ["b200"]
    with pytest.raises(ValueError):
        ops.unregister_backend("rms_norm", "b200")
