"""The whole-group fused all-reduce entry point that allocates nothing
(rn_allreduce_fused_add_rms_norm_local: exchange buffers and signal pads in a
static device array of the library) against the entry point with
caller-provided exchange memory, bit for bit, over calls in a row. The file
is collected last, so it also runs after every other test has used the
device; it passes on its own as well."""
import pytest
import torch

import oracle
import residual_add_rmsnorm_rms_b200 as rn
import synth
from residual_add_rmsnorm_rms_b200.allreduce import AllReduceComm
from tests.cmp_util import bits16
from tests.gpu_util import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    yield
    assert rn.device_errors() == 0


def _inputs(W, T, H, seed):
    wl = synth.make_tp_inputs("bf16", W, T, H, seed=seed, device="cuda")
    return wl, wl.residual.unsqueeze(0).repeat(W, 1, 1).contiguous()


def _both(W, T, H, seed, comm):
    """One call through each entry point on the same inputs."""
    wl, res = _inputs(W, T, H, seed)
    ra, rb = res.clone(), res.clone()
    oa, ob = torch.empty_like(wl.x), torch.empty_like(wl.x)
    rn.allreduce_fused_add_rms_norm(oa, wl.x, ra, wl.weight, wl.eps, comm)
    rn.allreduce_fused_add_rms_norm_local(ob, wl.x, rb, wl.weight, wl.eps, W)
    torch.cuda.synchronize()
    return wl, (oa, ra), (ob, rb)


def test_no_alloc_matches_caller_memory_calls_in_a_row():
    W, T, H = 4, 64, 3840
    comm = AllReduceComm.single_device(W, T, H, "cuda")
    for i in range(2):
        wl, (oa, ra), (ob, rb) = _both(W, T, H, 900 + i, comm)
        assert torch.equal(ob.view(torch.int16), oa.view(torch.int16))
        assert torch.equal(rb.view(torch.int16), ra.view(torch.int16))
    # and the last one against the oracle
    _, r2, out = oracle.allreduce_fused_add_rms_norm(bits16(wl.x.cpu()), bits16(wl.residual.cpu()),
                                                    bits16(wl.weight.cpu()), "bf16", wl.eps)
    compare("fused", {"residual": rb[W - 1], "out": ob[W - 1]}, {"residual": r2, "out": out},
            "bf16")


def test_no_alloc_group_size_changes():
    """Changing `world` clears the pads; every size still matches."""
    H = 4096
    for W, T in [(2, 33), (8, 16), (2, 5), (1, 3)]:
        comm = AllReduceComm.single_device(W, T, H, "cuda")
        _, (oa, ra), (ob, rb) = _both(W, T, H, 950 + W + T, comm)
        assert torch.equal(ob.view(torch.int16), oa.view(torch.int16)), (W, T)
        assert torch.equal(rb.view(torch.int16), ra.view(torch.int16)), (W, T)


def test_no_alloc_two_shot_then_one_shot_then_two_shot():
    """Calls the automatic choice runs two-shot in the static memory (eight
    ranks of [40 x 8192]: two-shot saves 8.75 * 40 * 8192 = 2.87 MB of peer
    reads per rank, above the 2.3 MB threshold, and eight buffers of
    round_up(12 * 40 * 8192 + 32, 256) bytes, 31.5 MB, fit the 32 MiB), with a
    one-shot call of the same group size ([2 x 8192] per rank) in between,
    each bit for bit against the entry point with caller memory."""
    W, H = 8, 8192
    for T in (40, 2, 40):
        comm = AllReduceComm.single_device(W, T, H, "cuda")
        _, (oa, ra), (ob, rb) = _both(W, T, H, 970 + T, comm)
        assert torch.equal(ob.view(torch.int16), oa.view(torch.int16)), T
        assert torch.equal(rb.view(torch.int16), ra.view(torch.int16)), T


def test_no_alloc_capacity_and_arguments():
    W, H = 8, 4096
    T = (32 << 20) // (W * 4 * H) + 1  # one row per rank too many
    x = torch.zeros(W, T, H, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rn.RmsNormError) as e:
        rn.allreduce_fused_add_rms_norm_local(torch.empty_like(x), x, x.clone(), None, 1e-6, W)
    assert e.value.name == "RN_ERR_CAPACITY"
    T -= 2  # fits
    x = torch.zeros(W, T, H, dtype=torch.bfloat16, device="cuda")
    rn.allreduce_fused_add_rms_norm_local(torch.empty_like(x), x, x.clone(), None, 1e-6, W)
    for world in (0, 9):
        with pytest.raises(rn.RmsNormError) as e:
            rn.allreduce_fused_add_rms_norm_local(torch.empty_like(x), x, x.clone(), None, 1e-6,
                                                  world)
        assert e.value.name == "RN_ERR_COMM"
    torch.cuda.synchronize()


def test_no_alloc_graph_capture_after_setup():
    """After an uncaptured call sets the group size up, captured calls replay
    correctly; a new group size inside a capture is refused."""
    W, T, H = 2, 24, 3840
    wl, res = _inputs(W, T, H, 990)
    out = torch.empty_like(wl.x)
    rn.allreduce_fused_add_rms_norm_local(out, wl.x, res.clone(), wl.weight, wl.eps, W)
    torch.cuda.synchronize()
    r = res.clone()
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            rn.allreduce_fused_add_rms_norm_local(out, wl.x, r, wl.weight, wl.eps, W)
            with pytest.raises(rn.RmsNormError) as e:
                rn.allreduce_fused_add_rms_norm_local(out, wl.x, r, wl.weight, wl.eps, W + 1)
            assert e.value.name == "RN_ERR_CONFIG"
    for _ in range(2):
        r.copy_(res)
        g.replay()
        torch.cuda.synchronize()
        comm = AllReduceComm.single_device(W, T, H, "cuda")
        _, (oa, ra), _ = _both(W, T, H, 990, comm)
        assert torch.equal(out.view(torch.int16), oa.view(torch.int16))
        assert torch.equal(r.view(torch.int16), ra.view(torch.int16))
    del g
