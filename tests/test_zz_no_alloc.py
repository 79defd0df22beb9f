"""ckda_chunk_fwd_noalloc: the segmented chunk path on the library's fixed device
scratch instead of a caller workspace. Two consecutive calls, on different inputs so
that the second one reuses scratch the first one filled, must give results
bit-identical to ckda_chunk_fwd on the same inputs (same kernels, same launch plan),
and a warmed-up call must not change the device's free memory."""
import ctypes

import pytest
import torch

from ckda_inputs import make_inputs, make_workload
from parity_util import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ck():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from delta_rule_attention_ckda_b200 import build
    build.build()
    import delta_rule_attention_ckda_b200 as m
    m.load()
    return m


def _pair(ck, inp):
    q, k, v, a, b, s0 = to_dev(inp)
    o_ref, S_ref = ck.chunk_fwd(q, k, v, a, b, s0)
    o = torch.full_like(o_ref, float("nan"))
    S = torch.full_like(S_ref, float("nan"))
    return (q, k, v, a, b, s0), (o_ref, S_ref), (o, S)


@pytest.mark.parametrize("shape", [(1, 1000, 2, 128, 128), (1, 1100, 2, 64, 128), (2, 300, 2, 128, 128)])
def test_two_consecutive_calls_match_workspace_entry(ck, shape):
    B, T, H, dk, dv = shape
    need = ck.workspace_bytes(B, T, H, dk, dv)
    assert need <= ck.noalloc_scratch_bytes()
    first = _pair(ck, make_inputs(B, T, H, dk, dv, torch.bfloat16, seed=1, gate="tanh15", s0_std=0.1))
    second = _pair(ck, make_inputs(B, T, H, dk, dv, torch.bfloat16, seed=2, gate="signmag", s0_std=0.1))
    for args, _, (o, S) in (first, second):
        ck.chunk_fwd_noalloc(*args, o=o, S_T=S)
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    for _, (o_ref, S_ref), (o, S) in (first, second):
        assert torch.equal(o, o_ref) and torch.equal(S, S_ref)


def test_long_workload_fits_and_matches(ck):
    """B=1, T=65536, H=16, d=128: the segmented launch the long-context forward takes. The
    capacity is sized for this problem on a 148-SM GPU; the segment plan follows the SM
    count, so a GPU that needs more scratch for it is outside what this test checks."""
    inp = make_workload("long")
    B, T, H, dk = inp.q.shape
    assert ck.chunk_segments(B, T, H, dk, dk) > 1
    need = ck.workspace_bytes(B, T, H, dk, dk)
    if need > ck.noalloc_scratch_bytes():
        pytest.skip(f"this GPU's segment plan needs {need} bytes of scratch for the long workload")
    assert need > 0
    args, (o_ref, S_ref), (o, S) = _pair(ck, inp)
    for _ in range(2):
        o.fill_(float("nan"))
        ck.chunk_fwd_noalloc(*args, o=o, S_T=S)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(S, S_ref)


def test_oversize_problem_is_rejected_before_launch(ck):
    """A problem whose segment buffers exceed the fixed scratch returns
    CKDA_ERR_WORKSPACE without touching its (dummy, aligned) pointers. The shape is
    found from the segment plan of this device (one long sequence per head)."""
    lib = ck.load()
    T, d = 1 << 20, 128
    over = [H for H in range(1, 160) if ck.workspace_bytes(1, T, H, d, d) > ck.noalloc_scratch_bytes()]
    assert over, "no head count needs more scratch than the capacity"
    p = ctypes.c_void_p(256)
    fp = ctypes.cast(p, ctypes.POINTER(ctypes.c_float))
    for H in over[:3]:
        st = lib.ckda_chunk_fwd_noalloc(p, p, p, fp, fp, fp, fp, fp, 1, T, H, d, d, 1, 0, None)
        assert st == 6, (H, st)   # CKDA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0


def test_warm_call_allocates_no_device_memory(ck):
    """Once the library's module is loaded and the scratch address looked up (the first
    call on the device), a call changes neither the driver's free memory nor torch's
    allocator: the scratch is the fixed array, and o / S_T are the caller's."""
    inp = make_inputs(1, 1000, 2, 128, 128, torch.bfloat16, seed=3, gate="tanh15", s0_std=0.1)
    B, T, H, dk, dv = inp.shape
    assert ck.workspace_bytes(B, T, H, dk, dv) > 0          # the call really uses the scratch
    q, k, v, a, b, s0 = to_dev(inp)
    o = torch.empty(B, T, H, dv, device="cuda")
    S = torch.empty(B, H, dk, dv, device="cuda")
    ck.chunk_fwd_noalloc(q, k, v, a, b, s0, o=o, S_T=S)      # warm-up: module and address set up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(3):
        ck.chunk_fwd_noalloc(q, k, v, a, b, s0, o=o, S_T=S)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0, (free0, free1)
    assert ck.get_device_error() == 0
