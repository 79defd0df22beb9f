"""GPU checks of the tcgen05 / TMEM / TMA building blocks (libckda_selftest.so):
small GEMMs through shared-memory and tensor-memory operand paths against an fp64
matmul of the same bf16 operands, and TMA box loads against the 128-byte swizzle
formula the kernels assume."""
import ctypes
import os

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def st():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from delta_rule_attention_ckda_b200 import build
    build.build()
    lib = ctypes.CDLL(build.SELFTEST_LIB)
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.ckda_selftest_gemm.argtypes = [vp, vp, vp, i, i, i, i, i, vp]
    lib.ckda_selftest_gemm_sub.argtypes = [vp, vp, vp] + [i] * 7 + [vp]
    lib.ckda_selftest_tma.argtypes = [vp, i, i, i, i, i, i, i, i, i, i, vp, vp]
    lib.ckda_selftest_wait.argtypes = [ctypes.c_uint, i, vp]
    lib.ckda_selftest_error_word.argtypes = [ctypes.POINTER(ctypes.c_uint)]
    return lib


@pytest.mark.parametrize("arrive", [0, 1])
def test_bounded_wait_gives_up_and_reports(st, arrive):
    """A wait on an mbarrier that nothing completes returns after its poll limit with the
    timeout bit set in the device error word; the context stays usable afterwards (a
    GEMM self-test still passes). With the barrier completed first, the wait succeeds
    and nothing is reported."""
    word = ctypes.c_uint(0)
    assert st.ckda_selftest_error_word(ctypes.byref(word)) == 0      # clear
    res = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    assert st.ckda_selftest_wait(1024, arrive, res.data_ptr()) == 0
    assert st.ckda_selftest_error_word(ctypes.byref(word)) == 0
    assert int(res.item()) == arrive
    assert (word.value & 1) == (0 if arrive else 1)
    test_gemm_paths(st, 0, 0, 64, 64, 0)


def swz(off):
    return off ^ (((off >> 7) & 7) << 4)


@pytest.mark.parametrize("a_mode", [0, 1, 2])
@pytest.mark.parametrize("b_mode", [0, 1])
@pytest.mark.parametrize("N,K", [(64, 64), (128, 128), (256, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("neg", [0, 1])
def test_gemm_paths(st, a_mode, b_mode, N, K, neg):
    g = torch.Generator().manual_seed(N * 1000 + K + 10 * a_mode + b_mode)
    A = torch.randn(128, K, generator=g).to(torch.bfloat16)
    B = torch.randn(K, N, generator=g).to(torch.bfloat16)
    dA, dB = A.cuda(), B.cuda()
    D = torch.full((128, N), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = st.ckda_selftest_gemm(dA.data_ptr(), dB.data_ptr(), D.data_ptr(), N, K, a_mode, b_mode, neg,
                               status.data_ptr())
    assert rc == 0
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = A.double() @ B.double()
    if neg:
        ref = -ref
    err = (D.double().cpu() - ref).abs().max().item()
    assert err <= 1e-5 * ref.abs().max().item(), f"max err {err}"


@pytest.mark.parametrize("b_mode,N,K,n0,ns,kb,kn", [
    (0, 128, 64, 16, 48, 0, 16), (0, 128, 64, 80, 48, 0, 16), (0, 128, 64, 32, 32, 0, 32),
    (0, 128, 64, 112, 16, 0, 48), (1, 64, 128, 0, 16, 16, 48), (1, 64, 128, 16, 16, 32, 32),
    (1, 64, 128, 32, 16, 48, 16), (1, 64, 128, 0, 64, 64, 64), (1, 64, 64, 48, 16, 16, 16)])
def test_gemm_sub_tiles(st, b_mode, N, K, n0, ns, kb, kn):
    """Sub-tiles of a staged operand through the descriptors alone: rows of a K-major B,
    16-wide column ranges inside the swizzle atom of an MN-major B, and a range of K steps
    (the gate gradient's partial products over earlier or later token blocks)."""
    g = torch.Generator().manual_seed(N + 7 * K + n0 + 3 * kb + b_mode)
    A = torch.randn(128, K, generator=g).to(torch.bfloat16)
    B = torch.randn(K, N, generator=g).to(torch.bfloat16)
    dA, dB = A.cuda(), B.cuda()
    D = torch.full((128, ns), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = st.ckda_selftest_gemm_sub(dA.data_ptr(), dB.data_ptr(), D.data_ptr(), N, K, b_mode, n0, ns, kb, kn,
                                   status.data_ptr())
    assert rc == 0
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = A[:, kb:kb + kn].double() @ B[kb:kb + kn, n0:n0 + ns].double()
    err = (D.double().cpu() - ref).abs().max().item()
    assert err <= 1e-5 * ref.abs().max().item(), f"max err {err}"


@pytest.mark.parametrize("dtype,box_d", [(torch.bfloat16, 64), (torch.float32, 32)])
@pytest.mark.parametrize("t0", [0, 64])
def test_tma_box_layout_and_tail_fill(st, dtype, box_d, t0):
    B, T, H, d = 2, 100, 3, 128
    g = torch.Generator().manual_seed(3)
    X = torch.randn(B, T, H, d, generator=g).to(dtype)
    dX = X.cuda()
    out = torch.zeros(64 * 128, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    b, h, c0 = 1, 2, box_d
    rc = st.ckda_selftest_tma(dX.data_ptr(), 1 if dtype == torch.bfloat16 else 0, B, T, H, d, box_d, c0, h, t0, b,
                              out.data_ptr(), status.data_ptr())
    assert rc == 0
    torch.cuda.synchronize()
    assert status.item() == 0
    raw = out.cpu().numpy()
    es = 2 if dtype == torch.bfloat16 else 4
    npdt = np.uint16 if es == 2 else np.uint32
    src = X.view(torch.int16 if es == 2 else torch.int32).numpy().view(npdt)
    for r in range(64):
        for c in range(box_d):
            off = swz(r * 128 + c * es)
            got = raw[off:off + es].view(npdt)[0]
            exp = src[b, t0 + r, h, c0 + c] if t0 + r < T else 0
            assert got == exp, (r, c, got, exp)
