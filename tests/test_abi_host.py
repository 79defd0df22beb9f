"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
symbol include/ckda.h declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ckda.h")


@pytest.fixture(scope="module")
def lib():
    from delta_rule_attention_ckda_b200 import build
    build.build()
    import delta_rule_attention_ckda_b200 as ck
    return ck.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"CKDA_API\s+[\w\s\*]+?\b(ckda_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ["ckda_chunk_fwd", "ckda_decode_step", "ckda_chunk_fwd_workspace_bytes",
                 "ckda_status_string", "ckda_get_device_error", "ckda_recurrent_fwd"]:
        assert name in syms


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_exports_match_nm(lib):
    import subprocess
    import delta_rule_attention_ckda_b200 as ck
    out = subprocess.run(["nm", "-D", "--defined-only", ck.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (ckda_\w+)", out))
    assert set(declared_symbols()) <= exported


def test_status_strings(lib):
    for code in range(7):
        s = lib.ckda_status_string(code)
        assert isinstance(s, bytes) and len(s) > 0
    assert lib.ckda_status_string(99) == b"unknown status"
    assert lib.ckda_abi_version() == 9


NULL = None


def call_fwd(lib, fn, q=NULL, k=NULL, v=NULL, a=NULL, b=NULL, S0=NULL, o=NULL, ST=NULL,
             B=1, T=4, H=1, dk=16, dv=16, dt=1):
    args = [ctypes.c_void_p(x) if x is not None else None for x in (q, k, v, a, b, S0, o, ST)]
    if fn == "ckda_chunk_fwd":
        return lib.ckda_chunk_fwd(*args, B, T, H, dk, dv, dt, None, 0, None)
    return lib.ckda_recurrent_fwd(*args, B, T, H, dk, dv, dt, None)


@pytest.mark.parametrize("fn", ["ckda_chunk_fwd", "ckda_recurrent_fwd"])
def test_rejects_bad_sizes_before_launch(lib, fn):
    # none of these reaches a launch, so the fake pointers are never dereferenced
    p = 0x10000
    assert call_fwd(lib, fn, p, p, p, p, p, None, p, None, dk=0) == 1
    assert call_fwd(lib, fn, p, p, p, p, p, None, p, None, dv=129) == 1
    assert call_fwd(lib, fn, p, p, p, p, p, None, p, None, B=-1) == 1
    assert call_fwd(lib, fn, p, p, p, p, p, None, p, None, T=-5) == 1
    assert call_fwd(lib, fn, p, p, p, p, p, None, p, None, dt=7) == 1


@pytest.mark.parametrize("fn", ["ckda_chunk_fwd", "ckda_recurrent_fwd"])
def test_rejects_null_and_misaligned(lib, fn):
    p = 0x10000
    assert call_fwd(lib, fn, None, p, p, p, p, None, p, None) == 1       # q missing
    assert call_fwd(lib, fn, p, p, p, p, p, None, None, None) == 1       # o missing
    assert call_fwd(lib, fn, p + 4, p, p, p, p, None, p, None) == 3      # q misaligned
    assert call_fwd(lib, fn, p, p, p, p, p, p + 8, p, None) == 3         # S0 misaligned
    assert call_fwd(lib, fn, p, p, p, p, p, None, p, p + 2) == 3         # S_T misaligned


def test_decode_rejects(lib):
    p = ctypes.c_void_p(0x10000)
    bad = ctypes.c_void_p(0x10004)
    assert lib.ckda_decode_step(p, p, p, p, p, p, p, 4, 2, 0, 16, 1, None) == 1
    assert lib.ckda_decode_step(p, p, p, p, p, p, p, 4, 2, 16, 200, 1, None) == 1
    assert lib.ckda_decode_step(p, p, p, p, p, None, p, 4, 2, 16, 16, 1, None) == 1
    assert lib.ckda_decode_step(p, p, p, p, p, bad, p, 4, 2, 16, 16, 1, None) == 3
    assert lib.ckda_decode_step(p, p, p, p, p, p, p, 4, 2, 16, 16, 3, None) == 1


def test_empty_problems_launch_nothing(lib):
    # B*H == 0 returns OK without touching CUDA
    assert call_fwd(lib, "ckda_chunk_fwd", None, None, None, None, None, None, None, None,
                    B=0) == 0
    assert lib.ckda_decode_step(None, None, None, None, None, None, None, 0, 4, 16, 16, 1,
                                None) == 0


def test_workspace_query_and_path(lib):
    assert lib.ckda_chunk_fwd_workspace_bytes(1, 10, 1, 0, 16, 1) == 0
    for dt in (0, 1):
        assert lib.ckda_chunk_fwd_path(2, 100, 4, 16, 16, dt) in (0, 1)
    # fp32 inputs always take the recurrent path (the tensor-core path is bf16-only)
    assert lib.ckda_chunk_fwd_path(8, 4096, 16, 128, 128, 0) == 0


def test_segment_plan(lib):
    """Host-side segment plan of the tensor-core path (148 SMs assumed without a device):
    a batch that fills the GPU runs in one pass with no workspace; one long sequence per
    head is split, and its workspace holds nseg entering states (dk x dv) and transition
    products (dk x dk) per sequence, fp32."""
    bf = 1
    assert lib.ckda_chunk_fwd_segments(8, 4096, 16, 128, 128, bf) == 1
    assert lib.ckda_chunk_fwd_workspace_bytes(8, 4096, 16, 128, 128, bf) == 0
    nseg = lib.ckda_chunk_fwd_segments(1, 65536, 16, 128, 128, bf)
    assert 1 < nseg <= 64
    assert lib.ckda_chunk_fwd_workspace_bytes(1, 65536, 16, 128, 128, bf) == 16 * nseg * 128 * 256 * 4
    n64 = lib.ckda_chunk_fwd_segments(1, 65536, 16, 64, 128, bf)
    assert lib.ckda_chunk_fwd_workspace_bytes(1, 65536, 16, 64, 128, bf) == 16 * n64 * 64 * 192 * 4
    # segments are whole chunks: never more segments than chunks
    for T in (1, 64, 65, 128, 640, 1000):
        assert 1 <= lib.ckda_chunk_fwd_segments(1, T, 1, 128, 128, bf) <= (T + 63) // 64
    # the recurrent path and empty problems are never split
    assert lib.ckda_chunk_fwd_segments(1, 65536, 16, 128, 128, 0) == 1
    assert lib.ckda_chunk_fwd_segments(0, 65536, 16, 128, 128, bf) == 1
    assert lib.ckda_chunk_fwd_segments(1, 65536, 16, 32, 32, bf) == 1


def test_bwd_workspace_and_argument_checks(lib):
    """ckda_bwd's workspace: 8-token checkpoints, recomputed states and row partials;
    argument errors return before anything touches the device."""
    import ctypes
    # 6 sequences, 3 checkpoint blocks, one 32-column slab: checkpoints + states + partials
    assert lib.ckda_bwd_workspace_bytes(2, 17, 3, 16, 8, 0) == (
        6 * 3 * 16 * 8 + 6 * 8 * 128 * 32 + 6 * 17 * (3 * 16 + 1)) * 4
    assert lib.ckda_bwd_workspace_bytes(1, 8, 1, 128, 100, 0) == (
        1 * 128 * 100 + 4 * 8 * 128 * 32 + 4 * 8 * (3 * 128 + 1)) * 4
    assert lib.ckda_bwd_workspace_bytes(0, 17, 3, 16, 8, 0) == 0
    assert lib.ckda_bwd_workspace_bytes(1, 0, 3, 16, 8, 0) == 0
    assert lib.ckda_bwd_workspace_bytes(1, 4, 1, 0, 8, 0) == 0
    p = ctypes.c_void_p(256)
    fp = ctypes.cast(p, ctypes.POINTER(ctypes.c_float))
    null = ctypes.POINTER(ctypes.c_float)()
    ws = ctypes.c_void_p(4096)
    big = 1 << 40
    # missing grad_o
    assert lib.ckda_bwd(p, p, p, fp, fp, null, null, null, fp, fp, fp, fp, fp, null,
                        1, 4, 1, 16, 16, 0, 0, ws, big, None) == 1
    # unknown gate mode, bad head size
    assert lib.ckda_bwd(p, p, p, fp, fp, null, fp, null, fp, fp, fp, fp, fp, null,
                        1, 4, 1, 16, 16, 0, 7, ws, big, None) == 1
    assert lib.ckda_bwd(p, p, p, fp, fp, null, fp, null, fp, fp, fp, fp, fp, null,
                        1, 4, 1, 129, 16, 0, 0, ws, big, None) == 1
    # misaligned output
    bad = ctypes.cast(ctypes.c_void_p(260), ctypes.POINTER(ctypes.c_float))
    assert lib.ckda_bwd(p, p, p, fp, fp, null, fp, null, bad, fp, fp, fp, fp, null,
                        1, 4, 1, 16, 16, 0, 0, ws, big, None) == 3
    # workspace too small
    assert lib.ckda_bwd(p, p, p, fp, fp, null, fp, null, fp, fp, fp, fp, fp, null,
                        1, 4, 1, 16, 16, 0, 0, ws, 16, None) == 6


def test_mode_option_bits(lib):
    """mode = gate form | option bits; unknown bits and gate forms are argument errors,
    returned before anything touches the (dummy) pointers."""
    import ctypes
    from delta_rule_attention_ckda_b200 import _lib
    assert _lib._mode("signed", True) == 0x100 and _lib._mode("log", False) == 1
    p = ctypes.c_void_p(256)
    fp = ctypes.cast(p, ctypes.POINTER(ctypes.c_float))
    null = ctypes.POINTER(ctypes.c_float)()
    for mode in (0x200, 0x101 | 0x400, 2, 0x1FF):
        assert lib.ckda_chunk_fwd_ex(p, p, p, fp, fp, null, fp, null, 1, 4, 1, 16, 16, 0, mode,
                                     None, 0, None) == 1, hex(mode)
        assert lib.ckda_recurrent_fwd_ex(p, p, p, fp, fp, null, fp, null, 1, 4, 1, 16, 16, 0, mode,
                                         None) == 1, hex(mode)


def test_python_binding_refuses_cpu_tensors():
    import torch
    import delta_rule_attention_ckda_b200 as ck
    x = torch.zeros(1, 4, 1, 16)
    with pytest.raises(ValueError):
        ck.chunk_fwd(x, x, x, x, torch.zeros(1, 4, 1))


def test_gate_mode_names():
    """The binding maps gate names onto ckda_gate_t and rejects unknown ones (host only)."""
    from delta_rule_attention_ckda_b200 import _lib
    assert _lib.GATES == {"signed": 0, "log": 1}
    with pytest.raises(ValueError):
        _lib._gate("exp")
    text = open(os.path.join(ROOT, "include", "ckda.h")).read()
    assert "CKDA_GATE_SIGNED = 0" in text and "CKDA_GATE_LOG = 1" in text


def test_maps_workspace_and_argument_checks(lib):
    """ckda_chunk_fwd_maps: workspace only when the sequences are too few to fill the GPU
    (then (nsub + 1) slots of [M | N] per sequence), argument errors before any launch."""
    bf = 1
    assert lib.ckda_chunk_fwd_maps_workspace_bytes(64, 256, 16, 128, 128, bf) == 0      # 2048 CTAs already
    wl = lib.ckda_chunk_fwd_maps_workspace_bytes(8, 4096, 16, 128, 128, bf)             # 256 CTAs: split
    assert wl % (128 * 128 * 256 * 4) == 0
    assert lib.ckda_chunk_fwd_maps_workspace_bytes(1, 65536, 16, 128, 128, 0) == 0     # fp32: recurrent
    w = lib.ckda_chunk_fwd_maps_workspace_bytes(1, 65536, 16, 128, 128, bf)
    slot = 16 * 128 * 256 * 4
    assert w > 0 and w % slot == 0 and 3 <= w // slot <= 65
    assert lib.ckda_chunk_fwd_maps_workspace_bytes(1, 65536, 16, 64, 128, bf) % (16 * 64 * 192 * 4) == 0
    assert lib.ckda_chunk_fwd_maps_workspace_bytes(-1, 64, 1, 128, 128, bf) == 0
    p = ctypes.c_void_p(256)
    fp = ctypes.cast(p, ctypes.POINTER(ctypes.c_float))
    null = ctypes.POINTER(ctypes.c_float)()
    bad = ctypes.cast(ctypes.c_void_p(260), ctypes.POINTER(ctypes.c_float))
    args = (1, 64, 1, 16, 16, 0)
    assert lib.ckda_chunk_fwd_maps(p, p, p, fp, fp, null, fp, *args, 0, None, 0, None) == 1     # no M
    assert lib.ckda_chunk_fwd_maps(p, p, p, fp, fp, fp, null, *args, 0, None, 0, None) == 1     # no N
    assert lib.ckda_chunk_fwd_maps(None, p, p, fp, fp, fp, fp, *args, 0, None, 0, None) == 1    # no q
    assert lib.ckda_chunk_fwd_maps(p, p, p, fp, fp, bad, fp, *args, 0, None, 0, None) == 3
    assert lib.ckda_chunk_fwd_maps(p, p, p, fp, fp, fp, fp, *args, 0x200, None, 0, None) == 1   # mode
    assert lib.ckda_chunk_fwd_maps(p, p, p, fp, fp, fp, fp, 1, 64, 1, 0, 16, 0, 0, None, 0, None) == 1
    assert lib.ckda_chunk_fwd_maps(p, p, p, fp, fp, fp, fp, 1, 65536, 16, 128, 128, bf, 0, None, 0,
                                   None) == 6                                                  # workspace
    assert lib.ckda_chunk_fwd_maps(None, None, None, null, null, null, null, 0, 64, 4, 16, 16, 0, 0, None, 0,
                                   None) == 0                                                  # empty: nothing


def test_cp_prefix_argument_checks(lib):
    p = ctypes.cast(ctypes.c_void_p(256), ctypes.POINTER(ctypes.c_float))
    null = ctypes.POINTER(ctypes.c_float)()
    bad = ctypes.cast(ctypes.c_void_p(260), ctypes.POINTER(ctypes.c_float))
    assert lib.ckda_cp_prefix(p, 0, 1, 1, 16, 16, None) == 1          # R < 1
    assert lib.ckda_cp_prefix(p, 2, 1, 1, 0, 16, None) == 1           # d_k = 0
    assert lib.ckda_cp_prefix(p, 2, 1, 1, 16, 129, None) == 1         # d_v > 128
    assert lib.ckda_cp_prefix(null, 2, 1, 1, 16, 16, None) == 1
    assert lib.ckda_cp_prefix(bad, 2, 1, 1, 16, 16, None) == 3
    assert lib.ckda_cp_prefix(p, 2, 1, 1, 6, 16, None) == 2           # d_k not a multiple of 4
    assert lib.ckda_cp_prefix(null, 1, 1, 1, 16, 16, None) == 0       # one rank: nothing to chain
    assert lib.ckda_cp_prefix(null, 3, 0, 4, 16, 16, None) == 0       # no sequences


def test_python_binding_refuses_cpu_tensors_for_maps_and_prefix():
    """No CPU path: the map and prefix calls raise on host tensors before any library call."""
    import torch
    import delta_rule_attention_ckda_b200 as ck
    x = torch.zeros(1, 4, 1, 16)
    with pytest.raises(ValueError):
        ck.chunk_fwd_maps(x, x, x, x, torch.zeros(1, 4, 1))
    with pytest.raises(ValueError):
        ck.cp_prefix(torch.zeros(2, 1 * 1 * 16 * 32), 2, 1, 1, 16, 16)


def test_noalloc_capacity_getter(lib):
    """The fixed scratch capacity is read from the library, not restated in Python."""
    import delta_rule_attention_ckda_b200 as ck
    text = open(HEADER).read()
    assert "#define CKDA_NOALLOC_SCRATCH_BYTES ((size_t)20 << 20)" in text
    assert lib.ckda_noalloc_scratch_bytes() == 20 << 20
    assert ck.noalloc_scratch_bytes() == 20 << 20


class _FakeCuda(__import__("torch").Tensor):
    """A host tensor that reports a CUDA device: lets the binding's device checks run on a
    machine without a GPU (the checks raise before any library call or device access)."""
    _dev = None

    @property
    def device(self):
        return self._dev


def _on(t, dev):
    import torch
    f = t.as_subclass(_FakeCuda)
    f._dev = torch.device(dev)
    return f


@pytest.mark.parametrize("entry", ["chunk_fwd", "recurrent_fwd", "chunk_fwd_noalloc", "chunk_fwd_maps",
                                   "bwd", "decode_step"])
def test_python_binding_refuses_mixed_devices(entry):
    """Every tensor of a call must sit on the first tensor's device: the library launches on
    the current device with that device's stream, so a tensor on another GPU is an error,
    raised on the host before any launch."""
    import torch
    import delta_rule_attention_ckda_b200 as ck
    if entry == "decode_step":
        q, k, v, a = (_on(torch.zeros(2, 1, 16), "cuda:0") for _ in range(4))
        b = _on(torch.zeros(2, 1), "cuda:0")
        S = _on(torch.zeros(2, 1, 16, 16), "cuda:1")
        with pytest.raises(ValueError, match="cuda:1"):
            ck.decode_step(q, k, v, a, b, S)
        return
    q, v, a = (_on(torch.zeros(1, 4, 1, 16), "cuda:0") for _ in range(3))
    k = _on(torch.zeros(1, 4, 1, 16), "cuda:1")
    b = _on(torch.zeros(1, 4, 1), "cuda:0")
    args = (q, k, v, a, b)
    if entry == "bwd":
        args = args + (_on(torch.zeros(1, 4, 1, 16), "cuda:0"),)
    with pytest.raises(ValueError, match="cuda:1"):
        getattr(ck, entry)(*args)
