"""ctypes binding of libckda.so (argument marshalling only; every step runs in CUDA).

The functions here take torch CUDA tensors, check dtype/shape/contiguity on the host,
and pass raw device pointers plus the current CUDA stream to the C ABI declared in
include/ckda.h. There is no fallback: if the library is missing or the tensors are
not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libckda.so")

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported request", 3: "pointer not 16-byte aligned",
          4: "CUDA error", 5: "device wait timed out", 6: "workspace missing or too small"}
F32, BF16 = 0, 1
PATH_RECURRENT, PATH_CHUNK_TC = 0, 1


class CkdaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, 'unknown')} (status {status})")
        self.status = status


_lib = None


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libckda.so (built in-tree by build.py). Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"libckda.so not found at {path}; run delta_rule_attention_ckda_b200/build.py")
    lib = ctypes.CDLL(path)
    vp, fp, i, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.ckda_abi_version.restype = i
    lib.ckda_status_string.argtypes = [i]
    lib.ckda_status_string.restype = ctypes.c_char_p
    lib.ckda_chunk_fwd_workspace_bytes.argtypes = [i] * 6
    lib.ckda_chunk_fwd_workspace_bytes.restype = sz
    lib.ckda_chunk_fwd_path.argtypes = [i] * 6
    lib.ckda_chunk_fwd_path.restype = i
    lib.ckda_chunk_fwd_segments.argtypes = [i] * 6
    lib.ckda_chunk_fwd_segments.restype = i
    lib.ckda_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp] + [i] * 6 + [vp, sz, vp]
    lib.ckda_chunk_fwd.restype = i
    lib.ckda_recurrent_fwd.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp] + [i] * 6 + [vp]
    lib.ckda_recurrent_fwd.restype = i
    lib.ckda_chunk_fwd_ex.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp] + [i] * 7 + [vp, sz, vp]
    lib.ckda_chunk_fwd_ex.restype = i
    lib.ckda_recurrent_fwd_ex.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp] + [i] * 7 + [vp]
    lib.ckda_recurrent_fwd_ex.restype = i
    lib.ckda_chunk_fwd_noalloc.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp] + [i] * 7 + [vp]
    lib.ckda_chunk_fwd_noalloc.restype = i
    lib.ckda_noalloc_scratch_bytes.argtypes = []
    lib.ckda_noalloc_scratch_bytes.restype = sz
    lib.ckda_chunk_fwd_maps_workspace_bytes.argtypes = [i] * 6
    lib.ckda_chunk_fwd_maps_workspace_bytes.restype = sz
    lib.ckda_chunk_fwd_maps.argtypes = [vp, vp, vp, fp, fp, fp, fp] + [i] * 7 + [vp, sz, vp]
    lib.ckda_chunk_fwd_maps.restype = i
    lib.ckda_cp_prefix.argtypes = [fp] + [i] * 5 + [vp]
    lib.ckda_cp_prefix.restype = i
    lib.ckda_bwd_workspace_bytes.argtypes = [i] * 6
    lib.ckda_bwd_workspace_bytes.restype = sz
    lib.ckda_bwd_workspace_bytes_ex.argtypes = [i] * 7
    lib.ckda_bwd_workspace_bytes_ex.restype = sz
    lib.ckda_bwd_path.argtypes = [i] * 7
    lib.ckda_bwd_path.restype = i
    lib.ckda_bwd.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, fp, fp, fp, fp, fp, fp] + [i] * 7 + [vp, sz, vp]
    lib.ckda_bwd.restype = i
    lib.ckda_decode_step.argtypes = [vp, vp, vp, fp, fp, fp, fp] + [i] * 5 + [vp]
    lib.ckda_decode_step.restype = i
    lib.ckda_decode_step_ex.argtypes = [vp, vp, vp, fp, fp, fp, fp] + [i] * 6 + [vp]
    lib.ckda_decode_step_ex.restype = i
    lib.ckda_get_device_error.argtypes = [vp]
    lib.ckda_get_device_error.restype = i
    _lib = lib
    return lib


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(t: torch.Tensor, name: str, shape, dtype=None, device=None):
    """Type, device, shape, dtype and contiguity of one tensor argument. `device`: the device
    every tensor of the call must be on (that of its first tensor)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the call's tensors are on {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _device(t: torch.Tensor, name: str = "q") -> torch.device:
    """The device of a call: that of its first tensor, which must be a CUDA tensor. The
    library launches on the current device, so every call runs under
    torch.cuda.device(this device)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    return t.device


def _stream(stream, device: torch.device) -> ctypes.c_void_p:
    """The stream to launch on: the given one, which must belong to `device`, else the
    current stream of `device`."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the call's tensors are on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _raise(status: int, where: str):
    if status != 0:
        raise CkdaError(status, where)


def workspace_bytes(B, T, H, dk, dv, dtype=torch.bfloat16) -> int:
    return int(load().ckda_chunk_fwd_workspace_bytes(B, T, H, dk, dv, _dt(torch.empty(0, dtype=dtype))))


def chunk_path(B, T, H, dk, dv, dtype=torch.bfloat16) -> int:
    return int(load().ckda_chunk_fwd_path(B, T, H, dk, dv, _dt(torch.empty(0, dtype=dtype))))


def chunk_segments(B, T, H, dk, dv, dtype=torch.bfloat16) -> int:
    """Segments per sequence ckda_chunk_fwd runs side by side on the current device (1 = one pass)."""
    return int(load().ckda_chunk_fwd_segments(B, T, H, dk, dv, _dt(torch.empty(0, dtype=dtype))))


def _fwd_common(q, k, v, alpha, beta, S0, o, S_T):
    dev = _device(q)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _check(q, "q", (B, T, H, dk), None, dev)
    _check(k, "k", (B, T, H, dk), dt, dev)
    _check(v, "v", (B, T, H, dv), dt, dev)
    _check(alpha, "alpha", (B, T, H, dk), torch.float32, dev)
    _check(beta, "beta", (B, T, H), torch.float32, dev)
    if S0 is not None:
        _check(S0, "S0", (B, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(B, T, H, dv, device=dev, dtype=torch.float32)
    _check(o, "o", (B, T, H, dv), torch.float32, dev)
    if S_T is not None:
        _check(S_T, "S_T", (B, H, dk, dv), torch.float32, dev)
    return B, T, H, dk, dv, _dt(q), o


GATES = {"signed": 0, "log": 1}       # ckda_gate_t: alpha in [-1,1], or g = ln(alpha) (KDA form)


OPT_NORMALIZE_QK = 0x100              # CKDA_OPT_NORMALIZE_QK


def _gate(gate: str) -> int:
    if gate not in GATES:
        raise ValueError(f"gate must be one of {sorted(GATES)}, got {gate!r}")
    return GATES[gate]


def _mode(gate: str, normalize_qk: bool) -> int:
    """The C mode argument: the gate form, OR-ed with CKDA_OPT_NORMALIZE_QK if asked."""
    return _gate(gate) | (OPT_NORMALIZE_QK if normalize_qk else 0)


def chunk_fwd(q, k, v, alpha, beta, S0=None, *, o=None, S_T=None, want_state=True,
              workspace=None, stream=None, gate="signed",
              normalize_qk=False) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """ckda_chunk_fwd_ex. Returns (o, S_T). `alpha` is the gate in the form `gate` names:
    "signed" (alpha in [-1,1], CKDA) or "log" (g = ln(alpha) of a non-negative gate, KDA).
    normalize_qk: q and k are L2-normalised per token and head inside the kernels.
    Allocates o / S_T / workspace with torch when not given (the library never allocates)."""
    B, T, H, dk, dv, dt, o = _fwd_common(q, k, v, alpha, beta, S0, o, S_T)
    dev = q.device
    if S_T is None and want_state:
        S_T = torch.empty(B, H, dk, dv, device=dev, dtype=torch.float32)
    lib = load()
    with torch.cuda.device(dev):
        need = int(lib.ckda_chunk_fwd_workspace_bytes(B, T, H, dk, dv, dt))
        if need and workspace is None:
            workspace = torch.empty(need, device=dev, dtype=torch.uint8)
        if workspace is not None:
            _check(workspace, "workspace", tuple(workspace.shape), None, dev)
        wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = lib.ckda_chunk_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S0), _ptr(o),
                                   _ptr(S_T), B, T, H, dk, dv, dt, _mode(gate, normalize_qk), _ptr(workspace),
                                   wbytes, _stream(stream, dev))
    _raise(st, "ckda_chunk_fwd_ex")
    return o, S_T


def noalloc_scratch_bytes() -> int:
    """Capacity of the fixed device scratch of chunk_fwd_noalloc (CKDA_NOALLOC_SCRATCH_BYTES,
    read from the library)."""
    return int(load().ckda_noalloc_scratch_bytes())


def chunk_fwd_noalloc(q, k, v, alpha, beta, S0=None, *, o=None, S_T=None, want_state=True,
                      stream=None, gate="signed",
                      normalize_qk=False) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """ckda_chunk_fwd_noalloc: ckda_chunk_fwd_ex on the library's fixed device scratch
    (no workspace argument; the call allocates nothing). Raises CkdaError(WORKSPACE)
    when the problem needs more than noalloc_scratch_bytes() of scratch. o / S_T are
    allocated with torch only when not given."""
    B, T, H, dk, dv, dt, o = _fwd_common(q, k, v, alpha, beta, S0, o, S_T)
    dev = q.device
    if S_T is None and want_state:
        S_T = torch.empty(B, H, dk, dv, device=dev, dtype=torch.float32)
    with torch.cuda.device(dev):
        st = load().ckda_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S0),
                                           _ptr(o), _ptr(S_T), B, T, H, dk, dv, dt, _mode(gate, normalize_qk),
                                           _stream(stream, dev))
    _raise(st, "ckda_chunk_fwd_noalloc")
    return o, S_T


def maps_workspace_bytes(B, T, H, dk, dv, dtype=torch.bfloat16) -> int:
    return int(load().ckda_chunk_fwd_maps_workspace_bytes(B, T, H, dk, dv, _dt(torch.empty(0, dtype=dtype))))


def chunk_fwd_maps(q, k, v, alpha, beta, *, M=None, N=None, workspace=None, stream=None, gate="signed",
                   normalize_qk=False) -> Tuple[torch.Tensor, torch.Tensor]:
    """ckda_chunk_fwd_maps: the affine map S_T = M S_0 + N of every (b, h) sequence.
    Returns (M [B,H,dk,dk], N [B,H,dk,dv]), fp32; allocated with torch when not given."""
    dev = _device(q)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _check(q, "q", (B, T, H, dk), None, dev)
    _check(k, "k", (B, T, H, dk), dt, dev)
    _check(v, "v", (B, T, H, dv), dt, dev)
    _check(alpha, "alpha", (B, T, H, dk), torch.float32, dev)
    _check(beta, "beta", (B, T, H), torch.float32, dev)
    f32 = dict(device=dev, dtype=torch.float32)
    M = torch.empty(B, H, dk, dk, **f32) if M is None else M
    N = torch.empty(B, H, dk, dv, **f32) if N is None else N
    _check(M, "M", (B, H, dk, dk), torch.float32, dev)
    _check(N, "N", (B, H, dk, dv), torch.float32, dev)
    lib = load()
    with torch.cuda.device(dev):
        need = int(lib.ckda_chunk_fwd_maps_workspace_bytes(B, T, H, dk, dv, _dt(q)))
        if need and workspace is None:
            workspace = torch.empty(need, device=dev, dtype=torch.uint8)
        if workspace is not None:
            _check(workspace, "workspace", tuple(workspace.shape), None, dev)
        wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = lib.ckda_chunk_fwd_maps(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(M), _ptr(N),
                                     B, T, H, dk, dv, _dt(q), _mode(gate, normalize_qk), _ptr(workspace),
                                     wbytes, _stream(stream, dev))
    _raise(st, "ckda_chunk_fwd_maps")
    return M, N


def cp_prefix(blocks: torch.Tensor, R: int, B: int, H: int, dk: int, dv: int, stream=None) -> torch.Tensor:
    """ckda_cp_prefix, in place on `blocks` ([R, B*H*dk*(dk+dv)] fp32, rank r's M then N)."""
    dev = _device(blocks, "blocks")
    _check(blocks, "blocks", (R, B * H * dk * (dk + dv)), torch.float32, dev)
    with torch.cuda.device(dev):
        st = load().ckda_cp_prefix(_ptr(blocks), R, B, H, dk, dv, _stream(stream, dev))
    _raise(st, "ckda_cp_prefix")
    return blocks


BWD_RECURRENT, BWD_CHUNK_TC = 0, 1


def bwd_workspace_bytes(B, T, H, dk, dv, dtype=torch.bfloat16, gate="signed", normalize_qk=False) -> int:
    return int(load().ckda_bwd_workspace_bytes_ex(B, T, H, dk, dv, _dt(torch.empty(0, dtype=dtype)),
                                                  _mode(gate, normalize_qk)))


def bwd_path(B, T, H, dk, dv, dtype=torch.bfloat16, gate="signed", normalize_qk=False) -> int:
    """ckda_bwd_path: BWD_CHUNK_TC (tensor cores) or BWD_RECURRENT (CUDA cores, fp32)."""
    return int(load().ckda_bwd_path(B, T, H, dk, dv, _dt(torch.empty(0, dtype=dtype)), _mode(gate, normalize_qk)))


def bwd(q, k, v, alpha, beta, grad_o, S0=None, grad_S_T=None, *, want_dS0=True, grads=None,
        workspace=None, stream=None, gate="signed", normalize_qk=False):
    """ckda_bwd: gradients of L = <grad_o, o> + <grad_S_T, S_T> for the forward of chunk_fwd.
    Returns a dict with dq, dk, dv, dalpha (dL/dg for gate="log"), dbeta and dS0 (None
    unless want_dS0). Output tensors may be passed in `grads` (same keys); the workspace
    is allocated with torch when not given."""
    dev = _device(q)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _check(q, "q", (B, T, H, dk), None, dev)
    _check(k, "k", (B, T, H, dk), dt, dev)
    _check(v, "v", (B, T, H, dv), dt, dev)
    _check(alpha, "alpha", (B, T, H, dk), torch.float32, dev)
    _check(beta, "beta", (B, T, H), torch.float32, dev)
    _check(grad_o, "grad_o", (B, T, H, dv), torch.float32, dev)
    if S0 is not None:
        _check(S0, "S0", (B, H, dk, dv), torch.float32, dev)
    if grad_S_T is not None:
        _check(grad_S_T, "grad_S_T", (B, H, dk, dv), torch.float32, dev)
    g = dict(grads or {})
    f32 = dict(device=dev, dtype=torch.float32)
    shapes = {"dq": (B, T, H, dk), "dk": (B, T, H, dk), "dv": (B, T, H, dv), "dalpha": (B, T, H, dk),
              "dbeta": (B, T, H), "dS0": (B, H, dk, dv)}
    for name, shp in shapes.items():
        if name == "dS0" and not want_dS0:
            g[name] = None
            continue
        if g.get(name) is None:
            g[name] = torch.empty(shp, **f32)
        _check(g[name], name, shp, torch.float32, dev)
    lib = load()
    with torch.cuda.device(dev):
        need = int(lib.ckda_bwd_workspace_bytes_ex(B, T, H, dk, dv, _dt(q), _mode(gate, normalize_qk)))
        if need and workspace is None:
            workspace = torch.empty(need, device=dev, dtype=torch.uint8)
        if workspace is not None:
            _check(workspace, "workspace", tuple(workspace.shape), None, dev)
        wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = lib.ckda_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S0), _ptr(grad_o),
                          _ptr(grad_S_T), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dalpha"]),
                          _ptr(g["dbeta"]), _ptr(g["dS0"]), B, T, H, dk, dv, _dt(q),
                          _mode(gate, normalize_qk), _ptr(workspace), wbytes, _stream(stream, dev))
    _raise(st, "ckda_bwd")
    return g


def recurrent_fwd(q, k, v, alpha, beta, S0=None, *, o=None, S_T=None, want_state=True,
                  stream=None, gate="signed", normalize_qk=False) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """ckda_recurrent_fwd_ex (fp32 SIMT token-by-token kernel). Returns (o, S_T)."""
    B, T, H, dk, dv, dt, o = _fwd_common(q, k, v, alpha, beta, S0, o, S_T)
    dev = q.device
    if S_T is None and want_state:
        S_T = torch.empty(B, H, dk, dv, device=dev, dtype=torch.float32)
    with torch.cuda.device(dev):
        st = load().ckda_recurrent_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S0),
                                          _ptr(o), _ptr(S_T), B, T, H, dk, dv, dt, _mode(gate, normalize_qk),
                                          _stream(stream, dev))
    _raise(st, "ckda_recurrent_fwd_ex")
    return o, S_T


def decode_step(q, k, v, alpha, beta, S, *, o=None, stream=None, gate="signed",
                normalize_qk=False) -> torch.Tensor:
    """ckda_decode_step_ex: updates S [N,H,dk,dv] in place, returns o [N,H,dv]. `alpha` is
    the gate in the form `gate` names; normalize_qk L2-normalises q and k in the step."""
    dev = _device(q)
    N, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _check(q, "q", (N, H, dk), None, dev)
    _check(k, "k", (N, H, dk), dt, dev)
    _check(v, "v", (N, H, dv), dt, dev)
    _check(alpha, "alpha", (N, H, dk), torch.float32, dev)
    _check(beta, "beta", (N, H), torch.float32, dev)
    _check(S, "S", (N, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(N, H, dv, device=dev, dtype=torch.float32)
    _check(o, "o", (N, H, dv), torch.float32, dev)
    with torch.cuda.device(dev):
        st = load().ckda_decode_step_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S),
                                        _ptr(o), N, H, dk, dv, _dt(q), _mode(gate, normalize_qk),
                                        _stream(stream, dev))
    _raise(st, "ckda_decode_step_ex")
    return o


def get_device_error(stream=None, device=None) -> int:
    """ckda_get_device_error on `device` (default: the stream's, else the current device):
    synchronises the stream; returns the status code."""
    if device is None:
        device = stream.device if stream is not None else torch.device("cuda", torch.cuda.current_device())
    device = torch.device(device)
    with torch.cuda.device(device):
        return int(load().ckda_get_device_error(_stream(stream, device)))
