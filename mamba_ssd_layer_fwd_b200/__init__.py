"""Mamba-2 SSD forward layer for NVIDIA B200 (sm_100a): Python binding.

A thin ctypes layer over the C ABI in include/ssd_fwd.h (libssd_b200.so).
It only marshals arguments: PyTorch provides device memory and the stream,
every step of the computation runs in the library's CUDA kernels. There is no
CPU fallback; calling without the built library raises.

    import torch, mamba_ssd_layer_fwd_b200 as ssd
    y, final = ssd.ssd_fwd(x, dt, A_log, B, C, D, chunk_len=256,
                           return_final_states=True)

Shapes (contiguous): x (batch, seqlen, nheads, headdim), dt (batch, seqlen,
nheads), B and C (batch, seqlen, ngroups, dstate), A_log and D (nheads,)
float32, initial_states (nseq, nheads, headdim, dstate) float32, cu_seqlens
(nseq + 1,) int32 for a packed batch (batch == 1).
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

__all__ = [
    "ssd_fwd", "ssd_bwd", "ssd_fwd_summary", "ssd_state_combine", "ssd_decode_step", "SsdParams", "SsdStepParams", "SsdInstrumentation", "make_instrumentation", "workspace_size",
    "launch_count", "resolved_path", "library", "library_path", "STATUS", "PATHS", "SsdError",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "_lib", "libssd_b200.so")
_lib = None
_lock = threading.Lock()

STATUS = {0: "SSD_OK", -1: "SSD_ERR_INVALID_ARG", -2: "SSD_ERR_UNSUPPORTED", -3: "SSD_ERR_CUDA",
          -4: "SSD_ERR_TIMEOUT", -5: "SSD_ERR_BAD_SEQLENS"}
PATHS = {"auto": 0, "simt": 1, "tensor": 2}
DTYPES = {"f32": 0, "bf16": 1}

EXPORTED = ("ssd_fwd", "ssd_fwd_instrumented", "ssd_fwd_gated_norm", "ssd_bwd", "ssd_bwd_workspace_size", "ssd_fwd_summary",
            "ssd_fwd_summary_workspace_size", "ssd_state_combine", "ssd_decode_step", "ssd_fwd_workspace_size", "ssd_get_status", "ssd_fwd_launch_count",
            "ssd_fwd_resolved_path", "ssd_status_string", "ssd_abi_version")


class SsdError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({_status_string(code)})")


class SsdParams(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("seqlen", ctypes.c_int), ("nheads", ctypes.c_int),
        ("headdim", ctypes.c_int), ("dstate", ctypes.c_int), ("ngroups", ctypes.c_int),
        ("chunk_len", ctypes.c_int), ("num_seqs", ctypes.c_int), ("io_dtype", ctypes.c_int),
        ("dt_softplus", ctypes.c_int), ("path", ctypes.c_int),
    ]


class SsdInstrumentation(ctypes.Structure):
    """ssd_fwd_instrumentation: CUDA events recorded around the compute
    kernels, and the failure-injection switch used by the timeout test."""
    _fields_ = [
        ("ev_begin", ctypes.c_void_p), ("ev_main", ctypes.c_void_p), ("ev_end", ctypes.c_void_p),
        ("withhold_first_tile", ctypes.c_int),
    ]


class SsdStepParams(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("nheads", ctypes.c_int), ("headdim", ctypes.c_int),
        ("dstate", ctypes.c_int), ("ngroups", ctypes.c_int), ("io_dtype", ctypes.c_int),
        ("dt_softplus", ctypes.c_int),
    ]


def library_path() -> str:
    return _LIB_PATH


def library():
    """Load libssd_b200.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                                   "`python -m mamba_ssd_layer_fwd_b200.build`")
            lib = ctypes.CDLL(_LIB_PATH)
            vp, sz, i32, pp = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.POINTER(SsdParams)
            lib.ssd_fwd.restype = i32
            lib.ssd_fwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            lib.ssd_fwd_instrumented.restype = i32
            lib.ssd_fwd_instrumented.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp,
                                                 ctypes.POINTER(SsdInstrumentation)]
            lib.ssd_bwd.restype = i32
            lib.ssd_bwd.argtypes = [pp] + [vp] * 17 + [vp, sz, vp]
            lib.ssd_bwd_workspace_size.restype = sz
            lib.ssd_bwd_workspace_size.argtypes = [pp]
            lib.ssd_fwd_gated_norm.restype = i32
            lib.ssd_fwd_gated_norm.argtypes = [pp] + [vp] * 11 + [ctypes.c_float, vp, vp, vp, sz, vp]
            lib.ssd_fwd_summary.restype = i32
            lib.ssd_fwd_summary.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            lib.ssd_fwd_summary_workspace_size.restype = sz
            lib.ssd_fwd_summary_workspace_size.argtypes = [pp]
            lib.ssd_state_combine.restype = i32
            lib.ssd_state_combine.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp]
            lib.ssd_decode_step.restype = i32
            lib.ssd_decode_step.argtypes = [ctypes.POINTER(SsdStepParams), vp, vp, vp, vp, vp, vp, vp, vp, vp]
            lib.ssd_fwd_workspace_size.restype = sz
            lib.ssd_fwd_workspace_size.argtypes = [pp]
            lib.ssd_get_status.restype = i32
            lib.ssd_get_status.argtypes = [vp, vp]
            lib.ssd_fwd_launch_count.restype = i32
            lib.ssd_fwd_launch_count.argtypes = [pp]
            lib.ssd_fwd_resolved_path.restype = i32
            lib.ssd_fwd_resolved_path.argtypes = [pp]
            lib.ssd_status_string.restype = ctypes.c_char_p
            lib.ssd_status_string.argtypes = [i32]
            lib.ssd_abi_version.restype = i32
            lib.ssd_abi_version.argtypes = []
            _lib = lib
    return _lib


def _status_string(code: int) -> str:
    try:
        return library().ssd_status_string(int(code)).decode()
    except Exception:  # library missing: keep the error message usable
        return "?"


def make_params(*, batch, seqlen, nheads, headdim, dstate, ngroups, chunk_len, num_seqs=0,
                io_dtype="bf16", dt_softplus=True, path="auto") -> SsdParams:
    return SsdParams(int(batch), int(seqlen), int(nheads), int(headdim), int(dstate), int(ngroups),
                     int(chunk_len), int(num_seqs), DTYPES[io_dtype], int(bool(dt_softplus)),
                     PATHS[path])


def make_instrumentation(events=None, withhold_first_tile=False) -> SsdInstrumentation:
    """events = (begin, main, end) torch.cuda.Event objects (or None each)."""
    ev = [None, None, None] if events is None else [None if e is None else int(e.cuda_event) for e in events]
    return SsdInstrumentation(ev[0], ev[1], ev[2], int(bool(withhold_first_tile)))


def workspace_size(params: SsdParams) -> int:
    return int(library().ssd_fwd_workspace_size(ctypes.byref(params)))


def launch_count(params: SsdParams) -> int:
    return int(library().ssd_fwd_launch_count(ctypes.byref(params)))


def resolved_path(params: SsdParams) -> str:
    r = int(library().ssd_fwd_resolved_path(ctypes.byref(params)))
    return {1: "simt", 2: "tensor"}.get(r, "unsupported")


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


# ---------------------------------------------------------------- argument checks
# The kernels dereference every pointer they are given, over the extent the
# shapes imply: a host tensor, a tensor on another GPU, a short buffer or a
# strided view would be read or written out of bounds on the device.  These
# checks look at tensor metadata only (dtype, shape, contiguity, device), so
# they run before anything is launched.

def _check(name, t, dev, dtype, shape=None, required=False):
    """`t` (None when optional) must be a contiguous `dtype` tensor on `dev`
    with exactly `shape` (when given)."""
    if t is None:
        if required:
            raise ValueError(f"{name} is required")
        return
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != dev:
        raise ValueError(f"{name} must be on {dev}, got {t.device}")


def _io_dtype(x):
    import torch
    if x.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError(f"x must be bfloat16 or float32, got {x.dtype}")
    return x.dtype


def _check_workspace(workspace, dev):
    if workspace is not None and (not workspace.is_contiguous() or workspace.device != dev):
        raise ValueError(f"workspace must be a contiguous tensor on {dev}")


def _check_sequence_inputs(x, dt, A_log, B, cu_seqlens):
    """Shared checks of x, dt, A_log, B and cu_seqlens; returns
    (b, T, H, P, G, N, nseq)."""
    import torch
    io = _io_dtype(x)
    if x.dim() != 4:
        raise ValueError(f"x must be (batch, seqlen, nheads, headdim), got {tuple(x.shape)}")
    if B is None or B.dim() != 4:
        raise ValueError("B must be (batch, seqlen, ngroups, dstate)")
    dev = x.device
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    _check("x", x, dev, io)
    _check("dt", dt, dev, io, (b, T, H), required=True)
    _check("B", B, dev, io, (b, T, G, N))
    _check("A_log", A_log, dev, torch.float32, (H,), required=True)
    nseq = b
    if cu_seqlens is not None:
        _check("cu_seqlens", cu_seqlens, dev, torch.int32)
        if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
            raise ValueError("cu_seqlens must be 1-D with nseq + 1 >= 2 entries")
        nseq = cu_seqlens.numel() - 1
    return b, T, H, P, G, N, nseq


def _validate_fwd(x, dt, A_log, B, C, D=None, initial_states=None, cu_seqlens=None, y=None, final_states=None,
                  workspace=None, z=None, norm_weight=None, norm_bias=None):
    """Every tensor argument of ssd_fwd (metadata only); returns nseq."""
    import torch
    b, T, H, P, G, N, nseq = _check_sequence_inputs(x, dt, A_log, B, cu_seqlens)
    dev, io = x.device, x.dtype
    _check("C", C, dev, io, (b, T, G, N), required=True)
    _check("D", D, dev, torch.float32, (H,))
    _check("initial_states", initial_states, dev, torch.float32, (nseq, H, P, N))
    _check("y", y, dev, io, (b, T, H, P))
    _check("final_states", final_states, dev, torch.float32, (nseq, H, P, N))
    _check_workspace(workspace, dev)
    if z is None:
        if norm_weight is not None or norm_bias is not None:
            raise ValueError("norm_weight and norm_bias are used only together with z")
        return nseq
    _check("z", z, dev, io, (b, T, H, P))
    _check("norm_weight", norm_weight, dev, torch.float32, required=True)
    _check("norm_bias", norm_bias, dev, torch.float32)
    for name, t in (("norm_weight", norm_weight), ("norm_bias", norm_bias)):
        if t is not None and t.numel() != H * P:
            raise ValueError(f"{name} must hold nheads * headdim = {H * P} values, got {t.numel()}")
    return nseq


def _validate_summary(x, dt, A_log, B, cu_seqlens=None, workspace=None):
    """Every tensor argument of ssd_fwd_summary; returns nseq."""
    nseq = _check_sequence_inputs(x, dt, A_log, B, cu_seqlens)[-1]
    _check_workspace(workspace, x.device)
    return nseq


def _validate_bwd(x, dt, A_log, B, C, D, dy, initial_states=None, cu_seqlens=None, dfinal_states=None,
                  workspace=None):
    """Every tensor argument of ssd_bwd; returns nseq."""
    import torch
    b, T, H, P, G, N, nseq = _check_sequence_inputs(x, dt, A_log, B, cu_seqlens)
    dev, io = x.device, x.dtype
    _check("C", C, dev, io, (b, T, G, N), required=True)
    _check("D", D, dev, torch.float32, (H,))
    _check("dy", dy, dev, io, (b, T, H, P), required=True)
    _check("initial_states", initial_states, dev, torch.float32, (nseq, H, P, N))
    _check("dfinal_states", dfinal_states, dev, torch.float32, (nseq, H, P, N))
    _check_workspace(workspace, dev)
    return nseq


def _validate_decode(x, dt, A_log, B, C, D, state, y=None):
    """Every tensor argument of ssd_decode_step."""
    import torch
    io = _io_dtype(x)
    if x.dim() != 3:
        raise ValueError(f"x must be (batch, nheads, headdim), got {tuple(x.shape)}")
    if B is None or B.dim() != 3:
        raise ValueError("B must be (batch, ngroups, dstate)")
    dev = x.device
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    _check("x", x, dev, io)
    _check("dt", dt, dev, io, (b, H), required=True)
    _check("B", B, dev, io, (b, G, N))
    _check("C", C, dev, io, (b, G, N), required=True)
    _check("A_log", A_log, dev, torch.float32, (H,), required=True)
    _check("D", D, dev, torch.float32, (H,))
    _check("state", state, dev, torch.float32, (b, H, P, N), required=True)
    _check("y", y, dev, io, (b, H, P))


def _validate_combine(end_states_all, logdecay_all, rank, initial_states=None, out=None):
    """Every tensor argument of ssd_state_combine."""
    import torch
    if end_states_all is None or end_states_all.dim() != 5:
        raise ValueError("end_states_all must be (world, nseq, nheads, headdim, dstate)")
    dev = end_states_all.device
    world, nseq, H, P, N = end_states_all.shape
    _check("end_states_all", end_states_all, dev, torch.float32)
    _check("logdecay_all", logdecay_all, dev, torch.float32, (world, nseq, H), required=True)
    _check("initial_states", initial_states, dev, torch.float32, (nseq, H, P, N))
    _check("out", out, dev, torch.float32, (nseq, H, P, N))
    if not 0 <= int(rank) <= world:
        raise ValueError(f"rank must be in 0..{world}, got {rank}")


def _stream_handle(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) or None


def params_for(x, B, chunk_len: int, cu_seqlens=None, dt_softplus=True, path="auto") -> SsdParams:
    import torch
    if x.dtype == torch.bfloat16:
        io = "bf16"
    elif x.dtype == torch.float32:
        io = "f32"
    else:
        raise TypeError(f"x must be bfloat16 or float32, got {x.dtype}")
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    nseq = 0 if cu_seqlens is None else int(cu_seqlens.numel()) - 1
    return make_params(batch=b, seqlen=T, nheads=H, headdim=P, dstate=N, ngroups=G,
                       chunk_len=chunk_len, num_seqs=nseq, io_dtype=io, dt_softplus=dt_softplus,
                       path=path)


def ssd_fwd(x, dt, A_log, B, C, D=None, chunk_len: int = 256, initial_states=None,
            cu_seqlens=None, dt_softplus: bool = True, return_final_states: bool = False,
            y=None, final_states=None, workspace=None, stream=None, path: str = "auto",
            instrumentation: Optional[SsdInstrumentation] = None, check_status: bool = False,
            z=None, norm_weight=None, norm_bias=None, norm_eps: float = 1e-5):
    """SSD forward on the GPU through the C ABI. Returns y, or (y, final_states)
    when `return_final_states` is true (or `final_states` is given).

    x, dt, B, C share the io dtype (bfloat16 or float32); A_log, D,
    initial_states are float32; cu_seqlens is int32. Outputs and the workspace
    are allocated with torch on x's device unless passed in. `instrumentation`
    (make_instrumentation) routes the call through ssd_fwd_instrumented.
    With `z` (x's layout and dtype) and `norm_weight` (float32, nheads * headdim)
    the call returns the Mamba-2 block's normalised output instead of y:
    GroupNorm(y * silu(z)) over each head's channels, times norm_weight, plus
    norm_bias (ssd_fwd_gated_norm).
    """
    import torch
    lib = library()
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("ssd_fwd runs on CUDA tensors only")
    nseq = _validate_fwd(x, dt, A_log, B, C, D, initial_states, cu_seqlens, y, final_states, workspace, z,
                         norm_weight, norm_bias)
    p = params_for(x, B, chunk_len, cu_seqlens, dt_softplus, path)
    b, T, H, P = x.shape
    N = B.shape[3]
    if y is None:
        y = torch.empty_like(x)
    want_final = return_final_states or final_states is not None
    if want_final and final_states is None:
        final_states = torch.empty((nseq, H, P, N), dtype=torch.float32, device=dev)
    need = int(lib.ssd_fwd_workspace_size(ctypes.byref(p)))
    if need == 0:
        raise SsdError(-2 if lib.ssd_fwd_resolved_path(ctypes.byref(p)) == -1 else -1, "ssd_fwd_workspace_size")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    st = _stream_handle(stream)
    args = (ctypes.byref(p), _ptr(x), _ptr(dt), _ptr(A_log), _ptr(B), _ptr(C), _ptr(D),
            _ptr(initial_states), _ptr(cu_seqlens), _ptr(y), _ptr(final_states),
            _ptr(workspace), workspace.numel() * workspace.element_size(), st)
    if z is not None:
        rc = lib.ssd_fwd_gated_norm(ctypes.byref(p), _ptr(x), _ptr(dt), _ptr(A_log), _ptr(B), _ptr(C), _ptr(D),
                                    _ptr(initial_states), _ptr(cu_seqlens), _ptr(z), _ptr(norm_weight),
                                    _ptr(norm_bias), float(norm_eps), _ptr(y), _ptr(final_states),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(), st)
    elif instrumentation is None:
        rc = lib.ssd_fwd(*args)
    else:
        rc = lib.ssd_fwd_instrumented(*args, ctypes.byref(instrumentation))
    if rc != 0:
        raise SsdError(rc, "ssd_fwd")
    if check_status:
        rc = lib.ssd_get_status(_ptr(workspace), st)
        if rc != 0:
            raise SsdError(rc, "ssd_fwd (device status)")
    return (y, final_states) if want_final else y


def ssd_fwd_summary(x, dt, A_log, B, chunk_len: int = 256, cu_seqlens=None, dt_softplus: bool = True,
                    path: str = "auto", workspace=None, stream=None, check_status: bool = False):
    """Every sequence's end state from a zero state, (nseq, H, P, N) float32,
    and its total log decay sum_t delta_t A, (nseq, H) float32, through the
    C ABI (the summary one worker of a context-parallel forward exchanges)."""
    import torch
    lib = library()
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("ssd_fwd_summary runs on CUDA tensors only")
    nseq = _validate_summary(x, dt, A_log, B, cu_seqlens, workspace)
    p = params_for(x, B, chunk_len, cu_seqlens, dt_softplus, path)
    b, T, H, P = x.shape
    N = B.shape[3]
    S = torch.empty((nseq, H, P, N), dtype=torch.float32, device=dev)
    L = torch.empty((nseq, H), dtype=torch.float32, device=dev)
    need = int(lib.ssd_fwd_summary_workspace_size(ctypes.byref(p)))
    if need == 0:
        raise SsdError(-2 if lib.ssd_fwd_resolved_path(ctypes.byref(p)) == -1 else -1, "ssd_fwd_summary_workspace_size")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    st = _stream_handle(stream)
    rc = lib.ssd_fwd_summary(ctypes.byref(p), _ptr(x), _ptr(dt), _ptr(A_log), _ptr(B), _ptr(cu_seqlens), _ptr(S),
                             _ptr(L), _ptr(workspace), workspace.numel() * workspace.element_size(), st)
    if rc != 0:
        raise SsdError(rc, "ssd_fwd_summary")
    if check_status:
        rc = lib.ssd_get_status(_ptr(workspace), st)
        if rc != 0:
            raise SsdError(rc, "ssd_fwd_summary (device status)")
    return S, L


def ssd_state_combine(end_states_all, logdecay_all, rank: int, initial_states=None, out=None, stream=None):
    """Fold the summaries of workers 0 .. rank-1 (end_states_all (world, nseq,
    H, P, N), logdecay_all (world, nseq, H), float32) from initial_states:
    the state entering worker `rank` (rank == world: after the last piece)."""
    import torch
    lib = library()
    if end_states_all.device.type != "cuda":
        raise ValueError("ssd_state_combine runs on CUDA tensors only")
    _validate_combine(end_states_all, logdecay_all, rank, initial_states, out)
    world, nseq, H, P, N = end_states_all.shape
    if out is None:
        out = torch.empty((nseq, H, P, N), dtype=torch.float32, device=end_states_all.device)
    rc = lib.ssd_state_combine(int(world), int(rank), int(nseq), int(H), int(P), int(N), _ptr(end_states_all),
                               _ptr(logdecay_all), _ptr(initial_states), _ptr(out), _stream_handle(stream))
    if rc != 0:
        raise SsdError(rc, "ssd_state_combine")
    return out


def ssd_bwd(x, dt, A_log, B, C, D, dy, initial_states=None, cu_seqlens=None, dfinal_states=None,
            dt_softplus: bool = True, want_dinitial: bool = True, workspace=None, stream=None,
            check_status: bool = False) -> dict:
    """Gradients of L given dy = dL/dy (and dL/dfinal_states) through the C ABI.
    Returns float32 tensors: dx, ddt (with respect to the raw dt), dA_log, dB,
    dC, dD and dinitial_states (when `want_dinitial`), each shaped like its input."""
    import torch
    lib = library()
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("ssd_bwd runs on CUDA tensors only")
    nseq = _validate_bwd(x, dt, A_log, B, C, D, dy, initial_states, cu_seqlens, dfinal_states, workspace)
    p = params_for(x, B, 256, cu_seqlens, dt_softplus, "auto")
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"dx": torch.empty(x.shape, **f32), "ddt": torch.empty(dt.shape, **f32),
           "dA_log": torch.empty(H, **f32), "dB": torch.empty(B.shape, **f32), "dC": torch.empty(C.shape, **f32),
           "dD": torch.empty(H, **f32),
           "dinitial_states": torch.empty((nseq, H, P, N), **f32) if want_dinitial else None}
    need = int(lib.ssd_bwd_workspace_size(ctypes.byref(p)))
    if need == 0:
        raise SsdError(-2, "ssd_bwd_workspace_size")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    st = _stream_handle(stream)
    rc = lib.ssd_bwd(ctypes.byref(p), _ptr(x), _ptr(dt), _ptr(A_log), _ptr(B), _ptr(C), _ptr(D),
                     _ptr(initial_states), _ptr(cu_seqlens), _ptr(dy), _ptr(dfinal_states),
                     _ptr(out["dx"]), _ptr(out["ddt"]), _ptr(out["dA_log"]), _ptr(out["dB"]), _ptr(out["dC"]),
                     _ptr(out["dD"]), _ptr(out["dinitial_states"]), _ptr(workspace),
                     workspace.numel() * workspace.element_size(), st)
    if rc != 0:
        raise SsdError(rc, "ssd_bwd")
    if check_status:
        rc = lib.ssd_get_status(_ptr(workspace), st)
        if rc != 0:
            raise SsdError(rc, "ssd_bwd (device status)")
    return out


def ssd_decode_step(x, dt, A_log, B, C, D, state, y=None, dt_softplus: bool = True, stream=None):
    """One decoding step of every row through the C ABI; updates `state` in
    place and returns y.

    x (batch, nheads, headdim) and dt (batch, nheads), B and C (batch, ngroups,
    dstate) share the io dtype (bfloat16 or float32); A_log, D (nheads) and
    state (batch, nheads, headdim, dstate) are float32 on x's device.
    """
    import torch
    lib = library()
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("ssd_decode_step runs on CUDA tensors only")
    _validate_decode(x, dt, A_log, B, C, D, state, y)
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    if y is None:
        y = torch.empty_like(x)
    p = SsdStepParams(int(b), int(H), int(P), int(N), int(G), DTYPES["bf16" if x.dtype == torch.bfloat16 else "f32"],
                      int(bool(dt_softplus)))
    rc = lib.ssd_decode_step(ctypes.byref(p), _ptr(x), _ptr(dt), _ptr(A_log), _ptr(B), _ptr(C), _ptr(D),
                             _ptr(state), _ptr(y), _stream_handle(stream))
    if rc != 0:
        raise SsdError(rc, "ssd_decode_step")
    return y
