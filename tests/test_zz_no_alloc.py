"""ssd_fwd_noalloc: the allocation-free entry point for callers that cannot
allocate device memory (it takes its workspace from a fixed __device__ array
inside the library). Called through the C ABI and checked against ssd_fwd on
the same inputs, twice in a row, since every call reuses the same scratch.

This file sorts last so that a run stopping at its first failure has already
run every other test."""
import ctypes

import numpy as np
import pytest

import ssd_inputs
from _helpers import BF16_TOL, F32_TOL, rel_max_err, small_inputs, to_device

pytestmark = pytest.mark.gpu


def _lib():
    import mamba_ssd_layer_fwd_b200 as ssd
    lib = ssd.library()
    vp = ctypes.c_void_p
    lib.ssd_fwd_noalloc.restype = ctypes.c_int
    lib.ssd_fwd_noalloc.argtypes = [ctypes.POINTER(ssd.SsdParams), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                    ctypes.c_int]
    return lib


def _call_noalloc(inp, t, y, fin):
    import torch
    import mamba_ssd_layer_fwd_b200 as ssd
    lib = _lib()
    p = ssd.params_for(t["x"], t["B"], inp["chunk_len"], t["cu_seqlens"], inp.get("dt_softplus", True))
    ptr = lambda a: None if a is None else a.data_ptr()
    stream = torch.cuda.current_stream().cuda_stream or None
    return lib.ssd_fwd_noalloc(ctypes.byref(p), ptr(t["x"]), ptr(t["dt"]), ptr(t["A_log"]), ptr(t["B"]),
                               ptr(t["C"]), ptr(t["D"]), ptr(t["initial_states"]), ptr(t["cu_seqlens"]), ptr(y),
                               ptr(fin), stream, 1)


def _reference(inp, t):
    import mamba_ssd_layer_fwd_b200 as ssd
    return ssd.ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], chunk_len=inp["chunk_len"],
                       initial_states=t["initial_states"], cu_seqlens=t["cu_seqlens"],
                       return_final_states=True, check_status=True)


CASES = {
    "bf16_tensor_core": lambda: small_inputs(batch=2, seqlen=700, H=4, P=64, N=128, G=1, Q=256, init=True, seed=21),
    "bf16_varlen": lambda: small_inputs(H=4, P=64, N=64, G=1, Q=256, varlen=[300, 0, 129, 411], init=True, seed=22),
    "f32_tiny": lambda: ssd_inputs.make_inputs(ssd_inputs.workload("tiny_f32", with_initial_states=True,
                                                                   with_final_states=True)),
}


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_ssd_fwd_twice(name):
    import torch
    inp = CASES[name]()
    tol = F32_TOL if inp["io_dtype"] == "f32" else BF16_TOL
    t = to_device(inp)
    y_ref, f_ref = _reference(inp, t)
    torch.cuda.synchronize()
    y_ref = y_ref.double().cpu().numpy()
    f_ref = f_ref.double().cpu().numpy()
    for _ in range(2):   # the second call runs on the scratch the first one left behind
        y = torch.full_like(t["x"], float("nan"))
        fin = torch.full(f_ref.shape, float("nan"), dtype=torch.float32, device="cuda")
        rc = _call_noalloc(inp, t, y, fin)
        assert rc == 0, f"ssd_fwd_noalloc returned {rc}"
        torch.cuda.synchronize()
        assert rel_max_err(y.double().cpu().numpy(), y_ref) <= tol
        assert rel_max_err(fin.double().cpu().numpy(), f_ref) <= tol


def test_noalloc_rejects_problems_beyond_its_scratch():
    import torch
    import mamba_ssd_layer_fwd_b200 as ssd
    # the float32 path keeps fp32 chunk states: 64 chunks x 64 heads x 64 x 128 x 4 B = 128 MiB of workspace
    p = ssd.make_params(batch=1, seqlen=64 * 64, nheads=64, headdim=64, dstate=128, ngroups=1, chunk_len=64,
                        io_dtype="f32")
    assert ssd.workspace_size(p) > (16 << 20)
    lib = _lib()
    buf = torch.empty(16, dtype=torch.float32, device="cuda")
    a = buf.data_ptr()
    rc = lib.ssd_fwd_noalloc(ctypes.byref(p), a, a, a, a, a, None, None, None, a, None, None, 0)
    assert rc == -2   # SSD_ERR_UNSUPPORTED, nothing launched
