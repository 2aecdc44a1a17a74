"""The C-ABI library: it loads, exports every declared entry point, and its
host-side validation rejects bad arguments before touching the device (no GPU
needed: every call here fails validation or only queries sizes)."""
import ctypes
import os
import re

import pytest

import mamba_ssd_layer_fwd_b200 as ssd
from mamba_ssd_layer_fwd_b200 import build as ssd_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    ssd_build.build()
    return ssd.library()


def declared_symbols():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            body = src.split("#endif\n", 1)[-1] if "#define SSD_API" in src else src
            names += re.findall(r"^SSD_API\s+[\w\s\*]*?\b(\w+)\s*\(", body, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert "ssd_fwd" in names and "ssd_fwd_workspace_size" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert lib.ssd_abi_version() == 2


def test_only_abi_symbols_exported(lib):
    # the .so hides everything but the C ABI (-fvisibility=hidden)
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", ssd.library_path()], capture_output=True,
                         text=True).stdout
    ours = {l.split()[-1] for l in out.splitlines() if " T " in l and l.split()[-1].startswith("ssd_")}
    assert ours == set(declared_symbols())


def params(**kw):
    base = dict(batch=2, seqlen=2048, nheads=24, headdim=64, dstate=64, ngroups=1, chunk_len=256,
                num_seqs=0, io_dtype="bf16", dt_softplus=True, path="auto")
    base.update(kw)
    return ssd.make_params(**base)


def test_workspace_size_valid_and_invalid(lib):
    assert ssd.workspace_size(params()) > 0
    assert ssd.workspace_size(params(path="simt")) > 0
    for bad in (dict(nheads=24, ngroups=5), dict(chunk_len=100), dict(batch=0), dict(headdim=0),
                dict(num_seqs=3, batch=2), dict(dstate=300), dict(headdim=256)):
        assert ssd.workspace_size(params(**bad)) == 0, bad


def test_resolved_path_and_launch_count(lib):
    p = params(path="simt")
    assert ssd.resolved_path(p) == "simt"
    assert ssd.launch_count(p) == 5
    assert ssd.resolved_path(params(io_dtype="f32")) == "simt"


def _call(lib, p, **ptrs):
    args = dict(x=16, dt=16, A_log=16, B=16, C=16, D=None, init=None, cu=None, y=16, final=None,
                ws=256, ws_bytes=1 << 40)
    args.update(ptrs)
    return lib.ssd_fwd(ctypes.byref(p), args["x"], args["dt"], args["A_log"], args["B"], args["C"],
                       args["D"], args["init"], args["cu"], args["y"], args["final"], args["ws"],
                       args["ws_bytes"], None)


def test_validation_errors(lib):
    INVALID, UNSUPPORTED = -1, -2
    assert lib.ssd_fwd(None, 16, 16, 16, 16, 16, None, None, None, 16, None, 256, 1 << 40, None) == INVALID
    assert _call(lib, params(), x=None) == INVALID
    assert _call(lib, params(), y=None) == INVALID
    assert _call(lib, params(), ws=None) == INVALID
    assert _call(lib, params(), x=24) == INVALID                 # misaligned
    assert _call(lib, params(), ws=128) == INVALID               # workspace not 256-aligned
    assert _call(lib, params(), ws_bytes=16) == INVALID          # workspace too small
    assert _call(lib, params(nheads=6, ngroups=4)) == INVALID
    assert _call(lib, params(chunk_len=32)) == INVALID
    assert _call(lib, params(num_seqs=2, batch=1)) == INVALID    # cu_seqlens missing
    assert _call(lib, params(), cu=16) == INVALID                # cu_seqlens without num_seqs
    assert _call(lib, params(headdim=200)) == UNSUPPORTED
    assert _call(lib, params(path="tensor", io_dtype="f32")) == UNSUPPORTED


def test_status_strings(lib):
    for code in ssd.STATUS:
        assert lib.ssd_status_string(code)


def _step(lib, batch=2, nheads=4, headdim=64, dstate=64, ngroups=1, io="bf16", softplus=1, **ptrs):
    p = ssd.SsdStepParams(batch, nheads, headdim, dstate, ngroups, ssd.DTYPES[io], softplus)
    a = dict(x=16, dt=16, A_log=16, B=16, C=16, D=None, state=16, y=16)
    a.update(ptrs)
    return lib.ssd_decode_step(ctypes.byref(p), a["x"], a["dt"], a["A_log"], a["B"], a["C"], a["D"],
                               a["state"], a["y"], None)


def test_decode_step_validation(lib):
    # every call is rejected on the host before anything is launched
    assert _step(lib, nheads=6, ngroups=4) == -1                 # H % G
    assert _step(lib, dstate=0) == -1
    assert _step(lib, softplus=2) == -1
    assert _step(lib, dstate=30) == -2                           # not a multiple of 4
    assert _step(lib, dstate=260) == -2                          # above 256
    assert _step(lib, B=None) == -1
    assert _step(lib, state=None) == -1
    assert _step(lib, B=24) == -1                                # misaligned vector operand
    assert _step(lib, state=8) == -1
    assert _step(lib, batch=0, x=None, B=None) == 0              # nothing to do


def _tc_params(batch, seqlen, nheads, dstate, ngroups=1, num_seqs=0):
    return ssd.make_params(batch=batch, seqlen=seqlen, nheads=nheads, headdim=64, dstate=dstate,
                           ngroups=ngroups, chunk_len=256, num_seqs=num_seqs, io_dtype="bf16", path="auto")


def test_tensor_path_work_split(lib):
    """Host-side work planning of the tensor-core path (no GPU needed): how
    many kernels one forward launches for each kind of problem."""
    # 8 x 80 heads: 320 two-head items = 2 whole waves of 148 in one launch; the
    # 24 pairs left over as 48 one-head items in a second launch
    p = _tc_params(8, 2048, 80, 128)
    assert ssd.resolved_path(p) == "tensor"
    assert ssd.launch_count(p) == 2
    # exactly one wave of two-head items: one launch
    assert ssd.launch_count(_tc_params(148, 256, 2, 64)) == 1
    # one short row: one item, one launch
    assert ssd.launch_count(_tc_params(1, 128, 2, 64)) == 1
    # a 16K-token row with 32 heads: 16 pairs cut into 9 segments, state-only walks,
    # exchange and full walks in one launch
    assert ssd.launch_count(_tc_params(1, 16384, 32, 256, ngroups=8)) == 1
    # 160 two-head items of 3 blocks: 148 whole rows + 24 one-head items
    assert ssd.launch_count(_tc_params(2, 300, 160, 64)) == 2
    # packed variable-length batch: planner + walk when there are enough items for
    # the SMs (16 x 24 here), + state pass + scan when it must be cut (one sequence)
    assert ssd.launch_count(_tc_params(1, 32768, 48, 128, num_seqs=16)) == 2
    assert ssd.launch_count(_tc_params(1, 32768, 48, 128, num_seqs=1)) == 4
    assert ssd.launch_count(_tc_params(1, 512, 48, 128, num_seqs=4)) == 2
    # the segmented launches keep their segment states in the workspace: 16 pairs x 9 segments
    # x 2 heads x 64 x 256 fp32 for the 16K row; the 4 pairs left over after a whole wave of
    # 148 rows of 32 blocks are cut into 32 segments; the one-head tail needs none
    seg16k = 16 * 9 * 2 * 64 * 256 * 4
    assert ssd.workspace_size(_tc_params(1, 16384, 32, 256, ngroups=8)) >= seg16k
    assert ssd.launch_count(_tc_params(4, 4096, 76, 64)) == 2
    assert ssd.workspace_size(_tc_params(4, 4096, 76, 64)) >= 4 * 32 * 2 * 64 * 64 * 4
    assert ssd.workspace_size(_tc_params(8, 2048, 80, 128)) < 64 * 1024
    for p in (_tc_params(8, 2048, 80, 128), _tc_params(1, 16384, 32, 256, ngroups=8),
              _tc_params(1, 32768, 48, 128, num_seqs=16)):
        assert ssd.workspace_size(p) > 0
