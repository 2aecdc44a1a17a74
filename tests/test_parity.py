"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle,
element by element, on seeded inputs. Tolerance: max|dy| / max|y_oracle| <=
2e-2 for bf16 inputs, <= 1e-4 for float32; final states to the same bound."""
import numpy as np
import pytest

import oracle
import ssd_inputs
from _helpers import BF16_TOL, F32_TOL, record_parity, rel_max_err, run_gpu, small_inputs

pytestmark = pytest.mark.gpu

PATHS = ["simt", "tensor"]


def _maybe_skip_path(inp, path):
    import mamba_ssd_layer_fwd_b200 as ssd
    x, B = inp["x"], inp["B"]
    nseq = 0 if inp.get("cu_seqlens") is None else len(inp["cu_seqlens"]) - 1
    p = ssd.make_params(batch=x.shape[0], seqlen=x.shape[1], nheads=x.shape[2], headdim=x.shape[3],
                        dstate=B.shape[3], ngroups=B.shape[2], chunk_len=inp["chunk_len"],
                        num_seqs=nseq, io_dtype=inp["io_dtype"], path=path)
    if ssd.resolved_path(p) != path:
        pytest.skip(f"{path} path does not take this shape")


def _test_name():
    import os
    return os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0].split("::")[-1]


def check_full(inp, path="auto", chunk_len=None, tol=None, label=None):
    tol = tol or (F32_TOL if inp["io_dtype"] == "f32" else BF16_TOL)
    y, fin = run_gpu(inp, path=path, chunk_len=chunk_len)
    y_ref, fin_ref = oracle.recurrence(inp)
    ey, ef = rel_max_err(y, y_ref), rel_max_err(fin, fin_ref)
    record_parity(label or _test_name(), ey, ef, tol)
    assert ey <= tol, f"y rel err {ey:.3e} > {tol}"
    assert ef <= tol, f"final-state rel err {ef:.3e} > {tol}"
    return y, fin, ey, ef


# ------------------------------------------------------------- tiny float32

def test_tiny_f32_workload():
    """The tiny float32 workload (T=256, H=2, P=N=16, chunk 64) to 1e-4."""
    inp = ssd_inputs.make_inputs(ssd_inputs.workload("tiny_f32", with_final_states=True))
    check_full(inp)


@pytest.mark.parametrize("Q", [64, 128, 256])
def test_f32_ragged_with_initial_state(Q):
    inp = small_inputs(batch=2, seqlen=333, H=3, P=16, N=24, G=1, Q=Q, io="f32", init=True,
                       xbc_std=1.0, dt_shift=2.0, a_log_hi=1.5)
    check_full(inp)


# ----------------------------------------------------------------- bf16

@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("N,G,H", [(64, 1, 4), (128, 1, 6), (256, 2, 4), (128, 4, 8)])
def test_bf16_shapes_ragged(path, N, G, H):
    inp = small_inputs(batch=2, seqlen=700, H=H, P=64, N=N, G=G, Q=256, init=True, seed=N + G)
    _maybe_skip_path(inp, path)
    check_full(inp, path=path)


@pytest.mark.parametrize("path", PATHS)
def test_bf16_dstate256_long_segments(path):
    """dstate 256 with several 128-token blocks per segment (one B/C stage)."""
    inp = small_inputs(batch=1, seqlen=3000, H=2, P=64, N=256, G=1, Q=256, init=True, seed=31)
    _maybe_skip_path(inp, path)
    check_full(inp, path=path)


@pytest.mark.parametrize("path", PATHS)
def test_bf16_varlen_with_states(path):
    lens = [1, 255, 256, 257, 0, 700, 64, 3]
    inp = small_inputs(H=4, P=64, N=128, G=1, Q=256, varlen=lens, init=True, seed=3)
    _maybe_skip_path(inp, path)
    check_full(inp, path=path)


def test_chunk_length_invariance_simt():
    """Sec. 6: the block decomposition is exact for any chunk length; the SIMT
    path evaluates chunks of Q = 64, 128 and 256 tokens."""
    inp = small_inputs(batch=1, seqlen=1024, H=4, P=64, N=64, G=1, Q=256, init=True, seed=5)
    outs = []
    for Q in (64, 128, 256):
        inp["chunk_len"] = Q
        y, fin, _, _ = check_full(inp, path="simt", chunk_len=Q, label=f"chunk_length_invariance simt Q={Q}")
        outs.append((y, fin))
    for y, fin in outs[1:]:
        assert rel_max_err(y, outs[0][0]) <= BF16_TOL
        assert rel_max_err(fin, outs[0][1]) <= BF16_TOL


def test_tensor_path_agrees_with_simt_chunk_lengths():
    """The tensor-core path (128-token diagonal blocks whatever chunk_len is)
    against the SIMT path's chunk decompositions at Q = 64, 128 and 256 on the
    same inputs: two independent implementations and four block lengths."""
    inp = small_inputs(batch=1, seqlen=1000, H=4, P=64, N=128, G=2, Q=256, init=True, seed=25)
    simt = {}
    for Q in (64, 128, 256):
        inp["chunk_len"] = Q
        simt[Q] = run_gpu(inp, path="simt", chunk_len=Q)
    for Q in (128, 256):
        inp["chunk_len"] = Q
        y, fin = run_gpu(inp, path="tensor", chunk_len=Q)
        for Qs, (ys, fs) in simt.items():
            ey, ef = rel_max_err(y, ys), rel_max_err(fin, fs)
            record_parity(f"tensor Q={Q} vs simt Q={Qs}", ey, ef, BF16_TOL)
            assert ey <= BF16_TOL and ef <= BF16_TOL


@pytest.mark.parametrize("path", PATHS)
def test_decay_one_and_zero(path):
    inp = small_inputs(batch=1, seqlen=520, H=2, P=64, N=64, G=1, Q=256, init=True, seed=6)
    _maybe_skip_path(inp, path)
    inp["A_log"] = np.array([-np.inf, 30.0], dtype=np.float32)   # head 0: a == 1, head 1: a == 0
    check_full(inp, path=path)


@pytest.mark.parametrize("path", PATHS)
def test_single_token_and_empty(path):
    inp = small_inputs(batch=3, seqlen=1, H=2, P=64, N=64, G=1, Q=256, init=True, seed=7)
    _maybe_skip_path(inp, path)
    check_full(inp, path=path)


def test_tail_items_split_into_single_heads():
    """160 two-head work items on 148 SMs: the first 148 run as two-head items,
    the 12 left over as 24 one-head items in a second launch."""
    inp = small_inputs(batch=2, seqlen=300, H=160, P=64, N=64, G=1, Q=256, init=True, seed=15)
    check_full(inp, path="tensor")


def _plan(inp):
    """(launches, workspace bytes) of the tensor path for these inputs."""
    import mamba_ssd_layer_fwd_b200 as ssd
    from _helpers import to_device
    t = to_device(inp)
    p = ssd.params_for(t["x"], t["B"], 256, None, True, "tensor")
    return ssd.launch_count(p), ssd.workspace_size(p)


@pytest.mark.parametrize("N,G,H,seqlen", [(128, 2, 4, 1000), (256, 1, 2, 1300), (64, 1, 6, 1500), (128, 1, 3, 1400)])
def test_segmented_single_launch(N, G, H, seqlen):
    """Equal-length rows with fewer (row, head block) pairs than SMs: every pair is
    cut into segments (the last one ragged) and one launch runs the state-only
    walks, the exchange of segment states and the full walks (Sec. 8.2); with
    initial and final states, two-head and one-head items (H = 3)."""
    inp = small_inputs(batch=2, seqlen=seqlen, H=H, P=64, N=N, G=G, Q=256, init=True, seed=N + H + seqlen)
    launches, ws = _plan(inp)
    assert launches == 1 and ws >= 2 * 64 * N * 4     # one launch, with segment states in the workspace
    check_full(inp, path="tensor")


def test_segmented_tail_after_whole_waves():
    """152 two-head items of 32 blocks on 148 SMs: 148 walk whole rows, the 4
    pairs left over are cut into segments and run by the single-launch segmented
    walk, started as SMs free up behind the first launch."""
    inp = small_inputs(batch=4, seqlen=4096, H=76, P=64, N=64, G=1, Q=256, init=True, seed=16)
    launches, ws = _plan(inp)
    assert launches == 2 and ws >= 2 * 64 * 64 * 4
    check_full(inp, path="tensor")


def test_zero_length_batch_passes_initial_state():
    inp = small_inputs(batch=2, seqlen=0, H=2, P=64, N=64, G=1, Q=256, init=True, seed=8)
    y, fin = run_gpu(inp)
    assert y.size == 0
    np.testing.assert_array_equal(fin, inp["initial_states"].astype(np.float64))


def test_deterministic():
    inp = small_inputs(batch=1, seqlen=900, H=4, P=64, N=128, G=1, Q=256, init=True, seed=9)
    a, fa = run_gpu(inp)
    b, fb = run_gpu(inp)
    assert np.array_equal(a, b) and np.array_equal(fa, fb)


def test_bad_cu_seqlens_reported_in_status():
    import torch
    import mamba_ssd_layer_fwd_b200 as ssd
    from _helpers import to_device
    inp = small_inputs(H=2, P=64, N=64, G=1, Q=256, varlen=[100, 100], init=False, seed=10)
    t = to_device(inp)
    t["cu_seqlens"] = torch.tensor([0, 150, 120], dtype=torch.int32, device="cuda")
    with pytest.raises(ssd.SsdError) as e:
        ssd.ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], chunk_len=256,
                    cu_seqlens=t["cu_seqlens"], check_status=True)
    assert e.value.code == -5


def test_bad_cu_seqlens_on_segmented_path_with_reused_workspace():
    """Two long packed sequences are cut into segments (planner, state-only
    pass, segment scan, walk).  A malformed cu_seqlens on the workspace the
    previous good call left behind is reported, and the next good call on the
    same workspace is still correct."""
    import torch
    import mamba_ssd_layer_fwd_b200 as ssd
    from _helpers import to_device
    inp = small_inputs(H=2, P=64, N=64, G=1, Q=256, varlen=[6000, 6000], init=True, seed=13)
    t = to_device(inp)
    p = ssd.params_for(t["x"], t["B"], 256, t["cu_seqlens"], True, "tensor")
    assert ssd.launch_count(p) == 4          # segmented
    ws = torch.empty(ssd.workspace_size(p), dtype=torch.uint8, device="cuda")
    kw = dict(chunk_len=256, initial_states=t["initial_states"], workspace=ws, return_final_states=True)
    ssd.ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], cu_seqlens=t["cu_seqlens"],
                check_status=True, **kw)
    bad = torch.tensor([0, 13000, 12000], dtype=torch.int32, device="cuda")
    with pytest.raises(ssd.SsdError) as e:
        ssd.ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], cu_seqlens=bad, check_status=True, **kw)
    assert e.value.code == -5
    y, fin = ssd.ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], cu_seqlens=t["cu_seqlens"],
                         check_status=True, **kw)
    torch.cuda.synchronize()
    y_ref, fin_ref = oracle.recurrence(inp)
    ey = rel_max_err(y.double().cpu().numpy(), y_ref)
    ef = rel_max_err(fin.double().cpu().numpy(), fin_ref)
    record_parity("segmented varlen after a rejected plan", ey, ef, BF16_TOL)
    assert ey <= BF16_TOL and ef <= BF16_TOL


def test_device_wait_timeout_reported():
    """Failure detection without a fault: work item 0 withholds a tile, its
    bounded waits run out (about 2 s), the CTA drains, frees TMEM and exits,
    and the host reads SSD_ERR_TIMEOUT; the context stays usable."""
    import ctypes
    import torch
    import mamba_ssd_layer_fwd_b200 as ssd
    from _helpers import to_device
    inp = small_inputs(batch=1, seqlen=512, H=2, P=64, N=64, G=1, Q=256, init=False, seed=12)
    t = to_device(inp)
    p = ssd.params_for(t["x"], t["B"], 256, None, True, "tensor")
    ins = ssd.make_instrumentation(withhold_first_tile=True)
    lib = ssd.library()
    ws = torch.empty(ssd.workspace_size(p), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(t["x"])
    st = torch.cuda.current_stream().cuda_stream or None
    rc = lib.ssd_fwd_instrumented(ctypes.byref(p), t["x"].data_ptr(), t["dt"].data_ptr(), t["A_log"].data_ptr(),
                                  t["B"].data_ptr(), t["C"].data_ptr(), t["D"].data_ptr(), None, None, y.data_ptr(),
                                  None, ws.data_ptr(), ws.numel(), st, ctypes.byref(ins))
    assert rc == 0
    assert lib.ssd_get_status(ws.data_ptr(), st) == -4      # SSD_ERR_TIMEOUT
    # the same context keeps working
    check_full(inp, path="tensor")


def test_segment_exchange_timeout_reported():
    """The waits between CTAs of the single-launch segmented walk are bounded too:
    work item 0 withholds a tile, so segment 0 never publishes its state; the
    other segments' exchange waits run out (about 2 s), every CTA frees TMEM and
    exits, and the host reads SSD_ERR_TIMEOUT; the context stays usable."""
    import ctypes
    import torch
    import mamba_ssd_layer_fwd_b200 as ssd
    from _helpers import to_device
    inp = small_inputs(batch=1, seqlen=3000, H=2, P=64, N=256, G=1, Q=256, init=True, seed=13)
    assert _plan(inp)[0] == 1
    t = to_device(inp)
    p = ssd.params_for(t["x"], t["B"], 256, None, True, "tensor")
    ins = ssd.make_instrumentation(withhold_first_tile=True)
    lib = ssd.library()
    ws = torch.empty(ssd.workspace_size(p), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(t["x"])
    st = torch.cuda.current_stream().cuda_stream or None
    rc = lib.ssd_fwd_instrumented(ctypes.byref(p), t["x"].data_ptr(), t["dt"].data_ptr(), t["A_log"].data_ptr(),
                                  t["B"].data_ptr(), t["C"].data_ptr(), t["D"].data_ptr(),
                                  t["initial_states"].data_ptr(), None, y.data_ptr(), None, ws.data_ptr(),
                                  ws.numel(), st, ctypes.byref(ins))
    assert rc == 0
    assert lib.ssd_get_status(ws.data_ptr(), st) == -4      # SSD_ERR_TIMEOUT
    check_full(inp, path="tensor")


# ------------------------------------------ benchmark shapes, element-wise

BENCH_WORKLOADS = ["small_bf16", "mamba2_2p7b", "long16k_gva", "varlen32k"]


@pytest.mark.parametrize("name", BENCH_WORKLOADS)
def test_benchmark_workload_full(name):
    """Full-size benchmark shapes in the bench's launch configuration, every
    output element and every final state against the oracle's whole-workload
    recurrence (fp64 on the host cores)."""
    w = ssd_inputs.workload(name, with_final_states=True)
    inp = ssd_inputs.make_inputs(w)
    y, fin = run_gpu(inp)
    y_ref, fin_ref = oracle.recurrence(inp)
    ey, ef = rel_max_err(y, y_ref), rel_max_err(fin, fin_ref)
    record_parity(f"benchmark workload {name} (every element)", ey, ef, BF16_TOL)
    assert ey <= BF16_TOL, f"{name}: y rel err {ey:.3e}"
    assert ef <= BF16_TOL, f"{name}: final rel err {ef:.3e}"
