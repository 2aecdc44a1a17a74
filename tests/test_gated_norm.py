"""The Mamba-2 block's output normalisation fused after the SSD forward
(ssd_fwd_gated_norm): out = GroupNorm(y * silu(z)) over each head's headdim
channels, times a per-channel weight, plus a bias ("Transformers are SSMs",
Sec. 7.1 and 8.1), against oracle.recurrence followed by
oracle.gated_group_norm (fp64), every element.

Tolerance: max|d| / max|oracle| <= 2e-2 for bf16 inputs (y * silu(z) is
staged as bf16 before the normalisation on the tensor-core path, and the
output is bf16), 1e-4 for float32."""
import numpy as np
import pytest

import oracle
from _helpers import BF16_TOL, F32_TOL, record_parity, small_inputs, to_device

pytestmark = pytest.mark.gpu


def run_gated(inp, z, w, b, eps, path="auto"):
    import torch
    import mamba_ssd_layer_fwd_b200 as ssd
    t = to_device(inp)
    zt = torch.from_numpy(np.ascontiguousarray(z)).to(device="cuda", dtype=t["x"].dtype)
    wt = torch.from_numpy(np.ascontiguousarray(w, dtype=np.float32)).cuda()
    bt = None if b is None else torch.from_numpy(np.ascontiguousarray(b, dtype=np.float32)).cuda()
    out, fin = ssd.ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], chunk_len=inp["chunk_len"],
                           initial_states=t["initial_states"], cu_seqlens=t["cu_seqlens"], return_final_states=True,
                           path=path, check_status=True, z=zt, norm_weight=wt, norm_bias=bt, norm_eps=eps)
    torch.cuda.synchronize()
    return out.double().cpu().numpy(), fin.double().cpu().numpy()


def check_gated(inp, label, path="auto", seed=0, bias=True, eps=1e-5):
    import ssd_inputs
    rng = np.random.default_rng(seed)
    H, P = inp["x"].shape[2], inp["x"].shape[3]
    z = rng.standard_normal(inp["x"].shape).astype(np.float32) * 2.0
    if inp["io_dtype"] == "bf16":
        z = ssd_inputs.round_to_bf16(z)
    w = (1.0 + 0.5 * rng.standard_normal(H * P)).astype(np.float32)
    b = (0.1 * rng.standard_normal(H * P)).astype(np.float32) if bias else None
    out, fin = run_gated(inp, z, w, b, eps, path)
    y_ref, fin_ref = oracle.recurrence(inp)
    want = oracle.gated_group_norm(y_ref, z, w, b, eps)
    tol = F32_TOL if inp["io_dtype"] == "f32" else BF16_TOL
    e = float(np.max(np.abs(out - want)) / np.max(np.abs(want)))
    ef = float(np.max(np.abs(fin - fin_ref)) / np.max(np.abs(fin_ref)))
    record_parity(f"gated norm {label}", e, ef, tol)
    assert np.all(np.isfinite(out))
    assert e <= tol and ef <= tol, (e, ef)


@pytest.mark.parametrize("N,G,H", [(64, 1, 4), (128, 2, 4), (256, 2, 4)])
def test_gated_norm_tensor_path_ragged(N, G, H):
    inp = small_inputs(batch=2, seqlen=700, H=H, P=64, N=N, G=G, Q=256, init=True, seed=60 + N)
    check_gated(inp, f"tensor ragged N={N}", path="tensor", seed=1)


@pytest.mark.parametrize("N", [128, 256])
def test_gated_norm_single_launch_segmented(N):
    """Equal-length rows cut into segments: the gated norm in the epilogue of the
    segmented walk's second (full) walk."""
    import mamba_ssd_layer_fwd_b200 as ssd
    inp = small_inputs(batch=1, seqlen=3000, H=2, P=64, N=N, G=1, Q=256, init=True, seed=65 + N)
    t = to_device(inp)
    assert ssd.launch_count(ssd.params_for(t["x"], t["B"], 256, None, True, "tensor")) == 1
    check_gated(inp, f"tensor single-launch segmented N={N}", path="tensor", seed=3)


def test_gated_norm_one_head_items_and_tail():
    """Odd heads per group (one-head items), and 160 two-head items on 148 SMs
    (whole waves of two-head items, the rest as one-head items in a second,
    overlapping launch), each with the gated norm in the epilogue."""
    inp = small_inputs(batch=2, seqlen=300, H=3, P=64, N=128, G=1, Q=256, init=True, seed=66)
    check_gated(inp, "tensor one-head items", path="tensor", seed=4)
    inp = small_inputs(batch=2, seqlen=300, H=160, P=64, N=64, G=1, Q=256, init=True, seed=67)
    check_gated(inp, "tensor two-head waves + one-head tail", path="tensor", seed=5)


def test_gated_norm_tensor_path_segmented_varlen():
    inp = small_inputs(H=2, P=64, N=128, G=1, Q=256, varlen=[6000, 0, 129, 3000], init=True, seed=61)
    check_gated(inp, "tensor packed, segmented", path="tensor", seed=2, bias=False)


def test_gated_norm_simt_path():
    inp = small_inputs(batch=2, seqlen=333, H=3, P=16, N=24, G=1, Q=64, io="f32", init=True, seed=62,
                       xbc_std=1.0, dt_shift=2.0, a_log_hi=1.5)
    check_gated(inp, "simt f32", path="simt", seed=3, eps=1e-3)


def test_gated_norm_simt_bf16_headdim_128():
    inp = small_inputs(batch=1, seqlen=300, H=2, P=128, N=32, G=1, Q=64, init=True, seed=63)
    check_gated(inp, "simt bf16 headdim 128", path="simt", seed=4)


def test_gated_norm_closed_gate_gives_bias():
    """z == 0 closes the gate: every channel of the output is its bias."""
    import torch
    inp = small_inputs(batch=1, seqlen=256, H=2, P=64, N=64, G=1, Q=256, init=False, seed=64)
    H, P = 2, 64
    b = np.linspace(-1, 1, H * P).astype(np.float32)
    out, _ = run_gated(inp, np.zeros(inp["x"].shape, np.float32), np.ones(H * P, np.float32), b, 1e-5,
                       path="tensor")
    bb = np.asarray(torch.tensor(b).to(torch.bfloat16).float())
    assert np.max(np.abs(out - bb.reshape(1, 1, H, P))) == 0.0
