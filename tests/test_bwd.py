"""GPU backward pass (ssd_bwd, through the C ABI) against the fp64 gradient
oracle, every element of every gradient: dx, ddt, dA_log, dB, dC, dD and the
initial-state gradient, for L = <dy, y> + <dfinal, final_states>.

The pass computes in fp32 from the exact input values (bf16 inputs are read
as they are), so the bound is an fp32 one: max|d| / max|oracle| <= 1e-3 per
gradient (accumulation over up to a few thousand terms and exponentials of
cumulative sums, each with fp32 rounding ~6e-8)."""
import numpy as np
import pytest

import oracle
import ssd_inputs
from _helpers import record_parity, rel_max_err, small_inputs, to_device

pytestmark = pytest.mark.gpu

BWD_TOL = 1e-3
KEYS = ("dx", "ddt", "dA_log", "dB", "dC", "dD", "dinit")


def run_bwd(inp, dy, dfin, want_dinit=True):
    import torch
    import mamba_ssd_layer_fwd_b200 as ssd
    t = to_device(inp)
    io = t["x"].dtype
    dy_t = torch.from_numpy(np.ascontiguousarray(dy)).to(device="cuda", dtype=io)
    df_t = None if dfin is None else torch.from_numpy(np.ascontiguousarray(dfin, dtype=np.float32)).cuda()
    g = ssd.ssd_bwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], dy_t,
                    initial_states=t["initial_states"], cu_seqlens=t["cu_seqlens"], dfinal_states=df_t,
                    dt_softplus=inp.get("dt_softplus", True), want_dinitial=want_dinit, check_status=True)
    torch.cuda.synchronize()
    out = {k: (None if v is None else v.double().cpu().numpy()) for k, v in g.items()}
    out["dinit"] = out.pop("dinitial_states")
    return out


def check_bwd(inp, label, seed=0, with_dfinal=True, tol=BWD_TOL):
    rng = np.random.default_rng(seed)
    dy = rng.standard_normal(inp["x"].shape).astype(np.float32)
    if inp["io_dtype"] == "bf16":
        dy = ssd_inputs.round_to_bf16(dy)
    nseq = len(ssd_inputs.seq_bounds(inp))
    H, P, N = inp["x"].shape[2], inp["x"].shape[3], inp["B"].shape[3]
    dfin = rng.standard_normal((nseq, H, P, N)).astype(np.float32) if with_dfinal else None
    got = run_bwd(inp, dy, dfin)
    want = oracle.recurrence_grad(inp, dy, dfin)
    bad = {k: int(np.sum(~np.isfinite(got[k]))) for k in KEYS if not np.all(np.isfinite(got[k]))}
    assert not bad, f"{label}: non-finite gradients (count per output): {bad}"
    errs = {}
    for k in KEYS:
        errs[k] = rel_max_err(got[k].reshape(want[k].shape), want[k])
    worst = max(errs.values())
    record_parity(f"bwd {label} (worst of {', '.join(KEYS)})", worst, None, tol)
    for k, e in errs.items():
        assert e <= tol, f"{label}: {k} rel err {e:.3e} > {tol} (all: {errs})"
    return errs


def test_bwd_f32_tiny_workload():
    inp = ssd_inputs.make_inputs(ssd_inputs.workload("tiny_f32", with_initial_states=True, with_final_states=True))
    check_bwd(inp, "tiny_f32")


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("N,G,H,P", [(24, 1, 3, 16), (64, 2, 4, 64), (128, 1, 2, 64), (256, 2, 4, 64),
                                     (32, 1, 2, 128)])
def test_bwd_shapes_ragged(io, N, G, H, P):
    inp = small_inputs(batch=2, seqlen=333, H=H, P=P, N=N, G=G, Q=64, io=io, init=True, seed=N + G + P,
                       **({"xbc_std": 1.0, "dt_shift": 2.0, "a_log_hi": 1.5} if io == "f32" else {}))
    check_bwd(inp, f"ragged {io} N={N} G={G} H={H} P={P}", seed=1)


def test_bwd_varlen_with_empty_and_single_token_sequences():
    inp = small_inputs(H=4, P=64, N=128, G=2, Q=64, varlen=[1, 255, 0, 97, 33, 3], init=True, seed=41)
    check_bwd(inp, "varlen bf16", seed=2)


def test_bwd_without_softplus_without_D_and_states():
    inp = small_inputs(batch=1, seqlen=200, H=2, P=32, N=64, G=1, Q=64, io="f32", init=False, seed=42,
                       xbc_std=1.0)
    inp["dt_softplus"] = False
    inp["dt"] = np.abs(inp["dt"]).astype(np.float32) * np.float32(0.2)
    inp["D"] = None
    check_bwd(inp, "no softplus, no D, no initial state", seed=3, with_dfinal=False)


def test_bwd_decay_one_and_zero():
    inp = small_inputs(batch=1, seqlen=150, H=2, P=64, N=64, G=1, Q=64, init=True, seed=43)
    inp["A_log"] = np.array([-np.inf, 30.0], dtype=np.float32)   # head 0: a == 1, head 1: a == 0
    check_bwd(inp, "decay one and zero", seed=4)


def test_bwd_longer_sequence():
    """Two rows of 1500 tokens, 8 heads in 2 groups, the 2.7B layer's value distributions."""
    inp = small_inputs(batch=2, seqlen=1500, H=8, P=64, N=128, G=2, Q=256, init=True, seed=44)
    check_bwd(inp, "2 x 1500 tokens", seed=5)


def test_bwd_zero_length():
    inp = small_inputs(batch=2, seqlen=0, H=2, P=64, N=64, G=1, Q=64, init=True, seed=45)
    rng = np.random.default_rng(6)
    dfin = rng.standard_normal((2, 2, 64, 64)).astype(np.float32)
    got = run_bwd(inp, np.zeros(inp["x"].shape, np.float32), dfin)
    np.testing.assert_array_equal(got["dinit"], dfin.astype(np.float64))
    assert np.all(got["dA_log"] == 0.0) and np.all(got["dD"] == 0.0)
