"""GPU parity of the decoding step (recurrent mode, one token per call)
against the fp64 oracle's recurrence over the same tokens: T calls of
ssd_decode_step from the initial state must give the oracle's y at every step
and its final state.  Same tolerances as the forward: max|dy| / max|y_oracle|
<= 2e-2 for bf16 inputs, <= 1e-4 for float32."""
import numpy as np
import pytest

import oracle
import ssd_inputs
from _helpers import BF16_TOL, F32_TOL, rel_max_err, small_inputs

pytestmark = pytest.mark.gpu


def _steps(inp, state0=None):
    """Run every token of `inp` (batch rows of equal length) through the decode
    step; returns y (b, T, H, P) and the final state, float64."""
    import torch
    import mamba_ssd_layer_fwd_b200 as ssd
    io = torch.bfloat16 if inp["io_dtype"] == "bf16" else torch.float32
    dev = "cuda"
    x = torch.from_numpy(inp["x"]).to(dev, io)
    dt = torch.from_numpy(inp["dt"]).to(dev, io)
    Bm = torch.from_numpy(inp["B"]).to(dev, io)
    Cm = torch.from_numpy(inp["C"]).to(dev, io)
    A_log = torch.from_numpy(inp["A_log"]).to(dev)
    D = None if inp.get("D") is None else torch.from_numpy(inp["D"]).to(dev)
    b, T, H, P = x.shape
    N = Bm.shape[3]
    if state0 is not None:
        state = state0.clone()
    elif inp.get("initial_states") is not None:
        state = torch.from_numpy(inp["initial_states"]).to(dev).contiguous()
    else:
        state = torch.zeros((b, H, P, N), dtype=torch.float32, device=dev)
    ys = []
    for t in range(T):
        y = ssd.ssd_decode_step(x[:, t].contiguous(), dt[:, t].contiguous(), A_log, Bm[:, t].contiguous(),
                                Cm[:, t].contiguous(), D, state, dt_softplus=inp.get("dt_softplus", True))
        ys.append(y)
    torch.cuda.synchronize()
    y = torch.stack(ys, dim=1) if ys else torch.empty((b, 0, H, P), dtype=io, device=dev)
    return y.double().cpu().numpy(), state.double().cpu().numpy()


def _check(inp, tol):
    y, fin = _steps(inp)
    y_ref, fin_ref = oracle.recurrence(inp)
    assert rel_max_err(y, y_ref) <= tol, rel_max_err(y, y_ref)
    assert rel_max_err(fin, fin_ref) <= tol, rel_max_err(fin, fin_ref)


def test_decode_f32_odd_shapes():
    inp = small_inputs(batch=3, seqlen=6, H=4, P=16, N=24, G=2, Q=64, io="f32", init=True, seed=41,
                       xbc_std=1.0, dt_shift=1.0, a_log_hi=1.5)
    _check(inp, F32_TOL)


@pytest.mark.parametrize("P,N,G,H", [(64, 128, 1, 8), (64, 256, 2, 8), (128, 64, 1, 4), (64, 16, 1, 2),
                                     (32, 252, 3, 6)])
def test_decode_bf16_shapes(P, N, G, H):
    inp = small_inputs(batch=5, seqlen=5, H=H, P=P, N=N, G=G, Q=64, init=True, seed=P + N + G)
    _check(inp, BF16_TOL)


def test_decode_without_softplus_and_without_D():
    inp = small_inputs(batch=2, seqlen=4, H=4, P=64, N=64, G=1, Q=64, io="f32", init=True, seed=43)
    raw = inp["dt"].astype(np.float64)
    inp["dt"] = (np.maximum(raw, 0) + np.log1p(np.exp(-np.abs(raw)))).astype(np.float32)
    inp["dt_softplus"] = False
    inp["D"] = None
    _check(inp, F32_TOL)


def test_decode_zero_rows_is_a_no_op():
    import torch
    import mamba_ssd_layer_fwd_b200 as ssd
    x = torch.empty((0, 2, 64), dtype=torch.bfloat16, device="cuda")
    dt = torch.empty((0, 2), dtype=torch.bfloat16, device="cuda")
    Bm = torch.empty((0, 1, 64), dtype=torch.bfloat16, device="cuda")
    st = torch.empty((0, 2, 64, 64), dtype=torch.float32, device="cuda")
    A = torch.zeros(2, dtype=torch.float32, device="cuda")
    y = ssd.ssd_decode_step(x, dt, A, Bm, Bm, None, st)
    assert y.shape == x.shape


def test_prefill_then_decode_equals_one_forward():
    """ssd_fwd over the first tokens (final states out), then decode steps
    from that state, reproduce the oracle over all tokens."""
    import torch
    import mamba_ssd_layer_fwd_b200 as ssd
    from _helpers import to_device
    T0, K = 300, 6
    full = small_inputs(batch=2, seqlen=T0 + K, H=4, P=64, N=128, G=1, Q=256, init=True, seed=44)
    y_ref, fin_ref = oracle.recurrence(full)
    pre = dict(full)
    tail = dict(full)
    for k in ("x", "dt", "B", "C"):
        pre[k] = np.ascontiguousarray(full[k][:, :T0])
        tail[k] = np.ascontiguousarray(full[k][:, T0:])
    t = to_device(pre)
    y0, state = ssd.ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"], chunk_len=256,
                            initial_states=t["initial_states"], return_final_states=True, check_status=True)
    y1, fin = _steps(tail, state0=state)
    torch.cuda.synchronize()
    y = np.concatenate([y0.double().cpu().numpy(), y1], axis=1)
    assert rel_max_err(y, y_ref) <= BF16_TOL
    assert rel_max_err(fin, fin_ref) <= BF16_TOL


def test_decode_benchmark_shape_sampled():
    """The decode benchmark's shape (64 rows of the 2.7B layer), one step,
    against the oracle on every row."""
    w = ssd_inputs.workload("decode_2p7b")
    inp = ssd_inputs.make_inputs(w)
    _check(inp, BF16_TOL)
