"""Pins of the CPU oracle against facts fixed by the pages and by mathematics
(no GPU). Source: "Transformers are SSMs: Generalized Models and Efficient
Algorithms Through Structured State Space Duality"."""
import json
import math
import os

import numpy as np
import pytest
import scipy.signal

import oracle
import ssd_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny(T=48, H=4, P=3, N=5, G=2, b=2, seed=0, init=False, D=True, varlen=None, **kw):
    """Small random problem (float32 values, not bf16-rounded)."""
    rng = np.random.default_rng(seed)
    tot = T * b
    if varlen is not None:
        b, tot = 1, int(sum(varlen))
    f = np.float32
    inp = {
        "x": rng.standard_normal((b, tot // b, H, P)).astype(f),
        "dt": (rng.standard_normal((b, tot // b, H)) - 1.0).astype(f),
        "A_log": rng.uniform(-1.0, 1.0, H).astype(f),
        "B": rng.standard_normal((b, tot // b, G, N)).astype(f),
        "C": rng.standard_normal((b, tot // b, G, N)).astype(f),
        "D": rng.standard_normal(H).astype(f) if D else None,
        "initial_states": None,
        "cu_seqlens": None,
        "dt_softplus": True,
    }
    nseq = b
    if varlen is not None:
        inp["cu_seqlens"] = np.concatenate([[0], np.cumsum(varlen)]).astype(np.int32)
        nseq = len(varlen)
    if init:
        inp["initial_states"] = rng.standard_normal((nseq, H, P, N)).astype(f)
    inp.update(kw)
    return inp


def rel_err(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# ---------------------------------------------------------------- golden values

_EXPR = {"log(ln(2)/2)": math.log(math.log(2) / 2), "0": 0.0, "30": 30.0,
         "log(ln(2))": math.log(math.log(2)), "ln(3)": math.log(3.0), "-ln(3)": -math.log(3.0)}


def _golden_inp(case):
    dt = [_EXPR[e] for e in case["dt_expr"]] if "dt_expr" in case else case["dt"]
    T = len(dt)
    P, N = case["P"], case["N"]
    A_log = _EXPR[case["A_log_expr"]]
    inp = {
        "x": np.array(case["x"], dtype=np.float32).reshape(1, T, 1, P),
        "dt": np.array(dt, dtype=np.float32).reshape(1, T, 1),
        "A_log": np.array([A_log], dtype=np.float32),
        "B": np.array(case["B"], dtype=np.float32).reshape(1, T, 1, N),
        "C": np.array(case["C"], dtype=np.float32).reshape(1, T, 1, N),
        "D": np.array([case["D"]], dtype=np.float32),
        "initial_states": None if case["h0"] is None else np.full((1, 1, P, N), case["h0"], np.float32),
        "cu_seqlens": None,
        "dt_softplus": case["dt_softplus"],
    }
    return inp


@pytest.mark.parametrize("idx", [0, 1, 2, 3, 4])
def test_golden_hand_worked(idx):
    """Hand-worked values of the recurrence (tests/golden/scalar_recurrence.json).
    Cases 3 and 4 pin the discretisation delta = softplus(dt) = log(1 + e^dt)
    away from dt = 0 (both signs, and |dt| up to 1000 where the naive form
    overflows): a sign flip or a dropped max(dt, 0) term fails them."""
    case = json.load(open(os.path.join(GOLDEN, "scalar_recurrence.json")))["cases"][idx]
    inp = _golden_inp(case)
    y, fin = oracle.recurrence(inp)
    ln2, ln3 = math.log(2.0), math.log(3.0)
    if "y_ln2" in case:
        want_y = np.array([c0 + c1 * ln2 for c0, c1 in case["y_ln2"]])
        want_f = case["final_ln2"][0] + case["final_ln2"][1] * ln2
    elif "y_ln23" in case:
        want_y = np.array([c0 + c1 * ln2 + c2 * ln3 for c0, c1, c2 in case["y_ln23"]])
        want_f = case["final_ln23"][0] + case["final_ln23"][1] * ln2 + case["final_ln23"][2] * ln3
    else:
        want_y = np.array(case["y"], dtype=np.float64)
        want_f = np.array(case["final"], dtype=np.float64)
    # A_log and dt are stored in float32, so a = 1/2 (or ln 3) holds to ~1e-7 relative
    rtol = case.get("rtol", 2e-6)
    np.testing.assert_allclose(y.reshape(want_y.shape), want_y, rtol=rtol, atol=1e-6)
    np.testing.assert_allclose(fin.reshape(np.shape(want_f)), want_f, rtol=rtol, atol=1e-6)


def test_discretize_softplus_matches_logaddexp():
    """delta = softplus(r) = log(e^0 + e^r): numpy's logaddexp is an independent
    evaluation of the same definition (Sec. 2.1 discretisation step size)."""
    r = np.array([-1000.0, -30.0, -5.0, -math.log(3.0), -1e-3, 0.0, 1e-3, math.log(3.0), 2.0, 30.0, 1000.0])
    inp = {"x": np.zeros((1, r.size, 1, 1)), "dt": r.reshape(1, -1, 1), "A_log": np.array([0.0]),
           "dt_softplus": True}
    delta, a = oracle.discretize(inp)
    want = np.logaddexp(0.0, r)
    np.testing.assert_allclose(delta[:, 0], want, rtol=1e-15, atol=0.0)
    np.testing.assert_allclose(a[:, 0], np.exp(-want), rtol=1e-15, atol=0.0)


# ---------------------------------------------------- brute-force quadratic form

@pytest.mark.parametrize("init,D", [(False, True), (True, True), (True, False)])
def test_recurrence_equals_quadratic_form(init, D):
    """Sec. 3.4.2 / 5.1: the SSM equals multiplication by the explicit semiseparable M."""
    inp = tiny(T=40, H=4, P=3, N=5, G=2, b=2, init=init, D=D, seed=1)
    y_rec, _ = oracle.recurrence(inp)
    y_quad = oracle.quadratic_form(inp)
    assert rel_err(y_rec, y_quad) < 1e-12


def test_recurrence_equals_quadratic_form_varlen():
    inp = tiny(H=2, P=2, N=3, G=1, varlen=[7, 1, 20, 12], init=True, seed=2)
    y_rec, _ = oracle.recurrence(inp)
    assert rel_err(y_rec, oracle.quadratic_form(inp)) < 1e-12


def test_impulse_columns_match_semiseparable_matrix():
    """Column j of M is the response to a unit input at time j (one channel)."""
    T, N = 24, 4
    inp = tiny(T=T, H=1, P=1, N=N, G=1, b=1, D=False, seed=3)
    M = oracle.semiseparable_matrix(inp, 0, 0)
    cols = []
    for j in range(T):
        e = np.zeros_like(inp["x"])
        e[0, j, 0, 0] = 1.0
        y, _ = oracle.recurrence(dict(inp, x=e))
        cols.append(y[0, :, 0, 0])
    M_imp = np.stack(cols, axis=1)
    assert rel_err(M_imp, M) < 1e-12
    # Def. 3.1: every block on or below the diagonal has rank <= N
    for i0 in (8, 12, 17):
        blk = M_imp[i0:, :i0]
        s = np.linalg.svd(blk, compute_uv=False)
        assert np.sum(s > 1e-9 * s[0]) <= N


# ------------------------------------------------------------------ closed forms

def test_decay_one_is_causal_linear_attention():
    """a == 1 (A_log = -inf, so A = -0): masked attention with the all-ones causal
    mask, i.e. a cumulative sum over time (Sec. 4.2 / 5.2)."""
    inp = tiny(T=33, H=2, P=3, N=4, G=1, b=1, init=True, seed=4)
    inp["A_log"] = np.full(2, -np.inf, dtype=np.float32)
    y, fin = oracle.recurrence(inp)
    delta, a = oracle.discretize(inp)
    assert np.all(a == 1.0)
    x = inp["x"][0].astype(np.float64)
    Bm = inp["B"][0, :, 0].astype(np.float64)
    Cm = inp["C"][0, :, 0].astype(np.float64)
    for h in range(2):
        kv = np.einsum("tp,tn->tpn", delta[:, h, None] * x[:, h], Bm)
        S = np.cumsum(kv, axis=0) + inp["initial_states"][0, h][None].astype(np.float64)
        want = np.einsum("tpn,tn->tp", S, Cm) + float(inp["D"][h]) * x[:, h]
        assert rel_err(y[0, :, h], want) < 1e-12
        assert rel_err(fin[0, h], S[-1]) < 1e-12


def test_decay_zero_keeps_only_the_diagonal():
    """a == 0 (A_log = +30 underflows exp(delta * A) to 0): y_t = (C_t . B_t) delta_t x_t + D x_t."""
    inp = tiny(T=20, H=2, P=3, N=4, G=2, b=1, init=True, seed=5)
    inp["A_log"] = np.full(2, 30.0, dtype=np.float32)
    y, _ = oracle.recurrence(inp)
    delta, a = oracle.discretize(inp)
    assert np.all(a == 0.0)
    x = inp["x"][0].astype(np.float64)
    for h in range(2):
        g = h // 1
        cb = np.sum(inp["C"][0, :, g].astype(np.float64) * inp["B"][0, :, g], axis=1)
        want = (cb * delta[:, h])[:, None] * x[:, h] + float(inp["D"][h]) * x[:, h]
        assert rel_err(y[0, :, h], want) < 1e-12


def test_scalar_lti_is_first_order_filter():
    """N = P = 1, B = C = 1, constant delta: y_t = a y_{t-1} + delta x_t, the textbook
    first-order IIR filter (scipy.signal.lfilter)."""
    T = 64
    inp = tiny(T=T, H=1, P=1, N=1, G=1, b=1, D=False, seed=6)
    inp["B"][:] = 1.0
    inp["C"][:] = 1.0
    inp["dt"][:] = 0.3
    y, _ = oracle.recurrence(inp)
    delta, a = oracle.discretize(inp)
    want = scipy.signal.lfilter([delta[0, 0]], [1.0, -a[0, 0]], inp["x"][0, :, 0, 0].astype(np.float64))
    assert rel_err(y[0, :, 0, 0], want) < 1e-12


def test_lti_is_causal_convolution():
    """Constant a, B, C (Sec. 2.1 LTI case): y = K * x with K_k = (C . B) a^k delta."""
    T, N = 50, 3
    inp = tiny(T=T, H=1, P=2, N=N, G=1, b=1, D=False, seed=7)
    inp["dt"][:] = -0.5
    inp["B"][:] = inp["B"][0, 0]
    inp["C"][:] = inp["C"][0, 0]
    y, _ = oracle.recurrence(inp)
    delta, a = oracle.discretize(inp)
    cb = float(inp["C"][0, 0, 0].astype(np.float64) @ inp["B"][0, 0, 0].astype(np.float64))
    K = cb * delta[0, 0] * a[0, 0] ** np.arange(T)
    for p in range(2):
        want = np.convolve(K, inp["x"][0, :, 0, p].astype(np.float64))[:T]
        assert rel_err(y[0, :, 0, p], want) < 1e-12


# ------------------------------------------------------------------- invariants

def test_split_sequence_state_passing():
    """Sec. 8.2 (context parallelism): running [0, T/2) then [T/2, T) from the
    first half's final state equals the whole run."""
    inp = tiny(T=60, H=2, P=3, N=4, G=1, b=1, init=True, seed=8)
    y, fin = oracle.recurrence(inp)
    half = lambda a, s: None if a is None else a[:, s]
    first = dict(inp, x=inp["x"][:, :30], dt=inp["dt"][:, :30], B=inp["B"][:, :30], C=inp["C"][:, :30])
    y1, f1 = oracle.recurrence(first)
    second = dict(inp, x=inp["x"][:, 30:], dt=inp["dt"][:, 30:], B=inp["B"][:, 30:], C=inp["C"][:, 30:],
                  initial_states=f1.astype(np.float32))
    y2, f2 = oracle.recurrence(second)
    # f1 is rounded to float32 when passed back in: compare at float32 resolution
    assert rel_err(np.concatenate([y1, y2], axis=1), y) < 1e-6
    assert rel_err(f2, fin) < 1e-6


def test_linearity_in_input_and_initial_state():
    inp1 = tiny(T=30, H=2, P=2, N=3, G=1, b=1, init=True, D=True, seed=9)
    inp2 = tiny(T=30, H=2, P=2, N=3, G=1, b=1, init=True, D=True, seed=10)
    inp2.update({k: inp1[k] for k in ("dt", "A_log", "B", "C", "D")})
    al, be = 0.75, -1.25
    mix = dict(inp1, x=(al * inp1["x"].astype(np.float64) + be * inp2["x"]),
               initial_states=(al * inp1["initial_states"].astype(np.float64) + be * inp2["initial_states"]))
    # float32 inputs: keep the mixed values exactly representable by rounding first
    mix["x"] = mix["x"].astype(np.float32)
    mix["initial_states"] = mix["initial_states"].astype(np.float32)
    y1, f1 = oracle.recurrence(inp1)
    y2, f2 = oracle.recurrence(inp2)
    ym, fm = oracle.recurrence(mix)
    assert rel_err(ym, al * y1 + be * y2) < 1e-6
    assert rel_err(fm, al * f1 + be * f2) < 1e-6


def test_varlen_equals_separate_runs():
    """Sec. 8.3: packed sequences exchange no state."""
    lens = [5, 17, 1, 30]
    inp = tiny(H=3, P=2, N=3, G=1, varlen=lens, init=True, seed=11)
    y, fin = oracle.recurrence(inp)
    cu = inp["cu_seqlens"]
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        one = dict(inp, x=inp["x"][:, a:b], dt=inp["dt"][:, a:b], B=inp["B"][:, a:b], C=inp["C"][:, a:b],
                   initial_states=inp["initial_states"][s:s + 1], cu_seqlens=None)
        ys, fs = oracle.recurrence(one)
        assert rel_err(y[:, a:b], ys) < 1e-14
        assert rel_err(fin[s], fs[0]) < 1e-14


def test_empty_sequence_passes_initial_state_through():
    inp = tiny(H=2, P=2, N=2, G=1, varlen=[4, 0, 3], init=True, seed=12)
    _, fin = oracle.recurrence(inp)
    np.testing.assert_array_equal(fin[1], inp["initial_states"][1].astype(np.float64))


def test_group_mapping_is_contiguous():
    """GVA (Sec. 7.2): head h reads B/C group h // (H / G)."""
    inp = tiny(T=16, H=4, P=2, N=3, G=2, b=1, seed=13)
    y, _ = oracle.recurrence(inp)
    for h in range(4):
        g = h // 2
        one = dict(inp, x=inp["x"][:, :, h:h + 1], dt=inp["dt"][:, :, h:h + 1], A_log=inp["A_log"][h:h + 1],
                   D=inp["D"][h:h + 1], B=inp["B"][:, :, g:g + 1], C=inp["C"][:, :, g:g + 1])
        yh, _ = oracle.recurrence(one)
        assert rel_err(y[:, :, h:h + 1], yh) < 1e-14


def test_pairs_subset_matches_full_run():
    inp = tiny(T=20, H=3, P=2, N=3, G=1, b=2, init=True, seed=14)
    y, fin = oracle.recurrence(inp)
    ys, fs = oracle.recurrence_pairs(inp, [(1, 2), (0, 1)])
    assert np.array_equal(ys[0], y[1, :, 2])
    assert np.array_equal(fs[1], fin[0, 1])


# ------------------------------------------------------------------- generator

def test_generator_shapes_and_bf16_rounding():
    w = ssd_inputs.workload("varlen32k", seqlen=4096, num_seqs=5)
    inp = ssd_inputs.make_inputs(w)
    assert inp["x"].shape == (1, 4096, 48, 64)
    cu = inp["cu_seqlens"]
    assert cu[0] == 0 and cu[-1] == 4096 and np.all(np.diff(cu) >= 64) and len(cu) == 6
    for k in ("x", "dt", "B", "C"):
        bits = inp[k].view(np.uint32)
        assert np.all(bits & 0xFFFF == 0)
    assert inp["initial_states"].shape == (5, 48, 64, 128)
    # reproducible
    again = ssd_inputs.make_inputs(w)
    assert np.array_equal(again["x"], inp["x"]) and np.array_equal(again["cu_seqlens"], cu)


def test_round_to_bf16_ties_to_even():
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: rounds to the even mantissa (1.0)
    v = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5], dtype=np.float32)
    r = ssd_inputs.round_to_bf16(v)
    assert r[0] == 1.0 and r[1] == 1.0 + 2.0 ** -6 and r[2] == -2.5


# ------------------------------------------------------- gradients (reverse mode)

def _loss(inp, dy, dfin):
    """L = <dy, y> + <dfinal, final_states> through the (pinned) forward oracle."""
    y, fin = oracle.recurrence(inp)
    L = float(np.sum(y * dy.astype(np.float64)))
    if dfin is not None:
        L += float(np.sum(fin * dfin.astype(np.float64)))
    return L


GRAD_OF = {"x": "dx", "dt": "ddt", "A_log": "dA_log", "B": "dB", "C": "dC", "D": "dD", "initial_states": "dinit"}


def _fd_check(inp, dy, dfin, eps=1e-3, rtol=2e-4):
    """Central differences of the forward oracle, element by element. Inputs
    are float32, so the perturbation actually applied is taken from the rounded
    values (exact in float64)."""
    g = oracle.recurrence_grad(inp, dy, dfin)
    worst = 0.0
    for k, gk in GRAD_OF.items():
        base = inp[k]
        if base is None:
            continue
        got = g[gk].reshape(-1)
        scale = max(np.max(np.abs(got)), 1e-12)
        for i in range(base.size):
            vp, vm = base.copy().reshape(-1), base.copy().reshape(-1)
            vp[i] = np.float32(vp[i] + eps)
            vm[i] = np.float32(vm[i] - eps)
            h = float(np.float64(vp[i]) - np.float64(vm[i]))
            Lp = _loss(dict(inp, **{k: vp.reshape(base.shape)}), dy, dfin)
            Lm = _loss(dict(inp, **{k: vm.reshape(base.shape)}), dy, dfin)
            fd = (Lp - Lm) / h
            err = abs(fd - got[i]) / scale
            worst = max(worst, err)
            assert err < rtol, f"d{k}[{i}]: finite difference {fd:.9g}, reverse mode {got[i]:.9g}"
    return worst


@pytest.mark.parametrize("softplus", [True, False])
def test_gradients_match_finite_differences(softplus):
    """Every input's gradient (x, dt, A_log, B, C, D, initial state) against
    central differences of the forward recurrence, with GVA groups, two rows
    and a loss on the final state too."""
    inp = tiny(T=10, H=4, P=3, N=2, G=2, b=2, init=True, seed=21)
    if not softplus:
        inp["dt_softplus"] = False
        inp["dt"] = np.abs(inp["dt"]) + np.float32(0.1)      # delta itself, kept positive
    rng = np.random.default_rng(5)
    dy = rng.standard_normal(inp["x"].shape).astype(np.float32)
    dfin = rng.standard_normal(inp["initial_states"].shape).astype(np.float32)
    _fd_check(inp, dy, dfin)


def test_gradients_match_finite_differences_varlen():
    """Packed sequences (one empty, one of length 1): per-sequence initial
    states, no gradient crossing a boundary."""
    inp = tiny(H=2, P=2, N=3, G=1, varlen=[5, 0, 1, 7], init=True, seed=22)
    rng = np.random.default_rng(6)
    dy = rng.standard_normal(inp["x"].shape).astype(np.float32)
    dfin = rng.standard_normal(inp["initial_states"].shape).astype(np.float32)
    _fd_check(inp, dy, dfin)


def test_input_gradient_is_transposed_semiseparable_matrix():
    """y = (M + D I) x for fixed dt, A, B, C (Sec. 3.4.2 / 5.1), so dL/dx = (M + D I)^T dy,
    with M built explicitly by the quadratic form (independent of the reverse sweep)."""
    inp = tiny(T=30, H=3, P=2, N=4, G=1, b=2, init=True, seed=23)
    rng = np.random.default_rng(7)
    dy = rng.standard_normal(inp["x"].shape).astype(np.float32)
    g = oracle.recurrence_grad(inp, dy)
    for s in range(2):
        for h in range(3):
            M = oracle.semiseparable_matrix(inp, s, h)
            dyd = dy[s, :, h].astype(np.float64)
            want = M.T @ dyd + float(inp["D"][h]) * dyd
            assert rel_err(g["dx"][s, :, h], want) < 1e-12


def test_gradients_along_random_directions():
    """Adjoint identity <grad L, v> = dL/d(eps) along random directions v through
    every input at once, on a larger packed problem (central differences)."""
    inp = tiny(H=4, P=8, N=16, G=2, varlen=[90, 33, 120], init=True, seed=24)
    rng = np.random.default_rng(8)
    dy = rng.standard_normal(inp["x"].shape).astype(np.float32)
    dfin = rng.standard_normal(inp["initial_states"].shape).astype(np.float32)
    g = oracle.recurrence_grad(inp, dy, dfin)
    for trial in range(3):
        plus, minus, proj = dict(inp), dict(inp), 0.0
        for k, gk in GRAD_OF.items():
            v = rng.standard_normal(inp[k].shape)
            vp = (inp[k] + 1e-3 * v).astype(np.float32)
            vm = (inp[k] - 1e-3 * v).astype(np.float32)
            plus[k], minus[k] = vp, vm
            # half the perturbation actually applied (after float32 rounding), exactly
            proj += float(np.sum(g[gk] * (vp.astype(np.float64) - vm.astype(np.float64)) / 2.0))
        fd = (_loss(plus, dy, dfin) - _loss(minus, dy, dfin)) / 2.0
        assert abs(fd - proj) <= 1e-5 * max(abs(proj), 1.0), (trial, fd, proj)


def test_gradients_decay_zero_closed_form():
    """a == 0 (A_log = +30): every token is independent, G_t = dy_t C_t^T, so
    dx_t = D dy_t + delta_t (C_t . B_t) dy_t, dB_t = delta_t (dy_t . x_t) C_t,
    dC_t = delta_t (dy_t . x_t) B_t, and nothing reaches the initial state."""
    inp = tiny(T=15, H=2, P=3, N=4, G=1, b=1, init=True, seed=25)
    inp["A_log"] = np.full(2, 30.0, dtype=np.float32)
    rng = np.random.default_rng(9)
    dy = rng.standard_normal(inp["x"].shape).astype(np.float32)
    g = oracle.recurrence_grad(inp, dy)
    delta, a = oracle.discretize(inp)
    assert np.all(a == 0.0)
    x, dyd = inp["x"][0].astype(np.float64), dy[0].astype(np.float64)
    Bm, Cm = inp["B"][0, :, 0].astype(np.float64), inp["C"][0, :, 0].astype(np.float64)
    cb = np.sum(Cm * Bm, axis=1)
    dB = np.zeros_like(Bm)
    dC = np.zeros_like(Cm)
    for h in range(2):
        d = delta[:, h]
        dyx = np.sum(dyd[:, h] * x[:, h], axis=1)
        want_dx = float(inp["D"][h]) * dyd[:, h] + (d * cb)[:, None] * dyd[:, h]
        assert rel_err(g["dx"][0, :, h], want_dx) < 1e-12
        dB += (d * dyx)[:, None] * Cm
        dC += (d * dyx)[:, None] * Bm
    assert rel_err(g["dB"][0, :, 0], dB) < 1e-12
    assert rel_err(g["dC"][0, :, 0], dC) < 1e-12
    assert np.all(g["dinit"] == 0.0)


def test_gradient_of_empty_sequence_passes_dfinal_through():
    inp = tiny(H=2, P=2, N=2, G=1, varlen=[4, 0, 3], init=True, seed=26)
    rng = np.random.default_rng(10)
    dy = rng.standard_normal(inp["x"].shape).astype(np.float32)
    dfin = rng.standard_normal(inp["initial_states"].shape).astype(np.float32)
    g = oracle.recurrence_grad(inp, dy, dfin)
    np.testing.assert_array_equal(g["dinit"][1], dfin[1].astype(np.float64))


# ------------------------------------------------ gated norm of the Mamba-2 block

def test_gated_group_norm_matches_torch_group_norm():
    """Sec. 7.1 / 8.1: y * silu(z) followed by GroupNorm with one group per
    head, against torch's own silu and group_norm (library routines, float64)."""
    import torch
    rng = np.random.default_rng(30)
    T, H, P = 37, 6, 16
    y = rng.standard_normal((T, H, P))
    z = rng.standard_normal((T, H, P)) * 2.0
    w = rng.standard_normal(H * P)
    b = rng.standard_normal(H * P)
    got = oracle.gated_group_norm(y, z, w, b, eps=1e-5)
    g = torch.from_numpy(y) * torch.nn.functional.silu(torch.from_numpy(z))
    want = torch.nn.functional.group_norm(g.reshape(T, H * P), H, torch.from_numpy(w), torch.from_numpy(b), 1e-5)
    assert rel_err(got.reshape(T, H * P), want.numpy()) < 1e-12
    # groups of 8 channels (two per head)
    got8 = oracle.gated_group_norm(y, z, w, None, eps=1e-3, group_size=8)
    want8 = torch.nn.functional.group_norm(g.reshape(T, H * P), H * P // 8, torch.from_numpy(w), None, 1e-3)
    assert rel_err(got8.reshape(T, H * P), want8.numpy()) < 1e-12


def test_gated_group_norm_closed_forms():
    rng = np.random.default_rng(31)
    T, H, P = 5, 3, 8
    y = rng.standard_normal((T, H, P))
    b = rng.standard_normal(H * P)
    # z == 0 closes the gate: every group is constant 0, so the output is the bias
    out = oracle.gated_group_norm(y, np.zeros_like(y), np.ones(H * P), b)
    assert rel_err(out.reshape(T, H * P), np.broadcast_to(b, (T, H * P))) < 1e-15
    # unit weight, no bias: every group has mean 0 and variance var / (var + eps)
    z = rng.standard_normal((T, H, P))
    out = oracle.gated_group_norm(y, z, np.ones(H * P), None, eps=1e-2).reshape(T, H, P)
    g = y * z / (1 + np.exp(-z))
    var = g.var(axis=-1)
    assert np.max(np.abs(out.mean(axis=-1))) < 1e-14
    assert rel_err(out.var(axis=-1), var / (var + 1e-2)) < 1e-12
