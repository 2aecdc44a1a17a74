"""Property tests of the CPU oracle over random shapes (no GPU).

The fixed-shape pins in test_oracle.py fix the values; these vary the shapes
(head and group counts, head and state sizes, packed batches with empty and
one-token sequences, with and without D, initial state and softplus) so that
an indexing slip that only shows at some shape fails too.  Two independent
facts are checked ("Transformers are SSMs", Sec. 3.4 and 5.1):

- the recurrence (C, fp64) equals multiplication by the explicit
  semiseparable matrix (numpy quadratic form);
- the reverse mode is the adjoint of the forward map: y and the final states
  are linear in x, B, C, D and the initial state, so for each of those
  L(v) - L(0) = <dL/dinput, v> holds up to fp64 rounding, with
  L = <dy, y> + <dfinal, final_states>; dt and A_log enter nonlinearly and
  are checked by central differences.
"""
import numpy as np
import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings, HealthCheck, strategies as st  # noqa: E402

import oracle  # noqa: E402

SETTINGS = dict(max_examples=30, deadline=None, derandomize=True,
                suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])


@st.composite
def problems(draw):
    G = draw(st.sampled_from([1, 2, 3]))
    H = G * draw(st.sampled_from([1, 2, 3]))
    P = draw(st.integers(1, 5))
    N = draw(st.integers(1, 6))
    packed = draw(st.booleans())
    if packed:
        lens = draw(st.lists(st.sampled_from([0, 1, 2, 5, 17, 30]), min_size=1, max_size=5))
        b, T = 1, int(sum(lens))
    else:
        lens = None
        b, T = draw(st.integers(1, 3)), draw(st.sampled_from([0, 1, 3, 24, 41]))
    softplus = draw(st.booleans())
    seed = draw(st.integers(0, 2 ** 16))
    rng = np.random.default_rng(seed)
    f = np.float32
    dt = rng.standard_normal((b, T, H)) - 1.0
    if not softplus:
        dt = np.abs(dt)             # delta given directly must be >= 0
    inp = {
        "x": rng.standard_normal((b, T, H, P)).astype(f),
        "dt": dt.astype(f),
        "A_log": rng.uniform(-1.5, 1.0, H).astype(f),
        "B": rng.standard_normal((b, T, G, N)).astype(f),
        "C": rng.standard_normal((b, T, G, N)).astype(f),
        "D": rng.standard_normal(H).astype(f) if draw(st.booleans()) else None,
        "initial_states": None,
        "cu_seqlens": None,
        "dt_softplus": softplus,
    }
    nseq = b
    if packed:
        inp["cu_seqlens"] = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        nseq = len(lens)
    if draw(st.booleans()):
        inp["initial_states"] = rng.standard_normal((nseq, H, P, N)).astype(f)
    return inp


def _loss(inp, dy, dfin):
    y, fin = oracle.recurrence(inp)
    return float(np.sum(y * dy) + np.sum(fin * dfin))


def _scale(*arrays):
    return max([1.0] + [float(np.max(np.abs(a))) for a in arrays if a is not None and a.size])


@settings(**SETTINGS)
@given(problems())
def test_recurrence_equals_quadratic_form_any_shape(inp):
    y_rec, _ = oracle.recurrence(inp)
    y_quad = oracle.quadratic_form(inp)
    assert y_rec.shape == inp["x"].shape
    assert np.max(np.abs(y_rec - y_quad), initial=0.0) <= 1e-11 * _scale(y_quad)


@settings(**SETTINGS)
@given(problems())
def test_reverse_mode_is_the_adjoint_of_the_linear_inputs(inp):
    rng = np.random.default_rng(int(inp["x"].size) + 7)
    H, P = inp["x"].shape[2], inp["x"].shape[3]
    N = inp["B"].shape[3]
    nseq = len(oracle.seq_bounds(inp))
    dy = rng.standard_normal(inp["x"].shape).astype(np.float32)
    dfin = rng.standard_normal((nseq, H, P, N)).astype(np.float32)
    g = oracle.recurrence_grad(inp, dy, dfin)
    grad_of = {"x": "dx", "B": "dB", "C": "dC", "D": "dD", "initial_states": "dinit"}
    for k, gk in grad_of.items():
        if inp[k] is None:
            continue
        zero = dict(inp, **{k: np.zeros_like(inp[k])})
        # D and the initial state may be absent (= 0), which is the same map at 0
        lin = _loss(inp, dy, dfin) - _loss(zero, dy, dfin)
        proj = float(np.sum(g[gk] * inp[k].astype(np.float64)))
        assert abs(lin - proj) <= 1e-9 * max(abs(proj), _scale(dy, dfin)), (k, lin, proj)


@settings(**dict(SETTINGS, max_examples=15))
@given(problems())
def test_reverse_mode_of_dt_and_A_log_matches_central_differences(inp):
    rng = np.random.default_rng(int(inp["x"].size) + 11)
    H, P = inp["x"].shape[2], inp["x"].shape[3]
    N = inp["B"].shape[3]
    nseq = len(oracle.seq_bounds(inp))
    dy = rng.standard_normal(inp["x"].shape).astype(np.float32)
    dfin = rng.standard_normal((nseq, H, P, N)).astype(np.float32)
    g = oracle.recurrence_grad(inp, dy, dfin)
    for k, gk in (("dt", "ddt"), ("A_log", "dA_log")):
        v = rng.standard_normal(inp[k].shape)
        eps = 1e-3
        plus = (inp[k] + eps * v).astype(np.float32)
        minus = (inp[k] - eps * v).astype(np.float32)
        if k == "dt" and not inp["dt_softplus"]:
            if np.any(minus < 0):
                continue               # delta must stay >= 0 without the softplus
        fd = (_loss(dict(inp, **{k: plus}), dy, dfin) - _loss(dict(inp, **{k: minus}), dy, dfin)) / 2.0
        # the perturbation actually applied after float32 rounding, halved
        proj = float(np.sum(g[gk] * (plus.astype(np.float64) - minus.astype(np.float64)) / 2.0))
        assert abs(fd - proj) <= 2e-5 * max(abs(proj), 1.0), (k, fd, proj)
