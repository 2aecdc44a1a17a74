"""CPU oracle of the Mamba-2 SSD forward layer (fp64).

TEST INFRASTRUCTURE. Only tests/, the smoke check and the bench's CPU
baseline may import this package. The library's product path never does, and
this package imports nothing from the CUDA path.

Two independent formulations of the same map, both written from
"Transformers are SSMs: Generalized Models and Efficient Algorithms Through
Structured State Space Duality":

* `recurrence` - the linear (recurrent) mode, Sec. 3.4.1 eq. (8): expand by B,
  scalar recurrence, contract by C. Plain C in `ssd_ref.c`, fp64, threads over
  (sequence, head) pairs. This is the oracle the CUDA path is compared with.
* `recurrence_grad` - reverse mode of the same recurrence (every input's
  gradient given dL/dy and dL/dfinal), plain C, fp64.
* `gated_group_norm` - the block's output normalisation after the layer
  (y * silu(z), then GroupNorm over each head's channels), numpy fp64.
* `quadratic_form` - the dual (attention-like) mode, Sec. 3.4.2 / Sec. 5.1: build
  the T x T semiseparable matrix M[i, j] = C_i . (a_{j+1} ... a_i) B_j delta_j
  (lower triangle) explicitly and multiply. numpy, tiny sizes only. It pins the
  recurrence.

Readings where the pages are silent (the CUDA path makes the same ones): the input is
discretised as delta * x; A = -exp(A_log); D multiplies raw x; the initial
state is decayed by the first token's a; packed sequences exchange no state.
Every function here is pinned by tests/test_oracle.py (brute force, closed
forms, invariants, hand-worked values), except for the input discretisation
itself: the pages omit it, so that one choice (delta * x) is parity unpinned,
a recorded reading that both formulations above share.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Iterable, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_ref.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libssd_ref.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile ssd_ref.c with gcc (plain -O2, no fast-math) into _build/."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64p = ctypes.POINTER(ctypes.c_int64)
            i32p = ctypes.POINTER(ctypes.c_int32)
            fp = ctypes.POINTER(ctypes.c_float)
            dp = ctypes.POINTER(ctypes.c_double)
            lib.ssd_ref_pairs.restype = ctypes.c_int
            lib.ssd_ref_pairs.argtypes = [ctypes.c_int, i64p, i64p, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          fp, fp, fp, fp, fp, fp, fp,
                                          ctypes.c_int, i32p, i32p, i64p, dp, dp, ctypes.c_int]
            lib.ssd_ref_max_threads.restype = ctypes.c_int
            lib.ssd_ref_bwd.restype = ctypes.c_int
            lib.ssd_ref_bwd.argtypes = [ctypes.c_int, i64p, i64p, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        fp, fp, fp, fp, fp, fp, fp, fp, fp, ctypes.c_int64,
                                        dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().ssd_ref_max_threads())


def _ptr(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct)) if a is not None else None


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def seq_bounds(inp: dict):
    x = inp["x"]
    b, T = x.shape[0], x.shape[1]
    cu = inp.get("cu_seqlens")
    if cu is None:
        return [(i * T, T) for i in range(b)]
    cu = np.asarray(cu, dtype=np.int64)
    return [(int(cu[i]), int(cu[i + 1] - cu[i])) for i in range(len(cu) - 1)]


def recurrence_pairs(inp: dict, pairs: Iterable[tuple[int, int]], nthreads: int = 0):
    """Run the recurrence for the given (sequence, head) pairs only.

    Returns (ys, finals): ys[i] is (len_i, P) float64, finals[i] is (P, N).
    """
    lib = _load()
    x, dt, Bm, Cm = (_f32(inp[k]) for k in ("x", "dt", "B", "C"))
    A_log, D, init = _f32(inp["A_log"]), _f32(inp.get("D")), _f32(inp.get("initial_states"))
    H, P = x.shape[2], x.shape[3]
    G, N = Bm.shape[2], Bm.shape[3]
    bounds = seq_bounds(inp)
    pairs = list(pairs)
    ps = np.array([p[0] for p in pairs], dtype=np.int32)
    ph = np.array([p[1] for p in pairs], dtype=np.int32)
    lens = np.array([bounds[s][1] for s, _ in pairs], dtype=np.int64)
    offs = np.zeros(len(pairs), dtype=np.int64)
    if len(pairs):
        offs[1:] = np.cumsum(lens * P)[:-1]
    y = np.zeros(int((lens * P).sum()), dtype=np.float64)
    fin = np.zeros(len(pairs) * P * N, dtype=np.float64)
    starts = np.array([b[0] for b in bounds], dtype=np.int64)
    slens = np.array([b[1] for b in bounds], dtype=np.int64)
    rc = lib.ssd_ref_pairs(len(bounds), _ptr(starts, ctypes.c_int64), _ptr(slens, ctypes.c_int64),
                           H, P, N, G, int(bool(inp.get("dt_softplus", True))),
                           _ptr(x, ctypes.c_float), _ptr(dt, ctypes.c_float),
                           _ptr(A_log, ctypes.c_float), _ptr(Bm, ctypes.c_float),
                           _ptr(Cm, ctypes.c_float), _ptr(D, ctypes.c_float),
                           _ptr(init, ctypes.c_float), len(pairs), _ptr(ps, ctypes.c_int32),
                           _ptr(ph, ctypes.c_int32), _ptr(offs, ctypes.c_int64),
                           _ptr(y, ctypes.c_double), _ptr(fin, ctypes.c_double), int(nthreads))
    if rc != 0:
        raise ValueError("ssd_ref_pairs rejected its arguments")
    ys = [y[o:o + n * P].reshape(n, P) for o, n in zip(offs, lens)]
    finals = [fin[i * P * N:(i + 1) * P * N].reshape(P, N) for i in range(len(pairs))]
    return ys, finals


def recurrence(inp: dict, nthreads: int = 0):
    """Full oracle output: y with x's shape (float64) and final states (nseq, H, P, N)."""
    x = inp["x"]
    H, P = x.shape[2], x.shape[3]
    N = inp["B"].shape[3]
    bounds = seq_bounds(inp)
    pairs = [(s, h) for s in range(len(bounds)) for h in range(H)]
    ys, finals = recurrence_pairs(inp, pairs, nthreads)
    y = np.zeros(x.shape, dtype=np.float64).reshape(-1, H, P)
    for (s, h), ysh in zip(pairs, ys):
        t0, n = bounds[s]
        y[t0:t0 + n, h, :] = ysh
    fin = np.stack(finals).reshape(len(bounds), H, P, N) if pairs else np.zeros((len(bounds), H, P, N))
    return y.reshape(x.shape), fin


def recurrence_grad(inp: dict, dy, dfinal=None, nthreads: int = 0) -> dict:
    """Reverse mode of the recurrence (fp64, plain C): the gradients of
    L = <dy, y> + <dfinal, final_states> with respect to x, dt (raw, before the
    softplus), A_log, B, C, D and the initial states. Written by differentiating
    the per-token update of Sec. 3.4.1 eq. (8) step by step (see ssd_ref.c).
    Returns float64 arrays shaped like the inputs: dx, ddt, dA_log, dB, dC, dD,
    dinit (dinit has the initial-state shape (nseq, H, P, N))."""
    lib = _load()
    x, dt, Bm, Cm = (_f32(inp[k]) for k in ("x", "dt", "B", "C"))
    A_log, D, init = _f32(inp["A_log"]), _f32(inp.get("D")), _f32(inp.get("initial_states"))
    dyf = _f32(dy)
    dfin = _f32(dfinal)
    H, P = x.shape[2], x.shape[3]
    G, N = Bm.shape[2], Bm.shape[3]
    bounds = seq_bounds(inp)
    nseq = len(bounds)
    tokens = x.shape[0] * x.shape[1]
    starts = np.array([b[0] for b in bounds], dtype=np.int64)
    slens = np.array([b[1] for b in bounds], dtype=np.int64)
    out = {"dx": np.zeros((tokens, H, P)), "ddt": np.zeros((tokens, H)), "dB": np.zeros((tokens, G, N)),
           "dC": np.zeros((tokens, G, N)), "dA_log": np.zeros(H), "dD": np.zeros(H),
           "dinit": np.zeros((nseq, H, P, N))}
    rc = lib.ssd_ref_bwd(nseq, _ptr(starts, ctypes.c_int64), _ptr(slens, ctypes.c_int64), H, P, N, G,
                         int(bool(inp.get("dt_softplus", True))), _ptr(x, ctypes.c_float),
                         _ptr(dt, ctypes.c_float), _ptr(A_log, ctypes.c_float), _ptr(Bm, ctypes.c_float),
                         _ptr(Cm, ctypes.c_float), _ptr(D, ctypes.c_float), _ptr(init, ctypes.c_float),
                         _ptr(dyf, ctypes.c_float), _ptr(dfin, ctypes.c_float), tokens,
                         *(_ptr(out[k], ctypes.c_double) for k in ("dx", "ddt", "dB", "dC", "dA_log", "dD", "dinit")),
                         int(nthreads))
    if rc != 0:
        raise ValueError("ssd_ref_bwd rejected its arguments")
    out["dx"] = out["dx"].reshape(x.shape)
    out["ddt"] = out["ddt"].reshape(dt.shape)
    out["dB"] = out["dB"].reshape(Bm.shape)
    out["dC"] = out["dC"].reshape(Cm.shape)
    return out


def silu(z):
    """z * sigmoid(z) in float64."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def gated_group_norm(y, z, weight, bias=None, eps: float = 1e-5, group_size=None):
    """The Mamba-2 block's output normalisation ("Transformers are SSMs",
    Sec. 7.1 extra normalisation before the output projection, Sec. 8.1
    GroupNorm): g = y * silu(z), then every group of `group_size` consecutive
    channels of a token (default: one head's headdim channels) is normalised
    by its mean and variance, out = (g - mean) / sqrt(var + eps) * weight + bias.
    y, z: (..., H, P); weight, bias: (H * P,). float64 result, y's shape."""
    y = np.asarray(y, dtype=np.float64)
    z = np.asarray(z, dtype=np.float64)
    H, P = y.shape[-2], y.shape[-1]
    gs = P if group_size is None else int(group_size)
    g = (y * silu(z)).reshape(-1, H * P // gs, gs)
    mean = g.mean(axis=-1, keepdims=True)
    var = ((g - mean) ** 2).mean(axis=-1, keepdims=True)
    out = ((g - mean) / np.sqrt(var + eps)).reshape(-1, H * P) * np.asarray(weight, dtype=np.float64)
    if bias is not None:
        out = out + np.asarray(bias, dtype=np.float64)
    return out.reshape(y.shape)


def _softplus(r):
    return np.maximum(r, 0.0) + np.log1p(np.exp(-np.abs(r)))


def discretize(inp: dict):
    """delta (tokens, H) and a = exp(delta * A) (tokens, H), float64."""
    x = inp["x"]
    H = x.shape[2]
    r = np.asarray(inp["dt"], dtype=np.float64).reshape(-1, H)
    delta = _softplus(r) if inp.get("dt_softplus", True) else r
    A = -np.exp(np.asarray(inp["A_log"], dtype=np.float64))
    return delta, np.exp(delta * A[None, :])


def semiseparable_matrix(inp: dict, seq: int, head: int) -> np.ndarray:
    """The T x T matrix M of one (sequence, head): M[i, j] = (C_i . B_j) *
    (a_{j+1} * ... * a_i) * delta_j for j <= i, else 0 ("Transformers are SSMs",
    Sec. 5.1, the SSS form M_ij = C_i^T A_{j+1:i} B_j with A_k = a_k I and the
    input scaled by delta). The products of a's are taken one by one (O(T^3));
    tiny T only."""
    x = inp["x"]
    H = x.shape[2]
    G = inp["B"].shape[2]
    g = head // (H // G)
    t0, T = seq_bounds(inp)[seq]
    delta, a = discretize(inp)
    Bm = np.asarray(inp["B"], dtype=np.float64).reshape(-1, G, inp["B"].shape[3])[t0:t0 + T, g]
    Cm = np.asarray(inp["C"], dtype=np.float64).reshape(-1, G, inp["C"].shape[3])[t0:t0 + T, g]
    ah = a[t0:t0 + T, head]
    dh = delta[t0:t0 + T, head]
    M = np.zeros((T, T))
    for i in range(T):
        for j in range(i + 1):
            decay = 1.0
            for k in range(j + 1, i + 1):
                decay *= ah[k]
            M[i, j] = float(Cm[i] @ Bm[j]) * decay * dh[j]
    return M


def quadratic_form(inp: dict):
    """y = M x + D x + (a_0 ... a_t) C_t . h0 for every (sequence, head), built from
    the explicit semiseparable matrix. Returns (y like x, float64)."""
    x = inp["x"]
    H, P = x.shape[2], x.shape[3]
    G, N = inp["B"].shape[2], inp["B"].shape[3]
    xf = np.asarray(x, dtype=np.float64).reshape(-1, H, P)
    Cf = np.asarray(inp["C"], dtype=np.float64).reshape(-1, G, N)
    D = inp.get("D")
    init = inp.get("initial_states")
    _, a = discretize(inp)
    y = np.zeros_like(xf)
    for s, (t0, T) in enumerate(seq_bounds(inp)):
        for h in range(H):
            g = h // (H // G)
            M = semiseparable_matrix(inp, s, h)
            yh = M @ xf[t0:t0 + T, h, :]
            if D is not None:
                yh = yh + float(D[h]) * xf[t0:t0 + T, h, :]
            if init is not None:
                h0 = np.asarray(init[s, h], dtype=np.float64)          # (P, N)
                cum = np.cumprod(a[t0:t0 + T, h])                     # a_0 ... a_t
                yh = yh + cum[:, None] * (Cf[t0:t0 + T, g, :] @ h0.T)
            y[t0:t0 + T, h, :] = yh
    return y.reshape(x.shape)
