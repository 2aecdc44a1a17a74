"""Seeded synthetic inputs for the Mamba-2 SSD forward layer.

This module only draws random numbers and shapes them. It holds none of the
layer's arithmetic, so both the CPU oracle (tests, bench baseline) and the
CUDA path (tests, bench) can take their inputs from here.

Workloads follow the shapes and value distributions of the SSD benchmark
configurations (tensor layouts follow the `ssd(X, A, B, C, block_len,
initial_states)` listing of "Transformers are SSMs", Section 6 / Listing 1):

    x, y            (batch, seqlen, nheads, headdim)      io dtype
    dt              (batch, seqlen, nheads)               io dtype (raw, pre-softplus)
    B, C            (batch, seqlen, ngroups, dstate)      io dtype
    A_log, D        (nheads,)                             fp32
    initial_states  (nseq, nheads, headdim, dstate)       fp32
    cu_seqlens      (nseq + 1,)                           int32 (packed varlen only; batch == 1)

Every tensor draws from its own stream, seeded by (seed, tensor id), so adding
a tensor never changes the others. Values of bf16 tensors are rounded to the
nearest bf16 (ties to even) here, once; the float32 arrays returned hold those
exact bf16 values, so the oracle and the GPU read identical numbers.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "workload",
    "make_inputs",
    "round_to_bf16",
    "varlen_lengths",
]

_TENSOR_IDS = {"x": 1, "dt": 2, "A_log": 3, "B": 4, "C": 5, "D": 6, "init": 7, "lengths": 8}


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and value recipe of one synthetic SSD forward workload."""

    name: str
    batch: int
    seqlen: int          # per-row length, or total packed tokens when varlen
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk_len: int
    io_dtype: str        # "f32" or "bf16"
    num_seqs: int = 0    # > 0: packed varlen (batch must be 1)
    with_initial_states: bool = False
    with_final_states: bool = False
    min_seqlen: int = 64
    # value distributions
    xbc_std: float = 1.0           # std of x, B, C
    dt_shift: float = 2.0          # raw dt ~ N(0,1) - dt_shift, delta = softplus(raw)
    a_log_hi: float = 1.5          # A_log ~ U(0, a_log_hi), A = -exp(A_log)
    init_std: float = 0.1
    seed: int = 0

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen

    @property
    def nseq(self) -> int:
        return self.num_seqs if self.num_seqs > 0 else self.batch

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _scaled(n: int) -> float:
    return 1.0 / math.sqrt(n)


# The five benchmark shapes of the SSD forward (tiny fp32 parity case, a small
# bf16 case, the Mamba-2 2.7B layer shape, a 16K-token GVA case, packed varlen).
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 256, 2, 16, 16, 1, 64, "f32",
                          xbc_std=1.0, dt_shift=2.0, a_log_hi=1.5),
    "small_bf16": Workload("small_bf16", 2, 2048, 24, 64, 64, 1, 256, "bf16",
                            xbc_std=_scaled(64), dt_shift=3.0, a_log_hi=2.7),
    "mamba2_2p7b": Workload("mamba2_2p7b", 8, 2048, 80, 64, 128, 1, 256, "bf16",
                             xbc_std=_scaled(128), dt_shift=3.0, a_log_hi=2.7),
    "long16k_gva": Workload("long16k_gva", 1, 16384, 32, 64, 256, 8, 256, "bf16",
                             with_final_states=True,
                             xbc_std=_scaled(256), dt_shift=3.0, a_log_hi=2.7),
    "varlen32k": Workload("varlen32k", 1, 32768, 48, 64, 128, 1, 256, "bf16",
                           num_seqs=16, with_initial_states=True, with_final_states=True,
                           xbc_std=_scaled(128), dt_shift=3.0, a_log_hi=2.7, init_std=0.1),
    # one decoding step (recurrent mode) of 64 rows of the 2.7B layer shape,
    # from a carried state; seqlen 1, chunk_len unused by the step
    "decode_2p7b": Workload("decode_2p7b", 64, 1, 80, 64, 128, 1, 256, "bf16",
                             with_initial_states=True, with_final_states=True,
                             xbc_std=_scaled(128), dt_shift=3.0, a_log_hi=2.7, init_std=0.1),
}


def workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return w.replace(**overrides) if overrides else w


def _rng(seed: int, name: str) -> np.random.Generator:
    return np.random.default_rng([int(seed), _TENSOR_IDS[name]])


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((u >> 16) & 1)
    r = ((u + bias) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).reshape(a.shape)


def varlen_lengths(total: int, nseq: int, min_len: int, seed: int) -> np.ndarray:
    """Seeded sequence lengths: min_len + the gaps between sorted uniform integer
    cut points of [0, total - nseq*min_len]. They sum to `total`."""
    slack = total - nseq * min_len
    if slack < 0:
        raise ValueError("total tokens too small for nseq * min_len")
    cuts = np.sort(_rng(seed, "lengths").integers(0, slack + 1, size=nseq - 1))
    edges = np.concatenate([[0], cuts, [slack]])
    return (np.diff(edges) + min_len).astype(np.int64)


def make_inputs(w: Workload, seed: Optional[int] = None) -> dict:
    """Draw the inputs of workload `w`. Returns numpy arrays (float32 holding
    io-dtype-exact values, int32 cu_seqlens) plus metadata."""
    seed = w.seed if seed is None else seed
    b, T, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    if w.num_seqs > 0 and b != 1:
        raise ValueError("packed varlen workloads have batch 1")
    f = np.float32

    def normal(name, shape, std=1.0, shift=0.0):
        v = _rng(seed, name).standard_normal(size=shape, dtype=np.float64) * std - shift
        return v.astype(f)

    x = normal("x", (b, T, H, P), w.xbc_std)
    dt = normal("dt", (b, T, H), 1.0, w.dt_shift)
    Bm = normal("B", (b, T, G, N), w.xbc_std)
    Cm = normal("C", (b, T, G, N), w.xbc_std)
    A_log = _rng(seed, "A_log").uniform(0.0, w.a_log_hi, size=(H,)).astype(f)
    D = normal("D", (H,), 1.0)
    if w.io_dtype == "bf16":
        x, dt, Bm, Cm = (round_to_bf16(t) for t in (x, dt, Bm, Cm))
    elif w.io_dtype != "f32":
        raise ValueError(w.io_dtype)

    cu = None
    if w.num_seqs > 0:
        lens = varlen_lengths(T, w.num_seqs, w.min_seqlen, seed)
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    nseq = w.nseq
    init = normal("init", (nseq, H, P, N), w.init_std) if w.with_initial_states else None
    return {
        "x": x, "dt": dt, "A_log": A_log, "B": Bm, "C": Cm, "D": D,
        "initial_states": init, "cu_seqlens": cu,
        "dt_softplus": True, "chunk_len": w.chunk_len, "io_dtype": w.io_dtype,
        "want_final_states": w.with_final_states, "workload": w,
    }


def seq_bounds(inputs: dict) -> list[tuple[int, int]]:
    """(start, length) of every sequence in the flattened (batch*seqlen) token axis."""
    x = inputs["x"]
    b, T = x.shape[0], x.shape[1]
    cu = inputs.get("cu_seqlens")
    if cu is None:
        return [(i * T, T) for i in range(b)]
    return [(int(cu[i]), int(cu[i + 1] - cu[i])) for i in range(len(cu) - 1)]
