"""Context-parallel SSD forward (Sec. 8.2 item 2): pieces of one sequence on
several workers, one exchange of state summaries.

CPU (gloo, world sizes 2 and 3): the orchestration and the exchange, with the
three local steps done by the oracle (end state from zero via the recurrence,
the fold in float64, the forward via the recurrence).  GPU: the library's
summary and combine kernels against the oracle, and four pieces emulated in
one process (no kernel waits on another) against the whole-sequence oracle."""
import os
import sys

import numpy as np
import pytest

import oracle
import ssd_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _piece(inp, t0, t1):
    return dict(inp, x=inp["x"][:, t0:t1], dt=inp["dt"][:, t0:t1], B=inp["B"][:, t0:t1], C=inp["C"][:, t0:t1])


class OracleOps:
    """The three local steps on the CPU, from the oracle (test only)."""

    def __init__(self, inp):
        self.inp = inp

    def _np(self, t):
        return None if t is None else t.detach().cpu().numpy()

    def summary(self, x, dt, A_log, B):
        import torch
        piece = dict(self.inp, x=self._np(x), dt=self._np(dt), B=self._np(B), C=np.zeros_like(self._np(B)),
                     initial_states=None, D=None)
        _, fin = oracle.recurrence(piece)
        delta, a = oracle.discretize(piece)
        A = -np.exp(self.inp["A_log"].astype(np.float64))
        b, T = piece["x"].shape[:2]
        L = (delta * A[None, :]).reshape(b, T, -1).sum(axis=1)
        return torch.from_numpy(fin.astype(np.float32)), torch.from_numpy(L.astype(np.float32))

    def combine(self, S_all, L_all, rank, initial_states):
        import torch
        S, L = S_all.double().numpy(), L_all.double().numpy()
        h = np.zeros(S.shape[1:]) if initial_states is None else initial_states.double().numpy()
        for r in range(rank):
            h = np.exp(L[r])[..., None, None] * h + S[r]
        return torch.from_numpy(h.astype(np.float32))

    def forward(self, x, dt, A_log, B, C, D, initial_states):
        import torch
        piece = dict(self.inp, x=self._np(x), dt=self._np(dt), B=self._np(B), C=self._np(C),
                     initial_states=self._np(initial_states))
        y, fin = oracle.recurrence(piece)
        return torch.from_numpy(y.astype(np.float32)), torch.from_numpy(fin.astype(np.float32))


def _problem():
    w = ssd_inputs.Workload("cp", 2, 300, 3, 4, 5, 1, 64, "f32", with_initial_states=True,
                            xbc_std=1.0, dt_shift=1.0, a_log_hi=1.0)
    return ssd_inputs.make_inputs(w)


def _worker(rank, world, cuts, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        import datetime
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        from mamba_ssd_layer_fwd_b200.context_parallel import ssd_fwd_context_parallel
        inp = _problem()
        p = _piece(inp, cuts[rank], cuts[rank + 1])
        t = {k: torch.from_numpy(np.ascontiguousarray(p[k])) for k in ("x", "dt", "B", "C")}
        y, fin = ssd_fwd_context_parallel(t["x"], t["dt"], torch.from_numpy(inp["A_log"]), t["B"], t["C"],
                                          torch.from_numpy(inp["D"]),
                                          initial_states=torch.from_numpy(inp["initial_states"]),
                                          ops=OracleOps(inp), return_final_states=True)
        q.put((rank, y.numpy(), fin.numpy()))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, repr(e), None))


@pytest.mark.parametrize("cuts", [[0, 170, 300], [0, 64, 65, 300]])
def test_context_parallel_gloo(cuts):
    import multiprocessing as mp
    world = len(cuts) - 1
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000) + world
    procs = [ctx.Process(target=_worker, args=(r, world, cuts, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, y, fin = q.get(timeout=120)
        res[r] = (y, fin)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert not isinstance(res[r][0], str), res[r][0]
    inp = _problem()
    y_ref, fin_ref = oracle.recurrence(inp)
    y = np.concatenate([res[r][0] for r in range(world)], axis=1)
    assert np.max(np.abs(y - y_ref)) / np.max(np.abs(y_ref)) < 1e-5
    for r in range(world):   # every worker holds the state after the whole sequence
        assert np.max(np.abs(res[r][1] - fin_ref)) / np.max(np.abs(fin_ref)) < 1e-5


# ------------------------------------------------------------------- GPU

def _dev(inp, t0=None, t1=None):
    import torch
    from _helpers import to_device
    p = inp if t0 is None else _piece(inp, t0, t1)
    return to_device(p)


@pytest.mark.gpu
@pytest.mark.parametrize("kind", ["tensor", "simt", "tensor_varlen", "simt_varlen", "tensor_short"])
def test_summary_matches_oracle(kind):
    """End state from a zero state and total log decay of every sequence (tensor_short:
    sequences of one and two 128-token blocks, where the end state is read right
    after the last state update)."""
    import torch
    import mamba_ssd_layer_fwd_b200 as ssd
    from _helpers import small_inputs, record_parity
    varlen = {"tensor_varlen": [300, 0, 129, 411], "simt_varlen": [300, 0, 129, 411],
              "tensor_short": [129, 1, 256, 129, 2]}.get(kind)
    inp = small_inputs(batch=2, seqlen=700, H=4, P=64, N=128, G=2, Q=256, init=False, varlen=varlen, seed=51)
    path = "tensor" if kind.startswith("tensor") else "simt"
    t = _dev(inp)
    S, L = ssd.ssd_fwd_summary(t["x"], t["dt"], t["A_log"], t["B"], chunk_len=256, cu_seqlens=t["cu_seqlens"],
                               path=path, check_status=True)
    torch.cuda.synchronize()
    _, fin = oracle.recurrence(dict(inp, initial_states=None))
    delta, _ = oracle.discretize(inp)
    A = -np.exp(inp["A_log"].astype(np.float64))
    L_ref = np.stack([(delta[t0:t0 + n] * A).sum(axis=0) for t0, n in ssd_inputs.seq_bounds(inp)])
    es = np.max(np.abs(S.double().cpu().numpy() - fin)) / max(np.max(np.abs(fin)), 1e-30)
    el = np.max(np.abs(L.double().cpu().numpy() - L_ref)) / np.max(np.abs(L_ref))
    record_parity(f"summary {kind} (end state, log decay)", es, el, 2e-2)
    assert es <= 2e-2 and el <= 1e-5


@pytest.mark.gpu
def test_state_combine_matches_fold():
    import torch
    import mamba_ssd_layer_fwd_b200 as ssd
    rng = np.random.default_rng(52)
    S = rng.standard_normal((4, 2, 3, 8, 16)).astype(np.float32)
    L = -rng.uniform(0, 3, (4, 2, 3)).astype(np.float32)
    h0 = rng.standard_normal((2, 3, 8, 16)).astype(np.float32)
    dev = lambda a: torch.from_numpy(a).cuda()
    for rank in range(5):
        got = ssd.ssd_state_combine(dev(S), dev(L), rank, initial_states=dev(h0)).cpu().numpy()
        want = h0.astype(np.float64)
        for r in range(rank):   # H <- exp(L_r) H + S_r
            want = np.exp(L[r].astype(np.float64))[..., None, None] * want + S[r]
        assert np.max(np.abs(got - want)) <= 1e-5 * np.max(np.abs(want))


@pytest.mark.gpu
@pytest.mark.parametrize("io,cuts", [("bf16", [0, 300, 557, 1069, 1197]), ("f32", [0, 100, 101, 333, 600])])
def test_context_parallel_pieces_on_one_gpu(io, cuts):
    """Four workers emulated in one process: every piece summarised by the
    library, the summaries stacked as the all-gather would, then every piece
    finished from the fold of the pieces before it; the concatenation matches
    the oracle over the whole sequence."""
    import torch
    from mamba_ssd_layer_fwd_b200.context_parallel import LibraryOps, finish_piece, summarize_piece
    from _helpers import small_inputs, record_parity, BF16_TOL, F32_TOL
    T = cuts[-1]
    kw = {} if io == "bf16" else {"xbc_std": 1.0, "dt_shift": 2.0, "a_log_hi": 1.5}
    inp = small_inputs(batch=2, seqlen=T, H=4, P=64 if io == "bf16" else 16, N=128 if io == "bf16" else 24,
                       G=2, Q=256 if io == "bf16" else 64, io=io, init=True, seed=53, **kw)
    ops = LibraryOps(chunk_len=inp["chunk_len"])
    pieces = [_dev(inp, cuts[r], cuts[r + 1]) for r in range(len(cuts) - 1)]
    init = pieces[0]["initial_states"]
    summ = [summarize_piece(p["x"], p["dt"], p["A_log"], p["B"], ops) for p in pieces]
    S_all = torch.stack([s for s, _ in summ]).contiguous()
    L_all = torch.stack([l for _, l in summ]).contiguous()
    ys, fins = [], []
    for r, p in enumerate(pieces):
        y, fin = finish_piece(p["x"], p["dt"], p["A_log"], p["B"], p["C"], p["D"], S_all, L_all, r, init, ops)
        ys.append(y)
        fins.append(fin)
    torch.cuda.synchronize()
    y = torch.cat(ys, dim=1).double().cpu().numpy()
    y_ref, fin_ref = oracle.recurrence(inp)
    tol = BF16_TOL if io == "bf16" else F32_TOL
    ey = np.max(np.abs(y - y_ref)) / np.max(np.abs(y_ref))
    ef = max(np.max(np.abs(f.double().cpu().numpy() - fin_ref)) for f in fins) / np.max(np.abs(fin_ref))
    record_parity(f"context parallel, 4 pieces, {io}", ey, ef, tol)
    assert ey <= tol and ef <= tol
