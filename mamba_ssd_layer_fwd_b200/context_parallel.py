"""Context-parallel SSD forward: a long sequence split along its length over
the workers of a process group ("Transformers are SSMs", Sec. 8.2 item 2 and
Fig. 7 right: each worker receives an initial state, runs the SSM on its piece
and passes its final state on).

A piece maps the state entering it to exp(L) H + S (S: its end state from a
zero state, L: its total log decay), so every worker summarises its own piece
at the same time, the summaries are exchanged once (an all-gather of
nseq * H * (P * N + 1) floats per worker), and each worker folds the summaries
of the pieces before its own, in order, into the state entering its piece,
then runs the forward on its piece from that state.  All arithmetic runs in
the library's kernels (ssd_fwd_summary, ssd_state_combine, ssd_fwd); the
process group carries the exchange (NCCL between GPUs).

Worker `rank` holds tokens [t_rank, t_rank+1) of every row (rows of equal
length; pieces may differ in length).  `ops` replaces the three local steps
(for tests on machines without the library)."""
from __future__ import annotations

from typing import Optional


class LibraryOps:
    """The three local steps on the GPU, through the C ABI."""

    def __init__(self, chunk_len: int = 256, dt_softplus: bool = True, path: str = "auto"):
        self.chunk_len, self.dt_softplus, self.path = chunk_len, dt_softplus, path

    def summary(self, x, dt, A_log, B):
        from . import ssd_fwd_summary
        return ssd_fwd_summary(x, dt, A_log, B, chunk_len=self.chunk_len, dt_softplus=self.dt_softplus,
                               path=self.path)

    def combine(self, S_all, L_all, rank, initial_states):
        from . import ssd_state_combine
        return ssd_state_combine(S_all, L_all, rank, initial_states=initial_states)

    def forward(self, x, dt, A_log, B, C, D, initial_states):
        from . import ssd_fwd
        return ssd_fwd(x, dt, A_log, B, C, D, chunk_len=self.chunk_len, initial_states=initial_states,
                       dt_softplus=self.dt_softplus, return_final_states=True, path=self.path)


def summarize_piece(x, dt, A_log, B, ops=None):
    """Step 1 on one worker: (S, L) of its piece."""
    ops = ops or LibraryOps()
    return ops.summary(x, dt, A_log, B)


def finish_piece(x, dt, A_log, B, C, D, S_all, L_all, rank: int, initial_states=None, ops=None):
    """Steps 3-4 on worker `rank`, given every worker's summary: the piece's y,
    and the state after the whole sequence (the fold of all the summaries)."""
    ops = ops or LibraryOps()
    world = S_all.shape[0]
    h_in = ops.combine(S_all, L_all, rank, initial_states)
    y, _ = ops.forward(x, dt, A_log, B, C, D, h_in)
    final = ops.combine(S_all, L_all, world, initial_states)
    return y, final


def ssd_fwd_context_parallel(x, dt, A_log, B, C, D=None, *, initial_states=None, group=None,
                             ops=None, return_final_states: bool = False):
    """Forward of this worker's piece of every row, exchanging one summary per
    worker over `group` (torch.distributed; every worker calls this together).
    Returns y of the piece, and (if asked) the state after the whole sequence
    (identical on every worker)."""
    import torch
    import torch.distributed as dist
    ops = ops or LibraryOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    S, L = summarize_piece(x, dt, A_log, B, ops)
    # one exchange: every worker's (S, L), packed into one buffer per worker
    flat = torch.cat([S.reshape(-1), L.reshape(-1)]).contiguous()
    parts = [torch.empty_like(flat) for _ in range(world)]
    dist.all_gather(parts, flat, group=group)
    nS = S.numel()
    S_all = torch.stack([q[:nS].view(S.shape) for q in parts]).contiguous()
    L_all = torch.stack([q[nS:].view(L.shape) for q in parts]).contiguous()
    y, final = finish_piece(x, dt, A_log, B, C, D, S_all, L_all, rank, initial_states, ops)
    return (y, final) if return_final_states else y
