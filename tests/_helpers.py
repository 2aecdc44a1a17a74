"""Shared helpers for the GPU parity tests: move seeded inputs to the device,
run the library through its C ABI, compare with the oracle."""
import numpy as np

import ssd_inputs

BF16_TOL = 2e-2   # max|dy| / max|y_oracle| for bf16 inputs
F32_TOL = 1e-4    # same, float32 path

# (test, y error, final-state error, tolerance) of the parity checks that ran,
# printed in pytest's terminal summary so that every margin is on record
PARITY_LOG = []


def record_parity(name, ey, ef, tol):
    PARITY_LOG.append((name, float(ey), None if ef is None else float(ef), float(tol)))


def to_device(inp: dict, device="cuda"):
    import torch
    io = torch.bfloat16 if inp["io_dtype"] == "bf16" else torch.float32
    t = {}
    for k in ("x", "dt", "B", "C"):
        t[k] = torch.from_numpy(np.ascontiguousarray(inp[k])).to(device=device, dtype=io)
    for k in ("A_log", "D", "initial_states"):
        v = inp.get(k)
        t[k] = None if v is None else torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).to(device)
    cu = inp.get("cu_seqlens")
    t["cu_seqlens"] = None if cu is None else torch.from_numpy(np.asarray(cu, dtype=np.int32)).to(device)
    return t


def run_gpu(inp: dict, path="auto", chunk_len=None, final=True, stream=None):
    """Returns (y float64 numpy with x's shape, final states float64 or None)."""
    import torch
    import mamba_ssd_layer_fwd_b200 as ssd
    t = to_device(inp)
    out = ssd.ssd_fwd(t["x"], t["dt"], t["A_log"], t["B"], t["C"], t["D"],
                      chunk_len=chunk_len or inp["chunk_len"], initial_states=t["initial_states"],
                      cu_seqlens=t["cu_seqlens"], dt_softplus=inp.get("dt_softplus", True),
                      return_final_states=final, path=path, stream=stream, check_status=True)
    torch.cuda.synchronize()
    if final:
        y, f = out
        return y.double().cpu().numpy(), f.double().cpu().numpy()
    return out.double().cpu().numpy(), None


def rel_max_err(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), "non-finite output"
    scale = float(np.max(np.abs(want)))
    return float(np.max(np.abs(got - want))) / max(scale, 1e-30)


def small_inputs(batch=2, seqlen=700, H=4, P=64, N=128, G=1, Q=256, io="bf16", init=True,
                 varlen=None, seed=0, **kw):
    """A seeded problem with the value distributions of the bf16 benchmark shapes."""
    nseq = len(varlen) if varlen is not None else 0
    if varlen is not None:
        kw.setdefault("min_seqlen", 0)
    kw.setdefault("xbc_std", 1.0 / np.sqrt(N))
    kw.setdefault("dt_shift", 3.0)
    kw.setdefault("a_log_hi", 2.7)
    w = ssd_inputs.Workload("test", 1 if varlen is not None else batch,
                            int(sum(varlen)) if varlen is not None else seqlen, H, P, N, G, Q, io,
                            num_seqs=nseq, with_initial_states=init, with_final_states=True,
                            seed=seed, **kw)
    inp = ssd_inputs.make_inputs(w)
    if varlen is not None:
        inp["cu_seqlens"] = np.concatenate([[0], np.cumsum(varlen)]).astype(np.int32)
    return inp
