"""The Python binding's argument checks (CPU, no library calls).

The kernels read and write every buffer over the extent the shapes imply, so a
host tensor, a short output, a strided view or a tensor on another device must
be refused before anything is launched.  The checks use tensor metadata only;
these tests drive them with `meta` tensors, which carry dtype, shape, stride
and device but no storage, so they run without a GPU.  One valid argument set
per entry point (the shapes the parity tests and the benchmark use) must pass,
and every single-argument fault must raise.
"""
import pytest

torch = pytest.importorskip("torch")

import mamba_ssd_layer_fwd_b200 as ssd  # noqa: E402

META = torch.device("meta")
BF16, F32, I32 = torch.bfloat16, torch.float32, torch.int32


def t(*shape, dtype=F32, device=META):
    return torch.empty(shape, dtype=dtype, device=device)


def fwd_args(b=2, T=700, H=4, P=64, G=2, N=128, io=BF16, varlen=None):
    nseq = b if varlen is None else varlen
    return dict(x=t(b, T, H, P, dtype=io), dt=t(b, T, H, dtype=io), A_log=t(H), B=t(b, T, G, N, dtype=io),
                C=t(b, T, G, N, dtype=io), D=t(H), initial_states=t(nseq, H, P, N),
                cu_seqlens=None if varlen is None else t(varlen + 1, dtype=I32), y=t(b, T, H, P, dtype=io),
                final_states=t(nseq, H, P, N), workspace=t(4096, dtype=torch.uint8))


def test_fwd_accepts_valid_arguments():
    assert ssd._validate_fwd(**fwd_args()) == 2
    assert ssd._validate_fwd(**fwd_args(b=1, T=1200, varlen=4)) == 4
    assert ssd._validate_fwd(**fwd_args(io=F32, G=1, N=16, P=16)) == 2
    a = fwd_args()
    for k in ("D", "initial_states", "y", "final_states", "workspace"):
        a[k] = None
    assert ssd._validate_fwd(**a) == 2
    # empty batch and gated norm
    e = fwd_args(T=0)
    e["z"], e["norm_weight"], e["norm_bias"] = t(2, 0, 4, 64, dtype=BF16), t(4 * 64), None
    assert ssd._validate_fwd(**e) == 2


@pytest.mark.parametrize("name,bad", [
    ("dt", t(2, 700, 3, dtype=BF16)),               # wrong head count
    ("dt", t(2, 700, 4, dtype=F32)),                # dtype differs from x
    ("dt", None),                                    # required
    ("A_log", t(5)),                                 # one value per head
    ("A_log", t(4, dtype=BF16)),
    ("A_log", None),
    ("B", t(2, 700, 2, 128, dtype=F32)),
    ("C", t(2, 700, 2, 64, dtype=BF16)),             # dstate differs from B
    ("C", t(2, 699, 2, 128, dtype=BF16)),
    ("C", None),
    ("D", t(3)),
    ("initial_states", t(2, 4, 64, 64)),
    ("initial_states", t(2, 4, 64, 128, dtype=BF16)),
    ("y", t(2, 700, 4, 32, dtype=BF16)),             # short output
    ("y", t(2, 700, 4, 64, dtype=F32)),
    ("final_states", t(1, 4, 64, 128)),
    ("x", t(2, 700, 4, 64, dtype=BF16).transpose(0, 1)),   # strided view, (700, 2, ...) shape
])
def test_fwd_rejects_each_bad_argument(name, bad):
    a = fwd_args()
    a[name] = bad
    with pytest.raises((ValueError, TypeError)):
        ssd._validate_fwd(**a)


def test_fwd_rejects_non_contiguous_and_foreign_device():
    a = fwd_args()
    a["y"] = t(2, 700, 4, 128, dtype=BF16)[..., ::2]            # right shape, strided
    with pytest.raises(ValueError, match="contiguous"):
        ssd._validate_fwd(**a)
    for name in ("dt", "A_log", "D", "y", "final_states", "initial_states"):
        a = fwd_args()
        a[name] = torch.empty(tuple(a[name].shape), dtype=a[name].dtype)   # host memory
        with pytest.raises(ValueError, match="must be on"):
            ssd._validate_fwd(**a)
    a = fwd_args()
    a["workspace"] = torch.empty(16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="workspace"):
        ssd._validate_fwd(**a)


def test_fwd_cu_seqlens_checks():
    a = fwd_args(b=1, T=1200, varlen=4)
    a["cu_seqlens"] = torch.zeros(5, dtype=I32)                 # a host array would be read by the planner kernel
    with pytest.raises(ValueError, match="must be on"):
        ssd._validate_fwd(**a)
    a["cu_seqlens"] = t(5, dtype=torch.int64)
    with pytest.raises(ValueError):
        ssd._validate_fwd(**a)
    a["cu_seqlens"] = t(1, dtype=I32)
    with pytest.raises(ValueError, match="entries"):
        ssd._validate_fwd(**a)
    a = fwd_args(b=1, T=1200, varlen=4)
    a["initial_states"] = t(1, 4, 64, 128)                      # one state per sequence, not per row
    with pytest.raises(ValueError, match="initial_states"):
        ssd._validate_fwd(**a)


def test_fwd_dtype_of_x():
    a = fwd_args()
    a["x"] = t(2, 700, 4, 64, dtype=torch.float16)
    with pytest.raises(TypeError):
        ssd._validate_fwd(**a)


def test_gated_norm_arguments():
    a = fwd_args()
    a["z"], a["norm_weight"], a["norm_bias"] = t(2, 700, 4, 64, dtype=BF16), t(256), t(256)
    assert ssd._validate_fwd(**a) == 2
    for name, bad in (("z", t(2, 700, 4, 64, dtype=F32)), ("z", t(2, 700, 4, 32, dtype=BF16)),
                      ("norm_weight", None), ("norm_weight", t(255)), ("norm_bias", t(128)),
                      ("norm_weight", torch.empty(256))):
        b = dict(a)
        b[name] = bad
        with pytest.raises(ValueError):
            ssd._validate_fwd(**b)
    c = fwd_args()
    c["norm_weight"] = t(256)                                   # without z it would be ignored silently
    with pytest.raises(ValueError, match="only together with z"):
        ssd._validate_fwd(**c)


def test_summary_arguments():
    a = fwd_args(b=1, T=1200, varlen=4)
    assert ssd._validate_summary(a["x"], a["dt"], a["A_log"], a["B"], a["cu_seqlens"], a["workspace"]) == 4
    with pytest.raises(ValueError):
        ssd._validate_summary(a["x"], a["dt"], a["A_log"], t(1, 1200, 2, 128, dtype=F32), a["cu_seqlens"])
    with pytest.raises(ValueError):
        ssd._validate_summary(a["x"], a["dt"], None, a["B"])


def test_bwd_arguments():
    a = fwd_args()
    dy = t(2, 700, 4, 64, dtype=BF16)
    ok = dict(x=a["x"], dt=a["dt"], A_log=a["A_log"], B=a["B"], C=a["C"], D=a["D"], dy=dy,
              initial_states=a["initial_states"], dfinal_states=t(2, 4, 64, 128), workspace=a["workspace"])
    assert ssd._validate_bwd(**ok) == 2
    assert ssd._validate_bwd(**dict(ok, D=None, initial_states=None, dfinal_states=None)) == 2
    for name, bad in (("dy", t(2, 700, 4, 64, dtype=F32)), ("dy", None), ("dfinal_states", t(2, 4, 64, 64)),
                      ("C", t(2, 700, 1, 128, dtype=BF16)), ("dt", t(2, 700, 4))):
        with pytest.raises(ValueError):
            ssd._validate_bwd(**dict(ok, **{name: bad}))


def test_decode_arguments():
    b, H, P, G, N = 64, 80, 64, 1, 128
    ok = dict(x=t(b, H, P, dtype=BF16), dt=t(b, H, dtype=BF16), A_log=t(H), B=t(b, G, N, dtype=BF16),
              C=t(b, G, N, dtype=BF16), D=t(H), state=t(b, H, P, N), y=t(b, H, P, dtype=BF16))
    ssd._validate_decode(**ok)
    ssd._validate_decode(**dict(ok, D=None, y=None))
    ssd._validate_decode(**dict(ok, x=t(0, 2, 64, dtype=BF16), dt=t(0, 2, dtype=BF16), A_log=t(2),
                                B=t(0, 1, 64, dtype=BF16), C=t(0, 1, 64, dtype=BF16), D=None,
                                state=t(0, 2, 64, 64), y=None))
    for name, bad in (("state", t(b, H, P, 64)), ("state", None), ("state", t(b, H, P, N, dtype=BF16)),
                      ("y", t(b, H, 32, dtype=BF16)), ("A_log", t(H - 1)), ("C", t(b, 2, N, dtype=BF16)),
                      ("dt", t(b, H + 1, dtype=BF16)), ("B", t(b, G, N))):
        with pytest.raises(ValueError):
            ssd._validate_decode(**dict(ok, **{name: bad}))


def test_combine_arguments():
    S, L = t(4, 2, 3, 8, 16), t(4, 2, 3)
    for rank in range(5):
        ssd._validate_combine(S, L, rank, t(2, 3, 8, 16), t(2, 3, 8, 16))
    for kw in (dict(rank=5), dict(rank=-1), dict(logdecay_all=t(4, 2, 2)), dict(initial_states=t(2, 3, 8, 8)),
               dict(out=t(2, 3, 8, 16, dtype=BF16)), dict(logdecay_all=torch.empty(4, 2, 3))):
        args = dict(end_states_all=S, logdecay_all=L, rank=1, initial_states=None, out=None)
        args.update(kw)
        with pytest.raises(ValueError):
            ssd._validate_combine(**args)
