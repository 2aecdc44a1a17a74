"""The bench's reference arm (the fp64 oracle timed on the host cores) prints
one JSON line with the fields of the bench contract; it needs no GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "small_bf16", "--steps", "1", "--warmup", "3", "--ref-seconds", "0.5"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["warmup"] >= 3
    assert d["config"]["workload"] == "small_bf16"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_traffic_figures_follow_code_not_comments():
    """The committed ncu traffic applies while the CUDA code (not its comments)
    is unchanged."""
    sys.path.insert(0, ROOT)
    import bench
    a = "int f() { return 1; } // one\n/* block\ncomment */ int g;"
    b = "int f() {  return 1; }   // another comment\nint g;"
    c = "int f() { return 2; } // one\nint g;"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)
    h = bench.kernel_source_hash()
    assert len(h) == 16 and h == bench.kernel_source_hash()


def test_timed_loop_with_and_without_flush(monkeypatch):
    """Forward.timed runs warm-up + timed steps with the L2 flush before each,
    or with none (the warm-L2 figures), and a device error during the warm-L2
    run ends up in the JSON line instead of ending the bench.  Fake CUDA
    events stand in for the GPU."""
    import types
    import torch
    sys.path.insert(0, ROOT)
    import bench

    class Ev:
        clock = 0

        def __init__(self, enable_timing=False):
            self.t = None

        def record(self, stream=None):
            Ev.clock += 1
            self.t = Ev.clock

        def elapsed_time(self, other):
            return float(other.t - self.t)

    class Flush:
        def __init__(self):
            self.n = 0

        def zero_(self):
            self.n += 1

    monkeypatch.setattr(torch.cuda, "Event", Ev)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    fw = object.__new__(bench.Forward)
    calls = []
    fw.stream = None
    fw.step = lambda events=None: calls.append(events)
    fw.status = lambda: 0
    fw.ssd = types.SimpleNamespace(SsdError=lambda rc, what: RuntimeError(f"{what}: {rc}"))
    fl = Flush()
    s, c, m, _ = fw.timed(4, 3, fl)
    assert fl.n == 7 and len(calls) == 7 and len(s) == len(c) == len(m) == 4
    assert all(e is not None and len(e) == 3 for e in calls[3:]) and all(e is None for e in calls[:3])
    assert all(v > 0 for v in s + c + m)
    calls.clear()
    s, c, m, _ = fw.timed(5, 3, None)
    assert len(calls) == 8 and len(s) == 5 and fl.n == 7
    w = bench.warm_l2_stats(fw, 6)
    assert w["steps"] == 6 and set(w) == {"steps", "step_ms", "compute_ms", "output_pass_ms"}
    assert w["step_ms"]["min"] > 0
    fw.status = lambda: -4
    w = bench.warm_l2_stats(fw, 6)
    assert set(w) == {"error"} and "-4" in w["error"]


def test_accounting_of_the_benchmark_workloads():
    """Bytes and FLOPs per forward, worked out by hand from the shapes:
    2.7B-shaped layer (8 x 2048 tokens, H 80, P 64, N 128, G 1, bf16):
    x + y = 2 * 167,772,160 B, dt 2,621,440 B, B + C = 2 * 4,194,304 B;
    16K GVA (H 32, P 64, N 256, G 8) adds 32 * 64 * 256 = 524,288 floats of final state."""
    sys.path.insert(0, ROOT)
    import bench
    import ssd_inputs
    inp = ssd_inputs.make_inputs(ssd_inputs.workload("mamba2_2p7b"), seed=0)
    assert bench.algorithmic_bytes(inp) == 2 * 167_772_160 + 2_621_440 + 2 * 4_194_304
    tok = 8 * 2048
    assert bench.algorithmic_flops(inp, 128) == tok * (80 * (4 * 64 * 128 + 128 * 64) + 128 * 128)
    assert bench.full_tile_flops(inp, 256) == tok * (80 * (4 * 64 * 128 + 2 * 256 * 64) + 2 * 256 * 128)
    inp = ssd_inputs.make_inputs(ssd_inputs.workload("long16k_gva"), seed=0)
    assert bench.algorithmic_bytes(inp) == 2 * 67_108_864 + 1_048_576 + 2 * 67_108_864 + 4 * 524_288
