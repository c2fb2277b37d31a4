"""The benchmark's reference arm (the CPU oracle on the host cores) runs
without a GPU and prints one JSON line with the contract's keys."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "GB/s"
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in d["config"] and d["metric"]


def _bench():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_runs_of_equal_names():
    b = _bench()
    assert b.runs_of_equal_names([]) == []
    assert b.runs_of_equal_names(["w", "g", "g", "g", "g"]) == [(0, 1), (1, 5)]
    assert b.runs_of_equal_names(["w", "q", "g", "q", "g"]) == [(0, 1), (1, 2), (2, 3), (3, 4), (4, 5)]
    assert b.runs_of_equal_names(["a", "a", "b", "a"]) == [(0, 2), (2, 3), (3, 4)]


def test_detail_capture_brackets_runs_of_one_kernel():
    """The per-kernel timing capture (a stand-in for torch.cuda's graph and
    events; nothing runs on a GPU): one event pair per run of consecutive
    launches of one kernel, with the run's launches, bytes and flops, and
    every op called once per step in order."""
    import contextlib
    import types

    b = _bench()
    called = []

    class Ev:
        def __init__(self, **kw):
            self.recorded = 0

        def record(self):
            self.recorded += 1

    fake_torch = types.SimpleNamespace(cuda=types.SimpleNamespace(
        CUDAGraph=lambda: object(), graph=lambda g: contextlib.nullcontext(), Event=Ev))
    gw = b.GpuWorkload.__new__(b.GpuWorkload)
    gw.torch = fake_torch

    def ops_of_step(s):
        names = ["prune"] + ["fused"] * 4
        return [(nm, (lambda s=s, i=i: called.append((s, i))), 10 + i, 100 * i, 1) for i, nm in enumerate(names)]

    gw.ops_of_step = ops_of_step
    g, evs = gw.capture(2, 3, events=True)
    assert called == [(s, i) for s in (3, 4) for i in range(5)]
    assert [(e[0], e[1], e[2], e[3]) for e in evs] == [("prune", 10, 0, 1), ("fused", 11 + 12 + 13 + 14, 1000, 4)] * 2
    assert all(e[4].recorded == 1 and e[5].recorded == 1 for e in evs)
    called.clear()
    g, evs = gw.capture(1, 0, events=False)
    assert evs == [] and called == [(0, i) for i in range(5)]
