"""The benchmark's command-line contract on CPU: the reference arm's JSON line (the
oracle timed on the host cores), its behaviour on ranks other than 0, and the
warm-up floor. The GPU arm's line is produced only on a GPU machine.
"""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args, env=None):
    e = dict(os.environ)
    for key in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        e.pop(key, None)
    e.update(env or {})
    return subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, env=e, capture_output=True, text=True,
                          timeout=600)


def _last_json(stdout):
    lines = [line for line in stdout.splitlines() if line.startswith("{")]
    assert len(lines) == 1, stdout
    return json.loads(lines[0])


def test_reference_arm_line():
    r = _bench("--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    d = _last_json(r.stdout)
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["config"]["workload"] == "tiny" and "model" not in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] == d["value"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_without_work():
    r = _bench("--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "3", "--gpus", "2",
               env={"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [line for line in r.stdout.splitlines() if line.startswith("{")]


def test_warmup_floor():
    r = _bench("--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "2")
    assert r.returncode == 2 and "--warmup must be >= 3" in r.stderr


def test_traffic_digest_ignores_comments_and_layout_only():
    sys.path.insert(0, ROOT)
    import bench

    code = "__global__ void k(int *p)\n{\n    p[0] = 1; // one\n}\n"
    same = "/* a new comment */\n__global__ void k(int *p) {\n  p[0] = 1;   // changed comment\n}\n"
    other = "__global__ void k(int *p)\n{\n    p[0] = 2; // one\n}\n"
    assert bench._code_only(code) == bench._code_only(same)
    assert bench._code_only(code) != bench._code_only(other)
    assert bench.stored_traffic("permute", "no_such_workload") is None


def test_clock_window_tail():
    """The clock record's window: the timed region plus untimed repetitions up to ~30 ms."""
    import bench

    assert bench.clock_tail_reps(3.3) == 9  # 3.3 ms timed + 9 x 3.3 ms = 33 ms
    assert bench.clock_tail_reps(bench.CLOCK_WINDOW_MS) == 0
    assert bench.clock_tail_reps(100.0) == 0
    assert bench.clock_tail_reps(0.0) > 0


def test_pipelined_schedule_applies_to_plain_forward_steps():
    """Two batches in flight only where a step is route -> layout -> permute -> combine on
    one rank (no backward, TP folding, dedup view or exchange)."""
    import bench
    from synthetic import get_workload

    eligible = {name for name in ["tiny", "ht", "qwen3", "capacity", "ultraep"] + list(bench.EXTRA_WORKLOADS)
                if bench.pipelined_eligible(get_workload(name))}
    assert eligible == {"tiny", "ht", "qwen3", "capacity", "ht_align16"}


def test_kernels_per_call():
    import bench

    assert bench.kernels_per_call("layout") == 2 and bench.kernels_per_call("layout.1") == 2
    assert bench.kernels_per_call("dispatch") == 2 and bench.kernels_per_call("permute") == 1
    # the pipelined headline's step: route, layout (count + fill), permute, combine
    assert sum(bench.kernels_per_call(n) for n in ("route", "layout", "permute", "combine")) == 5
