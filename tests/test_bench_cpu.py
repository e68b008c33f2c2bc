"""bench.py on the host alone: the reference arm (the fp64 oracle on the host cores) prints one JSON
line with the bench keys, ranks other than 0 exit without work, and fewer than 3 warm-up steps are
refused.  No GPU is touched."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, env=e, capture_output=True, text=True,
                          timeout=300)


def test_reference_arm_prints_one_contract_line():
    # the default arm times every request of the workload; 8 keep this test short
    import bench
    from paged_kv_cache_461_b200 import workloads as W
    r = _bench("--impl", "reference", "--steps", "3", "--warmup", "3", "--reference-requests", "8")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["value"] > 0 and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1
    # the same config object as our arm's line (the whole workload), so the two lines compare
    assert d["config"] == bench.job_config(W.workload_layout(bench.HEADLINE), 1)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert cb["sample"].startswith("the first 8 of 256 requests") and d["oracle_kv_write_ms"] > 0
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_without_work():
    r = _bench("--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3",
               env={"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0 and not r.stdout.strip()


def test_fewer_than_three_warmups_are_refused():
    r = _bench("--impl", "reference", "--steps", "3", "--warmup", "2")
    assert r.returncode != 0 and "warm-up" in r.stderr


def test_clock_sampler_always_ends_its_child():
    # stop() (and the exit hook) end the background sampler process; a stand-in child replaces nvidia-smi
    import shutil
    import threading

    import bench
    if shutil.which("sleep") is None:
        return
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.rows, s.first = [], threading.Event()
    s.proc = subprocess.Popen(["sleep", "30"], stdout=subprocess.PIPE, text=True)
    s.t = threading.Thread(target=s._read, daemon=True)
    s.t.start()
    r = s.stop(0.0, 1.0)
    assert s.proc.poll() is not None and r["samples"] == 0
    s._kill()                                            # a second end is harmless


def test_clock_sampler_without_nvidia_smi_reports_it():
    import shutil

    import bench
    if shutil.which("nvidia-smi") is not None:
        return
    r = bench.ClockSampler(0).stop(0.0, 1.0)
    assert r["reasons"] == ["nvidia-smi unavailable"] and r["samples"] == 0
