"""bench.py's output contract, checked on the host.

The reference arm (the CPU oracle timed on a bounded sample) runs without a
GPU, so its JSON line is checked here in full; the GPU arm must fail loudly
when no CUDA device is present (there is no CPU fallback)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SMALL = "gmm16-n2048-d64-f32"


def _run(args, env=None, timeout=300):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          cwd=ROOT, env=e, timeout=timeout)


def test_reference_arm_prints_one_complete_line():
    r = _run(["--impl", "reference", "--workload", SMALL, "--steps", "2", "--warmup", "1"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["impl"] == "reference" and j["unit"] == "calls/s" and j["higher_is_better"] is True
    assert j["steps"] == 2 and j["warmup"] == 1 and j["value"] > 0
    # a step is one bounded sample: steps x ms_per_step is the measured wall
    # time, and value extrapolates the samples to whole calls
    assert j["extrapolated"] is True
    cb = j["cpu_baseline"]
    assert cb["samples_timed"] == 2 and abs(cb["wall_s"] - 2 * j["ms_per_step"] / 1e3) < 1e-6 * cb["wall_s"]
    assert cb["scale_per_sample"] > 1
    assert j["config"]["workload"] == SMALL
    import bench
    from clustered_sparse_attention_head_b200 import workloads as W
    assert j["config"] == bench.config_of(W.WORKLOADS[SMALL], 1), "the reference config must equal the GPU arm's"
    assert "flushed" in j["config"]["l2"], "a workload smaller than L2 is timed with an L2 flush"
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == j["value"] and cb["sample"]
    assert j["e2e"] == {"value": j["value"], "unit": "calls/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    r = _run(["--impl", "reference", "--workload", SMALL, "--steps", "1", "--warmup", "0"],
             env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and not r.stdout.strip()


def test_l2_policy_follows_the_tensor_size():
    import bench
    from clustered_sparse_attention_head_b200 import workloads as W
    big = bench.config_of(W.WORKLOADS["wan21-n75600-h40-d128"], 1)["l2"]
    assert big.startswith("inputs larger than L2 (774 MB per tensor)")
    assert "flushed" in bench.config_of(W.WORKLOADS["cogvideox2b-n17776-h30-d64"], 1)["l2"]


def test_gpu_arm_fails_loudly_without_a_device():
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    r = _run(["--workload", SMALL, "--steps", "1", "--warmup", "0", "--no-cpu-baseline"])
    assert r.returncode != 0
    assert not any(ln.startswith("{") for ln in r.stdout.splitlines())


def test_select_mode_names_config_fields():
    """--select-mode accepts only the listed options, and every option sets
    fields the binding's Config has (the main call's contexts take them)."""
    import bench
    from clustered_sparse_attention_head_b200 import workloads as W
    from clustered_sparse_attention_head_b200.api import Config
    r = _run(["--select-mode", "no_such_mode", "--steps", "1"])
    assert r.returncode == 2 and "invalid choice" in r.stderr
    cfg = Config.from_workload(W.WORKLOADS["wan21-n75600-h40-d128"])
    assert bench.SELECT_MODES, "no selection options listed"
    for name, over in bench.SELECT_MODES.items():
        for key in over:
            assert hasattr(cfg, key), f"{name}: Config has no field {key}"
    assert bench.SELECT_MODES["per_query_top_k64"] == {"top_k": 64, "per_query": True}


def test_cluster_count_overrides_reach_the_config():
    r = _run(["--impl", "reference", "--workload", SMALL, "--kq", "9", "--kk", "13", "--steps", "1",
              "--warmup", "0"])
    assert r.returncode == 0, r.stderr[-2000:]
    j = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][0])
    assert j["config"]["kq"] == 9 and j["config"]["kk"] == 13
