"""bench.py --impl reference (the oracle timed on the host cores) keeps the
JSON-line contract, and only rank 0 prints under a multi-rank launch.
CPU only; the arm runs on a 16-token sample so the test takes seconds."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra, extra_args=("--impl", "reference", "--workload", "qwen3_0.6b_attn_qv",
                                 "--steps", "1", "--warmup", "3", "--ref-rows", "16")):
    env = dict(os.environ, **env_extra)
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *extra_args],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    return [l for l in out.stdout.splitlines() if l.startswith("{")]


def test_reference_arm_prints_one_contract_line():
    lines = _run({"RANK": "0", "WORLD_SIZE": "1"})
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 3 and d["value"] > 0
    assert d["config"]["workload"] == "qwen3_0.6b_attn_qv"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    assert _run({"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_default_workload_is_the_largest_single_gpu_config():
    import bench
    assert bench.DEFAULT_WORKLOAD == "14b_layer"
    assert set(bench.OTHER_WORKLOADS) == {"qwen3_0.6b_attn_qv", "8b_mlp"}


def test_gpus_flag_starts_one_rank_per_gpu():
    """--gpus 2 outside torchrun re-launches itself with torch.distributed.run:
    two ranks start, each sees its own RANK / LOCAL_RANK and WORLD_SIZE 2."""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    # The launcher picks its rendezvous port by binding port 0 and releasing
    # it; another process can take the port in between, so one retry.
    for attempt in range(2):
        out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--print-ranks"],
                             cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
        if out.returncode == 0:
            break
    assert out.returncode == 0, out.stderr[-2000:]
    ranks = sorted((json.loads(l)["rank"], json.loads(l)["local_rank"], json.loads(l)["world"])
                   for l in out.stdout.splitlines() if l.startswith("{"))
    assert ranks == [(0, 0, 2), (1, 1, 2)]


def test_default_sample_is_bounded():
    import bench
    import synth
    for name in ("qwen3_0.6b_attn_qv", "8b_mlp", "14b_layer"):
        wl = synth.workload(name)
        rows = bench.default_sample_rows(wl)
        assert 16 <= rows <= 1024 and bench.algorithmic_flops(wl, rows) <= 1.5e11
