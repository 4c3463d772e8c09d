"""bench.py's JSON line: the reference arm (the CPU oracle) runs here without a
GPU and must print the keys the benchmark contract names."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=e,
                       capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    return [json.loads(l) for l in lines]


@pytest.mark.parametrize("config", ["glam_small_bf16", "glm_small_bf16", "glam_dense_small_bf16"])
def test_reference_arm_line(config):
    (out,) = run_bench("--impl", "reference", "--config", config, "--steps", "2", "--warmup", "1",
                       "--ref-seconds", "3")
    assert out["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in out, key
    assert out["value"] > 0 and out["unit"] == "tokens/s" and out["higher_is_better"] is True
    assert out["config"]["workload"] == config
    cb = out["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == out["value"] and cb["sample"]
    assert out["e2e"] == {"value": out["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
    dense = config.startswith("glam_dense")
    assert out["metric"].startswith("dense FFN layer" if dense else "MoE-layer")


def test_reference_arm_other_ranks_print_nothing():
    assert run_bench("--impl", "reference", "--config", "glam_small_bf16", "--steps", "1", "--warmup", "1",
                     "--ref-seconds", "1", env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []


@pytest.mark.parametrize("config", ["glam_small_bf16", "glm_small_bf16"])
def test_backward_cpu_baseline_sample(config):
    """The backward leg's CPU baseline (the fp64 backward oracle on the first
    tokens, restricted to the experts they chose) runs on host tensors."""
    sys.path.insert(0, ROOT)
    import torch

    import bench
    import moe_synth as ms
    import oracle

    cfg = ms.get_config(config)
    inp = ms.layer_inputs(cfg, "cpu")
    dy = ms.upstream_grad(cfg, "cpu")
    f64 = lambda t: None if t is None else t.to(torch.float64).numpy()  # noqa: E731
    r = oracle.route(f64(inp["x"]), f64(inp["w_r"]), f64(inp["e_bias"]), cfg["k"], cfg["gate"],
                     cfg["norm_topk_prob"], cfg["alpha"], cfg["eps"])
    cb = bench.backward_cpu_baseline(cfg, inp, dy, r["idx"], target_s=0.05, max_experts=6)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["unit"] == "tokens/s" and cb["cores"] >= 1
    assert "experts they chose" in cb["sample"]
