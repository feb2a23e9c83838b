"""bench.py's output contract: one JSON line with the keys the benchmark
promises, from the reference arm (the oracle on the host, CPU) and from the
GPU arm (on a B200)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
             "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "e2e"}


def _run(args, timeout):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                         capture_output=True, text=True, timeout=timeout)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


@pytest.mark.timeout(600)
def test_reference_arm_json():
    r = _run(["--impl", "reference", "--config", "tiny", "--steps", "2", "--warmup", "3"], 500)
    assert BASE_KEYS <= set(r) and r["impl"] == "reference"
    assert r["value"] > 0 and r["unit"] == "tokens/s" and r["higher_is_better"] is True
    assert r["steps"] == 2 and r["warmup"] == 3 and r["n_gpus"] == 1
    cb = r["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == r["value"]
    assert r["e2e"]["h2d_bytes_per_step"] == 0 and r["e2e"]["value"] == r["value"]
    assert r["config"]["workload"].startswith("tiny")


@pytest.mark.gpu
@pytest.mark.timeout(900)
@pytest.mark.parametrize("extra", [[], ["--fp8"], ["--fused"], ["--layout", "padded"]],
                         ids=["bf16", "fp8", "fused", "padded"])
def test_gpu_arm_json(extra):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    r = _run(["--config", "tiny", "--steps", "3", "--warmup", "3", "--no-cpu-baseline",
              "--no-per-config", *extra], 800)
    assert BASE_KEYS <= set(r)
    assert r["value"] > 0 and r["device_status"] == 0 and r["gpu_launches"] > 0
    rf = r["roofline"]
    assert rf["bound"] in ("hbm", "tensor") and rf["achieved"] > 0 and rf["peak"] > 0
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-3
    assert set(r["clocks"]) == {"sm_mhz", "sm_max_mhz", "reasons"}
    e2e = r["e2e"]
    assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] == 64 * 128 * 2
    assert e2e["d2h_bytes_per_step"] == 64 * 128 * 2
    assert set(r["stages_ms"]) >= {"route", "permute", "gate_up", "down", "combine"}


def test_launches_per_step():
    """The gpu_launches arithmetic (checked against the CUDA profiler's count by
    tests/test_gpu_launch_count.py): 8 launches with a split router K, one fewer
    when the router's top-k runs in its GEMM epilogue, one more for the
    permutation's scan when the chunk histograms hold more than 4096
    counters, +2 row quantizers for FP8 experts, +1 fill for the padded
    layout."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_36_b200 import configs
    assert bench.launches_per_step(configs.MIXTRAL, 148) == 8              # 32 row tiles
    assert bench.launches_per_step(configs.SKEWED, 148) == 7               # 128 row tiles
    assert bench.launches_per_step(configs.SKEWED, 148, fp8=True) == 9
    assert bench.launches_per_step(configs.FINE, 148) == 9                 # + permutation scan
    assert bench.launches_per_step(configs.FINE, 148, padded=True) == 10
    assert bench.launches_per_step(configs.FINE, 148, fused=True) == 9
    assert bench.launches_per_step(configs.DECODE.with_tokens(16), 148, fp8=True) == 10
    assert bench.launches_per_step(configs.TINY.with_tokens(0), 148) == 0


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun_two_ranks():
    """Launched the way the multi-GPU runs are (torchrun, two ranks): rank 0
    alone times the oracle and prints the one JSON line; rank 1 exits 0."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    out = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                          "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
                          "--master-port", str(port), os.path.join(ROOT, "bench.py"),
                          "--impl", "reference", "--config", "tiny", "--gpus", "2",
                          "--steps", "2", "--warmup", "3"],
                         cwd=ROOT, capture_output=True, text=True, timeout=500)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    r = json.loads(lines[0])
    assert r["impl"] == "reference" and r["n_gpus"] == 2 and r["value"] > 0


@pytest.mark.parametrize("extra,stages", [
    ([], ["route", "permute", "gate_up", "down", "combine"]),
    (["--fp8"], ["route", "quant_x", "permute", "gate_up", "quant_h", "down", "combine"]),
    (["--fused"], ["route", "permute", "gate_up", "down", "combine"]),
    (["--layout", "padded"], ["route", "permute", "gate_up", "down", "combine"]),
], ids=["bf16", "fp8", "fused", "padded"])
def test_gpu_arm_json_assembly_on_cpu(monkeypatch, capsys, extra, stages):
    """bench.py's JSON line from the GPU arm's measurements, with the GPU arm
    replaced by fixed numbers (CPU): every contract key present and the
    roofline arithmetic (algorithmic work / mean duration / peak) consistent."""
    import sys
    import types
    sys.path.insert(0, ROOT)
    import bench
    import torch
    from mixture_experts_layer_36_b200 import configs
    cfg = configs.by_name("skewed")
    mean = {n: 0.1 * (i + 1) for i, n in enumerate(stages)}
    fake = {"elapsed_ms": 12.0, "stage_ms": {n: v * 0.9 for n, v in mean.items()},
            "stage_mean": mean, "status": 0, "N": 30000, "active_experts": 60,
            "n_dropped": 5, "clocks": {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": []},
            "e2e_ms": 15.0, "h2d": cfg.T * cfg.d * 2, "d2h": cfg.T * cfg.d * 2,
            "layer": types.SimpleNamespace(rows=cfg.E * 1536)}
    monkeypatch.setattr(bench, "gpu_arm", lambda *a, **k: fake)
    monkeypatch.setattr(torch.cuda, "get_device_properties",
                        lambda *_: types.SimpleNamespace(multi_processor_count=148))
    monkeypatch.setattr(sys, "argv", ["bench.py", "--config", "skewed", "--steps", "4",
                                      "--warmup", "3", "--no-cpu-baseline", "--no-per-config",
                                      *extra])
    bench.main()
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    r = json.loads(lines[0])
    assert BASE_KEYS <= set(r) and {"roofline", "clocks", "gpu_launches"} <= set(r)
    assert r["value"] == pytest.approx(cfg.T * 4 / 12e-3, rel=1e-6)
    assert r["e2e"]["value"] == pytest.approx(cfg.T * 4 / 15e-3, rel=1e-6)
    assert r["gpu_launches"] == 4 * bench.launches_per_step(
        cfg, 148, "--fp8" in extra, "padded" in extra, "--fused" in extra)
    rf = r["roofline"]
    assert rf["duration_ms"] == pytest.approx(mean["gate_up"])
    assert rf["frac"] == pytest.approx(rf["achieved"] / rf["peak"], abs=1e-3)
    if rf["bound"] == "tensor":
        assert rf["achieved"] == pytest.approx(
            4.0 * 30000 * cfg.d * cfg.f / (mean["gate_up"] / 1e3) / 1e12, rel=1e-3)
    assert r["stages_mean_ms"] == {n: round(v, 4) for n, v in mean.items()}
    assert set(r["stages_ms"]) == set(stages)


def test_per_config_assembly_on_cpu(monkeypatch, capsys):
    """per_config from fixed numbers (CPU): one entry per workload, the headline
    first, each roofline fraction recomputing from its own line."""
    import sys
    import types
    sys.path.insert(0, ROOT)
    import bench
    import torch
    from mixture_experts_layer_36_b200 import configs
    stages = ["route", "permute", "gate_up", "down", "combine"]
    seen = []

    def fake_arm(args, c, rank, world, local_rank, with_e2e=True):
        seen.append((c.name, with_e2e))
        mean = {n: 0.05 * (i + 1) for i, n in enumerate(stages)}
        N = min(c.T * c.k, bench.moe_max_rows_host(c))
        r = {"elapsed_ms": 2.0 * args.steps, "stage_ms": dict(mean), "stage_mean": mean,
             "status": 0, "N": N, "active_experts": min(c.E, N), "n_dropped": c.T * c.k - N,
             "clocks": {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": []},
             "layer": types.SimpleNamespace(rows=N)}
        if with_e2e:
            r.update(e2e_ms=3.0 * args.steps, h2d=c.T * c.d * 2, d2h=c.T * c.d * 2)
        return r

    monkeypatch.setattr(bench, "gpu_arm", fake_arm)
    monkeypatch.setattr(torch.cuda, "get_device_properties",
                        lambda *_: types.SimpleNamespace(multi_processor_count=148))
    monkeypatch.setattr(sys, "argv", ["bench.py", "--steps", "4", "--warmup", "3",
                                      "--no-cpu-baseline"])
    bench.main()
    r = json.loads([ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")][0])
    per = r["per_config"]
    want = [configs.by_name(n).name for n in bench.PER_CONFIG]
    assert list(per)[0] == "mixtral" and sorted(per) == sorted(want)
    assert seen[0] == ("mixtral", True) and all(not e for _, e in seen[1:])
    for name, e in per.items():
        c = configs.by_name(name)
        assert e["tokens_per_s"] == pytest.approx(c.T * 4 / (8.0e-3), rel=1e-6)
        rf = e["roofline"]
        assert rf["frac"] == pytest.approx(rf["achieved"] / rf["peak"], abs=1e-3)
        for st in ("permute", "combine"):
            h = e["stage_rooflines"][st]
            assert h["achieved"] == pytest.approx(
                h["algorithmic_bytes"] / (h["duration_ms"] / 1e3) / 1e9, rel=1e-3)
            assert h["frac"] == pytest.approx(h["achieved"] / h["peak"], abs=1e-3)
    # decode sizes are weight-streaming: bound by HBM on the active experts' weights
    assert per["decode@T16"]["roofline"]["bound"] == "hbm"
    assert per["mixtral"]["roofline"]["bound"] == "tensor"


def test_reference_arm_config_equals_gpu_arm_config():
    """Both arms describe the workload with the same `config` object."""
    import argparse
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_36_b200 import configs
    args = argparse.Namespace(fp8=False, fused=False, layout="ragged")
    for name in bench.PER_CONFIG:
        c = configs.by_name(name)
        assert bench.workload_config(c, args, 1) == bench.workload_config(c, args, 1)
    ref = _run(["--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "3"], 300)
    assert ref["config"] == bench.workload_config(configs.TINY, args, 1)
