"""Host logic of the multi-GPU (replica) benchmark, as two gloo ranks on the
CPU: distinct token batches per rank, identical weights, and the timed value
taken as the max over ranks."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    from mixture_experts_layer_36_b200 import configs, synth
    cfg = configs.TINY
    x = synth.make_tokens(cfg, "cpu", seed=bench.rank_token_seed(cfg, rank))
    w = synth.make_weights(cfg, "cpu")
    # gather a fingerprint of each rank's batch and weights on every rank
    fp = torch.tensor([x.float().sum().item(), w["w_gate"].float().sum().item()],
                      dtype=torch.float64)
    allfp = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(allfp, fp)
    slowest = bench.max_over_ranks(10.0 * (rank + 1), "cpu", True)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, [t.tolist() for t in allfp], slowest))


@pytest.mark.timeout(180)
def test_two_replicas_on_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=170) for _ in range(world)]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, fps, slowest in res:
        assert slowest == 10.0 * world          # max over ranks, seen by every rank
        (x0, w0), (x1, w1) = fps
        assert x0 != x1                         # each replica has its own tokens
        assert w0 == w1                         # and the same weights


def _bench_worker(rank, world, port, out):
    """bench.main() on a gloo rank with the GPU arm replaced by a stand-in
    that takes the same collective steps (a barrier-free max over ranks)."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK="0")
    import datetime
    import io
    import contextlib
    import json
    import types
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    calls = []

    def fake_arm(args, c, r, wsize, local_rank, with_e2e=True):
        calls.append(c.name)
        t = bench.max_over_ranks(1.0 + r, "cpu", True)       # a collective on every rank
        mean = {n: 0.05 for n in ("route", "permute", "gate_up", "down", "combine")}
        N = min(c.T * c.k, bench.moe_max_rows_host(c))
        res = {"elapsed_ms": t * args.steps, "stage_ms": dict(mean), "stage_mean": mean,
               "status": 0, "N": N, "active_experts": min(c.E, N), "n_dropped": 0,
               "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []},
               "layer": types.SimpleNamespace(rows=N)}
        if with_e2e:
            res.update(e2e_ms=2.0 * t * args.steps, h2d=8, d2h=8)
        return res

    bench.gpu_arm = fake_arm
    torch.cuda.get_device_properties = lambda *_: types.SimpleNamespace(multi_processor_count=148)
    sys.argv = ["bench.py", "--gpus", str(world), "--steps", "2", "--warmup", "3",
                "--no-cpu-baseline"]
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main()                 # destroys the process group at the end
    lines = [ln for ln in buf.getvalue().splitlines() if ln.startswith("{")]
    out.put((rank, calls, [json.loads(ln) for ln in lines]))


@pytest.mark.timeout(180)
def test_bench_main_on_two_gloo_ranks():
    """The multi-GPU bench path with its per-workload runs: every rank runs the
    same workloads in the same order (same collective steps), the time is the
    slowest rank's, and rank 0 alone prints one line with every workload."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bench_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=170) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    (r0, calls0, lines0), (r1, calls1, lines1) = res
    assert calls0 == calls1 and calls0[0] == "mixtral" and len(calls0) == 7
    assert len(lines0) == 1 and lines1 == []
    line = lines0[0]
    assert line["n_gpus"] == 2 and line["ms_per_step"] == pytest.approx(2.0)   # max over ranks
    assert line["value"] == pytest.approx(4096 * 2 * 2 / (4.0e-3))          # both ranks' tokens
    assert len(line["per_config"]) == 7 and "cpu_baseline" not in line
