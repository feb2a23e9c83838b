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
