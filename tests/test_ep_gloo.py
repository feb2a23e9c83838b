"""Host logic of the expert-parallel layer (mixture_experts_layer_36_b200.ep)
on CPU ranks over gloo: the count and row exchanges, the slot-to-expert
mapping of the received buckets and the return exchange, with the compute
steps done by the oracle.  Each rank's output must equal the single-process
oracle layer on that rank's tokens with all experts (the same fp64 sums), for
P = 2 and 4 ranks, with and without dropped tokens.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The layer's compute steps on the CPU oracle (test infrastructure).
    Activations travel as fp64 tensors holding exact bf16 values."""

    def __init__(self, oracle):
        self.o = oracle

    @staticmethod
    def _bits(t):
        v = t.to(torch.float32).to(torch.bfloat16)
        return v.view(torch.int16).numpy().view(np.uint16)

    def route(self, x, w_router, bias, k):
        lg = self.o.router_logits(self._bits(x), w_router.numpy(),
                                  None if bias is None else bias.numpy())
        idx, w = self.o.topk(lg.astype(np.float32), k)
        return torch.from_numpy(lg), torch.from_numpy(idx), torch.from_numpy(w)

    def capacity(self, T, E, k, cf):
        return self.o.capacity(T, E, k, cf)

    def permute_padded(self, x, topk_idx, E, cf):
        T = x.shape[0]
        k = topk_idx.shape[1]
        C = self.o.capacity(T, E, k, cf)
        counts, _, slot, _, _ = self.o.permute(topk_idx.numpy(), E, C)
        pad, _ = self.o.dispatch_padded(self._bits(x), topk_idx.numpy(), slot, E, C)
        x_pad = torch.from_numpy(self.o.bits_to_f64(pad))
        offsets = torch.arange(E + 1, dtype=torch.int32) * C
        return torch.from_numpy(counts), offsets, torch.from_numpy(slot), x_pad

    def mlp_buckets(self, x_rows, offsets, bucket_rows, w_gate, w_up, w_down):
        B = offsets.shape[0] - 1
        E_w = w_gate.shape[0]
        y = torch.zeros(x_rows.shape[0], w_down.shape[2], dtype=torch.float64)
        xb = self._bits(x_rows)
        for b in range(B):
            lo, n = int(offsets[b]), int(bucket_rows[b])
            if n == 0:
                continue
            e = b % E_w
            _, o = self.o.swiglu_rows(xb[lo:lo + n], self._bits(w_gate[e]), self._bits(w_up[e]),
                                      self._bits(w_down[e]))
            y[lo:lo + n] = torch.from_numpy(o)
        self.rows_max = float(y.abs().max()) if y.numel() else 0.0
        return y

    def combine(self, y_rows, x, topk_idx, topk_w, slot, offsets):
        return torch.from_numpy(self.o.combine(y_rows.numpy(), self._bits(x), topk_idx.numpy(),
                                               topk_w.numpy(), slot.numpy(), offsets.numpy()))

    def rows_to_bf16(self, y_rows):
        # each value rounded to bf16 by the oracle's rounding (ties to even)
        return torch.from_numpy(np.vectorize(self.o.round_bf16)(y_rows.numpy()))

    combine_bf16rows = combine


def _worker(rank, world, port, case, out, return_bf16=False):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    import oracle
    from mixture_experts_layer_36_b200 import ep, synth
    from mixture_experts_layer_36_b200.configs import MoEConfig
    T, d, E, k, f, cf, zipf_s = case
    cfg = MoEConfig("ep_case", T=T, d=d, E=E, k=k, f=f, cf=cf, seed=5, zipf_s=zipf_s)
    w = synth.make_weights(cfg, "cpu")                    # the same weights on every rank
    x = synth.make_tokens(cfg, "cpu", seed=100 + rank)    # each rank its own tokens
    layer = ep.ExpertParallelMoE(w["w_router"], w["bias"],
                                 ep.shard_experts(w["w_gate"], rank, world),
                                 ep.shard_experts(w["w_up"], rank, world),
                                 ep.shard_experts(w["w_down"], rank, world), k, cf,
                                 ops=OracleOps(oracle), return_bf16=return_bf16)
    y = layer(x).numpy()
    # the largest expert output any rank computed (a rank combines rows of all)
    rows_max = torch.tensor([layer.ops.rows_max], dtype=torch.float64)
    dist.all_reduce(rows_max, op=dist.ReduceOp.MAX)
    rows_max = float(rows_max.item())
    log = dict(layer.exchange_log)
    xb = OracleOps._bits(x)
    ops = OracleOps(oracle)
    bias = None if w["bias"] is None else w["bias"].numpy()
    lg32 = oracle.router_logits(xb, w["w_router"].numpy(), bias).astype(np.float32)
    ref = oracle.moe_forward(xb, w["w_router"].numpy(), bias, ops._bits(w["w_gate"]),
                             ops._bits(w["w_up"]), ops._bits(w["w_down"]), k, cf,
                             decision_logits=lg32)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, float(np.max(np.abs(y - ref["y"]))), float(np.max(np.abs(ref["y"]))),
             int(ref["n_dropped"]), log, oracle.capacity(T, E, k, cf), rows_max))


CASES = [
    # (T, d, E, k, f, cf, zipf_s)
    (24, 16, 8, 2, 32, 0.0, None),    # dropless
    (40, 16, 8, 3, 32, 0.75, None),   # with drops
    (48, 16, 8, 2, 32, 1.0, 1.2),     # Zipf-hot low experts (router bias), drops on rank 0's
]


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("case", CASES, ids=["dropless", "drops", "skewed"])
def test_expert_parallel_matches_single_process(world, case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=280) for _ in range(world)]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    dropped = 0
    T, d, E, k, f, cf, _ = case
    # dispatch volume per rank on the neelmishra page: T*k*d*2*(P-1)/P bytes
    page = T * k * d * 2 * (world - 1) / world
    for rank, err, scale, n_drop, log, C, _ in res:
        assert err <= 1e-12 * max(scale, 1.0), (rank, err)
        dropped += n_drop
        # the padded exchange moves E*C rows where the formula counts T*k:
        # the page's volume times E*C / (T*k); the rows come back in fp32
        assert log["dispatch"] == E * C * d * 2 * (world - 1) // world
        assert log["dispatch"] == pytest.approx(page * E * C / (T * k))
        assert log["combine"] == 2 * log["dispatch"]
        assert log["counts"] == E * 4 * (world - 1) // world
    if case[5] > 0:
        assert dropped > 0                    # the capacity limit was exercised


@pytest.mark.timeout(300)
@pytest.mark.parametrize("case", CASES[:2], ids=["dropless", "drops"])
def test_expert_parallel_bf16_return(case):
    """The return exchange in bf16: half the bytes of the fp32 return (the
    same as the dispatch), and the layer off the fp64 one by at most the
    rounding of each expert output (2^-9 of the largest, the gate weights
    summing to at most 1)."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q, True))
             for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=280) for _ in range(world)]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, err, scale, n_drop, log, C, rows_max in res:
        assert err <= 2.0 ** -9 * rows_max * (1 + 1e-9) + 1e-12 * max(scale, 1.0), (rank, err)
        assert "combine" not in log
        assert log["combine_bf16"] == log["dispatch"]


def test_layer_rejects_expert_counts_that_do_not_split():
    """Without a process group the layer is one rank holding all E experts;
    wrong local expert counts are refused before any compute."""
    from mixture_experts_layer_36_b200 import ep
    E, d, f = 8, 16, 32
    wr = torch.zeros(d, E)
    wg, wu, wd = torch.zeros(E, d, f), torch.zeros(E, d, f), torch.zeros(E, f, d)
    layer = ep.ExpertParallelMoE(wr, None, wg, wu, wd, 2, 1.0, ops=object())
    assert (layer.P, layer.rank, layer.E_loc) == (1, 0, E)
    with pytest.raises(ValueError):
        ep.ExpertParallelMoE(wr, None, wg[:4], wu[:4], wd[:4], 2, 1.0, ops=object())
    # shard_experts hands rank r experts r*E/P .. (r+1)*E/P - 1
    w = torch.arange(E).reshape(E, 1, 1).float()
    assert ep.shard_experts(w, 1, 4).flatten().tolist() == [2.0, 3.0]
