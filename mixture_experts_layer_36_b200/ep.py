"""Expert-parallel MoE layer forward across the ranks of a torch.distributed
group (one process per GPU; NCCL over NVLink / NVSwitch on B200).

The experts are spread over the P ranks, E/P consecutive experts each, and
every rank keeps its own batch of tokens.  One layer pass on rank p:

  1. route its tokens (moe_route);
  2. permute them into the fixed-size expert buffers [E, C, d]
     (moe_permute_padded): rank q's experts occupy one contiguous slot of
     E/P * C rows, so every rank sends every other rank the same number of
     rows and no host-side split sizes are needed;
  3. exchange the per-expert kept counts and the row slots (all-to-all);
  4. run the grouped SwiGLU MLP over the P * E/P received slots, slot
     b = q * E/P + e through local expert e, only its received count of rows
     (moe_expert_mlp_buckets);
  5. send the output rows back (all-to-all) to their source slots;
  6. combine locally (moe_combine on the padded offsets e * C).

This follows the dispatch / expert compute / combine pipeline of "Expert
Parallelism & All-to-All" (neelmishra.github.io, sections "All-to-all: the
distributed transpose" and "Why fixed-size buffers matter here": static
shapes, padded rows) and of the "Expert Parallelism" guide (infra.bea.ai,
section 2, "The Dispatch Pattern").  Capacity is applied per source rank to
its own tokens (each rank's buffers hold C = ceil(cf*k*T/E) rows per expert),
so with P = 1 the layer is exactly the single-GPU layer; all ranks must hold
the same number of tokens T (equal slot sizes).

The exchange itself is NCCL's all-to-all through torch.distributed; the
compute steps go through an ``ops`` object (``CudaOps``: the library's C-ABI
calls), which keeps the exchange logic testable with CPU ranks.

Exchange volume.  The neelmishra page's dispatch volume per rank is
T*k*d*2*(P-1)/P bytes (bf16 rows, the share of each rank's rows that leaves
it).  The padded exchange here sends E*C rows per rank instead of T*k, a
factor E*C/(T*k) (about cf, or E/k when dropless, C = T).  The rows come
back as fp32 by default (the expert outputs are rounded to bf16 only once,
in the combine), twice the bytes of the dispatch; with ``return_bf16`` they
are rounded to bf16 before the return exchange (moe_rows_to_bf16) and
combined from bf16 (moe_combine_bf16rows): the same bytes as the dispatch,
for one more rounding of each expert output (at most 2^-9 of its magnitude
per term of the weighted sum).  ``exchange_log`` records, per exchange of the
last forward, the bytes this rank sent to other ranks.
"""
import torch
import torch.distributed as dist


class CudaOps:
    """The layer's compute steps as libmoe calls (on the current CUDA stream)."""

    def __init__(self):
        from . import binding
        self.b = binding

    def route(self, x, w_router, bias, k):
        return self.b.moe_route(x, w_router, bias, k)

    def capacity(self, T, E, k, cf):
        return self.b.moe_capacity(T, E, k, cf)

    def permute_padded(self, x, topk_idx, E, cf):
        p = self.b.moe_permute_padded(x, topk_idx, E, cf)
        return p["counts"], p["offsets"], p["slot"], p["x_pad"]

    def mlp_buckets(self, x_rows, offsets, bucket_rows, w_gate, w_up, w_down):
        _, y_rows = self.b.moe_expert_mlp_buckets(x_rows, offsets, bucket_rows, w_gate, w_up,
                                                  w_down)
        return y_rows

    def combine(self, y_rows, x, topk_idx, topk_w, slot, offsets):
        return self.b.moe_combine(y_rows, x, topk_idx, topk_w, slot, offsets)

    def rows_to_bf16(self, y_rows):
        return self.b.moe_rows_to_bf16(y_rows)

    def combine_bf16rows(self, y_rows, x, topk_idx, topk_w, slot, offsets):
        return self.b.moe_combine_bf16rows(y_rows, x, topk_idx, topk_w, slot, offsets)


class ExpertParallelMoE:
    """One rank's part of an expert-parallel MoE layer.

    w_router f32 [d, E] and bias f32 [E] (or None) are replicated; w_gate /
    w_up [E/P, d, f] and w_down [E/P, f, d] are this rank's experts
    rank*E/P .. (rank+1)*E/P - 1.  return_bf16: send the expert outputs back
    in bf16 (half the return bytes) instead of fp32.
    """

    def __init__(self, w_router, bias, w_gate, w_up, w_down, k, cf, group=None, ops=None,
                 return_bf16=False):
        self.group = group
        self.P = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.E = w_router.shape[1]
        if self.E % self.P != 0:
            raise ValueError(f"{self.E} experts do not split over {self.P} ranks")
        self.E_loc = self.E // self.P
        if w_gate.shape[0] != self.E_loc:
            raise ValueError(f"expected {self.E_loc} local experts, got {w_gate.shape[0]}")
        self.w_router, self.bias = w_router, bias
        self.w_gate, self.w_up, self.w_down = w_gate, w_up, w_down
        self.k, self.cf = k, cf
        self.ops = ops if ops is not None else CudaOps()
        self.return_bf16 = return_bf16
        self.exchange_log = []

    # bytes per element on the wire: int32 counts, bf16 rows out, fp32 (or
    # bf16) rows back
    WIRE_BYTES = {"counts": 4, "dispatch": 2, "combine": 4, "combine_bf16": 2}

    def _all_to_all(self, out, inp, name):
        # each rank keeps 1/P of its buffer (its own slot) and sends the rest
        if inp.is_cuda and inp.element_size() != self.WIRE_BYTES[name]:
            raise TypeError(f"{name}: {inp.dtype} on the wire")
        nbytes = inp.numel() * self.WIRE_BYTES[name]
        self.exchange_log.append((name, nbytes * (self.P - 1) // self.P))
        if self.P == 1:
            out.copy_(inp)
        else:
            dist.all_to_all_single(out, inp, group=self.group)
        return out

    def forward(self, x):
        """y for this rank's tokens x [T, d] (bf16); T equal on every rank."""
        T, d = x.shape
        E, k, cf = self.E, self.k, self.cf
        C = self.ops.capacity(T, E, k, cf)
        logits, topk_idx, topk_w = self.ops.route(x, self.w_router, self.bias, k)
        counts, offsets, slot, x_pad = self.ops.permute_padded(x, topk_idx, E, cf)
        self.exchange_log = []
        # rank q receives counts[q*E_loc : (q+1)*E_loc] from every rank: bucket
        # b = source * E_loc + local expert
        recv_counts = self._all_to_all(torch.empty_like(counts), counts, "counts")
        x_recv = self._all_to_all(torch.empty_like(x_pad), x_pad, "dispatch")
        B = self.P * self.E_loc
        recv_offsets = torch.arange(B + 1, dtype=torch.int32, device=x.device) * C
        y_recv = self.ops.mlp_buckets(x_recv, recv_offsets, recv_counts, self.w_gate, self.w_up,
                                      self.w_down)
        if self.return_bf16:
            y_send = self.ops.rows_to_bf16(y_recv)
            y_pad = self._all_to_all(torch.empty_like(y_send), y_send, "combine_bf16")
            return self.ops.combine_bf16rows(y_pad, x, topk_idx, topk_w, slot, offsets)
        y_pad = self._all_to_all(torch.empty_like(y_recv), y_recv, "combine")
        return self.ops.combine(y_pad, x, topk_idx, topk_w, slot, offsets)

    __call__ = forward


def shard_experts(w, rank, world):
    """This rank's experts of a full [E, ...] expert weight tensor."""
    E = w.shape[0]
    n = E // world
    return w[rank * n:(rank + 1) * n].contiguous()
