"""Benchmark of the MoE layer forward pass on B200: tokens/s of the whole layer,
with the dominant kernel's roofline fraction and the CPU oracle beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one pass of the whole layer (router + top-k, permute, grouped
gate/up GEMM with SwiGLU, grouped down GEMM, combine) over one batch of T
seeded synthetic tokens, inputs and weights resident in HBM.  Multi-GPU runs
(torchrun, one process per GPU) are independent replicas: every rank runs the
same layer on its own token batch; there is no data-path collective, only a
barrier around the timed region and a max-over-ranks of the device time.

Prints one JSON line on rank 0.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_layer_36_b200 import configs, synth  # noqa: E402

METRIC = "MoE layer tokens/s at 1 B200; grouped-GEMM % bf16 peak; permute/combine % HBM"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ROUTER_TILE_M = 128      # tokens per router GEMM row tile
# buffer rows per expert from which the GEMMs use CTA-pair tiles, and (bf16)
# CTA-pair tiles with the expert tails inside full tiles
PAIR_MIN_ROWS = 512
PAIR_TAIL_MIN_ROWS = 256
ROOFLINE_TIMING = ("mean launch duration over the timed steps: CUDA events recorded around "
                   "the launch on its stream")
FP8_OVER_BF16 = 2.0      # nominal dense e4m3 / bf16 tensor throughput (4.5 / 2.25 PFLOP/s)
PERMUTE_DIRECT_SUM = 4096   # chunk-histogram counters the scatter sums without a scan kernel


def launches_per_step(cfg, sms, fp8=False, padded=False, fused=False):
    """libmoe kernels one layer step launches: router weight split, router
    GEMM and top-k (the top-k runs in the GEMM's epilogue when the router's K
    is not split, i.e. when there are more 128-token row tiles than half the
    SMs); permutation rank and scatter, with a scan between them when there
    are more than PERMUTE_DIRECT_SUM chunk-histogram counters (chunks of 256
    tokens x E) (+ the padded layout's fill); the FP8 row quantizers on x and
    on h; the two expert GEMMs; the combine (the fused path's finalize)."""
    if cfg.T == 0:
        return 0
    m_tiles = -(-cfg.T // ROUTER_TILE_M)
    splits = max(1, min(min(sms, 256) // m_tiles, cfg.d // 64))
    n = 2 if splits == 1 else 3
    n += 2 + (1 if -(-cfg.T // 256) * cfg.E > PERMUTE_DIRECT_SUM else 0) + (1 if padded else 0)
    n += 2 if fp8 else 0
    return n + 2 + 1


def moe_max_rows_host(cfg):
    """min(T*k, E*C): the rows of the permuted buffers (decides the GEMM tiles)."""
    C = cfg.T if cfg.cf == 0 else math.ceil(((cfg.cf * cfg.k) * cfg.T) / cfg.E)
    return min(cfg.T * cfg.k, cfg.E * C)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            return json.load(fh), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def describe(cfg):
    cf = "dropless" if cfg.cf == 0 else f"cf={cfg.cf}"
    extra = f", zipf bias s={cfg.zipf_s}" if cfg.zipf_s else ""
    return (f"{cfg.name}: T={cfg.T} d={cfg.d} E={cfg.E} k={cfg.k} SwiGLU f={cfg.f} {cf}{extra}, "
            f"seed {cfg.seed}")


# ----------------------------------------------------------------- clocks sampling

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        props = torch.cuda.get_device_properties(device)
        uuid = str(getattr(props, "uuid", "") or "")
        self.gpu = ("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else (uuid or "0")
        self.proc = None

    def __enter__(self):
        import threading
        self.lines = []
        self.first = threading.Event()
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self

        def reader():
            for line in self.proc.stdout:
                self.lines.append(line)
                self.first.set()
        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()
        self.first.wait(timeout=10)      # sampling has started before timing begins
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)
        self.out = "".join(self.lines)
        return False

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r)
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": rows[0][1],
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------- replicas

def rank_token_seed(cfg, rank):
    """Each replica draws its own token batch; weights share the workload seed."""
    return cfg.seed * 1000 + rank


def max_over_ranks(value, device, dist):
    """The slowest rank's time (every rank takes the same collective step)."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if dist:
        import torch.distributed as td
        td.all_reduce(t, op=td.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- the GPU arm

class Layer:
    """Inputs, weights and buffers of one workload, resident on the device,
    and the step as C-ABI calls on one stream (five; seven with FP8 experts)."""

    def __init__(self, cfg, device, token_seed, fp8=False, padded=False, fused=False):
        import mixture_experts_layer_36_b200 as moe
        self.moe = moe
        self.cfg = cfg
        self.dev = device
        w = synth.make_weights(cfg, device)
        self.w = w
        self.fp8 = fp8
        if fp8:
            # one-time preprocessing, outside any timed region: e4m3 codes and
            # per-column scales of the expert weights
            self.q = {n: moe.moe_quantize_weights_fp8(w[n]) for n in ("w_gate", "w_up", "w_down")}
            torch.cuda.synchronize(device)
        self.x = synth.make_tokens(cfg, device, seed=token_seed)
        T, d, E, k, f = cfg.T, cfg.d, cfg.E, cfg.k, cfg.f
        self.padded = padded
        self.fused = fused
        # padded [E, C, d] layout: every bucket is C rows, all of them computed
        self.rows = moe.moe_padded_rows(T, E, k, cfg.cf) if padded else \
            moe.moe_max_rows(T, E, k, cfg.cf)
        z = lambda *s, dt: torch.empty(*s, dtype=dt, device=device)  # noqa: E731
        self.logits = z(T, E, dt=torch.float32)
        self.idx = z(T, k, dt=torch.int32)
        self.tw = z(T, k, dt=torch.float32)
        self.perm = {"counts": z(E, dt=torch.int32), "offsets": z(E + 1, dt=torch.int32),
                     "slot": z(T, k, dt=torch.int32), "row_src": z(self.rows, dt=torch.int32),
                     "n_dropped": z(1, dt=torch.int32)}
        if fp8:
            # the FP8 layer quantizes each token once and permutes codes + scales
            self.perm.update(xq=z(self.rows, d, dt=torch.uint8), sx=z(self.rows, dt=torch.float32))
            self.xq_tok, self.sx_tok = z(T, d, dt=torch.uint8), z(T, dt=torch.float32)
        elif padded:
            self.perm["x_pad"] = z(self.rows, d, dt=torch.bfloat16)
        elif fused:
            # no permuted copies: row_pair for the scatter, an fp32 token accumulator
            self.perm.update(row_pair=z(self.rows, dt=torch.int32),
                             y32=z(T, d, dt=torch.float32),
                             x_perm=z(self.rows, d, dt=torch.bfloat16))
        else:
            self.perm["x_perm"] = z(self.rows, d, dt=torch.bfloat16)
        self.pws = z(max(moe.moe_permute_workspace_size(T, E, k), 16), dt=torch.uint8)
        self.rws = z(max(moe.moe_route_workspace_size(T, d, E, k), 16), dt=torch.uint8)
        self.h = z(self.rows, f, dt=torch.bfloat16)
        self.y_perm = z(self.rows, d, dt=torch.float32)
        self.y = z(T, d, dt=torch.bfloat16)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        if fp8:
            self.hq, self.sh = z(self.rows, f, dt=torch.uint8), z(self.rows, dt=torch.float32)
            self.ws = z(moe.moe_workspace_size_fp8(T, d, E, k, f, cfg.cf), dt=torch.uint8)
        elif fused:
            self.ws = z(moe.moe_workspace_size_fused(T, d, E, k, f, cfg.cf), dt=torch.uint8)
        else:
            self.ws = z(moe.moe_workspace_size(T, d, E, k, f, cfg.cf), dt=torch.uint8)
        self.steps = self.stages()
        self.stage_names = [n for n, _ in self.steps]

    def stages(self):
        """The step as (name, call) pairs, in launch order."""
        m, w, c = self.moe, self.w, self.cfg
        p = self.perm
        st = [("route", lambda: m.moe_route(self.x, w["w_router"], w["bias"], c.k, self.logits,
                                            self.idx, self.tw, ws=self.rws,
                                            dev_status=self.status))]
        if self.fp8:
            q, n_rows = self.q, p["offsets"][c.E:]
            st += [("quant_x", lambda: m.moe_quantize_rows_fp8(self.x, q=self.xq_tok,
                                                               scale=self.sx_tok)),
                   ("permute", lambda: m.moe_permute_fp8(self.xq_tok, self.sx_tok, self.idx, c.E,
                                                         c.cf, out=p, ws=self.pws)),
                   ("gate_up", lambda: m.moe_expert_gate_up_fp8(
                       p["xq"], p["sx"], p["offsets"], *q["w_gate"], *q["w_up"], h=self.h,
                       dev_status=self.status)),
                   ("quant_h", lambda: m.moe_quantize_rows_fp8(self.h, n_rows=n_rows, q=self.hq,
                                                               scale=self.sh)),
                   ("down", lambda: m.moe_expert_down_fp8(self.hq, self.sh, p["offsets"],
                                                          *q["w_down"], y_perm=self.y_perm,
                                                          dev_status=self.status))]
        elif self.fused:
            st += [("permute", lambda: m.moe_permute_fused(self.x, self.idx, c.E, c.cf, out=p,
                                                           ws=self.pws)),
                   ("gate_up", lambda: m.moe_expert_gate_up(p["x_perm"], p["offsets"],
                                                            w["w_gate"], w["w_up"], h=self.h,
                                                            dev_status=self.status)),
                   ("down", lambda: m.moe_expert_down_scatter(
                       self.h, p["offsets"], w["w_down"], p["row_pair"], self.tw, p["y32"],
                       dev_status=self.status)),
                   ("combine", lambda: m.moe_combine_finalize(p["y32"], self.x, p["slot"],
                                                              y=self.y))]
            return st
        else:
            if self.padded:
                st.append(("permute", lambda: m.moe_permute_padded(self.x, self.idx, c.E, c.cf,
                                                                   out=p, ws=self.pws)))
            else:
                st.append(("permute", lambda: m.moe_permute(self.x, self.idx, c.E, c.cf, out=p,
                                                            ws=self.pws)))
            xin = p["x_pad"] if self.padded else p["x_perm"]
            st += [("gate_up", lambda: m.moe_expert_gate_up(xin, p["offsets"], w["w_gate"],
                                                            w["w_up"], h=self.h,
                                                            dev_status=self.status)),
                   ("down", lambda: m.moe_expert_down(self.h, p["offsets"], w["w_down"],
                                                      y_perm=self.y_perm,
                                                      dev_status=self.status))]
        st.append(("combine", lambda: m.moe_combine(self.y_perm, self.x, self.idx, self.tw,
                                                    p["slot"], p["offsets"], y=self.y)))
        return st

    def step(self, ev=None):
        """One layer pass; ev = events recorded around every stage."""
        for i, (_, call) in enumerate(self.steps):
            if ev:
                ev[i].record()
            call()
        if ev:
            ev[len(self.steps)].record()

    def layer_forward(self, x, y):
        w, c = self.w, self.cfg
        if self.padded:
            # no one-shot call for this layout: the stage entry points on x, y
            x0, y0 = self.x, self.y
            self.x, self.y = x, y
            for _, call in self.steps:
                call()
            self.x, self.y = x0, y0
            return
        if self.fused:
            self.moe.moe_layer_forward_fused(x, w["w_router"], w["bias"], w["w_gate"], w["w_up"],
                                             w["w_down"], c.k, c.cf, y=y, ws=self.ws)
            return
        if self.fp8:
            q = self.q
            self.moe.moe_layer_forward_fp8(x, w["w_router"], w["bias"], *q["w_gate"], *q["w_up"],
                                           *q["w_down"], c.k, c.cf, y=y, ws=self.ws)
            return
        self.moe.moe_layer_forward(x, w["w_router"], w["bias"], w["w_gate"], w["w_up"],
                                   w["w_down"], c.k, c.cf, y=y, ws=self.ws)


def gpu_arm(args, cfg, rank, world, local_rank, with_e2e=True):
    """Time K layer steps (CUDA events around every stage, max over ranks), and
    with_e2e the one-shot public call with host buffers in and out."""
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = world > 1
    if dist:
        import torch.distributed as td
    layer = Layer(cfg, dev, token_seed=rank_token_seed(cfg, rank), fp8=args.fp8,
                  padded=args.layout == "padded", fused=args.fused)
    stream = torch.cuda.current_stream()

    K = args.steps
    nst = len(layer.stage_names)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(K)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # the clock sampler starts before the warm-up so that it is running
    # (nvidia-smi takes a moment to start) when the timed region begins
    with ClockSampler(dev) as clk:
        for _ in range(args.warmup):
            layer.step()
        torch.cuda.synchronize()
        if dist:
            td.barrier()
        torch.cuda.synchronize()
        start.record(stream)
        for i in range(K):
            layer.step(evs[i])
        stop.record(stream)
        torch.cuda.synchronize()
    if dist:
        td.barrier()
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), dev, dist)

    names = layer.stage_names
    stage_ms = {n: statistics.median(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(K))
                for j, n in enumerate(names)}
    # the rooflines divide by a kernel's average duration over the timed steps
    stage_mean = {n: statistics.fmean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(K))
                  for j, n in enumerate(names)}
    status = int(layer.status.item())
    N = int(layer.perm["counts"].sum().item())          # kept pairs (either layout)
    active = int((layer.perm["counts"] > 0).sum().item())
    n_drop = int(layer.perm["n_dropped"].item())
    out = {"elapsed_ms": elapsed_ms, "stage_ms": stage_ms, "stage_mean": stage_mean,
           "status": status, "N": N, "active_experts": active, "n_dropped": n_drop,
           "clocks": clk.summary(), "layer": layer}
    if not with_e2e:
        return out

    # end to end through the one-shot public call, host buffers in and out:
    # every step copies its tokens host->device, runs moe_layer_forward and
    # copies the result device->host.  Copies run on their own streams and
    # overlap the previous / next step's compute (two device buffer sets).
    x_host = layer.x.cpu().pin_memory()
    y_host = torch.empty_like(x_host).pin_memory()
    x_dev = [torch.empty_like(layer.x) for _ in range(2)]
    y_dev = [torch.empty_like(layer.x) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[b])       # compute i-2 finished reading x_dev[b]
                x_dev[b].copy_(x_host, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])          # copy-out i-2 finished reading y_dev[b]
            layer.layer_forward(x_dev[b], y_dev[b])
            ev_done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[b])
                y_host.copy_(y_dev[b], non_blocking=True)
                ev_out[b].record(s_out)

    e2e_steps(max(2, args.warmup))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        td.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    s_in.wait_event(e0)
    e2e_steps(K)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize()
    out["e2e_ms"] = max_over_ranks(e0.elapsed_time(e1), dev, dist)
    out["h2d"] = x_host.numel() * 2
    out["d2h"] = y_host.numel() * 2
    return out


def traffic_from_profile(kernel_tag, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}.{workload}.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        prof = json.load(fh)
    src = os.path.join(ROOT, prof.get("source", ""))
    if not os.path.exists(src):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()
    return prof.get("dram_bytes_per_launch") if h == prof.get("source_sha256") else None


# ----------------------------------------------------------------- the CPU oracle

def oracle_sample(cfg, weights_host, x_host_bits, n_tokens):
    """Time the oracle (as it stands) on the first n_tokens tokens of the batch,
    whole layer (capacity recomputed for the sample size).  Returns seconds."""
    import oracle
    bias = None if weights_host["bias"] is None else weights_host["bias"]
    t0 = time.perf_counter()
    oracle.moe_forward(x_host_bits[:n_tokens], weights_host["w_router"], bias,
                       weights_host["w_gate"], weights_host["w_up"], weights_host["w_down"],
                       cfg.k, cfg.cf)
    return time.perf_counter() - t0, oracle.num_threads()


def host_weights(w):
    import oracle
    return {"w_router": w["w_router"].cpu().numpy(),
            "bias": None if w["bias"] is None else w["bias"].cpu().numpy(),
            "w_gate": oracle.bf16_bits(w["w_gate"]), "w_up": oracle.bf16_bits(w["w_up"]),
            "w_down": oracle.bf16_bits(w["w_down"])}


def calibrated_tokens(cfg, wh, xb, seconds):
    """Tokens whose oracle pass takes about `seconds` on this host: time a
    small pass, scale, re-time once if far off; clamp to [2, T]."""
    n = 8 if cfg.T >= 8 else cfg.T
    for _ in range(3):
        t, _ = oracle_sample(cfg, wh, xb, n)
        want = int(max(2, min(cfg.T, round(n * seconds / max(t, 1e-6)))))
        if t > 0.3 * seconds or want == n or n == cfg.T:
            return want
        n = min(want, max(n * 4, 2))
    return n


# the oracle runs the whole layer on these workloads when their pass is
# estimated under FULL_LAYER_MAX_S on the host; otherwise a token sample
# (extrapolated to the batch: the oracle's cost is linear in the tokens)
FULL_LAYER = ("tiny", "mixtral", "skewed", "decode")
FULL_LAYER_MAX_S = 90.0


def oracle_timing(cfg, layer, host_cache=None, sample_s=5.0):
    """The oracle's tokens/s on this workload: the whole batch where planned
    (and affordable), else a calibrated sample of about sample_s seconds.
    host_cache keeps the host copy of weights that several workloads share
    (the decode sweep draws the same weights at every T)."""
    import oracle
    key = (cfg.seed, cfg.E, cfg.d, cfg.f, cfg.zipf_s)
    if host_cache is not None and key in host_cache:
        wh = host_cache[key]
    else:
        wh = host_weights(layer.w)
        if host_cache is not None:
            host_cache.clear()
            host_cache[key] = wh
    xb = oracle.bf16_bits(layer.x)
    n = calibrated_tokens(cfg, wh, xb, sample_s)
    whole = cfg.name.split("@")[0] in FULL_LAYER
    if whole and n < cfg.T:
        est = sample_s * cfg.T / max(n, 1)
        whole = est <= FULL_LAYER_MAX_S
    if whole:
        secs, cores = oracle_sample(cfg, wh, xb, cfg.T)
        what = f"whole layer, all {cfg.T} tokens, {secs:.1f} s"
        n = cfg.T
    else:
        secs, cores = oracle_sample(cfg, wh, xb, n)
        what = (f"first {n} of {cfg.T} tokens through the whole layer, {secs:.1f} s "
                "(capacity recomputed for the sample; extrapolated: cost is linear in tokens)")
    return {"value": round(n / secs, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": what}


# ----------------------------------------------------------------- the JSON line

def path_name(args):
    return "fused (down GEMM + weighted scatter)" if args.fused else "staged"


def workload_config(cfg, args, world):
    """The `config` object of both arms' lines: a function of the workload and
    the command line only."""
    wb = 1 if args.fp8 else 2
    return {"workload": describe(cfg), "T": cfg.T, "d": cfg.d, "E": cfg.E, "k": cfg.k,
            "f": cfg.f, "cf": cfg.cf,
            "parallelism": f"replicas x{world} (token batches, no collective)",
            "layout": args.layout, "path": path_name(args),
            "experts": ("e4m3 weights (fp32 column scales) x e4m3 activations (fp32 row "
                        "scales)") if args.fp8 else "bf16",
            "l2": "inputs larger than L2 (expert weights "
                  f"{3 * cfg.E * cfg.d * cfg.f * wb / 1e9:.1f} GB); no flush"}


def summarize(cfg, args, r, pk, pk_kind, world):
    """Throughput, the dominant kernel's roofline and the per-stage rooflines
    of one timed run (r from gpu_arm)."""
    K = args.steps
    value = cfg.T * world * K / (r["elapsed_ms"] / 1e3)
    gemm1_flop = 4.0 * r["N"] * cfg.d * cfg.f
    gemm2_flop = 2.0 * r["N"] * cfg.d * cfg.f
    t_g1 = r["stage_mean"]["gate_up"] / 1e3
    t_g2 = r["stage_mean"]["down"] / 1e3
    # a kernel timed inside a long run under the power cap is compared with
    # the sustained peak, otherwise with the burst peak
    capped = "sw_power_cap" in (r["clocks"].get("reasons") or [])
    peak_tf = pk["bf16_tflops_sustained"] if capped else pk["bf16_tflops"]
    peak_src = f"{pk_kind} bf16 {'sustained (power cap active)' if capped else 'burst'}"
    burst_tf = pk["bf16_tflops"]
    if args.fp8:
        # e4m3 MMAs: the measured bf16 peak times the nominal fp8 / bf16 ratio (2)
        peak_tf *= FP8_OVER_BF16
        burst_tf *= FP8_OVER_BF16
        peak_src += f" x {FP8_OVER_BF16:g} (nominal e4m3 / bf16 dense ratio)"
    # the library's tile choice by buffer rows per expert: CTA pairs from
    # PAIR_MIN_ROWS, (bf16) CTA pairs with the expert tails from PAIR_TAIL_MIN_ROWS
    rows_per_expert = moe_max_rows_host(cfg) / cfg.E
    pair = rows_per_expert >= PAIR_MIN_ROWS
    pair_tail = not args.fp8 and not pair and rows_per_expert >= PAIR_TAIL_MIN_ROWS
    if args.fp8:
        kname = ("grouped_gemm_pair_kernel<true,true> (gate/up + SwiGLU, e4m3, CTA pairs)"
                 if pair else "grouped_gemm_e4m3_kernel<256,true> (gate/up + SwiGLU, e4m3)")
        ktag = "gemm_e4m3_pair_gate_up" if pair else "gemm_e4m3_gate_up"
    elif pair_tail:
        kname = ("grouped_gemm_pair_tail_kernel<true> (gate/up + SwiGLU, CTA pairs, expert tails "
                 "inside full tiles)")
        ktag = "gemm_pair_tail_gate_up"
    else:
        kname = ("grouped_gemm_pair_kernel<true> (gate/up + SwiGLU, CTA pairs)" if pair else
                 "grouped_gemm_kernel<256,true> (gate/up + SwiGLU)")
        ktag = "gemm_pair_gate_up" if pair else "gemm_gate_up"
    achieved = gemm1_flop / t_g1 / 1e12
    # bytes the gate/up GEMM must move: weights of the experts that got rows,
    # x_perm rows in, h rows out
    A = r["active_experts"]
    # operand bytes per element: bf16 2; e4m3 1 (plus 4-byte row / column scales)
    wb = 1 if args.fp8 else 2
    g1_bytes = A * 2.0 * cfg.d * cfg.f * wb + r["N"] * cfg.d * wb + r["N"] * cfg.f * 2
    g2_bytes = A * 1.0 * cfg.d * cfg.f * wb + r["N"] * cfg.f * wb + r["N"] * cfg.d * 4
    if args.fp8:
        g1_bytes += A * 2.0 * cfg.f * 4 + r["N"] * 4
        g2_bytes += A * 1.0 * cfg.d * 4 + r["N"] * 4
    ridge = peak_tf * 1e12 / (pk["hbm_gbs"] * 1e9)
    hbm_bound = gemm1_flop / g1_bytes < ridge
    bytes_perm = cfg.T * cfg.d * wb + r["N"] * cfg.d * wb
    bytes_comb = r["N"] * cfg.d * 4 + cfg.T * cfg.d * 2
    if args.fused:
        # the permutation also zeroes the fp32 accumulator; the finishing pass
        # reads it and writes y
        bytes_perm += cfg.T * cfg.d * 4
        bytes_comb = cfg.T * cfg.d * 4 + cfg.T * cfg.d * 2

    def hbm(nbytes, name):
        t = r["stage_mean"][name] / 1e3
        return {"bound": "hbm", "unit": "GB/s", "algorithmic_bytes": nbytes,
                "duration_ms": round(t * 1e3, 6), "achieved": float(f"{nbytes / t / 1e9:.6g}"),
                "peak": pk["hbm_gbs"], "frac": round(nbytes / t / 1e9 / pk["hbm_gbs"], 4)}

    quant_rooflines = {}
    if args.fp8:
        # the row quantizers: bf16 rows read once (the second pass hits cache),
        # codes + fp32 scales written
        for name, rows, width in (("quant_x", cfg.T, cfg.d), ("quant_h", r["N"], cfg.f)):
            quant_rooflines[name] = hbm(rows * width * 3 + rows * 4, name)
    if not hbm_bound:
        roofline = {"kernel": kname, "bound": "tensor", "achieved": round(achieved, 1),
                    "peak": peak_tf, "unit": "TFLOP/s", "frac": round(achieved / peak_tf, 4),
                    "peak_source": peak_src,
                    "frac_of_burst_peak": round(achieved / burst_tf, 4),
                    "algorithmic_flop": gemm1_flop, "duration_ms": round(t_g1 * 1e3, 4),
                    "timing": ROOFLINE_TIMING, "traffic": traffic_from_profile(ktag, cfg.name)}
    else:
        roofline = {"kernel": kname, "bound": "hbm", "achieved": round(g1_bytes / t_g1 / 1e9, 1),
                    "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": round(g1_bytes / t_g1 / 1e9 / pk["hbm_gbs"], 4),
                    "peak_source": f"{pk_kind} HBM copy", "algorithmic_bytes": g1_bytes,
                    "active_experts": A, "duration_ms": round(t_g1 * 1e3, 4),
                    "timing": ROOFLINE_TIMING, "traffic": traffic_from_profile(ktag, cfg.name)}
    return {
        "value": round(value, 1),
        "ms_per_step": round(r["elapsed_ms"] / K, 4),
        "roofline": roofline,
        "stages_ms": {k_: round(v, 4) for k_, v in r["stage_ms"].items()},     # medians
        "stages_mean_ms": {k_: round(v, 4) for k_, v in r["stage_mean"].items()},
        "stage_rooflines": {
            "gate_up_gemm": {"bound": "tensor", "achieved": round(achieved, 1), "unit": "TFLOP/s",
                             "peak": peak_tf, "frac": round(achieved / peak_tf, 4),
                             "frac_of_burst_peak": round(achieved / burst_tf, 4),
                             "hbm_GBps": round(g1_bytes / t_g1 / 1e9, 1),
                             "hbm_frac": round(g1_bytes / t_g1 / 1e9 / pk["hbm_gbs"], 4),
                             "active_experts": A},
            "down_gemm": {"bound": "tensor", "achieved": round(gemm2_flop / t_g2 / 1e12, 1),
                          "unit": "TFLOP/s", "peak": peak_tf,
                          "frac": round(gemm2_flop / t_g2 / 1e12 / peak_tf, 4),
                          "frac_of_burst_peak": round(gemm2_flop / t_g2 / 1e12 / burst_tf, 4),
                          "hbm_GBps": round(g2_bytes / t_g2 / 1e9, 1),
                          "hbm_frac": round(g2_bytes / t_g2 / 1e9 / pk["hbm_gbs"], 4)},
            "permute": hbm(bytes_perm, "permute"),
            "combine": hbm(bytes_comb, "combine"),
            **quant_rooflines,
        },
        "routing": {"kept_pairs": r["N"], "dropped_pairs": r["n_dropped"], "active_experts": A,
                    "gemm_rows_computed": (r["layer"].rows if args.layout == "padded"
                                           else r["N"])},
        "device_status": r["status"],
        "clocks": {k_: r["clocks"][k_] for k_ in ("sm_mhz", "sm_max_mhz", "reasons")},
    }


# the other workloads measured beside the headline one (per_config)
PER_CONFIG = ("tiny", "mixtral", "fine_grained", "skewed", "decode@T16", "decode@T64",
              "decode@T256")


# ----------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="mixtral")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the named workload (by default every other workload is "
                         "also timed, with the oracle beside it, into per_config)")
    ap.add_argument("--layout", choices=["ragged", "padded"], default="ragged",
                    help="padded: the static [E, C, d] expert buffers (every bucket C rows, all "
                         "computed) in place of the ragged buckets")
    ap.add_argument("--fused", action="store_true",
                    help="the fused path: the down GEMM adds gate-weighted rows into an fp32 "
                         "token accumulator (no y_perm, no separate combine)")
    ap.add_argument("--fp8", action="store_true",
                    help="expert weights as e4m3 codes + fp32 column scales (quantized once "
                         "before timing); activations and accumulation as in the bf16 path")
    ap.add_argument("--profile", action="store_true",
                    help="run W + K layer steps only (no timing, e2e or oracle): a short, "
                         "fixed launch sequence for ncu")
    args = ap.parse_args()
    if args.fused and (args.fp8 or args.layout != "ragged"):
        ap.error("--fused runs the bf16 experts on ragged buckets")
    if args.fp8 and args.layout != "ragged":
        ap.error("--fp8 runs on ragged buckets")
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    cfg = configs.by_name(args.config)

    if args.impl == "reference":
        return reference_arm(args, cfg, rank, world)
    if args.profile:
        layer = Layer(cfg, torch.device("cuda", local_rank), token_seed=rank_token_seed(cfg, 0),
                      fp8=args.fp8, padded=args.layout == "padded", fused=args.fused)
        for _ in range(args.warmup + args.steps):
            layer.step()
        torch.cuda.synchronize()
        assert int(layer.status.item()) == 0
        sms = torch.cuda.get_device_properties(local_rank).multi_processor_count
        kps = launches_per_step(cfg, sms, args.fp8, args.layout == "padded", args.fused)
        print(json.dumps({"profile_run": cfg.name, "launches": kps * (args.warmup + args.steps)}))
        return

    if world > 1:
        import datetime
        import torch.distributed as td
        if not td.is_initialized():        # (a caller may have set up the group already)
            torch.cuda.set_device(local_rank)
            td.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                  device_id=torch.device("cuda", local_rank))
    r = gpu_arm(args, cfg, rank, world, local_rank)
    pk, pk_kind = peaks()
    K = args.steps
    summ = summarize(cfg, args, r, pk, pk_kind, world)
    oracle_here = rank == 0 and world == 1 and not args.no_cpu_baseline
    out = {
        "metric": METRIC,
        "value": summ["value"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": summ["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3 (expert GEMM operands; fp32 accumulation)" if args.fp8 else "bf16",
        "data": "synthetic (seeded; random-init weights of the named shape)",
        "config": workload_config(cfg, args, world),
        **{k_: summ[k_] for k_ in ("roofline", "stages_ms", "stages_mean_ms", "stage_rooflines",
                                   "routing", "device_status", "clocks")},
        "e2e": {"value": round(cfg.T * world * K / (r["e2e_ms"] / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "api": ("the stage entry points (moe_route, moe_permute_padded, "
                        "moe_expert_gate_up, moe_expert_down, moe_combine)"
                        if args.layout == "padded" else
                        ("moe_layer_forward_fused" if args.fused else
                         "moe_layer_forward_fp8" if args.fp8 else "moe_layer_forward") +
                        " (one-shot C-ABI call)") +
                       "; every step copies x from pinned host memory and y back, on copy "
                       "streams overlapping adjacent steps' compute"},
        "gpu_launches": launches_per_step(
            cfg, torch.cuda.get_device_properties(local_rank).multi_processor_count, args.fp8,
            args.layout == "padded", args.fused) * K,
    }
    if oracle_here:
        wh = host_weights(r["layer"].w)
        import oracle
        xb = oracle.bf16_bits(r["layer"].x)
        n = calibrated_tokens(cfg, wh, xb, seconds=15.0)
        secs, cores = oracle_sample(cfg, wh, xb, n)
        out["cpu_baseline"] = {"value": round(n / secs, 3), "unit": "tokens/s", "cores": cores,
                               "kind": "oracle",
                               "sample": f"first {n} tokens of the batch through the whole "
                                         f"layer (fp64 C oracle, OpenMP), {secs:.1f} s"}
    if not args.no_per_config:
        # every other workload, same path and step count: throughput, the
        # dominant kernel's roofline, the permute / combine HBM fractions, and
        # the oracle on the host beside it
        per = {}
        names = [cfg.name] + [n for n in PER_CONFIG if configs.by_name(n).name != cfg.name]
        host_cache = {}
        for name in names:
            c = configs.by_name(name)
            if c.name == cfg.name:
                rc, sc = r, summ
            else:
                torch.cuda.empty_cache()
                rc = gpu_arm(args, c, rank, world, local_rank, with_e2e=False)
                sc = summarize(c, args, rc, pk, pk_kind, world)
            entry = {"workload": describe(c), "tokens_per_s": sc["value"],
                     "ms_per_step": sc["ms_per_step"], "steps": K,
                     **{k_: sc[k_] for k_ in ("roofline", "stage_rooflines", "stages_mean_ms",
                                              "routing", "device_status", "clocks")}}
            if oracle_here:
                entry["oracle"] = oracle_timing(c, rc["layer"], host_cache)
            per[c.name] = entry
            rc.pop("layer", None)        # frees this workload's buffers before the next
        out["per_config"] = per
    if world > 1:
        import torch.distributed as td
        td.barrier()
        td.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def reference_arm(args, cfg, rank, world):
    """The oracle timed as it stands on the host cores (rank 0 only)."""
    if rank != 0:
        return
    import oracle
    # weights drawn on the CPU with the same recipe (one step is a bounded sample)
    w = synth.make_weights(cfg, "cpu")
    x = synth.make_tokens(cfg, "cpu")
    wh = host_weights(w)
    xb = oracle.bf16_bits(x)
    # each step is a sample sized so that warm-up + steps take about 90 s
    per_step = min(2.0, 90.0 / (args.steps + 1))
    n = calibrated_tokens(cfg, wh, xb, per_step)
    oracle_sample(cfg, wh, xb, n)     # one untimed warm-up pass
    t = 0.0
    for _ in range(args.steps):
        s, cores = oracle_sample(cfg, wh, xb, n)
        t += s
    value = n * args.steps / t
    out = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t / args.steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; random-init weights of the named shape)",
        "config": workload_config(cfg, args, world),
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"each step: first {n} tokens of the batch through the whole "
                                   f"layer (fp64 C oracle, OpenMP)"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
