#!/usr/bin/env python
"""Benchmark of the B200 MoE layer: tokens/s of the whole layer step and
TFLOP/s of the grouped expert GEMMs, as a fraction of the measured peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

A step is one pass of the whole layer over one batch of seeded synthetic
tokens: router -> permute -> grouped SwiGLU MLP -> combine (a forward pass,
plus the grouped-MLP backward for workloads that train). It is one call of
moe_layer_forward (and moe_grouped_mlp_backward) through the C ABI. Inputs
are already resident in HBM when the timed region starts. The weights exceed
L2 (126 MB), which keeps the steps L2-cold without a flush. Rank 0 prints one
JSON line.

The default workload is the largest single-GPU one, the Llama-4-17Bx16E-shaped
forward with its shared expert. On one GPU the line also carries the other
workloads under "workloads": the Mixtral-8x7B-shaped forward, the
Qwen3-30B-A3B-shaped forward + backward, the skewed sweep at T = 1, 8, 64
and 16384, and the 64-token tie case, whose near-tied logits spread the
batch over most experts (each batch of at most 64 tokens timed with L2
flushed before every step, since their weights can fit in L2).

With N > 1 (torchrun), each rank runs its own replica of the layer on its own
tokens (data-parallel replicas; the forward has no exchange step). value =
tokens of all ranks / the slowest rank's time. --impl reference times the CPU
oracle (the plain restatement the tests compare against) on the host cores of
rank 0, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s and grouped-GEMM TFLOP/s (% of B200 bf16 peak), 1 GPU"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "llama4_17bx16e"
NOMINAL_BF16_TFLOPS = 2250.0   # dense bf16 tensor peak of one B200 (vendor figure, no sparsity)
EXTRA_WORKLOADS = ["mixtral_8x7b", "qwen3_30b_a3b", "skew_t1", "skew_t8", "skew_t64", "skew_t16384", "tie_t64"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--T", type=int, default=None,
                    help="override the token count (small cases for profiling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay timing")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only --workload (not the other workloads of the \"workloads\" key)")
    ap.add_argument("--router-sweep", action="store_true",
                    help="also time the router alone at E=128, k=8, T = 2^16 .. 2^20")
    ap.add_argument("--router-calls", type=int, default=None, metavar="LOGT",
                    help="only call the router three times at T = 2^LOGT, E=128, k=8 on N(0,1) logits "
                         "(a small program for ncu captures of the router), then exit")
    ap.add_argument("--scaled-compare", action="store_true",
                    help="also time the Qwen3-30B-A3B fwd+bwd with the routing weights applied "
                         "before FC2 (ScaledSwiGLU) on a padded dispatch, beside the default layer")
    ap.add_argument("--gather-compare", action="store_true",
                    help="also time the Qwen3-30B-A3B-shaped forward (no saved state) through x_perm and "
                         "with the gate_up GEMM gathering its rows from x")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.15)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [r.strip().split(",") for r in self.tmp.read().splitlines() if r.strip()]
        os.unlink(self.tmp.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ dist
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=120)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            # a host without GPUs (the reference arm, the multi-rank tests): gloo
            dist.init_process_group("gloo", timeout=timeout)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(tokens_per_rank: int, world: int, steps: int, ms_max: float) -> float:
    """Tokens per second of the whole job: every rank's tokens over the slowest
    rank's time (weak scaling: each rank runs the same per-rank workload)."""
    return tokens_per_rank * world * steps / (ms_max / 1e3)


# ------------------------------------------------------------------ CPU baseline
class OracleRunner:
    """The oracle's per-token layer (and, for training workloads, its
    backward for dx and the routing-weight gradient) on host copies of the
    workload's inputs."""

    def __init__(self, w, inputs_cpu, threads):
        import oracle
        bits = oracle.bf16_bits
        self.w, self.threads, self.oracle = w, threads, oracle
        self.x = bits(inputs_cpu["x"])
        self.logits = inputs_cpu["logits"].numpy()
        self.wgu = bits(inputs_cpu["w_gate_up"])
        self.wd = bits(inputs_cpu["w_down"])
        sg, sd = inputs_cpu["shared_gate_up"], inputs_cpu["shared_down"]
        self.sgu = None if sg is None else bits(sg[0])
        self.sd = None if sd is None else bits(sd[0])
        self.dout = bits(inputs_cpu["dout"]) if "dout" in inputs_cpu else None

    def run(self, tokens):
        w, o = self.w, self.oracle
        o.moe_forward_tokens(self.x, self.logits, self.wgu, self.wd, w.k, tokens=tokens,
                             score=w.score, renormalize=w.renormalize, shared_gu_bits=self.sgu,
                             shared_d_bits=self.sd, threads=self.threads)
        if self.dout is not None:
            r = o.router_topk(self.logits[tokens], w.k, w.score, w.renormalize, with_map=False)
            o.moe_backward(self.x[tokens], r["topk_idx"], r["topk_prob"], self.wgu, self.wd,
                           self.dout[tokens], want=("dx", "dprob"))

    def sample_for(self, budget_s):
        """Tokens (spread over the batch) that take about budget_s seconds."""
        import numpy as np
        n = max(1, self.threads)
        t0 = time.perf_counter()
        self.run(np.arange(n))
        dt = time.perf_counter() - t0
        n2 = int(max(n, min(self.w.T, n * budget_s / max(dt, 1e-6))))
        n2 = max(n, (n2 // n) * n)
        return np.linspace(0, self.w.T - 1, n2).astype(np.int64)

    def time(self, tokens):
        t0 = time.perf_counter()
        self.run(tokens)
        return time.perf_counter() - t0


def cpu_inputs(w, d):
    """Host copies of the device inputs (the oracle reads exactly these bytes)."""
    return {k: (None if v is None else v.detach().to("cpu")) for k, v in d.items()}


def reference_arm(args, world, rank):
    if rank != 0:
        return 0
    import torch

    import workloads as wl
    w = workload(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    d = wl.make_inputs(w, dev)
    threads = os.cpu_count() or 1
    runner = OracleRunner(w, cpu_inputs(w, d), threads)
    tokens = runner.sample_for(0.5)
    for _ in range(args.warmup):
        runner.time(tokens)
    elapsed = sum(runner.time(tokens) for _ in range(args.steps))
    value = len(tokens) * args.steps / elapsed
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * elapsed / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(w, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{len(tokens)} of {w.T} tokens of the workload per step "
                                   f"(plain C oracle, fp64 accumulation, {threads} host threads)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def workload(args):
    import workloads as wl
    w = wl.WORKLOADS[args.workload]
    return w.scaled(T=args.T) if args.T else w


def config_dict(w, args):
    return {"workload": w.name, "T": w.T, "H": w.H, "I": w.I, "E": w.E, "top_k": w.k,
            "score": "sigmoid" if w.score == 1 else "softmax",
            "shared_expert": w.shared_expert, "pass": "fwd+bwd" if w.backward else "fwd",
            "global_batch_tokens": w.T * max(1, args.gpus),
            "l2": "inputs larger than L2 (weights exceed 126 MB); no flush",
            "parallelism": f"replicas x{args.gpus}" if args.gpus > 1 else "single GPU"}


def source_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_for(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if the
    kernel's source has not changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    e = t.get(kernel)
    if not e:
        return None
    src = os.path.join(ROOT, e["source"])
    if not os.path.exists(src) or source_sha(src) != e.get("source_sha"):
        return None
    return e.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ our arm
FWD_STAGES = ["router", "permute", "gate_up_swiglu", "down", "shared_expert", "combine"]
BWD_STAGES = ["combine_bwd", "down_dgrad_swiglu_bwd", "gate_up_dgrad", "dx_token_sum", "down_wgrad",
              "gate_up_wgrad"]
GEMM_STAGES = ["fwd_gate_up_swiglu", "fwd_down", "fwd_shared_expert", "bwd_down_dgrad_swiglu_bwd",
               "bwd_gate_up_dgrad", "bwd_down_wgrad", "bwd_gate_up_wgrad"]


def bandwidth_bytes(w):
    """Algorithmic bytes of the bandwidth-bound stages: what each must read
    and write once (bf16 rows 2 B per element, indices and weights 4 B)."""
    T, H, k, E, A = w.T, w.H, w.k, w.E, w.A
    b = {"fwd_router": T * E * 4 + T * k * 8 + E * 8,
         "fwd_permute": T * H * 2 + A * H * 2 + A * 4 + T * k * 4,
         "fwd_combine": A * H * 2 + T * H * 2 + T * k * 8 + (T * H * 2 if w.shared_expert else 0)}
    if w.backward:
        b["bwd_combine_bwd"] = T * H * 2 + 2 * A * H * 2 + T * k * 12
        b["bwd_dx_token_sum"] = A * H * 2 + T * H * 2 + T * k * 4
    return b


class Layer:
    """One workload's inputs, workspace and outputs on the device, and its
    step (the fused forward, plus the grouped-MLP backward when it trains)."""

    def __init__(self, m, w, d):
        import torch
        self.m, self.w, self.d = m, w, d
        self.opts = m.RouterOpts(w.score, w.renormalize)
        self.ws = m.LayerWorkspace(w.T, w.H, w.I, w.E, w.k, w.shared_expert, backward=w.backward)
        self.out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device="cuda")
        # the routing and saved state are kept so the combine can be timed alone
        _, self.state = m.moe_layer_forward(d["logits"], d["x"], d["w_gate_up"], d["w_down"], w.k, self.opts,
                                            d["shared_gate_up"], d["shared_down"], save_for_backward=True,
                                            workspace=self.ws, out=self.out)
        self.grads = None
        if w.backward:
            self.grads = m.moe_grouped_mlp_backward(d["dout"], self.state, d["w_gate_up"], d["w_down"], self.ws)
        if not w.backward:   # the forward-only step saves nothing beyond the routing
            self.state = {k_: self.state[k_] for k_ in ("topk_idx", "topk_prob", "counts", "offsets", "row_of",
                                                        "y_perm")}
            self.fwd_state = None
        else:
            self.fwd_state = self.state

    def step(self, fev=None, bev=None):
        m, w, d = self.m, self.w, self.d
        if fev:
            m.moe_trace_set(fev)
        m.moe_layer_forward(d["logits"], d["x"], d["w_gate_up"], d["w_down"], w.k, self.opts,
                            d["shared_gate_up"], d["shared_down"], save_for_backward=w.backward,
                            workspace=self.ws, out=self.out, state=self.fwd_state)
        if w.backward:
            if bev:
                m.moe_trace_set(bev)
            m.moe_grouped_mlp_backward(d["dout"], self.state, d["w_gate_up"], d["w_down"], self.ws, self.grads)
        if fev or bev:
            m.moe_trace_set(None)

    def launches(self):
        # router, scan (done by the router itself for one token block, T <= 8),
        # permute (also done by the router there for at most 64 KB of rows), gate_up, down (one launch with gate_up when every expert has
        # at most T <= 64 rows on swap-AB tiles and the experts that can hold
        # rows have at least one gate_up tile per SM), combine; the shared expert's
        # two GEMMs (the combine then folded into the second, above 16 tokens);
        # the backward's six
        import torch
        w = self.w
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        fused_mlp = (w.T <= 64 and w.T * w.k <= 16 * w.E and w.E <= 256
                     and min(w.E, w.T * w.k) * -(-w.I // 64) >= sms)
        # the router's one token block (T <= 8) also permutes up to 64 KB of rows
        router_permutes = w.T <= 8 and w.T * w.k * w.H * 2 <= 65536
        return (6 - (1 if w.T <= 8 else 0) - (1 if router_permutes else 0) - (1 if fused_mlp else 0)
                + (2 if w.shared_expert else 0) - (1 if combine_folded(w) else 0) + (6 if w.backward else 0))


def _events(n):
    import torch
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in evs:
        e.record()           # materialise the events before handing them to the library
    return evs


def stage_medians(layer, fevs, bevs):
    """Per-stage device time (ms), the median over the traced steps."""
    st = {}
    for i, n in enumerate(FWD_STAGES):
        st[f"fwd_{n}"] = statistics.median(evs[i].elapsed_time(evs[i + 1]) for evs in fevs)
    if layer.w.backward:
        for i, n in enumerate(BWD_STAGES):
            st[f"bwd_{n}"] = statistics.median(evs[i].elapsed_time(evs[i + 1]) for evs in bevs)
    return st


def gemm_summary(w, stages, peaks):
    """Grouped-GEMM TFLOP/s over the GEMM stages' device time, against the
    burst and sustained measured peaks and the nominal dense bf16 peak."""
    ms = sum(stages.get(k_, 0.0) for k_ in GEMM_STAGES if k_ != "fwd_shared_expert" or w.shared_expert)
    flop = w.fwd_flops() + (w.bwd_flops() if w.backward else 0.0)
    tf = flop / (ms / 1e3) / 1e12
    return {"tflops": tf, "flop_per_step": flop, "gemm_ms": ms,
            "frac_of_burst_peak": tf / peaks["bf16_tflops"],
            "frac_of_sustained_peak": tf / peaks["bf16_tflops_sustained"],
            "frac_of_nominal_peak": tf / NOMINAL_BF16_TFLOPS,
            "note": "expert GEMM FLOPs (6AHI fwd incl. shared expert, 12AHI bwd) / device time of the GEMM stages"}


def combine_folded(w):
    """Whether moe_layer_forward runs the combine in the shared expert's down
    GEMM epilogue (a shared expert on CTA-pair tiles: more than 16 tokens),
    so that the step has no combine kernel (its traced combine stage is empty)."""
    return w.shared_expert and w.T > 16


def warm_bandwidth(w, stages, hbm):
    out = {}
    for key, nbytes in bandwidth_bytes(w).items():
        if key == "fwd_combine" and combine_folded(w):
            out[key] = {"bytes": nbytes, "warm_us": None, "warm_frac_of_hbm": None,
                        "in_step": "folded into the shared expert's down GEMM epilogue; the cold figures "
                                   "time the combine kernel alone on the step's stored rows"}
            continue
        gbs = nbytes / (stages[key] / 1e3) / 1e9
        out[key] = {"bytes": nbytes, "warm_us": stages[key] * 1e3, "warm_frac_of_hbm": gbs / hbm}
    return out


def cold_bandwidth(layer, hbm, flush, reps=50, warm=10):
    """The bandwidth-bound stages with L2 flushed (a 256 MB read) before each
    timed call; median of `reps` after `warm`. The fused forward's router and
    permute run first after the flush; the combine (and the backward's dx
    token sum, the same kernel without weights) is timed as its own call on
    the step's saved rows; the backward's combine-bwd runs first in its call."""
    import torch
    m, w, d, st = layer.m, layer.w, layer.d, layer.state
    res = {"fwd_router": [], "fwd_permute": [], "fwd_combine": []}
    if w.backward:
        res.update({"bwd_combine_bwd": [], "bwd_dx_token_sum": []})
    shared = None
    if w.shared_expert:
        shared = torch.zeros((w.T, w.H), dtype=torch.bfloat16, device="cuda")

    def timed(fn):
        flush.sum()
        torch.cuda._sleep(200000)      # the GPU is busy while the call is issued: device time only
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        return s, e

    for it in range(warm + reps):
        fev = _events(7)
        flush.sum()
        torch.cuda._sleep(200000)
        m.moe_trace_set(fev)
        m.moe_layer_forward(d["logits"], d["x"], d["w_gate_up"], d["w_down"], w.k, layer.opts,
                            d["shared_gate_up"], d["shared_down"], save_for_backward=w.backward,
                            workspace=layer.ws, out=layer.out, state=layer.fwd_state)
        m.moe_trace_set(None)
        c = timed(lambda: m.moe_unpermute_combine(st["y_perm"], st["row_of"], st["topk_prob"], shared,
                                                  out=layer.out))
        if w.backward:
            bev = _events(7)
            flush.sum()
            torch.cuda._sleep(200000)
            m.moe_trace_set(bev)
            m.moe_grouped_mlp_backward(d["dout"], st, d["w_gate_up"], d["w_down"], layer.ws, layer.grads)
            m.moe_trace_set(None)
            dxs = timed(lambda: m.moe_unpermute_combine(st["y_perm"], st["row_of"], None, out=layer.out))
        torch.cuda.synchronize()
        if it < warm:
            continue
        res["fwd_router"].append(fev[0].elapsed_time(fev[1]))
        res["fwd_permute"].append(fev[1].elapsed_time(fev[2]))
        res["fwd_combine"].append(c[0].elapsed_time(c[1]))
        if w.backward:
            res["bwd_combine_bwd"].append(bev[0].elapsed_time(bev[1]))
            res["bwd_dx_token_sum"].append(dxs[0].elapsed_time(dxs[1]))
    nbytes = bandwidth_bytes(w)
    out = {}
    for key, v in res.items():
        ms = statistics.median(v)
        out[key] = {"cold_us": ms * 1e3, "cold_frac_of_hbm": nbytes[key] / (ms / 1e3) / 1e9 / hbm}
    return out


def bandwidth_report(layer, stages, hbm, flush):
    bw = warm_bandwidth(layer.w, stages, hbm)
    for key, v in cold_bandwidth(layer, hbm, flush).items():
        bw[key].update(v)
    return bw


def nonempty_experts(layer):
    return int((layer.state["counts"] > 0).sum().item())


def traced_pass(layer, steps, flush=None):
    """Per-stage events on `steps` further steps (the stage boundaries break
    the programmatic overlap of consecutive kernels, so the step times are
    taken without them); with `flush`, L2 is flushed before each step."""
    import torch
    fevs, bevs = [], []
    for _ in range(steps):
        fev = _events(7)
        bev = _events(7) if layer.w.backward else None
        if flush is not None:
            flush.sum()
            torch.cuda._sleep(200000)
        layer.step(fev, bev)
        fevs.append(fev)
        bevs.append(bev)
    torch.cuda.synchronize()
    return fevs, bevs


def measure_flushed(layer, steps, warmup, flush):
    """Each step timed on its own after an L2 flush (for workloads whose
    weights could stay in L2 between steps); median over the steps."""
    import torch
    totals = []
    for it in range(warmup + steps):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.sum()
        torch.cuda._sleep(200000)   # the GPU is busy while the step is issued: device time only
        s.record()
        layer.step()
        e.record()
        torch.cuda.synchronize()
        if it >= warmup:
            totals.append(s.elapsed_time(e))
    fevs, bevs = traced_pass(layer, steps, flush)
    return statistics.median(totals), fevs, bevs


def measure_back_to_back(layer, steps, warmup):
    """`steps` steps back to back between two events (no flush: the weights
    exceed L2), then a traced pass for the stage times."""
    import torch
    for _ in range(warmup):
        layer.step()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(steps):
        layer.step()
    e.record()
    torch.cuda.synchronize()
    fevs, bevs = traced_pass(layer, steps)
    return s.elapsed_time(e) / steps, fevs, bevs


def workload_entry(m, name, peaks, flush, steps, warmup, local):
    """One extra workload, timed like the main line: after a one-second idle
    (so each workload starts from the same power state), `warmup` steps,
    then `steps` timed steps with the clocks sampled. Reports the median step
    time, tokens/s, grouped-GEMM fractions, the warm bandwidth stages, and for
    the small batches the HBM roofline of the non-empty experts' weights.
    Returns (entry, layer); the L2-cold bandwidth stages are measured later
    (cold_pass), so that their loops do not heat the GPU before the next
    workload's timing."""
    import torch
    import workloads as wl
    w = wl.WORKLOADS[name]
    d = wl.make_inputs(w, "cuda")
    layer = Layer(m, w, d)
    small = w.T <= 64
    torch.cuda.synchronize()
    time.sleep(1.0)
    sampler = ClockSampler(local)
    sampler.start()
    if small:
        ms, fevs, bevs = measure_flushed(layer, steps, warmup, flush)
    else:
        ms, fevs, bevs = measure_back_to_back(layer, steps, warmup)
    clocks = sampler.stop()
    if m.moe_get_device_status() != 0:
        raise RuntimeError(f"device status error in {name}")
    stages = stage_medians(layer, fevs, bevs)
    hbm = peaks["hbm_gbs"]
    e = {"T": w.T, "H": w.H, "I": w.I, "E": w.E, "top_k": w.k, "pass": "fwd+bwd" if w.backward else "fwd",
         "steps": steps, "warmup": warmup, "ms_per_step": ms, "tokens_per_s": w.T / (ms / 1e3),
         "l2": "flushed (256 MB read) before each step" if small else "weights exceed L2; steps back to back",
         "clocks": clocks,
         "grouped_gemm": gemm_summary(w, stages, peaks),
         "stages_us": {k_: v * 1e3 for k_, v in stages.items()}}
    if small:
        ne = nonempty_experts(layer)
        wbytes = ne * 3 * w.H * w.I * 2
        gemm_ms = stages["fwd_gate_up_swiglu"] + stages["fwd_down"]
        e["roofline"] = {"bound": "hbm", "unit": "GB/s",
                         "weight_bytes": wbytes, "nonempty_experts": ne,
                         "gemm_us": gemm_ms * 1e3, "achieved": wbytes / (gemm_ms / 1e3) / 1e9, "peak": hbm,
                         "frac": wbytes / (gemm_ms / 1e3) / 1e9 / hbm,
                         "layer_frac": wbytes / (ms / 1e3) / 1e9 / hbm,
                         "note": "bytes = the non-empty experts' weights (3 H I bf16 each), read once per step; "
                                 "frac over the two GEMM stages, layer_frac over the whole step"}
        return e, None
    e["bandwidth_kernels"] = warm_bandwidth(w, stages, hbm)
    return e, layer


def extra_workloads(m, args, peaks, flush, local, skip):
    """Every other workload, timed one after another, then their L2-cold
    bandwidth stages in a second pass."""
    import torch
    steps, warmup = max(args.steps, 20), max(args.warmup, 5)
    out, layers = {}, {}
    for n in EXTRA_WORKLOADS:
        if n == skip:
            continue
        out[n], layers[n] = workload_entry(m, n, peaks, flush, steps, warmup, local)
    for n, layer in layers.items():
        if layer is None:
            continue
        for key, v in cold_bandwidth(layer, peaks["hbm_gbs"], flush).items():
            out[n]["bandwidth_kernels"][key].update(v)
    layers.clear()
    torch.cuda.empty_cache()
    return out


def our_arm(args, world, rank, local):
    import torch

    import routing_grouped_gemm_score_b200 as m
    import workloads as wl
    from routing_grouped_gemm_score_b200 import build as bld
    bld.build()
    torch.cuda.set_device(local)
    w = workload(args)
    # each rank its own tokens (seeded per rank), the same weights
    d = wl.make_inputs(w, "cuda")
    if rank:
        wr = w.scaled(seed=w.seed + 1000 * rank)
        d["logits"] = wl.make_logits(wr, "cuda")
        d["x"] = wl.make_x(wr, "cuda")
        if w.backward:
            d["dout"] = wl.make_dout(wr, "cuda")
    layer = Layer(m, w, d)

    for _ in range(args.warmup):
        layer.step()
    torch.cuda.synchronize()
    if m.moe_get_device_status() != 0:
        raise RuntimeError("device status error after warm-up")

    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    start.record()
    for i in range(K):
        layer.step()
    end.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    ms = start.elapsed_time(end)
    ms_max = max_over_ranks(ms, world)
    if m.moe_get_device_status() != 0:
        raise RuntimeError("device status error in the timed region")
    # stage times: a separate pass of K steps with an event at every stage
    # boundary (events between kernels break their programmatic overlap),
    # after a second of idle so that it starts from the timed region's power
    # state rather than from the end of it; its clocks are reported with it
    time.sleep(1.0)
    tsampler = ClockSampler(local)
    tsampler.start()
    fevs, bevs = traced_pass(layer, K)
    traced_clocks = tsampler.stop()
    stages = stage_medians(layer, fevs, bevs)

    graph = None if args.no_graph else graph_measure(args, layer.step, w, world, m)

    value = whole_job_value(w.T, world, K, ms_max)
    peaks, peaks_src = load_peaks()
    # Under dense tensor load the 1 kW part settles at its power cap within
    # about a hundred milliseconds, so a timed region of a quarter second or
    # more is measured against the sustained peak; a shorter one against the
    # burst peak.
    long_region = ms / 1e3 >= 0.25
    peak_tf = peaks["bf16_tflops_sustained" if long_region else "bf16_tflops"]
    burst_tf = peaks["bf16_tflops"]
    gate_up_flop = 4.0 * w.A * w.H * w.I
    gate_up_ms = stages["fwd_gate_up_swiglu"]
    achieved = gate_up_flop / (gate_up_ms / 1e3) / 1e12
    gg = gemm_summary(w, stages, peaks)
    gg["frac_of_peak"] = gg["tflops"] / peak_tf
    gg["peak_tflops"] = peak_tf
    hbm = peaks["hbm_gbs"]
    flush = torch.ones(64 << 20, dtype=torch.float32, device="cuda")   # a 256 MB read evicts L2

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_max / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict(w, args),
        "grouped_gemm": gg,
        "roofline": {"bound": "tensor", "kernel": "gate_up + SwiGLU grouped GEMM (routed experts)",
                     "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": achieved / peak_tf, "frac_of_burst_peak": achieved / burst_tf,
                     "frac_of_nominal_peak": achieved / NOMINAL_BF16_TFLOPS,
                     "traffic": traffic_for(f"gate_up_swiglu/{w.name}"),
                     "peak_source": f"{peaks_src} {'sustained' if long_region else 'burst'} bf16",
                     "flop_per_launch": gate_up_flop, "ms_per_launch": gate_up_ms,
                     "ms_per_launch_is": "median over a traced pass of as many steps as the timed region, events on the launching stream",
                     "clocks_traced_pass": traced_clocks},
        "stages_ms": stages,
        "stages_note": ("the combine runs in the shared expert's down GEMM epilogue: fwd_shared_expert holds it "
                        "and fwd_combine is empty") if combine_folded(w) else None,
        "bandwidth_kernels": bandwidth_report(layer, stages, hbm, flush),
        "hbm_peak_gbs": hbm,
        "gpu_launches": K * layer.launches(),
        "clocks": clocks,
    }

    if graph:
        line["cuda_graph"] = graph
    if not args.no_e2e:
        line["e2e"] = e2e_measure(args, w, d, m, layer.opts, layer.ws, world)
    if world == 1 and not args.no_extra and args.T is None:
        del layer
        torch.cuda.empty_cache()
        line["workloads"] = extra_workloads(m, args, peaks, flush, local, w.name)
    if args.router_sweep:
        line["router_sweep"] = router_sweep(m, hbm)
    if args.gather_compare:
        line["gather_compare"] = gather_compare(m)
    if args.scaled_compare:
        line["scaled_compare"] = scaled_compare(m)
    if not args.no_cpu_baseline and world == 1 and rank == 0:
        threads = os.cpu_count() or 1
        runner = OracleRunner(w, cpu_inputs(w, d), threads)
        tokens = runner.sample_for(10.0)
        n = len(tokens)
        tps = n / runner.time(tokens)
        line["cpu_baseline"] = {"value": tps, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": f"{n} of {w.T} tokens of the same workload"
                                          f"{' (fwd + dx/dprob bwd)' if w.backward else ''}, "
                                          f"plain C oracle, fp64 accumulation"}
    if rank == 0:
        print(json.dumps(line))
    return 0


def router_sweep(m, hbm):
    """The router alone (score + top-k + weights + counts/offsets) at E=128,
    k=8 on N(0,1) logits, large T, each launch L2-cold (logits > L2 from
    T = 2^18 on; before every launch a 256 MB read evicts them). A short GPU
    spin between the flush and the start event keeps the host's launch time
    out of the measured interval."""
    import ctypes

    import torch
    out = []
    # a 256 MB read evicts the logits from L2 and leaves only clean lines there
    flush = torch.ones(64 << 20, dtype=torch.float32, device="cuda")
    for logT in (16, 18, 20):
        T, E, k = 1 << logT, 128, 8
        g = torch.Generator(device="cuda").manual_seed(77 + logT)
        logits = torch.randn((T, E), generator=g, device="cuda")
        res = m.moe_router_topk(logits, k)
        ws = torch.empty(m.lib().moe_router_workspace_size(T, E, k), dtype=torch.uint8, device="cuda")
        times = []
        for it in range(8):
            flush.sum()
            torch.cuda._sleep(200000)   # the GPU is busy while the call is issued: device time only
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            oc = m.RouterOpts().c()
            s.record()
            m.lib().moe_router_topk(logits.data_ptr(), T, E, k, ctypes.byref(oc),
                                    res["topk_idx"].data_ptr(), res["topk_prob"].data_ptr(), None,
                                    res["counts"].data_ptr(), res["offsets"].data_ptr(),
                                    ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
            e.record()
            torch.cuda.synchronize()
            if it >= 2:
                times.append(s.elapsed_time(e))
        ms = statistics.median(times)
        nbytes = T * E * 4 + T * k * 8 + E * 8
        gbs = nbytes / (ms / 1e3) / 1e9
        entry = {"T": T, "E": E, "k": k, "us": ms * 1e3, "GB/s": gbs, "frac_of_hbm": gbs / hbm}
        # the backward through the score function on the same routing:
        # reads logits, topk_idx and dprob, writes dlogits
        dprob = torch.randn((T, k), generator=g, device="cuda")
        dl = torch.empty_like(logits)
        btimes = []
        for it in range(8):
            flush.sum()
            torch.cuda._sleep(200000)   # the GPU is busy while the call is issued: device time only
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            m.moe_router_backward(logits, res["topk_idx"], dprob, out=dl)
            e.record()
            torch.cuda.synchronize()
            if it >= 2:
                btimes.append(s.elapsed_time(e))
        bms = statistics.median(btimes)
        bbytes = 2 * T * E * 4 + T * k * 8
        entry["backward"] = {"us": bms * 1e3, "GB/s": bbytes / (bms / 1e3) / 1e9,
                             "frac_of_hbm": bbytes / (bms / 1e3) / 1e9 / hbm}
        # the auxiliary load-balancing loss on the same logits and counts: the
        # forward reads the logits once; its backward reads them and writes dlogits
        aws = torch.empty(m.lib().moe_aux_loss_workspace_size(T, E), dtype=torch.uint8, device="cuda")
        for name, call, nb in (
                ("aux_loss", lambda: m.moe_aux_loss(logits, res["counts"], k, 1e-2, workspace=aws),
                 T * E * 4 + E * 4),
                ("aux_loss_backward", lambda: m.moe_aux_loss_backward(logits, res["counts"], k, 1e-2, dlogits=dl),
                 2 * T * E * 4 + E * 4)):
            atimes = []
            for it in range(8):
                flush.sum()
                torch.cuda._sleep(200000)   # the GPU is busy while the call is issued: device time only
                s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                s.record()
                call()
                e.record()
                torch.cuda.synchronize()
                if it >= 2:
                    atimes.append(s.elapsed_time(e))
            ams = statistics.median(atimes)
            entry[name] = {"us": ams * 1e3, "GB/s": nb / (ams / 1e3) / 1e9,
                           "frac_of_hbm": nb / (ams / 1e3) / 1e9 / hbm}
        out.append(entry)
        del logits, res, ws, dprob, dl, aws
    return out


def scaled_compare(m):
    """The Qwen3-30B-A3B-shaped training step (T=4096, H=2048, I=768, E=128,
    k=8, forward and backward) three ways, each L2-flushed before the step
    and timed by CUDA events on the device (median of 10 after 3):
    - the default layer: moe_layer_forward (weights applied in combine) and
      moe_grouped_mlp_backward;
    - ScaledSwiGLU on a padded dispatch (align 16 and 128):
      moe_permute_padded -> moe_grouped_mlp_scaled (h = p silu(g) u) ->
      unweighted moe_unpermute_combine_rows, then
      moe_grouped_mlp_scaled_backward on the saved rows.
    The router runs in every step. GEMM rates count the real rows only (the
    pad rows' products are zeros)."""
    import torch
    import workloads as wl
    w = wl.WORKLOADS["qwen3_30b_a3b"]
    d = wl.make_inputs(w, "cuda", with_dout=True)
    opts = m.RouterOpts(w.score, w.renormalize)
    flush = torch.ones(64 << 20, dtype=torch.float32, device="cuda")
    flops = 2.0 * w.T * w.k * w.H * 3 * w.I * 3   # forward and backward grouped GEMMs

    ws = m.LayerWorkspace(w.T, w.H, w.I, w.E, w.k, w.shared_expert, backward=True)
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device="cuda")
    _, state = m.moe_layer_forward(d["logits"], d["x"], d["w_gate_up"], d["w_down"], w.k, opts,
                                   save_for_backward=True, workspace=ws, out=out)
    grads = m.moe_grouped_mlp_backward(d["dout"], state, d["w_gate_up"], d["w_down"], ws)

    def layer_step():
        m.moe_layer_forward(d["logits"], d["x"], d["w_gate_up"], d["w_down"], w.k, opts, save_for_backward=True,
                            workspace=ws, out=out, state=state)
        m.moe_grouped_mlp_backward(d["dout"], state, d["w_gate_up"], d["w_down"], ws, grads)

    def scaled_step(align):
        def step():
            r = m.moe_router_topk(d["logits"], w.k, opts)
            p = m.moe_permute_padded(d["x"], r["topk_idx"], r["offsets"], align, r["topk_prob"])
            mlp = m.moe_grouped_mlp_scaled(p["x_perm"], p["padded_offsets"], d["w_gate_up"], d["w_down"],
                                           p["prob_perm"], save=True)
            m.moe_unpermute_combine(mlp["y_perm"], p["row_of"], None)
            m.moe_grouped_mlp_scaled_backward(d["dout"], p["row_of"], p["sorted_token"], p["prob_perm"],
                                              p["padded_offsets"], p["x_perm"], mlp["gu"], mlp["h"],
                                              d["w_gate_up"], d["w_down"])
        return step

    res = {"workload": "qwen3_30b_a3b fwd+bwd (T=4096), L2 flushed before each step"}
    for name, step in (("default_layer", layer_step), ("scaled_align16", scaled_step(16)),
                       ("scaled_align128", scaled_step(128))):
        times = []
        for it in range(13):
            flush.sum()
            torch.cuda._sleep(200000)   # the GPU is busy while the calls are issued: device time only
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            step()
            e.record()
            torch.cuda.synchronize()
            if it >= 3:
                times.append(s.elapsed_time(e))
        ms = statistics.median(times)
        res[name] = {"ms_per_step": ms, "tokens_per_s": w.T / (ms / 1e3),
                     "gemm_tflop_per_step_time": flops / (ms / 1e3) / 1e12}
    if m.moe_get_device_status() != 0:
        raise RuntimeError("device status after the ScaledSwiGLU comparison")
    res["note"] = ("gemm_tflop_per_step_time divides the grouped GEMMs' FLOPs by the whole step's time "
                   "(router, permute and combine included); the padded steps also allocate their outputs "
                   "through torch's caching allocator inside the timed region")
    return res


def gather_compare(m):
    """The forward of the Qwen3-30B-A3B-shaped layer (T=4096, H=2048, I=768,
    E=128, k=8), no saved state, L2-flushed before each call: the permute
    writes x_perm and the gate_up GEMM loads it with TMA tiles, against the
    permute computing only the rows and the GEMM gathering its A rows from x
    (the folded permute of moe_testing_set_kernels). The outputs are
    bit-identical (tested)."""
    import torch
    import workloads as wl
    w = wl.WORKLOADS["qwen3_30b_a3b"]
    d = wl.make_inputs(w, "cuda", with_dout=False)
    opts = m.RouterOpts(w.score, w.renormalize)
    flush = torch.ones(64 << 20, dtype=torch.float32, device="cuda")
    res = {"workload": "qwen3_30b_a3b forward, no saved state"}
    for name, fold in (("x_perm_us", 0), ("gather_us", 1)):
        m.moe_testing_set_kernels(fold_permute=fold)
        times = []
        for it in range(12):
            flush.sum()
            torch.cuda._sleep(200000)   # the GPU is busy while the call is issued: device time only
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            m.moe_layer_forward(d["logits"], d["x"], d["w_gate_up"], d["w_down"], w.k, opts)
            e.record()
            torch.cuda.synchronize()
            if it >= 2:
                times.append(s.elapsed_time(e) * 1e3)
        res[name] = statistics.median(times)
    m.moe_testing_set_kernels()
    if m.moe_get_device_status() != 0:
        raise RuntimeError("device status after the gather comparison")
    return res


def graph_measure(args, step, w, world, m):
    """The same step captured once in a CUDA graph and replayed: the device
    time without per-launch host overhead (the calls allocate nothing and
    never sync, so a whole step captures as is)."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    K = max(1, args.steps)   # as many steps as the main timed region, under the same power state
    barrier(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(K):
        g.replay()
    end.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(end), world)
    if m.moe_get_device_status() != 0:
        raise RuntimeError("device status error in the graph replays")
    del g
    return {"value": w.T * world * K / (ms / 1e3), "unit": UNIT, "ms_per_step": ms / K, "steps": K,
            "note": "one step captured in a CUDA graph, replayed back to back"}


def e2e_measure(args, w, d, m, opts, ws, world):
    """Same metric through the public calls with host buffers: every step
    copies its inputs (logits, x, and dout for a training step) from pinned
    host memory to the device and reads the step's result back (the layer
    output, or dx for a training step), inside the timed region.

    The steps are pipelined the way a serving or training loop runs them: the
    copy-in of step i+1 (one stream) and the read-back of step i-1 (another)
    overlap the compute of step i, with two device slots for the inputs and
    the result. Every step still moves all of its bytes inside the region."""
    import torch
    h_logits = d["logits"].cpu().pin_memory()
    h_x = d["x"].cpu().pin_memory()
    h_dout = d["dout"].cpu().pin_memory() if w.backward else None
    h_res = [torch.empty((w.T, w.H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    dl = [torch.empty_like(d["logits"]) for _ in range(2)]
    dx = [torch.empty_like(d["x"]) for _ in range(2)]
    ddo = [torch.empty_like(d["dout"]) for _ in range(2)] if w.backward else None
    out = [torch.empty((w.T, w.H), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    K = max(1, args.steps)   # as many steps as the main timed region
    state = None
    grads = None
    if w.backward:
        _, state = m.moe_layer_forward(d["logits"], d["x"], d["w_gate_up"], d["w_down"], w.k, opts,
                                       save_for_backward=True, workspace=ws, out=out[0])
        g0 = m.moe_grouped_mlp_backward(d["dout"], state, d["w_gate_up"], d["w_down"], ws)
        # the weight gradients are consumed on the device; dx is read back, so it has two slots
        grads = [dict(g0), dict(g0, dx=torch.empty_like(g0["dx"]))]

    compute = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready = [ev(), ev()]      # the slot's inputs have landed
    in_free = [ev(), ev()]       # the compute has finished reading the slot's inputs
    res_ready = [ev(), ev()]     # the slot's result is complete
    res_free = [ev(), ev()]      # the slot's result has been read back
    for e in in_free + res_free:
        e.record(compute)

    def step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(in_free[b])
            dl[b].copy_(h_logits, non_blocking=True)
            dx[b].copy_(h_x, non_blocking=True)
            if w.backward:
                ddo[b].copy_(h_dout, non_blocking=True)
            in_ready[b].record(s_in)
        compute.wait_event(in_ready[b])
        compute.wait_event(res_free[b])
        m.moe_layer_forward(dl[b], dx[b], d["w_gate_up"], d["w_down"], w.k, opts, d["shared_gate_up"],
                            d["shared_down"], save_for_backward=w.backward, workspace=ws, out=out[b],
                            state=state)
        if w.backward:
            m.moe_grouped_mlp_backward(ddo[b], state, d["w_gate_up"], d["w_down"], ws, grads[b])
        in_free[b].record(compute)
        res_ready[b].record(compute)
        res = grads[b]["dx"] if w.backward else out[b]
        with torch.cuda.stream(s_out):
            s_out.wait_event(res_ready[b])
            h_res[b].copy_(res, non_blocking=True)
            res_free[b].record(s_out)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(compute)
    s_in.wait_stream(compute)      # the first copy-in starts after the start event
    for i in range(K):
        step(i)
    compute.wait_stream(s_out)     # the end event follows the last read-back
    e.record(compute)
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e), world)
    h2d = h_logits.numel() * 4 + h_x.numel() * 2 + (h_dout.numel() * 2 if w.backward else 0)
    return {"value": w.T * world * K / (ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": h_res[0].numel() * 2, "steps": K,
            "pass": "fwd+bwd" if w.backward else "fwd",
            "pipelined": "copy-in of step i+1 and read-back of step i-1 overlap step i on two copy streams",
            "note": "weights resident on the device; the step's result read back is "
                    + ("dx" if w.backward else "the layer output")}


def router_calls(log_t: int) -> int:
    """Three router calls at T = 2^log_t, E=128, k=8 on seeded N(0,1) logits:
    the program the router's ncu captures run."""
    import torch

    import routing_grouped_gemm_score_b200 as m
    T = 1 << log_t
    g = torch.Generator(device="cuda").manual_seed(77)
    logits = torch.randn((T, 128), generator=g, device="cuda")
    for _ in range(3):
        m.moe_router_topk(logits, 8)
    torch.cuda.synchronize()
    if m.moe_get_device_status() != 0:
        raise RuntimeError("device status after the router calls")
    print(json.dumps({"router_calls": 3, "T": T, "E": 128, "k": 8}))
    return 0


def main():
    args = parse()
    if args.router_calls is not None:
        return router_calls(args.router_calls)
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            return reference_arm(args, world, rank)
        return our_arm(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
