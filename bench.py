#!/usr/bin/env python
"""Benchmark of the MoE expert-MLP + Split-LoRA layer, forward + backward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one pass of the whole hot path on one batch: top-k routing,
counting-sort permute, grouped GEMM forward (gate_up + SwiGLU, down, Split-LoRA
fused), weighted combine, grouped GEMM backward (dX, dA, dB with W frozen) and
the dX combine.  Default workload: the Qwen3-30B-A3B-shaped layer (T=4096,
m=2048, n=768, E=128, k=8, r=16), synthetic seeded inputs resident in HBM.

N > 1 (torchrun, one process per GPU): data parallel.  Every rank runs its own
batch of T tokens against the same expert weights and the adapter gradients
are summed across ranks with one NCCL all-reduce per step (weak scaling).

Rank 0 prints ONE JSON line.  `--impl reference` times the fp64 CPU oracle on
bounded token samples of the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from moe_inputs import CONFIGS, generate  # noqa: E402
from mixture_experts_lora_b200 import accounting as acc  # noqa: E402

METRIC = "MoE-layer fwd+bwd tokens/s and TFLOP/s as % of B200 bf16 dense peak"
UNIT = "tokens/s"
FLUSH_BYTES = 256 << 20          # > 126 MB L2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="qwen3_30b_a3b", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every kernel from the host in the timed steps instead of replaying "
                         "one captured CUDA graph per step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-tokens", type=int, default=0,
                    help="tokens per oracle sample (0: sized for ~15 s)")
    ap.add_argument("--plain", action="store_true",
                    help="run W + K layer steps with host launches and no timing, tracing or "
                         "JSON line, then exit (a short command for profilers; one GPU)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def workload_name(cfg):
    return (f"{cfg.name}: MoE expert-MLP + Split-LoRA layer fwd+bwd, T={cfg.T} m={cfg.m} "
            f"n={cfg.n} E={cfg.E} k={cfg.k} r={cfg.r} alpha={cfg.alpha:g}")


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples every 100 ms while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]), "power": float(parts[3]),
                             "hw": parts[5], "hw_thermal": parts[6], "sw_thermal": parts[7],
                             "sw_power": parts[8]})
            except ValueError:
                continue
        if not rows:
            return None
        load = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                              ("sw_thermal", "sw_thermal_slowdown"), ("sw_power", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load)}


# ---------------------------------------------------------------- accounting
def kernel_work(cfg, active_experts=None):
    """Algorithmic work of each kernel kind for one step: {kind: {"flop": F, "byte": B}}.
    Byte counts read and write each tensor once (rank-r outputs included); X and dY
    are read once (the kernels gather their rows, k copies per token, from L2); a GEMM
    reads the frozen weights of the experts that received tokens once."""
    T, m, n, E, k, r = cfg.T, cfg.m, cfg.n, cfg.E, cfg.k, cfg.r
    Ea = E if active_experts is None else active_experts
    P = T * k
    rp = 16 if r <= 16 else 32 if r <= 32 else 64 if r <= 64 else 128
    tok = T * m * 2                                       # X or dY, read once
    rows = P * m * 2                                      # expert-ordered X or w dY
    lrc = P * rp * 2                                      # one [P, rp] rank-r operand
    return {
        "gemm_gateup_fwd": {"flop": acc.flops_gemm_gate_up_fwd(T, m, n, k, r),
                            "byte": Ea * m * 2 * n * 2 + rows + lrc + Ea * r * 2 * n * 2
                                    + P * 2 * n * 2 + P * n * 2},            # GU and H written
        "gemm_down_fwd": {"flop": acc.flops_gemm_down_fwd(T, m, n, k, r),
                          "byte": Ea * n * m * 2 + P * n * 2 + lrc + Ea * r * m * 2 + P * m * 2},
        "gemm_down_bwd": {"flop": acc.flops_gemm_down_bwd(T, m, n, k, r),
                          "byte": Ea * n * m * 2 + rows + lrc + Ea * n * r * 2 + P * n * 2},
        "gemm_gateup_bwd": {"flop": acc.flops_gemm_gate_up_bwd(T, m, n, k, r),
                            "byte": Ea * m * 2 * n * 2 + P * 2 * n * 2 + lrc + Ea * m * r * 2 + P * m * 2},
        # gathered X rows written in expert order, XA (saved) and bf16(c XA)
        "rank_xa": {"byte": tok + P * 4 + rows + E * m * r * 2 + P * r * 2 + lrc},
        "rank_ha": {"byte": P * n * 2 + E * n * r * 2 + P * r * 2 + lrc},
        # gathered w dY rows written in expert order, T1 and bf16(c T1)
        "rank_t1": {"byte": tok + P * 8 + rows + E * r * m * 2 + 2 * lrc},
        # the SwiGLU backward (dH and GU read, dGU written) with T2 and bf16(c T2)
        "rank_t2": {"byte": P * n * 2 + P * 2 * n * 2 + P * 2 * n * 2 + E * r * 2 * n * 2 + 2 * lrc},
        # two launches: (H, w dY) -> dA_d, dB_d; (dGU, X) -> dB_gu, dA_gu
        "lora_wgrad": {"byte": P * n * 2 + rows + lrc + P * r * 2 + E * r * (n + m) * 2
                               + P * 2 * n * 2 + rows + P * r * 2 + lrc + E * r * (m + 2 * n) * 2},
        # routing with the whole counting sort (one launch): logits read, ids and
        # weights written, ids read back, sorted_pairs and pair_pos written
        "route_topk": {"byte": acc.bytes_route(T, E, k) + P * 12},
        "unpermute_combine": {"byte": 2 * acc.bytes_combine(T, m, k)},  # Y and dX
        # full fine-tuning only: the expert-weight gradients (sorted operands read once,
        # every expert's gradient written once)
        "gemm_dw_gu": {"flop": 4 * P * m * n, "byte": P * m * 2 + P * 2 * n * 2 + E * m * 2 * n * 2},
        "gemm_dw_d": {"flop": 2 * P * n * m, "byte": P * n * 2 + P * m * 2 + E * n * m * 2},
    }


def roof_entry(work, per_launch_ms, launches_per_step, peaks):
    """Roofline of one kernel kind: achieved rate of each resource it uses and the
    binding one (the larger ideal time at the measured peaks)."""
    ent = {}
    sec = per_launch_ms / 1e3
    opts = []
    if "flop" in work:
        f = work["flop"] / launches_per_step
        a = f / sec / 1e12
        ent["tensor"] = {"achieved": a, "unit": "TFLOP/s", "peak": peaks["bf16_tflops_sustained"],
                         "frac": a / peaks["bf16_tflops_sustained"], "per_launch": f}
        opts.append(("tensor", f / (peaks["bf16_tflops_sustained"] * 1e12)))
    if "byte" in work:
        b = work["byte"] / launches_per_step
        a = b / sec / 1e9
        ent["hbm"] = {"achieved": a, "unit": "GB/s", "peak": peaks["hbm_gbs"],
                      "frac": a / peaks["hbm_gbs"], "per_launch": b}
        opts.append(("hbm", b / (peaks["hbm_gbs"] * 1e9)))
    if opts:
        ent["bound"] = max(opts, key=lambda o: o[1])[0]
    return ent


def src_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mixture_experts_lora_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, cfg_name: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, or None if
    there is none for this workload or the kernel sources changed since."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("src_hash") != src_hash():
        return None
    ent = d.get("kernels", {}).get(cfg_name, {}).get(kernel)
    return None if ent is None else ent.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- CPU oracle
def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        nums = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if nums:
            return max(nums)
    except Exception:
        pass
    return os.cpu_count() or 1


def time_oracle_sample(cfg, cpu_inp, W64, tok0, ntok):
    """Forward + backward of the oracle on tokens [tok0, tok0 + ntok) of the workload."""
    import numpy as np
    import oracle.moe_lora_oracle as O
    sl = slice(tok0, tok0 + ntok)
    inp = dict(W64)
    inp["logits"] = cpu_inp["logits"][sl].numpy().astype(np.float32)
    inp["X"] = O.to64(cpu_inp["X"][sl])
    dY = O.to64(cpu_inp["dY"][sl])
    t0 = time.perf_counter()
    Y, aux = O.moe_forward(inp, cfg.k, cfg.scale)
    O.moe_backward(inp, aux, dY, cfg.k, cfg.scale)
    return time.perf_counter() - t0


def oracle_setup(cfg, cpu_inp):
    import oracle.moe_lora_oracle as O
    return {k: O.to64(cpu_inp[k]) for k in ("W_gu", "W_d", "A_gu", "B_gu", "A_d", "B_d")}


def pick_sample_tokens(cfg, cpu_inp, W64, target_s, requested):
    """Tokens per oracle step for a step time of about target_s.  A step costs a fixed
    part (every touched expert's fp64 weights are streamed whatever its row count) plus
    a part per token, so a few tokens cost almost as much as a few hundred: the sample
    doubles from 64 tokens while a timed step stays under half the budget, instead of
    extrapolating from a handful of tokens."""
    if requested > 0:
        return requested
    n = min(64, cfg.T)
    time_oracle_sample(cfg, cpu_inp, W64, 0, n)     # first call: thread pool, page-in
    spent = 0.0
    while n < cfg.T and spent < 30.0:
        ts = [time_oracle_sample(cfg, cpu_inp, W64, 0, n) for _ in range(2)]
        spent += sum(ts)
        if min(ts) >= target_s / 2:          # the better of two: host timing is noisy
            break
        n = min(cfg.T, 2 * n)
    return n


def cpu_baseline(cfg, cpu_inp, requested, target_s=12.0, cap_s=40.0):
    """The oracle on the host cores: whole-workload passes (or `requested`-token
    samples) repeated until about target_s seconds of CPU work."""
    W64 = oracle_setup(cfg, cpu_inp)
    ntok = requested if requested > 0 else cfg.T
    done, spent, reps = 0, 0.0, 0
    while spent < target_s and spent < cap_s:
        tok0 = (reps * ntok) % max(1, cfg.T - ntok + 1)
        spent += time_oracle_sample(cfg, cpu_inp, W64, tok0, ntok)
        done += ntok
        reps += 1
    return {"value": done / spent, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
            "sample": f"fp64 NumPy oracle fwd+bwd, {reps} pass(es) of {ntok} of the {cfg.T} tokens "
                      f"of the same workload with all {cfg.E} experts' weights, {spent:.1f} s of "
                      f"wall clock; fp64 weight conversion done once outside the timing"}


def run_reference(args, cfg):
    """The oracle arm: rank 0 only; other ranks exit without work."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    cpu = generate(cfg, seed=0, device="cpu")
    W64 = oracle_setup(cfg, cpu)
    # each step a bounded sample: about two minutes for the whole run
    per_step_s = min(2.0, 120.0 / max(1, args.steps + args.warmup))
    ntok = pick_sample_tokens(cfg, cpu, W64, per_step_s, args.cpu_sample_tokens)
    for s in range(args.warmup):
        time_oracle_sample(cfg, cpu, W64, (s * ntok) % max(1, cfg.T - ntok), ntok)
    times = []
    for s in range(args.steps):
        times.append(time_oracle_sample(cfg, cpu, W64, (s * ntok) % max(1, cfg.T - ntok), ntok))
    step_s = statistics.mean(times)
    value = ntok / step_s
    cores = oracle_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": workload_name(cfg),
                                        "tokens_per_step_sample": ntok},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{ntok} tokens per step of the {cfg.T}-token workload"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our arm
def run_ours(args, cfg):
    import torch.distributed as dist
    import mixture_experts_lora_b200 as ml

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    ml.lib()  # fails loudly if the CUDA library is missing

    # inputs: weights shared by every rank (seed 0), tokens per rank
    from mixture_experts_lora_b200 import dp
    inp = dp.rank_inputs(cfg, rank, device=dev)
    buf = ml.alloc_buffers(cfg.T, cfg.m, cfg.n, cfg.E, cfg.k, cfg.r, cfg.scale, device=dev)
    grads = (buf.dA_gu, buf.dB_gu, buf.dA_d, buf.dB_d)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ml.layer_step(inp, cfg.k, cfg.scale, buf)
        dp.allreduce_adapter_grads(grads)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = ml.moe_get_device_error()
    if st != ml.MOE_OK:
        raise SystemExit(f"device error after warm-up: {ml.status_string(st)}")

    # ---- traced pass (not the timed value): every kernel kind bracketed by CUDA
    # events, for the per-kernel breakdown and to find the dominant kernel.  With
    # graphs the events are event-record nodes of each step's captured graph, so a
    # small kernel is not charged for the host's launch gaps (the records still
    # split the launches' programmatic overlap).
    ml.moe_profile_select(None)
    if args.no_graph:
        ml.moe_profile_enable(True)
        for _ in range(args.steps):
            flush.zero_()
            step()
    else:
        traced = []
        torch.cuda.synchronize()
        ml.moe_profile_enable(True)
        for _ in range(args.steps):
            gph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gph):
                ml.layer_step(inp, cfg.k, cfg.scale, buf)
            traced.append(gph)
        ml.moe_profile_enable(False)
        for gph in traced:
            flush.zero_()
            gph.replay()
            dp.allreduce_adapter_grads(grads)
        torch.cuda.synchronize()
        del traced
    torch.cuda.synchronize()
    ml.moe_profile_enable(False)
    prof_all = ml.moe_profile_read()
    launches_per_step = sum(v[0] for v in prof_all.values()) / args.steps
    top = max(prof_all, key=lambda k: prof_all[k][1]) if prof_all else None

    # ---- timed region (device time, CUDA events per step, L2 flushed before each
    # step outside the events); only the dominant kernel kind is traced, so its
    # events add two records per launch and nothing to the other kernels.  By
    # default each timed step replays its own CUDA graph of the layer's launches
    # (captured here, with the dominant kernel's trace events as graph nodes), so
    # the step carries no host launch gaps; the gradient all-reduce (N > 1) runs
    # after the replay, inside the step's events.
    if top is not None:
        ml.moe_profile_select(top)
        ml.moe_profile_enable(True)
    graphs = []
    if not args.no_graph:
        torch.cuda.synchronize()
        for i in range(args.steps):
            gph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gph):
                ml.layer_step(inp, cfg.k, cfg.scale, buf)
            graphs.append(gph)
        ml.moe_profile_enable(False)
        for gph in graphs:                 # upload; the trace records are read after the timed replays
            gph.replay()
        torch.cuda.synchronize()

    def timed_step(i):
        if graphs:
            graphs[i].replay()
            dp.allreduce_adapter_grads(grads)
        else:
            step()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(1.0)                       # nvidia-smi's first sample precedes the timed steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if top is not None and not graphs:
        ml.moe_profile_enable(True)
    for i in range(args.steps):
        flush.zero_()
        evs[i][0].record(stream)
        timed_step(i)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    ml.moe_profile_enable(False)
    prof_top = ml.moe_profile_read()
    ml.moe_profile_select(None)
    del graphs
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    mean_ms = statistics.mean(step_ms)
    median_ms = statistics.median(step_ms)
    if world > 1:
        t = torch.tensor([mean_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        mean_ms = float(t.item())
    st = ml.moe_get_device_error()
    if st != ml.MOE_OK:
        raise SystemExit(f"device error in timed region: {ml.status_string(st)}")
    active_experts = int((buf.counts > 0).sum().item())

    # ---- rows beyond the step, timed on their own (not part of the step's value):
    # the router backward (gradient into the logits), inputs from the last step
    extras = {}
    dlog = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=dev)

    def router_bwd():
        ml.moe_router_backward(inp["dY"], buf.Y_sorted, buf.ids, buf.w, buf.pair_pos, cfg.E, dlog)

    for _ in range(3):
        router_bwd()
    rb_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(min(args.steps, 50))]
    for a, b in rb_evs:
        flush.zero_()
        a.record(stream)
        router_bwd()
        b.record(stream)
    torch.cuda.synchronize()
    rb_ms = statistics.mean(a.elapsed_time(b) for a, b in rb_evs)
    P = cfg.T * cfg.k
    rb_bytes = P * cfg.m * 2 + cfg.T * cfg.m * 2 + cfg.T * cfg.E * 4 + P * 12
    extras["router_backward"] = {
        "what": "dlogits [T, E] from dY and the expert outputs (router backward; not part of the step)",
        "ms_per_launch": rb_ms, "algorithmic_bytes": rb_bytes,
        "achieved": rb_bytes / (rb_ms / 1e3) / 1e9, "unit": "GB/s"}

    def extra_ms(fn, n):
        """Mean device time of fn over n runs, L2 flushed before each outside the events:
        one captured CUDA graph replayed like the timed steps (host launches with
        --no-graph)."""
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        gph = None
        if not args.no_graph:
            gph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gph):
                fn()
            gph.replay()
            torch.cuda.synchronize()
        xevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(n)]
        for a, b in xevs:
            flush.zero_()
            a.record(stream)
            if gph is not None:
                gph.replay()
            else:
                fn()
            b.record(stream)
        torch.cuda.synchronize()
        del gph
        return statistics.mean(a.elapsed_time(b) for a, b in xevs)

    # the shared expert (dense MLP + LoRA on every token): the layer with one
    # expert at the same token count and dimensions
    from moe_inputs import LayerConfig
    scfg = LayerConfig("shared_expert", T=cfg.T, m=cfg.m, n=cfg.n, E=1, k=1, r=cfg.r, alpha=cfg.alpha)
    sinp = generate(scfg, seed=7, device=dev)
    sbuf = ml.alloc_buffers(scfg.T, scfg.m, scfg.n, 1, 1, scfg.r, scfg.scale, device=dev)
    se_ms = extra_ms(lambda: ml.shared_expert_step(sinp, scfg.scale, sbuf), min(args.steps, 50))
    if ml.moe_get_device_error() != ml.MOE_OK:
        raise SystemExit("device error in the shared-expert timing")
    se_flops = acc.flops_step(scfg.T, scfg.m, scfg.n, 1, scfg.r)
    extras["shared_expert"] = {
        "what": f"dense SwiGLU MLP + LoRA on all {scfg.T} tokens, fwd+bwd (shared expert; not part of the step)",
        "ms_per_step": se_ms, "tokens_per_s": scfg.T / (se_ms / 1e3),
        "tflops": se_flops / (se_ms / 1e3) / 1e12}

    # the routed layer and the shared expert together, on two streams of one graph, the
    # way a model with a shared expert runs them, against the two timed alone
    side = torch.cuda.Stream(device=dev)

    def routed_and_shared():
        main = torch.cuda.current_stream(dev)
        side.wait_stream(main)
        ml.layer_step(inp, cfg.k, cfg.scale, buf)
        with torch.cuda.stream(side):
            ml.shared_expert_step(sinp, scfg.scale, sbuf)
        main.wait_stream(side)

    routed_ms = extra_ms(lambda: ml.layer_step(inp, cfg.k, cfg.scale, buf), min(args.steps, 50))
    both_ms = extra_ms(routed_and_shared, min(args.steps, 50))
    if ml.moe_get_device_error() != ml.MOE_OK:
        raise SystemExit("device error in the routed + shared timing")
    extras["routed_plus_shared_expert"] = {
        "what": "the routed layer and the shared expert concurrently on two streams (one graph), "
                "fwd+bwd; alone they take routed_ms and shared_ms",
        "ms_per_step": both_ms, "routed_ms": routed_ms, "shared_ms": se_ms,
        "tokens_per_s": world * cfg.T / (both_ms / 1e3),
        "tflops": (acc.flops_step(cfg.T, cfg.m, cfg.n, cfg.k, cfg.r) + se_flops) / (both_ms / 1e3) / 1e12}
    del sinp, sbuf

    # separate gate/up adapters of rank r: the same workload run as the fused
    # rank-2r adapter (skipped when 2r > 128)
    if 2 * cfg.r <= 128:
        ad = ml.SplitGateUpAdapters(cfg.E, cfg.m, cfg.n, cfg.r, device=dev)
        gsp = torch.Generator(device=dev).manual_seed(5)
        for name in ("A_g", "A_u"):
            getattr(ad, name).copy_(torch.randn(getattr(ad, name).shape, generator=gsp, device=dev)
                                    / cfg.m ** 0.5)
        for name in ("B_g", "B_u"):
            getattr(ad, name).copy_(torch.randn(getattr(ad, name).shape, generator=gsp, device=dev) * 0.02)
        ad.A_d.copy_(inp["A_d"])
        ad.B_d.copy_(inp["B_d"])
        sp_inp = ad.layer_inputs(inp)
        sp_buf = ml.alloc_buffers(cfg.T, cfg.m, cfg.n, cfg.E, cfg.k, 2 * cfg.r, cfg.scale, device=dev)
        sp_ms = extra_ms(lambda: ml.layer_step(sp_inp, cfg.k, cfg.scale, sp_buf), min(args.steps, 50))
        if ml.moe_get_device_error() != ml.MOE_OK:
            raise SystemExit("device error in the separate-adapter timing")
        extras["separate_gate_up_adapters"] = {
            "what": f"the step with separate gate and up adapters of rank {cfg.r} (fused rank {2 * cfg.r})",
            "ms_per_step": sp_ms, "tokens_per_s": world * cfg.T / (sp_ms / 1e3)}
        del sp_buf, sp_inp, ad

    # routing and the counting sort alone (moe_route_permute: a memset and one cooperative
    # launch, logits to sorted pairs), one event pair around the call; the per-kernel
    # table's event nodes around the launch add several us.  A single replayed call also
    # carries the graph's launch latency, so the call is timed a second way too: a graph
    # of 20 calls back to back, divided by 20 (logits, 2 MB at this shape, stay in L2
    # between those calls, as they do after the router GEMM that writes them)
    def route_call():
        ml.moe_route_permute(inp["logits"], cfg.k, buf.ids, buf.w, buf.counts, buf.offsets,
                             buf.sorted_pairs, buf.pair_pos, buf.ws)

    def route_20():
        for _ in range(20):
            route_call()

    rp_ms = extra_ms(route_call, min(args.steps, 50))
    rp20_ms = extra_ms(route_20, min(args.steps, 20)) / 20
    if ml.moe_get_device_error() != ml.MOE_OK:
        raise SystemExit("device error in the routing timing")
    extras["route_permute"] = {
        "what": "routing and the counting-sort permutation (a memset and one cooperative "
                "launch) timed as one call, and per call in a graph of 20 calls",
        "ms_per_call": rp_ms, "ms_per_call_in_sequence": rp20_ms}

    # the same step at LoRA rank 64, the rank the pages work their numbers at
    # (adapters drawn with the same distributions; alpha = r, so c = 1)
    if cfg.r != 64:
        g64 = torch.Generator(device=dev).manual_seed(7)
        r64 = dict(inp)
        for name, shape, std in (("A_gu", (cfg.E, cfg.m, 64), cfg.m ** -0.5),
                                 ("B_gu", (cfg.E, 64, 2 * cfg.n), 0.02),
                                 ("A_d", (cfg.E, cfg.n, 64), cfg.n ** -0.5),
                                 ("B_d", (cfg.E, 64, cfg.m), 0.02)):
            r64[name] = (torch.randn(shape, generator=g64, device=dev) * std).to(torch.bfloat16)
        b64 = ml.alloc_buffers(cfg.T, cfg.m, cfg.n, cfg.E, cfg.k, 64, 1.0, device=dev)
        r64_ms = extra_ms(lambda: ml.layer_step(r64, cfg.k, 1.0, b64), min(args.steps, 50))
        if ml.moe_get_device_error() != ml.MOE_OK:
            raise SystemExit("device error in the rank-64 timing")
        r64_flops = acc.flops_step(cfg.T, cfg.m, cfg.n, cfg.k, 64)
        extras["rank_64"] = {
            "what": "the step at LoRA rank 64 (alpha 64) on the same workload",
            "ms_per_step": r64_ms, "tokens_per_s": world * cfg.T / (r64_ms / 1e3),
            "tflops": r64_flops / (r64_ms / 1e3) / 1e12}
        del b64, r64

    # full fine-tuning: forward, then the backward with the expert-weight
    # gradients dW_gu, dW_d and no adapter gradients
    dWg = torch.empty(cfg.E, cfg.m, 2 * cfg.n, dtype=torch.bfloat16, device=dev)
    dWd = torch.empty(cfg.E, cfg.n, cfg.m, dtype=torch.bfloat16, device=dev)

    def fft_step():
        ml.layer_forward(inp, cfg.k, cfg.scale, buf)
        ml.layer_backward_full(inp, inp["dY"], cfg.k, cfg.scale, buf, dWg, dWd, adapters=False)

    ft_ms = extra_ms(fft_step, min(args.steps, 50))
    # the two weight-gradient kernels, timed on their own launches in a few more steps
    ml.moe_profile_select(["gemm_dw_gu", "gemm_dw_d"])
    ml.moe_profile_enable(True)
    for _ in range(10):
        flush.zero_()
        fft_step()
    ml.moe_profile_enable(False)
    ft_prof = ml.moe_profile_read()
    ml.moe_profile_select(None)
    if ml.moe_get_device_error() != ml.MOE_OK:
        raise SystemExit("device error in the full fine-tuning timing")
    ft_flops = (acc.flops_step(cfg.T, cfg.m, cfg.n, cfg.k, cfg.r)
                - acc.flops_lora_wgrad(cfg.T, cfg.m, cfg.n, cfg.k, cfg.r) + 6 * P * cfg.m * cfg.n)
    ft_kern = {}
    ft_work, (ft_peaks, _) = kernel_work(cfg, active_experts), load_peaks()
    for name in ("gemm_dw_gu", "gemm_dw_d"):
        if name in ft_prof and ft_prof[name][0] > 0:
            launches, tot = ft_prof[name]
            ft_kern[name] = {"ms_per_launch": tot / launches,
                             **roof_entry(ft_work[name], tot / launches, 1, ft_peaks)}
    extras["full_fine_tuning"] = {
        "what": "forward + backward with the expert-weight gradients dW_gu, dW_d (no adapter "
                "gradients; not part of the step)",
        "ms_per_step": ft_ms, "tokens_per_s": world * cfg.T / (ft_ms / 1e3),
        "tflops": ft_flops / (ft_ms / 1e3) / 1e12, "kernels": ft_kern}
    del dWg, dWd

    # ---- end to end through the public API with host buffers
    # Every step copies its inputs (logits, X, dY) in from pinned host memory and its
    # results (Y, dX and the four adapter gradients) back out, inside the timed region.
    # As an input pipeline does, step i + 1's inputs move in and step i - 1's results
    # move out while step i computes: two sets of device inputs and layer buffers, one
    # copy stream per direction, all ordered by events.
    e2e = None
    if not args.no_e2e:
        keys = ("logits", "X", "dY")
        h_in = {k: inp[k].cpu().pin_memory() for k in keys}
        bufs = [buf, ml.alloc_buffers(cfg.T, cfg.m, cfg.n, cfg.E, cfg.k, cfg.r, cfg.scale, device=dev)]
        d_ins = []
        for _ in range(2):
            d_in = dict(inp)
            d_in.update({k: torch.empty_like(inp[k]) for k in keys})
            d_ins.append(d_in)

        def outs_of(b):
            return (b.Y, b.dX, b.dA_gu, b.dB_gu, b.dA_d, b.dB_d)

        h_outs = [[torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs_of(b)] for b in bufs]
        h2d = sum(t.numel() * t.element_size() for t in h_in.values())
        d2h = sum(t.numel() * t.element_size() for t in outs_of(buf))
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of the slot landed
        ev_comp = [torch.cuda.Event() for _ in range(2)]   # the slot's step computed
        ev_out = [torch.cuda.Event() for _ in range(2)]    # the slot's results copied out

        def e2e_step(i):
            sl = i % 2
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_comp[sl])               # step i - 2 is done with these inputs
                for k in keys:
                    d_ins[sl][k].copy_(h_in[k], non_blocking=True)
                ev_in[sl].record(s_in)
            stream.wait_event(ev_in[sl])
            stream.wait_event(ev_out[sl])                  # step i - 2's results are out
            ml.layer_step(d_ins[sl], cfg.k, cfg.scale, bufs[sl])
            dp.allreduce_adapter_grads(outs_of(bufs[sl])[2:])
            ev_comp[sl].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[sl])
                for o, h in zip(outs_of(bufs[sl]), h_outs[sl]):
                    h.copy_(o, non_blocking=True)
                ev_out[sl].record(s_out)

        for i in range(max(1, args.warmup)):
            e2e_step(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_stream(stream)
        for i in range(args.steps):
            e2e_step(i)
        stream.wait_event(ev_out[0])
        stream.wait_event(ev_out[1])
        e1.record(stream)
        torch.cuda.synchronize()
        if ml.moe_get_device_error() != ml.MOE_OK:
            raise SystemExit("device error in the end-to-end timing")
        e_ms = e0.elapsed_time(e1) / args.steps
        if world > 1:
            t = torch.tensor([e_ms], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t.item())
        e2e = {"value": world * cfg.T / (e_ms / 1e3), "unit": UNIT, "ms_per_step": e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipeline": "inputs of step i+1 copied in and results of step i-1 copied out "
                           "while step i computes (two copy streams, double-buffered)"}
        del bufs, d_ins, h_outs

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    # ---- report
    peaks, peak_src = load_peaks()
    for ex in extras.values():
        if "achieved" in ex:
            ex["peak"] = peaks["hbm_gbs"]
            ex["frac"] = ex["achieved"] / peaks["hbm_gbs"]
        if "tflops" in ex:
            ex["frac_bf16_sustained"] = ex["tflops"] / peaks["bf16_tflops_sustained"]
    flops = acc.flops_step(cfg.T, cfg.m, cfg.n, cfg.k, cfg.r)
    tflops = flops / (mean_ms / 1e3) / 1e12
    work = kernel_work(cfg, active_experts)
    total_traced = max(1e-9, sum(v[1] for v in prof_all.values()))
    kernels = {}
    for name, (launches, tot_ms) in prof_all.items():
        ent = {"launches": launches, "ms_per_step": tot_ms / args.steps, "share": tot_ms / total_traced}
        if name in work:
            ent.update(roof_entry(work[name], tot_ms / launches, launches / args.steps, peaks))
        kernels[name] = ent
    roof = None
    if top is not None and top in prof_top and top in work:
        launches, tot_ms = prof_top[top]
        re_ = roof_entry(work[top], tot_ms / launches, launches / args.steps, peaks)
        b = re_["bound"]
        pk = "bf16_tflops_sustained" if b == "tensor" else "hbm_gbs"
        roof = {"kernel": top, "bound": b, "achieved": re_[b]["achieved"], "peak": re_[b]["peak"],
                "unit": re_[b]["unit"], "frac": re_[b]["frac"],
                "peak_source": f"{peak_src} ({pk}, MEASURED_PEAKS.json)",
                "traffic": ncu_traffic(top, cfg.name),
                "algorithmic_per_launch": re_[b]["per_launch"],
                "ms_per_launch": tot_ms / launches,
                "measured_in": "timed region (CUDA events on the launch stream around this kernel only)"}
        other = "hbm" if b == "tensor" else "tensor"
        if other in re_:
            roof["other_resource"] = {"resource": other, "achieved": re_[other]["achieved"],
                                      "unit": re_[other]["unit"], "frac": re_[other]["frac"]}
    launches_total = int(round(launches_per_step * args.steps))
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu_inp = {k: v.cpu() for k, v in inp.items()}
        cpu = cpu_baseline(cfg, cpu_inp, args.cpu_sample_tokens)
    line = {
        "metric": METRIC, "value": world * cfg.T / (mean_ms / 1e3), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; layer shapes of the named model family, random weights)",
        "config": {"workload": workload_name(cfg), "tokens_per_rank": cfg.T,
                   "global_tokens": world * cfg.T, "parallelism": f"dp{world}",
                   "l2": "flushed before every timed step (256 MiB write outside the step events)",
                   "lora_scale": cfg.scale},
        "tflops": tflops,
        "pct_bf16_peak": {"burst": tflops / peaks["bf16_tflops"],
                          "sustained": tflops / peaks["bf16_tflops_sustained"],
                          "source": peak_src},
        "algorithmic_flop_per_step": flops,
        "roofline": roof,
        "kernels": kernels,
        "kernels_source": ("separate traced pass of the same steps (every launch bracketed by CUDA events"
                           + (", host launches)" if args.no_graph else ", graph replay)")),
        "launch": "host launches" if args.no_graph else "one CUDA graph replay per timed step",
        "gpu_launches": launches_total,
        "step_ms_min_max": [min(step_ms), max(step_ms)],
        "step_ms_median": median_ms,
        "active_experts": active_experts,
        "clocks": clk,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "extras": extras,
    }
    print(json.dumps(line), flush=True)


def run_plain(args, cfg):
    """W + K steps of the layer through the public API, nothing else."""
    import mixture_experts_lora_b200 as ml
    torch.cuda.set_device(0)
    inp = generate(cfg, seed=0, device="cuda")
    buf = ml.alloc_buffers(cfg.T, cfg.m, cfg.n, cfg.E, cfg.k, cfg.r, cfg.scale)
    for _ in range(args.warmup + args.steps):
        ml.layer_step(inp, cfg.k, cfg.scale, buf)
    torch.cuda.synchronize()
    st = ml.moe_get_device_error()
    if st != ml.MOE_OK:
        raise SystemExit(f"device error: {ml.status_string(st)}")


def main():
    args = parse_args()
    cfg = CONFIGS[args.config]
    if args.plain:
        run_plain(args, cfg)
    elif args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
