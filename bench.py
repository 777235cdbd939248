"""Benchmark of the routed Q2_K MoE layer.  Default workload: single-token decode, H=4096,
256 experts, top-8 (the configuration the headline metric is quoted on).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one forward of the layer over one batch of synthetic input (decode: one token;
prefill workloads: the whole token batch, through every chained layer with the RMS
renormalisation between layers), a different batch every step (so the routed experts
change), with the L2 cache flushed between timed steps (a 256 MiB buffer is written).  Inputs are resident in HBM when the
timed region starts; each step is timed with CUDA events on the launching stream and
the step times are summed.  Under torchrun every rank runs its own replica on its own
token stream (weak scaling, no data-path collective); the job time is the max over ranks.

Printed (rank 0, one JSON line): tokens/s of the whole job, ms per step, an end-to-end
figure through ds4moe_forward_host (host buffers, copies inside the timed region), the
roofline of the dominant kernel (from a second, profiled pass with events around each
kernel), the SM clocks sampled during the timed region, and the fp64 oracle timed on the
host cores on a bounded sample (rank 0, N=1).  ``--impl reference`` times the oracle
alone on the same workload and metric.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "decode_t1_h4096_e256_k8"
PREFILL_STAGES = ["route", "gather_tiles", "gemm1", "gemm2", "combine"]
PREFILL_LAUNCHES_PER_LAYER = 9   # router GEMM, top-k, scatter, gather, 2 tile lists, 2 GEMMs, combine
METRIC = "routed-MoE layer tokens/s; decode expert-weight HBM GB/s as % of B200 peak"
UNIT = "tokens/s"
FLUSH_BYTES = 256 << 20


def flush_l2(buf, i):
    """Write then read a buffer twice the size of L2: the next step starts with a cold L2
    that holds no dirty lines of ours or of the flush (its write-backs finish here)."""
    buf.fill_(float(i))
    return buf.sum()
TOKEN_POOL = 512
PROFILES = os.path.join(ROOT, "profiles")
STAGES = ["decode_route", "decode_stream"]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d.get("bf16_tflops"), "measured"
    return 6650.0, 1590.0, "fallback"


def kernel_source_hash(files) -> str:
    """Hash of the CUDA sources a kernel is built from (files under the package's csrc/)."""
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "bit_quantized_routed_sqrt_b200", "csrc")
    for f in files:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, when it was taken on
    the kernel's current sources (null otherwise)."""
    p = os.path.join(PROFILES, "traffic.json")
    if not os.path.exists(p):
        return None
    k = json.load(open(p)).get("kernels", {}).get(kernel)
    if k is None or k.get("source_hash") != kernel_source_hash(k.get("files", [])):
        return None
    return k.get("dram_bytes_per_launch")


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.device = device
        self.proc = None
        self.path = os.path.join(ROOT, "gpurun_out", "clocks_rank%d.csv" % device)

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.device), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = [l.split(",") for l in open(self.path).read().strip().splitlines() if l.strip()]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1])); mx.append(float(r[2]))
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def algorithmic_bytes(cfg, n_active: int):
    """Unique bytes each launch of one decode step must move: the routing launch reads the
    router weights and the tokens; the streaming launch reads the active experts' Q2_K
    gate/up/down and the shared expert's bf16 weights and writes the output."""
    H, E, I, Is, T, k = cfg["hidden"], cfg["n_experts"], cfg["inter"], cfg["shared_inter"], cfg["T"], cfg["top_k"]
    q2k = I * H // 256 * 84
    route = E * H * 2 + T * H * 2
    stream = n_active * 3 * q2k + 3 * Is * H * 2 + T * H * 2 + T * H * 4
    return {"decode_route": route, "decode_stream": stream}


def prefill_flops(cfg, pairs: int):
    """Algorithmic FLOPs of the grouped path's stages for one layer (padding, dequant and
    gather not counted): router 2*T*E*H; GEMM1 (gate and up) 4*pairs*H*I + 4*T*H*I_s; GEMM2
    (down) 2*pairs*H*I + 2*T*H*I_s."""
    H, E, I, Is, T = cfg["hidden"], cfg["n_experts"], cfg["inter"], cfg["shared_inter"], cfg["T"]
    return {"route": 2 * T * E * H, "gather_tiles": 0, "gemm1": 4 * pairs * H * I + 4 * T * H * Is,
            "gemm2": 2 * pairs * H * I + 2 * T * H * Is, "combine": 0}


def cpu_baseline(lw, w, x_pool, budget_s: float = 12.0):
    import oracle
    ora = oracle.oracle()
    n = 0
    t0 = time.perf_counter()
    while True:
        ora.layer_forward(lw, x_pool[n % len(x_pool)][None, :], w.top_k)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= len(x_pool):
            break
    # one token per oracle call: the oracle's cost is per token
    return {"value": n / el, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": "%d single tokens of the same workload (fp64 C oracle, one thread)" % n}


def cpu_baseline_prefill(lws, w, x, budget_s: float = 12.0):
    """Oracle tokens/s of a multi-token workload, from the time of single tokens through the
    first layer, extrapolated to all chained layers (the oracle's cost is per token and per
    layer; routing of one token is part of it)."""
    import oracle
    ora = oracle.oracle()
    n = 0
    t0 = time.perf_counter()
    while True:
        ora.layer_forward(lws[0], x[n:n + 1], w.top_k)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= len(x):
            break
    per_token = el / n * len(lws)
    return {"value": 1.0 / per_token, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": "%d tokens of the workload through layer 1 (fp64 C oracle, one thread), extrapolated to "
                      "%d layer(s)" % (n, len(lws))}


def job_time_ms(local_ms: float, device) -> float:
    """The job's time: the maximum over ranks of each rank's device time (every rank takes
    part; a single process returns its own time)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(tokens_per_step: int, steps: int, world: int, job_ms: float) -> float:
    """Whole-job tokens/s: every rank processes its own batch each step (weak scaling)."""
    return world * tokens_per_step * steps / (job_ms / 1e3)


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def run_reference(args):
    """The fp64 oracle on the same workload and metric, time-capped (rank 0 only)."""
    ws, rank, local = dist_env()
    if rank != 0:
        return
    import synth
    w = synth.workload(args.workload)
    lws = [synth.make_layer(w, l) for l in range(w.layers)]
    x_pool = synth.make_tokens(w, tokens=max(4, min(args.steps + args.warmup, 64)))
    import oracle
    ora = oracle.oracle()
    for i in range(min(args.warmup, 1)):
        ora.layer_forward(lws[0], x_pool[i][None, :], w.top_k)
    times = []
    cap = 90.0
    t_all = time.perf_counter()
    for s in range(args.steps):
        # one sampled token through every layer (a decode step is exactly one token)
        t0 = time.perf_counter()
        for lw in lws:
            ora.layer_forward(lw, x_pool[s % len(x_pool)][None, :], w.top_k)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_all > cap:
            break
    tot = sum(times)
    value = len(times) / tot
    if w.tokens == 1:
        sample = "%d of %d steps (time cap %.0f s), one token per step, fp64 C oracle on one host core" % (
            len(times), args.steps, cap)
    else:
        sample = ("%d sampled tokens of the %d-token batch (time cap %.0f s), each through all %d layer(s); "
                  "fp64 C oracle on one host core; tokens/s of the batch extrapolated from the sample" % (
                      len(times), w.tokens, cap, w.layers))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": len(times), "warmup": min(args.warmup, 1), "ms_per_step": 1e3 * tot / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, "tokens_per_step": w.tokens, "hidden": w.hidden,
                                           "n_experts": w.n_experts, "top_k": w.top_k, "inter": w.inter,
                                           "shared_inter": w.shared_inter, "parallelism": "replicas"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_prefill(args):
    """Multi-token workloads: the grouped tensor-core path, every chained layer per step."""
    import torch
    import torch.distributed as dist

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))

    import bit_quantized_routed_sqrt_b200 as ds4
    import synth

    w = synth.workload(args.workload)
    T, H, L = w.tokens, w.hidden, w.layers
    lws = [synth.make_layer(w, l) for l in range(L)]
    layers = []
    for lw in lws:
        h = ds4.Ds4Moe(H, w.n_experts, w.top_k, w.inter, w.shared_inter, max_tokens=T)
        h.load(lw)
        layers.append(h)
    prof = ds4.Ds4Moe(H, w.n_experts, w.top_k, w.inter, w.shared_inter, max_tokens=T, flags=ds4.FLAG_PROFILE)
    prof.load(lws[0])
    n_batches = 2
    x_np = synth.make_tokens(w, tokens=T * n_batches, stream=1 + rank)
    x_dev = torch.from_numpy(x_np.view(np.int16)).cuda()
    y_dev = torch.empty((T, H), dtype=torch.float32, device="cuda")
    xb = torch.empty((T, H), dtype=torch.int16, device="cuda")   # bf16 input of the next layer
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def batch(i):
        j = i % n_batches
        return x_dev[j * T:(j + 1) * T]

    def step(x):
        for l, h in enumerate(layers):
            h.ds4moe_forward(x, T, y_dev)
            if l + 1 < L:
                ds4.ds4moe_rms_renorm(y_dev, T, H, xb)
                x = xb

    for i in range(args.warmup):
        step(batch(i))
    torch.cuda.synchronize()
    for h in layers:
        h.ds4moe_sync_status()

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for i in range(args.steps):
        flush_l2(flush, i)
        starts[i].record(stream)
        step(batch(args.warmup + i))
        ends[i].record(stream)
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    clk = clocks.stop()
    for h in layers:
        h.ds4moe_sync_status()
    total_max = job_time_ms(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), "cuda")
    value = job_value(T, args.steps, ws, total_max)

    # ---- end to end: pinned host tokens in, host output back, every step
    x_host = torch.from_numpy(x_np.view(np.int16)).pin_memory()
    y_host = torch.empty((T, H), dtype=torch.float32).pin_memory()
    e2e_steps = min(args.steps, 20)
    x_in = torch.empty((T, H), dtype=torch.int16, device="cuda")
    e_st = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    e_en = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    for i in range(e2e_steps):
        flush_l2(flush, i)
        j = (args.warmup + i) % n_batches
        e_st[i].record(stream)
        if L == 1:
            layers[0].ds4moe_forward_host(x_host[j * T:(j + 1) * T], T, y_host)
        else:
            x_in.copy_(x_host[j * T:(j + 1) * T], non_blocking=True)
            step(x_in)
            y_host.copy_(y_dev, non_blocking=True)
        e_en[i].record(stream)
    torch.cuda.synchronize()
    e2e_value = job_value(T, e2e_steps, ws, job_time_ms(sum(s.elapsed_time(e) for s, e in zip(e_st, e_en)), "cuda"))

    # ---- profiled pass on layer 1: per-stage device time (events between the launches)
    prof_steps = min(args.steps, 20)
    cfg = dict(hidden=H, n_experts=w.n_experts, inter=w.inter, shared_inter=w.shared_inter, T=T)
    stage_sum = [0.0] * len(PREFILL_STAGES)
    for i in range(prof_steps):
        flush_l2(flush, i)
        prof.ds4moe_forward(batch(args.warmup + i), T, y_dev)
        st = prof.ds4moe_get_stats()
        for s_ in range(len(PREFILL_STAGES)):
            stage_sum[s_] += st.stage_ms[s_]
    stage_avg = [v / prof_steps for v in stage_sum]
    fl = prefill_flops(cfg, T * w.top_k)
    hbm_gbs, bf16_tf, peak_kind = peaks()
    kname = "gemm1"
    achieved = fl[kname] / (stage_avg[PREFILL_STAGES.index(kname)] * 1e-3) / 1e12
    layer_flops = sum(fl.values())
    roofline = {"bound": "tensor", "kernel": kname, "achieved": achieved, "peak": bf16_tf, "unit": "TFLOP/s",
                "frac": achieved / bf16_tf, "peak_kind": peak_kind + " (bf16 dense burst; fp16 dense has the same "
                                                                  "nominal rate)",
                "traffic": ncu_traffic("pf_gemm1"),
                "algorithmic_flops_per_launch": fl[kname],
                "stage_ms": dict(zip(PREFILL_STAGES, stage_avg)),
                "stage_share": dict(zip(PREFILL_STAGES, [v / sum(stage_avg) for v in stage_avg])),
                "step_algorithmic_flops": layer_flops * L,
                "step_frac_of_peak": layer_flops * L / (total_max / args.steps * 1e-3) / 1e12 / bf16_tf,
                "measured": "profiled pass of %d steps on layer 1, CUDA events between the launches on the "
                            "launching stream" % prof_steps}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_prefill(lws, w, x_np[:64])

    if ws > 1:
        dist.barrier()
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": total_max / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "q2k->f16 MMA/f32 accumulate",
                "data": "synthetic (seeded Q2_K experts, bf16 router/shared, N(0,1) tokens)",
                "config": {"workload": w.name, "tokens_per_step": T, "layers": L, "hidden": H,
                           "n_experts": w.n_experts, "top_k": w.top_k, "inter": w.inter,
                           "shared_inter": w.shared_inter, "parallelism": "replicas" if ws > 1 else "single",
                           "l2": "flushed between timed steps (256 MiB written, then read)"},
                "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": T * H * 2,
                        "d2h_bytes_per_step": T * H * 4, "steps": e2e_steps},
                "gpu_launches": (PREFILL_LAUNCHES_PER_LAYER * L + (L - 1)) * args.steps,
                "roofline": roofline, "cpu_baseline": cpu, "clocks": clk}
        print(json.dumps(line), flush=True)
    for h in layers:
        h.close()
    prof.close()
    if ws > 1:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=["decode_t1_h4096_e256_k8", "decode_t16_h4096_e256_k8",
                             "prefill_t2048_h4096_e256_k8_bias", "prefill4_t8192_h7168_e256_k8_zipf"])
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    args.warmup = max(args.warmup, 3)
    import synth
    if synth.workload(args.workload).tokens > 32:
        return run_prefill(args)

    import torch
    import torch.distributed as dist

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))

    import bit_quantized_routed_sqrt_b200 as ds4
    import synth

    w = synth.workload(args.workload)
    lw = synth.make_layer(w)
    layer = ds4.Ds4Moe(w.hidden, w.n_experts, w.top_k, w.inter, w.shared_inter, max_tokens=w.tokens)
    layer.load(lw)
    prof = ds4.Ds4Moe(w.hidden, w.n_experts, w.top_k, w.inter, w.shared_inter, max_tokens=w.tokens,
                      flags=ds4.FLAG_PROFILE)
    prof.load(lw)
    T = w.tokens
    n_pool = max(2, TOKEN_POOL // T)   # batches of T tokens, a different one every step
    x_np = synth.make_tokens(w, tokens=n_pool * T, stream=1 + rank)
    x_dev = torch.from_numpy(x_np.view(np.int16)).cuda()
    y_dev = torch.empty((w.tokens, w.hidden), dtype=torch.float32, device="cuda")
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def xs(i):
        j = i % n_pool
        return x_dev[j * T:(j + 1) * T]

    for i in range(args.warmup):
        layer.forward(xs(i), y_dev)
    torch.cuda.synchronize()
    layer.ds4moe_sync_status()

    # ---- timed region: device-resident inputs
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for i in range(args.steps):
        flush_l2(flush, i)
        starts[i].record(stream)
        layer.ds4moe_forward(xs(args.warmup + i), T, y_dev)
        ends[i].record(stream)
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    clk = clocks.stop()
    layer.ds4moe_sync_status()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_max = job_time_ms(sum(step_ms), "cuda")
    value = job_value(T, args.steps, ws, total_max)

    # ---- end to end through ds4moe_forward_host (pinned host buffers)
    x_host = torch.from_numpy(x_np.view(np.int16)).pin_memory()
    y_host = torch.empty((T, w.hidden), dtype=torch.float32).pin_memory()
    e2e_steps = min(args.steps, 500)
    e_st = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    e_en = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    for i in range(3):
        layer.ds4moe_forward_host(x_host[i * T:(i + 1) * T], T, y_host)
    for i in range(e2e_steps):
        flush_l2(flush, i)
        e_st[i].record(stream)
        j = (args.warmup + i) % n_pool
        layer.ds4moe_forward_host(x_host[j * T:(j + 1) * T], T, y_host)
        e_en[i].record(stream)
    torch.cuda.synchronize()
    e2e_value = job_value(T, e2e_steps, ws, job_time_ms(sum(s.elapsed_time(e) for s, e in zip(e_st, e_en)), "cuda"))

    # ---- profiled pass: per-kernel device time (events between the kernels)
    prof_steps = min(args.steps, 400)
    stage_sum = [0.0] * len(STAGES)
    act_sum = 0
    cfg = dict(hidden=w.hidden, n_experts=w.n_experts, inter=w.inter, shared_inter=w.shared_inter, T=T,
               top_k=w.top_k)
    byt_sum = {k: 0 for k in STAGES}
    for i in range(prof_steps):
        flush_l2(flush, i)
        xi = xs(args.warmup + i)
        prof.ds4moe_forward(xi, T, y_dev)
        st = prof.ds4moe_get_stats()
        for s in range(len(STAGES)):
            stage_sum[s] += st.stage_ms[s]
        idx, *_ = prof.route(xi)
        n_act = int(torch.unique(idx).numel())
        act_sum += n_act
        for kname, b in algorithmic_bytes(cfg, n_act).items():
            byt_sum[kname] += b
    stage_avg = [s / prof_steps for s in stage_sum]
    dom = int(np.argmax(stage_avg))
    kname = STAGES[dom]
    hbm_gbs, bf16_tf, peak_kind = peaks()
    achieved = byt_sum[kname] / prof_steps / (stage_avg[dom] * 1e-3) / 1e9
    step_bytes = sum(byt_sum.values()) / prof_steps
    roofline = {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                "frac": achieved / hbm_gbs, "peak_kind": peak_kind, "traffic": ncu_traffic(kname),
                "algorithmic_bytes_per_launch": byt_sum[kname] / prof_steps,
                "stage_ms": dict(zip(STAGES, stage_avg)),
                "stage_share": dict(zip(STAGES, [s / sum(stage_avg) for s in stage_avg])),
                "step_algorithmic_bytes": step_bytes,
                "step_frac_of_peak": step_bytes / (total_max / args.steps * 1e-3) / 1e9 / hbm_gbs,
                "avg_active_experts": act_sum / prof_steps,
                "measured": "profiled pass of %d steps, CUDA events between the kernels on the launching stream"
                            % prof_steps}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(lw, w, x_np[:64])

    if ws > 1:
        dist.barrier()
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": total_max / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "q2k-int16/f32",
                "data": "synthetic (seeded Q2_K experts, bf16 router/shared, N(0,1) tokens)",
                "config": {"workload": w.name, "tokens_per_step": T, "hidden": w.hidden,
                           "n_experts": w.n_experts, "top_k": w.top_k, "inter": w.inter,
                           "shared_inter": w.shared_inter, "parallelism": "replicas" if ws > 1 else "single",
                           "l2": "flushed between timed steps (256 MiB written, then read)"},
                "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": T * w.hidden * 2,
                        "d2h_bytes_per_step": T * w.hidden * 4, "steps": e2e_steps},
                "gpu_launches": len(STAGES) * args.steps,
                "roofline": roofline, "cpu_baseline": cpu, "clocks": clk}
        print(json.dumps(line), flush=True)
    layer.close()
    prof.close()
    if ws > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
