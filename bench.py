"""Benchmark of the routed Q2_K MoE layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Default: the headline workload is the single-token decode (H=4096, 256 experts, top-8,
I=2048), the configuration the headline metric is quoted on; the same JSON line carries a
``per_config`` object with the other three workloads measured the same way (16-token
decode, 2048-token prefill, and the 4-layer 8192-token chain with fewer steps).
``--workload NAME`` measures that workload alone as the headline.

One step = one forward of the layer over one batch of synthetic input (decode: T tokens;
prefill workloads: the whole token batch through every chained layer with the RMS
renormalisation between layers), a different batch every step (so the routed experts
change), with the L2 cache flushed between timed steps (a 256 MiB buffer is written, then
read).  Inputs are resident in HBM when the timed region starts; each step is timed with
CUDA events on the launching stream and the step times are summed.  Under torchrun every
rank runs its own replica on its own token stream (weak scaling, no data-path collective);
the job time is the max over ranks.

Printed (rank 0, one JSON line): tokens/s of the whole job, ms per step, an end-to-end
figure through ds4moe_forward_host (host buffers, copies inside the timed region), the
roofline of the dominant kernel (from a second, profiled pass with events around each
kernel), the SM clocks sampled during the timed region, and the fp64 oracle timed on the
host cores on a bounded sample (rank 0, N=1).  ``--impl reference`` times the oracle alone
on the same workload and metric.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "decode_t1_h4096_e256_k8"
OTHER_CONFIGS = ["decode_t16_h4096_e256_k8", "prefill_t2048_h4096_e256_k8_bias", "prefill4_t8192_h7168_e256_k8_zipf"]
PREFILL_STAGES = ["route", "gather_tiles", "gemm1", "gemm2", "combine"]
PREFILL_LAUNCHES_PER_LAYER = 9   # router GEMM, top-k, scatter, gather, 2 tile lists, 2 GEMMs, combine
DECODE_STAGES = ["decode"]       # one launch: routing and the whole layer
METRIC = "routed-MoE layer tokens/s; decode expert-weight HBM GB/s as % of B200 peak"
UNIT = "tokens/s"
FLUSH_BYTES = 256 << 20
TOKEN_POOL = 512
PROFILES = os.path.join(ROOT, "profiles")


def flush_l2(buf, i):
    """Write then read a buffer twice the size of L2: the next step starts with a cold L2
    that holds no dirty lines of ours or of the flush (its write-backs finish here)."""
    buf.fill_(float(i))
    return buf.sum()


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


def ncu_traffic(kernel: str, scale: float = 1.0):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, when it was taken on
    the kernel's current sources (null otherwise); `scale` converts a capture of a smaller
    case to the measured one (traffic grows with the units processed)."""
    p = os.path.join(PROFILES, "traffic.json")
    if not os.path.exists(p):
        return None
    k = json.load(open(p)).get("kernels", {}).get(kernel)
    if k is None or k.get("source_hash") != kernel_source_hash(k.get("files", [])):
        return None
    return k.get("dram_bytes_per_launch") * scale


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.device = device
        self.proc = None
        fd, self.path = tempfile.mkstemp(prefix="ds4moe_clocks_%d_" % device, suffix=".csv")
        os.close(fd)

    def start(self):
        try:
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
        try:
            os.unlink(self.path)
        except OSError:
            pass
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


def algorithmic_bytes(cfg, n_active: int) -> int:
    """Unique bytes one decode launch must move: the router weights and the tokens, the
    active experts' Q2_K gate/up/down, the shared expert's bf16 weights, and the output."""
    H, E, I, Is, T = cfg["hidden"], cfg["n_experts"], cfg["inter"], cfg["shared_inter"], cfg["T"]
    q2k = I * H // 256 * 84
    return E * H * 2 + T * H * 2 + n_active * 3 * q2k + 3 * Is * H * 2 + T * H * 4


def prefill_flops(cfg, pairs: int):
    """Algorithmic FLOPs of the grouped path's stages for one layer (padding, dequant and
    gather not counted): router 2*T*E*H; GEMM1 (gate and up) 4*pairs*H*I + 4*T*H*I_s; GEMM2
    (down) 2*pairs*H*I + 2*T*H*I_s."""
    H, E, I, Is, T = cfg["hidden"], cfg["n_experts"], cfg["inter"], cfg["shared_inter"], cfg["T"]
    return {"route": 2 * T * E * H, "gather_tiles": 0, "gemm1": 4 * pairs * H * I + 4 * T * H * Is,
            "gemm2": 2 * pairs * H * I + 2 * T * H * Is, "combine": 0}


def cpu_baseline(lws, w, x, budget_s: float):
    """Oracle tokens/s of a workload, from the time of single tokens through the first
    layer, extrapolated to all chained layers (the oracle's cost is per token and per layer;
    routing of one token is part of it)."""
    import oracle
    ora = oracle.oracle()
    n = 0
    t0 = time.perf_counter()
    while True:
        ora.layer_forward(lws[0], x[n % len(x)][None, :], w.top_k)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= len(x):
            break
    per_token = el / n * len(lws)
    sample = "%d single tokens of the same workload (fp64 C oracle, one thread)" % n
    if len(lws) > 1:
        sample += ", through layer 1, extrapolated to %d layers" % len(lws)
    return {"value": 1.0 / per_token, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample}


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


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


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


_LAYER_CACHE = {}


def layer_weights(w, l=0):
    """Seeded layer weights; workloads that share a layer seed share the arrays."""
    import synth
    key = (w.hidden, w.n_experts, w.top_k, w.inter, w.shared_inter, w.router_sigma, w.bias, w.bias_sigma, w.zipf_s,
           w.layer_seeds[l], w.shared_sigma)
    if key not in _LAYER_CACHE:
        _LAYER_CACHE[key] = synth.make_layer(w, l)
    return _LAYER_CACHE[key]


def run_decode(name, steps, warmup, ws, rank, local, cpu_budget):
    """T <= 32 workloads: the batched-GEMV path, one launch per step."""
    import torch
    import bit_quantized_routed_sqrt_b200 as ds4
    import synth

    w = synth.workload(name)
    lw = layer_weights(w)
    layer = ds4.Ds4Moe(w.hidden, w.n_experts, w.top_k, w.inter, w.shared_inter, max_tokens=w.tokens)
    layer.load(lw)
    prof = ds4.Ds4Moe(w.hidden, w.n_experts, w.top_k, w.inter, w.shared_inter, max_tokens=w.tokens,
                      flags=ds4.FLAG_PROFILE)
    prof.load(lw)
    T = w.tokens
    n_pool = max(2, TOKEN_POOL // T)   # batches of T tokens, a different one every step
    x_np = synth.make_tokens(w, tokens=n_pool * T, stream=1 + rank)
    x_dev = torch.from_numpy(x_np.view(np.int16)).cuda()
    y_dev = torch.empty((T, w.hidden), dtype=torch.float32, device="cuda")
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def xs(i):
        j = i % n_pool
        return x_dev[j * T:(j + 1) * T]

    for i in range(warmup):
        layer.ds4moe_forward(xs(i), T, y_dev)
    torch.cuda.synchronize()
    layer.ds4moe_sync_status()

    # ---- timed region: device-resident inputs
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    for i in range(steps):
        flush_l2(flush, i)
        starts[i].record(stream)
        layer.ds4moe_forward(xs(warmup + i), T, y_dev)
        ends[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    layer.ds4moe_sync_status()
    total_max = job_time_ms(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), "cuda")
    value = job_value(T, steps, ws, total_max)

    # ---- end to end through ds4moe_forward_host (pinned host buffers)
    x_host = torch.from_numpy(x_np.view(np.int16)).pin_memory()
    y_host = torch.empty((T, w.hidden), dtype=torch.float32).pin_memory()
    e2e_steps = steps
    e_st = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    e_en = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    for i in range(3):
        layer.ds4moe_forward_host(x_host[i * T:(i + 1) * T], T, y_host)
    for i in range(e2e_steps):
        flush_l2(flush, i)
        e_st[i].record(stream)
        j = (warmup + i) % n_pool
        layer.ds4moe_forward_host(x_host[j * T:(j + 1) * T], T, y_host)
        e_en[i].record(stream)
    torch.cuda.synchronize()
    e2e_value = job_value(T, e2e_steps, ws, job_time_ms(sum(s.elapsed_time(e) for s, e in zip(e_st, e_en)), "cuda"))

    # ---- profiled pass: the kernel's device time (events around the launch)
    prof_steps = steps
    kern_ms, act_sum, byt_sum = 0.0, 0, 0
    cfg = dict(hidden=w.hidden, n_experts=w.n_experts, inter=w.inter, shared_inter=w.shared_inter, T=T,
               top_k=w.top_k)
    for i in range(prof_steps):
        flush_l2(flush, i)
        xi = xs(warmup + i)
        prof.ds4moe_forward(xi, T, y_dev)
        st = prof.ds4moe_get_stats()
        kern_ms += st.stage_ms[0]
        idx, *_ = prof.route(xi)
        n_act = int(torch.unique(idx).numel())
        act_sum += n_act
        byt_sum += algorithmic_bytes(cfg, n_act)
    kern_avg = kern_ms / prof_steps
    hbm_gbs, bf16_tf, peak_kind = peaks()
    achieved = byt_sum / prof_steps / (kern_avg * 1e-3) / 1e9
    roofline = {"bound": "hbm", "kernel": "decode_kernel", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                "frac": achieved / hbm_gbs, "peak_kind": peak_kind + " (burst copy bandwidth)",
                "traffic": ncu_traffic("decode_kernel_" + name),
                "algorithmic_bytes_per_launch": byt_sum / prof_steps,
                "kernel_ms": kern_avg,
                "step_frac_of_peak": byt_sum / prof_steps / (total_max / steps * 1e-3) / 1e9 / hbm_gbs,
                "avg_active_experts": act_sum / prof_steps,
                "measured": "profiled pass of %d steps, CUDA events around the launch on the launching stream"
                            % prof_steps}
    cpu = None
    if rank == 0 and ws == 1 and cpu_budget > 0:
        cpu = cpu_baseline([lw], w, x_np[:64], cpu_budget)
    layer.close()
    prof.close()
    del x_dev, flush
    return {"value": value, "ms_per_step": total_max / steps, "steps": steps, "warmup": warmup,
            "dtype": "q2k-int16/f32",
            "config": {"workload": w.name, "tokens_per_step": T, "hidden": w.hidden, "n_experts": w.n_experts,
                       "top_k": w.top_k, "inter": w.inter, "shared_inter": w.shared_inter,
                       "l2": "flushed between timed steps (256 MiB written, then read)"},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": T * w.hidden * 2,
                    "d2h_bytes_per_step": T * w.hidden * 4, "steps": e2e_steps},
            "gpu_launches": len(DECODE_STAGES) * steps,
            "roofline": roofline, "cpu_baseline": cpu, "clocks": clk}


def run_prefill(name, steps, warmup, ws, rank, local, cpu_budget):
    """Multi-token workloads: the grouped tensor-core path, every chained layer per step."""
    import torch
    import bit_quantized_routed_sqrt_b200 as ds4
    import synth

    w = synth.workload(name)
    T, H, L = w.tokens, w.hidden, w.layers
    lws = [layer_weights(w, l) for l in range(L)]
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

    for i in range(warmup):
        step(batch(i))
    torch.cuda.synchronize()
    for h in layers:
        h.ds4moe_sync_status()

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    for i in range(steps):
        flush_l2(flush, i)
        starts[i].record(stream)
        step(batch(warmup + i))
        ends[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    for h in layers:
        h.ds4moe_sync_status()
    total_max = job_time_ms(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), "cuda")
    value = job_value(T, steps, ws, total_max)

    # ---- end to end: pinned host tokens in, host output back, every step
    x_host = torch.from_numpy(x_np.view(np.int16)).pin_memory()
    y_host = torch.empty((T, H), dtype=torch.float32).pin_memory()
    e2e_steps = steps
    x_in = torch.empty((T, H), dtype=torch.int16, device="cuda")
    e_st = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    e_en = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    for i in range(e2e_steps):
        flush_l2(flush, i)
        j = (warmup + i) % n_batches
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
    prof_steps = steps
    cfg = dict(hidden=H, n_experts=w.n_experts, inter=w.inter, shared_inter=w.shared_inter, T=T)
    stage_sum = [0.0] * len(PREFILL_STAGES)
    for i in range(prof_steps):
        flush_l2(flush, i)
        prof.ds4moe_forward(batch(warmup + i), T, y_dev)
        st = prof.ds4moe_get_stats()
        for s_ in range(len(PREFILL_STAGES)):
            stage_sum[s_] += st.stage_ms[s_]
    stage_avg = [v / prof_steps for v in stage_sum]
    fl = prefill_flops(cfg, T * w.top_k)
    hbm_gbs, bf16_tf, peak_kind = peaks()
    kname = "gemm1"
    achieved = fl[kname] / (stage_avg[PREFILL_STAGES.index(kname)] * 1e-3) / 1e12
    layer_flops = sum(fl.values())
    roofline = {"bound": "tensor", "kernel": "pf_gemm_kernel<1>", "achieved": achieved, "peak": bf16_tf,
                "unit": "TFLOP/s", "frac": achieved / bf16_tf,
                "peak_kind": peak_kind + " (bf16 dense burst; fp16 dense has the same nominal rate)",
                "traffic": ncu_traffic("pf_gemm1_" + name),
                "algorithmic_flops_per_launch": fl[kname],
                "stage_ms": dict(zip(PREFILL_STAGES, stage_avg)),
                "stage_share": dict(zip(PREFILL_STAGES, [v / sum(stage_avg) for v in stage_avg])),
                "step_algorithmic_flops": layer_flops * L,
                "step_frac_of_peak": layer_flops * L / (total_max / steps * 1e-3) / 1e12 / bf16_tf,
                "measured": "profiled pass of %d steps on layer 1, CUDA events between the launches on the "
                            "launching stream" % prof_steps}
    cpu = None
    if rank == 0 and ws == 1 and cpu_budget > 0:
        cpu = cpu_baseline(lws, w, x_np[:64], cpu_budget)
    for h in layers:
        h.close()
    prof.close()
    del x_dev, flush, xb
    return {"value": value, "ms_per_step": total_max / steps, "steps": steps, "warmup": warmup,
            "dtype": "q2k->f16 MMA/f32 accumulate",
            "config": {"workload": w.name, "tokens_per_step": T, "layers": L, "hidden": H, "n_experts": w.n_experts,
                       "top_k": w.top_k, "inter": w.inter, "shared_inter": w.shared_inter,
                       "l2": "flushed between timed steps (256 MiB written, then read)"},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * H * 4,
                    "steps": e2e_steps},
            "gpu_launches": (PREFILL_LAUNCHES_PER_LAYER * L + (L - 1)) * steps,
            "roofline": roofline, "cpu_baseline": cpu, "clocks": clk}


def run_config(name, steps, warmup, ws, rank, local, cpu_budget):
    import synth
    fn = run_prefill if synth.workload(name).tokens > 32 else run_decode
    return fn(name, steps, warmup, ws, rank, local, cpu_budget)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=None,
                    choices=[WORKLOAD] + OTHER_CONFIGS)
    args = ap.parse_args()
    if args.impl == "reference":
        args.workload = args.workload or WORKLOAD
        return run_reference(args)
    args.warmup = max(args.warmup, 3)

    import torch
    import torch.distributed as dist

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))

    cpu = 0.0 if args.no_cpu_baseline else 12.0
    head_name = args.workload or WORKLOAD
    head = run_config(head_name, args.steps, args.warmup, ws, rank, local, cpu)
    per_config = None
    if args.workload is None:
        per_config = {}
        for name in OTHER_CONFIGS:
            # the 4-layer chain holds 14.8 GB of weights and runs ~50 ms per step: fewer steps
            steps = min(args.steps, 10) if name.startswith("prefill4") else args.steps
            per_config[name] = run_config(name, steps, args.warmup, ws, rank, local, 0.0 if args.no_cpu_baseline else 4.0)
            _LAYER_CACHE.clear()
    if rank == 0:
        line = {"metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": ws, "steps": head["steps"],
                "warmup": head["warmup"], "ms_per_step": head["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": head["dtype"],
                "data": "synthetic (seeded Q2_K experts, bf16 router/shared, N(0,1) tokens)",
                "config": dict(head["config"], parallelism="replicas" if ws > 1 else "single"),
                "e2e": head["e2e"], "gpu_launches": head["gpu_launches"], "roofline": head["roofline"],
                "cpu_baseline": head["cpu_baseline"], "clocks": head["clocks"]}
        if per_config is not None:
            line["per_config"] = per_config
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
