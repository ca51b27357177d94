#!/usr/bin/env python
"""HSTU layer forward throughput on one or more B200s (one process per GPU).

Default workload: the long-sequence configuration -- 2 HSTU layers, bf16,
d_model 512, 8 heads x 64, 8 users x 8192 tokens, log-normal timestamp gaps,
8192 position / 128 time buckets.  A step is one full forward pass (f1 ->
attention -> f2 per layer, both layers) over that batch.  With --gpus N each
rank runs its own batch of that shape (users are independent, so the batch
shards with no collective: weak scaling).

Prints one JSON line (rank 0).  `value` is whole-job tokens/s with inputs
resident in HBM; `e2e` is the same metric through the public API with the
inputs copied from pinned host memory and the output copied back inside the
timed region.  At N = 1 the line also carries `workloads`: the other
configurations (tiny fp32, small bf16, Stochastic Length, M-FALCON scoring)
timed the same way, each with its own roofline.  `--impl reference` times the
float64 CPU oracle instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HSTU layer fwd tokens/sec at 1 B200; attention TFLOP/s as % of bf16 dense peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
WORKLOAD_TEXT = {
    "long-bf16": "long sequence: 2 HSTU layers bf16, d_model 512, 8 heads x 64, 8 users x 8192 "
                 "tokens, lognormal gaps (mu=7, sigma=2), 8192 pos + 128 time buckets, causal",
    "small-bf16": "2 HSTU layers bf16, d_model 256, 4 heads x 64, 32 users, lengths U{64..512}",
    "sl-bf16": "4 HSTU layers bf16, d_model 512, 8 heads x 64, 64 users, Stochastic Length "
               "(alpha 1.6) subsample of 4096",
    "tiny-fp32": "1 HSTU layer fp32, d_model 64, 1 head x 64, 4 users, lengths U{8..64}",
    "mfalcon": "M-FALCON ranking: 4 HSTU layers bf16, d_model 512, 8 heads x 64, 16 users x 4096 "
               "cached history, 2048 candidates per user in microbatches of 256",
    "long-bf16-softmax": "the long-sequence workload with the (-rab, Softmax) ablation: softmax "
                         "over the visible keys instead of the pointwise phi2, zero bias tables",
    "long-bf16-mtgr": "the long-sequence workload with generalised (MTGR-style) masks: per user "
                      "1024 U+S tokens, 6144 R tokens, 1024 candidates timed across R",
    "sl-sampler": "GPU Stochastic Length sampler on 64 users x 4096 events (alpha 1.6), d_model "
                  "512 bf16 rows gathered",
    "long-bf16-train": "training step on the long-sequence workload: forward and backward of "
                       "both layers (hstu_layer_fwd, hstu_layer_bwd), synthetic dL/dY",
    "long-bf16-fused": "the long-sequence workload with f2 inside the attention kernel "
                       "(HSTU_FLAG_FUSED_F2: the last head CTA of each query tile pair runs it)",
}
# workloads that are another workload with a changed configuration:
# name -> (base workload, config changes, zero the rab tables)
VARIANTS = {"long-bf16-softmax": ("long-bf16", {"phi2": "softmax"}, True),
            "long-bf16-mtgr": ("long-bf16", {}, False)}


def make_workload(name, batch=None):
    from gen import make_case
    base, changes, zero_rab = VARIANTS.get(name, (name, {}, False))
    case = make_case(base, batch=batch)
    if changes:
        case = make_case(case.cfg.replace(**changes), seed=case.seed, batch=batch)
    if zero_rab:
        for lw in case.layers:
            lw.rab_pos[:] = 0.0
            lw.rab_time[:] = 0.0
    if name == "long-bf16-mtgr":
        # U+S 1024, R 6144, candidates 1024 with timestamps spread over R's span
        import numpy as np
        rng = np.random.default_rng(7)
        n_us, n_r = 1024, 6144
        segs = []
        for u in range(len(case.lengths)):
            s0, n = int(case.offsets[u]), int(case.lengths[u])
            lo, hi = case.timestamps[s0 + n_us], case.timestamps[s0 + n_us + n_r - 1]
            case.timestamps[s0 + n_us + n_r:s0 + n] = np.sort(rng.integers(lo, hi + 1, n - n_us - n_r))
            segs.append([n_us, n_r])
        case.extra["segments"] = np.array(segs, dtype=np.int32)
    return case


def visible_pairs(case) -> int:
    """Causal pairs, or the visible (query, key) pairs of the generalised masks."""
    import numpy as np
    segs = case.extra.get("segments")
    n = case.lengths.astype(np.int64)
    if segs is None:
        return int((n * (n + 1) // 2).sum())
    total = 0
    for u, seg in enumerate(segs):
        n_us, n_r = int(seg[0]), int(seg[1])
        s0, nu = int(case.offsets[u]), int(n[u])
        r_end = n_us + n_r
        ts = case.timestamps[s0:s0 + nu]
        total += n_us * n_us                                         # U+S rows
        total += int(np.arange(n_us + 1, r_end + 1).sum())           # R rows: i + 1
        r_vis = np.searchsorted(ts[n_us:r_end], ts[r_end:], side="right")
        total += int((n_us + r_vis + 1).sum())                       # candidates
    return total

MFALCON_METRIC = "M-FALCON candidate scores/sec at 1 B200 (cached history K/V)"
# The attention launches of these workloads last about a millisecond inside
# steps of a few milliseconds, far from the seconds-long matmul loop that
# defines the sustained figure, so their roofline uses the burst peak.
PEAK_RULE = ("burst: the kernel is timed per launch (~0.05-1.2 ms) inside short steps; "
             "the sustained figure belongs to a seconds-long loop")
# fp32 FFMA peak for the fp32 SIMT workload: 148 SMs x 128 FMA/clk x 2 flop x clock
FP32_LANES_PER_SM = 128


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks

def gpu_selector(torch, local: int) -> str:
    """nvidia-smi id of the GPU torch calls cuda:local.  nvidia-smi ignores
    CUDA_VISIBLE_DEVICES, so the CUDA ordinal is not an NVML index: select by
    UUID (or PCI bus id when the UUID is unavailable)."""
    props = torch.cuda.get_device_properties(local)
    u = str(getattr(props, "uuid", "") or "")
    if u:
        return u if u.startswith("GPU-") else "GPU-" + u
    return f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.2)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "gpu": self.gpu}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "gpu": self.gpu}
        sm = sorted(float(r[1]) for r in rows if r[1].replace(".", "").isdigit())
        mx = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "gpu": self.gpu}


# ----------------------------------------------------------------------------- oracle baseline

def _oracle_cores():
    cores = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 0) for i in threadpool_info()), default=cores)
    except Exception:
        threads = cores
    return threads, cores


def oracle_extrapolated(case, target_s: float = 15.0):
    """The float64 oracle's rate on the whole workload, extrapolated from two
    timed causal prefixes of user 0.

    Rows 0..m-1 of a user depend only on its first m tokens, so a prefix is an
    exact piece of the workload.  The oracle's cost per user is a per-token
    term (projection, LayerNorm, f2) plus a per-(query, key) term (it forms
    dense n x n matrices per head): t(m) = a m + b m^2.  Prefixes m and m/2 are
    timed (all layers), a and b solved, and t = sum_u (a n_u + b n_u^2) gives
    the whole-workload time.  Labelled extrapolated."""
    from oracle import hstu as O
    n0 = int(case.offsets[1] - case.offsets[0])

    def run(m):
        t0 = time.perf_counter()
        O.forward(case.x, case.offsets, case.timestamps, case.layers, case.cfg,
                  users=[0], prefix=[m])
        return time.perf_counter() - t0

    m = min(256, n0)
    dt = run(m)
    while m < n0 and dt < 0.45 * target_s:
        m = min(n0, int(m * min(4.0, max(1.25, math.sqrt(0.6 * target_s / max(dt, 1e-3))))))
        dt = run(m)
    m1 = max(1, m // 2)
    dt1 = run(m1)
    # t = a m + b m^2 through both points (b >= 0, a >= 0)
    if m1 == m:
        a, b = dt / m, 0.0
    else:
        b = max(0.0, (dt / m - dt1 / m1) / (m - m1))
        a = max(0.0, dt / m - b * m)
    n = case.lengths.astype(float)
    t_full = float(sum(a * x + b * x * x for x in n))
    tokens = float(n.sum())
    threads, cores = _oracle_cores()
    return {"value": tokens / t_full, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "extrapolated": True,
            "sample": f"float64 oracle on causal prefixes of user 0 ({m1} and {m} of {n0} tokens, "
                      f"all {case.cfg.num_layers} layers: {dt1:.2f} s and {dt:.2f} s); "
                      f"t(m) = a m + b m^2 fitted (a={a:.3e} s/token, b={b:.3e} s/pair) and "
                      f"extrapolated to the whole workload ({int(tokens)} tokens, "
                      f"{len(n)} users): {t_full:.0f} s",
            "host_cpu_count": cores, "seconds_timed": dt + dt1, "seconds_extrapolated": t_full}


def run_reference(args, rank, world):
    """The reference arm: the float64 oracle on the host cores (rank 0 only)."""
    if rank != 0:
        return
    case = make_workload(args.workload)
    # each step a bounded sample: the whole run stays near 2.5 minutes of host time
    per_step = max(0.5, min(args.ref_seconds, 150.0 / max(1, args.steps)))
    for _ in range(args.warmup):
        oracle_extrapolated(case, target_s=0.5)
    samples = [oracle_extrapolated(case, target_s=per_step) for _ in range(args.steps)]
    vals = sorted(s["value"] for s in samples)
    v = vals[len(vals) // 2]
    last = samples[-1]
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * last["seconds_extrapolated"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT.get(args.workload, args.workload)},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": last["cores"],
                             "kind": "oracle", "extrapolated": True, "sample": last["sample"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- helpers

def traffic_from_profiles(kernel: str):
    """DRAM bytes per launch of `kernel` from a committed ncu summary, if its
    recorded source hash still matches the kernel source."""
    import hashlib
    summ = os.path.join(ROOT, "profiles", f"{kernel}_traffic.txt")
    if not os.path.exists(summ):
        return None
    vals = {}
    with open(summ) as f:
        for line in f:
            if "=" in line and not line.startswith("#"):
                k, v = line.split("=", 1)
                vals[k.strip()] = v.strip()
    src = os.path.join(ROOT, "hstu_sequential_transduction_jagged_b200", "csrc", vals.get("source", ""))
    if not os.path.exists(src):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if h != vals.get("source_sha256_16"):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def pipelined_e2e(torch, n_steps, nb, copy_in, compute, copy_out, stream):
    """Run `n_steps` host-in / compute / host-out steps with `nb` sets of
    buffers: the host-to-device copy of step i+1 and the device-to-host copy of
    step i-1 run on their own streams while step i computes on `stream`.
    Every step still copies its own inputs from pinned host memory and its own
    result back.  `copy_in(k)`, `compute(k)` and `copy_out(k)` enqueue on the
    current stream for buffer set k."""
    s_in, s_out = torch.cuda.Stream(stream.device), torch.cuda.Stream(stream.device)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    ev_in = [torch.cuda.Event() for _ in range(nb)]
    ev_cmp = [torch.cuda.Event() for _ in range(nb)]
    ev_out = [torch.cuda.Event() for _ in range(nb)]
    for i in range(n_steps):
        k = i % nb
        if i >= nb:
            s_in.wait_event(ev_cmp[k])    # step i-nb has finished reading buffer set k
        with torch.cuda.stream(s_in):
            copy_in(k)
        ev_in[k].record(s_in)
        stream.wait_event(ev_in[k])
        if i >= nb:
            stream.wait_event(ev_out[k])  # step i-nb's result has left buffer set k
        with torch.cuda.stream(stream):
            compute(k)
        ev_cmp[k].record(stream)
        s_out.wait_event(ev_cmp[k])
        with torch.cuda.stream(s_out):
            copy_out(k)
        ev_out[k].record(s_out)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)


class Ctx:
    """Per-process GPU context shared by the workload measurements."""

    def __init__(self, args, rank, world, local):
        import torch
        import torch.distributed as dist
        from hstu_sequential_transduction_jagged_b200 import build as hbuild
        from hstu_sequential_transduction_jagged_b200 import hstu as H
        self.torch, self.dist, self.H = torch, dist, H
        self.args, self.rank, self.world, self.local = args, rank, world, local
        torch.cuda.set_device(local)
        self.dev = torch.device("cuda", local)
        if world > 1:
            from datetime import timedelta
            dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=self.dev)
        if rank == 0:
            hbuild.build()
        if world > 1:
            dist.barrier()
        self.flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=self.dev)  # > L2
        self.stream = torch.cuda.current_stream()
        self.peaks, self.peak_src = load_peaks()
        self.gpu_id = gpu_selector(torch, local)

    def max_over_ranks(self, x: float) -> float:
        if self.world == 1:
            return x
        t = self.torch.tensor([x], dtype=self.torch.float64, device=self.dev)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def timed_steps(self, step, steps, sample_clocks=True):
        """`steps` calls of step(), each bracketed by CUDA events on the launching
        stream, an L2 flush (256 MiB write) before each outside the events.
        Returns (per-step ms list, library per-kernel times, clocks)."""
        torch, H = self.torch, self.H
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        sampler = ClockSampler(self.gpu_id) if sample_clocks else None
        if sampler:
            sampler.start()
        if self.world > 1:
            self.dist.barrier()
        torch.cuda.synchronize()
        H.profiler_start()
        for i in range(steps):
            self.flush.zero_()
            evs[i][0].record(self.stream)
            step()
            evs[i][1].record(self.stream)
        torch.cuda.synchronize()
        kernels = H.profiler_stop()
        if self.world > 1:
            self.dist.barrier()
        clocks = sampler.stop() if sampler else None
        assert H.device_status() == 0
        return [a.elapsed_time(b) for a, b in evs], kernels, clocks


def _median(xs):
    s = sorted(xs)
    n = len(s)
    return s[n // 2] if n % 2 else 0.5 * (s[n // 2 - 1] + s[n // 2])


def _kernel_table(kernels):
    tot = max(1e-9, sum(v[1] for v in kernels.values()))
    return {k: {"launches": n, "ms_per_launch": m / n, "share": m / tot}
            for k, (n, m) in kernels.items()}


def _roofline(ctx, kernels, name, flop, kernel_label, bound="tensor"):
    n, ms = kernels.get(name, (0, 0.0))
    if not n:
        return None
    per = ms / n
    achieved = flop / (per / 1000.0) / 1e12
    if bound == "alu":
        # fp32 SIMT kernels: FFMA lanes x 2 flop x max SM clock
        peak = 148 * FP32_LANES_PER_SM * 2 * ctx.peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        src = "derived: 148 SMs x 128 fp32 FMA lanes x 2 flop x max SM clock"
    else:
        peak = ctx.peaks["bf16_tflops"]
        src = f"{ctx.peak_src} bf16 dense, burst ({PEAK_RULE})"
    out = {"kernel": kernel_label, "bound": bound, "achieved": achieved, "peak": peak,
           "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None, "peak_source": src,
           "algorithmic_flop_per_launch": flop, "ms_per_launch": per}
    if bound == "tensor":
        sus = ctx.peaks.get("bf16_tflops_sustained")
        if sus:
            out["frac_of_sustained"] = achieved / sus
    return out


# ----------------------------------------------------------------------------- workloads

def measure_forward(ctx, name, steps, warmup, with_e2e, sample_clocks=True, batch=None):
    """Time hstu_forward over one workload; returns a dict (value, rooflines...)."""
    torch, H = ctx.torch, ctx.H
    from gen import algorithmic_counts
    from gen.device import case_tensors
    fused = name.endswith("-fused")
    case = make_workload(name[:-len("-fused")] if fused else name, batch=batch)
    c = case.cfg
    counts = algorithmic_counts(case)
    counts["attn_flop_per_layer"] = visible_pairs(case) * c.num_heads * (2 * c.dqk + 2 * c.dv)
    t = case_tensors(case, ctx.dev)
    segs = case.extra.get("segments")
    jag = H.Jagged(t["offsets"], t["timestamps"], case.max_len, case.total_tokens,
                   None if segs is None else torch.from_numpy(segs).to(ctx.dev),
                   0 if segs is None else int(segs[:, 0].max()))
    weights = [H.LayerWeights(**lw) for lw in t["layers"]]
    cfg = H.LayerConfig(c.d_model, c.num_heads, c.num_pos_buckets, c.num_time_buckets,
                        dqk=c.dqk, dv=c.dv, phi1=c.phi1, phi2=c.phi2, ln_eps=c.ln_eps,
                        dtype=c.dtype, fused_f2=fused)
    L, T = c.num_layers, case.total_tokens
    ws = torch.empty(H.forward_workspace_bytes(cfg, L, T), dtype=torch.uint8, device=ctx.dev)
    y = torch.empty((T, c.d_model), dtype=torch.float32, device=ctx.dev)

    def step():
        H.forward(cfg, weights, jag, t["x"], y_out=y, workspace=ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert H.device_status() == 0
    step_ms, kernels, clocks = ctx.timed_steps(step, steps, sample_clocks)
    total = ctx.max_over_ranks(sum(step_ms))
    ms = total / steps
    value = ctx.world * T / (ms / 1000.0)
    world = ctx.world
    bf16 = c.dtype == "bf16"
    if bf16 and "attention_f2_fused" in kernels:
        # the layer-fused kernel: attention plus f2 (Norm(AV) (.) U, W2, residual)
        roof = _roofline(ctx, kernels, "attention_f2_fused",
                         counts["attn_flop_per_layer"] + counts["f2_flop_per_layer"],
                         "hstu_attn_kernel (causal, layer-fused f2)", "tensor")
        if roof is not None:
            roof["algorithmic_flop_attention"] = counts["attn_flop_per_layer"]
            roof["algorithmic_flop_f2"] = counts["f2_flop_per_layer"]
            if name == "long-bf16-fused" and batch is None:
                roof["traffic"] = traffic_from_profiles("attention_f2_fused")
    else:
        attn_name = "attention" if bf16 else "fp32_attention"
        roof = _roofline(ctx, kernels, attn_name, counts["attn_flop_per_layer"],
                         "hstu_attn_kernel (causal)" if bf16 else "hstu_f32_attn_kernel (causal)",
                         "tensor" if bf16 else "alu")
        if roof is not None and name == "long-bf16" and batch is None:
            roof["traffic"] = traffic_from_profiles("attention")
    kern = _kernel_table(kernels)
    for kname, key in (("f1_gemm", "f1_flop_per_layer"), ("f2_gemm", "f2_flop_per_layer")):
        if kname in kern:
            per = kern[kname]["ms_per_launch"]
            kern[kname]["tflops"] = counts[key] / (per / 1000.0) / 1e12
            kern[kname]["frac_of_bf16_burst"] = kern[kname]["tflops"] / ctx.peaks["bf16_tflops"]
    if "f2_gemm" in kern:
        # algorithmic bytes of f2: AV and U (fp32), residual (fp32 after layer 0), Y fp32 + bf16 copy
        d, hv = c.d_model, c.num_heads * c.dv
        byt = T * (hv * 4 * 2 + d * 4 + d * 4 + d * 2) + d * hv * 2
        kern["f2_gemm"]["algorithmic_bytes"] = byt
        kern["f2_gemm"]["gbs"] = byt / (kern["f2_gemm"]["ms_per_launch"] / 1000.0) / 1e9
        kern["f2_gemm"]["frac_of_hbm"] = kern["f2_gemm"]["gbs"] / ctx.peaks["hbm_gbs"]
    out = {"metric": "tokens/s", "value": value, "unit": "tokens/s",
           "workload": WORKLOAD_TEXT[name], "ms_per_step": ms,
           "ms_per_step_median": _median(step_ms), "tokens_per_step": world * T,
           "layer_tokens_per_s": value * L, "layers": L, "dtype": c.dtype,
           "roofline": roof, "kernels": kern, "gpu_launches": sum(n for n, _ in kernels.values()),
           "clocks": clocks, "_case": case}
    if with_e2e:
        out.update(forward_e2e(ctx, case, t, cfg, weights, ws, y, steps))
    return out


def forward_e2e(ctx, case, t, cfg, weights, ws, y, steps):
    """Same forward through the public API with host buffers: X, offsets and
    timestamps copied from pinned host memory and Y copied back, every step.
    Serial: one step after another.  Pipelined (reported as e2e): two buffer
    sets, the copy-in of step i+1 and copy-out of step i-1 overlap step i."""
    torch, H = ctx.torch, ctx.H
    T = case.total_tokens
    x_host = t["x"].cpu().pin_memory()
    off_host = t["offsets"].cpu().pin_memory()
    ts_host = t["timestamps"].cpu().pin_memory()
    NB = 2
    y_hosts = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(NB)]
    x_devs = [torch.empty_like(t["x"]) for _ in range(NB)]
    off_devs = [torch.empty_like(t["offsets"]) for _ in range(NB)]
    ts_devs = [torch.empty_like(t["timestamps"]) for _ in range(NB)]
    y_devs = [torch.empty_like(y) for _ in range(NB)]
    jags = [H.Jagged(off_devs[k], ts_devs[k], case.max_len, T) for k in range(NB)]

    def copy_in(k):
        x_devs[k].copy_(x_host, non_blocking=True)
        off_devs[k].copy_(off_host, non_blocking=True)
        ts_devs[k].copy_(ts_host, non_blocking=True)

    def compute(k):
        H.forward(cfg, weights, jags[k], x_devs[k], y_out=y_devs[k], workspace=ws,
                  stream=torch.cuda.current_stream())

    def copy_out(k):
        y_hosts[k].copy_(y_devs[k], non_blocking=True)

    def run_serial(n):
        for _ in range(n):
            copy_in(0)
            compute(0)
            copy_out(0)

    def run_pipe(n):
        pipelined_e2e(torch, n, NB, copy_in, compute, copy_out, ctx.stream)

    def timed(run, n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if ctx.world > 1:
            ctx.dist.barrier()
        torch.cuda.synchronize()
        a.record(ctx.stream)
        run(n)
        b.record(ctx.stream)
        torch.cuda.synchronize()
        return ctx.max_over_ranks(a.elapsed_time(b) / n)

    n_e2e = max(3, min(steps, 20))
    run_serial(2)
    torch.cuda.synchronize()
    e_serial_ms = timed(run_serial, n_e2e)
    run_pipe(2 * NB)
    torch.cuda.synchronize()
    e_ms = timed(run_pipe, n_e2e)
    h2d = x_host.numel() * x_host.element_size() + off_host.numel() * 8 + ts_host.numel() * 8
    d2h = y_hosts[0].numel() * y_hosts[0].element_size()
    w = ctx.world
    return {"e2e": {"value": w * T / (e_ms / 1000.0), "unit": "tokens/s", "ms_per_step": e_ms,
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                    "pipelining": "2 buffer sets; copy-in of step i+1 and copy-out of step i-1 "
                                  "on their own streams overlap step i"},
            "e2e_serial": {"value": w * T / (e_serial_ms / 1000.0), "unit": "tokens/s",
                           "ms_per_step": e_serial_ms}}


def measure_sl_sampler(ctx, steps, warmup):
    """Time the GPU Stochastic Length sampler on the sl-bf16 batch before
    subsampling: 64 users with full timelines of 4096 events, d_model 512 bf16
    rows gathered.  The gather is HBM-bound: algorithmic bytes are the kept
    rows read and written plus their index and timestamp (8 bytes each, read
    and written)."""
    torch, H = ctx.torch, ctx.H
    from gen import make_case
    from gen.device import case_tensors
    cfg = make_case("sl-bf16").cfg.replace(len_kind="fixed")
    case = make_case(cfg, seed=3, num_layers=1)
    t = case_tensors(case, ctx.dev)
    jag = H.Jagged(t["offsets"], t["timestamps"], case.max_len, case.total_tokens)
    seeds = iter(range(10 ** 6))

    def step():
        H.stochastic_length(jag, cfg.sl_alpha, 7, next(seeds), x=t["x"])

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    step_ms, kernels, _ = ctx.timed_steps(step, steps, sample_clocks=False)
    ms = sum(step_ms) / steps
    out = H.stochastic_length(jag, cfg.sl_alpha, 7, 0, x=t["x"])
    T_out = int(out["offsets"][-1].item())
    row = cfg.d_model * 2
    n_g, ms_g = kernels.get("sl_gather", (0, 0.0))
    byt = T_out * (2 * row + 2 * 8 + 2 * 8)
    gbs = byt / (ms_g / n_g / 1000.0) / 1e9 if n_g else None
    return {"metric": "events kept/s", "value": T_out / (ms / 1000.0), "unit": "events/s",
            "workload": "Stochastic Length (alpha 1.6) of 64 users x 4096 events, d_model 512 "
                        "bf16 rows gathered", "ms_per_step": ms, "events_in": case.total_tokens,
            "events_kept_example": T_out, "kernels": _kernel_table(kernels),
            "gpu_launches": sum(n for n, _ in kernels.values()),
            "roofline": None if gbs is None else {
                "kernel": "hstu_sl_gather_kernel", "bound": "hbm", "achieved": gbs,
                "peak": ctx.peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / ctx.peaks["hbm_gbs"],
                "traffic": None, "algorithmic_bytes_per_launch": byt,
                "ms_per_launch": ms_g / n_g}}


TRAIN_METRIC = "HSTU training step (forward + backward of every layer) tokens/sec at 1 B200"


def measure_train(ctx, steps, warmup, sample_clocks=False, batch=None):
    """Forward and backward of both layers of the long-sequence workload: layer
    0 from the bf16 input, layer 1 from layer 0's fp32 output; backward with a
    fixed synthetic dL/dY through layer 1, then layer 0 (all parameter
    gradients and dX).  No optimizer."""
    torch, H = ctx.torch, ctx.H
    from gen.device import case_tensors
    case = make_workload("long-bf16", batch=batch)
    c = case.cfg
    T, L = case.total_tokens, c.num_layers
    t = case_tensors(case, ctx.dev)
    jag = H.Jagged(t["offsets"], t["timestamps"], case.max_len, T)
    weights = [H.LayerWeights(**lw) for lw in t["layers"]]
    cfg = H.LayerConfig(c.d_model, c.num_heads, c.num_pos_buckets, c.num_time_buckets,
                        dqk=c.dqk, dv=c.dv, phi1=c.phi1, phi2=c.phi2, ln_eps=c.ln_eps,
                        dtype=c.dtype)
    fws = torch.empty(H.layer_workspace_bytes(cfg, T), dtype=torch.uint8, device=ctx.dev)
    bws = torch.empty(H.layer_bwd_workspace_bytes(cfg, T), dtype=torch.uint8, device=ctx.dev)
    ys = [torch.empty((T, c.d_model), dtype=torch.float32, device=ctx.dev) for _ in range(L)]
    g = torch.Generator(device=ctx.dev).manual_seed(0)
    dy_top = torch.randn((T, c.d_model), generator=g, device=ctx.dev, dtype=torch.float32)

    def step():
        for l in range(L):
            if l == 0:
                H.layer_fwd(cfg, weights[0], jag, t["x"], y_out=ys[0], workspace=fws)
            else:
                H.layer_fwd(cfg, weights[l], jag, None, x_res=ys[l - 1], y_out=ys[l], workspace=fws)
        dy = dy_top
        for l in reversed(range(L)):
            if l == 0:
                r = H.layer_bwd(cfg, weights[0], jag, t["x"], dy, workspace=bws)
            else:
                r = H.layer_bwd(cfg, weights[l], jag, None, dy, x_res=ys[l - 1], workspace=bws)
            dy = r["dx"]

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert H.device_status() == 0
    step_ms, kernels, clocks = ctx.timed_steps(step, steps, sample_clocks)
    total = ctx.max_over_ranks(sum(step_ms))
    ms = total / steps
    value = ctx.world * T / (ms / 1000.0)
    pairs = visible_pairs(case)
    # attention backward, FlashAttention convention: five 2*64-flop products
    # per visible (i, j, head): S (recomputed), dP, dV, dQ, dK
    bwd_flop = pairs * c.num_heads * 5 * 2 * 64
    n_b, ms_b = kernels.get("attention_bwd", (0, 0.0))
    roof = None
    if n_b:
        per = ms_b / n_b
        ach = bwd_flop / (per / 1000.0) / 1e12
        roof = {"kernel": "hstu_attn_bwd_kernel (dK, dV and dQ, one launch per layer)",
                "bound": "tensor",
                "achieved": ach, "peak": ctx.peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": ach / ctx.peaks["bf16_tflops"],
                "traffic": traffic_from_profiles("attention_bwd") if batch is None else None,
                "peak_source": f"{ctx.peak_src} bf16 dense, burst ({PEAK_RULE})",
                "algorithmic_flop_per_launch": bwd_flop,
                "flop_rule": "5 x 2 x 64 flop per visible (i, j, head): S, dP, dV, dQ, dK",
                "ms_per_launch": per}
    return {"metric": TRAIN_METRIC, "value": value, "unit": "tokens/s",
            "workload": "training step on the long-sequence workload (2 layers bf16, d_model "
                        "512, 8 heads, 8 users x 8192): forward and backward of both layers, "
                        "synthetic dL/dY, no optimizer",
            "ms_per_step": ms, "ms_per_step_median": _median(step_ms), "tokens_per_step": T,
            "layers": L, "roofline": roof, "kernels": _kernel_table(kernels),
            "gpu_launches": sum(n for n, _ in kernels.values()), "clocks": clocks}


def measure_mfalcon(ctx, steps, warmup, with_e2e, sample_clocks=True, batch=None):
    """Time mfalcon_score over every candidate of the M-FALCON workload (the
    history is encoded once beforehand, with its K/V kept per layer)."""
    import numpy as np
    torch, H = ctx.torch, ctx.H
    from gen import make_case
    from gen.device import case_tensors
    case = make_case("mfalcon", batch=batch)
    c = case.cfg
    t = case_tensors(case, ctx.dev)
    jag = H.Jagged(t["offsets"], t["timestamps"], case.max_len, case.total_tokens)
    weights = [H.LayerWeights(**lw) for lw in t["layers"]]
    cfg = H.LayerConfig(c.d_model, c.num_heads, c.num_pos_buckets, c.num_time_buckets)
    L, T, hv = c.num_layers, case.total_tokens, c.num_heads * 64
    M = t["cand_emb"].shape[0]
    kv = torch.empty((L, T, 2 * hv), dtype=cfg.cache_dtype, device=ctx.dev)
    ws_h = torch.empty(H.forward_workspace_bytes(cfg, L, T), dtype=torch.uint8, device=ctx.dev)
    ws_c = torch.empty(H.mfalcon_workspace_bytes(cfg, M), dtype=torch.uint8, device=ctx.dev)
    scores = torch.empty(M, dtype=torch.float32, device=ctx.dev)
    for _ in range(2):
        H.forward(cfg, weights, jag, t["x"], kv_cache_out=kv, workspace=ws_h)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(ctx.stream)
    H.forward(cfg, weights, jag, t["x"], kv_cache_out=kv, workspace=ws_h)
    b.record(ctx.stream)
    torch.cuda.synchronize()
    hist_ms = a.elapsed_time(b)

    def step():
        H.mfalcon_score(cfg, weights, jag, kv, t["cand_offsets"], t["cand_emb"], t["request_ts"],
                        c.microbatch, c.num_cand, scores=scores, workspace=ws_c)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert H.device_status() == 0
    step_ms, kernels, clocks = ctx.timed_steps(step, steps, sample_clocks)
    ms = ctx.max_over_ranks(sum(step_ms)) / steps
    value = ctx.world * M / (ms / 1000.0)
    n_u = case.lengths.astype(np.float64)
    cand_flop = float(((n_u + 1) * c.num_cand).sum()) * c.num_heads * 256  # per layer
    roof = _roofline(ctx, kernels, "mfalcon_attention", cand_flop, "hstu_attn_kernel (candidate)")
    out = {"metric": MFALCON_METRIC, "value": value, "unit": "candidates/s",
           "workload": WORKLOAD_TEXT["mfalcon"], "ms_per_step": ms,
           "ms_per_step_median": _median(step_ms), "candidates_per_step": ctx.world * M,
           "history_tokens": T, "layers": L, "microbatch": c.microbatch,
           "history_encode_ms": hist_ms, "roofline": roof, "kernels": _kernel_table(kernels),
           "gpu_launches": sum(n for n, _ in kernels.values()), "clocks": clocks}
    if with_e2e:
        emb_host = t["cand_emb"].cpu().pin_memory()
        NB = 2
        sc_hosts = [torch.empty(M, dtype=torch.float32).pin_memory() for _ in range(NB)]
        emb_devs = [torch.empty_like(t["cand_emb"]) for _ in range(NB)]
        sc_devs = [torch.empty(M, dtype=torch.float32, device=ctx.dev) for _ in range(NB)]

        def score_into(k):
            H.mfalcon_score(cfg, weights, jag, kv, t["cand_offsets"], emb_devs[k],
                            t["request_ts"], c.microbatch, c.num_cand, scores=sc_devs[k],
                            workspace=ws_c, stream=torch.cuda.current_stream())

        def run_pipe(n):
            pipelined_e2e(torch, n, NB, lambda k: emb_devs[k].copy_(emb_host, non_blocking=True),
                          score_into, lambda k: sc_hosts[k].copy_(sc_devs[k], non_blocking=True),
                          ctx.stream)

        n_e2e = max(3, min(steps, 10))
        run_pipe(2 * NB)
        torch.cuda.synchronize()
        a.record(ctx.stream)
        run_pipe(n_e2e)
        b.record(ctx.stream)
        torch.cuda.synchronize()
        e_ms = ctx.max_over_ranks(a.elapsed_time(b) / n_e2e)
        out["e2e"] = {"value": ctx.world * M / (e_ms / 1000.0), "unit": "candidates/s",
                      "ms_per_step": e_ms, "h2d_bytes_per_step": int(emb_host.numel() * 2),
                      "d2h_bytes_per_step": int(M * 4),
                      "pipelining": "2 buffer sets; copy-in of step i+1 and copy-out of step "
                                    "i-1 on their own streams overlap step i"}
    return out


# ----------------------------------------------------------------------------- main

def _public(d):
    return {k: v for k, v in d.items() if not k.startswith("_")}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="long-bf16", choices=sorted(WORKLOAD_TEXT))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other configurations (profiling runs)")
    ap.add_argument("--ref-seconds", type=float, default=15.0)
    ap.add_argument("--batch", type=int, default=None,
                    help="fewer users than the workload (profiling runs only)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    ctx = Ctx(args, rank, world, local)
    if args.workload == "sl-sampler":
        r = measure_sl_sampler(ctx, args.steps, args.warmup)
        if rank == 0:
            print(json.dumps({**r, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                              "higher_is_better": True, "data": "synthetic"}), flush=True)
    elif args.workload == "long-bf16-train":
        r = measure_train(ctx, args.steps, args.warmup, batch=args.batch)
        if rank == 0:
            print(json.dumps({**r, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                              "higher_is_better": True, "data": "synthetic"}), flush=True)
    elif args.workload == "mfalcon":
        r = measure_mfalcon(ctx, args.steps, args.warmup, not args.no_e2e, batch=args.batch)
        line = {"metric": MFALCON_METRIC, "value": r["value"], "unit": "candidates/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": WORKLOAD_TEXT["mfalcon"],
                           "candidates_per_step": r["candidates_per_step"],
                           "l2": "flushed between timed steps (256 MiB write outside the events)",
                           "parallelism": f"dp{world}: users sharded, no collective"}}
        line.update({k: v for k, v in r.items() if k not in line and k != "metric"})
        if rank == 0:
            print(json.dumps(line), flush=True)
    else:
        r = measure_forward(ctx, args.workload, args.steps, args.warmup, not args.no_e2e,
                            batch=args.batch)
        case = r["_case"]
        line = {"metric": METRIC, "value": r["value"], "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
                "ms_per_step_median": r["ms_per_step_median"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": case.cfg.dtype,
                "data": "synthetic",
                "config": {"workload": WORKLOAD_TEXT[args.workload],
                           "global_batch": world * len(case.lengths), "seq_len": case.max_len,
                           "tokens_per_step": world * case.total_tokens,
                           "layers": case.cfg.num_layers,
                           "l2": "flushed between timed steps (256 MiB write outside the events)",
                           "parallelism": f"dp{world}: users sharded, no collective"},
                "layer_tokens_per_s": r["layer_tokens_per_s"], "roofline": r["roofline"],
                "kernels": r["kernels"], "gpu_launches": r["gpu_launches"],
                "clocks": r["clocks"], "e2e": r.get("e2e"), "e2e_serial": r.get("e2e_serial")}
        if r["roofline"]:
            line["attention"] = {"kernel": r["roofline"]["kernel"],
                                 "tflops": r["roofline"]["achieved"],
                                 "pct_of_bf16_peak_burst": 100 * r["roofline"]["frac"],
                                 "pct_of_bf16_peak_sustained":
                                     100 * r["roofline"].get("frac_of_sustained", 0.0)}
        if world == 1 and not args.no_workloads and args.batch is None:
            subs = {}
            for name in ("long-bf16-fused", "small-bf16", "sl-bf16", "tiny-fp32",
                         "long-bf16-softmax", "long-bf16-mtgr"):
                if name == args.workload:
                    continue
                subs[name] = _public(measure_forward(ctx, name, min(args.steps, 20), args.warmup,
                                                     False, sample_clocks=(name == "sl-bf16")))
            subs["mfalcon"] = measure_mfalcon(ctx, min(args.steps, 20), args.warmup, True)
            subs["sl-sampler"] = measure_sl_sampler(ctx, min(args.steps, 20), args.warmup)
            subs["long-bf16-train"] = measure_train(ctx, min(args.steps, 10), args.warmup)
            line["workloads"] = subs
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = oracle_extrapolated(case)
        if rank == 0:
            print(json.dumps(line), flush=True)
    if world > 1:
        ctx.dist.barrier()
        ctx.dist.destroy_process_group()


if __name__ == "__main__":
    main()
