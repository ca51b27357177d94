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
timed region.  `--impl reference` times the float64 CPU oracle instead.
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
}
MFALCON_METRIC = "M-FALCON candidate scores/sec at 1 B200 (cached history K/V)"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
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
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
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
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = sorted(float(r[1]) for r in rows if r[1].replace(".", "").isdigit())
        mx = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------- oracle baseline

def oracle_sample(case, target_s: float = 15.0):
    """Time the float64 oracle on a causal prefix of user 0 (both layers).

    Rows 0..m-1 of a user depend only on its first m tokens, so the prefix is
    an exact piece of the workload; m is grown until one run takes about
    target_s seconds (or the whole user is covered)."""
    from oracle import hstu as O
    import numpy as np
    n0 = int(case.offsets[1] - case.offsets[0])
    m = min(512, n0)
    while True:
        t0 = time.perf_counter()
        O.forward(case.x, case.offsets, case.timestamps, case.layers, case.cfg,
                  users=[0], prefix=[m])
        dt = time.perf_counter() - t0
        if m >= n0 or dt >= target_s * 0.5:
            break
        # causal work grows about quadratically in the prefix length
        m = min(n0, int(m * min(4.0, max(1.2, math.sqrt(target_s / max(dt, 1e-3))))))
    cores = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 0) for i in threadpool_info()), default=cores)
    except Exception:
        threads = cores
    return {"value": m / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"float64 oracle, user 0 causal prefix of {m} of {n0} tokens, "
                      f"all {case.cfg.num_layers} layers, {dt:.1f} s",
            "host_cpu_count": cores, "seconds": dt}


def run_reference(args, rank, world):
    """The reference arm: the float64 oracle on the host cores (rank 0 only)."""
    if rank != 0:
        return
    from gen import make_case
    case = make_case(args.workload)
    samples = []
    for _ in range(args.warmup):
        oracle_sample(case, target_s=2.0)
    for _ in range(args.steps):
        samples.append(oracle_sample(case, target_s=args.ref_seconds))
    v = sum(s["value"] for s in samples) / len(samples)
    last = samples[-1]
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * last["seconds"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT.get(args.workload, args.workload)},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": last["cores"],
                             "kind": "oracle", "sample": last["sample"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- main arm

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


def run_mfalcon(args, rank, world, local):
    """Time mfalcon_score over every candidate of the M-FALCON workload (the
    history is encoded once beforehand, with its K/V kept per layer)."""
    import numpy as np
    import torch
    import torch.distributed as dist
    from gen import make_case
    from gen.device import case_tensors
    from hstu_sequential_transduction_jagged_b200 import build as hbuild
    from hstu_sequential_transduction_jagged_b200 import hstu as H

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    if rank == 0:
        hbuild.build()
    if world > 1:
        dist.barrier()
    case = make_case("mfalcon", batch=args.batch)
    c = case.cfg
    t = case_tensors(case, dev)
    jag = H.Jagged(t["offsets"], t["timestamps"], case.max_len, case.total_tokens)
    weights = [H.LayerWeights(**lw) for lw in t["layers"]]
    cfg = H.LayerConfig(c.d_model, c.num_heads, c.num_pos_buckets, c.num_time_buckets)
    L, T, hv = c.num_layers, case.total_tokens, c.num_heads * 64
    M = t["cand_emb"].shape[0]
    kv = torch.empty((L, T, 2 * hv), dtype=torch.bfloat16, device=dev)
    ws_h = torch.empty(H.forward_workspace_bytes(cfg, L, T), dtype=torch.uint8, device=dev)
    ws_c = torch.empty(H.mfalcon_workspace_bytes(cfg, M), dtype=torch.uint8, device=dev)
    scores = torch.empty(M, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    # history encode (timed on its own)
    for _ in range(2):
        H.forward(cfg, weights, jag, t["x"], kv_cache_out=kv, workspace=ws_h)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    H.forward(cfg, weights, jag, t["x"], kv_cache_out=kv, workspace=ws_h)
    b.record(stream)
    torch.cuda.synchronize()
    hist_ms = a.elapsed_time(b)

    def step(emb):
        H.mfalcon_score(cfg, weights, jag, kv, t["cand_offsets"], emb, t["request_ts"],
                        c.microbatch, c.num_cand, scores=scores, workspace=ws_c)

    for _ in range(args.warmup):
        step(t["cand_emb"])
    torch.cuda.synchronize()
    assert H.device_status() == 0
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    sampler = ClockSampler(local)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    H.profiler_start()
    for i in range(args.steps):
        flush.zero_()
        evs[i][0].record(stream)
        step(t["cand_emb"])
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    kernels = H.profiler_stop()
    clocks = sampler.stop()
    assert H.device_status() == 0
    total_ms = sum(x.elapsed_time(y) for x, y in evs)
    if world > 1:
        tt = torch.tensor([total_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        total_ms = float(tt.item())
    ms = total_ms / args.steps
    value = world * M / (ms / 1000.0)
    # end to end: candidate embeddings in, scores out, through the public API.
    # Serial: copy in, score, copy out, one step after another on one stream.
    # Pipelined (reported as e2e): two buffer sets, copies of neighbouring steps
    # overlap the scoring of the current one.
    emb_host = t["cand_emb"].cpu().pin_memory()
    NB = 2
    sc_hosts = [torch.empty(M, dtype=torch.float32).pin_memory() for _ in range(NB)]
    emb_devs = [torch.empty_like(t["cand_emb"]) for _ in range(NB)]
    sc_devs = [torch.empty(M, dtype=torch.float32, device=dev) for _ in range(NB)]

    def score_into(k):
        H.mfalcon_score(cfg, weights, jag, kv, t["cand_offsets"], emb_devs[k], t["request_ts"],
                        c.microbatch, c.num_cand, scores=sc_devs[k], workspace=ws_c,
                        stream=torch.cuda.current_stream())

    def e2e_serial_step():
        emb_devs[0].copy_(emb_host, non_blocking=True)
        score_into(0)
        sc_hosts[0].copy_(sc_devs[0], non_blocking=True)

    n_e2e = max(3, min(args.steps, 10))
    e2e_serial_step()
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(n_e2e):
        e2e_serial_step()
    b.record(stream)
    torch.cuda.synchronize()
    e_serial_ms = a.elapsed_time(b) / n_e2e

    def run_pipe(n):
        pipelined_e2e(torch, n, NB, lambda k: emb_devs[k].copy_(emb_host, non_blocking=True),
                      score_into, lambda k: sc_hosts[k].copy_(sc_devs[k], non_blocking=True),
                      stream)

    run_pipe(2 * NB)
    torch.cuda.synchronize()
    a.record(stream)
    run_pipe(n_e2e)
    b.record(stream)
    torch.cuda.synchronize()
    e_ms = a.elapsed_time(b) / n_e2e
    peaks, peak_src = load_peaks()
    peak_sus = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    n_u = case.lengths.astype(np.float64)
    cand_flop = float(((n_u + 1) * c.num_cand).sum()) * c.num_heads * 256  # per layer
    ca_n, ca_ms = kernels.get("mfalcon_attention", (0, 0.0))
    ca_tf = cand_flop / (ca_ms / ca_n / 1000.0) / 1e12 if ca_n else None
    kern = {k: {"launches": n, "ms_per_launch": m / n} for k, (n, m) in kernels.items()}
    line = {"metric": MFALCON_METRIC, "value": value, "unit": "candidates/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT["mfalcon"], "candidates_per_step": world * M,
                       "history_tokens": T, "layers": L, "microbatch": c.microbatch,
                       "l2": "flushed between timed steps (256 MiB write outside the events)",
                       "parallelism": f"dp{world}: users sharded, no collective"},
            "history_encode_ms": hist_ms,
            "roofline": {"kernel": "hstu_attn_kernel (candidate)", "bound": "tensor",
                         "achieved": ca_tf, "peak": peak_sus, "unit": "TFLOP/s",
                         "frac": ca_tf / peak_sus if ca_tf else None, "traffic": None,
                         "peak_source": f"{peak_src} bf16 dense, sustained",
                         "algorithmic_flop_per_launch": cand_flop},
            "kernels": kern, "gpu_launches": sum(n for n, _ in kernels.values()),
            "clocks": clocks,
            "e2e": {"value": world * M / (e_ms / 1000.0), "unit": "candidates/s",
                    "ms_per_step": e_ms, "h2d_bytes_per_step": int(emb_host.numel() * 2),
                    "d2h_bytes_per_step": int(M * 4),
                    "pipelining": "2 buffer sets; copy-in of step i+1 and copy-out of step i-1 "
                                  "on their own streams overlap step i"},
            "e2e_serial": {"value": world * M / (e_serial_ms / 1000.0), "unit": "candidates/s",
                           "ms_per_step": e_serial_ms}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="long-bf16", choices=sorted(WORKLOAD_TEXT))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
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
    if args.workload == "mfalcon":
        run_mfalcon(args, rank, world, local)
        return

    import numpy as np
    import torch
    import torch.distributed as dist
    from gen import make_case, algorithmic_counts
    from gen.device import case_tensors
    from hstu_sequential_transduction_jagged_b200 import build as hbuild
    from hstu_sequential_transduction_jagged_b200 import hstu as H

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=dev)
    if rank == 0:
        hbuild.build()
    if world > 1:
        dist.barrier()

    case = make_case(args.workload, batch=args.batch)
    cfgd = case.cfg
    counts = algorithmic_counts(case)
    t = case_tensors(case, dev)
    jag = H.Jagged(t["offsets"], t["timestamps"], case.max_len, case.total_tokens)
    weights = [H.LayerWeights(**lw) for lw in t["layers"]]
    cfg = H.LayerConfig(cfgd.d_model, cfgd.num_heads, cfgd.num_pos_buckets, cfgd.num_time_buckets,
                        dqk=cfgd.dqk, dv=cfgd.dv, phi1=cfgd.phi1, phi2=cfgd.phi2,
                        ln_eps=cfgd.ln_eps, dtype=cfgd.dtype)
    L = cfgd.num_layers
    T = case.total_tokens
    ws = torch.empty(H.forward_workspace_bytes(cfg, L, T), dtype=torch.uint8, device=dev)
    y = torch.empty((T, cfgd.d_model), dtype=torch.float32, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)  # > 126 MB L2
    stream = torch.cuda.current_stream()

    def step(x_in):
        H.forward(cfg, weights, jag, x_in, y_out=y, workspace=ws)

    for _ in range(args.warmup):
        step(t["x"])
    torch.cuda.synchronize()
    assert H.device_status() == 0

    # ---------------- timed region: inputs resident in HBM, L2 flushed between steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    sampler = ClockSampler(local)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    H.profiler_start()
    for i in range(args.steps):
        flush.zero_()
        evs[i][0].record(stream)
        step(t["x"])
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    kernels = H.profiler_stop()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = sum(step_ms)
    assert H.device_status() == 0
    if world > 1:
        tt = torch.tensor([total_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        total_ms = float(tt.item())
    ms_per_step = total_ms / args.steps
    value = world * T / (ms_per_step / 1000.0)

    # ---------------- end to end through the public API, host buffers
    # Every step copies X, offsets and timestamps from pinned host memory and
    # Y back.  Serial: one step after another on one stream.  Pipelined
    # (reported as e2e): two buffer sets, the copy-in of step i+1 and the
    # copy-out of step i-1 overlap the forward of step i.
    e2e = None
    e2e_serial = None
    if not args.no_e2e:
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

        def serial_step():
            copy_in(0)
            compute(0)
            copy_out(0)

        def timed(run, n):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            a.record(stream)
            run(n)
            b.record(stream)
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / n
            if world > 1:
                tt = torch.tensor([ms], dtype=torch.float64, device=dev)
                dist.all_reduce(tt, op=dist.ReduceOp.MAX)
                ms = float(tt.item())
            return ms

        def run_serial(n):
            for _ in range(n):
                serial_step()

        def run_pipe(n):
            pipelined_e2e(torch, n, NB, copy_in, compute, copy_out, stream)

        n_e2e = max(3, min(args.steps, 20))
        run_serial(2)
        torch.cuda.synchronize()
        e_serial_ms = timed(run_serial, n_e2e)
        run_pipe(2 * NB)
        torch.cuda.synchronize()
        e_ms = timed(run_pipe, n_e2e)
        h2d = (x_host.numel() * x_host.element_size() + off_host.numel() * 8
               + ts_host.numel() * 8)
        d2h = y_hosts[0].numel() * y_hosts[0].element_size()
        e2e = {"value": world * T / (e_ms / 1000.0), "unit": "tokens/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "pipelining": "2 buffer sets; copy-in of step i+1 and copy-out of step i-1 "
                             "on their own streams overlap step i"}
        e2e_serial = {"value": world * T / (e_serial_ms / 1000.0), "unit": "tokens/s",
                      "ms_per_step": e_serial_ms}

    # ---------------- roofline of the dominant kernel (attention), from device events
    peaks, peak_src = load_peaks()
    attn_launches, attn_ms = kernels.get("attention", (0, 0.0))
    attn_flop = counts["attn_flop_per_layer"]  # algorithmic: causal pairs x H x 256
    attn_tflops = attn_flop / (attn_ms / attn_launches / 1000.0) / 1e12 if attn_launches else None
    peak_sus = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    roofline = {"kernel": "hstu_attn_kernel (causal)", "bound": "tensor",
                "achieved": attn_tflops, "peak": peak_sus, "unit": "TFLOP/s",
                "frac": (attn_tflops / peak_sus) if attn_tflops else None,
                "traffic": traffic_from_profiles("attention"),
                "peak_source": f"{peak_src} bf16 dense, sustained (kernel timed inside a long step)",
                "algorithmic_flop_per_launch": attn_flop,
                "ms_per_launch": attn_ms / attn_launches if attn_launches else None}
    kern = {}
    for name, (n, ms) in kernels.items():
        ent = {"launches": n, "ms_per_launch": ms / n, "share": ms / max(1e-9, sum(
            v[1] for v in kernels.values()))}
        if name == "f1_gemm":
            ent["tflops"] = counts["f1_flop_per_layer"] / (ms / n / 1000.0) / 1e12
            ent["frac_of_peak"] = ent["tflops"] / peak_sus
        if name == "f2_gemm":
            ent["tflops"] = counts["f2_flop_per_layer"] / (ms / n / 1000.0) / 1e12
            ent["frac_of_peak"] = ent["tflops"] / peak_sus
            # algorithmic bytes: AV, U (fp32), X residual (bf16 or fp32), Y fp32 (+bf16), W2
            T_, d, hv = T, cfgd.d_model, cfgd.num_heads * cfgd.dv
            byt = T_ * (hv * 4 * 2 + d * 4 + d * 4 + d * 2) + d * hv * 2
            ent["gbs_approx"] = byt / (ms / n / 1000.0) / 1e9
        if name == "attention":
            ent["tflops"] = attn_tflops
        kern[name] = ent
    gpu_launches = sum(n for n, _ in kernels.values())

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": cfgd.dtype, "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT[args.workload], "global_batch": world * case.cfg.batch
                       if args.workload != "sl-bf16" else world * len(case.lengths),
                       "seq_len": case.max_len, "tokens_per_step": world * T, "layers": L,
                       "l2": "flushed between timed steps (256 MiB write outside the events)",
                       "parallelism": f"dp{world}: users sharded, no collective"},
            "layer_tokens_per_s": value * L,
            "attention": {"tflops": attn_tflops,
                          "pct_of_bf16_peak_sustained": 100 * attn_tflops / peak_sus if attn_tflops else None,
                          "pct_of_bf16_peak_burst": 100 * attn_tflops / peaks["bf16_tflops"] if attn_tflops else None},
            "roofline": roofline, "kernels": kern, "gpu_launches": gpu_launches,
            "clocks": clocks, "e2e": e2e, "e2e_serial": e2e_serial}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_sample(case)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
