"""Benchmark: varlen block-diagonal attention of the 50-layer ViT-G/14 tower at 16384 tokens.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one forward of all 50 attention layers of the tower on a 128x128
patch grid (16384 tokens, H = 16, D = 96, bf16): 37 window layers (16 segments
of 32x32 = 1024 tokens) and 13 full layers (one 16384-token segment), fresh
N(0,1) Q/K/V per layer from seed + layer.  All 50 layers' inputs (7.5 GB) stay
resident, so every layer reads inputs larger than L2.

Metric: attention TFLOP/s (FLOPs = 4 * sum(L^2) * H * D, block-diagonal work
only) and ms per tower.  Prints ONE JSON line on rank 0.

--impl reference times the CPU oracle (plain f64 C) on a bounded sample of the
same workload: the reference arm, since the source pages ship no runnable
implementation of this path.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "vision attn TFLOP/s & % bf16 tensor peak; ms per 50-layer tower @16384 tok"
WORKLOAD = "tower16k: 50-layer ViT-G/14 vision-tower attention, 128x128 patches = 16384 tok, H=16, D=96"
GRID = 128
SCALE = 1.0 / math.sqrt(workloads.HEAD_DIM)
INLINE_SEGMENTS = 32  # the bf16 kernel builds the work list of calls this small itself
KERNEL_SRC = os.path.join(ROOT, "flash_attention_varlen_b200", "csrc", "attn_bf16_sm100.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_bf16_traffic.json")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-configuration timings of the smaller workloads")
    ap.add_argument("--e2e-steps", type=int, default=None,
                    help="steps of the host-buffer end-to-end measurement (default: min(steps, 3))")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="approximate CPU time budget of the oracle sample")
    ap.add_argument("--single-layer", choices=["full", "window", "varlen8", "f32_4096", "img448",
                                               "decoder_sliding", "decoder_full", "rope2d_window"],
                    default=None,
                    help="profiling aid: run only one layer (full = 1 x 16384 tok, window = "
                         "16 x 1024 tok, varlen8 = eight images of unequal size) warmup + "
                         "steps times and print its timing")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------- helpers

def rank_info():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_base_seed(rank: int) -> int:
    """Each rank runs its own image (weak scaling): layer l of rank r uses seed 1000*r + l."""
    return 1000 * rank


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """Max of a per-rank float over the process group (identity when not distributed)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return (float(d["bf16_tflops"]), float(d.get("hbm_gbs", 0.0)),
                "measured burst dense bf16 (MEASURED_PEAKS.json bf16_tflops)")
    return 1590.0, 6650.0, ("fallback: 1.59 PFLOP/s dense bf16 and 6.65 TB/s, an earlier "
                            "measurement on this pool (MEASURED_PEAKS.json absent)")


def kernel_sha() -> str:
    """Fingerprint of the hot kernel's code: sha256 of the source with comments and
    whitespace removed, so that a comment edit does not orphan committed counters."""
    with open(KERNEL_SRC) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    src = re.sub(r"\s+", "", src)
    return hashlib.sha256(src.encode()).hexdigest()[:16]


def traffic_per_launch():
    """DRAM bytes per launch from the committed ncu summary, if it is for this exact kernel source."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    if d.get("kernel_sha") != kernel_sha():
        return None, None
    return d.get("full_layer_bytes"), d.get("window_layer_bytes")


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        def num(x):
            try:
                return float(x)
            except ValueError:
                return float("nan")
        sm = [num(r[1]) for r in rows]
        mx = max(num(r[2]) for r in rows)
        power = [num(r[3]) for r in rows]
        loaded = [s for s, p in zip(sm, power) if p > 300] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(power)}


# ----------------------------------------------------------------------------- oracle timing

def oracle_sample(seconds: float, base_seed: int = 0):
    """Time the CPU oracle on a bounded sample of the tower and scale to tower TFLOP/s.

    Sample: one 1024-token window (all 16 heads) of window layer 0 and a growing
    number of (token, head) rows of full layer 3 until ~`seconds` elapse.
    Tower time estimate = 37 * 16 * t_window + 13 * (16384 * 16) * t_row.
    """
    import oracle
    threads = oracle.default_threads()
    lw = workloads.tower_layer_case(0, GRID, base_seed)
    L = 1024
    q, k, v = workloads.qkv(lw.seed, L, dtype="bf16")  # first window of layer 0's stream layout
    cu = np.array([0, L], np.int32)
    t0 = time.perf_counter()
    oracle.attn_fwd(q, k, v, cu, SCALE, threads=threads)
    t_window = time.perf_counter() - t0

    lf = workloads.tower_layer_case(3, GRID, base_seed)
    qf, kf, vf = lf.inputs()
    rows_done, t_rows = 0, 0.0
    rng = np.random.default_rng(0)
    batch = max(threads, 16)
    budget = max(0.5, seconds - t_window)
    while t_rows < budget and rows_done < 16384 * 16:
        tok = rng.integers(0, lf.T, batch).astype(np.int32)
        hd = rng.integers(0, lf.H, batch).astype(np.int32)
        t0 = time.perf_counter()
        oracle.attn_rows(qf, kf, vf, lf.cu_seqlens, SCALE, tok, hd, threads=threads)
        t_rows += time.perf_counter() - t0
        rows_done += batch
    t_row = t_rows / rows_done
    tower_s = 37 * 16 * t_window + 13 * (GRID * GRID * workloads.HEADS) * t_row
    tower_flops = sum(c.flops() for c in workloads.tower_cases(GRID, base_seed))
    value = tower_flops / tower_s / 1e12
    sample = (f"oracle f64 on 1 window (1024 tok x 16 heads, {t_window:.2f} s) + {rows_done} "
              f"(token, head) rows of a 16384-tok full layer ({t_rows:.2f} s); tower time "
              f"extrapolated as 37*16*t_window + 13*262144*t_row = {tower_s:.1f} s")
    return {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": sample, "tower_s_estimate": tower_s,
            "cpu_seconds": t_window + t_rows}


# ----------------------------------------------------------------------------- our arm

def run_ours(args):
    import torch
    import flash_attention_varlen_b200 as fa

    rank, world, local = rank_info()
    distributed = world > 1
    if distributed:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local if distributed else 0)
    torch.cuda.set_device(dev)

    base = rank_base_seed(rank)
    cases = workloads.tower_cases(GRID, base)
    T, H, D = GRID * GRID, workloads.HEADS, workloads.HEAD_DIM
    n_layers = len(cases)
    layer_flops = [c.flops() for c in cases]
    step_flops = sum(layer_flops)

    # inputs: generated on the host into pinned memory (also the e2e source), copied once
    pinned, dev_q, dev_k, dev_v, dev_o, dev_cu = [], [], [], [], [], []
    for c in cases:
        hq = torch.empty((T, H, D), dtype=torch.bfloat16, pin_memory=True)
        hk, hv = torch.empty_like(hq).pin_memory(), torch.empty_like(hq).pin_memory()
        for t, stream_id in ((hq, workloads.STREAM_Q), (hk, workloads.STREAM_K), (hv, workloads.STREAM_V)):
            workloads.normal(c.seed, stream_id, T * H * D, "bf16", out=t.view(torch.int16).numpy().view(np.uint16).reshape(-1))
        cu = torch.from_numpy(c.cu_seqlens.copy())
        pinned.append((hq, hk, hv, cu))
        dev_q.append(hq.to(dev, non_blocking=True))
        dev_k.append(hk.to(dev, non_blocking=True))
        dev_v.append(hv.to(dev, non_blocking=True))
        dev_o.append(torch.empty((T, H, D), dtype=torch.bfloat16, device=dev))
        dev_cu.append(cu.to(dev, non_blocking=True))
    torch.cuda.synchronize(dev)

    stream = torch.cuda.current_stream(dev)
    handle = stream.cuda_stream

    def one_step(ev=None):
        for l in range(n_layers):
            if ev is not None:
                ev[l][0].record(stream)
            rc = fa.vt_attn_fwd(dev_q[l].data_ptr(), dev_k[l].data_ptr(), dev_v[l].data_ptr(),
                                dev_o[l].data_ptr(), dev_cu[l].data_ptr(), cases[l].num_segments,
                                T, H, D, SCALE, fa.VT_DTYPE_BF16, handle)
            if rc != 0:
                raise fa.VtAttnError(rc, "vt_attn_fwd")
            if ev is not None:
                ev[l][1].record(stream)

    for _ in range(args.warmup):
        one_step()
    fa.check_device_status(stream)

    ev = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
           for _ in range(n_layers)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index)
    if distributed:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    t_start.record(stream)
    for s in range(args.steps):
        one_step(ev[s])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clock_info = clocks.stop()
    fa.check_device_status(stream)
    total_ms = t_start.elapsed_time(t_end)
    if distributed:
        total_ms = max_over_ranks(total_ms, dist, dev)
        dist.barrier()

    per_layer = np.array([[ev[s][l][0].elapsed_time(ev[s][l][1]) for l in range(n_layers)]
                          for s in range(args.steps)])  # ms
    full_idx = [l for l, c in enumerate(cases) if c.meta["full"]]
    win_idx = [l for l, c in enumerate(cases) if not c.meta["full"]]
    full_ms = float(per_layer[:, full_idx].mean())
    win_ms = float(per_layer[:, win_idx].mean())
    calls_ms = float(per_layer.sum())
    achieved = step_flops * args.steps / (calls_ms * 1e-3) / 1e12
    peak, hbm_peak, peak_src = measured_peaks()
    ms_per_step = total_ms / args.steps
    value = step_flops * args.steps * world / (total_ms * 1e-3) / 1e12

    # SM cycles per key-tile period of the busiest CTA (two 128-row Q tiles against one
    # 128-key tile): a guard on the kernel's per-clock speed that the power-capped clock
    # does not move (a build whose hot loop is laid out worse shows up here)
    num_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    sm_mhz = clock_info.get("sm_mhz") if isinstance(clock_info, dict) else None

    def cycles_per_period(case, ms):
        periods = key_tile_periods(case.cu_seqlens, H, num_sms)
        return round(ms * 1e-3 * sm_mhz * 1e6 / periods) if sm_mhz else None

    full_traffic, win_traffic = traffic_per_launch()
    traffic = None
    if full_traffic is not None and win_traffic is not None:
        traffic = (13 * full_traffic + 37 * win_traffic) / 50.0

    # end-to-end through the public API with host buffers (pinned H2D, kernel, D2H)
    e2e_steps = args.e2e_steps if args.e2e_steps is not None else min(args.steps, 3)
    e2e = run_e2e(fa, torch, dev, pinned, cases, e2e_steps, step_flops, world,
                  dist if distributed else None)

    # the other configurations of the workload, one layer each (informational): after the
    # timed region, on this rank's GPU
    outputs = {} if (rank == 0 and not args.no_cpu_baseline) else None
    configs = time_configs(fa, torch, dev, keep_outputs=outputs) if not args.no_configs else None

    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic: Q,K,V ~ N(0,1) bf16 per layer from a seeded SplitMix64/Box-Muller stream",
        "config": {
            "workload": WORKLOAD,
            "layers": "37 window (16 x 1024 tok) + 13 full (1 x 16384 tok)",
            "tokens": T, "heads": H, "head_dim": D, "scale": "1/sqrt(96)",
            "flops_per_step": step_flops,
            "l2": "inputs larger than L2: 150 MB of Q/K/V per layer, 7.5 GB resident over 50 layers",
            "parallelism": f"replica per GPU x{world} (independent towers, no collective)",
        },
        "pct_of_bf16_peak": round(100.0 * achieved / peak, 2),
        "layers": {
            "full_16384": {"ms": round(full_ms, 4),
                           "tflops": round(layer_flops[full_idx[0]] / (full_ms * 1e-3) / 1e12, 2),
                           "sm_cycles_per_key_tile_period": cycles_per_period(cases[full_idx[0]], full_ms)},
            "window_16x1024": {"ms": round(win_ms, 4),
                               "tflops": round(layer_flops[win_idx[0]] / (win_ms * 1e-3) / 1e12, 2),
                               "sm_cycles_per_key_tile_period": cycles_per_period(cases[win_idx[0]], win_ms)},
        },
        "roofline": {
            "bound": "tensor",
            "achieved": round(achieved, 2),
            "peak": peak,
            "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "peak_source": peak_src,
            "traffic": traffic,
            "kernel": "attn_bf16_kernel (calls of at most 32 segments, as in the tower, schedule themselves; a prepass would be timed with its call)",
            "per_launch": "4*sum(L^2)*H*D FLOPs of the call / CUDA-event duration of the call, "
                          "averaged FLOP-weighted over the 50 calls of a step",
        },
        "configs": configs,
        # one launch per call; a call of more than 32 segments adds the scheduling prepass
        "gpu_launches": args.steps * sum(1 if c.num_segments <= INLINE_SEGMENTS else 2 for c in cases),
        "e2e": e2e,
        "clocks": clock_info,
    }
    if rank == 0 and not args.no_cpu_baseline:
        result["cpu_baseline"] = oracle_sample(args.cpu_seconds)
        if configs:
            for name, entry in oracle_per_config(outputs).items():
                configs[name]["vs_oracle"] = entry
    if distributed:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def key_tile_periods(cu_seqlens, H: int, num_sms: int) -> int:
    """Key-tile periods of the busiest CTA of a bf16 call with equal-cost units: units of
    256 query rows per (segment, head), dealt over min(units, SMs) persistent CTAs, each
    unit taking one period per 128-key tile of its segment (the longest segment's count)."""
    lengths = np.diff(np.asarray(cu_seqlens, np.int64))
    units = int(sum(-(-int(n) // 256) for n in lengths if n > 0)) * H
    per_cta = -(-units // min(units, num_sms))
    return per_cta * -(-int(lengths.max()) // 128)


def config_cases():
    return [workloads.tiny_case("bf16"), workloads.tiny_case("f32"), workloads.image448_case(),
            workloads.image448_case(True), *workloads.image896_cases(), workloads.varlen8_case()]


def bf16_round(x):
    """f64 values rounded to the nearest bf16 (ties to even), kept in f64."""
    x = np.asarray(x, np.float64)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126))) - 7)
    return np.round(x / ulp) * ulp


def oracle_per_config(outputs):
    """CPU-baseline leg, per configuration: the oracle (f64, all host cores) timed on each
    configuration's whole input, and the GPU output's error against it: max/mean-abs, the
    max-abs against the oracle rounded to bf16 (the output's own rounding floor), and
    max |O|.  Runs after the timed region; `outputs` maps a configuration name to
    (case, GPU output as f64)."""
    import oracle
    threads = oracle.default_threads()
    res = {}
    for name, item in outputs.items():
        if item[0] == "decoder":
            res[name] = decoder_vs_oracle(*item[1:])
            continue
        if item[0] == "rope2d":
            res[name] = rope2d_vs_oracle(*item[1:])
            continue
        c, got = item
        q, k, v = c.inputs()
        t0 = time.perf_counter()
        ref = oracle.attn_fwd(q, k, v, c.cu_seqlens, SCALE, threads=threads)
        dt = time.perf_counter() - t0
        err = np.abs(got - ref)
        entry = {"max_abs": float(err.max()), "mean_abs": float(err.mean()),
                 "max_abs_O": float(np.abs(ref).max()), "finite": bool(np.isfinite(got).all()),
                 "oracle_s": round(dt, 3), "oracle_tflops": round(c.flops() / dt / 1e12, 5),
                 "cores": threads}
        if c.dtype == "bf16":
            entry["max_abs_vs_bf16_oracle"] = float(np.abs(got - bf16_round(ref)).max())
            entry["within_bound"] = bool(err.max() <= 1e-2 and err.mean() <= 1e-3)
        else:
            entry["within_bound"] = bool(err.max() <= 1e-5)
        res[name] = entry
    return res


def rope2d_vs_oracle(inputs, got):
    """The RoPE attention output against the oracle (rotate in f64, then attention) on one
    row of every (256-row block, head) unit, alternating ends of the block."""
    from oracle import rope
    q, k, v, cu, pos = inputs
    T, H = q.shape[0], q.shape[1]
    blocks = np.arange(0, T, 256)
    tok = np.concatenate([blocks + (h % 2) * 255 for h in range(H)])
    head = np.repeat(np.arange(H), len(blocks))
    t0 = time.perf_counter()
    ref = rope.attn_rows_rope2d(q, k, v, cu, SCALE, pos, tok, head)
    dt = time.perf_counter() - t0
    err = np.abs(got[tok, head] - ref)
    return {"rows": int(len(tok)), "max_abs": float(err.max()), "mean_abs": float(err.mean()),
            "max_abs_O": float(np.abs(ref).max()), "finite": bool(np.isfinite(got).all()),
            "within_bound": bool(err.max() <= 1e-2 and err.mean() <= 1e-3),
            "oracle_s_rows": round(dt, 3)}


def decoder_vs_oracle(inputs, got):
    """The decoder output against its oracle on one row of every 128-row block of each
    query head, alternating ends of the block: errors, max |O| and the oracle's time."""
    from oracle import decoder
    q, k, v, cu, window, scale = inputs
    T, Hq = q.shape[0], q.shape[1]
    blocks = np.arange(0, T, 128)
    tok = np.concatenate([blocks + (h % 2) * 127 for h in range(Hq)])
    head = np.repeat(np.arange(Hq), len(blocks))
    t0 = time.perf_counter()
    ref = decoder.attn_rows(q, k, v, cu, scale, window, tok, head)
    dt = time.perf_counter() - t0
    err = np.abs(got[tok, head] - ref)
    return {"rows": int(len(tok)), "max_abs": float(err.max()), "mean_abs": float(err.mean()),
            "max_abs_O": float(np.abs(ref).max()), "finite": bool(np.isfinite(got).all()),
            "max_abs_vs_bf16_oracle": float(np.abs(got[tok, head] - bf16_round(ref)).max()),
            "within_bound": bool(err.max() <= 1e-2 and err.mean() <= 1e-3),
            "oracle_s_rows": round(dt, 3), "cores": 1}


def time_configs(fa, torch, dev, calls: int = 20, warmup: int = 3, keep_outputs=None):
    """ms per call and TFLOP/s of each smaller configuration of the workload (one layer, the
    inputs resident; calls back to back, so these small cases run partly out of L2).  With
    `keep_outputs` (a dict), each configuration's output is stored there, as f64 on the host,
    for the error check after the timed region."""
    cases = config_cases()
    stream = torch.cuda.current_stream(dev)
    out = {}
    for c in cases:
        q, k, v = c.inputs()
        if c.dtype == "bf16":
            to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
            code = fa.VT_DTYPE_BF16
        else:
            to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
            code = fa.VT_DTYPE_F32
        dq, dk, dv = to(q), to(k), to(v)
        do = torch.empty_like(dq)
        cu = torch.from_numpy(c.cu_seqlens.copy()).to(dev)

        def call():
            rc = fa.vt_attn_fwd(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), do.data_ptr(),
                                cu.data_ptr(), c.num_segments, c.T, c.H, c.D, SCALE, code,
                                stream.cuda_stream)
            if rc != 0:
                raise fa.VtAttnError(rc, "vt_attn_fwd")
        for _ in range(warmup):
            call()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(calls):
            call()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        fa.check_device_status(stream)
        ms = e0.elapsed_time(e1) / calls
        out[c.name] = {"dtype": c.dtype, "segments": c.num_segments, "tokens": c.T,
                       "ms": round(ms, 4), "tflops": round(c.flops() / (ms * 1e-3) / 1e12, 2)}
        if keep_outputs is not None:
            keep_outputs[c.name] = (c, do.float().cpu().numpy().astype(np.float64))
    try:  # informational: must never cost the headline line
        out["window_segmentation_128x128"] = time_window_segmentation(fa, torch, dev, calls)
    except Exception as exc:  # noqa: BLE001
        out["window_segmentation_128x128"] = {"error": str(exc)[:200]}
    try:  # informational
        out["rope2d_window_16x1024"] = time_rope2d(fa, torch, dev, calls, keep_outputs)
    except Exception as exc:  # noqa: BLE001
        out["rope2d_window_16x1024"] = {"error": str(exc)[:200]}
    for window in (workloads.DECODER_WINDOW, 0):
        name = f"decoder_{'sliding' if window else 'full'}_16384"
        try:  # informational, like the segmentation timings
            out[name] = time_decoder(fa, torch, dev, window, 10, keep_outputs, name)
        except Exception as exc:  # noqa: BLE001
            out[name] = {"error": str(exc)[:200]}
    return out


def time_rope2d(fa, torch, dev, calls: int, keep_outputs):
    """The tower's window layer (16 x 1024 tokens in window order) with the 2D RoPE: the
    attention over rope(Q), rope(K) (one pass rotates both, then the attention) beside the
    plain attention on the same inputs, and the rotation pass over K alone in GB/s, timed
    as a CUDA graph of 20 passes so the host's per-call cost does not hide in it."""
    case = workloads.tower_layer_case(0, GRID)
    q, k, v = case.inputs()
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    dq, dk, dv = to(q), to(k), to(v)
    do, k_rot = torch.empty_like(dq), torch.empty_like(dk)
    cu = torch.from_numpy(case.cu_seqlens.copy()).to(dev)
    perm, _ = fa.window_partition([(GRID, GRID)], 32, device=dev)
    pos = torch.from_numpy(workloads.patch_positions(GRID, GRID)).to(dev)[perm.long()].contiguous()
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(calls):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        fa.check_device_status(stream)
        return e0.elapsed_time(e1) / calls
    plain = timed(lambda: fa.attn_fwd(dq, dk, dv, cu, scale=SCALE, out=do))
    rope = timed(lambda: fa.attn_fwd_rope2d(dq, dk, dv, cu, pos, scale=SCALE, out=do, k_rot=k_rot))
    side = torch.cuda.Stream(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        fa.rope2d(dk, pos, out=k_rot, stream=side)
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(graph, stream=side):
            for _ in range(20):
                fa.rope2d(dk, pos, out=k_rot, stream=side)
    torch.cuda.synchronize(dev)
    kpass = timed(graph.replay) / 20
    del graph
    moved = 2 * dk.numel() * dk.element_size() + pos.numel() * pos.element_size()
    _, hbm_peak, _ = measured_peaks()
    gbs = moved / (kpass * 1e-3) / 1e9
    if keep_outputs is not None:
        keep_outputs["rope2d_window_16x1024"] = ("rope2d", (q, k, v, case.cu_seqlens, pos.cpu().numpy()),
                                                  do.float().cpu().numpy().astype(np.float64))
    return {"dtype": "bf16", "tokens": case.T, "segments": case.num_segments,
            "ms_attn_rope2d": round(rope, 4), "ms_attn_plain": round(plain, 4),
            "rope_overhead_pct": round(100.0 * (rope - plain) / plain, 1),
            "tflops_attn_rope2d": round(case.flops() / (rope * 1e-3) / 1e12, 2),
            "ms_k_rotation": round(kpass, 4), "k_rotation_gbs": round(gbs, 1),
            "k_rotation_frac_of_hbm_peak": round(gbs / hbm_peak, 3) if hbm_peak else None}


def time_decoder(fa, torch, dev, window: int, calls: int, keep_outputs, name: str):
    """The text decoder's attention (causal, GQA 32/2, head size 128) on one 16384-token
    sequence: a sliding layer (window 2048) or a full one (window 0); ms per call and
    TFLOP/s of the attended (query, key) pairs."""
    T = 16384
    cu_np = workloads.cu_from_lengths([T])
    q, k, v = workloads.decoder_qkv(77, T)
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    dq, dk, dv = to(q), to(k), to(v)
    do = torch.empty_like(dq)
    cu = torch.from_numpy(cu_np.copy()).to(dev)
    stream = torch.cuda.current_stream(dev)
    scale = 1.0 / math.sqrt(workloads.DECODER_D)

    def call():
        rc = fa._binding.vt_attn_fwd_swa(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), do.data_ptr(),
                                         cu.data_ptr(), 1, T, workloads.DECODER_HQ, workloads.DECODER_HKV,
                                         workloads.DECODER_D, scale, window, stream.cuda_stream)
        if rc != 0:
            raise fa.VtAttnError(rc, "vt_attn_fwd_swa")
    for _ in range(3):
        call()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(calls):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    fa.check_device_status(stream)
    ms = e0.elapsed_time(e1) / calls
    flops = workloads.decoder_flops(cu_np, window)
    if keep_outputs is not None:
        keep_outputs[name] = ("decoder", (q, k, v, cu_np, window, scale),
                              do.float().cpu().numpy().astype(np.float64))
    return {"dtype": "bf16", "kind": "causal, GQA 32/2, head size 128", "window": window,
            "tokens": T, "ms": round(ms, 4), "tflops": round(flops / (ms * 1e-3) / 1e12, 2)}


def time_window_segmentation(fa, torch, dev, calls: int = 20):
    """The tower image's window order built on the device, and one [16384, 16, 96] bf16
    tensor put in that order (the tower does this once before its layers and once after)."""
    stream = torch.cuda.current_stream(dev)
    perm, cu = fa.window_partition([(GRID, GRID)], 32, device=dev)
    x = torch.empty((GRID * GRID, workloads.HEADS, workloads.HEAD_DIM), dtype=torch.bfloat16,
                    device=dev).normal_()
    y = torch.empty_like(x)
    for _ in range(3):
        fa.window_partition([(GRID, GRID)], 32, device=dev)
        fa.permute_rows(x, perm, out=y)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    ev[0].record(stream)
    for _ in range(calls):
        fa.window_partition([(GRID, GRID)], 32, device=dev)
    ev[1].record(stream)
    ev[2].record(stream)
    for _ in range(calls):
        fa.permute_rows(x, perm, out=y)
    ev[3].record(stream)
    torch.cuda.synchronize(dev)
    part_ms = ev[0].elapsed_time(ev[1]) / calls
    perm_ms = ev[2].elapsed_time(ev[3]) / calls
    moved = 2 * x.numel() * x.element_size()  # read + write of every row
    _, hbm_peak, _ = measured_peaks()
    gbs = moved / (perm_ms * 1e-3) / 1e9
    return {"partition_us": round(1e3 * part_ms, 2), "windows": int(cu.numel() - 1),
            "permute_ms": round(perm_ms, 4), "permute_gbs": round(gbs, 1),
            "permute_frac_of_hbm_peak": round(gbs / hbm_peak, 3) if hbm_peak else None,
            "note": "partition includes its host-side checks and launch; permute moves "
                    "2 x 50.3 MB per call"}


def run_e2e(fa, torch, dev, pinned, cases, steps, step_flops, world, dist):
    """Same tower through attn_fwd_host: per layer H2D of Q/K/V/cu from pinned memory,
    the kernel, D2H of the output; two streams with their own device buffers overlap
    one layer's copies with the other's compute."""
    T, H, D = GRID * GRID, workloads.HEADS, workloads.HEAD_DIM
    streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
    bufs = []
    for _ in range(2):
        dq = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
        bufs.append((dq, torch.empty_like(dq), torch.empty_like(dq), torch.empty_like(dq),
                     torch.empty(cases[0].num_segments + 1, dtype=torch.int32, device=dev)))
    outs = [torch.empty((T, H, D), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    cu_bufs = {}

    def step():
        for l, c in enumerate(cases):
            i = l & 1
            hq, hk, hv, cu = pinned[l]
            dq, dk, dv, do, _ = bufs[i]
            key = (i, c.num_segments)
            if key not in cu_bufs:
                cu_bufs[key] = torch.empty(c.num_segments + 1, dtype=torch.int32, device=dev)
            fa.attn_fwd_host(hq, hk, hv, cu, outs[i], scale=SCALE,
                             device_buffers=(dq, dk, dv, do, cu_bufs[key]), stream=streams[i])

    step()
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    t0 = time.perf_counter()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(streams[0])
    streams[1].wait_event(ev0)
    for _ in range(steps):
        step()
    ev_end1 = torch.cuda.Event()
    ev_end1.record(streams[1])
    streams[0].wait_event(ev_end1)
    ev1.record(streams[0])
    torch.cuda.synchronize(dev)
    wall = time.perf_counter() - t0
    ms = max_over_ranks(ev0.elapsed_time(ev1), dist, dev)
    h2d = sum(3 * T * H * D * 2 + (c.num_segments + 1) * 4 for c in cases)
    d2h = len(cases) * T * H * D * 2
    return {"value": round(step_flops * steps * world / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms / steps, 3), "steps": steps,
            "wall_ms_per_step": round(1e3 * wall / steps, 3),
            "path": "flash_attention_varlen_b200.attn_fwd_host (pinned H2D -> vt_attn_fwd -> D2H), "
                    "2 streams"}


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    rank, world, _ = rank_info()
    if rank != 0:
        return
    per_step = max(1.0, min(20.0, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(per_step)
    vals, cpu_s, info = [], 0.0, None
    for _ in range(args.steps):
        info = oracle_sample(per_step)
        vals.append(info["value"])
        cpu_s += info["cpu_seconds"]
    value = statistics.median(vals)
    tower_s = info["tower_s_estimate"]
    out = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * tower_s, 1),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic: the same seeded bf16 Q,K,V as the GPU arm, widened to f64",
        "config": {"workload": WORKLOAD, "tokens": GRID * GRID, "heads": workloads.HEADS,
                   "head_dim": workloads.HEAD_DIM},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": info["cores"],
                         "kind": "oracle", "sample": info["sample"]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "note": "reference arm = the plain f64 CPU oracle, each step a bounded sample of the tower",
    }
    print(json.dumps(out), flush=True)


def run_single_layer(args):
    """One layer, called warmup + steps times (for ncu captures): a tower layer type, the
    eight-image batch, a 4096-token f32 segment (the f32 arm), the text decoder's sliding
    or full layer on a 16384-token sequence, or the tower's window layer with the 2D RoPE
    (the rotation pass over Q and K, then the attention)."""
    import torch
    import flash_attention_varlen_b200 as fa
    dev = torch.device("cuda", 0)
    bf16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    if args.single_layer.startswith("decoder_"):
        window = workloads.DECODER_WINDOW if args.single_layer == "decoder_sliding" else 0
        cu_np = workloads.cu_from_lengths([GRID * GRID])
        q, k, v = workloads.decoder_qkv(77, GRID * GRID)
        dq, dk, dv = bf16(q), bf16(k), bf16(v)
        flops = workloads.decoder_flops(cu_np, window)
        cu = torch.from_numpy(cu_np.copy()).to(dev)
        out = torch.empty_like(dq)
        call = lambda: fa.attn_fwd_swa(dq, dk, dv, cu, window=window, out=out)
    else:
        if args.single_layer == "varlen8":  # eight images of unequal size (the scheduler's case)
            case = workloads.varlen8_case(0)
        elif args.single_layer == "img448":  # one 448 x 448 image: split-key units
            case = workloads.image448_case()
        elif args.single_layer == "f32_4096":
            case = workloads.Case("f32_4096", workloads.cu_from_lengths([4096]), seed=5, dtype="f32")
        else:
            case = workloads.tower_layer_case(3 if args.single_layer == "full" else 0, GRID)
        q, k, v = case.inputs()
        to = bf16 if case.dtype == "bf16" else (lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev))
        dq, dk, dv = to(q), to(k), to(v)
        flops = case.flops()
        cu = torch.from_numpy(case.cu_seqlens.copy()).to(dev)
        out = torch.empty_like(dq)
        call = lambda: fa.attn_fwd(dq, dk, dv, cu, scale=SCALE, out=out)
        if args.single_layer == "rope2d_window":
            perm, _ = fa.window_partition([(GRID, GRID)], 32, device=dev)
            pos = torch.from_numpy(workloads.patch_positions(GRID, GRID)).to(dev)[perm.long()].contiguous()
            k_rot = torch.empty_like(dk)
            call = lambda: fa.attn_fwd_rope2d(dq, dk, dv, cu, pos, scale=SCALE, out=out, k_rot=k_rot)
    for _ in range(args.warmup):
        call()
    fa.check_device_status()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        call()
    e1.record()
    torch.cuda.synchronize()
    fa.check_device_status()
    ms = e0.elapsed_time(e1) / max(1, args.steps)
    print(json.dumps({"single_layer": args.single_layer, "ms_per_call": round(ms, 4),
                      "tflops": round(flops / (ms * 1e-3) / 1e12, 2),
                      "calls": args.steps, "note": "back-to-back calls on one layer's inputs"}))


def check_world(args):
    """--gpus N must match the number of ranks launched (torchrun sets WORLD_SIZE; a plain
    `python bench.py` is one rank): N replicas come from torchrun, never from this flag."""
    _, world, _ = rank_info()
    if args.gpus != world:
        sys.stderr.write(f"bench.py: --gpus {args.gpus} but {world} rank(s) were launched; run "
                         f"`python -m torch.distributed.run --nproc-per-node {args.gpus} bench.py "
                         f"--gpus {args.gpus} ...` for more than one GPU\n")
        sys.exit(2)


def main(argv=None):
    args = parse_args(argv)
    check_world(args)
    if args.single_layer:
        run_single_layer(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
