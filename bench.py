"""Benchmark of the fused LoRA-adapted linear layer, forward + backward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config q_proj]

One step = one forward (lora_linear_fwd) and one backward (lora_linear_bwd)
over one batch of synthetic bf16 inputs of the workload (default: the
Llama-3-8B q_proj shape, M = 16384 tokens, 4096 -> 4096, r = 8, alpha = 16).
Algorithmic work per step: 4 M d_in d_out + 6 M r (d_in + d_out) FLOPs.

Timing: W untimed warm-up steps, then K steps, each timed with CUDA events on
the stream the library launches on; the L2 cache is flushed (a 512 MiB write)
before every timed step, outside the events; a barrier + synchronize brackets
the timed region and the time is the max over ranks.  N > 1 runs N independent
replicas (one process per GPU, launched by torch.distributed.run): the layer
has no exchange step, so there is no collective on the data path.

Prints one JSON line (rank 0).  ``--impl reference`` times the fp64 CPU oracle
on the host cores instead (a bounded sample of the same workload per step).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import seeded_inputs  # noqa: E402

METRIC = "LoRA-linear fwd+bwd TFLOP/s (M=16384, 4096², r=8) & % of B200 roofline"
METRIC_QKV = "LoRA attention-input block (RMSNorm + q/k/v + rotary) fwd+bwd TFLOP/s & % of B200 roofline"
UNIT = "TFLOP/s"


def step_flops(M, d_in, d_out, r, act="identity"):
    """Algorithmic FLOPs of one forward + backward (SwiGLU: two projections)."""
    np_ = 2 if act == "swiglu" else 1
    return np_ * (4.0 * M * d_in * d_out + 6.0 * M * r * (d_in + d_out))


def fwd_flops(M, d_in, d_out, r, act="identity"):
    np_ = 2 if act == "swiglu" else 1
    return np_ * (2.0 * M * d_in * d_out + 2.0 * M * r * (d_in + d_out))


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        # scratch: the samples are summarised into the JSON line
        self.path = os.path.join(tempfile.gettempdir(), f"lora_bench_clocks_rank{gpu_index}_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        # nvidia-smi takes a moment to start: wait (at most 2 s) for its first
        # sample so that a short timed region is still sampled
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < 2.0 and self.proc.poll() is None:
            self.f.flush()
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.01)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return None
        busy = [r for r in rows if r[2] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in busy for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in busy), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(busy)}


# ---------------------------------------------------------------------------
# the oracle on the host cores (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------
def is_qkv(cfg):
    return "d_kv" in cfg


def cfg_step_flops(cfg, M):
    """FLOPs of one step of a workload at M tokens: the attention-input block
    counts its three projections (the norm and the rotation are O(M d) and not
    counted)."""
    if is_qkv(cfg):
        return sum(step_flops(M, cfg["d_in"], n, cfg["r"]) for n in qkv_douts(cfg))
    return step_flops(M, cfg["d_in"], cfg["d_out"], cfg["r"], cfg["act"])


def qkv_douts(cfg):
    return (cfg["d_out"], cfg["d_kv"], cfg["d_kv"])


def qkv_inputs(cfg, M, seed):
    """Host inputs of the attention-input block: bf16 bits (X, g, W_j, A_j, B_j,
    dY_j for j = q, k, v), int32 positions (whole sequences), fp32 tables."""
    d, r = cfg["d_in"], cfg["r"]
    out = {"X": seeded_inputs.draw("X", (M, d), seed, d), "g": seeded_inputs.draw_norm_weight(d, seed)}
    for j, d_out in enumerate(qkv_douts(cfg)):
        inp = seeded_inputs.make_inputs(M, d, d_out, r, "identity", seed=seed * 10 + j)
        for k in ("W", "A", "B", "dY"):
            out[f"{k}{j}"] = inp[k]
    out["pos"] = seeded_inputs.sequence_positions(M, cfg["seq_len"])
    out["cos"], out["sin"] = seeded_inputs.rotary_tables(cfg["seq_len"], cfg["head_dim"])
    return out


def oracle_sample_run(cfg, rows, inp_f64):
    import oracle
    g = inp_f64
    if is_qkv(cfg):
        from oracle import norm_rope_oracle
        projs = [{k: g[f"{k}{j}"] for k in ("W", "A", "B")} for j in range(3)]
        t0 = time.perf_counter()
        norm_rope_oracle.qkv_backward([g[f"dY{j}"][:rows] for j in range(3)], g["X"][:rows], g["g"],
                                      float(np.float32(cfg["eps"])), projs, cfg["alpha"] / cfg["r"],
                                      [True, True, False], g["pos"][:rows], g["cos"], g["sin"], cfg["head_dim"])
        return time.perf_counter() - t0
    X = g["X"][:rows]
    dY = g["dY"][:rows]
    t0 = time.perf_counter()
    oracle.lora_backward(dY, X, g["W"], g["A"], g["B"], cfg["alpha"] / cfg["r"], cfg["act"],
                         g.get("W_up"), g.get("A_up"), g.get("B_up"))
    return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(cfg, budget_s=12.0, max_rows=None):
    """Time the oracle on growing row samples until ~budget_s of CPU work."""
    import oracle
    M, d_in, d_out, r = cfg["M"], cfg["d_in"], cfg["d_out"], cfg["r"]
    rows_cap = max_rows or (4096 if is_qkv(cfg) else M)
    g = oracle_inputs(cfg, min(M, rows_cap))
    rows = 16
    spent = 0.0
    best = None
    while True:
        dt = oracle_sample_run(cfg, rows, g)
        spent += dt
        best = (rows, dt)
        if dt > budget_s / 3 or rows >= min(M, rows_cap) or spent > budget_s:
            break
        rows = min(rows * 4, min(M, rows_cap))
    rows, dt = best
    # repeat the chosen sample until ~budget_s / 2 of work has been timed
    times = [dt]
    while sum(times) < budget_s / 2 and len(times) < 20:
        times.append(oracle_sample_run(cfg, rows, g))
    dt = statistics.mean(times)
    val = cfg_step_flops(cfg, rows) / dt / 1e12
    what = (f"the norm, q/k/v projections ({d_in}->{'/'.join(map(str, qkv_douts(cfg)))}) and rotation"
            if is_qkv(cfg) else f"({d_in}->{d_out})")
    return {"value": val, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"fp64 numpy oracle fwd+bwd on the first {rows} of {M} tokens "
                      f"{what}, r={r}; mean of {len(times)} runs of {dt:.2f} s; FLOPs by the same formula"}


def oracle_inputs(cfg, M):
    """The workload's inputs for the oracle (float64; positions and tables as given)."""
    import oracle
    if is_qkv(cfg):
        raw = qkv_inputs(cfg, M, 0)
        return {k: (v.astype(np.float64) if k in ("cos", "sin") else v if k == "pos" else oracle.bf16_to_f64(v))
                for k, v in raw.items()}
    inp = seeded_inputs.make_inputs(M, cfg["d_in"], cfg["d_out"], cfg["r"], cfg["act"], seed=0)
    return {k: oracle.bf16_to_f64(v) for k, v in inp.items()}


def run_reference(args, cfg, world, rank):
    if rank != 0:
        return
    steps, warm = args.steps, args.warmup
    g = oracle_inputs(cfg, min(cfg["M"], 4096))
    # rows per step: sized so the whole warm-up + timed run stays within a few minutes
    rows = 64
    while rows < 4096:
        dt = oracle_sample_run(cfg, rows, g)
        if dt * (steps + warm) > 60.0 or dt > 2.0:
            break
        rows *= 2
    for _ in range(warm):
        oracle_sample_run(cfg, rows, g)
    tot = 0.0
    for _ in range(steps):
        tot += oracle_sample_run(cfg, rows, g)
    val = cfg_step_flops(cfg, rows) * steps / tot / 1e12
    shape = (f"norm + {cfg['d_in']}->{'/'.join(map(str, qkv_douts(cfg)))} + rotary" if is_qkv(cfg)
             else f"{cfg['d_in']}->{cfg['d_out']}")
    sample = f"fp64 numpy oracle fwd+bwd on {rows} of {cfg['M']} tokens per step ({shape}, r={cfg['r']})"
    line = {"impl": "reference", "metric": METRIC_QKV if is_qkv(cfg) else METRIC, "value": val, "unit": UNIT, "n_gpus": world, "steps": steps,
            "warmup": warm, "ms_per_step": tot / steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.config, "M": cfg["M"], "d_in": cfg["d_in"], "d_out": cfg["d_out"],
                       "r": cfg["r"], "alpha": cfg["alpha"], "act": cfg["act"], "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# multi-rank helpers (replicas: one process per GPU, no collective on the data
# path; ranks only meet for the timing barrier and the max over ranks)
# ---------------------------------------------------------------------------
def max_over_ranks(x, dist, device):
    """The largest value of x over all ranks (x itself without a process group)."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_step, steps, world, max_ms):
    """Whole-job throughput: the units all ranks processed / the slowest rank's time."""
    return units_per_step * steps * world / (max_ms * 1e-3)


def committed_traffic(workload, record="gemm_traffic.json", source="lora_mma.cuh"):
    """DRAM bytes per launch of a kernel from a committed ncu summary, valid
    only while the kernel source is unchanged (else None)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", record)) as f:
            rec = json.load(f)
        src = open(os.path.join(ROOT, "lora_linear_fine_b200", "csrc", source), "rb").read()
        if rec.get("kernel_sha256") != hashlib.sha256(src).hexdigest():
            return None
        return rec.get("per_launch_bytes", {}).get(workload)
    except Exception:
        return None


def run_small_m(args, cfg, fwd, flush, stream, L, world, rank, dist):
    """Few tokens: forward only, bound by reading W once (HBM roofline)."""
    import torch
    M, d_in, d_out, r = cfg["M"], cfg["d_in"], cfg["d_out"], cfg["r"]
    for _ in range(args.warmup):
        fwd()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    launches0 = L.lora_linear_launch_count()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        fwd()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    launches = L.lora_linear_launch_count() - launches0
    ms = [a.elapsed_time(b) for a, b in ev]
    med = statistics.median(ms)
    F = fwd_flops(M, d_in, d_out, r)
    w4 = cfg.get("weight") == "w4"
    # the base weight: bf16, or 4-bit codes plus one bf16 scale per row and 64 features
    w_bytes = (d_out * d_in / 2.0 + 2.0 * d_out * (d_in // 64)) if w4 else 2.0 * d_out * d_in
    byts = w_bytes + 2.0 * (M * d_in + r * d_in + d_out * r + M * d_out) + 4.0 * M * r
    peaks = read_peaks()
    gbs = byts / (med * 1e-3) / 1e9
    line = {"metric": "LoRA-linear forward (few tokens), HBM roofline", "value": round(F / (med * 1e-3) / 1e12, 3),
            "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(med, 5), "timing": "median of per-step CUDA events",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": args.config, "M": M, "d_in": d_in, "d_out": d_out, "r": r,
                       "alpha": cfg["alpha"], "act": cfg["act"], "weight": "w4g64" if w4 else "bf16",
                       "l2": "flushed before each timed step (512 MiB write)"},
            "roofline": {"kernel": "small_m_kernel" if M <= 64 else "lora_gemm_kernel (forward)", "bound": "hbm",
                         "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4),
                         "traffic": committed_traffic(args.config, "small_m_traffic.json", "lora_small_m.cuh")
                         if M <= 64 else None,
                         "bytes_per_launch": byts},
            "gpu_launches": int(launches)}
    if rank == 0:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_qkv(args, cfg, L, world, rank, local, dist):
    """The attention-input block: RMSNorm, the q, k, v projections (q and k
    rotated in the GEMM epilogue), their backward, and the norm's backward over
    the three input gradients; every step through the C ABI."""
    import torch
    M, d, r, hd, eps = cfg["M"], cfg["d_in"], cfg["r"], cfg["head_dim"], cfg["eps"]
    douts = qkv_douts(cfg)
    s = cfg["alpha"] / r
    n_pos = cfg["seq_len"]
    raw = qkv_inputs(cfg, M, rank)
    host = {k: (torch.from_numpy(v.view(np.int16)).view(torch.bfloat16) if v.dtype == np.uint16
                else torch.from_numpy(v)).pin_memory() for k, v in raw.items()}
    t = {k: v.to("cuda", non_blocking=True) for k, v in host.items()}
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    p = lambda x: None if x is None else x.data_ptr()  # noqa: E731
    descs = [L.make_desc(M, d, n, r, s, "identity") for n in douts]
    ws = L.Workspace(max(max(L.lora_linear_workspace_size_rope(x, 1), L.lora_linear_workspace_size(x, 1))
                         for x in descs))
    bf, f32 = torch.bfloat16, torch.float32
    Xn = torch.empty((M, d), dtype=bf, device="cuda")
    rstd = torch.empty(M, dtype=f32, device="cuda")
    o = {"Y": [torch.empty((M, n), dtype=bf, device="cuda") for n in douts],
         "T": [torch.empty((M, r), dtype=f32, device="cuda") for _ in douts],
         "dXn": torch.empty((M, d), dtype=f32, device="cuda"),     # fp32 sum of the three input gradients
         "dA": [torch.empty((r, d), dtype=f32, device="cuda") for _ in douts],
         "dB": [torch.empty((n, r), dtype=f32, device="cuda") for n in douts],
         "dX": torch.empty((M, d), dtype=bf, device="cuda")}
    rope = L.make_rope_desc(p(t["pos"]), p(t["cos"]), p(t["sin"]), n_pos, hd)
    wsp = (ws.buf.data_ptr(), ws.nbytes, sh)

    def fwd(norm_done=None):
        assert L.lora_linear_rmsnorm_fwd(p(t["X"]), p(t["g"]), M, d, eps, p(Xn), p(rstd), sh) == 0
        if norm_done is not None:
            norm_done.record(stream)
        for j in range(3):
            w = (p(t[f"W{j}"]), p(t[f"A{j}"]), p(t[f"B{j}"]))
            if j < 2:
                st = L.lora_linear_fwd_rope(descs[j], rope, p(Xn), *w, p(o["Y"][j]), p(o["T"][j]), *wsp)
            else:
                st = L.lora_linear_fwd(descs[j], p(Xn), *w, None, None, None, p(o["Y"][j]), p(o["T"][j]), None, *wsp)
            assert st == 0, L.status_string(st)

    def bwd():
        # q writes the fp32 dx_n, k and v add to it (v is not rotated)
        for j in range(3):
            w = (p(t[f"W{j}"]), p(t[f"A{j}"]), p(t[f"B{j}"]))
            st = L.lora_linear_bwd_rope(descs[j], rope if j < 2 else None, p(t[f"dY{j}"]), p(Xn), *w, p(o["T"][j]),
                                        p(o["dXn"]), 1 if j else 0, p(o["dA"][j]), p(o["dB"][j]), *wsp)
            assert st == 0, L.status_string(st)
        assert L.lora_linear_rmsnorm_bwd(p(t["X"]), p(t["g"]), p(rstd), p(o["dXn"]), M, d, p(o["dX"]), sh) == 0

    if args.calls > 0:
        for _ in range(args.calls):
            fwd()
            if not args.fwd_only:
                bwd()
        torch.cuda.synchronize()
        print("ok", flush=True)
        return
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize()
    launches0 = L.lora_linear_launch_count()
    L.lora_linear_timing_enable(1)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        fwd(norm_done=ev[i][1])
        ev[i][2].record(stream)
        bwd()
        ev[i][3].record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    launches = L.lora_linear_launch_count() - launches0
    _, gemm_fwd_ms, gemm_fwd_n, gemm_bwd_ms, gemm_bwd_n = L.lora_linear_timing_read()
    L.lora_linear_timing_enable(0)
    tot_ms = max_over_ranks(sum(e[0].elapsed_time(e[3]) for e in ev), dist, "cuda")
    norm_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    F = cfg_step_flops(cfg, M)
    value = job_throughput(F, args.steps, world, tot_ms) / 1e12

    # e2e: every step copies its inputs from pinned host memory and its results
    # (Y_q, Y_k, Y_v, dX, dA_j, dB_j) back, serialised with the compute
    out_host = {k: torch.empty_like(v, device="cpu").pin_memory()
                for k, v in [(f"Y{j}", o["Y"][j]) for j in range(3)] + [(f"dA{j}", o["dA"][j]) for j in range(3)]
                + [(f"dB{j}", o["dB"][j]) for j in range(3)] + [("dX", o["dX"])]}
    dev_out = {**{f"Y{j}": o["Y"][j] for j in range(3)}, **{f"dA{j}": o["dA"][j] for j in range(3)},
               **{f"dB{j}": o["dB"][j] for j in range(3)}, "dX": o["dX"]}
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(v.numel() * v.element_size() for v in out_host.values())
    ee0, ee1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ee0.record(stream)
    for _ in range(args.e2e_steps):
        for k, v in host.items():
            t[k].copy_(v, non_blocking=True)
        fwd()
        bwd()
        for k, v in dev_out.items():
            out_host[k].copy_(v, non_blocking=True)
    ee1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(ee0.elapsed_time(ee1), dist, "cuda")
    e2e = job_throughput(F, args.e2e_steps, world, e2e_ms) / 1e12

    peaks = read_peaks()
    f_fwd = sum(2.0 * M * d * n + 2.0 * M * r * n for n in douts)     # the three forward GEMMs per step
    f_bwd = sum(2.0 * M * d * n + 2.0 * M * r * d for n in douts)     # the three dX GEMMs per step
    ach_f = f_fwd * args.steps / (gemm_fwd_ms * 1e-3) / 1e12 if gemm_fwd_n else None
    ach_b = f_bwd * args.steps / (gemm_bwd_ms * 1e-3) / 1e12 if gemm_bwd_n else None
    pk = peaks["bf16_tflops"]
    norm_bytes = 2.0 * M * d * 2 + 4.0 * M + 2.0 * d                # read X, write x_n, rstd, g
    norm_gbs = norm_bytes / (norm_ms * 1e-3) / 1e9
    roof = {"kernel": "lora_mma_kernel (forward GEMMs of q, k, v; q and k with the rotary epilogue)",
            "bound": "tensor", "achieved": round(ach_f, 2) if ach_f else None, "peak": pk, "unit": "TFLOP/s",
            "frac": round(ach_f / pk, 4) if ach_f else None,
            "peak_kind": f"bf16 burst, {peaks['source']} (sustained {peaks['bf16_tflops_sustained']})",
            "flop_per_step": f_fwd, "launches_per_step": 3, "traffic": None,
            "backward_gemms": {"achieved": round(ach_b, 2) if ach_b else None,
                               "frac": round(ach_b / pk, 4) if ach_b else None, "flop_per_step": f_bwd},
            "rmsnorm_fwd": {"bound": "hbm", "achieved": round(norm_gbs, 1), "peak": peaks["hbm_gbs"],
                            "unit": "GB/s", "frac": round(norm_gbs / peaks["hbm_gbs"], 4),
                            "bytes_per_launch": norm_bytes, "ms_per_launch": round(norm_ms, 5)},
            "step_frac": round(value / world / pk, 4)}
    line = {"metric": METRIC_QKV, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(tot_ms / args.steps, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.config, "M": M, "d_in": d, "d_out_q": douts[0], "d_out_kv": douts[1],
                       "r": r, "alpha": cfg["alpha"], "head_dim": hd, "seq_len": n_pos, "eps": eps,
                       "parallelism": f"replicas x{world}", "l2": "flushed before each timed step (512 MiB write)"},
            "roofline": roof, "gpu_launches": int(launches),
            "e2e": {"value": round(e2e, 2), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h), "copies": "serialised with the compute"},
            "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="q_proj", choices=sorted(seeded_inputs.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--shape", default=None,
                    help="M,d_in,d_out,r,act: this shape instead of --config (profiling, with --calls)")
    ap.add_argument("--calls", type=int, default=0,
                    help="run this many untimed forward(+backward) calls, print nothing else, exit (for profilers)")
    ap.add_argument("--fwd-only", action="store_true", help="with --calls: forward calls only")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    cfg = dict(seeded_inputs.CONFIGS[args.config])
    if args.shape:
        f = args.shape.split(",")
        cfg = dict(M=int(f[0]), d_in=int(f[1]), d_out=int(f[2]), r=int(f[3]), alpha=16.0, act=f[4])
        args.config = "shape " + args.shape

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, cfg, world, rank)
        return

    import torch
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    import lora_linear_fine_b200 as L

    if is_qkv(cfg):
        run_qkv(args, cfg, L, world, rank, local, dist)
        return
    M, d_in, d_out, r, act = cfg["M"], cfg["d_in"], cfg["d_out"], cfg["r"], cfg["act"]
    s = cfg["alpha"] / r if r else 0.0
    inp = seeded_inputs.make_inputs(M, d_in, d_out, r, act, seed=rank)
    w4 = cfg.get("weight") == "w4"
    if w4:   # the 4-bit base weight replaces W (forward-only few-token workload)
        inp.pop("W")
        Wq, Ws = seeded_inputs.draw_w4("W", d_out, d_in, rank)
    host = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).pin_memory() for k, v in inp.items()}
    t = {k: v.to("cuda", non_blocking=True) for k, v in host.items()}
    if w4:
        t["Wq"] = torch.from_numpy(Wq).cuda()
        t["Ws"] = torch.from_numpy(Ws.view(np.int16)).view(torch.bfloat16).cuda()
        # the frozen weight's codes in the few-token kernel's tiled layout (a load-time step)
        t["Wt"] = torch.empty(L.lora_linear_w4_tiled_bytes(d_out, d_in), dtype=torch.uint8, device="cuda")
        assert L.lora_linear_w4_tile(t["Wq"].data_ptr(), d_out, d_in, t["Wt"].data_ptr(),
                                     torch.cuda.current_stream().cuda_stream) == 0
    p_drop = cfg.get("dropout")
    if p_drop is not None:   # dropout on the adapter input: one mask per projection, an input like X
        for name in ("mask", "mask_up") if act == "swiglu" else ("mask",):
            host[name] = torch.from_numpy(seeded_inputs.draw_mask(name, M, d_in, p_drop, rank)).pin_memory()
            t[name] = host[name].to("cuda", non_blocking=True)
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    desc = L.make_desc(M, d_in, d_out, r, s, act)
    np_ = 2 if act == "swiglu" else 1
    if w4:
        ws = L.Workspace(L.lora_linear_workspace_size_w4(desc, 0))
    elif p_drop is not None:
        ws = L.Workspace(L.lora_linear_workspace_size_dropout(desc, 1))
    else:
        ws = L.Workspace(max(L.lora_linear_workspace_size(desc, 0), L.lora_linear_workspace_size(desc, 1)))
    Y = torch.empty((M, d_out), dtype=torch.bfloat16, device="cuda")
    T = torch.empty((np_, M, r), dtype=torch.float32, device="cuda")
    Z = torch.empty((np_, M, d_out), dtype=torch.float32, device="cuda") if act != "identity" else None
    dX = torch.empty((M, d_in), dtype=torch.bfloat16, device="cuda")
    dA = torch.empty((np_, r, d_in), dtype=torch.float32, device="cuda")
    dB = torch.empty((np_, d_out, r), dtype=torch.float32, device="cuda")
    p = lambda x: None if x is None else x.data_ptr()  # noqa: E731

    def fwd():
        if w4 and M <= 64:
            st = L.lora_linear_fwd_w4_tiled(desc, p(t["X"]), p(t["Wt"]), p(t["Ws"]), p(t["A"]), p(t["B"]), p(Y),
                                            p(T), p(Z), ws.buf.data_ptr(), ws.nbytes, sh)
        elif w4:
            st = L.lora_linear_fwd_w4(desc, p(t["X"]), p(t["Wq"]), p(t["Ws"]), p(t["A"]), p(t["B"]), None, None,
                                      None, None, p(Y), p(T), p(Z), ws.buf.data_ptr(), ws.nbytes, sh)
        elif p_drop is not None:
            st = L.lora_linear_fwd_dropout(desc, p(t["X"]), p(t["W"]), p(t["A"]), p(t["B"]), p(t.get("W_up")),
                                           p(t.get("A_up")), p(t.get("B_up")), p(t["mask"]), p(t.get("mask_up")),
                                           p_drop, p(Y), p(T), p(Z), ws.buf.data_ptr(), ws.nbytes, sh)
        else:
            st = L.lora_linear_fwd(desc, p(t["X"]), p(t["W"]), p(t["A"]), p(t["B"]), p(t.get("W_up")),
                                   p(t.get("A_up")), p(t.get("B_up")), p(Y), p(T), p(Z), ws.buf.data_ptr(),
                                   ws.nbytes, sh)
        assert st == 0, L.status_string(st)

    def bwd():
        if p_drop is not None:
            st = L.lora_linear_bwd_dropout(desc, p(t["dY"]), p(t["X"]), p(t["W"]), p(t["A"]), p(t["B"]),
                                           p(t.get("W_up")), p(t.get("A_up")), p(t.get("B_up")), p(t["mask"]),
                                           p(t.get("mask_up")), p_drop, p(T), p(Z), p(dX), p(dA[0]), p(dB[0]),
                                           p(dA[1]) if np_ == 2 else None, p(dB[1]) if np_ == 2 else None,
                                           ws.buf.data_ptr(), ws.nbytes, sh)
            assert st == 0, L.status_string(st)
            return
        st = L.lora_linear_bwd(desc, p(t["dY"]), p(t["X"]), p(t["W"]), p(t["A"]), p(t["B"]), p(t.get("W_up")),
                               p(t.get("A_up")), p(t.get("B_up")), p(T), p(Z), p(dX), p(dA[0]), p(dB[0]),
                               p(dA[1]) if np_ == 2 else None, p(dB[1]) if np_ == 2 else None,
                               ws.buf.data_ptr(), ws.nbytes, sh)
        assert st == 0, L.status_string(st)

    if args.calls > 0:
        for _ in range(args.calls):
            fwd()
            if not args.fwd_only:
                bwd()
        torch.cuda.synchronize()
        print("ok", flush=True)
        return
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    if args.config.startswith("small_m"):
        run_small_m(args, cfg, fwd, flush, stream, L, world, rank, dist)
        return
    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize()

    launches0 = L.lora_linear_launch_count()
    L.lora_linear_timing_enable(1)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        e0, e1, e2 = ev[i]
        e0.record(stream)
        fwd()
        e1.record(stream)
        bwd()
        e2.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    launches = L.lora_linear_launch_count() - launches0
    _, gemm_fwd_ms, gemm_fwd_n, gemm_bwd_ms, gemm_bwd_n = L.lora_linear_timing_read()
    L.lora_linear_timing_enable(0)
    step_ms = [a.elapsed_time(c) for a, _, c in ev]
    fwd_ms = [a.elapsed_time(b) for a, b, _ in ev]
    tot_ms = sum(step_ms)
    tot_ms = max_over_ranks(tot_ms, dist, "cuda")
    F = step_flops(M, d_in, d_out, r, act)
    value = job_throughput(F, args.steps, world, tot_ms) / 1e12

    # e2e: the same step through the C ABI from pinned HOST buffers, copies
    # included: every step copies its inputs host -> device and its results
    # device -> host.  Two buffer sets and one copy stream per direction let
    # step i+1's input copy and step i-1's result copy run while step i
    # computes (PCIe is full duplex), as a training loop feeding the layer
    # would arrange them.
    bufs = [dict(t=t, Y=Y, dX=dX, dA=dA, dB=dB),
            dict(t={k: torch.empty_like(v) for k, v in t.items()}, Y=torch.empty_like(Y),
                 dX=torch.empty_like(dX), dA=torch.empty_like(dA), dB=torch.empty_like(dB))]
    for k in bufs[1]["t"]:
        if k not in host:                 # inputs that are not copied per step (none in the bf16 path)
            bufs[1]["t"][k].copy_(t[k])
    out_host = [{k: torch.empty_like(bufs[0][k], device="cpu").pin_memory() for k in ("Y", "dX", "dA", "dB")}
                for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(v.numel() * v.element_size() for v in out_host[0].values())
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    ee0, ee1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ee0.record(stream)
    s_in.wait_event(ee0)
    s_out.wait_event(ee0)
    for i in range(args.e2e_steps):
        b = i % 2
        cur = bufs[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[b])        # step i-2 no longer reads these inputs
            for k, v in host.items():
                cur["t"][k].copy_(v, non_blocking=True)
            in_ready[b].record(s_in)
        stream.wait_event(in_ready[b])
        if i >= 2:
            stream.wait_event(out_done[b])           # step i-2's results are on the host
        t, Y, dX, dA, dB = cur["t"], cur["Y"], cur["dX"], cur["dA"], cur["dB"]
        fwd()
        bwd()
        comp_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            for k in ("Y", "dX", "dA", "dB"):
                out_host[b][k].copy_(cur[k], non_blocking=True)
            out_done[b].record(s_out)
    for b in range(min(2, args.e2e_steps)):
        stream.wait_event(out_done[b])
    ee1.record(stream)
    torch.cuda.synchronize()
    t, Y, dX, dA, dB = bufs[0]["t"], bufs[0]["Y"], bufs[0]["dX"], bufs[0]["dA"], bufs[0]["dB"]
    e2e_ms = ee0.elapsed_time(ee1)
    e2e_ms = max_over_ranks(e2e_ms, dist, "cuda")
    e2e = job_throughput(F, args.e2e_steps, world, e2e_ms) / 1e12

    peaks = read_peaks()
    # Dominant kernels: the forward and backward GEMMs (lora_mma_kernel), each
    # timed by the library's event pair around its launch on this stream.
    np_ = 2 if act == "swiglu" else 1
    f_fwd = np_ * (2.0 * M * d_in * d_out + 2.0 * M * r * d_out)       # X W^T + (sT) B^T
    f_bwd = np_ * (2.0 * M * d_in * d_out + 2.0 * M * r * d_in)        # dZ W + (sU) A
    ach_f = f_fwd / (gemm_fwd_ms / max(gemm_fwd_n, 1) * 1e-3) / 1e12 if gemm_fwd_n else None
    ach_b = f_bwd / (gemm_bwd_ms / max(gemm_bwd_n, 1) * 1e-3) / 1e12 if gemm_bwd_n else None
    pk = peaks["bf16_tflops"]
    traffic = committed_traffic(args.config)
    roof = {"kernel": "lora_mma_kernel (forward GEMM)", "bound": "tensor",
            "achieved": round(ach_f, 2) if ach_f else None, "peak": pk, "unit": "TFLOP/s",
            "frac": round(ach_f / pk, 4) if ach_f else None,
            "peak_kind": f"bf16 burst, {peaks['source']} (sustained {peaks['bf16_tflops_sustained']})",
            "frac_of_sustained": round(ach_f / peaks["bf16_tflops_sustained"], 4) if ach_f else None,
            "flop_per_launch": f_fwd, "ms_per_launch": round(gemm_fwd_ms / max(gemm_fwd_n, 1), 5),
            "traffic": traffic,
            "backward_gemm": {"achieved": round(ach_b, 2) if ach_b else None,
                              "frac": round(ach_b / pk, 4) if ach_b else None, "flop_per_launch": f_bwd,
                              "ms_per_launch": round(gemm_bwd_ms / max(gemm_bwd_n, 1), 5)},
            "step_frac": round(value / world / pk, 4)}

    line = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(tot_ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.config, "M": M, "d_in": d_in, "d_out": d_out, "r": r,
                       "alpha": cfg["alpha"], "act": act, "parallelism": f"replicas x{world}",
                       "l2": "flushed before each timed step (512 MiB write)",
                       **({"dropout": p_drop} if p_drop is not None else {})},
            "roofline": roof, "gpu_launches": int(launches),
            "e2e": {"value": round(e2e, 2), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h)},
            "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
