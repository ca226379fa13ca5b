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
METRIC_CE = "LoRA fine-tuning output projection + cross-entropy fwd+bwd TFLOP/s & % of B200 roofline"
METRIC_SMALL_M = "LoRA-linear forward (few tokens) TFLOP/s & % of B200 HBM roofline"
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
    if cfg["act"] == "ce":       # logits + dH of the output projection fused with the loss
        return 4.0 * M * cfg["d_in"] * cfg["d_out"]
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


def oracle_sample_run(cfg, rows, inp_f64, fwd_only=False):
    """Seconds the oracle takes for one sample of `rows` tokens of the
    workload: the plain C fp64 oracle for the layer, the numpy block oracle
    (norm, three projections, rotation) for the attention-input block."""
    g = inp_f64
    if is_qkv(cfg):
        from oracle import norm_rope_oracle
        projs = [{k: g[f"{k}{j}"] for k in ("W", "A", "B")} for j in range(3)]
        t0 = time.perf_counter()
        norm_rope_oracle.qkv_backward([g[f"dY{j}"][:rows] for j in range(3)], g["X"][:rows], g["g"],
                                      float(np.float32(cfg["eps"])), projs, cfg["alpha"] / cfg["r"],
                                      [True, True, False], g["pos"][:rows], g["cos"], g["sin"], cfg["head_dim"])
        return time.perf_counter() - t0
    if cfg["act"] == "ce":
        from oracle import linear_ce_oracle
        t0 = time.perf_counter()
        linear_ce_oracle.linear_ce_backward(g["H"][:rows], g["W"], g["labels"][:rows])
        return time.perf_counter() - t0
    from oracle import lora_oracle_c
    X = g["X"][:rows]
    s = cfg["alpha"] / cfg["r"]
    t0 = time.perf_counter()
    if fwd_only:
        lora_oracle_c.lora_forward(X, g["W"], g["A"], g["B"], s, cfg["act"], g.get("W_up"), g.get("A_up"),
                                   g.get("B_up"))
    else:
        lora_oracle_c.lora_backward(g["dY"][:rows], X, g["W"], g["A"], g["B"], s, cfg["act"], g.get("W_up"),
                                    g.get("A_up"), g.get("B_up"))
    return time.perf_counter() - t0


def oracle_cores(cfg):
    """Threads the oracle runs on: the C oracle's POSIX threads, or numpy's BLAS pool."""
    if is_qkv(cfg) or cfg["act"] == "ce":
        try:
            from threadpoolctl import threadpool_info
            n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
            return max(n) if n else os.cpu_count()
        except Exception:
            return os.cpu_count()
    from oracle import lora_oracle_c
    return lora_oracle_c.threads()


def oracle_kind(cfg):
    return ("fp64 numpy oracle (matmul through the BLAS)" if is_qkv(cfg) or cfg["act"] == "ce"
            else "plain C fp64 oracle (scalar loops, POSIX threads over output rows)")


def cpu_baseline(cfg, budget_s=12.0, max_rows=None, fwd_only=False):
    """Time the oracle on growing row samples until ~budget_s of CPU work."""
    M, d_in, d_out, r = cfg["M"], cfg["d_in"], cfg["d_out"], cfg["r"]
    rows_cap = max_rows or (4096 if is_qkv(cfg) else M)
    g = oracle_inputs(cfg, min(M, rows_cap))
    rows = 16
    spent = 0.0
    best = None
    while True:
        dt = oracle_sample_run(cfg, rows, g, fwd_only)
        spent += dt
        best = (rows, dt)
        if dt > budget_s / 3 or rows >= min(M, rows_cap) or spent > budget_s:
            break
        rows = min(rows * 4, min(M, rows_cap))
    rows, dt = best
    # repeat the chosen sample until ~budget_s / 2 of work has been timed
    times = [dt]
    while sum(times) < budget_s / 2 and len(times) < 20:
        times.append(oracle_sample_run(cfg, rows, g, fwd_only))
    dt = statistics.mean(times)
    flops = fwd_flops(rows, d_in, d_out, r, cfg["act"]) if fwd_only else cfg_step_flops(cfg, rows)
    val = flops / dt / 1e12
    what = (f"the norm, q/k/v projections ({d_in}->{'/'.join(map(str, qkv_douts(cfg)))}) and rotation"
            if is_qkv(cfg) else f"(output projection {d_in}->{d_out} + cross-entropy)" if cfg["act"] == "ce"
            else f"({d_in}->{d_out}, {cfg['act']})")
    return {"value": val, "unit": UNIT, "cores": oracle_cores(cfg), "kind": "oracle",
            "sample": f"{oracle_kind(cfg)}, {'forward' if fwd_only else 'fwd+bwd'} on the first {rows} of {M} "
                      f"tokens {what}, r={r}; mean of {len(times)} runs of {dt:.2f} s; FLOPs by the same formula"}


def oracle_inputs(cfg, M):
    """The workload's inputs for the oracle (float64; positions and tables as given)."""
    import oracle
    if cfg["act"] == "ce":
        H, W, labels = seeded_inputs.draw_ce(M, cfg["d_in"], cfg["d_out"], 0)
        return {"H": oracle.bf16_to_f64(H), "W": oracle.bf16_to_f64(W), "labels": labels}
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
    fwd_only = args.config.startswith("small_m")
    g = oracle_inputs(cfg, min(cfg["M"], 256 if cfg["act"] == "ce" else 4096))
    # rows per step: sized so the whole warm-up + timed run stays within a few minutes
    rows = 16
    cap = min(cfg["M"], 256 if cfg["act"] == "ce" else 4096)
    while rows < cap:
        dt = oracle_sample_run(cfg, rows, g, fwd_only)
        if dt * (steps + warm) > 60.0 or dt > 2.0:
            break
        rows = min(rows * 2, cap)
    for _ in range(warm):
        oracle_sample_run(cfg, rows, g, fwd_only)
    tot = 0.0
    for _ in range(steps):
        tot += oracle_sample_run(cfg, rows, g, fwd_only)
    flops = fwd_flops(rows, cfg["d_in"], cfg["d_out"], cfg["r"], cfg["act"]) if fwd_only else cfg_step_flops(cfg, rows)
    val = flops * steps / tot / 1e12
    shape = (f"norm + {cfg['d_in']}->{'/'.join(map(str, qkv_douts(cfg)))} + rotary" if is_qkv(cfg)
             else f"output projection {cfg['d_in']}->{cfg['d_out']} + cross-entropy" if cfg["act"] == "ce"
             else f"{cfg['d_in']}->{cfg['d_out']}")
    sample = (f"{oracle_kind(cfg)}, {'forward' if fwd_only else 'fwd+bwd'} on {rows} of {cfg['M']} tokens per "
              f"step ({shape}, r={cfg['r']})")
    metric = (METRIC_QKV if is_qkv(cfg) else METRIC_CE if cfg["act"] == "ce"
              else METRIC_SMALL_M if fwd_only else METRIC)
    line = {"impl": "reference", "metric": metric, "value": val, "unit": UNIT, "n_gpus": world,
            "steps": steps, "warmup": warm, "ms_per_step": tot / steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.config, "M": cfg["M"], "d_in": cfg["d_in"], "d_out": cfg["d_out"],
                       "r": cfg["r"], "alpha": cfg["alpha"], "act": cfg["act"], "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": oracle_cores(cfg), "kind": "oracle",
                             "sample": sample},
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


# ---------------------------------------------------------------------------
# one LoRA-linear workload on the device
# ---------------------------------------------------------------------------
class Layer:
    """Device inputs, outputs and workspace of one LoRA-linear workload, with
    fwd() / bwd() closures that call the C ABI.  The input tensors live in
    self.t and may be re-pointed (a chained MLP feeds one layer's output to the
    next)."""

    def __init__(self, L, cfg, seed, pin_host=False):
        import torch
        self.L, self.cfg = L, cfg
        M, d_in, d_out, r, act = cfg["M"], cfg["d_in"], cfg["d_out"], cfg["r"], cfg["act"]
        self.M, self.d_in, self.d_out, self.r, self.act = M, d_in, d_out, r, act
        self.s = cfg["alpha"] / r if r else 0.0
        inp = seeded_inputs.make_inputs(M, d_in, d_out, r, act, seed=seed)
        self.w4 = cfg.get("weight") == "w4"
        if self.w4:   # the 4-bit base weight replaces W (forward-only few-token workload)
            inp.pop("W")
            Wq, Ws = seeded_inputs.draw_w4("W", d_out, d_in, seed)
        host = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16) for k, v in inp.items()}
        self.p_drop = cfg.get("dropout")
        if self.p_drop is not None:   # dropout on the adapter input: one mask per projection, an input like X
            for name in ("mask", "mask_up") if act == "swiglu" else ("mask",):
                host[name] = torch.from_numpy(seeded_inputs.draw_mask(name, M, d_in, self.p_drop, seed))
        if pin_host:
            host = {k: v.pin_memory() for k, v in host.items()}
        self.host = host
        self.t = {k: v.to("cuda", non_blocking=True) for k, v in host.items()}
        self.stream = torch.cuda.current_stream()
        self.sh = self.stream.cuda_stream
        if self.w4:
            self.t["Wq"] = torch.from_numpy(Wq).cuda()
            self.t["Ws"] = torch.from_numpy(Ws.view(np.int16)).view(torch.bfloat16).cuda()
            # the frozen weight's codes in the few-token kernel's tiled layout (a load-time step)
            self.t["Wt"] = torch.empty(L.lora_linear_w4_tiled_bytes(d_out, d_in), dtype=torch.uint8, device="cuda")
            assert L.lora_linear_w4_tile(self.t["Wq"].data_ptr(), d_out, d_in, self.t["Wt"].data_ptr(), self.sh) == 0
        self.desc = L.make_desc(M, d_in, d_out, r, self.s, act)
        self.np = 2 if act == "swiglu" else 1
        if self.w4:
            nb = L.lora_linear_workspace_size_w4(self.desc, 0)
        elif self.p_drop is not None:
            nb = L.lora_linear_workspace_size_dropout(self.desc, 1)
        else:
            nb = max(L.lora_linear_workspace_size(self.desc, 0), L.lora_linear_workspace_size(self.desc, 1))
        self.ws = L.Workspace(nb)
        bf, f32 = torch.bfloat16, torch.float32
        self.Y = torch.empty((M, d_out), dtype=bf, device="cuda")
        self.T = torch.empty((self.np, M, r), dtype=f32, device="cuda")
        self.Z = torch.empty((self.np, M, d_out), dtype=f32, device="cuda") if act != "identity" else None
        self.dX = torch.empty((M, d_in), dtype=bf, device="cuda")
        self.dA = torch.empty((self.np, r, d_in), dtype=f32, device="cuda")
        self.dB = torch.empty((self.np, d_out, r), dtype=f32, device="cuda")

    @staticmethod
    def p(x):
        return None if x is None else x.data_ptr()

    def fwd(self):
        L, t, p, sh = self.L, self.t, self.p, self.sh
        ws = (self.ws.buf.data_ptr(), self.ws.nbytes, sh)
        if self.w4 and self.M <= 64:
            st = L.lora_linear_fwd_w4_tiled(self.desc, p(t["X"]), p(t["Wt"]), p(t["Ws"]), p(t["A"]), p(t["B"]),
                                            p(self.Y), p(self.T), p(self.Z), *ws)
        elif self.w4:
            st = L.lora_linear_fwd_w4(self.desc, p(t["X"]), p(t["Wq"]), p(t["Ws"]), p(t["A"]), p(t["B"]), None,
                                      None, None, None, p(self.Y), p(self.T), p(self.Z), *ws)
        elif self.p_drop is not None:
            st = L.lora_linear_fwd_dropout(self.desc, p(t["X"]), p(t["W"]), p(t["A"]), p(t["B"]), p(t.get("W_up")),
                                           p(t.get("A_up")), p(t.get("B_up")), p(t["mask"]), p(t.get("mask_up")),
                                           self.p_drop, p(self.Y), p(self.T), p(self.Z), *ws)
        else:
            st = L.lora_linear_fwd(self.desc, p(t["X"]), p(t["W"]), p(t["A"]), p(t["B"]), p(t.get("W_up")),
                                   p(t.get("A_up")), p(t.get("B_up")), p(self.Y), p(self.T), p(self.Z), *ws)
        assert st == 0, L.status_string(st)

    def bwd(self):
        L, t, p, sh = self.L, self.t, self.p, self.sh
        ws = (self.ws.buf.data_ptr(), self.ws.nbytes, sh)
        two = self.np == 2
        grads = (p(self.dX), p(self.dA[0]), p(self.dB[0]), p(self.dA[1]) if two else None,
                 p(self.dB[1]) if two else None)
        if self.p_drop is not None:
            st = L.lora_linear_bwd_dropout(self.desc, p(t["dY"]), p(t["X"]), p(t["W"]), p(t["A"]), p(t["B"]),
                                           p(t.get("W_up")), p(t.get("A_up")), p(t.get("B_up")), p(t["mask"]),
                                           p(t.get("mask_up")), self.p_drop, p(self.T), p(self.Z), *grads, *ws)
        else:
            st = L.lora_linear_bwd(self.desc, p(t["dY"]), p(t["X"]), p(t["W"]), p(t["A"]), p(t["B"]),
                                   p(t.get("W_up")), p(t.get("A_up")), p(t.get("B_up")), p(self.T), p(self.Z),
                                   *grads, *ws)
        assert st == 0, L.status_string(st)

    # algorithmic work
    def step_flops(self):
        return step_flops(self.M, self.d_in, self.d_out, self.r, self.act)

    def fwd_gemm_flops(self):    # X W^T + (sT) B^T, per projection
        return self.np * (2.0 * self.M * self.d_in * self.d_out + 2.0 * self.M * self.r * self.d_out)

    def t_in_gemm(self):
        """Whether the library accumulates T = X A^T inside the forward GEMM
        (then that launch also does T's 2 M d_in r FLOPs): one identity
        projection with 0 < r <= 64, no dropout, more than 64 tokens, and
        either one GEMM tile per CTA pair or at most one 256-row block per
        pair (the library's own test, with its switches)."""
        if os.environ.get("LORA_LINEAR_FUSED_T", "1")[:1] == "0":
            return False
        if not (0 < self.r <= 64) or self.np != 1 or self.act != "identity" or self.p_drop is not None:
            return False
        if self.M <= 64:
            return False
        import torch
        sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
        pair = self.M > 128
        units = sms // 2 if pair else sms
        m_tiles = -(-self.M // (256 if pair else 128))
        if m_tiles * -(-self.d_out // 256) <= units:
            return True
        return m_tiles <= units and os.environ.get("LORA_LINEAR_SHARED_T", "1")[:1] != "0"

    def fwd_launch_flops(self):  # the forward GEMM launch's work: + T when it is accumulated there
        return self.fwd_gemm_flops() + (2.0 * self.M * self.d_in * self.r if self.t_in_gemm() else 0.0)

    def dx_gemm_flops(self):     # dZ W + (sU) A, per projection
        return self.np * (2.0 * self.M * self.d_in * self.d_out + 2.0 * self.M * self.r * self.d_in)

    def fwd_bytes(self):
        """Algorithmic bytes of the forward: X, W (bf16, or 4-bit codes + scales), A, B
        read once, Y written once, T (fp32) written once."""
        d_in, d_out, M, r = self.d_in, self.d_out, self.M, self.r
        w = (d_out * d_in / 2.0 + 2.0 * d_out * (d_in // 64)) if self.w4 else 2.0 * d_out * d_in
        return self.np * (w + 2.0 * (r * d_in + d_out * r)) + 2.0 * (M * d_in + M * d_out) + 4.0 * self.np * M * r


def time_steps(L, step, steps, warmup, flush, stream, local, dist=None, sample_clocks=True):
    """Warm up, then time `steps` calls of step() with CUDA events on `stream`,
    the L2 flushed (a 512 MiB write) before each, outside the events; the
    library's own event pairs time its GEMM launches.  Returns per-step
    milliseconds, the GEMM times, the launch count and the clock record."""
    import torch
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    launches0 = L.lora_linear_launch_count()
    L.lora_linear_timing_enable(1)
    L.lora_linear_timing_read()              # start from zero
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    clocks = ClockSampler(local) if sample_clocks else None
    if clocks:
        clocks.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    launches = L.lora_linear_launch_count() - launches0
    _, gf_ms, gf_n, gb_ms, gb_n = L.lora_linear_timing_read()
    L.lora_linear_timing_enable(0)
    return {"ms": [a.elapsed_time(b) for a, b in ev], "gemm_fwd_ms": gf_ms, "gemm_fwd_n": gf_n,
            "gemm_bwd_ms": gb_ms, "gemm_bwd_n": gb_n, "launches": int(launches), "clocks": clk}


def gemm_record(flop_per_step, ms_total, n_launch, launches_per_step, peak):
    """Achieved TFLOP/s of the GEMM launches of one direction: their FLOPs over
    their summed CUDA-event durations (the library times at most 1024 launches
    per direction between reads, a whole number of steps)."""
    if not n_launch:
        return None
    steps_timed = n_launch / launches_per_step
    ach = flop_per_step * steps_timed / (ms_total * 1e-3) / 1e12
    return {"achieved": round(ach, 2), "frac": round(ach / peak, 4), "flop_per_step": flop_per_step,
            "launches_per_step": launches_per_step, "ms_per_launch": round(ms_total / n_launch, 5)}


def steps_for(seconds, ms_guess, lo=10, hi=1000):
    return int(max(lo, min(hi, seconds * 1e3 / max(ms_guess, 1e-3))))


def measure_layer_workload(L, name, local, flush, seconds=0.5, peaks=None):
    """A fwd+bwd workload timed on its own (the `workloads` entries)."""
    import torch
    cfg = dict(seeded_inputs.CONFIGS[name])
    lay = Layer(L, cfg, seed=0)

    def step():
        lay.fwd()
        lay.bwd()
    probe = time_steps(L, step, 3, 3, flush, lay.stream, local, sample_clocks=False)
    steps = steps_for(seconds, statistics.median(probe["ms"]))
    r = time_steps(L, step, steps, 2, flush, lay.stream, local)
    ms = statistics.median(r["ms"])
    pk = peaks["bf16_tflops"]
    F = lay.step_flops()
    tf = F / (ms * 1e-3) / 1e12
    out = {"M": cfg["M"], "d_in": cfg["d_in"], "d_out": cfg["d_out"], "r": cfg["r"], "act": cfg["act"],
           "steps": steps, "ms_per_step": round(ms, 5), "timing": "median of per-step CUDA events, L2 flushed",
           "value": round(tf, 2), "unit": UNIT,
           "roofline": {"bound": "tensor", "peak": pk, "unit": "TFLOP/s", "frac": round(tf / pk, 4),
                        "flop_per_step": F},
           "forward_gemm": gemm_record(lay.fwd_launch_flops(), r["gemm_fwd_ms"], r["gemm_fwd_n"], 1, pk),
           "dx_gemm": gemm_record(lay.dx_gemm_flops(), r["gemm_bwd_ms"], r["gemm_bwd_n"], 1, pk),
           "gpu_launches_per_step": r["launches"] // steps, "clocks": r["clocks"]}
    if name == "tiny":
        out["roofline"]["bound"] = "latency (parity workload: 1.8e7 FLOP per step)"
    del lay
    torch.cuda.empty_cache()
    return out


def measure_mlp(L, local, flush, seconds=0.5, peaks=None):
    """The Llama-3-8B MLP with LoRA r = 64 on gate, up and down, chained: the
    gate/up layer (SwiGLU in its epilogue) feeds H to the down projection; the
    down projection's input gradient is the gate/up layer's dY."""
    import torch
    gu = Layer(L, dict(seeded_inputs.CONFIGS["mlp_gate_up"]), seed=0)
    dn = Layer(L, dict(seeded_inputs.CONFIGS["mlp_down"]), seed=1)
    dn.t["X"] = gu.Y
    gu.t["dY"] = dn.dX

    def step():
        gu.fwd()
        dn.fwd()
        dn.bwd()
        gu.bwd()
    probe = time_steps(L, step, 2, 2, flush, gu.stream, local, sample_clocks=False)
    steps = steps_for(seconds, statistics.median(probe["ms"]), lo=10)
    r = time_steps(L, step, steps, 2, flush, gu.stream, local)
    ms = statistics.median(r["ms"])
    pk = peaks["bf16_tflops"]
    F = gu.step_flops() + dn.step_flops()
    tf = F / (ms * 1e-3) / 1e12
    out = {"M": gu.M, "d_model": gu.d_in, "d_ff": gu.d_out, "r": gu.r, "act": "swiglu (gate, up) -> down",
           "steps": steps, "ms_per_step": round(ms, 5), "timing": "median of per-step CUDA events, L2 flushed",
           "value": round(tf, 2), "unit": UNIT,
           "roofline": {"bound": "tensor", "peak": pk, "unit": "TFLOP/s", "frac": round(tf / pk, 4),
                        "flop_per_step": F},
           "forward_gemms": gemm_record(gu.fwd_launch_flops() + dn.fwd_launch_flops(), r["gemm_fwd_ms"],
                                        r["gemm_fwd_n"], 2, pk),
           "dx_gemms": gemm_record(gu.dx_gemm_flops() + dn.dx_gemm_flops(), r["gemm_bwd_ms"], r["gemm_bwd_n"],
                                   2, pk),
           "gpu_launches_per_step": r["launches"] // steps, "clocks": r["clocks"]}
    del gu, dn
    torch.cuda.empty_cache()
    return out


class CeWorkload:
    """The output projection fused with the cross-entropy loss: H [M x d],
    W [V x d] (bf16), int32 labels; one step = lora_linear_ce_fwd_bwd (loss,
    lse and dH in one call, the loss being the step's final scalar with
    upstream factor 1)."""

    def __init__(self, L, cfg, seed, pin_host=False):
        import torch
        self.L = L
        self.M, self.d, self.V = cfg["M"], cfg["d_in"], cfg["d_out"]
        H, W, labels = seeded_inputs.draw_ce(self.M, self.d, self.V, seed)
        host = {"H": torch.from_numpy(H.view(np.int16)).view(torch.bfloat16),
                "W": torch.from_numpy(W.view(np.int16)).view(torch.bfloat16),
                "labels": torch.from_numpy(labels)}
        if pin_host:
            host = {k: v.pin_memory() for k, v in host.items()}
        self.host = host
        self.t = {k: v.to("cuda", non_blocking=True) for k, v in host.items()}
        self.stream = torch.cuda.current_stream()
        self.sh = self.stream.cuda_stream
        self.desc = L.make_ce_desc(self.M, self.d, self.V)
        self.ws = L.Workspace(L.lora_linear_ce_workspace_size(self.desc, 2))
        self.loss = torch.empty((), dtype=torch.float32, device="cuda")
        self.lse = torch.empty(self.M, dtype=torch.float32, device="cuda")
        self.dloss = torch.ones((), dtype=torch.float32, device="cuda")
        self.dH = torch.empty((self.M, self.d), dtype=torch.bfloat16, device="cuda")

    def step(self):
        t = self.t
        st = self.L.lora_linear_ce_fwd_bwd(self.desc, t["H"].data_ptr(), t["W"].data_ptr(), t["labels"].data_ptr(),
                                           self.dloss.data_ptr(), self.loss.data_ptr(), self.lse.data_ptr(),
                                           self.dH.data_ptr(), self.ws.buf.data_ptr(), self.ws.nbytes, self.sh)
        assert st == 0, self.L.status_string(st)

    def logit_flops(self):      # H W^T, once per step (the chunk's logits are kept, not recomputed)
        return 2.0 * self.M * self.V * self.d

    def step_flops(self):       # the quantity: logits + dH = dz W, each executed once
        return 4.0 * self.M * self.V * self.d


def measure_ce(L, cfg, local, flush, steps=None, warmup=3, peaks=None, dist=None, ce=None):
    """Time the fused output projection + cross-entropy, forward + backward."""
    ce = ce or CeWorkload(L, cfg, seed=0)
    step = ce.step
    if steps is None:
        probe = time_steps(L, step, 2, 2, flush, ce.stream, local, sample_clocks=False)
        steps = steps_for(1.0, statistics.median(probe["ms"]), lo=5, hi=200)
    r = time_steps(L, step, steps, warmup, flush, ce.stream, local, dist)
    ms = statistics.median(r["ms"])
    pk = peaks["bf16_tflops"]
    F = ce.step_flops()
    tf = F / (ms * 1e-3) / 1e12
    # the logits GEMM (timing direction 0), the dH GEMM (direction 1)
    logits = gemm_record(ce.logit_flops(), r["gemm_fwd_ms"], r["gemm_fwd_n"], 1, pk)
    dh = gemm_record(ce.logit_flops(), r["gemm_bwd_ms"], r["gemm_bwd_n"], 1, pk)
    out = {"M": ce.M, "d": ce.d, "V": ce.V, "steps": steps, "ms_per_step": round(ms, 5),
           "timing": "median of per-step CUDA events, L2 flushed",
           "value": round(tf, 2), "unit": UNIT,
           "roofline": {"bound": "tensor", "peak": pk, "unit": "TFLOP/s", "frac": round(tf / pk, 4),
                        "flop_per_step": F, "flop_executed_per_step": F},
           "logit_gemms": logits, "dh_gemm": dh,
           "gpu_launches_per_step": r["launches"] // steps, "clocks": r["clocks"]}
    return out, ce, r


def small_m_roofline(lay, ms, peaks):
    """max(FLOPs / tensor peak, bytes / HBM bandwidth) against the measured time."""
    F = lay.fwd_gemm_flops() + (2.0 * lay.M * lay.d_in * lay.r)
    byts = lay.fwd_bytes()
    t_tensor = F / (peaks["bf16_tflops"] * 1e12)
    t_hbm = byts / (peaks["hbm_gbs"] * 1e9)
    bound = "hbm" if t_hbm >= t_tensor else "tensor"
    gbs = byts / (ms * 1e-3) / 1e9
    tf = F / (ms * 1e-3) / 1e12
    if bound == "hbm":
        return {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(gbs / peaks["hbm_gbs"], 4), "bytes_per_launch": byts, "flop_per_launch": F,
                "tflops": round(tf, 3)}
    return {"bound": "tensor", "achieved": round(tf, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(tf / peaks["bf16_tflops"], 4), "bytes_per_launch": byts, "flop_per_launch": F,
            "hbm_gbs": round(gbs, 1), "roofline_us": round(max(t_tensor, t_hbm) * 1e6, 2)}


def small_m_kernel_name(lay, launches_per_forward):
    """The kernel(s) one forward of a few-token workload runs: the cluster
    split-K kernel up to 64 tokens; above, one GEMM launch when T is
    accumulated inside it (one tile per CTA pair), else the T pass first."""
    if lay.M <= 64:
        return "small_m_kernel"
    if launches_per_forward == 1:
        return "lora_mma_kernel (forward GEMM, T accumulated in the GEMM)"
    return "rank_gemm_kernel (T) + lora_mma_kernel (forward GEMM)"


def small_m_back_to_back(L, lay, peaks, copies=None, reps=20):
    """Few-token forwards launched back to back over distinct copies of W (as
    the layers of one decode step), no flush between them: each launch streams
    its W from HBM (the copies together exceed twice the L2), and programmatic
    dependent launch lets a launch start while its predecessor drains.  One
    event pair around each chain of launches; returns the median per launch."""
    import torch
    if lay.w4 or "W" not in lay.t:
        return None
    wb = lay.t["W"].numel() * 2
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    n = copies or max(4, int(2 * l2 // wb) + 2)
    Ws = [lay.t["W"].clone() for _ in range(n)]
    orig = lay.t["W"]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ts = []
    launches0 = L.lora_linear_launch_count()
    for rep in range(reps + 2):
        e0.record(lay.stream)
        for w in Ws:
            lay.t["W"] = w
            lay.fwd()
        e1.record(lay.stream)
        torch.cuda.synchronize()
        if rep >= 2:
            ts.append(e0.elapsed_time(e1) / n)
    lay.t["W"] = orig
    launches = (L.lora_linear_launch_count() - launches0) // ((reps + 2) * n)
    ms = statistics.median(ts)
    roof = small_m_roofline(lay, ms, peaks)
    del Ws
    return {"ms_per_launch": round(ms, 5), "weight_copies": n, "chains": reps, "roofline": roof,
            "launches_per_forward": launches,
            "timing": "median over chains of (event pair around n back-to-back launches) / n"}


def measure_small_m(L, name, local, flush, seconds=0.3, peaks=None, lay=None):
    """A forward-only few-token workload: W read once (HBM roofline), or, for
    the ragged M = 1000 run, the larger of the tensor and HBM times."""
    import torch
    cfg = dict(seeded_inputs.CONFIGS[name])
    lay = lay or Layer(L, cfg, seed=0)
    probe = time_steps(L, lay.fwd, 5, 3, flush, lay.stream, local, sample_clocks=False)
    steps = steps_for(seconds, statistics.median(probe["ms"]) + 0.1, lo=50)
    r = time_steps(L, lay.fwd, steps, 3, flush, lay.stream, local)
    ms = statistics.median(r["ms"])
    roof = small_m_roofline(lay, ms, peaks)
    roof["kernel"] = small_m_kernel_name(lay, r["launches"] // steps)
    if lay.M <= 64:
        roof["traffic"] = committed_traffic(name, "small_m_traffic.json", "lora_small_m.cuh")
    F = roof["flop_per_launch"]
    out = {"M": lay.M, "d_in": lay.d_in, "d_out": lay.d_out, "r": lay.r, "act": lay.act,
           "weight": "w4g64" if lay.w4 else "bf16", "steps": steps, "ms_per_step": round(ms, 5),
           "timing": "median of per-launch CUDA events, L2 flushed before each (a single cold launch)",
           "value": round(F / (ms * 1e-3) / 1e12, 3), "unit": UNIT, "roofline": roof,
           "gpu_launches_per_step": r["launches"] // steps, "clocks": r["clocks"],
           "back_to_back": small_m_back_to_back(L, lay, peaks)}
    return out, lay, r


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
    # the three forward GEMMs per step; each also accumulates T = x_n A^T
    # (2 M d r) when r <= 64 and M <= 256 x (SMs / 2) (the library's test)
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    t_in = (0 < r <= 64 and -(-M // 256) <= sms // 2 and os.environ.get("LORA_LINEAR_FUSED_T", "1")[:1] != "0"
            and (os.environ.get("LORA_LINEAR_SHARED_T", "1")[:1] != "0"
                 or all(-(-M // 256) * -(-n // 256) <= sms // 2 for n in douts)))
    f_fwd = sum(2.0 * M * d * n + 2.0 * M * r * n + (2.0 * M * d * r if t_in else 0.0) for n in douts)
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


def layer_e2e(lay, steps, dist, fwd_only=False):
    """The same step through the C ABI from pinned HOST buffers, copies
    included: every step copies its inputs host -> device and its results
    device -> host.  Two buffer sets and one copy stream per direction let step
    i+1's input copy and step i-1's result copy run while step i computes (PCIe
    is full duplex), as a training loop feeding the layer would arrange them.
    Returns (milliseconds for `steps` steps, h2d bytes, d2h bytes per step)."""
    import copy
    import torch
    stream = lay.stream
    outs = ("Y",) if fwd_only else ("Y", "dX", "dA", "dB")
    host = {k: v if v.is_pinned() else v.pin_memory() for k, v in lay.host.items()
            if not (fwd_only and k == "dY")}
    second = copy.copy(lay)
    second.t = dict(lay.t)
    for k in host:
        second.t[k] = torch.empty_like(lay.t[k])
    for k in ("Y", "T", "Z", "dX", "dA", "dB"):
        v = getattr(lay, k)
        setattr(second, k, None if v is None else torch.empty_like(v))
    bufs = [lay, second]
    out_host = [{k: torch.empty_like(getattr(lay, k), device="cpu").pin_memory() for k in outs} for _ in range(2)]
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
    for i in range(steps):
        b = i % 2
        cur = bufs[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[b])        # step i-2 no longer reads these inputs
            for k, v in host.items():
                cur.t[k].copy_(v, non_blocking=True)
            in_ready[b].record(s_in)
        stream.wait_event(in_ready[b])
        if i >= 2:
            stream.wait_event(out_done[b])           # step i-2's results are on the host
        cur.fwd()
        if not fwd_only:
            cur.bwd()
        comp_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            for k in outs:
                out_host[b][k].copy_(getattr(cur, k), non_blocking=True)
            out_done[b].record(s_out)
    for b in range(min(2, steps)):
        stream.wait_event(out_done[b])
    ee1.record(stream)
    torch.cuda.synchronize()
    return ee0.elapsed_time(ee1), h2d, d2h


def run_small_m_line(args, cfg, L, world, rank, local, dist, flush, peaks):
    """Few tokens: forward only, bound by reading W once (HBM roofline); the
    ragged M = 1000 run against the larger of its tensor and HBM times."""
    lay = Layer(L, cfg, seed=rank, pin_host=True)
    r = time_steps(L, lay.fwd, args.steps, args.warmup, flush, lay.stream, local, dist)
    med = statistics.median(r["ms"])
    tot_ms = max_over_ranks(sum(r["ms"]), dist, "cuda")
    roof = small_m_roofline(lay, med, peaks)
    roof["kernel"] = small_m_kernel_name(lay, r["launches"] // max(args.steps, 1))
    if lay.M <= 64:
        roof["traffic"] = committed_traffic(args.config, "small_m_traffic.json", "lora_small_m.cuh")
    F = roof["flop_per_launch"]
    e2e_ms, h2d, d2h = layer_e2e(lay, args.e2e_steps, dist, fwd_only=True)
    e2e_ms = max_over_ranks(e2e_ms, dist, "cuda")
    b2b = small_m_back_to_back(L, lay, peaks)
    line = {"metric": METRIC_SMALL_M, "value": round(job_throughput(F, args.steps, world, tot_ms) / 1e12, 3),
            "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(tot_ms / args.steps, 5), "ms_median": round(med, 5),
            "timing": "per-launch CUDA events, L2 flushed before each (value: total; frac: median launch)",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.config, "M": lay.M, "d_in": lay.d_in, "d_out": lay.d_out, "r": lay.r,
                       "alpha": cfg["alpha"], "act": lay.act, "weight": "w4g64" if lay.w4 else "bf16",
                       "parallelism": f"replicas x{world}", "l2": "flushed before each timed step (512 MiB write)"},
            "roofline": roof, "gpu_launches": r["launches"],
            "back_to_back": b2b,
            "e2e": {"value": round(job_throughput(F, args.e2e_steps, world, e2e_ms) / 1e12, 3), "unit": UNIT,
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
            "clocks": r["clocks"]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, fwd_only=True)
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_ce_line(args, cfg, L, world, rank, local, dist, flush, peaks):
    """The output projection fused with the cross-entropy loss as the line's
    workload (forward + backward per step)."""
    import torch
    ce = CeWorkload(L, cfg, seed=rank, pin_host=True)
    ent, ce, r = measure_ce(L, cfg, local, flush, steps=args.steps, warmup=args.warmup, peaks=peaks, dist=dist,
                            ce=ce)
    tot_ms = max_over_ranks(sum(r["ms"]), dist, "cuda")
    F = ce.step_flops()
    value = job_throughput(F, args.steps, world, tot_ms) / 1e12
    # e2e: per step, H, W and the labels from pinned host memory, the loss and
    # dH back, serialised with the compute
    outs = {"loss": ce.loss, "dH": ce.dH}
    out_host = {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in outs.items()}
    h2d = sum(v.numel() * v.element_size() for v in ce.host.values())
    d2h = sum(v.numel() * v.element_size() for v in out_host.values())
    ee0, ee1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ee0.record(ce.stream)
    for _ in range(args.e2e_steps):
        for k, v in ce.host.items():
            ce.t[k].copy_(v, non_blocking=True)
        ce.step()
        for k, v in outs.items():
            out_host[k].copy_(v, non_blocking=True)
    ee1.record(ce.stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(ee0.elapsed_time(ee1), dist, "cuda")
    pk = peaks["bf16_tflops"]
    lg, dh = ent["logit_gemms"], ent["dh_gemm"]
    dom_is_dh = dh is not None and (lg is None or dh["ms_per_launch"] > lg["ms_per_launch"])
    dom = dh if dom_is_dh else lg
    roof = {"kernel": "lora_mma_kernel (dH = dz W, K = V)" if dom_is_dh
            else "lora_mma_kernel (logits with the cross-entropy epilogue)",
            "bound": "tensor", "achieved": dom["achieved"] if dom else None, "peak": pk, "unit": "TFLOP/s",
            "frac": dom["frac"] if dom else None,
            "peak_kind": f"bf16 burst, {peaks['source']} (sustained {peaks['bf16_tflops_sustained']})",
            "ms_per_launch": dom["ms_per_launch"] if dom else None, "traffic": None,
            "other_gemm": lg if dom_is_dh else dh, "step_frac": round(value / world / pk, 4)}
    line = {"metric": METRIC_CE,
            "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(tot_ms / args.steps, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.config, "M": ce.M, "d": ce.d, "V": ce.V,
                       "flops": "4 M V d per step (logits + dH), each executed once: the fused call keeps "
                                "each chunk's fp32 logits instead of recomputing them",
                       "parallelism": f"replicas x{world}", "l2": "flushed before each timed step (512 MiB write)"},
            "roofline": roof, "gpu_launches": r["launches"],
            "e2e": {"value": round(job_throughput(F, args.e2e_steps, world, e2e_ms) / 1e12, 2), "unit": UNIT,
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                    "copies": "serialised with the compute"},
            "clocks": ent["clocks"]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, max_rows=256)
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="q_proj", choices=sorted(seeded_inputs.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other workloads' entries of the default line")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--shape", default=None,
                    help="M,d_in,d_out,r,act[,p_drop]: this shape instead of --config (profiling, with --calls); "
                         "act 'ce': the output projection + cross-entropy with d_in = hidden, d_out = V; "
                         "p_drop: dropout on the adapter input")
    ap.add_argument("--calls", type=int, default=0,
                    help="run this many untimed forward(+backward) calls, print nothing else, exit (for profilers)")
    ap.add_argument("--fwd-only", action="store_true", help="with --calls: forward calls only")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    cfg = dict(seeded_inputs.CONFIGS[args.config])
    if args.shape:
        f = args.shape.split(",")
        cfg = dict(M=int(f[0]), d_in=int(f[1]), d_out=int(f[2]), r=int(f[3]), alpha=16.0 if int(f[3]) else 0.0,
                   act=f[4])
        if len(f) > 5:
            cfg["dropout"] = float(f[5])
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
    if args.calls > 0:
        lay = CeWorkload(L, cfg, seed=rank) if cfg["act"] == "ce" else Layer(L, cfg, seed=rank)
        for _ in range(args.calls):
            if cfg["act"] == "ce":
                lay.step()
                continue
            lay.fwd()
            if not args.fwd_only:
                lay.bwd()
        torch.cuda.synchronize()
        print("ok", flush=True)
        return
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    peaks = read_peaks()
    if cfg["act"] == "ce":
        run_ce_line(args, cfg, L, world, rank, local, dist, flush, peaks)
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return
    if args.config.startswith("small_m"):
        run_small_m_line(args, cfg, L, world, rank, local, dist, flush, peaks)
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return

    lay = Layer(L, cfg, seed=rank, pin_host=True)

    def step():
        lay.fwd()
        lay.bwd()
    r = time_steps(L, step, args.steps, args.warmup, flush, lay.stream, local, dist)
    tot_ms = max_over_ranks(sum(r["ms"]), dist, "cuda")
    F = lay.step_flops()
    value = job_throughput(F, args.steps, world, tot_ms) / 1e12
    e2e_ms, h2d, d2h = layer_e2e(lay, args.e2e_steps, dist)
    e2e_ms = max_over_ranks(e2e_ms, dist, "cuda")
    e2e = job_throughput(F, args.e2e_steps, world, e2e_ms) / 1e12

    # The dominant kernel: whichever of the two GEMM launches (lora_mma_kernel,
    # forward or dX) took longer per launch, each timed by the library's event
    # pair around its launch on this stream; the other is reported beside it.
    pk = peaks["bf16_tflops"]
    gf = gemm_record(lay.fwd_launch_flops(), r["gemm_fwd_ms"], r["gemm_fwd_n"], 1, pk)
    gb = gemm_record(lay.dx_gemm_flops(), r["gemm_bwd_ms"], r["gemm_bwd_n"], 1, pk)
    traffic = committed_traffic(args.config)
    dom_is_dx = gb is not None and (gf is None or gb["ms_per_launch"] > gf["ms_per_launch"])
    dom, other = (gb, gf) if dom_is_dx else (gf, gb)
    fwd_name = ("lora_mma_kernel (forward GEMM, T accumulated in the GEMM)" if lay.t_in_gemm()
                else "lora_mma_kernel (forward GEMM)")
    roof = {"kernel": "lora_mma_kernel (dX GEMM)" if dom_is_dx else fwd_name,
            "bound": "tensor", "achieved": dom["achieved"] if dom else None, "peak": pk, "unit": "TFLOP/s",
            "frac": dom["frac"] if dom else None,
            "peak_kind": f"bf16 burst, {peaks['source']} (sustained {peaks['bf16_tflops_sustained']})",
            "frac_of_sustained": round(dom["achieved"] / peaks["bf16_tflops_sustained"], 4) if dom else None,
            "flop_per_launch": dom["flop_per_step"] if dom else None,
            "ms_per_launch": dom["ms_per_launch"] if dom else None,
            "traffic": (traffic or {}).get("dx" if dom_is_dx else "forward") if isinstance(traffic, dict) else None,
            "other_gemm": dict(other or {}, kernel=fwd_name if dom_is_dx else "lora_mma_kernel (dX GEMM)",
                               traffic=(traffic or {}).get("forward" if dom_is_dx else "dx")
                               if isinstance(traffic, dict) else None),
            "step_frac": round(value / world / pk, 4)}

    line = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(tot_ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.config, "M": lay.M, "d_in": lay.d_in, "d_out": lay.d_out, "r": lay.r,
                       "alpha": cfg["alpha"], "act": lay.act, "parallelism": f"replicas x{world}",
                       "l2": "flushed before each timed step (512 MiB write)",
                       **({"dropout": lay.p_drop} if lay.p_drop is not None else {})},
            "roofline": roof, "gpu_launches": r["launches"],
            "e2e": {"value": round(e2e, 2), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h)},
            "clocks": r["clocks"]}
    if world == 1 and args.config == "q_proj" and not args.no_workloads:
        # every other workload of the build, each timed on its own (N = 1)
        del lay
        torch.cuda.empty_cache()
        wl = {}

        def entry(name, fn):
            # a workload that fails is reported as such; the others still run
            try:
                wl[name] = fn()
            except Exception as e:  # noqa: BLE001
                wl[name] = {"error": f"{type(e).__name__}: {e}"[:300]}
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
        for name in ("tiny", "v_proj"):
            entry(name, lambda name=name: measure_layer_workload(L, name, local, flush, peaks=peaks))
        entry("mlp", lambda: measure_mlp(L, local, flush, peaks=peaks))
        for name in ("small_m", "small_m_ragged"):
            entry(name, lambda name=name: measure_small_m(L, name, local, flush, peaks=peaks)[0])
        entry("lm_head_ce",
              lambda: measure_ce(L, dict(seeded_inputs.CONFIGS["lm_head_ce"]), local, flush, peaks=peaks)[0])
        line["workloads"] = wl
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
