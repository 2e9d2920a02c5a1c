"""Benchmark of the SRNL four-direction scan forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one full forward (query projection, the four route scans, restore +
channel fusion) over one batch of the workload, inputs resident in HBM.  The
L2 cache (126 MB) is flushed before every timed step by writing a 256 MiB
buffer outside the timed events.  Rank 0 prints one JSON line.

Multi-GPU (torchrun, N > 1): the sequences are independent, so every rank runs
its own replica of the workload with no collective on the data path (weak
scaling); the time is the max over ranks.

``--impl reference`` times the float64 CPU oracle (the slow, plain definition
the parity tests use) on the host cores over a bounded sample of the same
workload; it is the baseline arm, not a target.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from srnl_inputs import CONFIGS, Sustain, make_inputs  # noqa: E402

METRIC = "SRNL 4-dir scan tokens/s (fwd, 1xB200) and % of roofline at 56x56x64"

# DRAM bytes (read + write) of one scan launch, from a 1-pass ncu capture of the current
# chunkwise kernel on the full workload (profiles/scan_dram_hier_s1_56x56.md): 13.08 MB read (x
# once; the scan forms q itself) + 2.17 MB written (the bf16 route partials stay in L2 for the
# fusion).  Keyed by (workload, B, generation dtype); absent entries report null.
SCAN_TRAFFIC_BYTES = {("hier_s1_56x56", 32, "bf16"): 13.08e6 + 2.17e6}
UNIT = "route-tokens/s"
DEFAULT_CONFIG = "hier_s1_56x56"
L2_FLUSH_BYTES = 256 << 20

# Fallback peaks only when the measured file is absent.
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                    sm_max_mhz=d.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm_gbs=FALLBACK_HBM_GBS, bf16_tflops=FALLBACK_BF16_TFLOPS,
                bf16_tflops_sustained=1400.0, sm_max_mhz=1965.0, source="fallback")


# ----------------------------------------------------------------- work model
def scan_fuses_query(cfg, gen):
    """Whether the library's scan forms the queries itself (no projection launch): bf16
    activations and generation, two 32-wide heads (C = 64), chunks of at most 64 tokens, column
    chunks inside a column.  Mirrors the library's launch rule, for the launch count."""
    lr, lc = cfg.chunk_row or cfg.W, cfg.chunk_col or cfg.H
    return (cfg.act_dtype == "bf16" and gen == "bf16" and cfg.d == 32 and cfg.C == 64 and lr <= 64 and lc <= 64
            and lc <= cfg.H and cfg.H % lc == 0)


def work_model(cfg, gen_bf16=True):
    """Algorithmic bytes and flops of one forward (per launch)."""
    B, H, W, C, heads, d = cfg.B, cfg.H, cfg.W, cfg.C, cfg.heads, cfg.d
    N = H * W
    tokens = B * N
    elt = 2 if cfg.act_dtype == "bf16" else 4
    param_bytes = 4 * (C * C + 4 * C + 4 * heads * (3 * d * d + 2 * d))
    hbm_bytes = 2 * tokens * C * elt + param_bytes          # x read once, y written once, params
    seq_tokens = 4 * tokens * heads                          # (route, head) token steps
    gen_flops = 2.0 * seq_tokens * (2 * d + 2) * d           # boundary generation contraction
    qproj_flops = 2.0 * tokens * C * C
    # Sequential update on the single-product state, per (route, head) token:
    #   s = row . u (2 d^2), row <- alpha row - (eta s) k (3 d^2), z = row . q (2 d^2),
    #   readout y = M_mem0 z (2 d^2); plus the boundary product G Q_b once per chunk.
    upd_flops_tok = 9.0 * d * d
    Lr = cfg.chunk_row or W
    Lc = cfg.chunk_col or H
    chunks = B * heads * 2 * (-(-N // Lr) + -(-N // Lc))
    boundary_flops = 2.0 * chunks * (2 * d + 2) * d * d
    scan_flops = seq_tokens * upd_flops_tok + gen_flops + boundary_flops
    return dict(tokens=tokens, route_tokens=4 * tokens, hbm_bytes=hbm_bytes, gen_flops=gen_flops,
                qproj_flops=qproj_flops, scan_flops=scan_flops, update_flops=seq_tokens * upd_flops_tok,
                seq_tokens=seq_tokens)


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.rows = []
        self._proc = None
        self._thr = None

    def start(self):
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self._proc = None
            return
        self._thr = threading.Thread(target=self._read, daemon=True)
        self._thr.start()

    def _read(self):
        for line in self._proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def stop(self):
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
        if self._thr is not None:
            self._thr.join(timeout=2)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


# ----------------------------------------------------------------- CPU oracle arm
def oracle_sample(cfg, n_images, seed=0):
    """Time the float64 oracle on the first n_images of the workload (1 host thread)."""
    from oracle import srnl_oracle as O
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:  # pragma: no cover
        threadpool_limits = None
    inp = make_inputs(cfg, seed=seed)
    ctx = threadpool_limits(1) if threadpool_limits else None
    t0 = time.perf_counter()
    try:
        O.operator_forward(inp.x32[:n_images], inp.params(), alpha_max=cfg.alpha, eps=cfg.eps,
                           chunk_row=cfg.chunk_row, chunk_col=cfg.chunk_col, heads=cfg.heads)
    finally:
        if ctx is not None:
            ctx.__exit__(None, None, None)
    dt = time.perf_counter() - t0
    return 4.0 * n_images * cfg.H * cfg.W / dt, dt


def cpu_baseline(cfg, budget_s=12.0):
    one_rate, one_dt = oracle_sample(cfg, 1)
    n = max(1, min(cfg.B, int(budget_s / max(one_dt, 1e-3))))
    rate, dt = oracle_sample(cfg, n) if n > 1 else (one_rate, one_dt)
    return {"value": rate, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{n} of {cfg.B} images of {cfg.name}, float64 numpy, 1 thread, {dt:.1f} s"}


def run_reference(args, cfg, rank, world):
    if rank != 0:
        return
    per_step = []
    n_images = 1
    for _ in range(args.warmup if args.warmup < 1 else 1):
        oracle_sample(cfg, n_images)
    for _ in range(args.steps):
        rate, dt = oracle_sample(cfg, n_images)
        per_step.append(dt)
    t = sum(per_step)
    value = 4.0 * n_images * cfg.H * cfg.W * args.steps / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "W": cfg.W,
                                            "C": cfg.C, "heads": cfg.heads, "d": cfg.d,
                                            "step_sample_images": n_images},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"{n_images} image of {cfg.name} per step, float64 numpy, 1 thread"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- GPU arm
def max_over_ranks(values, world, device=None):
    """Each value's maximum over the ranks: a replica job takes as long as its slowest rank.
    Every rank calls it (one all-reduce), with the same number of values."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def whole_job_rate(world, units_per_step, steps, total_ms):
    """Units all ranks processed (each rank runs the whole workload) over the job's time."""
    return world * units_per_step * steps / (total_ms * 1e-3)


def stages_per_sequence(cfg, stage=64):
    """Dependent stages of the longest route: chunks x ceil(chunk / stage)."""
    n = 0
    N = cfg.H * cfg.W
    for L in (cfg.chunk_row or cfg.W, cfg.chunk_col or cfg.H):
        chunks = -(-N // L)
        last = N - (chunks - 1) * L
        n = max(n, (chunks - 1) * (-(-L // stage)) + -(-last // stage))
    return n


def chain_latency_ms(S, cfgd, params, x, stream, steps=5):
    """Scan time of one image.  Its 4 x heads sequences each get an SM of their own, so the
    time is one sequence's chain of dependent stages with nothing else on the GPU: the bound
    that batching cannot go below."""
    import torch
    h1 = S.srnl_scan_create(dict(cfgd, B=1), params)
    x1 = x[:1].contiguous()
    y1 = torch.empty_like(x1)
    for _ in range(3):
        S.srnl_scan_forward(h1, x1, y1, None, stream)
    S.srnl_scan_enable_stage_timing(h1, steps)
    for _ in range(steps):
        S.srnl_scan_forward(h1, x1, y1, None, stream)
    torch.cuda.synchronize()
    stage, n = S.srnl_scan_stage_times(h1)
    h1.close()
    return float(stage[1])


def run_ours(args, cfg, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import self_referential_nested_b200 as S
    from self_referential_nested_b200 import build as B

    B.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    gen = args.gen or cfg.act_dtype
    act = cfg.act_dtype
    if args.sustain:
        inp = make_inputs(cfg, seed=rank, mem_scale=0.3, vec_scale=0.05, sustain=Sustain())
    else:
        inp = make_inputs(cfg, seed=rank)
    cfgd = dict(B=cfg.B, H=cfg.H, W=cfg.W, C=cfg.C, heads=cfg.heads, d=cfg.d, alpha=cfg.alpha,
                eps=cfg.eps, chunk_row=cfg.chunk_row, chunk_col=cfg.chunk_col, act_dtype=act,
                gen_dtype=gen, injection_cap=args.cap)
    h = S.srnl_scan_create(cfgd, inp.params())
    if act == "bf16":
        x = torch.from_numpy(inp.x_bits.view(np.int16)).to(dev).view(torch.bfloat16)
    else:
        x = torch.from_numpy(inp.x32).to(dev)
    y = torch.empty_like(x)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    S.srnl_scan_enable_stage_timing(h, 0)

    def barrier():
        if world > 1:
            dist.barrier()

    for i in range(args.warmup):
        flush.fill_(i & 0xFF)
        S.srnl_scan_forward(h, x, y, None, stream)
    torch.cuda.synchronize()

    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    S.srnl_scan_enable_stage_timing(h, max(args.steps, 1))
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_((i + 1) & 0xFF)                 # evict x / workspace from L2 (untimed)
        starts[i].record(stream)
        S.srnl_scan_forward(h, x, y, None, stream)
        ends[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    stage, n_timed = S.srnl_scan_stage_times(h)
    assert n_timed == args.steps
    S.srnl_scan_enable_stage_timing(h, 0)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = float(sum(step_ms))

    # warm: the same steps back to back, inputs left in L2 (reported beside the cold figure)
    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0.record(stream)
    for _ in range(args.steps):
        S.srnl_scan_forward(h, x, y, None, stream)
    w1.record(stream)
    torch.cuda.synchronize()
    warm_ms = w0.elapsed_time(w1) / args.steps

    # end to end through the host-buffer entry point: pinned x in, y out, every step
    xh = x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    # pipelined host-buffer forwards: step i+1's input copy and step i's output copy overlap
    # the neighbouring forwards; the end event waits for the last output copy
    for _ in range(2):
        S.srnl_scan_forward_host_async(h, xh, yh, stream)
    S.srnl_scan_host_sync(h)
    e2e_s, e2e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e2e_s.record(stream)
    for _ in range(args.steps):
        S.srnl_scan_forward_host_async(h, xh, yh, stream)
    S.srnl_scan_host_join(h, stream)
    e2e_e.record(stream)
    torch.cuda.synchronize()
    S.srnl_scan_host_sync(h)
    barrier()
    clocks.stop()
    e2e_ms = e2e_s.elapsed_time(e2e_e)

    total_ms, e2e_ms, warm_ms = max_over_ranks([total_ms, e2e_ms, warm_ms], world, dev)
    cap_active = S.srnl_scan_cap_count(h) if args.cap == "hard" else 0
    h.close()
    if rank != 0:
        return
    chain_ms = chain_latency_ms(S, cfgd, inp.params(), x, stream)
    n_stages = stages_per_sequence(cfg)

    wm = work_model(cfg)
    peaks = load_peaks()
    ms_step = total_ms / args.steps
    value = whole_job_rate(world, wm["route_tokens"], args.steps, total_ms)
    e2e_value = whole_job_rate(world, wm["route_tokens"], args.steps, e2e_ms)
    stage_ms = np.asarray(stage)
    scan_ms = float(stage_ms[1])
    # Roofline of the dominant kernel (the scan) as the hot-path table defines it: the larger of
    # the forward's algorithmic bytes (x read once, y written once, parameters) over HBM
    # bandwidth and its generation + projection flops over the dense bf16 tensor peak, against
    # the scan kernel's own launch time.
    t_bytes_us = wm["hbm_bytes"] / (peaks["hbm_gbs"] * 1e9) * 1e6
    t_tensor_us = (wm["gen_flops"] + wm["qproj_flops"]) / (peaks["bf16_tflops"] * 1e12) * 1e6
    roof_us = max(t_bytes_us, t_tensor_us)
    if t_bytes_us >= t_tensor_us:
        roof = {"bound": "hbm", "achieved": wm["hbm_bytes"] / (scan_ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": (wm["gen_flops"] + wm["qproj_flops"]) / (scan_ms * 1e-3) / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    # The token-order update, reported beside the roofline: its sequential-form fp32 flops
    # (9 d^2 per (route, head) token: the solve's row products, the rank-one write, the readout
    # and y = M_mem0 z) over the fp32 FMA peak.  Generation runs on the tensor cores and is not
    # counted here.
    fp32_peak_tflops = 148 * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12
    upd_tflops = wm["update_flops"] / (scan_ms * 1e-3) / 1e12
    elt = 2 if act == "bf16" else 4
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if gen == "bf16" else "f32",
        "data": ("synthetic (seeded normal features, random-init memories)" if not args.sustain else
                 "synthetic, sustained (constant feature channel, retention bias, alpha 0.999)"),
        "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "W": cfg.W, "C": cfg.C,
                   "heads": cfg.heads, "d": cfg.d, "alpha": cfg.alpha, "chunk_row": cfg.chunk_row or cfg.W,
                   "chunk_col": cfg.chunk_col or cfg.H, "act_dtype": act, "gen_dtype": gen,
                   "states": "f32", "l2": "flushed (256 MiB write before each timed step)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "raster_tokens_per_s": value / 4},
        "roofline": dict(roof, **{
            "traffic": SCAN_TRAFFIC_BYTES.get((cfg.name, cfg.B, gen)), "traffic_unit": "bytes/launch",
            "kernel": ("srnl_scan_d64_kernel" if cfg.d == 64 else
                       "srnl_scan_chunkwise_kernel" if gen == "bf16" else "srnl_scan_sequential_kernel"),
            "kernel_ms": scan_ms, "roofline_us": roof_us, "algorithmic_bytes": wm["hbm_bytes"],
            "algorithmic_tensor_flops": wm["gen_flops"] + wm["qproj_flops"],
            "peak_note": f"{peaks['source']} peaks ({peaks['hbm_gbs']} GB/s HBM copy, "
                         f"{peaks['bf16_tflops']} TF/s dense bf16)",
            "target_0_40_reached": bool(roof["frac"] >= 0.40)}),
        "sequential_update_share": {"bound": "alu", "achieved": upd_tflops, "peak": fp32_peak_tflops,
                                    "unit": "TFLOP/s", "frac": upd_tflops / fp32_peak_tflops,
                                    "flops": wm["update_flops"],
                                    "peak_note": "fp32 FMA peak 148 SM x 128 lanes x 2 x sm_max_mhz (derived)"},
        "forward_roofline": {"bound": "hbm" if t_bytes_us >= t_tensor_us else "tensor",
                                "roofline_us": roof_us, "forward_us": ms_step * 1e3,
                                "frac": roof_us / (ms_step * 1e3),
                                "hbm_bytes": wm["hbm_bytes"], "tensor_flops": wm["gen_flops"] + wm["qproj_flops"],
                                "peaks": f"{peaks['source']}: {peaks['hbm_gbs']} GB/s, {peaks['bf16_tflops']} TF/s bf16"},
        "stage_ms": {"query_projection": float(stage_ms[0]), "scan": scan_ms, "fusion": float(stage_ms[2])},
        "injection_cap": {"mode": args.cap,
                          "active_frac": cap_active / (4.0 * cfg.B * cfg.H * cfg.W * cfg.heads)
                          if args.cap == "hard" else None},
        "warm_ms_per_step": warm_ms,
        "chain": {"stages_per_sequence": n_stages, "one_image_scan_us": chain_ms * 1e3,
                  "per_stage_us": chain_ms * 1e3 / n_stages, "scan_us": scan_ms * 1e3,
                  "frac": chain_ms / scan_ms,
                  "note": "scan of one image (each sequence alone on an SM) over the full scan"},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(x.numel() * elt),
                "d2h_bytes_per_step": int(y.numel() * elt), "ms_per_step": e2e_ms / args.steps},
        # projection (unless the scan forms q), scan, fusion; + pad x, unpad y below 32
        "gpu_launches": ((2 if scan_fuses_query(cfg, gen) else 3) + (0 if cfg.d >= 32 else 2)) * args.steps,
        "clocks": clocks.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
        line["cpu_baseline"]["gpu_over_cpu"] = value / line["cpu_baseline"]["value"]
    print(json.dumps(line), flush=True)


def backward_flops_per_token(d=32):
    """Algorithmic fp32 flops of the backward per (route, head) token, as the scan-backward
    kernel restates it: the forward chain twice (checkpoint pass and in-chunk recompute,
    2 x 5 d^2), generation once (Q_b x and G w: 2 d^2 + 2 (2d+2) d), the reverse chain
    (dQ += a q^T, dQ k, Q_{t-1} u, Q_t q, <Q_{t-1}, dQ>, the three column products and the
    dQ update: 19 d^2), the per-token adjoints (M0^T dy, G^T dgen, Q_b x, M0 z, Q_b^T dh:
    8 d^2 + 2 (2d+2) d) and the rank-one parameter sums (dM0, dQ_b, dG: 4 d^2 + 2 (2d+2) d)."""
    gen = 2 * (2 * d + 2) * d
    return 10 * d * d + (2 * d * d + gen) + 19 * d * d + (8 * d * d + gen) + (4 * d * d + gen)


def backward_cpu_baseline(cfg, budget_s=10.0):
    from oracle import srnl_grad as GR
    from srnl_inputs import make_cotangent
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:  # pragma: no cover
        threadpool_limits = None
    inp = make_inputs(cfg, seed=0)
    dout = make_cotangent(inp.x32.shape, seed=0, act_dtype=cfg.act_dtype)
    n, dt = 1, 0.0
    ctx = threadpool_limits(1) if threadpool_limits else None
    try:
        while True:
            t0 = time.perf_counter()
            GR.operator_backward(inp.x32[:n], inp.params(), dout[:n], alpha_max=cfg.alpha, eps=cfg.eps,
                                 chunk_row=cfg.chunk_row, chunk_col=cfg.chunk_col, heads=cfg.heads)
            dt = time.perf_counter() - t0
            if dt * 2 > budget_s or n >= cfg.B:
                break
            n = min(cfg.B, max(n + 1, int(n * budget_s / max(dt, 1e-3) / 2)))
    finally:
        if ctx is not None:
            ctx.__exit__(None, None, None)
    return {"value": 4.0 * n * cfg.H * cfg.W / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"backward of {n} of {cfg.B} images of {cfg.name}, float64 numpy, 1 thread, {dt:.1f} s"}


def run_backward(args, cfg):
    """Backward pass: dL/dx and every parameter gradient for an upstream gradient dL/dy, on one
    GPU (fp32 arithmetic; x, dy and dx in the workload's activation dtype).  One step = one
    srnl_scan_backward over the batch, inputs resident in HBM, L2 flushed before each step."""
    import torch
    import self_referential_nested_b200 as S
    from self_referential_nested_b200 import build as Bld
    from srnl_inputs import make_cotangent

    Bld.build()
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    act = cfg.act_dtype
    inp = make_inputs(cfg, seed=0)
    params = inp.params()
    h = S.srnl_scan_create(dict(B=cfg.B, H=cfg.H, W=cfg.W, C=cfg.C, heads=cfg.heads, d=cfg.d, alpha=cfg.alpha,
                                eps=cfg.eps, chunk_row=cfg.chunk_row, chunk_col=cfg.chunk_col, act_dtype=act,
                                gen_dtype="f32", injection_cap=args.cap), params)
    g_np = make_cotangent(inp.x32.shape, seed=0, act_dtype=act)

    def to_dev(a32):
        if act == "bf16":
            from srnl_inputs import bf16_round_bits
            return torch.from_numpy(bf16_round_bits(a32).view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a32)).to(dev)

    x, dy = to_dev(inp.x32), to_dev(g_np)
    dx = torch.empty_like(x)
    grads = {k: torch.empty(np.shape(params[k]), dtype=torch.float32, device=dev) for k in S.GRAD_KEYS}
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for i in range(args.warmup):
        flush.fill_(i & 0xFF)
        S.srnl_scan_backward(h, x, dy, dx, grads, stream)
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    S.srnl_scan_enable_stage_timing(h, max(args.steps, 1))
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_((i + 1) & 0xFF)
        starts[i].record(stream)
        S.srnl_scan_backward(h, x, dy, dx, grads, stream)
        ends[i].record(stream)
    torch.cuda.synchronize()
    stage, n_timed = S.srnl_scan_stage_times(h)
    assert n_timed == args.steps
    S.srnl_scan_enable_stage_timing(h, 0)
    total_ms = float(sum(s_.elapsed_time(e_) for s_, e_ in zip(starts, ends)))
    # end to end: pinned x and dy copied in, dx and the parameter gradients copied out, each step
    xh, dyh = x.cpu().pin_memory(), dy.cpu().pin_memory()
    dxh = torch.empty_like(xh).pin_memory()
    gh = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in grads.items()}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        x.copy_(xh, non_blocking=True)
        dy.copy_(dyh, non_blocking=True)
        S.srnl_scan_backward(h, x, dy, dx, grads, stream)
        dxh.copy_(dx, non_blocking=True)
        for k in grads:
            gh[k].copy_(grads[k], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.stop()
    e2e_ms = e0.elapsed_time(e1)
    h.close()

    peaks = load_peaks()
    ms_step = total_ms / args.steps
    route_tokens = 4 * cfg.B * cfg.H * cfg.W
    scan_ms = float(stage[1])
    flops = backward_flops_per_token(cfg.d) * route_tokens * cfg.heads
    fp32_peak_tflops = 148 * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12
    achieved = flops / (scan_ms * 1e-3) / 1e12
    elt = 2 if act == "bf16" else 4
    grad_bytes = int(sum(v.numel() for v in grads.values()) * 4)
    line = {
        "metric": "SRNL 4-dir scan backward route-tokens/s (1xB200)", "value": route_tokens / (ms_step * 1e-3),
        "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded normal features and upstream gradients, random-init memories)",
        "config": {"workload": cfg.name, "pass": "backward", "B": cfg.B, "H": cfg.H, "W": cfg.W, "C": cfg.C,
                   "heads": cfg.heads, "d": cfg.d, "alpha": cfg.alpha, "act_dtype": act, "gen_dtype": "f32",
                   "injection_cap": args.cap, "l2": "flushed (256 MiB write before each timed step)"},
        "roofline": {"bound": "alu", "achieved": achieved, "peak": fp32_peak_tflops, "unit": "TFLOP/s",
                     "frac": achieved / fp32_peak_tflops, "traffic": None,
                     "kernel": "srnl_scan_backward64_kernel" if cfg.d == 64 else "srnl_scan_backward_kernel",
                     "kernel_ms": scan_ms, "flops_per_route_head_token": backward_flops_per_token(cfg.d),
                     "peak_note": "fp32 FMA peak 148 SM x 128 lanes x 2 x sm_max_mhz (derived)"},
        "stage_ms": {"query_projection": float(stage[0]), "scan_backward": scan_ms, "combine": float(stage[2])},
        "e2e": {"value": route_tokens * args.steps / (e2e_ms * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": int(2 * x.numel() * elt), "d2h_bytes_per_step": int(dx.numel() * elt) + grad_bytes,
                "ms_per_step": e2e_ms / args.steps},
        "gpu_launches": (7 if cfg.d >= 32 else 10) * args.steps,   # + pad x, pad dy, unpad dx below 32
        "clocks": clocks.summary(),
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = backward_cpu_baseline(cfg)
    print(json.dumps(line), flush=True)


def run_seq(args):
    """Standalone SRNL layer on sequences ([B, T, D], 64-token chunks, x as the query):
    B sequences x heads of T tokens, one direction.  One GPU; prints one JSON line."""
    import torch
    import self_referential_nested_b200 as S
    from self_referential_nested_b200 import build as Bld
    from srnl_inputs import make_seq_inputs

    Bld.build()
    B, T, D, heads = args.seq_batch, args.seq_tokens, 64, 2
    inp = make_seq_inputs(B, T, D, heads, "bf16", seed=0)
    cfg = dict(B=B, T=T, D=D, heads=heads, d=32, alpha=0.95, eps=1e-6, chunk=64, act_dtype="bf16",
               gen_dtype="bf16")
    h = S.srnl_seq_create(cfg, inp.params())
    x = torch.from_numpy(inp.x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    y = torch.empty_like(x)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        flush.fill_(i & 0xFF)
        S.srnl_seq_forward(h, x, y, stream=stream)
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    ts = []
    for i in range(args.steps):
        flush.fill_((i + 1) & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        S.srnl_seq_forward(h, x, y, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    clocks.stop()
    S.srnl_seq_device_status(h)
    h.close()
    ms = float(np.mean(ts))
    print(json.dumps({"metric": "SRNL sequence layer tokens/s (fwd, 1xB200)", "value": B * T / (ms * 1e-3),
                      "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
                      "ms_per_step": ms, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
                      "config": {"workload": f"seq_b{B}_t{T}_d{D}", "B": B, "T": T, "D": D, "heads": heads,
                                 "d": 32, "chunk": 64, "queries": "x", "l2": "flushed before each step"},
                      "clocks": clocks.summary()}), flush=True)


def run_block(args):
    """Time the residual block around the operator on the S1 map (B = 32, 56 x 56, dim 64,
    mixer_dim 64, head_dim 32, bf16): LayerNorm, four tensor-core projections, depthwise
    convolution, the operator and the FFN per forward."""
    import torch
    import self_referential_nested_b200 as S
    from self_referential_nested_b200 import build as Bld
    from srnl_inputs import make_block_inputs

    Bld.build()
    B, H, W, dim, m, hd = args.batch or 32, 56, 56, 64, 64, 32
    inp = make_block_inputs(B, H, W, dim, m, hd, "bf16", seed=0)
    h = S.srnl_block_create(dict(B=B, H=H, W=W, dim=dim, mixer_dim=m, head_dim=hd, alpha=0.95, gen_dtype="bf16"),
                            inp.p)
    x = torch.from_numpy(inp.x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    y = torch.empty_like(x)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        flush.fill_(i & 0xFF)
        S.srnl_block_forward(h, x, y, stream)
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    ts = []
    for i in range(args.steps):
        flush.fill_((i + 1) & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        S.srnl_block_forward(h, x, y, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    clocks.stop()
    S.srnl_block_device_status(h)
    h.close()
    ms = float(np.mean(ts))
    print(json.dumps({"metric": "VisionHOPE block tokens/s (fwd, 1xB200)", "value": B * H * W / (ms * 1e-3),
                      "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
                      "ms_per_step": ms, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
                      "config": {"workload": f"block_b{B}_56x56_dim{dim}_mixer{m}", "B": B, "H": H, "W": W,
                                 "dim": dim, "mixer_dim": m, "head_dim": hd, "l2": "flushed before each step"},
                      "clocks": clocks.summary()}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--gen", default=None, choices=[None, "f32", "bf16"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cap", default="soft", choices=["soft", "hard"],
                    help="injection cap: the soft cap (the method) or the hard clamp of its ablation")
    ap.add_argument("--batch", type=int, default=0, help="override B (small profiling cases)")
    ap.add_argument("--head-dim", type=int, default=0, choices=[0, 4, 8, 16, 32, 64],
                    help="override the head dim (C = heads x d); 64 defaults to the fp32-generation path")
    ap.add_argument("--seq", action="store_true", help="time the standalone sequence layer instead")
    ap.add_argument("--block", action="store_true", help="time the residual block around the operator instead")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (gradients of x and every parameter) instead")
    ap.add_argument("--sustain", action="store_true",
                    help="time the workload's shape on sustained inputs (retention cap 0.999, a constant "
                         "feature channel and a retention bias keep every chunk inside fp32 range)")
    ap.add_argument("--seq-batch", type=int, default=128)
    ap.add_argument("--seq-tokens", type=int, default=3136)
    args = ap.parse_args()
    if args.seq:
        run_seq(args)
        return
    if args.block:
        run_block(args)
        return
    cfg = CONFIGS[args.config]
    if args.batch > 0:
        cfg = cfg.replace(B=args.batch)
    if args.sustain:
        cfg = cfg.replace(alpha=0.999)
    if args.head_dim > 0:
        cfg = cfg.replace(d=args.head_dim, C=cfg.heads * args.head_dim)
        if args.head_dim == 64 and args.gen is None:
            args.gen = "f32"
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world == 1 and args.gpus > 1:
        print(json.dumps({"error": "launch N>1 with torchrun"}), flush=True)
        sys.exit(2)
    if args.impl == "reference":
        run_reference(args, cfg, rank, world)
        return
    if args.backward:
        run_backward(args, cfg)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, cfg, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
