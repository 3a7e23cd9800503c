"""Benchmark of the GSQ layer-reconstruction step on B200.

Default workload: the Llama-3.1-70B-shaped transformer block (hidden 8192,
64 query / 8 key-value heads of 128, SwiGLU 28672, 8 x 2048 tokens, 2-bit
grid).  One bench step is one GSQ step of every stage of the block: the Q
and K layers, the V/O joint stage and the MLP joint stage (seven weights,
8.55e8 grid coordinates).  Each stage step is the whole hot path: Philox
Gumbel soft weight, forward GEMMs with the fused loss / output gradient,
weight-gradient GEMMs, fused logit/scale gradients with Lion (and the next
step's soft weight).  Under torchrun each rank quantizes its own block (weak
scaling, no data-path collective).

    python bench.py [--gpus N] [--steps K] [--warmup W]     # the 70B block step
    python bench.py --config NAME [--split rows] ...          # one layer
    python bench.py --stage mlp|attn|scale|gptq|block|kquant  # one stage
    python bench.py --impl reference ...   # the oracle on the host cores

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import dataclasses
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

from post_weight_quantization_philox_b200 import synth  # noqa: E402

METRIC = "GSQ recon steps/s and grid coords updated/s per layer; % of TC / HBM roofline"
UNIT = "coords/s"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d["bf16_tflops_sustained"], "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi samples during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except FileNotFoundError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def phase_bytes_flops(cfg, layer, es=4):
    """Algorithmic bytes (HBM phases) and flops (GEMMs) of one launch: what
    the method itself must move per coordinate, es being the bytes of one
    logit / momentum element (4, or 2 in the bf16 state).

    soft weight:        read the L logit planes (+ the int8 initial level of
                        the 3-bit grid), write the bf16 weight; 4 B per group
                        of scales;
    backward + Lion:    read dW, read and write the L logit and L momentum
                        planes (+ initial level); 16 B per group (scale and
                        its momentum, read and written);
    ... + next soft:    also write the next step's bf16 weight.
    The kernels keep nothing else between launches: the backward draws the
    step's noise again from its counters."""
    NK = cfg.N * cfg.K
    L = layer.L
    extra = 1 if cfg.grid == synth.GRID_3BIT_LOCAL else 0  # initial level (int8)
    groups = cfg.N * (cfg.K // 128)
    soft = NK * (es * L + 2 + extra) + groups * 4
    back = NK * (4 + 4 * es * L + extra) + groups * 16
    back_next = back + NK * 2
    gemm = 2.0 * cfg.N * cfg.T * cfg.K
    return {"soft_weight": ("hbm", soft), "forward_gemm": ("tensor", gemm),
            "weight_grad_gemm": ("tensor", gemm), "backward_lion": ("hbm", back),
            "backward_lion_next_soft": ("hbm", back_next)}


def step_roofline(work, ms_step, tf, hbm):
    """A steady step (both GEMMs and the fused backward with the next soft
    weight) at the peaks: the GEMM flops at the bf16 rate tf plus the
    backward's algorithmic bytes at the copy rate, against the measured step."""
    gemm_ms = (work["forward_gemm"][1] + work["weight_grad_gemm"][1]) / (tf * 1e12) * 1e3
    hbm_ms = work["backward_lion_next_soft"][1] / (hbm * 1e9) * 1e3
    return {"gemm_ms": round(gemm_ms, 4), "hbm_ms": round(hbm_ms, 4),
            "ms": round(gemm_ms + hbm_ms, 4), "frac": round((gemm_ms + hbm_ms) / ms_step, 4),
            "how": "GEMM flops at the burst bf16 rate + the fused backward's algorithmic "
                   "bytes at the copy rate, over the measured step"}


def run_gsq(args, rank, world, local_rank):
    import torch
    from post_weight_quantization_philox_b200 import build
    if rank == 0 or not os.path.exists(os.path.join(ROOT, "post_weight_quantization_philox_b200", "libgsq.so")):
        build.build()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    from post_weight_quantization_philox_b200 import gsq

    torch.cuda.set_device(local_rank)
    full = synth.CONFIGS[args.config]
    cfg = full
    if args.rows:
        # the first rows of the layer (rows are independent problems): a
        # smaller case of the same kernels, e.g. for profiling
        if args.rows % 256 or not 0 < args.rows <= full.N:
            raise SystemExit(f"--rows must be a multiple of 256 in (0, {full.N}]")
        cfg = dataclasses.replace(full, N=args.rows, name=f"{full.name}_rows{args.rows}")
    split = args.split == "rows"
    row0 = None
    if split:
        # one layer split by rows over the ranks: the same layer and Philox
        # seed everywhere, rank r holds band r keyed by its global row offset
        w_seed, x_seed, philox_seed = layer_seeds(cfg, 0)
        row0, n = row_shard(cfg.N, rank, world)
        W = synth.make_weight(full, seed=w_seed, rows=slice(row0, row0 + n))
        cfg = dataclasses.replace(cfg, N=n)
    else:
        # each rank quantizes its own independent layer of the same shape
        w_seed, x_seed, philox_seed = layer_seeds(full, rank)
        W = synth.make_weight(full, seed=w_seed, rows=slice(0, cfg.N))
    X = synth.make_calib(full, seed=x_seed)
    Wd = torch.from_numpy(W).to(torch.bfloat16).cuda()
    Xd = torch.from_numpy(X).to(torch.bfloat16).cuda()
    stream = torch.cuda.current_stream()
    state16 = args.state == "bf16"
    lay = gsq.gsq_init(Wd, Xd, 128, cfg.grid, seed=philox_seed, state_bf16=state16, row0=row0)
    taus = synth.tau_schedule(cfg.tau0, cfg.tau1, cfg.steps)
    nt = len(taus)

    def dist_barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    sched = np.array([taus[i % nt] for i in range(args.warmup + args.steps)], np.float32)
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)  # sampler up before the GPU work starts
    # warm-up steps right before the timed region (clocks ramped up)
    lay.run(sched[:args.warmup], cfg.lr)
    dist_barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    # the timed region: the library's own launches only (no per-phase events
    # between its kernels, which would keep each from starting before the
    # previous one ends)
    e0.record(stream)
    lay.run(sched[args.warmup:], cfg.lr)
    e1.record(stream)
    torch.cuda.synchronize()
    dist_barrier()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    loss = lay.last_loss()
    # the per-phase breakdown from a second, instrumented run of the same
    # steps (its events separate the kernels)
    gsq.gsq_set_timing(lay, True)
    gsq.gsq_phase_times(lay)  # reset (syncs)
    lay.run(sched[args.warmup:], cfg.lr)
    phase_ms, phase_n = gsq.gsq_phase_times(lay)
    gsq.gsq_set_timing(lay, False)
    # the same steps through the per-step call: gsq_step_next announces the
    # next temperature, so its backward forms the next soft weight
    e0.record(stream)
    for i in range(args.warmup, args.warmup + args.steps):
        nxt = float(sched[i + 1]) if i + 1 < len(sched) else None
        lay.step(float(sched[i]), cfg.lr, tau_next=nxt)
    e1.record(stream)
    torch.cuda.synchronize()
    step_next_ms = e0.elapsed_time(e1) / args.steps
    # the unfused gsq_step loop, with phase events: the standalone soft-weight
    # kernel once per step
    gsq.gsq_set_timing(lay, True)
    gsq.gsq_phase_times(lay)
    for i in range(args.warmup, args.warmup + args.steps):
        lay.step(float(sched[i]), cfg.lr)
    loop_ms, loop_n = gsq.gsq_phase_times(lay)
    gsq.gsq_set_timing(lay, False)
    # harden + pack (A6) into device buffers
    pb = gsq.gsq_packed_bytes(cfg.grid, cfg.N, cfg.K)
    packed = torch.empty(pb // 4, dtype=torch.int32, device="cuda")
    s16 = torch.empty((cfg.N, cfg.K // 128), dtype=torch.int16, device="cuda")
    s32 = torch.empty((cfg.N, cfg.K // 128), dtype=torch.float32, device="cuda")
    gsq.gsq_harden_pack(lay, packed, s16, s32)
    reps = 5
    e0.record(stream)
    for _ in range(reps):
        gsq.gsq_harden_pack(lay, packed, s16, s32)
    e1.record(stream)
    torch.cuda.synchronize()
    harden_ms = e0.elapsed_time(e1) / reps
    del packed, s16, s32
    lay.close()
    del Wd, Xd
    torch.cuda.empty_cache()

    ms = max_over_ranks(ms, world)
    if split and world > 1:
        # the layer's loss is the sum of the bands' losses (a scalar; the
        # steps themselves exchange nothing)
        import torch.distributed as dist
        lt = torch.tensor([loss], dtype=torch.float64, device="cuda")
        dist.all_reduce(lt, op=dist.ReduceOp.SUM)
        loss = float(lt.item())

    # ---- end to end: host buffers through the C ABI, whole quantization job
    e2e = None if args.no_e2e else run_e2e(gsq, torch, cfg, W, X, rank, row0=row0)
    if e2e is not None and world > 1:
        # every rank ran its own job (or band); the whole job ends with the slowest
        sec = max_over_ranks(e2e["seconds"] * 1e3, world) / 1e3
        e2e["seconds"] = sec
        units = full.N * full.K * cfg.steps if split else world * cfg.N * cfg.K * cfg.steps
        e2e["value"] = whole_job_rate(1, units, sec * 1e3)
        e2e["ranks"] = world

    if rank != 0:
        return None
    hbm, tf_burst, tf_sus, peak_kind = peaks()
    steps_per_s = args.steps / (ms / 1e3)
    coords = cfg.N * cfg.K
    # coordinates all ranks updated per step: the whole layer when it is
    # split, one layer per rank otherwise
    job_coords = (full.N if not args.rows else args.rows) * full.K if split else world * coords
    value = whole_job_rate(1, job_coords * args.steps, ms)
    names = ["soft_weight", "forward_gemm", "weight_grad_gemm", "backward_lion",
             "backward_lion_next_soft"]
    es = 2 if state16 else 4
    work = phase_bytes_flops(cfg, lay, es)
    phases = {}
    # the soft weight alone from the gsq_step loop (one launch per step)
    phase_ms = list(phase_ms)
    phase_n = list(phase_n)
    phase_ms[0], phase_n[0] = loop_ms[0], loop_n[0]
    if phase_n[2] == 0 and phase_n[1] > 0:
        # both GEMMs of a step ran as one launch (layers whose X is at most
        # 64 MB): the forward slot holds them both
        names = list(names)
        names[1] = "gemms_merged"
        work["gemms_merged"] = ("tensor", work["forward_gemm"][1] + work["weight_grad_gemm"][1])
    for i, nm in enumerate(names):
        if phase_n[i] == 0:
            continue
        per = phase_ms[i] / phase_n[i]
        bound, amount = work[nm]
        if bound == "hbm":
            ach = amount / (per / 1e3) / 1e9
            peak, unit = hbm, "GB/s"
        else:
            # each GEMM launch is a ~0.1 ms burst: the burst bf16 rate
            ach = amount / (per / 1e3) / 1e12
            peak, unit = tf_burst, "TFLOP/s"
        phases[nm] = {"ms": round(per, 5), "launches": int(phase_n[i]),
                      "bound": bound, "achieved": round(ach, 1), "unit": unit,
                      "peak": peak, "frac": round(ach / peak, 4), "per_launch": amount}
        if bound == "tensor":
            phases[nm]["frac_of_sustained"] = round(ach / tf_sus, 4)
        if nm == "soft_weight":
            phases[nm]["note"] = ("standalone kernel, timed over a gsq_step loop (gsq_run "
                                  "and gsq_step_next form it inside the fused backward)")
    # harden + pack: logits (+ initial level) read, codes and fp16 / fp32
    # scales written, group scales read
    hb = (coords * (es * lay.L + (1 if cfg.grid == synth.GRID_3BIT_LOCAL else 0))
          + coords * (3 if cfg.grid == synth.GRID_3BIT_LOCAL else 2) // 8
          + (coords // 128) * (4 + 2 + 4))
    phases["harden_pack"] = {"ms": round(harden_ms, 5), "launches": 1, "bound": "hbm",
                             "achieved": round(hb / (harden_ms / 1e3) / 1e9, 1), "unit": "GB/s",
                             "peak": hbm, "frac": round(hb / (harden_ms / 1e3) / 1e9 / hbm, 4),
                             "per_launch": hb,
                             "note": "one gsq_harden_pack call (pack + scale export, syncs)"}
    dom = max(phases, key=lambda n: phases[n]["ms"] * phases[n]["launches"])
    d = phases[dom]
    traffic = load_traffic(dom, cfg.name + ("_bf16_state" if state16 else ""))
    state_mb = 2 * lay.L * coords * es / 1e6
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "steps_per_s": steps_per_s, "higher_is_better": True,
        "scaling": "strong" if split else "weak",
        "vs_baseline": None,
        "dtype": ("bf16 GEMM operands, bf16 logit/momentum state (stochastic rounding)"
                  if state16 else "bf16 GEMM operands, fp32 state"),
        "data": "synthetic (seeded; W ~ N(0,0.02^2) bf16, X ~ N(0,1) bf16 with 1% outlier channels x20)",
        "config": {"workload": cfg.name + ("_bf16_state" if state16 else ""),
                   "N": cfg.N, "K": cfg.K, "T": cfg.T,
                   "grid": ["2bit", "ternary", "3bit_local"][cfg.grid], "group": 128,
                   "parallelism": (f"one layer split by rows over {world} GPUs (global row offset)"
                                   if split else f"independent layer per GPU x{world}"),
                   "l2": f"state (logits + Lion momenta, {state_mb:.0f} MB) larger than L2; no flush"},
        "roofline": {"bound": d["bound"], "kernel": dom, "achieved": d["achieved"],
                     "peak": d["peak"], "unit": d["unit"], "frac": d["frac"],
                     "peak_kind": f"{peak_kind} ({'burst bf16' if d['bound'] == 'tensor' else 'HBM copy'})",
                     "traffic": traffic},
        "phases": phases,
        "step_roofline": step_roofline(work, ms / args.steps, tf_burst, hbm),
        "step_next_loop": {"ms_per_step": round(step_next_ms, 5),
                           "vs_run": round(step_next_ms / (ms / args.steps), 4),
                           "how": "the timed steps again through gsq_step_next calls"},
        "gpu_launches": int(sum(phase_n)),
        "clocks": clk,
        "last_loss": loss,
        "e2e": e2e,
    }
    if not args.no_cpu_baseline and world == 1:
        out["cpu_baseline"] = cpu_baseline(cfg, budget_s=args.cpu_seconds)
    return out


def run_e2e(gsq, torch, cfg, W, X, rank, row0=None):
    """Whole quantization job from pinned host buffers through the C ABI:
    upload + init, the config's steps, loss history read-back, harden+pack
    into host memory (of the rank's band when the layer is split by rows)."""
    Wh = torch.from_numpy(W).to(torch.bfloat16).pin_memory()
    Xh = torch.from_numpy(X).to(torch.bfloat16).pin_memory()
    taus = synth.tau_schedule(cfg.tau0, cfg.tau1, cfg.steps)
    pb = gsq.gsq_packed_bytes(cfg.grid, cfg.N, cfg.K)
    packed = torch.zeros(pb // 4, dtype=torch.int32).pin_memory()
    h16 = torch.zeros((cfg.N, cfg.K // 128), dtype=torch.int16).pin_memory()
    hist = np.zeros(min(cfg.steps, 4096), np.float64)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    lay = gsq.gsq_init(Wh, Xh, 128, cfg.grid, seed=0 if row0 is not None else rank, row0=row0)
    lay.run(taus, cfg.lr)
    gsq._check(gsq.lib().gsq_loss_history(lay.ctx, cfg.steps - hist.size, hist.size,
                                          hist.ctypes.data), "gsq_loss_history")
    gsq.gsq_harden_pack(lay, packed, h16, None)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    lay.close()
    h2d = W.size * 2 + X.size * 2
    d2h = pb + h16.numel() * 2 + hist.nbytes
    return {"value": cfg.N * cfg.K * cfg.steps / dt, "unit": UNIT,
            "h2d_bytes_per_step": h2d / cfg.steps, "d2h_bytes_per_step": d2h / cfg.steps,
            "job": f"init from pinned host + {cfg.steps} steps + harden/pack to host",
            "seconds": dt}


def cpu_baseline(cfg, budget_s=15.0, steps=None):
    """The oracle on the host cores: a row slice of the same layer (the loss
    decomposes over rows), full K and T, steps timed alone (init excluded).
    The slice is sized from one calibration step to fill about budget_s."""
    import oracle
    oracle.build()
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count()))
    W = synth.make_weight(cfg)
    X = synth.make_calib(cfg)
    nsteps = steps or 2
    taus = synth.tau_schedule(cfg.tau0, cfg.tau1, cfg.steps)
    r0 = min(8, cfg.N)
    st = oracle.init(cfg.grid, W[:r0], seed=0)
    Y = oracle.reference_output(W[:r0], X)
    t0 = time.perf_counter()
    oracle.step(st, X, Y, float(taus[0]), cfg.lr)
    per_row = (time.perf_counter() - t0) / r0
    rows = int(max(1, min(cfg.N, budget_s / max(per_row * nsteps, 1e-9))))
    st = oracle.init(cfg.grid, W[:rows], seed=0)
    Y = oracle.reference_output(W[:rows], X)
    t0 = time.perf_counter()
    for i in range(nsteps):
        oracle.step(st, X, Y, float(taus[i]), cfg.lr)
    dt = time.perf_counter() - t0
    return {"value": rows * cfg.K * nsteps / dt, "unit": UNIT, "cores": threads,
            "kind": "oracle",
            "sample": f"{rows} of {cfg.N} rows x K={cfg.K} x T={cfg.T}, {nsteps} steps, {dt:.1f} s"}


def load_traffic(kernel, config):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernels changed since those counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("_kernel_sources_sha256_16") != kernel_sources_hash():
        return None
    return d.get(config, {}).get(kernel)


# the sources that define the single-layer step's kernels and their launch
# configurations (the host orchestration in gsq_api.cu issues them)
STEP_KERNEL_SOURCES = ("gsq_device.cuh", "gsq_gemm.cu", "gsq_gemm_epi.cuh",
                       "gsq_gemm_pair.cu", "gsq_internal.h", "gsq_kernels.cu")


def code_hash(texts) -> str:
    """Hash of C/CUDA sources with comments and blank space removed."""
    import hashlib
    import re
    h = hashlib.sha256()
    for text in texts:
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def kernel_sources_hash():
    """Hash of the step kernels' code (comments and blank space removed), so
    that a comment edit keeps the counters valid and any code change drops
    them."""
    csrc = os.path.join(ROOT, "post_weight_quantization_philox_b200", "csrc")
    return code_hash(open(os.path.join(csrc, f), encoding="utf-8").read()
                     for f in STEP_KERNEL_SOURCES)


def rank_seed(base: int, rank: int) -> int:
    """Data seed of rank's own problem: every rank quantizes an independent
    layer (or stage) of the same shape, so the ranks never exchange data."""
    return base + 7919 * rank


def layer_seeds(cfg, rank):
    """(W seed, X seed, Philox seed) of rank's independent layer."""
    return rank_seed(1000 + cfg.number, rank), rank_seed(2000 + cfg.number, rank), rank


def row_shard(N: int, rank: int, world: int, align: int = 256):
    """(row0, rows) of rank's shard when the rows of one layer are split over
    world ranks: contiguous bands with boundaries on multiples of `align`
    rows (the GEMM tile) where the layer allows, the last band taking the
    remainder.  Rows are independent problems (the loss is a sum over output
    rows and groups lie inside rows), so the bands need no exchange."""
    units = max(1, N // align) if N >= align * world else 0
    if units:
        b = [min(N, (r * units // world) * align) for r in range(world)] + [N]
    else:
        b = [r * N // world for r in range(world)] + [N]
    return b[rank], b[rank + 1] - b[rank]


def max_over_ranks(ms: float, world: int, device="cuda") -> float:
    """The job's time: the slowest rank's device-timed region."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank: float, ms: float) -> float:
    """Units all ranks processed per second of the job's (max-over-ranks) time."""
    return world * units_per_rank / (ms / 1e3)


def run_mlp_stage(args, rank, world, local_rank):
    """The 70B block's MLP stage (gate/up/down quantized jointly on 16384
    tokens): whole-stage steps through gsq_mlp_run."""
    import torch
    from post_weight_quantization_philox_b200 import build
    build.build()
    from post_weight_quantization_philox_b200 import gsq
    torch.cuda.set_device(local_rank)
    cfg = synth.MLP_STAGE["c5_70b_mlp"]
    T, H, F = cfg["T"], cfg["H"], cfg["F"]
    Xn, Wg, Wu, Wd = synth.make_mlp_stage(T, H, F, seed=rank_seed(5005, rank))
    R = synth.random_target(T, H, 0.05, seed=rank_seed(5006, rank))
    dev = lambda x: torch.from_numpy(x).to(torch.bfloat16).cuda()
    m = gsq.gsq_mlp_init(dev(Xn), torch.from_numpy(R).cuda(), dev(Wg), dev(Wu), dev(Wd),
                         grid_mode=cfg["grid"], seed=rank)
    del Xn, Wg, Wu, Wd, R
    taus = synth.tau_schedule(1.0, 0.05, cfg["steps"])
    sched = np.array([taus[i % len(taus)] for i in range(args.warmup + args.steps)], np.float32)
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    m.run(sched[:args.warmup], 1e-3)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    m.run(sched[args.warmup:], 1e-3)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    loss = m.last_loss()
    m.close()
    ms = max_over_ranks(ms, world)
    if rank != 0:
        return None
    hbm, tf_burst, tf_sus, peak_kind = peaks()
    per = ms / args.steps
    coords = 3 * H * F
    flops = 7 * 2.0 * T * H * F
    ach = flops / (per / 1e3) / 1e12
    return {"metric": METRIC, "value": whole_job_rate(world, coords * args.steps, ms), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": per,
            "steps_per_s": 1e3 / per, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 GEMM operands, fp32 state", "data": "synthetic",
            "config": {"workload": "c5_70b_mlp_stage", "T": T, "H": H, "F": F, "grid": "2bit",
                       "weights": "gate, up, down (joint)"},
            "roofline": {"bound": "tensor", "kernel": "whole stage step (7 GEMMs + elementwise)",
                         "achieved": round(ach, 1), "peak": tf_sus, "unit": "TFLOP/s",
                         "frac": round(ach / tf_sus, 4), "peak_kind": f"{peak_kind} (sustained bf16)",
                         "traffic": None},
            "gpu_launches": int(args.steps * 20), "clocks": clk, "last_loss": loss}


def run_attn_stage(args, rank, world, local_rank):
    """The 70B block's attention V/O stage (value and output quantized
    jointly, 64/8 heads x 128, 8 x 2048 tokens) through gsq_attn_run."""
    import torch
    from post_weight_quantization_philox_b200 import build
    build.build()
    from post_weight_quantization_philox_b200 import gsq
    torch.cuda.set_device(local_rank)
    cfg = synth.ATTN_STAGE["c5_70b_attn"]
    dims = dict(nseq=cfg["nseq"], S=cfg["S"], nh=cfg["nh"], nkv=cfg["nkv"], d=cfg["d"])
    Xa, Wq, Wk, Wv, Wo = synth.make_attn_stage(**dims, seed=rank_seed(6006, rank))
    T, H = Xa.shape
    R = synth.random_target(T, H, 0.05, seed=rank_seed(6007, rank))
    dev = lambda x: torch.from_numpy(x).to(torch.bfloat16).cuda()
    a = gsq.gsq_attn_init(dev(Xa), torch.from_numpy(R).cuda(), dev(Wq), dev(Wk), dev(Wv),
                          dev(Wo), dims["nseq"], dims["S"], dims["nh"], dims["nkv"],
                          dims["d"], grid_mode=cfg["grid"], seed=rank)
    del Xa, Wq, Wk, Wv, Wo, R
    taus = synth.tau_schedule(1.0, 0.05, cfg["steps"])
    sched = np.array([taus[i % len(taus)] for i in range(args.warmup + args.steps)], np.float32)
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    a.run(sched[:args.warmup], 1e-3)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    a.run(sched[args.warmup:], 1e-3)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    loss = a.last_loss()
    a.close()
    ms = max_over_ranks(ms, world)
    if rank != 0:
        return None
    hbm, tf_burst, tf_sus, peak_kind = peaks()
    per = ms / args.steps
    S, nh, nkv, d = dims["S"], dims["nh"], dims["nkv"], dims["d"]
    Hk = nkv * d
    coords = Hk * H + H * H
    # useful flops per step: V, P.V, pred, dWo, do, P^T.do, dWv; the two
    # products with the causal P count its nonzero half only
    flops = 2.0 * (2 * T * H * Hk + 3 * T * H * H) + 2 * 2.0 * dims["nseq"] * nh * d * S * (S + 1) / 2
    ach = flops / (per / 1e3) / 1e12
    return {"metric": METRIC, "value": whole_job_rate(world, coords * args.steps, ms), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": per,
            "steps_per_s": 1e3 / per, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 GEMM operands, fp32 state", "data": "synthetic",
            "config": {"workload": "c5_70b_attn_vo_stage", **dims, "grid": "2bit",
                       "weights": "value, output (joint)"},
            "roofline": {"bound": "tensor", "kernel": "whole stage step (GEMMs + elementwise)",
                         "achieved": round(ach, 1), "peak": tf_sus, "unit": "TFLOP/s",
                         "frac": round(ach / tf_sus, 4), "peak_kind": f"{peak_kind} (sustained bf16)",
                         "traffic": None},
            "gpu_launches": int(args.steps * 17 + 2), "clocks": clk,
            "last_loss": loss}


def run_scale_stage(args, rank, world, local_rank):
    """Scale-only steps (assignments frozen at the hard choice, group scales
    trained) on the --config layer, after a short GSQ warm start."""
    import torch
    from post_weight_quantization_philox_b200 import build
    build.build()
    from post_weight_quantization_philox_b200 import gsq
    torch.cuda.set_device(local_rank)
    cfg = synth.CONFIGS[args.config]
    w_seed, x_seed, _ = layer_seeds(cfg, rank)
    W = synth.make_weight(cfg, seed=w_seed)
    X = synth.make_calib(cfg, seed=x_seed)
    lay = gsq.gsq_init(torch.from_numpy(W).to(torch.bfloat16).cuda(),
                       torch.from_numpy(X).to(torch.bfloat16).cuda(), 128, cfg.grid, seed=rank)
    lay.run(synth.tau_schedule(cfg.tau0, cfg.tau1, 20), cfg.lr)  # assignments to freeze
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    lay.scale_run(args.warmup, cfg.lr)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    lay.scale_run(args.steps, cfg.lr)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    loss = lay.last_loss()
    lay.close()
    ms = max_over_ranks(ms, world)
    if rank != 0:
        return None
    hbm, tf_burst, tf_sus, peak_kind = peaks()
    per = ms / args.steps
    flops = 4.0 * cfg.N * cfg.T * cfg.K  # forward + weight-gradient GEMMs
    ach = flops / (per / 1e3) / 1e12
    coords = cfg.N * cfg.K
    return {"metric": METRIC, "value": whole_job_rate(world, coords * args.steps, ms), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": per,
            "steps_per_s": 1e3 / per, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 GEMM operands, fp32 state", "data": "synthetic",
            "config": {"workload": cfg.name + "_scale_only", "N": cfg.N, "K": cfg.K,
                       "T": cfg.T, "grid": ["2bit", "ternary", "3bit_local"][cfg.grid],
                       "step": "scale-only (hard codes frozen)"},
            "roofline": {"bound": "tensor", "kernel": "whole scale-only step (2 GEMMs + 8 B/coord)",
                         "achieved": round(ach, 1), "peak": tf_sus, "unit": "TFLOP/s",
                         "frac": round(ach / tf_sus, 4),
                         "peak_kind": f"{peak_kind} (sustained bf16)", "traffic": None},
            "gpu_launches": int(args.steps * 4), "clocks": clk, "last_loss": loss}


# Llama-3.1-70B block on 8 sequences x 2048 tokens
BLOCK_70B = dict(nseq=8, S=2048, nh=64, nkv=8, d=128, F=28672)


def block_step_flops(nseq, S, nh, nkv, d, F):
    """GEMM flops of one step of each stage (Q, K, V/O, MLP) of the block."""
    T, H, Hk = nseq * S, nh * d, nkv * d
    q = 4.0 * T * H * H
    k = 4.0 * T * H * Hk
    vo = 2.0 * (2 * T * H * Hk + 3 * T * H * H) + 2 * 2.0 * nseq * nh * d * S * (S + 1) / 2
    mlp = 7 * 2.0 * T * H * F
    return [q, k, vo, mlp]


def run_block_pipeline(args, rank, world, local_rank):
    """GSQ's staged reconstruction of one 70B-shaped block (Q, K, V/O, MLP on
    the block output, then the quantized output for the next block) through
    gsq_block_quantize, --steps steps per stage; the timed region is the
    whole call (full-precision forward, four stage contexts, hardening,
    propagation)."""
    import torch
    from post_weight_quantization_philox_b200 import build
    build.build()
    from post_weight_quantization_philox_b200 import gsq
    torch.cuda.set_device(local_rank)
    dm = BLOCK_70B
    T, H, Hk, F = dm["nseq"] * dm["S"], dm["nh"] * dm["d"], dm["nkv"] * dm["d"], dm["F"]
    # seeded synthetic block: x ~ N(0, 1) residual stream, weights N(0, 0.02^2)
    gen = torch.Generator(device="cuda").manual_seed(rank_seed(7007, rank))
    x = torch.randn((T, H), generator=gen, device="cuda")
    shapes = gsq.block_weight_shapes(dm["nh"], dm["nkv"], dm["d"], F)
    W = {n: (torch.randn(shp, generator=gen, device="cuda") * 0.02).to(torch.bfloat16)
         for n, shp in shapes.items()}
    dims = (dm["nseq"], dm["S"], dm["nh"], dm["nkv"], dm["d"], F)
    warm = [synth.tau_schedule(1.0, 0.05, args.warmup)] * 4
    gsq.gsq_block_quantize(x, W, *dims, warm, 1e-3, seed=rank)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    taus = [synth.tau_schedule(1.0, 0.05, args.steps)] * 4
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    r = gsq.gsq_block_quantize(x, W, *dims, taus, 1e-3, seed=rank)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    ms = max_over_ranks(ms, world)
    if rank != 0:
        return None
    hbm, tf_burst, tf_sus, peak_kind = peaks()
    coords = sum(a * b for a, b in shapes.values())
    flops = block_step_flops(*dims)
    stage_ms = [r["stats"][s]["ms"] for s in gsq.BLOCK_STAGES]
    steps_ms = sum(stage_ms)
    ach = sum(flops) * args.steps / (ms / 1e3) / 1e12
    per_stage = {s: {"ms_per_step": m / args.steps,
                     "tflops": round(f * args.steps / (m / 1e3) / 1e12, 1) if m > 0 else None}
                 for s, m, f in zip(gsq.BLOCK_STAGES, stage_ms, flops)}
    return {"metric": METRIC, "value": whole_job_rate(world, coords * args.steps, ms), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps, "steps_per_s": 1e3 * args.steps / ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 GEMM operands, fp32 state and residual stream", "data":
            "synthetic (seeded torch generator: x ~ N(0,1), weights ~ N(0,0.02^2) bf16)",
            "config": {"workload": "c5_70b_block_pipeline", **dm, "grid": "2bit",
                       "steps_per_stage": args.steps,
                       "step": "one step of every stage; timed: the whole block call"},
            "roofline": {"bound": "tensor", "kernel": "whole block call (stage GEMM flops)",
                         "achieved": round(ach, 1), "peak": tf_sus, "unit": "TFLOP/s",
                         "frac": round(ach / tf_sus, 4),
                         "peak_kind": f"{peak_kind} (sustained bf16)", "traffic": None},
            "stages": per_stage, "stage_steps_share": round(steps_ms / ms, 4),
            "stage_stats": {s: {k: v for k, v in r["stats"][s].items() if k != "ms"}
                            for s in gsq.BLOCK_STAGES},
            "clocks": clk}


C5_WORKLOAD = "c5_70b_block_step"
C5_Q_LAYER = "c5_70b_qproj_8192x8192"


def block_step_coords(nseq, S, nh, nkv, d, F):
    """Grid coordinates of the block's seven weights: Q, K (layers), V, O
    (joint), gate, up, down (joint)."""
    H, Hk = nh * d, nkv * d
    return [H * H, Hk * H, Hk * H + H * H, 3 * H * F]


def block_backward_bytes(coords, L=4, es=4, next_soft=True):
    """Algorithmic bytes of the fused backward over `coords` coordinates (2-bit
    grid): dW read, L logit and L momentum planes read and written, 16 B per
    group of 128, plus the next bf16 soft weight."""
    return coords * (4 + 4 * es * L + (2 if next_soft else 0)) + coords // 128 * 16


def run_block_step(args, rank, world, local_rank):
    """The Llama-3.1-70B-shaped block (hidden 8192, 64 / 8 heads of 128, SwiGLU
    28672, 8 x 2048 tokens, 2-bit grid), one GSQ step of every stage per
    bench step: the Q and K layers (8192 x 8192 and 1024 x 8192 on the
    normalised attention input), the V/O joint stage (probabilities from the
    frozen query / key weights), the MLP joint stage (gate, up, down).  The
    timed region runs each stage's K steps through its run call, in the
    method's stage order.  Inputs are seeded on the device (torch generator):
    stage inputs normalised to unit RMS per token as after a unit-gain
    RMSNorm, weights N(0, 0.02^2) bf16, and for the joint stages N(0, 0.05^2)
    stand-ins of their targets (the step's work does not depend on the
    target's values).  The end-to-end leg is the whole job: gsq_block_quantize
    from pinned host buffers (full-precision forward, the four stages' inits
    and steps, hardening, the quantized output), outputs back in pinned host
    memory."""
    import torch
    from post_weight_quantization_philox_b200 import build
    build.build()
    from post_weight_quantization_philox_b200 import gsq
    torch.cuda.set_device(local_rank)
    dm = BLOCK_70B
    nseq, S, nh, nkv, d, F = (dm[k] for k in ("nseq", "S", "nh", "nkv", "d", "F"))
    T, H, Hk = nseq * S, nh * d, nkv * d
    gen = torch.Generator(device="cuda").manual_seed(rank_seed(8008, rank))

    def randn(shape, std):
        return torch.randn(shape, generator=gen, device="cuda") * std

    def normalised(shape):
        x = randn(shape, 1.0)
        return (x / x.pow(2).mean(1, keepdim=True).sqrt()).to(torch.bfloat16)

    xa, xm = normalised((T, H)), normalised((T, H))
    shapes = gsq.block_weight_shapes(nh, nkv, d, F)
    W = {n: randn(shp, 0.02).to(torch.bfloat16) for n, shp in shapes.items()}
    Ra, Rm = randn((T, H), 0.05), randn((T, H), 0.05)
    seed = rank
    q = gsq.gsq_init(W["q"], xa, 128, synth.GRID_2BIT, seed=seed)
    k = gsq.gsq_init(W["k"], xa, 128, synth.GRID_2BIT, seed=seed + 1)
    a = gsq.gsq_attn_init(xa, Ra, W["q"], W["k"], W["v"], W["o"], nseq, S, nh, nkv, d,
                          grid_mode=synth.GRID_2BIT, seed=seed + 2)
    m = gsq.gsq_mlp_init(xm, Rm, W["gate"], W["up"], W["down"], grid_mode=synth.GRID_2BIT,
                         seed=seed + 3)
    del Ra, Rm
    stages = [("q", q), ("k", k), ("vo", a), ("mlp", m)]
    lr = 1e-3
    taus = synth.tau_schedule(1.0, 0.05, 200)
    sched = np.array([taus[i % len(taus)] for i in range(args.warmup + args.steps)], np.float32)
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    for _, st in stages:
        st.run(sched[:args.warmup], lr)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    # the timed region: every stage's steps, the library's launches only
    e0.record(stream)
    for _, st in stages:
        st.run(sched[args.warmup:], lr)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    losses = {n: st.last_loss() for n, st in stages}
    # per-phase device time from a second, instrumented run of the same steps
    ph = {}
    for n, st in (("q", q), ("k", k)):
        gsq.gsq_set_timing(st, True)
        gsq.gsq_phase_times(st)
        st.run(sched[args.warmup:], lr)
        pm, pn = gsq.gsq_phase_times(st)
        gsq.gsq_set_timing(st, False)
        # soft weight, GEMMs (forward + weight gradient), backward (both kinds)
        ph[n] = (np.array([pm[0], pm[1] + pm[2], 0.0, pm[3] + pm[4]]),
                 np.array([pn[0], pn[1] + pn[2], 0, pn[3] + pn[4]]))
    for n, st in (("vo", a), ("mlp", m)):
        st.set_timing(True)
        st.phase_times()
        st.run(sched[args.warmup:], lr)
        ph[n] = st.phase_times()
        st.set_timing(False)
    for _, st in stages:
        st.close()
    del q, k, a, m, stages, xa, xm
    torch.cuda.empty_cache()
    ms = max_over_ranks(ms, world)

    # ---- end to end: the whole block job from pinned host buffers
    e2e = None
    if not args.no_e2e:
        e2e = block_e2e(gsq, torch, W, gen, dm, args.e2e_steps, rank)
        if world > 1:
            sec = max_over_ranks(e2e["seconds"] * 1e3, world) / 1e3
            e2e["seconds"] = sec
            e2e["value"] = whole_job_rate(world, e2e["coords_per_job"], sec * 1e3)
            e2e["ranks"] = world
    del W
    if rank != 0:
        return None
    hbm, tf_burst, tf_sus, peak_kind = peaks()
    K_ = args.steps
    coords = block_step_coords(nseq, S, nh, nkv, d, F)
    flops = block_step_flops(nseq, S, nh, nkv, d, F)
    names = ["q", "k", "vo", "mlp"]
    stage_out = {}
    gemm_ms = gemm_flops = bwd_ms = bwd_bytes = elem_ms = soft_ms = 0.0
    launches = 0
    for n, c, f in zip(names, coords, flops):
        pm, pn = ph[n]
        launches += int(pn.sum())
        # backward launches of a run: all but the last step also form the
        # next soft weight
        bb = (K_ - 1) * block_backward_bytes(c) + block_backward_bytes(c, next_soft=False)
        stage_out[n] = {
            "coords": c, "ms_per_step": round(float(pm.sum()) / K_, 4),
            "gemm": {"ms_per_step": round(pm[1] / K_, 4),
                     "tflops": round(f * K_ / (pm[1] / 1e3) / 1e12, 1) if pm[1] else None},
            "backward": {"ms_per_step": round(pm[3] / K_, 4),
                         "gbs": round(bb / (pm[3] / 1e3) / 1e9, 1) if pm[3] else None},
            "elementwise_ms_per_step": round(pm[2] / K_, 4),
            "soft_weight_ms_per_run": round(pm[0], 4),
            "last_loss": losses[n]}
        gemm_ms += pm[1]
        gemm_flops += f * K_
        bwd_ms += pm[3]
        bwd_bytes += bb
        elem_ms += pm[2]
        soft_ms += pm[0]
    gemm_ach = gemm_flops / (gemm_ms / 1e3) / 1e12
    bwd_ach = bwd_bytes / (bwd_ms / 1e3) / 1e9
    phases = {
        "gemm": {"ms": round(gemm_ms / K_, 4), "bound": "tensor", "achieved": round(gemm_ach, 1),
                 "unit": "TFLOP/s", "peak": tf_burst, "frac": round(gemm_ach / tf_burst, 4),
                 "frac_of_sustained": round(gemm_ach / tf_sus, 4)},
        "backward_lion": {"ms": round(bwd_ms / K_, 4), "bound": "hbm",
                          "achieved": round(bwd_ach, 1), "unit": "GB/s", "peak": hbm,
                          "frac": round(bwd_ach / hbm, 4)},
        "elementwise": {"ms": round(elem_ms / K_, 4)},
        "soft_weight": {"ms_per_run": round(soft_ms, 4)},
    }
    dom = "gemm" if gemm_ms >= bwd_ms else "backward_lion"
    dd = phases[dom]
    per = ms / K_
    gemm_floor = sum(flops) / (tf_burst * 1e12) * 1e3
    hbm_floor = sum(block_backward_bytes(c) for c in coords) / (hbm * 1e9) * 1e3
    out = {
        "metric": METRIC, "value": whole_job_rate(world, sum(coords) * K_, ms), "unit": UNIT,
        "n_gpus": world, "steps": K_, "warmup": args.warmup, "ms_per_step": per,
        "steps_per_s": 1e3 / per, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 GEMM operands, fp32 state",
        "data": ("synthetic (seeded torch generator on the device: unit-RMS stage inputs, "
                 "weights N(0,0.02^2) bf16, joint-stage targets N(0,0.05^2) stand-ins)"),
        "config": {"workload": C5_WORKLOAD, **dm, "T": T, "grid": "2bit", "group": 128,
                   "weights": "q, k (layers); v, o (joint); gate, up, down (joint)",
                   "step": "one GSQ step of every stage (Q, K, V/O, MLP), stage order",
                   "parallelism": f"independent block per GPU x{world}",
                   "l2": "every stage's state and activations far larger than L2; no flush"},
        "roofline": {"bound": dd["bound"], "kernel": ("k_gemm_pair (all GEMMs of the step)"
                                                      if dom == "gemm" else
                                                      "k_backward_lion (all weights)"),
                     "achieved": dd["achieved"], "peak": dd["peak"], "unit": dd["unit"],
                     "frac": dd["frac"],
                     "peak_kind": f"{peak_kind} ({'burst bf16' if dom == 'gemm' else 'HBM copy'})",
                     # the GEMMs run for tens of ms under the power cap: the
                     # sustained bf16 rate is the other fair denominator
                     **({"frac_of_sustained": dd["frac_of_sustained"]} if dom == "gemm" else {}),
                     "traffic": None},
        "phases": phases, "stages": stage_out,
        "step_roofline": {"gemm_ms": round(gemm_floor, 3), "hbm_ms": round(hbm_floor, 3),
                          "ms": round(gemm_floor + hbm_floor, 3),
                          "frac": round((gemm_floor + hbm_floor) / per, 4),
                          "how": "all GEMM flops at the burst bf16 rate + the fused backwards' "
                                 "algorithmic bytes at the copy rate, over the measured step"},
        "gpu_launches": launches, "clocks": clk, "e2e": e2e,
    }
    if not args.no_cpu_baseline and world == 1:
        cb = cpu_baseline(synth.CONFIGS[C5_Q_LAYER], budget_s=args.cpu_seconds, steps=1)
        cb["sample"] += " (the block's query projection, one step)"
        out["cpu_baseline"] = cb
    return out


def block_e2e(gsq, torch, W, gen, dm, steps, rank):
    """One gsq_block_quantize call (the whole block job, `steps` steps per
    stage) from pinned host buffers, outputs into pinned host memory."""
    nseq, S, nh, nkv, d, F = (dm[k] for k in ("nseq", "S", "nh", "nkv", "d", "F"))
    T, H = nseq * S, nh * d
    x = torch.randn((T, H), generator=gen, device="cuda").cpu().pin_memory()
    Wh = {n: w.cpu().pin_memory() for n, w in W.items()}
    taus = [synth.tau_schedule(1.0, 0.05, steps)] * 4
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    r = gsq.gsq_block_quantize(x, Wh, nseq, S, nh, nkv, d, F, taus, 1e-3, seed=rank,
                               host_outputs=True)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    coords = sum(a * b for a, b in gsq.block_weight_shapes(nh, nkv, d, F).values())
    h2d = x.numel() * 4 + sum(w.numel() * 2 for w in Wh.values())
    d2h = (r["x_out"].numel() * 4 + sum(p.numel() * 4 for p in r["packed"].values())
           + sum(s.numel() * 4 for s in r["scales"].values()))
    return {"value": coords * steps / dt, "unit": UNIT, "seconds": dt,
            "coords_per_job": coords * steps,
            "h2d_bytes_per_step": h2d / steps, "d2h_bytes_per_step": d2h / steps,
            "job": (f"gsq_block_quantize from pinned host buffers: full-precision forward, "
                    f"Q, K, V/O, MLP stages x {steps} steps, hardening, quantized output, "
                    f"outputs to pinned host memory")}


def gptq_flops(N: int, K: int) -> float:
    """fp32 flops of one GPTQ call (algorithmic): Cholesky of the damped K x K
    Hessian (K^3 / 3), inverse of its triangular factor (K^3 / 3), the
    trailing-column error updates (N K^2 in total) and the in-group feedback
    (N K 128)."""
    return 2.0 * K ** 3 / 3.0 + float(N) * K * K + float(N) * K * 128


def run_gptq_stage(args, rank, world, local_rank):
    """GPTQ initial assignment (Hessian, Cholesky, inverse, column-wise error
    feedback) of the --config layer, device inputs and outputs."""
    import torch
    from post_weight_quantization_philox_b200 import build
    build.build()
    from post_weight_quantization_philox_b200 import gsq
    torch.cuda.set_device(local_rank)
    cfg = synth.CONFIGS[args.config]
    w_seed, x_seed, _ = layer_seeds(cfg, rank)
    W = torch.from_numpy(synth.make_weight(cfg, seed=w_seed))
    X = torch.from_numpy(synth.make_calib(cfg, seed=x_seed))
    dt = torch.bfloat16 if cfg.w_bf16 else torch.float32
    W, X = W.to(dt).cuda(), X.to(dt).cuda()
    lev = torch.empty((cfg.N, cfg.K), dtype=torch.int8, device="cuda")
    sc = torch.empty((cfg.N, cfg.K // 128), dtype=torch.float32, device="cuda")
    for _ in range(args.warmup):
        gsq.gsq_gptq(W, X, 128, cfg.grid, levels=lev, scales=sc)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    clocks = ClockSampler(local_rank)
    clocks.start()
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        gsq.gsq_gptq(W, X, 128, cfg.grid, levels=lev, scales=sc)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    ms = max_over_ranks(ms, world)
    if rank != 0:
        return None
    per = ms / args.steps
    props = torch.cuda.get_device_properties(local_rank)
    sm_mhz = clk.get("sm_mhz") or 1965.0
    # fp32 FMA peak: 128 lanes per SM, 2 flops per FMA, at the sampled clock
    alu_peak = props.multi_processor_count * 128 * 2 * sm_mhz * 1e6 / 1e12
    # the trailing updates run on the tensor cores, each fp32 product formed
    # from six bf16 products (three-term split): that path's peak is the
    # measured burst bf16 rate / 6
    hbm, tf_burst, tf_sus, peak_kind = peaks()
    split_peak = tf_burst / 6.0
    flops = gptq_flops(cfg.N, cfg.K)
    ach = flops / (per / 1e3) / 1e12
    coords = cfg.N * cfg.K
    return {"metric": METRIC, "value": whole_job_rate(world, coords, per), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": per,
            "steps_per_s": 1e3 / per, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp32 (Hessian: bf16 operands, fp32 accumulate)",
            "data": "synthetic",
            "config": {"workload": cfg.name + "_gptq_init", "N": cfg.N, "K": cfg.K,
                       "T": cfg.T, "grid": ["2bit", "ternary", "3bit_local"][cfg.grid],
                       "step": "one GPTQ call (workspace allocated and freed inside)"},
            "roofline": {"bound": "tensor",
                         "kernel": "whole GPTQ call (fp32 flops of Cholesky, inverse and "
                                   "column updates)",
                         "achieved": round(ach, 2), "peak": round(split_peak, 1),
                         "unit": "TFLOP/s", "frac": round(ach / split_peak, 4),
                         "peak_kind": f"{peak_kind} burst bf16 / 6 (fp32 products from six "
                                      "bf16 products)",
                         "frac_of_fp32_simt": round(ach / alu_peak, 4),
                         "fp32_simt_peak": round(alu_peak, 1),
                         "traffic": None},
            "clocks": clk}


# one lr for the logits and the sub-block scales/mins: small enough that the
# noisy early steps leave the 16-weight sub-blocks' parameters near the start
KQ_LR = 1e-5


def run_kquant_stage(args, rank, world, local_rank):
    """GSQ on a GGUF K-Quant format (--kq-format q2k | q3k) on the --config
    layer: whole steps through gsq_kq_run from the min-max K-Quant start."""
    import torch
    from post_weight_quantization_philox_b200 import build
    build.build()
    from post_weight_quantization_philox_b200 import gsq
    torch.cuda.set_device(local_rank)
    cfg = synth.CONFIGS[args.config]
    fmt = gsq.GSQ_KQ_Q2_K if args.kq_format == "q2k" else gsq.GSQ_KQ_Q3_K
    w_seed, x_seed, _ = layer_seeds(cfg, rank)
    W = synth.make_weight(cfg, seed=w_seed)
    X = synth.make_calib(cfg, seed=x_seed)
    lay = gsq.gsq_kq_init(torch.from_numpy(W).to(torch.bfloat16).cuda(),
                          torch.from_numpy(X).to(torch.bfloat16).cuda(), fmt, seed=rank)
    e_start = lay.recon_error(1)[1]
    taus = synth.tau_schedule(cfg.tau0, cfg.tau1, cfg.steps)
    sched = np.array([taus[i % len(taus)] for i in range(args.warmup + args.steps)], np.float32)
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    lay.run(sched[:args.warmup], KQ_LR)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    lay.run(sched[args.warmup:], KQ_LR)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    loss = lay.last_loss()
    e_end = lay.recon_error(0)[1]
    lay.close()
    ms = max_over_ranks(ms, world)
    if rank != 0:
        return None
    hbm, tf_burst, tf_sus, peak_kind = peaks()
    per = ms / args.steps
    flops = 4.0 * cfg.N * cfg.T * cfg.K
    ach = flops / (per / 1e3) / 1e12
    coords = cfg.N * cfg.K
    # the step at the peaks: both GEMMs at the tensor rate plus the fused
    # backward's bytes at the copy rate (read dW 4, q0 1, logits and momenta
    # 8 L; write logits and momenta 8 L, the bf16 soft weight 2; sub-block
    # parameters and momenta 2 (Q2_K) or 1 B; the probabilities are drawn
    # again, not stored)
    q2 = args.kq_format == "q2k"
    L = 4 if q2 else 5
    bwd_bytes = coords * (7 + 16 * L + (2 if q2 else 1))
    gemm_ms = flops / (tf_sus * 1e12) * 1e3
    hbm_ms = bwd_bytes / (hbm * 1e9) * 1e3
    return {"metric": METRIC, "value": whole_job_rate(world, coords * args.steps, ms), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": per,
            "steps_per_s": 1e3 / per, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 GEMM operands, fp32 state", "data": "synthetic",
            "config": {"workload": cfg.name + "_" + args.kq_format, "N": cfg.N, "K": cfg.K,
                       "T": cfg.T, "format": args.kq_format.upper().replace("K", "_K"),
                       "step": "2 GEMMs, backward + Lion (16-weight sub-blocks) + next soft weight"},
            "roofline": {"bound": "tensor", "kernel": "whole step (2 GEMMs + elementwise)",
                         "achieved": round(ach, 1), "peak": tf_sus, "unit": "TFLOP/s",
                         "frac": round(ach / tf_sus, 4),
                         "peak_kind": f"{peak_kind} (sustained bf16)", "traffic": None},
            "step_roofline": {"gemm_ms": round(gemm_ms, 4), "hbm_ms": round(hbm_ms, 4),
                              "ms": round(gemm_ms + hbm_ms, 4),
                              "frac": round((gemm_ms + hbm_ms) / per, 4),
                              "how": "GEMM flops at the sustained bf16 rate + the backward's "
                                     "bytes at the copy rate, over the measured step"},
            "gpu_launches": int(args.steps * 3 + 1), "clocks": clk, "last_loss": loss,
            "recon_rel": {"start": e_start, "after": e_end}}


def run_reference(args, rank, world, block_default=False):
    """The oracle as the reference arm (rank 0 only), on the same workload
    as the GPU arm: for the 70B block step, rows of the block's query
    projection (every weight of the block costs the same two T-long
    contractions per coordinate, and the oracle's stage steps are the layer
    step's arithmetic)."""
    if rank != 0:
        return None
    cfg = synth.CONFIGS[args.config]
    per = []
    for _ in range(args.warmup):
        pass  # the oracle has no warm state to build
    cb = None
    for _ in range(args.steps):
        cb = cpu_baseline(cfg, budget_s=args.cpu_seconds / max(args.steps, 1), steps=1)
        per.append(cb["value"])
    v = statistics.median(per)
    return {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
            "impl": "reference",
            "config": ({"workload": C5_WORKLOAD, **BLOCK_70B, "T": cfg.T, "grid": "2bit",
                        "group": 128} if block_default else
                       {"workload": cfg.name, "N": cfg.N, "K": cfg.K, "T": cfg.T,
                        "grid": ["2bit", "ternary", "3bit_local"][cfg.grid], "group": 128}),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cb["cores"],
                             "kind": "oracle", "sample": cb["sample"]},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=None, choices=sorted(synth.CONFIGS),
                    help="time one layer of this shape (default: the 70B block step)")
    ap.add_argument("--impl", default="gsq", choices=["gsq", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--stage", default=None, choices=["mlp", "attn", "scale", "gptq", "block", "kquant"],
                    help="time a block stage instead of a single layer")
    ap.add_argument("--kq-format", default="q2k", choices=["q2k", "q3k"],
                    help="K-Quant format of --stage kquant")
    ap.add_argument("--state", default="fp32", choices=["fp32", "bf16"],
                    help="logit / momentum storage of the single-layer step")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end job (profiling runs)")
    ap.add_argument("--rows", type=int, default=0,
                    help="single layer: only its first ROWS rows (a multiple of 256)")
    ap.add_argument("--split", default="layers", choices=["layers", "rows"],
                    help="N > 1: one independent layer per GPU (weak scaling), or one "
                         "layer's rows split over the GPUs (strong scaling)")
    ap.add_argument("--e2e-steps", type=int, default=200,
                    help="block step: steps per stage of the end-to-end block job")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    block_default = args.config is None and args.stage is None
    if args.config is None:
        args.config = C5_Q_LAYER if block_default else "c2_qproj_4096x4096"

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        out = run_reference(args, rank, world, block_default)
        if out:
            print(json.dumps(out))
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    if args.stage == "mlp":
        out = run_mlp_stage(args, rank, world, local_rank)
    elif args.stage == "attn":
        out = run_attn_stage(args, rank, world, local_rank)
    elif args.stage == "scale":
        out = run_scale_stage(args, rank, world, local_rank)
    elif args.stage == "gptq":
        out = run_gptq_stage(args, rank, world, local_rank)
    elif args.stage == "block":
        out = run_block_pipeline(args, rank, world, local_rank)
    elif args.stage == "kquant":
        out = run_kquant_stage(args, rank, world, local_rank)
    elif block_default:
        out = run_block_step(args, rank, world, local_rank)
    else:
        out = run_gsq(args, rank, world, local_rank)
    if out:
        print(json.dumps(out))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
