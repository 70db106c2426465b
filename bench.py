"""Benchmark of one CD-RGE update (all probe losses, coefficients, update) on
B200 through the C ABI.  Prints one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is zo_probe_losses + zo_coeffs + zo_update over one synthetic batch of
the named workload (default "lstm1b", the ~1.1B-parameter 2-layer LSTM on
batch 1024 x sequence 10 with 16 probes, the largest configuration that the
pages' character-level language-modelling runs use and that fits one GPU;
also tiny, overfit, charlm, lstm270m, lstm4b).  `value` is CD-RGE steps/s of the whole
job (device time, inputs resident in HBM, L2 flushed before every step and
the flush not timed).  `e2e` is the same metric with the step's
tokens/targets copied from pinned host memory and L+/L- read back every step
(zo_step_host on one GPU).  With N > 1 (torchrun) the n_pert probes of each
step are split over the ranks (probe_parallel: each rank evaluates its probe
slice, the 2 n_pert scalar losses are all-gathered over NCCL, every rank
applies the same update): strong scaling, time = max over ranks.
`--impl reference` times the C++ fp64 CPU oracle instead (rank 0 only) on
bounded samples of the step, extrapolated (the line says so).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "CD-RGE steps/s and perturbed-forward tokens/s on 1 B200; % of roofline"
CELL_VARIANTS = {"single": 0, "single-exact-eps": 1, "pair": 2, "pair-exact-eps": 3,
                 "pair-direct-w": 4, "single-epi8": 5}
L2_BYTES = 126 * 1024 * 1024
CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "sm_max_mhz": d.get("sm_max_mhz", 1965.0), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sm_max_mhz": 1965.0, "source": "fallback"}


def fp32_alu_peak_tflops(sm_mhz):
    """fp32 CUDA-core peak: 148 SMs x 128 FP32 lanes x 2 flops (FMA) x clock."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def forward_macs_per_token(cfg):
    m = cfg.vocab * cfg.hidden
    for l in range(cfg.layers):
        m += 4 * cfg.hidden * ((cfg.embed if l == 0 else cfg.hidden) + cfg.hidden)
    return m


def batches(cfg, n, rank):
    """n (tokens, targets) batches for rank `rank`: fresh Markov batches per
    step for the LM workloads, the fixed batch for copy / overfit."""
    if cfg.task in ("copy", "overfit"):
        b = W.batch_for(cfg)
        return [b] * n
    return [W.markov_batch(cfg.batch, cfg.seq, step=1000 * rank + k, vocab=cfg.vocab) for k in range(n)]


class ClockSampler:
    """nvidia-smi samples (every 50 ms) with host timestamps; `summary` keeps
    the samples that fall inside a wall-clock window."""

    def __init__(self, gpu_index):
        import tempfile
        self.proc = None
        self.path = os.path.join(tempfile.mkdtemp(prefix="zo_clocks_"), "clocks.csv")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu=timestamp,{CLOCK_QUERY}",
                 "--format=csv,noheader", "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
            t0 = time.time()   # nvidia-smi takes a moment before its first line
            while time.time() - t0 < 3.0 and os.path.getsize(self.path) == 0:
                time.sleep(0.05)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()

    def summary(self, t0, t1):
        if self.proc is None:
            return None
        import datetime
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                sm, mx = float(f[2].split()[0]), float(f[3].split()[0])
            except ValueError:
                continue
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            rs = {nm for nm, v in zip(names, f[6:10]) if v.lower().startswith("active")}
            rows.append((ts, sm, mx, rs))
        if not rows:
            return None
        inside = [r for r in rows if t0 <= r[0] <= t1]
        if not inside:   # window shorter than the sampling period: nearest sample
            inside = [min(rows, key=lambda r: abs(r[0] - 0.5 * (t0 + t1)))]
        reasons = set().union(*[r[3] for r in inside])
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": sorted(reasons),
                "samples": len(inside)}


def run_ours(args, cfg):
    import torch
    import torch.distributed as dist

    import zero_order_recurrent_b200 as zo

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    zo.load_library()
    dev = torch.device("cuda", local)
    n, eps, eta = cfg.n_pert, cfg.eps, cfg.eta
    theta_h = W.init_theta(cfg)
    theta = torch.from_numpy(theta_h).to(dev)
    del theta_h
    K, Wm = args.steps, args.warmup
    bl = batches(cfg, Wm + K, 0)
    toks = [torch.from_numpy(t).to(dev) for t, _ in bl]
    tgts = [torch.from_numpy(g).to(dev) for _, g in bl]
    lp = torch.empty(n, device=dev)
    lm = torch.empty(n, device=dev)
    coef = torch.empty(n, device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    ctx = zo.Context.for_config(cfg)
    if args.cell_variant != "single":
        zo.zo_debug_cell_variant(ctx, CELL_VARIANTS[args.cell_variant])
    st = torch.cuda.current_stream()

    def step(k):
        if world > 1:
            from zero_order_recurrent_b200.probe_parallel import cdrge_step_sharded
            cdrge_step_sharded(ctx, theta, W.step_seed(k), n, eps, eta, toks[k], tgts[k], coef)
        else:
            zo.cdrge_step(ctx, theta, W.step_seed(k), n, eps, eta, toks[k], tgts[k], lp, lm, coef)

    sampler = ClockSampler(local)
    for k in range(Wm):
        step(k)
    torch.cuda.synchronize()
    s = zo.zo_sync_status(ctx)
    if s != zo.ZO_OK:
        raise RuntimeError(f"warm-up failed: {zo.status_string(s)}")
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = zo.zo_kernel_launches()
    t_start = time.time()
    zo.zo_profile(ctx, True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for k in range(K):
        flush.fill_(float(k))                      # L2 flush, outside the timed window
        ev[k][0].record(st)
        step(Wm + k)
        ev[k][1].record(st)
    torch.cuda.synchronize()
    t_end = time.time()
    zo.zo_profile(ctx, False)
    launches = zo.zo_kernel_launches() - launches0
    sampler.stop()
    clocks = sampler.summary(t_start, t_end)
    s = zo.zo_sync_status(ctx)
    if s != zo.ZO_OK:
        raise RuntimeError(f"timed steps failed: {zo.status_string(s)}")
    ms = sum(a.elapsed_time(b) for a, b in ev)
    kinds = {name: zo.zo_profile_read(ctx, kind) for name, kind in
             (("cell", zo.ZO_KIND_CELL), ("loss", zo.ZO_KIND_LOSS), ("update", zo.ZO_KIND_UPDATE),
              ("other", zo.ZO_KIND_OTHER))}
    if world > 1:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())

    # end-to-end through zo_step_host: pinned host inputs in, losses out
    e2e = None
    if not args.no_e2e:
        ht = [torch.from_numpy(t).pin_memory() for t, _ in bl]
        hg = [torch.from_numpy(g).pin_memory() for _, g in bl]
        hp = torch.empty(n, dtype=torch.float32).pin_memory()
        hm = torch.empty(n, dtype=torch.float32).pin_memory()
        Ke = max(1, min(K, 5))
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for k in range(Ke):
            seed = W.step_seed(Wm + K + k)
            if world > 1:
                from zero_order_recurrent_b200.probe_parallel import cdrge_step_sharded
                tk = ht[k % len(ht)].to(dev, non_blocking=True)
                tg = hg[k % len(hg)].to(dev, non_blocking=True)
                glp, glm = cdrge_step_sharded(ctx, theta, seed, n, eps, eta, tk, tg, coef)
                hp.copy_(glp, non_blocking=True)
                hm.copy_(glm, non_blocking=True)
                torch.cuda.current_stream().synchronize()
            else:
                zo.zo_step_host(ctx, theta, seed, n, eps, eta, ht[k % len(ht)], hg[k % len(hg)],
                                hp, hm)
        torch.cuda.synchronize()
        e_ms = (time.perf_counter() - t0) * 1e3
        if world > 1:
            t = torch.tensor([e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t.item())
        e2e = {"value": Ke / (e_ms / 1e3), "unit": "steps/s",
               "h2d_bytes_per_step": 2 * cfg.batch * cfg.seq * 4, "d2h_bytes_per_step": 2 * n * 4,
               "steps": Ke}
    ctx.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return {"ms": ms, "kinds": kinds, "clocks": clocks, "launches": launches, "e2e": e2e,
            "rank": rank, "world": world}


def captured_traffic(cfg):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary (profiles/traffic.json), or None when there is none or the
    kernel's source changed since the capture."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    e = json.load(open(p)).get(cfg.name)
    if not e:
        return None
    src = os.path.join(ROOT, e["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != e["sha256_16"]:
        return None
    return e["bytes_per_launch"]


def roofline_for(cfg, kinds, clocks, pk, steps, n_rank):
    n_cell, ms_cell, fl_cell, _ = kinds["cell"]
    if cfg.dtype == "bf16":
        achieved = fl_cell / (ms_cell / 1e3) / 1e12
        peak = pk["bf16_tflops_sustained"]
        out = {"bound": "tensor", "kernel": "cell_tc_kernel (tcgen05 perturbed LSTM cell)",
               "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
               "frac": round(achieved / peak, 4), "traffic": captured_traffic(cfg),
               "peak_source": f"{pk['source']} bf16 dense, sustained (a kernel timed inside a long step)",
               "frac_of_burst": round(achieved / pk["bf16_tflops"], 4),
               "frac_of_nominal_2250": round(achieved / 2250.0, 4),
               "launches": n_cell, "avg_launch_ms": round(ms_cell / max(n_cell, 1), 4),
               "flops": "executed"}
        if cfg.embed >= 512 and cfg.batch >= 256:
            # layer 0's input term comes from a per-chunk vocabulary table: the
            # cell launches execute fewer flops than a plain forward; the plain
            # forward's cell flops over the same time, for comparison
            H, E = cfg.hidden, cfg.embed
            per_token = sum(4 * H * ((E if l == 0 else H) + H) for l in range(cfg.layers))
            t0 = sum(4 * H * H for _ in range(cfg.layers))   # h_{-1} = 0 at t = 0
            plain = 2.0 * 2 * n_rank * cfg.batch * (cfg.seq * per_token - t0) * steps
            out["plain_forward_equiv_tflops"] = round(plain / (ms_cell / 1e3) / 1e12, 2)
            out["note"] = ("layer 0's input term from a vocabulary table built once per probe "
                           "chunk; achieved counts the flops executed")
        return out
    achieved = fl_cell / (ms_cell / 1e3) / 1e12
    mhz = pk["sm_max_mhz"]
    peak = fp32_alu_peak_tflops(mhz)
    # the context takes the probe-column kernel when E and H are multiples of 32
    wide = cfg.embed % 32 == 0 and cfg.hidden % 32 == 0
    name = ("fp32_wide_kernel (probe-column perturbed LSTM forward, 4 probes per CTA)" if wide
            else "fp32_forward_kernel (persistent perturbed LSTM forward)")
    return {"bound": "alu", "kernel": name,
            "achieved": round(achieved, 3), "peak": round(peak, 2), "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": captured_traffic(cfg),
            "peak_source": f"fp32 FMA: 148 SMs x 128 lanes x 2 x {mhz:.0f} MHz",
            "launches": n_cell, "avg_launch_ms": round(ms_cell / max(n_cell, 1), 4)}


class OracleSampler:
    """The C++ fp64 oracle (as it stands) on bounded samples of one CD-RGE step
    of `cfg`, on this host's cores.  A sample is one probe (both signs) over
    R2 = min(B, 16) batch rows plus the update of a contiguous run of m
    parameters with all n_pert probes.  The oracle's time for one probe grows
    linearly in the rows it evaluates, t(r) = t(1) + (r - 1) s, with an
    intercept that does not shrink with rows (it rebuilds every perturbed
    weight at every step), so one probe at 1 row and at R2 rows fix the line,
    and a full step is extrapolated as
        t_step = n_pert t(B) + t_update(m) d_pad / m.
    t(1) is the faster of two timings after an untimed first call (thread
    start-up and first touches would otherwise inflate the intercept and
    flatten the line)."""

    def __init__(self, cfg, rank=0):
        from oracle import native
        self.cfg = cfg
        self.N = native.Oracle()
        self.cores = native.cores()
        self.spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
        self.theta = W.init_theta(cfg)
        self.tok, self.tgt = batches(cfg, 1, rank)[0]
        self.d_pad = int(self.theta.size)
        self.m = min(self.d_pad, 1 << 22)
        self.coef = np.random.default_rng(0).standard_normal(cfg.n_pert) * 1e-3
        self.R2 = min(cfg.batch, 16)
        self.rows = np.arange(self.R2)
        self.t1 = None
        if cfg.batch > 1:
            ts = []
            for rep in range(3):                     # one probe, both signs, one row
                t0 = time.perf_counter()
                self.N.probe_row_losses(self.theta, self.spec, W.step_seed(rep), [0], cfg.eps,
                                        self.tok, self.tgt, rows=[0])
                ts.append(time.perf_counter() - t0)
            self.t1 = min(ts[1:])

    def sample(self, k):
        """One timed sample with probe k mod n_pert; returns (t_forward, t_update)."""
        cfg = self.cfg
        seed = W.step_seed(k)
        t0 = time.perf_counter()
        self.N.probe_row_losses(self.theta, self.spec, seed, [k % cfg.n_pert], cfg.eps, self.tok,
                                self.tgt, rows=self.rows)
        t1 = time.perf_counter()
        self.N.update_range(self.theta, self.spec, seed, cfg.n_pert, self.coef, 0, self.m)
        return t1 - t0, time.perf_counter() - t1

    def probe_seconds_full_batch(self, t_fwd):
        """One probe (both signs) over all B rows from the line through
        (1, t1) and (R2, t_fwd)."""
        B = self.cfg.batch
        if self.t1 is None or self.R2 <= 1:
            return t_fwd * B / self.R2
        slope = max(0.0, (t_fwd - self.t1) / (self.R2 - 1))
        return max(t_fwd, self.t1 + (B - 1) * slope)

    def step_seconds(self, t_fwd, t_upd):
        return (self.cfg.n_pert * self.probe_seconds_full_batch(t_fwd) +
                t_upd * self.d_pad / self.m)

    def describe(self, n_samples):
        cfg = self.cfg
        fit = ("" if self.t1 is None or self.R2 <= 1 else
               f"; one probe over 1 row took {self.t1:.2f} s, the line through that and the "
               f"{self.R2}-row samples gives the {cfg.batch}-row time")
        return (f"{n_samples} sample(s), each one probe (both signs) over {self.R2} of {cfg.batch} "
                f"rows at T={cfg.seq} plus the update of {self.m} of {self.d_pad} parameters with "
                f"all {cfg.n_pert} probes; extrapolated to the full step ({cfg.n_pert} probes x "
                f"{cfg.batch} rows, {self.d_pad} parameters){fit}")


def oracle_sample(cfg, budget_s=15.0, rank=0):
    """cpu_baseline: the C++ fp64 oracle timed on a bounded sample of one step."""
    t_all = time.perf_counter()
    S = OracleSampler(cfg, rank=rank)
    t_fwd, t_upd, n = 0.0, 0.0, 0
    while n < cfg.n_pert and (n == 0 or time.perf_counter() - t_all < budget_s):
        f, u = S.sample(n)
        t_fwd, t_upd, n = t_fwd + f, t_upd + u, n + 1
    step_s = S.step_seconds(t_fwd / n, t_upd / n)
    return {"value": 1.0 / step_s, "unit": "steps/s", "cores": S.cores, "kind": "oracle",
            "impl": "C++17 fp64, std::thread (oracle/zo_oracle_cpu.cpp)",
            "sample": S.describe(n), "extrapolated": True,
            "perturbed_tokens_per_s": 2 * n * S.R2 * cfg.seq / t_fwd,
            "seconds": round(time.perf_counter() - t_all, 2)}


def run_reference(args, cfg, config):
    """The reference arm: the C++ fp64 oracle as it stands, on this host's
    cores, W warm-up and K timed samples (each a bounded sample of one step,
    sized so the whole run stays within a few minutes), extrapolated."""
    S = OracleSampler(cfg)
    for k in range(args.warmup):
        S.sample(k)
    t0 = time.perf_counter()
    fs, us = [], []
    for k in range(args.steps):
        f, u = S.sample(args.warmup + k)
        fs.append(f)
        us.append(u)
    wall = time.perf_counter() - t0
    t_fwd, t_upd = sum(fs) / len(fs), sum(us) / len(us)
    v = 1.0 / S.step_seconds(t_fwd, t_upd)
    cb = {"value": v, "unit": "steps/s", "cores": S.cores, "kind": "oracle",
          "impl": "C++17 fp64, std::thread (oracle/zo_oracle_cpu.cpp)",
          "sample": S.describe(args.steps), "extrapolated": True}
    return {"metric": METRIC, "impl": "reference", "value": v, "unit": "steps/s",
            "perturbed_tokens_per_s": 2 * S.R2 * cfg.seq / t_fwd, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": wall / args.steps * 1e3,
            "ms_per_full_step_extrapolated": 1e3 / v,
            "extrapolated": True,
            "note": ("each timed step is one bounded sample (see cpu_baseline.sample); value is "
                     "the full step's rate extrapolated from the samples, ms_per_step the "
                     "samples' own time"),
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "config": config, "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="lstm1b", choices=sorted(W.CONFIGS))
    ap.add_argument("--chunk", type=int, default=None,
                    help="probes per pass (default: the workload's); smaller chunks hold less "
                         "workspace, e.g. for a profiler capture")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cell-variant", default="single", choices=sorted(CELL_VARIANTS),
                    help="how and on which tiles the cell GEMMs form W +- eps P "
                         "(include/zo_debug.h): single-CTA tiles with the bf16 tile perturbed in "
                         "shared memory (default), the separate +-eps P product (exact eps, twice "
                         "the MMA work), CTA-pair tiles, or pair tiles with W read into registers")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    cfg = W.CONFIGS[args.config]
    if args.chunk is not None:
        import dataclasses
        cfg = dataclasses.replace(cfg, chunk=args.chunk)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    tokens_per_step = 2 * cfg.n_pert * cfg.batch * cfg.seq
    config = {"workload": f"{cfg.name}: {cfg.layers}-layer LSTM V={cfg.vocab} E={cfg.embed} H={cfg.hidden}, "
                          f"batch {cfg.batch} x seq {cfg.seq}, n_pert={cfg.n_pert}, eps=eta={cfg.eps}",
              "params": int(W.segments(cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)[1]),
              "global_batch": cfg.batch, "seq_len": cfg.seq, "n_pert": cfg.n_pert,
              "parallelism": (f"probe-parallel x{world} (NCCL all-gather of the 2 n_pert losses)"
                              if world > 1 else "single GPU"),
              "l2": "flushed (256 MB write) before every timed step, flush untimed",
              "tokens": "seeded synthetic (workloads module)"}
    if args.cell_variant != "single":
        config["cell_variant"] = args.cell_variant
    dtype = "bf16" if cfg.dtype == "bf16" else "f32"

    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(args, cfg, config)), flush=True)
        return

    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    r = run_ours(args, cfg)
    if rank != 0:
        return
    from zero_order_recurrent_b200.probe_parallel import probe_slice
    pk = peaks()
    value = args.steps / (r["ms"] / 1e3)
    out = {"metric": METRIC, "value": value, "unit": "steps/s",
           "perturbed_tokens_per_s": value * tokens_per_step, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": r["ms"] / args.steps, "higher_is_better": True,
           "scaling": "strong", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
           "config": config,
           "roofline": roofline_for(cfg, r["kinds"], r["clocks"], pk, args.steps,
                                    probe_slice(cfg.n_pert, 0, world)[1])}
    if cfg.dtype == "bf16":
        # the whole step against the same peak: the plain dense forward's flops
        # (2 n_pert B T tokens, 2 flop per multiply-add) over the step time
        fl_step = 2.0 * forward_macs_per_token(cfg) * tokens_per_step
        out["roofline"]["whole_step_tflops"] = round(fl_step / (r["ms"] / args.steps / 1e3) / 1e12, 2)
        out["roofline"]["whole_step_frac"] = round(out["roofline"]["whole_step_tflops"] /
                                                   out["roofline"]["peak"], 4)
    nu, msu, _, byu = r["kinds"]["update"]
    if nu:
        gbs = byu / (msu / 1e3) / 1e9
        out["update_roofline"] = {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"],
                                  "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
                                  "avg_launch_ms": round(msu / nu, 4)}
    nl, msl, fll, byl = r["kinds"]["loss"]
    if nl:
        out["loss_kernel"] = {"launches": nl, "avg_launch_ms": round(msl / nl, 4),
                              "tflops": round(fll / (msl / 1e3) / 1e12, 2),
                              "gbs": round(byl / (msl / 1e3) / 1e9, 1)}
    out["kernel_time_share"] = {k: round(v[1] / r["ms"], 4) for k, v in r["kinds"].items()}
    out["e2e"] = r["e2e"]
    out["gpu_launches"] = r["launches"]
    out["clocks"] = r["clocks"]
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = oracle_sample(cfg)
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
