#!/usr/bin/env python
"""Benchmark of the SPIN decode step on B200.

One step = the whole hot path for one batch: query quantisation, predict +
block max-pool, budget / exploration select, paged FP8 indexer score on the
kept blocks (with the fused EMA update) and the token top-k, for 96 requests at
512K context (the serving-shaped workload).  Metric: decode rows/s (requests x
query rows per second), with index-key GB/s and the fraction of the HBM
roofline alongside.

Arms:
  default            libspin.so through its C ABI (device-resident inputs);
                     also an end-to-end pass with host buffers, a 0% / 40% / 50%
                     sparsity sweep, GPU-measured fidelity and the CPU oracle
                     baseline.
  --impl reference   the CPU oracle on this host's cores, on a bounded sample
                     of the same workload per step.

Multi-GPU (torchrun): every rank runs its own 96 requests (requests are
independent: weak scaling, no data-path collective); the time is the max over
ranks and the value counts every rank's rows.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "SPIN decode rows/s & index-key GB/s at 512K ctx x96 req; % of roofline"
POOLINGS = {"max": 0, "mean": 1, "top4": 2}
MTP_POLICIES = {"union-prefix": 0, "row0": 1}   # the method's policy, then the baseline it is compared with
WORKLOADS = {"serve-96x512K": 2, "mtp-32x128K-r4": 3, "ragged-8Lx8-256K-1M": 4, "dsa-1x64K": 1, "tiny-fp32-4K": 0}
KEY_BYTES_PER_SLOT = 128 + 4            # E4M3 key row + fp32 scale
SCORE_BYTES_PER_SLOT = 128 + 4 + 4 + 16  # + score write + fused EMA read/write of V and D
# DRAM traffic of one k_score_tc launch (dram__bytes_read.sum + dram__bytes_write.sum)
# per kept slot, from one ncu capture per launch plan (traffic grows with kept slots:
# each is read once), valid for the kernel source with this hash prefix:
#   "fused-r1": 16 requests at 512K, 50% sparsity, one row, fused EMA;
#   "deferred-r4": 32 requests at 128K, 40% sparsity, four MTP rows, no EMA in the launch
SCORE_TRAFFIC = {"src_sha256_16": "8ea7182b712ae393",
                 "bytes_per_kept_slot": {"fused-r1": 151.33, "deferred-r4": 146.20},
                 "sources": ("indexer_sparse_attention_b200/csrc/k_score_tc.cu",
                             "indexer_sparse_attention_b200/csrc/spin_internal.cuh")}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["spin", "reference"], default="spin")
    p.add_argument("--sparsity", type=float, default=0.5)
    p.add_argument("--requests", type=int, default=96, help="requests per GPU (96 = the serving workload)")
    p.add_argument("--no-sweep", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--workload", choices=list(WORKLOADS), default="serve-96x512K",
                   help="serve-96x512K is the headline; the others print their own line")
    p.add_argument("--pooling", choices=list(POOLINGS), default="max",
                   help="block reduction of the predicted scores (max is the method's)")
    p.add_argument("--mtp-policy", choices=list(MTP_POLICIES), default="union-prefix",
                   help="several query rows: row-local union + prefix-valid update (the method's) or row 0 alone")
    p.add_argument("--lookahead", action="store_true",
                   help="pipelined one-row steps (spin_set_lookahead): each step prepares the next step's "
                        "selection, whose select kernel runs beside the step's top-k")
    p.add_argument("--prepare-layers", action="store_true",
                   help="with --lookahead on a multi-layer workload: every layer's selection of a step is made "
                        "at once (spin_prepare_selections) before the first layer's step")
    p.add_argument("--ablation", choices=["pooling", "mtp", "predictors"], default=None,
                   help="pooling: miss and step time of max / mean / top-4 pooling over target sparsities; "
                        "mtp: p99 miss vs realized sparsity of the two MTP policies on the 4-row workload; "
                        "predictors: Pearson correlation and top-k recall of the random, previous-layer, "
                        "previous-iteration and SPIN predictors")
    return p.parse_args()


# ---------------------------------------------------------------------------
# process group (one rank per GPU) and device clocks
# ---------------------------------------------------------------------------
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's time: every rank takes the same collective step."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(rank: int, requests: int, spare_slots: int):
    """The serving workload a rank runs: the same shape on every rank, its
    own seeded data (requests are independent, so ranks share nothing)."""
    base = workloads.config(2)
    return workloads.config(2, seed=base.seed + 1000 * rank, steps=1, spare_slots=spare_slots,
                            requests=requests, ctx0=base.ctx0[:1] * requests)


def job_rows_per_s(rows_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank's rows over the slowest rank's time."""
    return world * rows_per_rank / (max_ms / 1e3)


class ClockSampler:
    """SM clock, utilisation and clock-event reasons of this GPU, read through
    NVML from a thread every 5 ms while the timed region runs (one reading at
    entry and one at exit as well, so a short region still has samples).
    Falls back to an nvidia-smi process when NVML cannot be opened.  Reads
    only; changes no setting."""

    FIELDS = ("clocks.sm,clocks.max.sm,utilization.gpu,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    # clock-event reason bits (NVML): name -> mask
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40}

    def __init__(self, device_index: int):
        self.proc = None
        self.thread = None
        self.rows = []
        self.path = tempfile.mktemp(suffix=".csv")
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            ident = str(device_index)
        self.ident = ident
        self.nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(ident)
            self.nvml = pynvml
        except Exception:
            self.nvml = None

    def _read(self):
        n, h = self.nvml, self.handle
        try:
            reasons = n.nvmlDeviceGetCurrentClocksEventReasons(h)
        except Exception:
            reasons = n.nvmlDeviceGetCurrentClocksThrottleReasons(h)
        return (float(n.nvmlDeviceGetClockInfo(h, n.NVML_CLOCK_SM)),
                float(n.nvmlDeviceGetMaxClockInfo(h, n.NVML_CLOCK_SM)),
                float(n.nvmlDeviceGetUtilizationRates(h).gpu), int(reasons))

    def _loop(self):
        import time
        while not self.stop:
            try:
                self.rows.append(self._read())
            except Exception:
                return
            time.sleep(0.005)

    def __enter__(self):
        if self.nvml is not None:
            import threading
            self.stop = False
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()
            return self
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.ident}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            try:
                self.rows.append(self._read())
            except Exception:
                pass
            self.stop = True
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.nvml is not None:
            if not self.rows:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
            sm = np.array([r[0] for r in self.rows])
            util = np.array([r[2] for r in self.rows])
            loaded = sm[util > 0] if np.any(util > 0) else sm
            reasons = sorted({k for r in self.rows for k, bit in self.REASONS.items() if r[3] & bit})
            return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": self.rows[0][1], "reasons": reasons,
                    "samples": len(self.rows), "samples_under_load": int(loaded.size), "source": "nvml, 5 ms"}
        rows = []
        try:
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        except Exception:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = np.array([float(r[0]) for r in rows])
        mx = float(rows[0][1])
        util = np.array([float(r[2]) if r[2].replace(".", "").isdigit() else 0.0 for r in rows])
        loaded = sm[util > 0] if np.any(util > 0) else sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "samples_under_load": int(loaded.size), "source": "nvidia-smi, 50 ms"}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def score_traffic_per_slot(plan="fused-r1"):
    """The captured DRAM bytes per kept slot of a launch plan, or None for a
    plan without a capture or once the kernel source differs from the one the
    counters were taken on."""
    import hashlib
    h = hashlib.sha256()
    for f in SCORE_TRAFFIC["sources"]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest()[:16] != SCORE_TRAFFIC["src_sha256_16"]:
        return None
    return SCORE_TRAFFIC["bytes_per_kept_slot"].get(plan)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class SpinRun:
    def __init__(self, wl, device, total_steps, pooling=0, lookahead=False):
        import indexer_sparse_attention_b200 as isa
        self.isa = isa
        self.wl = wl
        self.device = device
        self.cache = workloads.make_key_cache(wl, 0, device)
        self.positions = total_steps + 1
        q, w = workloads.make_queries(wl, 0, self.positions, device)
        self.q = [q[:, t:t + 1].contiguous() for t in range(self.positions)]
        self.w = [w[:, t:t + 1].contiguous() for t in range(self.positions)]
        del q, w
        ctx0 = torch.tensor(wl.ctx0, dtype=torch.int64, device=device)
        self.ctx = [(ctx0 + t + 1).to(torch.int32) for t in range(self.positions)]
        cfg = isa.make_config(num_layers=1, num_requests=wl.requests, max_slots=wl.max_slots, block_size=wl.b,
                              num_heads=wl.H, head_dim=wl.d, topk=wl.topk, max_rows=1, key_fp8=True, q_bf16=True,
                              alpha=wl.alpha, gamma=wl.gamma, target_sparsity=wl.sparsity, seed=wl.seed,
                              pooling=pooling)
        self.cfg = cfg
        self.st = isa.SpinState(cfg, device=device)
        self.lookahead = lookahead
        isa.spin_set_lookahead(self.st, lookahead)
        self.mask = self.st.new_mask()
        self.topk = torch.empty((wl.requests, 1, wl.topk), dtype=torch.int32, device=device)
        self.scores = self.st.new_scores()
        self.t = 0

    def set_sparsity(self, s):
        self.isa.spin_set_layer_sparsity(self.st, [s])

    def step(self, defer=False, q=None, w=None, ctx=None, mask=None, topk=None):
        t = self.t
        c = self.cache
        self.isa.spin_decode_step(self.st, 0, 1, t, c.keys, c.kscale, c.block_table,
                                  self.q[t] if q is None else q, self.w[t] if w is None else w,
                                  self.ctx[t] if ctx is None else ctx, defer,
                                  self.mask if mask is None else mask, self.topk if topk is None else topk,
                                  self.scores)
        self.t += 1

    def kept_slots(self):
        """Slots scored in the last step (kept blocks, visible part)."""
        ctx = self.ctx[self.t - 1].long()
        nb = (ctx + self.wl.b - 1) // self.wl.b
        m = self.mask.bool()
        kept_blocks = m.sum(dim=1)
        last = nb - 1
        tail_kept = m.gather(1, last[:, None])[:, 0]
        tail_slots = ctx - last * self.wl.b
        slots = kept_blocks * self.wl.b - tail_kept.long() * (self.wl.b - tail_slots)
        return int(slots.sum().item()), (kept_blocks.double() / nb.double())


def timed_steps(run, steps, world, defer=False):
    barrier(world)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(steps):
        run.step(defer=defer)
    e1.record(s)
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(e0.elapsed_time(e1), world)


def fidelity(run, n_steps=3):
    """Mean / p99 miss (share of the full indexer's top-k in skipped blocks)
    and realized block sparsity, measured on the GPU with a shadow full
    indexer on the same inputs; outside every timed region."""
    isa, wl = run.isa, run.wl
    full_scores = run.st.new_scores()
    full_topk = torch.empty_like(run.topk)
    missed = torch.zeros((wl.requests, 1), dtype=torch.int32, device=run.device)
    total = torch.zeros_like(missed)
    allk = torch.ones_like(run.mask)
    miss, realized = [], []
    c = run.cache
    for _ in range(n_steps):
        t = run.t
        run.step()
        isa.spin_indexer_score(run.st, 0, 1, c.keys, c.kscale, c.block_table, run.q[t], run.w[t], run.ctx[t],
                               allk, full_scores)
        isa.spin_topk(run.st, 1, full_scores, allk, run.ctx[t], full_topk)
        isa.spin_miss_count(run.st, 1, full_topk, run.mask, missed, total)
        miss += (missed.double() / total.double().clamp(min=1))[:, 0].tolist()
        realized += (1 - run.kept_slots()[1]).tolist()
    v = np.sort(np.array(miss))
    p99 = float(v[max(int(np.ceil(0.99 * v.size)), 1) - 1])
    return {"mean_miss": float(v.mean()), "p99_miss": p99, "realized_sparsity": float(np.mean(realized)),
            "rows": int(v.size)}


def e2e_pass(run, steps, world):
    """The same decode step through the public API with host buffers, run the
    way a server overlaps transfers: while step i computes, a copy stream
    brings step i+1's query, head weights and context lengths in from pinned
    host memory and reads step i-1's top-k indices and block mask back (two
    device buffers of each alternate).  Every step's copies lie inside the
    timed region, which ends when the last read-back has landed."""
    wl = run.wl
    t0 = run.t
    q_h = [run.q[t0 + i].cpu().pin_memory() for i in range(steps)]
    w_h = [run.w[t0 + i].cpu().pin_memory() for i in range(steps)]
    c_h = [run.ctx[t0 + i].cpu().pin_memory() for i in range(steps)]
    q_d = [torch.empty_like(run.q[0]) for _ in range(2)]
    w_d = [torch.empty_like(run.w[0]) for _ in range(2)]
    c_d = [torch.empty_like(run.ctx[0]) for _ in range(2)]
    topk_d = [torch.empty_like(run.topk) for _ in range(2)]
    mask_d = [torch.empty_like(run.mask) for _ in range(2)]
    topk_h = [torch.empty(run.topk.shape, dtype=torch.int32).pin_memory() for _ in range(2)]
    mask_h = [torch.empty(run.mask.shape, dtype=torch.uint8).pin_memory() for _ in range(2)]
    h2d = q_h[0].numel() * q_h[0].element_size() + w_h[0].numel() * 4 + c_h[0].numel() * 4
    d2h = topk_h[0].numel() * 4 + mask_h[0].numel()
    compute = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready, done, out_read = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(compute)
    copy.wait_stream(compute)

    def bring_in(i, b):
        with torch.cuda.stream(copy):
            q_d[b].copy_(q_h[i], non_blocking=True)
            w_d[b].copy_(w_h[i], non_blocking=True)
            c_d[b].copy_(c_h[i], non_blocking=True)
            in_ready[b].record(copy)

    bring_in(0, 0)
    for i in range(steps):
        b = i % 2
        if i + 1 < steps:
            if i >= 1:
                copy.wait_event(done[1 - b])   # step i-1 no longer reads buffer 1-b
            bring_in(i + 1, 1 - b)
        compute.wait_event(in_ready[b])
        if i >= 2:
            compute.wait_event(out_read[b])    # step i-2's results are out of buffer b
        run.step(q=q_d[b], w=w_d[b], ctx=c_d[b], mask=mask_d[b], topk=topk_d[b])
        done[b].record(compute)
        copy.wait_event(done[b])
        with torch.cuda.stream(copy):
            topk_h[b].copy_(topk_d[b], non_blocking=True)
            mask_h[b].copy_(mask_d[b], non_blocking=True)
            out_read[b].record(copy)
    compute.wait_stream(copy)
    e1.record(compute)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    # the last step's results as read back equal the device copy
    if not (torch.equal(topk_h[(steps - 1) % 2], topk_d[(steps - 1) % 2].cpu())
            and torch.equal(mask_h[(steps - 1) % 2], mask_d[(steps - 1) % 2].cpu())):
        raise RuntimeError("end-to-end read-back does not match the device results")
    return ms, h2d, d2h


def gpu_arm(args, world, rank, local):
    import indexer_sparse_attention_b200 as isa
    from indexer_sparse_attention_b200 import build
    if rank == 0 or world == 1:
        build.build()
    barrier(world)
    isa.load()
    device = torch.device("cuda", local if world > 1 else 0)
    W, K = args.warmup, args.steps
    sweep = [] if args.no_sweep else [0.4, 0.0]
    KS = min(K, 40)  # steps of the per-stage timing pass
    total = 1 + (W + K) * (1 + len(sweep)) + 9 + K + KS + 2
    wl = rank_workload(rank, args.requests, total + 8)
    run = SpinRun(wl, device, total, POOLINGS[args.pooling], lookahead=args.lookahead)
    Q = wl.requests
    # history bootstrap: all-keep step that fills V and D
    run.set_sparsity(0.0)
    run.step()
    # ---- headline: target sparsity, score kernel timed live -------------
    run.set_sparsity(args.sparsity)
    for _ in range(W):
        run.step()
    # CUDA events bracket only the dominant kernel inside the timed region,
    # so the other launches run back to back as in service; launches of every
    # stage are counted
    isa.spin_kernel_times(run.st)
    isa.spin_set_kernel_timing_mask(run.st, ["score"])
    with ClockSampler(device.index) as clk:
        ms = timed_steps(run, K, world)
    isa.spin_set_kernel_timing(run.st, False)
    stages = isa.spin_kernel_times(run.st)
    # per-stage breakdown from a separate pass with every launch bracketed
    isa.spin_set_kernel_timing(run.st, True)
    timed_steps(run, KS, world)
    isa.spin_set_kernel_timing(run.st, False)
    stage_pass = isa.spin_kernel_times(run.st)
    kept_slots, kept_frac = run.kept_slots()
    status, word = isa.spin_get_error(run.st)
    if status != 0:
        raise RuntimeError(f"device error word {word:#x} during the timed region")
    ms_step = ms / K
    rows_s = job_rows_per_s(Q * K, world, ms)
    key_gbs = kept_slots * KEY_BYTES_PER_SLOT / (ms_step / 1e3) / 1e9
    peak, peak_kind = peaks()
    score_ms, score_n = stages["score"]
    score_avg = score_ms / max(score_n, 1)
    score_b = score_bytes_per_slot(1, True, True, 128, args.pooling == "max")
    achieved = kept_slots * score_b / (score_avg / 1e3) / 1e9
    traffic_slot = score_traffic_per_slot()
    launches = sum(n for _, n in stages.values())
    step_tr = step_traffic(int(run.ctx[run.t - 1].long().sum().item()), kept_slots, ms_step, peak, args.pooling)
    out = {
        "metric": METRIC, "value": rows_s, "unit": "rows/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3xe4m3->f32 (selection f32, exact)", "data": "synthetic",
        "config": headline_config(wl, Q, args, world),
        "index_key_gbs": key_gbs,
        "key_roofline_frac": key_gbs / peak,
        "step_traffic": step_tr,
        "roofline": {"bound": "hbm", "kernel": "k_score_tc (paged FP8 indexer + fused EMA)",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": f"{peak_kind} hbm_gbs (copy, MEASURED_PEAKS.json)" if peak_kind == "measured"
                     else "fallback 6650 GB/s", "avg_launch_ms": score_avg,
                     "bytes_per_launch": kept_slots * score_b,
                     "traffic": (None if traffic_slot is None else traffic_slot * kept_slots),
                     "traffic_source": ("ncu dram__bytes_read.sum + dram__bytes_write.sum per kept slot "
                                        "(16-request capture, scaled by kept slots)" if traffic_slot is not None
                                        else "null: the kernel source has changed since the last ncu capture")},
        "pipelined": ("each step prepares the next step's selection, whose select kernel runs beside the "
                      "step's top-k on a second stream (spin_set_lookahead); results are those of the "
                      "sequential step" if run.lookahead else "no: sequential steps"),
        "stage_ms_per_step": {k: v[0] / KS for k, v in stage_pass.items() if v[1]},
        "stage_ms_source": (f"separate pass of {KS} steps with every launch bracketed by CUDA events"
                            + ("; the top-k overlaps the next step's select" if run.lookahead else "")),
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    # ---- sparsity sweep: 40% and the 0% all-keep control ------------------
    sw = {str(int(round(args.sparsity * 100))): ms_step}
    for s in sweep:
        run.set_sparsity(s)
        for _ in range(W):
            run.step(defer=(s == 0.0))
        sw[str(int(round(s * 100)))] = timed_steps(run, K, world, defer=(s == 0.0)) / K
    if sweep:
        out["sweep_ms_per_step"] = sw
        out["sweep_monotonic"] = bool(sw.get("0", 1e9) > sw.get("40", 0) > sw.get(str(int(round(args.sparsity * 100))), -1))
    # ---- fidelity (outside timed regions) ---------------------------------
    run.set_sparsity(args.sparsity)
    out["fidelity"] = fidelity(run)
    # the 1% planted vertical slots outnumber k, so at 40-50% nothing is
    # missed; higher targets are where the synthetic input tells policies apart
    by_s = {str(int(round(args.sparsity * 100))): out["fidelity"]}
    for s in (0.7, 0.8):
        run.set_sparsity(s)
        by_s[str(int(round(s * 100)))] = fidelity(run)
    out["fidelity_by_sparsity"] = by_s
    run.set_sparsity(args.sparsity)
    # ---- end to end with host buffers --------------------------------------
    e2e_ms, h2d, d2h = e2e_pass(run, K, world)
    out["e2e"] = {"value": job_rows_per_s(Q * K, world, e2e_ms), "unit": "rows/s", "h2d_bytes_per_step": h2d,
                  "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / K,
                  "transfers": "pinned host buffers; step i+1's inputs in and step i-1's results out on a copy "
                               "stream while step i computes (double-buffered), all inside the timed region"}
    # ---- the same step replayed from one captured CUDA graph ---------------
    out["graph_replay"] = graph_pass(run, W, K, world)
    status, word = isa.spin_get_error(run.st)
    if status != 0:
        raise RuntimeError(f"device error word {word:#x}")
    return out


def graph_pass(run, warmup, steps, world):
    """The decode step captured once in a CUDA graph -- the step number from
    the state's device counter, advanced inside the graph -- and replayed;
    every replay uses the same query rows and context lengths."""
    isa, wl = run.isa, run.wl
    t = run.t
    q_buf, w_buf, c_buf = run.q[t].clone(), run.w[t].clone(), run.ctx[t].clone()
    # the same ctx_len every replay breaks the one-slot-a-step contract of a
    # pipelined step: replay the sequential step
    isa.spin_set_lookahead(run.st, False)
    isa.spin_set_step(run.st, t)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    c = run.cache
    with torch.cuda.graph(graph):
        isa.spin_decode_step(run.st, 0, 1, isa.SPIN_STEP_DEVICE, c.keys, c.kscale, c.block_table, q_buf, w_buf,
                             c_buf, False, run.mask, run.topk, run.scores)
        isa.spin_advance_step(run.st)
    for _ in range(warmup):
        graph.replay()
    barrier(world)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(steps):
        graph.replay()
    e1.record(s)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    del graph
    return {"value": job_rows_per_s(wl.requests * steps, world, ms), "unit": "rows/s", "ms_per_step": ms / steps,
            "note": "one captured graph per step (device step counter), same inputs every replay; "
                    "the sequential step (no lookahead)"}


# ---------------------------------------------------------------------------
# The other workloads (MTP rows, multi-layer ragged contexts, single request,
# tiny fp32): one JSON line each, same keys as the headline where they apply
# ---------------------------------------------------------------------------
L2_BYTES = 126 * 1024 * 1024


def score_bytes_per_slot(rows: int, fused: bool, key_fp8: bool, d: int, vmax: bool = False) -> float:
    """Algorithmic bytes of the score kernel per kept slot: the key row and
    its scale, one score per row, (fused, one row) the EMA read/write of V
    and D, and with it (max pooling) V's maximum of each 32 kept slots."""
    key = (d + 4) if key_fp8 else 4 * d
    return key + 4 * rows + (16 if fused else 0) + (4 / 32 if fused and vmax else 0)


class WorkloadRun:
    """A workload through the C ABI with every layer's key cache and queries
    resident on the device.  The per-step inputs (each request's query rows
    at its committed position, context lengths, accepted lengths) are built
    before any timed region."""

    def __init__(self, wl, device, total_steps):
        import indexer_sparse_attention_b200 as isa
        self.isa, self.wl, self.device = isa, wl, device
        Q, R, Ly = wl.requests, wl.rows, wl.layers
        self.caches = [workloads.make_key_cache(wl, l, device) for l in range(Ly)]
        acc = workloads.accepted_lengths(wl, total_steps).numpy()
        committed = np.array(wl.ctx0, np.int64)
        ctx0 = committed.copy()
        plans = []
        for t in range(total_steps):
            plans.append((committed - ctx0, committed + 1, acc[t]))
            committed = committed + acc[t]
        self.ctx = [torch.from_numpy(c.astype(np.int32)).to(device) for _, c, _ in plans]
        self.acc = [torch.from_numpy(a.astype(np.int32)).to(device) for _, _, a in plans]
        self.qw = [[None] * Ly for _ in range(total_steps)]
        rows_idx = torch.arange(R)
        for l in range(Ly):
            q_all, w_all = workloads.make_queries(wl, l, total_steps * R + R, device)
            for t, (pos0, _, _) in enumerate(plans):
                idx = (torch.from_numpy(pos0)[:, None] + rows_idx[None, :]).to(device)
                ar = torch.arange(Q, device=device)[:, None]
                self.qw[t][l] = (q_all[ar, idx].contiguous(), w_all[ar, idx].contiguous())
            del q_all, w_all
        cfg = isa.make_config(num_layers=Ly, num_requests=Q, max_slots=wl.max_slots, block_size=wl.b,
                              num_heads=wl.H, head_dim=wl.d, topk=wl.topk, max_rows=R, key_fp8=wl.key_fp8,
                              q_bf16=wl.q_bf16, alpha=wl.alpha, gamma=wl.gamma, target_sparsity=wl.sparsity,
                              seed=wl.seed, pooling=wl.pooling, mtp_policy=wl.mtp_policy)
        self.cfg = cfg
        self.st = isa.SpinState(cfg, device=device)
        self.lookahead = False
        self.prepare = False              # spin_prepare_selections before each step's layers
        self.masks = [self.st.new_mask() for _ in range(Ly)]
        self.topks = [torch.empty((Q, R, wl.topk), dtype=torch.int32, device=device) for _ in range(Ly)]
        self.scores = self.st.new_scores()
        self.t = 0

    def set_sparsity(self, per_layer):
        self.isa.spin_set_layer_sparsity(self.st, list(per_layer))

    def restart(self, **cfg_fields):
        """A fresh state (never-observed V, D) with some config fields
        changed; the inputs are replayed from step 0."""
        for k, v in cfg_fields.items():
            setattr(self.cfg, k, v)
        self.st = self.isa.SpinState(self.cfg, device=self.device)
        self.isa.spin_set_lookahead(self.st, self.lookahead)
        self.t = 0

    def set_lookahead(self, on):
        self.lookahead = bool(on)
        self.isa.spin_set_lookahead(self.st, self.lookahead)

    def step(self, layers=None):
        """One decode step of every layer: a0..a5, and for MTP rows the
        prefix-valid EMA replay once the accepted lengths are known."""
        isa, wl, t = self.isa, self.wl, self.t
        R = wl.rows
        if self.prepare and self.lookahead and layers is None:
            isa.spin_prepare_selections(self.st, t, self.ctx[t])
        for l in (range(wl.layers) if layers is None else layers):
            c = self.caches[l]
            q, w = self.qw[t][l]
            isa.spin_decode_step(self.st, l, R, t, c.keys, c.kscale if wl.key_fp8 else None, c.block_table, q, w,
                                 self.ctx[t], R > 1, self.masks[l], self.topks[l], self.scores)
            if R > 1:
                isa.spin_ema_update(self.st, l, R, self.scores, self.masks[l], self.ctx[t], self.acc[t])
        self.t += 1

    def kept_slots(self, t):
        """Visible slots of the kept blocks at step t (row R-1 sees the most),
        summed over layers, and the realized sparsity per (layer, request)."""
        wl = self.wl
        ctx = self.ctx[t].long() + wl.rows - 1
        nb = (ctx + wl.b - 1) // wl.b
        total, realized = 0, []
        for m8 in self.masks:
            m = m8[:, : int(nb.max())].bool()
            kept = m.sum(dim=1)
            last = nb - 1
            tail_kept = m.gather(1, last[:, None])[:, 0]
            slots = kept * wl.b - tail_kept.long() * (wl.b - (ctx - last * wl.b))
            total += int(slots.sum().item())
            realized += (1 - kept.double() / nb.double()).tolist()
        return total, realized

    def miss(self):
        """Share of the full indexer's top-k in skipped blocks, per layer and
        (request, row), for the step just run (shadow all-keep indexer)."""
        isa, wl, t = self.isa, self.wl, self.t - 1
        R, Q = wl.rows, wl.requests
        full_scores = self.st.new_scores()
        full_topk = torch.empty((Q, R, wl.topk), dtype=torch.int32, device=self.device)
        missed = torch.zeros((Q, R), dtype=torch.int32, device=self.device)
        total = torch.zeros_like(missed)
        out = []
        for l in range(wl.layers):
            c = self.caches[l]
            q, w = self.qw[t][l]
            allk = torch.ones_like(self.masks[l])
            isa.spin_indexer_score(self.st, l, R, c.keys, c.kscale if wl.key_fp8 else None, c.block_table, q, w,
                                   self.ctx[t], allk, full_scores)
            isa.spin_topk(self.st, R, full_scores, allk, self.ctx[t], full_topk)
            isa.spin_miss_count(self.st, R, full_topk, self.masks[l], missed, total)
            out.append((missed.double() / total.double().clamp(min=1)).flatten().tolist())
        return out


def workload_arm(args, world, rank, local):
    """One of the non-headline workloads: history bootstrap, the workload's
    own warm-up protocol, then K timed steps (every layer, every row)."""
    import indexer_sparse_attention_b200 as isa
    from indexer_sparse_attention_b200 import build
    if rank == 0 or world == 1:
        build.build()
    barrier(world)
    isa.load()
    device = torch.device("cuda", local if world > 1 else 0)
    base = workloads.config(WORKLOADS[args.workload])
    W, K = max(args.warmup, 3), args.steps
    fid_steps = 3
    total = 1 + base.warmup_steps + W + K + fid_steps
    wl = workloads.config(WORKLOADS[args.workload], seed=base.seed + 1000 * rank, steps=total,
                          spare_slots=base.rows * 4, pooling=POOLINGS[args.pooling],
                          mtp_policy=MTP_POLICIES[args.mtp_policy])
    run = WorkloadRun(wl, device, total)
    run.set_lookahead(args.lookahead)   # applies to one-row steps
    run.prepare = bool(args.prepare_layers and args.lookahead and wl.rows == 1 and wl.key_fp8)
    Ly, Q, R = wl.layers, wl.requests, wl.rows
    # history bootstrap (all-keep), then the workload's warm-up protocol
    run.set_sparsity([0.0] * Ly)
    run.step()
    sparsity = [wl.sparsity] * Ly
    run.set_sparsity(sparsity)
    alloc = None
    if wl.warmup_steps:
        # uniform target with a shadow full indexer measuring each layer's miss,
        # then budgets in proportion to the measured miss (per-layer budget)
        miss = np.zeros(Ly)
        for _ in range(wl.warmup_steps):
            run.step()
            miss += np.array([np.mean(m) for m in run.miss()])
        miss /= wl.warmup_steps
        nblk = (np.array(wl.ctx0, np.float64) + wl.b - 1) // wl.b
        blocks = np.full(Ly, nblk.sum())
        lo = np.full(Ly, max(0.05, float(np.ceil(wl.topk / wl.b) / nblk.min())))
        sparsity = isa.spin_allocate_layer_sparsity(miss.tolist(), blocks.tolist(), lo.tolist(), wl.sparsity)
        run.set_sparsity(sparsity)
        alloc = {"warmup_miss": miss.tolist(), "layer_sparsity": sparsity}
    for _ in range(W):
        run.step()
    # L2-resident workloads are timed step by step with L2 flushed in between
    input_bytes = sum(c.keys.numel() * c.keys.element_size() for c in run.caches)
    flush = input_bytes < 2 * L2_BYTES
    scratch = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device) if flush else None
    isa.spin_kernel_times(run.st)
    isa.spin_set_kernel_timing(run.st, True)
    s = torch.cuda.current_stream()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(device.index) as clk:
        if flush:
            ms = 0.0
            for _ in range(K):
                scratch.fill_(1.0)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(s)
                run.step()
                e1.record(s)
                e1.synchronize()
                ms += e0.elapsed_time(e1)
        else:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            for _ in range(K):
                run.step()
            e1.record(s)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
    barrier(world)
    ms = max_over_ranks(ms, world)
    isa.spin_set_kernel_timing(run.st, False)
    stages = isa.spin_kernel_times(run.st)
    status, word = isa.spin_get_error(run.st)
    if status != 0:
        raise RuntimeError(f"device error word {word:#x} during the timed region")
    kept, _ = run.kept_slots(run.t - 1)
    ms_step = ms / K
    rows_step = Q * R
    peak, peak_kind = peaks()
    fused = R == 1
    per_slot = score_bytes_per_slot(R, fused, wl.key_fp8, wl.d, args.pooling == "max" and wl.b >= 32)
    key_slot = (wl.d + 4) if wl.key_fp8 else 4 * wl.d
    score_ms, score_n = stages["score"]
    score_avg = score_ms / max(score_n, 1)
    per_launch = kept / Ly * per_slot
    achieved = per_launch / (score_avg / 1e3) / 1e9
    # the MTP plan with a capture: four rows of 64 heads, FP8 keys, EMA deferred
    plan = "deferred-r4" if (R == 4 and wl.key_fp8 and wl.H == 64 and wl.d == 128) else None
    traffic_slot = score_traffic_per_slot(plan) if plan else None
    out = {
        "metric": METRIC, "value": job_rows_per_s(rows_step * K, world, ms),
        "unit": "rows/s" if Ly == 1 else f"rows/s (a row passes all {Ly} layers)",
        "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3xe4m3->f32 (selection f32, exact)" if wl.key_fp8 else "f32",
        "data": "synthetic",
        "config": {"workload": wl.name, "requests_per_gpu": Q, "layers": Ly, "rows": R,
                   "pooling": args.pooling, "mtp_policy": args.mtp_policy if R > 1 else None,
                   "context_slots": [min(wl.ctx0), max(wl.ctx0)], "block_size": wl.b, "heads": wl.H,
                   "head_dim": wl.d, "topk": wl.topk, "target_sparsity": wl.sparsity, "gamma": wl.gamma,
                   "parallelism": f"dp{world} (requests sharded, no collective)",
                   "l2": "flushed before every timed step (inputs L2-resident)" if flush
                   else f"inputs larger than L2: {input_bytes / 1e9:.2f} GB of keys"},
        "index_key_gbs": kept * key_slot / (ms_step / 1e3) / 1e9,
        "key_roofline_frac": kept * key_slot / (ms_step / 1e3) / 1e9 / peak,
        "roofline": {"bound": "hbm", "kernel": ("k_score_tc" if wl.key_fp8 else "k_score_simt"),
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": f"{peak_kind} hbm_gbs", "avg_launch_ms": score_avg,
                     "bytes_per_launch": per_launch, "bytes_per_kept_slot": per_slot,
                     "traffic": None if traffic_slot is None else traffic_slot * kept / Ly,
                     "traffic_source": (f"ncu dram__bytes_read.sum + dram__bytes_write.sum per kept slot "
                                        f"({plan} capture, scaled by kept slots)" if traffic_slot is not None
                                        else "null: no capture of this launch plan on the current kernel source")},
        "pipelined": bool(run.lookahead and R == 1 and wl.key_fp8),
        "layers_prepared_at_once": bool(run.prepare),
        "stage_ms_per_step": {k: v[0] / K for k, v in stages.items() if v[1]},
        "gpu_launches": sum(n for _, n in stages.values()),
        "clocks": clk.summary(),
    }
    if alloc:
        out["config"]["per_layer_budget"] = alloc
    miss_all, realized = [], []
    for _ in range(fid_steps):
        run.step()
        miss_all += [x for m in run.miss() for x in m]
        realized += run.kept_slots(run.t - 1)[1]
    v = np.sort(np.array(miss_all))
    out["fidelity"] = {"mean_miss": float(v.mean()),
                       "p99_miss": float(v[max(int(np.ceil(0.99 * v.size)), 1) - 1]),
                       "realized_sparsity": float(np.mean(realized)), "rows": int(v.size)}
    status, word = isa.spin_get_error(run.st)
    if status != 0:
        raise RuntimeError(f"device error word {word:#x}")
    return out


# ---------------------------------------------------------------------------
# Block-pooling ablation (SPIN listing, Figure 3 compares Mean and Top-4 with
# Max pooling by their P99 miss)
# ---------------------------------------------------------------------------
def pooling_ablation(args, world, rank, local):
    """The serving workload (args.requests requests at 512K) run three times,
    once per pooling, through the same target sparsities in rising order:
    after a bootstrap and W warm-up steps at each sparsity, mean / p99 miss
    and realized sparsity over 4 steps (shadow full indexer), then K timed
    steps.  One JSON line."""
    import indexer_sparse_attention_b200 as isa
    from indexer_sparse_attention_b200 import build
    if rank == 0 or world == 1:
        build.build()
    barrier(world)
    isa.load()
    device = torch.device("cuda", local if world > 1 else 0)
    sparsities = (0.5, 0.8, 0.9)
    W, K, F = max(args.warmup, 3), args.steps, 4
    total = 1 + len(sparsities) * (W + F + K) + 2
    wl = rank_workload(rank, args.requests, total + 8)
    run = SpinRun(wl, device, total, 0)
    results = {}
    for name, pooling in POOLINGS.items():
        cfg = run.cfg
        cfg.pooling = pooling
        run.st = isa.SpinState(cfg, device=device)
        run.t = 0
        run.set_sparsity(0.0)
        run.step()
        per = {}
        for s in sparsities:
            run.set_sparsity(s)
            for _ in range(W):
                run.step()
            fid = fidelity(run, n_steps=F)
            ms = timed_steps(run, K, world) / K
            per[str(s)] = {"mean_miss": fid["mean_miss"], "p99_miss": fid["p99_miss"],
                           "realized_sparsity": fid["realized_sparsity"], "ms_per_step": ms}
        status, word = isa.spin_get_error(run.st)
        if status != 0:
            raise RuntimeError(f"device error word {word:#x}")
        results[name] = per
    rel = {}
    for name in ("mean", "top4"):
        rel[name] = {}
        for s in sparsities:
            base = results["max"][str(s)]["p99_miss"]
            v = results[name][str(s)]["p99_miss"]
            rel[name][str(s)] = None if base == 0 else (v - base) / base
    return {"ablation": "block pooling: max (the method's) vs mean and top-4", "unit": "miss fraction / ms",
            "config": {"workload": wl.name, "requests_per_gpu": wl.requests, "context_slots": wl.ctx0[0],
                       "gamma": wl.gamma, "warmup_steps_per_sparsity": W, "fidelity_steps": F, "timed_steps": K},
            "results": results, "p99_change_vs_max": rel,
            "note": "relative change is null where max pooling misses nothing"}


# ---------------------------------------------------------------------------
# MTP policy ablation (SPIN listing, Figure 2: p99 miss against realized block
# sparsity, one point per target sparsity and policy, draft length three)
# ---------------------------------------------------------------------------
def mtp_ablation(args, world, rank, local):
    """The 4-row MTP workload (32 requests at 128K) run once per policy on the
    same inputs and accepted lengths, through the same target sparsities in
    rising order: after a bootstrap and W warm-up steps at each sparsity, the
    miss of every (request, row) and of the accepted rows alone, and realized
    sparsity, over F steps (shadow full indexer), then K timed steps.  One
    JSON line."""
    import indexer_sparse_attention_b200 as isa
    from indexer_sparse_attention_b200 import build
    if rank == 0 or world == 1:
        build.build()
    barrier(world)
    isa.load()
    device = torch.device("cuda", local if world > 1 else 0)
    sparsities = (0.4, 0.5, 0.6, 0.7, 0.8)
    W, K, F = max(args.warmup, 3), args.steps, 4
    total = 1 + len(sparsities) * (W + F + K) + 2
    base = workloads.config(WORKLOADS["mtp-32x128K-r4"])
    wl = workloads.config(WORKLOADS["mtp-32x128K-r4"], seed=base.seed + 1000 * rank, steps=total,
                          spare_slots=base.rows * 4)
    run = WorkloadRun(wl, device, total)
    Q, R = wl.requests, wl.rows
    s_ev = torch.cuda.current_stream()
    results = {}
    for name, pol in MTP_POLICIES.items():
        run.restart(mtp_policy=pol)
        run.set_sparsity([0.0])
        run.step()
        per = {}
        for sp in sparsities:
            run.set_sparsity([sp])
            for _ in range(W):
                run.step()
            miss_all, miss_acc, realized = [], [], []
            for _ in range(F):
                run.step()
                m = np.array(run.miss()[0]).reshape(Q, R)
                acc = run.acc[run.t - 1].cpu().numpy()
                miss_all += m.flatten().tolist()
                miss_acc += [m[q, r] for q in range(Q) for r in range(int(acc[q]))]
                realized += run.kept_slots(run.t - 1)[1]
            barrier(world)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s_ev)
            for _ in range(K):
                run.step()
            e1.record(s_ev)
            torch.cuda.synchronize()
            barrier(world)
            ms = max_over_ranks(e0.elapsed_time(e1), world) / K
            per[str(sp)] = {"p99_miss": p99_of(miss_all), "mean_miss": float(np.mean(miss_all)),
                            "p99_miss_accepted_rows": p99_of(miss_acc),
                            "realized_sparsity": float(np.mean(realized)), "ms_per_step": ms}
        status, word = isa.spin_get_error(run.st)
        if status != 0:
            raise RuntimeError(f"device error word {word:#x}")
        results[name] = per
    rel = {}
    for sp in sparsities:
        base_p99 = results["row0"][str(sp)]["p99_miss"]
        v = results["union-prefix"][str(sp)]["p99_miss"]
        rel[str(sp)] = None if base_p99 == 0 else (v - base_p99) / base_p99
    return {"ablation": "MTP policy: row-local union + prefix-valid update (the method's) vs row-0 sharing + "
                        "row-0 update", "unit": "miss fraction / ms",
            "config": {"workload": wl.name, "requests_per_gpu": Q, "rows": R, "context_slots": wl.ctx0[0],
                       "gamma": wl.gamma, "accept_probs": list(wl.accept_probs),
                       "warmup_steps_per_sparsity": W, "fidelity_steps": F, "timed_steps": K},
            "results": results, "p99_change_union_vs_row0": rel,
            "note": "miss over every (request, row) of the fidelity steps; accepted lengths drawn from the "
                    "workload's distribution, the same for both policies"}


# ---------------------------------------------------------------------------
# Predictor-quality profile (SPIN listing, Table 1: Pearson correlation and
# top-k recall per predictor, averaged over layers and decode iterations)
# ---------------------------------------------------------------------------
def predictor_profile(args, world, rank, local):
    """An 8-layer workload with two prompts of Table 1's lengths (94K and
    9.7K slots) decoded with every block kept.  Before each step of each
    layer, four predictors of that step's indexer scores are taken: the
    random baseline, the previous layer's scores of the same step, the
    previous step's scores of the same layer, and SPIN's z = max(V, D).  Per
    prompt, the Pearson correlation and the top-k recall of each, averaged
    over layers and steps 1..T.  Every figure comes from the library's
    kernels.  One JSON line."""
    import indexer_sparse_attention_b200 as isa
    from indexer_sparse_attention_b200 import build
    if rank == 0 or world == 1:
        build.build()
    barrier(world)
    isa.load()
    device = torch.device("cuda", local if world > 1 else 0)
    T = max(args.steps, 2)
    total = T + 1
    base = workloads.config(WORKLOADS["ragged-8Lx8-256K-1M"])
    wl = workloads.config(WORKLOADS["ragged-8Lx8-256K-1M"], requests=2, ctx0=(94_000, 9_700), steps=total,
                          seed=base.seed + 1000 * rank, spare_slots=8)
    run = WorkloadRun(wl, device, total)
    run.set_lookahead(args.lookahead)   # applies to one-row steps
    Ly, Q, R = wl.layers, wl.requests, wl.rows
    st = run.st
    run.set_sparsity([0.0] * Ly)
    allk = torch.ones_like(run.masks[0])
    names = ("random", "prev_layer", "prev_iter", "spin_ema")
    corr = {n: [[] for _ in range(Q)] for n in names}
    recall = {n: [[] for _ in range(Q)] for n in names}
    r_out = torch.zeros((Q, R), dtype=torch.float64, device=device)
    ov = torch.zeros((Q, R), dtype=torch.int32, device=device)
    ptop = torch.empty((Q, R, wl.topk), dtype=torch.int32, device=device)
    prev = [None] * Ly
    for t in range(total):
        cur = [None] * Ly
        ctx = run.ctx[t]
        vis = (ctx.long() + R - 1).clamp(max=wl.topk).cpu().numpy()     # k entries a top-k can hold
        for l in range(Ly):
            preds = {}
            if t >= 1:
                preds["spin_ema"] = st.new_scores()
                isa.spin_slot_prediction(st, l, R, isa.SPIN_PRED_EMA, t, ctx, preds["spin_ema"])
                preds["random"] = st.new_scores()
                isa.spin_slot_prediction(st, l, R, isa.SPIN_PRED_RANDOM, t, ctx, preds["random"])
                preds["prev_iter"] = prev[l]
                if l > 0:
                    preds["prev_layer"] = cur[l - 1]
            sc = st.new_scores()
            sc.fill_(float("-inf"))
            c = run.caches[l]
            q, w = run.qw[t][l]
            isa.spin_decode_step(st, l, R, t, c.keys, c.kscale if wl.key_fp8 else None, c.block_table, q, w, ctx,
                                 False, run.masks[l], run.topks[l], sc)
            for n, pred in preds.items():
                isa.spin_pearson(st, R, pred, sc, ctx, r_out)
                isa.spin_topk(st, R, pred, allk, ctx, ptop)
                isa.spin_topk_overlap(st, R, ptop, run.topks[l], ov)
                rr, oo = r_out.cpu().numpy(), ov.cpu().numpy()
                for qq in range(Q):
                    corr[n][qq].append(float(rr[qq, 0]))
                    recall[n][qq].append(float(oo[qq, 0]) / float(vis[qq]))
            cur[l] = sc
        prev = cur
    status, word = isa.spin_get_error(st)
    if status != 0:
        raise RuntimeError(f"device error word {word:#x}")
    prompts = {}
    for qq, L in enumerate(wl.ctx0):
        prompts[f"{L // 1000}K"] = {n: {"pearson": float(np.mean(corr[n][qq])), "topk_recall": float(np.mean(recall[n][qq])),
                                        "samples": len(corr[n][qq])} for n in names}
    return {"ablation": "predictor quality: Pearson correlation and top-k recall of the indexer scores",
            "unit": "correlation / recall", "config": {"layers": Ly, "prompts_slots": list(wl.ctx0), "steps": T,
                                                       "topk": wl.topk, "alpha": wl.alpha, "sparsity": 0.0},
            "results": prompts,
            "note": "synthetic keys: each layer draws its own keys, planted directions and vertical slots; "
                    "the layers share only the position pattern of the diagonal band"}


def p99_of(values):
    v = np.sort(np.asarray(values, np.float64))
    return float(v[max(int(np.ceil(0.99 * v.size)), 1) - 1]) if v.size else 0.0


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------
class OracleSample:
    """One request of the serving workload on the host, driven by the oracle
    (fp64 scores, OpenMP over blocks)."""

    def __init__(self, request_seed_offset=0):
        import oracle
        self.o = oracle
        self.o.build()
        wl = workloads.config(2, requests=1, ctx0=(512 * 1024,), steps=64, seed=2 + request_seed_offset)
        self.wl = wl
        cache = workloads.make_key_cache(wl, 0, "cpu")
        self.keys = cache.keys.numpy()
        self.ks = cache.kscale.numpy()
        self.bt = cache.block_table[0].numpy()
        q, w = workloads.make_queries(wl, 0, wl.steps, "cpu")
        self.q = q.float().numpy().astype(np.float64)
        self.w = w.numpy()
        nb = wl.max_blocks
        self.V = np.full(nb * wl.b, np.inf, np.float32)
        self.D = np.full(nb * wl.b, -np.inf, np.float32)
        self.t = 0

    def step(self, sparsity):
        wl = self.wl
        t = self.t % wl.steps
        ctx = wl.ctx0[0] + t + 1
        self.o.decode_step_request(V=self.V, D=self.D, ctx_len=ctx, rows=1, b=wl.b, sparsity=sparsity,
                                   gamma=wl.gamma, alpha=wl.alpha, seed=wl.seed, request=0, layer=0, step=self.t,
                                   topk=wl.topk, q=self.q[0, t:t + 1], w=self.w[0, t:t + 1], keys=self.keys,
                                   kscale=self.ks, block_table=self.bt, key_fp8=True)
        self.t += 1


def threads_used():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def cpu_baseline(sparsity, seconds):
    smp = OracleSample()
    smp.step(0.0)                      # history bootstrap (not timed)
    n, t0 = 0, time.perf_counter()
    while n < 2 or time.perf_counter() - t0 < seconds:
        smp.step(sparsity)
        n += 1
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": "rows/s", "cores": threads_used(), "kind": "oracle",
            "sample": f"{n} decode steps of 1 of the 96 requests (512K context, {int(sparsity * 100)}% sparsity) "
                      f"after an untimed all-keep bootstrap; fp64 scores, OpenMP over blocks; {dt:.1f} s"}


def step_traffic(context_slots, kept_slots, ms_step, peak, pooling="max"):
    """The whole step's algorithmic bytes against the measured copy bandwidth:
    per slot of context, what the predict kernel reads (max pooling: D and
    V's maximum per 32 slots, 4.125 B; otherwise V and D, 8 B), plus the score
    kernel's bytes per kept slot (key, scale, score, EMA read and write)."""
    ctx_b = 4 + 4 / 32 if pooling == "max" else 8
    kept_b = score_bytes_per_slot(1, True, True, 128, pooling == "max")
    b = ctx_b * context_slots + kept_b * kept_slots
    gbs = b / (ms_step / 1e3) / 1e9
    return {"bytes_per_step": b, "gbs": gbs, "frac": gbs / peak,
            "note": f"{ctx_b:g} B per slot of context + {kept_b:g} B per kept slot; the floor of a step"}


def headline_config(wl, Q, args, world):
    """The serving workload's config, the same in both arms."""
    return {"workload": wl.name, "requests_per_gpu": Q, "context_slots": wl.ctx0[0], "block_size": wl.b,
            "heads": wl.H, "head_dim": wl.d, "topk": wl.topk, "target_sparsity": args.sparsity,
            "gamma": wl.gamma, "pooling": args.pooling,
            "parallelism": f"dp{world} (requests sharded, no collective)",
            "l2": "inputs larger than L2: 6.4 GB paged FP8 key cache and 0.4 GB EMA state per GPU"}


def reference_arm(args, world, rank):
    if rank != 0:
        return None
    smp = OracleSample()
    smp.step(0.0)
    for _ in range(args.warmup):
        smp.step(args.sparsity)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        smp.step(args.sparsity)
    dt = time.perf_counter() - t0
    value = args.steps / dt
    wl = workloads.config(2)
    return {"metric": METRIC, "value": value, "unit": "rows/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": headline_config(wl, wl.requests, args, world),
            "cpu_baseline": {"value": value, "unit": "rows/s", "cores": threads_used(), "kind": "oracle",
                             "sample": f"each step one request of the 96 at 512K on the host cores: "
                                       f"{args.steps} timed steps after {args.warmup} warm-up steps"},
            "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        out = reference_arm(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    world, rank, local = dist_setup()
    try:
        if args.ablation in ("pooling", "mtp", "predictors"):
            fn = {"pooling": pooling_ablation, "mtp": mtp_ablation, "predictors": predictor_profile}[args.ablation]
            out = fn(args, world, rank, local)
            if rank == 0:
                print(json.dumps(out), flush=True)
            return
        if args.workload != "serve-96x512K":
            out = workload_arm(args, world, rank, local)
            if rank == 0:
                print(json.dumps(out), flush=True)
            return
        out = gpu_arm(args, world, rank, local)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline(args.sparsity, args.cpu_seconds)
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
