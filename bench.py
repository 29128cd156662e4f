#!/usr/bin/env python
"""Benchmark of the diffusion-LM noising-plus-loss hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
dlm_sample_t -> dlm_corrupt -> dlm_loss_fwd_bwd (fused forward + backward,
bf16 dlogits for every row), all through the C ABI of libdlm.so.

Default (the workload "suite"): the headline is the DiffusionGemma-like
uniform-noise loss, B=4, prefix 512 + canvas 1024, V=262,144 -- canvas CE
plus the encoder's causal CE, every row scored, 10.7 GB of logits read and
gradients written per step, the largest of the logits workloads.  The same
JSON line then carries, under "workloads", the LLaDA-like absorbing loss
(B=1 L=4096 V=126,464), the Dream-like shifted loss (B=8 L=2048 V=152,064)
and the fused-head loss on packed documents (T=16,384, D=4,096, V=126,464),
each timed the same way with its own clocks, roofline and end-to-end leg.
Inputs are larger than L2 in every workload, so no flush between steps is
needed.  Each timed step draws a new t (seed = 1000 + step), so the scored
rows vary like in training.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]
  python bench.py --workload abs_b1_l4096_v126464          # one workload alone
  python bench.py --workload lin_unif_b4_p512_c1024_d4096_v262144   # fused head, uniform

Besides the device-timed value, rank 0 at N=1 reports the CPU oracle on a
bounded sample of the same workload (all cores and one thread), and the same
metric end to end with each step's inputs copied from pinned host memory
(the logits workloads at every N, the fused-head workloads at N=1).

Multi-GPU: replicas only (the path has no data exchange); every rank runs the
same workload on its own GPU, timing is the max over ranks, value = scored
tokens of all ranks / that time ("scaling": "weak").

Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "diffusion-loss fwd+bwd scored tokens/s; achieved HBM GB/s vs B200 peak"
UNIT = "scored tokens/s"
SUITE = "suite"
SUITE_HEADLINE = "unif_b4_p512_c1024_v262144"
SUITE_OTHERS = ("abs_b1_l4096_v126464", "shift_b8_l2048_v152064", "lin_t16384_d4096_v126464",
                "dec_s128_k26_v126464")
DEFAULT_WORKLOAD = SUITE
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
CE_SOURCE = os.path.join(ROOT, "diffusion_lm_loss_b200", "csrc", "dlm_ce.cu")
DEC_SOURCE = os.path.join(ROOT, "diffusion_lm_loss_b200", "csrc", "dlm_decision.cu")
ABSORBING, UNIFORM = 0, 1          # noise modes, as numbered in include/dlm.h


def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def profile_traffic_ratio(name: str, source: str):
    """DRAM bytes / algorithmic bytes of a kernel from its committed ncu
    summary (profiles/<name>.md), or None when there is none or the kernel's
    source file changed since the capture."""
    try:
        txt = open(os.path.join(ROOT, "profiles", f"{name}.md")).read()
    except OSError:
        return None
    m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", txt)
    m_r = re.search(r"traffic_over_algorithmic:\s*([0-9.]+)", txt)
    if not (m_sha and m_r):
        return None
    sha = hashlib.sha256(open(source, "rb").read()).hexdigest()
    return float(m_r.group(1)) if sha == m_sha.group(1) else None


def ce_traffic_ratio(workload: str):
    """The CE kernel's ratio on `workload` (profiles/ce_stream_<workload>.md)."""
    return profile_traffic_ratio(f"ce_stream_{workload}", CE_SOURCE)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock, power and clock-event reasons sampled every few milliseconds
    by a background thread through NVML while the timed steps run (a timed
    region of a few tens of milliseconds still gets samples); falls back to
    `nvidia-smi -lms 50` when NVML is unavailable."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, gpu_index, device=None, period_s: float = 0.002):
        self.gpu = gpu_index
        self.device = device
        self.period = period_s
        self.proc = None
        self.thread = None
        self.samples = []
        self.t0 = self.t1 = None
        self.nvml = None

    def _nvml_handle(self):
        import pynvml
        import torch

        pynvml.nvmlInit()
        if self.device is not None:
            try:
                uuid = str(torch.cuda.get_device_properties(self.device).uuid)
                return pynvml, pynvml.nvmlDeviceGetHandleByUUID("GPU-" + uuid)
            except Exception:
                pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(int(self.gpu))

    def start(self):
        import threading

        try:
            nv, h = self._nvml_handle()
            self.nvml = (nv, h)
            self.sm_max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception:
            self.nvml = None
        if self.nvml is None:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu=timestamp,{self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "50"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except Exception:
                self.proc = None
            return
        self.stop_flag = threading.Event()

        def loop():
            nv, h = self.nvml
            while not self.stop_flag.is_set():
                try:
                    t = time.perf_counter()
                    sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                    pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                    self.samples.append((t, sm, rs, pw))
                except Exception:
                    pass
                time.sleep(self.period)

        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    def mark_begin(self):
        self.t0 = datetime.datetime.now()
        self.p0 = time.perf_counter()

    def mark_end(self):
        self.t1 = datetime.datetime.now()
        self.p1 = time.perf_counter()

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            inside = [s for s in self.samples if self.p0 <= s[0] <= self.p1]
            use = inside or self.samples[len(self.samples) // 2:len(self.samples) // 2 + 1]
            if not use:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "source": "nvml"}
            reasons = sorted({n for _, _, rs, _ in use for n, bit in self.REASONS if rs & bit})
            return {"sm_mhz": statistics.median(s[1] for s in use), "sm_max_mhz": self.sm_max,
                    "reasons": reasons, "power_w_max": max(s[3] for s in use), "samples": len(use),
                    "samples_in_timed_region": len(inside), "source": "nvml, every 2 ms"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f")
            except ValueError:
                continue
            rows.append((ts, f))
        inside = [r for r in rows if self.t0 and self.t1 and self.t0 <= r[0] <= self.t1]
        use = inside or rows[len(rows) // 2:len(rows) // 2 + 1]
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1][2]) for r in use if r[1][2].replace(".", "").isdigit()]
        smax = [float(r[1][3]) for r in use if r[1][3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for _, f in use:
            for n, v in zip(names, f[6:10]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(use),
                "samples_in_timed_region": len(inside), "source": "nvidia-smi, every 50 ms"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def reduce_over_ranks(ms: float, loss_ms: float, scored: float, device):
    """Whole-job numbers: the slowest rank's times (max) and the scored
    tokens of all ranks (sum).  Plumbing only (a few scalars); no-op on one
    rank."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([ms, loss_ms], dtype=torch.float64, device=device)
    n = torch.tensor([scored], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return float(t[0]), float(t[1]), float(n[0])


def algorithmic_ce_bytes(rows: int, scored: int, vocab: int) -> int:
    """Bytes the weighted-CE fwd+bwd must move per launch: each scored row is
    read once (2V) and every row's bf16 gradient written once (2V); plus the
    row list (16 B) read and the per-row loss (4 B) written."""
    return 2 * vocab * scored + 2 * vocab * rows + 20 * rows


def run_ours(args):
    """Our arm.  The default workload "suite" times the headline workload
    (the DiffusionGemma-like uniform loss, the largest logits workload) and
    then, each in the same way with its own clocks, roofline and end-to-end
    leg, the LLaDA-like, the Dream-like and the fused-head workloads; rank 0
    prints one JSON line, the headline at top level and the others under
    "workloads"."""
    import torch
    import torch.distributed as dist

    import dlm_inputs as di

    rank, local_rank, world = env_rank()
    if args.gpus != world:
        if world == 1 and args.gpus > 1:
            raise SystemExit("--gpus N>1 must be launched with torch.distributed.run (one rank per GPU)")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    keys = [SUITE_HEADLINE, *SUITE_OTHERS] if args.workload == SUITE else [args.workload]
    recs = []
    for i, key in enumerate(keys):
        spec = di.WORKLOADS[key]
        if args.slots and spec.kind == "decision":
            # the same recipe on another number of label slots
            spec = spec.scaled(key=key.replace(f"_s{spec.n_units}_", f"_s{args.slots}_"), n_units=args.slots,
                               description=spec.description.replace(
                                   f"{spec.n_units} label slots (16 canvases x 8 questions)",
                                   f"{args.slots} label slots"))
        run = {"linear": run_linear, "decision": run_decision}.get(spec.kind, run_logits)
        if i == 0 or world > 1:
            recs.append(run(args, spec, dev, rank, world, headline=(i == 0)))
        else:
            # one GPU: a failing sub-record is recorded and the line still prints
            try:
                recs.append(run(args, spec, dev, rank, world, headline=False))
            except Exception as ex:
                recs.append({"config": {"workload": key}, "value": None,
                             "error": f"{type(ex).__name__}: {ex}"[:300]})
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    res = recs[0]
    if len(recs) > 1:
        res["config"]["suite"] = ("headline: the largest logits workload; the other workloads of the suite "
                                  "under \"workloads\", each timed the same way")
        res["workloads"] = {r["config"]["workload"]: {k: v for k, v in r.items()
                                                      if k not in ("metric", "higher_is_better", "scaling",
                                                                   "vs_baseline", "data", "n_gpus")}
                            for r in recs[1:]}
    print(json.dumps(res), flush=True)


def run_logits(args, spec, dev, rank, world, headline=True):
    """One logits workload: time draw, corruption, weighted CE forward +
    backward through dlm_loss_fwd_bwd; returns the record of its JSON line."""
    import torch
    import torch.distributed as dist

    import dlm_inputs as di
    import diffusion_lm_loss_b200 as dlm

    local_rank = dev.index
    case = di.make_case(spec, dev, seed=spec.data_seed + rank)
    V = spec.vocab
    mode, align = spec.mode, spec.align
    B = spec.n_units
    uniform = mode == di.UNIFORM
    lay = dlm.make_layout(B, spec.seq_len)
    enc_lay = dlm.make_layout(B, spec.prefix + spec.seq_len) if uniform else None
    out = None
    # uniform noise, --objective rhine: DiffusionGemma's Rhine objectives --
    # 1/(1-t) time weighting capped at 10 (the pages give no default cap) and
    # the per-example mean
    if args.objective == "rhine" and not uniform:
        raise SystemExit("--objective rhine applies to uniform-noise workloads")
    options = (dlm.LossOptions(dlm.TIME_WEIGHT_INV_ONE_MINUS_T, 10.0, dlm.REDUCE_EXAMPLE_MEAN)
               if args.objective == "rhine" else None)
    # --keep-unscored: the secondary figure -- unscored rows of dlogits are not
    # written by the call; the step zeroes the buffer before the call, outside
    # the call's own events (the roofline counts the call's bytes only)
    if args.keep_unscored:
        options = options or dlm.LossOptions()
        options.keep_unscored_rows = 1

    def step(seed, logits, clean, enc_logits=None, enc_clean=None, ev=None):
        nonlocal out
        t, p = dlm.sample_t(seed, B, mode, spec.eps)
        _, corr = dlm.corrupt(lay, clean, p, mode, spec.mask_id, V, seed)
        if args.keep_unscored and out is not None:
            out.dlogits.zero_()
            if out.enc_dlogits is not None:
                out.enc_dlogits.zero_()
        if ev is not None:
            ev[0].record()
        out = dlm.loss_fwd_bwd(lay, logits, V, clean, corr, p, mode, align,
                               enc_layout=enc_lay, enc_logits=enc_logits, enc_ids=enc_clean,
                               enc_ar_weight=spec.enc_ar_weight, out=out, options=options)
        if ev is not None:
            ev[1].record()
        return corr

    K, W = args.steps, args.warmup
    for i in range(W):
        step(10 + i, case.logits, case.clean, case.enc_logits, case.enc_clean)
    torch.cuda.synchronize()

    vis = [v for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    clocks = ClockSampler(vis[local_rank] if local_rank < len(vis) else local_rank, device=dev)
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    loss_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark_begin()
    t_start.record()
    for i in range(K):
        step(1000 + i, case.logits, case.clean, case.enc_logits, case.enc_clean, ev=loss_ev[i])
    t_end.record()
    torch.cuda.synchronize()
    clocks.mark_end()
    if world > 1:
        dist.barrier()
    ms = t_start.elapsed_time(t_end)
    loss_ms = sum(a.elapsed_time(b) for a, b in loss_ev) / K
    clk = clocks.stop() if rank == 0 else None

    # scored rows of the timed steps (recomputed outside the timed region)
    scored = 0
    rows = case.n_tokens + (B * (spec.prefix + spec.seq_len) if uniform else 0)
    if uniform:
        enc_pairs = B * (spec.prefix + spec.seq_len - 1)
        scored = K * (case.n_tokens + enc_pairs) if align == di.ALIGNED else None
    if not uniform or scored is None:
        tot = torch.zeros((), dtype=torch.int64, device=dev)
        for i in range(K):
            t, p = dlm.sample_t(1000 + i, B, mode, spec.eps)
            _, corr = dlm.corrupt(lay, case.clean, p, mode, spec.mask_id, V, 1000 + i)
            if align == di.SHIFTED:
                c = corr.view(B, spec.seq_len)[:, 1:]
                tot += c.sum()
            else:
                tot += corr.sum(dtype=torch.int64)
        scored = int(tot.item())

    ms, loss_ms, scored_all = reduce_over_ranks(ms, loss_ms, scored, dev)
    value = scored_all / (ms / 1e3)

    # e2e: inputs from pinned host memory, H2D + step + D2H of the loss
    e2e = None
    if not args.no_e2e:
        Ke = max(1, min(K, args.e2e_steps))
        h_logits = case.logits.cpu().pin_memory()
        h_clean = case.clean.cpu().pin_memory()
        h_enc_logits = case.enc_logits.cpu().pin_memory() if uniform else None
        h_enc_clean = case.enc_clean.cpu().pin_memory() if uniform else None
        d_logits = torch.empty_like(case.logits)
        d_clean = torch.empty_like(case.clean)
        d_enc_logits = torch.empty_like(case.enc_logits) if uniform else None
        d_enc_clean = torch.empty_like(case.enc_clean) if uniform else None
        h_loss = torch.empty(Ke, dtype=torch.float32).pin_memory()
        h2d = h_logits.numel() * 2 + h_clean.numel() * 4
        if uniform:
            h2d += h_enc_logits.numel() * 2 + h_enc_clean.numel() * 4
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)

        def e2e_step(i):
            d_logits.copy_(h_logits, non_blocking=True)
            d_clean.copy_(h_clean, non_blocking=True)
            if uniform:
                d_enc_logits.copy_(h_enc_logits, non_blocking=True)
                d_enc_clean.copy_(h_enc_clean, non_blocking=True)
            step(1000 + i, d_logits, d_clean, d_enc_logits, d_enc_clean)
            h_loss[i:i + 1].copy_(out.loss, non_blocking=True)

        e2e_step(0)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s0.record()
        for i in range(Ke):
            e2e_step(i)
        s1.record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e_ms = torch.tensor([s0.elapsed_time(s1)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(e_ms, op=dist.ReduceOp.MAX)
        # the same seeds as the first Ke timed steps: scored rows in proportion
        e2e_val = scored_all * (Ke / K) / (float(e_ms[0]) / 1e3)
        e2e = {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 4,
               "steps": Ke, "ms_per_step": float(e_ms[0]) / Ke}
        del d_logits, h_logits

    hbm, _, peak_kind = peaks()
    alg_bytes = algorithmic_ce_bytes(rows, scored / K if world == 1 else scored_all / world / K, V)
    if args.keep_unscored:
        # no write for unscored rows: 2V read + 2V write per scored row, 20 B per row
        n_sc = scored / K if world == 1 else scored_all / world / K
        alg_bytes = 4.0 * V * n_sc + 20.0 * rows
    achieved = alg_bytes / (loss_ms / 1e3) / 1e9
    ratio = ce_traffic_ratio(spec.key)
    roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm,
            # the profiled traffic ratio belongs to the default (zero-writing) call
            "traffic": (ratio * alg_bytes) if (ratio and not args.keep_unscored) else None,
            "kernel": "k_ce_stream (timed as the whole dlm_loss_fwd_bwd call: plan + CE + reduce)",
            "algorithmic_bytes_per_launch": alg_bytes, "launch_ms": loss_ms,
            "peak_source": f"{peak_kind} hbm_gbs (copy bandwidth)",
            "frac_of_8TBps": achieved / 8000.0}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(spec) if headline else cpu_baseline(spec, budget_s=4.0, single_thread_s=0)
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": spec.key, "description": spec.description, "global_batch": B * world,
                   "seq_len": spec.seq_len, "vocab": V, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (logits %.2f GB per replica)" % (case.logits.numel() * 2 / 1e9),
                   "scored_tokens": scored_all, "seeds": "t/corruption seed 1000+step",
                   "objective": ("rhine: 1/(1-t) capped at 10, per-example mean" if args.objective == "rhine"
                                 else "plain"),
                   "unscored_rows": ("not written (buffer zeroed before each call, outside the call's events)"
                                     if args.keep_unscored else "written as zeros")},
        "roofline": roof, "cpu_baseline": cpu, "clocks": clk, "e2e": e2e,
        "gpu_launches": 5 * K,
    }
    return res


def run_linear(args, spec, dev, rank, world, headline=True):
    """The fused lm_head workload: time draw, corruption, and the loss from
    hidden states and the head (dlm_linear_loss_fwd_bwd, dH and dW; uniform
    workloads: dlm_linear_loss_uniform_fwd_bwd, canvas and encoder hidden
    states against one head, dH, dH_enc and dW)."""
    import torch
    import torch.distributed as dist

    import dlm_inputs as di
    import diffusion_lm_loss_b200 as dlm

    case = di.make_case(spec, dev, seed=spec.data_seed + rank)
    T, D, V = case.n_tokens, spec.d_model, spec.vocab
    out = None
    align = dlm.SHIFTED if args.align == "shifted" else dlm.ALIGNED
    uniform = spec.mode == dlm.UNIFORM
    if uniform:
        B, C, P = case.n_units, case.seq_len, spec.prefix
        lay = dlm.make_layout(B, C)
        enc = dlm.make_layout(B, P + C)
        T = B * C + B * (P + C)
    else:
        lay = dlm.make_layout(case.n_units, 0, case.cu_seqlens, None, n_tokens=T)

    def step(seed, ev=None):
        nonlocal out
        t, p = dlm.sample_t(seed, case.n_units, spec.mode, spec.eps)
        _, corr = dlm.corrupt(lay, case.clean, p, spec.mode, spec.mask_id, V, seed)
        if ev is not None:
            ev[0].record()
        if uniform:
            out = dlm.linear_loss_uniform_fwd_bwd(lay, case.hidden, case.weight, case.clean, enc, case.enc_hidden,
                                                  case.enc_clean, enc_ar_weight=spec.enc_ar_weight, align=align,
                                                  out=out)
        else:
            out = dlm.linear_loss_fwd_bwd(lay, case.hidden, case.weight, case.clean, corr, p, out=out, align=align)
        if ev is not None:
            ev[1].record()
        return corr

    K, W = args.steps, args.warmup
    for i in range(W):
        step(10 + i)
    torch.cuda.synchronize()
    vis = [v for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    lr = int(os.environ.get("LOCAL_RANK", "0"))
    clocks = ClockSampler(vis[lr] if lr < len(vis) else lr, device=dev)
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark_begin()
    t0.record()
    for i in range(K):
        step(1000 + i, evs[i])
    t1.record()
    torch.cuda.synchronize()
    clocks.mark_end()
    if world > 1:
        dist.barrier()
    ms = t0.elapsed_time(t1)
    call_ms = sum(a.elapsed_time(b) for a, b in evs) / K
    clk = clocks.stop() if rank == 0 else None
    per_step = []
    for i in range(K):
        if uniform:
            # every canvas target (each unit's first token is none when
            # shifted) and every encoder next-token pair
            per_step.append(B * (C - (1 if align == dlm.SHIFTED else 0)) + B * (P + C - 1))
            continue
        t, p = dlm.sample_t(1000 + i, case.n_units, spec.mode, spec.eps)
        _, corr = dlm.corrupt(lay, case.clean, p, spec.mode, spec.mask_id, V, 1000 + i)
        n = int(corr.sum().item())
        if align == dlm.SHIFTED:
            # a document's first token is never a target when rows score the next token
            cu = case.cu_seqlens.to(torch.int64)
            first = cu[:-1][cu[1:] > cu[:-1]]
            n -= int(corr[first].sum().item())
        per_step.append(n)
    scored = sum(per_step)
    ms, call_ms, scored_all = reduce_over_ranks(ms, call_ms, scored, dev)

    # e2e (one GPU): the step's inputs -- hidden states, ids, document
    # offsets -- copied from pinned host memory every step, the loss read back;
    # the head's weight is a resident parameter
    e2e = None
    if world == 1 and not args.no_e2e:
        try:
            e2e = _linear_e2e(args, spec, case, lay, enc if uniform else None, align, per_step, out)
        except Exception as ex:       # the device-timed figures above stand without it
            e2e = {"value": None, "error": f"{type(ex).__name__}: {ex}"[:300]}
    value = scored_all / (ms / 1e3)
    M = scored_all / world / K
    flops = 6.0 * M * D * V
    _, bf16, kind = peaks()
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            sustained = float(json.load(f)["bf16_tflops_sustained"])
    except Exception:
        sustained = 1400.0
    achieved = flops / (call_ms / 1e3) / 1e12
    roof = {"bound": "tensor", "achieved": achieved, "peak": sustained, "unit": "TFLOP/s",
            "frac": achieved / sustained, "traffic": None,
            "kernel": f"k_gemm (the whole {'dlm_linear_loss_uniform_fwd_bwd' if uniform else 'dlm_linear_loss_fwd_bwd'}"
                      " call: 6 GEMMs-worth of algorithmic flops "
                      "6*M*D*V; executed 8*M*D*V with the backward recompute)",
            "algorithmic_flops_per_call": flops, "launch_ms": call_ms,
            "frac_of_burst_peak": achieved / bf16, "peak_source": f"{kind} bf16 sustained (burst in frac_of_burst_peak)"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            cpu = cpu_baseline(spec) if headline else cpu_baseline(spec, budget_s=4.0, single_thread_s=0)
        except Exception as e:      # the GPU figures above stand without it
            cpu = {"value": None, "kind": "oracle", "error": f"{type(e).__name__}: {e}"[:300]}
    res = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
           "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "bf16", "data": "synthetic",
           "config": {"workload": spec.key, "description": spec.description, "align": args.align,
                      "tokens": T, "d_model": D, "encoder_ar_weight": spec.enc_ar_weight if uniform else None,
                      "vocab": V, "documents": case.n_units, "parallelism": f"replicas{world}",
                      "scored_tokens": scored_all, "l2": "inputs larger than L2 (W %.2f GB)" % (V * D * 2 / 1e9)},
           "roofline": roof, "cpu_baseline": cpu, "clocks": clk, "e2e": e2e,
           # per step: time draw, corruption, plan, gather, forward GEMM, lse,
           # dZ + dH + dW per 16,384-column vocabulary chunk, scatter, reduce
           "gpu_launches": K * (6 + 3 * ((V + 16383) // 16384) + 2)}
    return res


def run_decision(args, spec, dev, rank, world, headline=True):
    """The typed-decision workload: dlm_decision_loss_fwd_bwd on the logits
    rows of the label slots.  One call moves ~65 MB, less than the host
    takes to enqueue it from Python, so the timed steps run from a CUDA
    graph (captured once, replayed; the library's kernels run back to back
    with no host gap), and each step reads one of eight input sets in turn
    (8 x 32 MB of logits, larger than L2, so no step finds its input in
    L2)."""
    import torch

    import dlm_inputs as di
    import diffusion_lm_loss_b200 as dlm

    n, V = spec.n_units, spec.vocab
    sets = [di.make_case(spec, dev, seed=spec.data_seed + 101 * j + rank) for j in range(8)]
    e = sets[0].extra
    outs = [None] * len(sets)

    def call(j):
        outs[j] = dlm.decision_loss_fwd_bwd(sets[j].logits, V, sets[j].extra["cand_off"], sets[j].extra["cand_ids"],
                                            sets[j].extra["kind"], sets[j].extra["val"], brier_weight=0.1,
                                            out=outs[j])

    K, W = args.steps, args.warmup
    for i in range(max(W, len(sets))):
        call(i % len(sets))
    torch.cuda.synchronize()
    # every timed call in one graph (the sets in turn, K rounded up to use
    # each set equally): one graph launch for the whole timed region
    K = (K + len(sets) - 1) // len(sets) * len(sets)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(K):
            call(i % len(sets))
    graph.replay()
    torch.cuda.synchronize()
    vis = [v for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    lr = int(os.environ.get("LOCAL_RANK", "0"))
    clocks = ClockSampler(vis[lr] if lr < len(vis) else lr, device=dev)
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.mark_begin()
    t0.record()
    graph.replay()
    t1.record()
    torch.cuda.synchronize()
    clocks.mark_end()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop() if rank == 0 else None
    assert all(o.device_status() == 0 for o in outs)
    ms, call_ms, slots_all = reduce_over_ranks(t0.elapsed_time(t1), t0.elapsed_time(t1) / K, float(n * K), dev)
    value = slots_all / (ms / 1e3)
    del graph
    e2e = None
    if not args.no_e2e:
        Ke = max(1, min(K, args.e2e_steps))
        case = sets[0]
        dev_in = [case.logits, e["cand_off"], e["cand_ids"], e["kind"], e["val"]]
        host_in = [t.cpu().pin_memory() for t in dev_in]
        h_loss = torch.empty(Ke, dtype=torch.float32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host_in)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def e2e_step(i):
            for d, h in zip(dev_in, host_in):
                d.copy_(h, non_blocking=True)
            call(0)
            h_loss[i:i + 1].copy_(outs[0].loss, non_blocking=True)

        e2e_step(0)
        torch.cuda.synchronize()
        s0.record()
        for i in range(Ke):
            e2e_step(i)
        s1.record()
        torch.cuda.synchronize()
        e_ms = torch.tensor([s0.elapsed_time(s1)], dtype=torch.float64, device=dev)
        if world > 1:
            torch.distributed.all_reduce(e_ms, op=torch.distributed.ReduceOp.MAX)
        e2e = {"value": n * world * Ke / (float(e_ms[0]) / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": 4, "steps": Ke, "ms_per_step": float(e_ms[0]) / Ke}
    hbm, _, peak_kind = peaks()
    alg = 4.0 * n * V + 8.0 * n
    # DRAM bytes of the cluster kernel per call, from its committed capture
    # (the gradient it writes is still in L2 when the kernel ends)
    ratio = profile_traffic_ratio(f"dec_cluster_{spec.key}", DEC_SOURCE)
    roof = {"bound": "hbm", "achieved": alg / (call_ms / 1e3) / 1e9, "peak": hbm, "unit": "GB/s",
            "frac": alg / (call_ms / 1e3) / 1e9 / hbm, "traffic": ratio * alg if ratio else None,
            "kernel": "k_dec_cluster + k_dec_reduce (timed as the whole dlm_decision_loss_fwd_bwd call)",
            "algorithmic_bytes_per_launch": alg, "launch_ms": call_ms,
            "peak_source": f"{peak_kind} hbm_gbs (copy bandwidth)"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = _decision_cpu_baseline(spec, sets[0])
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": spec.key, "description": spec.description, "label_slots": n, "vocab": V,
                       "parallelism": f"replicas{world}", "label_softmax": "both", "brier_weight": 0.1,
                       "l2": f"eight input sets used in turn (8 x {n * V * 2 / 1e6:.0f} MB of logits, "
                             f"{'larger' if 8 * n * V * 2 > 126e6 else 'smaller'} than L2)",
                       "timing": "steps run from one CUDA graph of all timed calls (no host gap between calls); "
                                 "steps rounded up to a multiple of eight",
                       "unit_note": "scored tokens = label slots"},
            "roofline": roof, "cpu_baseline": cpu, "clocks": clk, "e2e": e2e, "gpu_launches": 2 * K}


def _decision_cpu_baseline(spec, case, budget_s=4.0):
    """The decision oracle on the whole workload, repeated for about
    budget_s seconds."""
    import dlm_inputs as di
    import oracle

    e = {k: v.cpu().numpy() for k, v in case.extra.items()}
    x = di.bf16_bits(case.logits)
    t0 = time.perf_counter()
    steps = 0
    while steps < 1 or time.perf_counter() - t0 < budget_s:
        oracle.decision_loss(x, spec.vocab, None, e["cand_off"], e["cand_ids"], e["kind"], e["val"])
        steps += 1
    dt = time.perf_counter() - t0
    return {"value": spec.n_units * steps / dt, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
            "sample": f"{steps} runs of the whole workload ({spec.n_units} label slots, V = {spec.vocab}; "
                      f"the three terms and the double-precision gradient of every logit): {dt:.1f} s"}


def _linear_e2e(args, spec, case, lay, enc, align, per_step, out):
    """The fused-head call end to end on one GPU: every step copies its inputs
    from pinned host memory, runs time draw, corruption and the loss through
    the public API, and reads the loss back.  Seeds 1000.. as the timed
    steps, so the scored rows are those steps' counts."""
    import torch

    import diffusion_lm_loss_b200 as dlm

    uniform = enc is not None
    Ke = max(1, min(args.steps, args.e2e_steps))
    dev_in = [case.hidden, case.clean] + ([case.enc_hidden, case.enc_clean] if uniform else [case.cu_seqlens])
    host_in = [t.cpu().pin_memory() for t in dev_in]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    h_loss = torch.empty(Ke, dtype=torch.float32).pin_memory()
    V = spec.vocab

    def e2e_step(i):
        nonlocal out
        for d, h in zip(dev_in, host_in):
            d.copy_(h, non_blocking=True)
        t, p = dlm.sample_t(1000 + i, case.n_units, spec.mode, spec.eps)
        _, corr = dlm.corrupt(lay, case.clean, p, spec.mode, spec.mask_id, V, 1000 + i)
        if uniform:
            out = dlm.linear_loss_uniform_fwd_bwd(lay, case.hidden, case.weight, case.clean, enc, case.enc_hidden,
                                                  case.enc_clean, enc_ar_weight=spec.enc_ar_weight, align=align,
                                                  out=out)
        else:
            out = dlm.linear_loss_fwd_bwd(lay, case.hidden, case.weight, case.clean, corr, p, out=out, align=align)
        h_loss[i:i + 1].copy_(out.loss, non_blocking=True)

    e2e_step(0)
    torch.cuda.synchronize()
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record()
    for i in range(Ke):
        e2e_step(i)
    s1.record()
    torch.cuda.synchronize()
    e_ms = s0.elapsed_time(s1)
    return {"value": sum(per_step[:Ke]) / (e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": 4, "steps": Ke, "ms_per_step": e_ms / Ke}


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------
def sample_spec(spec, rows):
    """The workload cut to its first `rows` rows per sequence (packed
    documents: to its first `rows` tokens, the same documents up to the cut)."""
    if spec.kind == "linear" and spec.mode == ABSORBING:
        return spec.scaled(n_tokens_packed=rows)
    return spec.scaled(seq_len=rows, prefix=min(spec.prefix, rows))


def sample_words(spec, rows):
    """How a bounded sample of the workload is described in the JSON line."""
    cut = (f"its first {rows} tokens of packed documents" if spec.kind == "linear" and spec.mode == ABSORBING
           else f"its first {rows} rows per sequence")
    work = ("time draw, corruption, CE of the scored rows, double-precision gradient of every row"
            + (", dH and dW through the head" if spec.kind == "linear" else ""))
    return cut, work


def oracle_inputs(spec, case_cpu):
    """Bit patterns of the fused-head inputs, converted once per case, before
    any timing (the logits workloads convert their sample inside the step)."""
    import dlm_inputs as di

    if spec.kind == "linear" and "W" not in case_cpu.extra:
        case_cpu.extra["W"] = di.bf16_bits(case_cpu.weight)
        case_cpu.extra["H"] = di.bf16_bits(case_cpu.hidden)
        if case_cpu.enc_hidden is not None:
            case_cpu.extra["He"] = di.bf16_bits(case_cpu.enc_hidden)


def oracle_host_bytes(spec, rows):
    """Peak host memory of one fused-head oracle step on `rows` rows per
    sequence (double-precision dW per term and their sum, W as bf16 in torch
    and numpy, Z and dZ of the rows), or 0 for the logits workloads."""
    if spec.kind != "linear":
        return 0
    V, D = spec.vocab, spec.d_model
    terms = 2 if spec.mode == UNIFORM else 1
    units = spec.n_units if spec.mode == UNIFORM else 1
    return V * D * (8 * (terms + 1) + 2 * 2) + 2 * rows * units * V * 8 + 16384 * D * 8


def oracle_step(spec, case_cpu, seed, rows_sample):
    """The oracle as it stands on the first `rows_sample` rows of each unit's
    sequence: time draw, corruption, CE of the scored rows, gradient of all
    rows.  Returns the number of scored rows."""
    import numpy as np

    import dlm_inputs as di
    import oracle

    if spec.kind == "linear":
        return _oracle_linear_step(spec, case_cpu, seed)

    B = spec.n_units
    L = min(spec.seq_len, rows_sample)
    lay = oracle.Layout(B, L, None, None)
    clean = case_cpu.clean.view(B, spec.seq_len)[:, :L].reshape(-1).numpy()
    x = di.bf16_bits(case_cpu.logits.view(B, spec.seq_len, -1)[:, :L].reshape(B * L, -1))
    _, p = oracle.sample_t(seed, B, spec.mode, spec.eps)
    _, corr = oracle.corrupt(lay, clean, p, spec.mode, spec.mask_id, spec.vocab, seed)
    if spec.mode == oracle.ABSORBING:
        loss, unit, tr = oracle.loss_absorbing(lay, x, spec.vocab, clean, corr, p, spec.align)
        oracle.term_grad(x, spec.vocab, tr, np.arange(B * L), 1.0)
        return int(tr.rows.shape[0])
    # uniform noise: the canvas term plus the encoder AR term over the first
    # rows of each (prefix + canvas) sequence
    S = spec.prefix + spec.seq_len
    Le = min(S, rows_sample)
    enc = oracle.Layout(B, Le, None, None)
    eclean = case_cpu.enc_clean.view(B, S)[:, :Le].reshape(-1).numpy()
    xe = di.bf16_bits(case_cpu.enc_logits.view(B, S, -1)[:, :Le].reshape(B * Le, -1))
    loss, unit, tc, te = oracle.loss_uniform(lay, x, clean, enc, xe, eclean, spec.vocab,
                                             spec.enc_ar_weight, spec.align)
    oracle.term_grad(x, spec.vocab, tc, np.arange(B * L), 1.0)
    oracle.term_grad(xe, spec.vocab, te, np.arange(B * Le), 1.0)
    return int(tc.rows.shape[0] + te.rows.shape[0])


def _oracle_linear_step(spec, case, seed):
    """The fused-head oracle on a case already cut to its sample: time draw,
    corruption, then the loss from hidden states and the head with dH and dW
    (absorbing: packed documents; uniform: canvas and encoder rows)."""
    import oracle

    oracle_inputs(spec, case)
    H, W = case.extra["H"], case.extra["W"]
    clean = case.clean.numpy()
    V = spec.vocab
    if spec.mode == UNIFORM:
        B, C, P = case.n_units, case.seq_len, spec.prefix
        lay = oracle.Layout(B, C, None, None)
        _, p = oracle.sample_t(seed, B, UNIFORM, spec.eps)
        oracle.corrupt(lay, clean, p, UNIFORM, spec.mask_id, V, seed)
        out = oracle.linear_loss_uniform(lay, H, W, clean, oracle.Layout(B, P + C, None, None),
                                         case.extra["He"], case.enc_clean.numpy(), spec.enc_ar_weight,
                                         spec.align)
        return int(out["rows"].shape[0] + out["enc_rows"].shape[0])
    lay = oracle.Layout(case.n_units, 0, case.cu_seqlens.numpy(), None)
    _, p = oracle.sample_t(seed, case.n_units, ABSORBING, spec.eps)
    _, corr = oracle.corrupt(lay, clean, p, ABSORBING, spec.mask_id, V, seed)
    out = oracle.linear_loss(lay, H, W, clean, corr, p, align=spec.align)
    return int(out["rows"].shape[0])


def _full_rows(spec):
    if spec.kind == "linear" and spec.mode == ABSORBING:
        return spec.n_tokens_packed
    return spec.seq_len


def _calibrated_rows(spec, per_step_s, cap=1024):
    """Rows per sequence such that one oracle step takes about per_step_s."""
    import dlm_inputs as di

    if spec.kind == "linear":
        # a large fixed cost per step (W converted to double for each GEMM):
        # two probe sizes separate it from the cost per row
        times = []
        for n in (16, 48):
            sub = sample_spec(spec, n)
            case = di.make_case(sub, "cpu")
            oracle_step(sub, case, 0, n)                    # conversions, first-call costs
            t0 = time.perf_counter()
            oracle_step(sub, case, 1, n)
            times.append(time.perf_counter() - t0)
        per_row = max((times[1] - times[0]) / 32, 1e-9)
        fixed = max(times[0] - 16 * per_row, 0.0)
        rows = int(max(per_step_s - fixed, 0.0) / per_row)
        return max(4, min(_full_rows(spec), cap, rows))
    probe = spec.scaled(seq_len=min(spec.seq_len, 16), prefix=min(spec.prefix, 16))
    case = di.make_case(probe, "cpu")
    oracle_step(probe, case, 0, probe.seq_len)          # first call builds / loads the oracle
    t0 = time.perf_counter()
    oracle_step(probe, case, 1, probe.seq_len)
    per_row = (time.perf_counter() - t0) / (probe.seq_len * probe.n_units)
    rows = int(per_step_s / max(per_row, 1e-9) / probe.n_units)
    return max(4, min(spec.seq_len, cap, rows))


def _oracle_threads():
    return int(os.environ.get("OMP_NUM_THREADS", len(os.sched_getaffinity(0))))


def cpu_baseline(spec, budget_s=15.0, min_steps=3, max_steps=100_000, single_thread_s=8.0):
    """The oracle on a bounded sample: rows per sequence sized so that one
    step takes about budget_s / min_steps (at most 1024 rows, which bounds
    the host memory of its double-precision gradient), then steps with fresh
    seeds until budget_s of CPU work has run.  With single_thread_s > 0 the
    same is timed again with one thread, in a child process started with
    OMP_NUM_THREADS=1 (the oracle's OpenMP and numpy's BLAS read it at
    start-up)."""
    import dlm_inputs as di
    import psutil

    need = oracle_host_bytes(spec, 1024)
    avail = psutil.virtual_memory().available
    if need > 0.6 * avail:
        return {"value": None, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
                "skipped": f"the oracle step needs ~{need / 1e9:.0f} GB of host memory, "
                           f"{avail / 1e9:.0f} GB available"}
    rows = _calibrated_rows(spec, budget_s / min_steps)
    sub = sample_spec(spec, rows)
    case = di.make_case(sub, "cpu")
    oracle_inputs(sub, case)
    t0 = time.perf_counter()
    scored = steps = 0
    while steps < min_steps or (steps < max_steps and time.perf_counter() - t0 < budget_s):
        scored += oracle_step(sub, case, 1000 + steps, rows)
        steps += 1
    dt = time.perf_counter() - t0
    res = {"value": scored / dt, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
           "sample": f"{steps} steps (seeds 1000..{999 + steps}) of the same workload cut to "
                     f"{sample_words(spec, rows)[0]} (V = {spec.vocab}; {sample_words(spec, rows)[1]}): "
                     f"{dt:.1f} s"}
    if single_thread_s > 0:
        env = dict(os.environ, OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1", MKL_NUM_THREADS="1")
        import dataclasses
        fields = json.dumps(dataclasses.asdict(spec))
        code = ("import json, bench, dlm_inputs as di; "
                f"spec = di.Spec(**json.loads({fields!r})); "
                f"print(json.dumps(bench.cpu_baseline(spec, budget_s={single_thread_s}, single_thread_s=0)))")
        try:
            r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                               text=True, timeout=20 * single_thread_s + 120)
            one = json.loads(r.stdout.strip().splitlines()[-1])
            res["single_thread"] = {"value": one["value"], "cores": one["cores"],
                                    "sample": one.get("sample", one.get("skipped"))}
        except Exception as e:   # the all-cores figure stands on its own
            res["single_thread"] = {"value": None, "error": f"{type(e).__name__}: {e}"[:200]}
    return res


def _decision_reference(args, spec, world):
    """The reference arm on a typed-decision workload: each step one run of
    the decision oracle over every label slot of the workload."""
    import dlm_inputs as di
    import oracle

    if args.slots:
        spec = spec.scaled(key=spec.key.replace(f"_s{spec.n_units}_", f"_s{args.slots}_"), n_units=args.slots)
    case = di.make_case(spec, "cpu")
    e = {k: v.numpy() for k, v in case.extra.items()}
    x = di.bf16_bits(case.logits)

    def step():
        oracle.decision_loss(x, spec.vocab, None, e["cand_off"], e["cand_ids"], e["kind"], e["val"])

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    val = spec.n_units * args.steps / dt
    sample = (f"each step: the whole workload ({spec.n_units} label slots, V = {spec.vocab}; the three terms "
              f"and the double-precision gradient of every logit)")
    print(json.dumps({"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
                      "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
                      "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                      "data": "synthetic",
                      "config": {"workload": spec.key, "description": spec.description,
                                 "label_slots": spec.n_units, "vocab": spec.vocab, "parallelism": "cpu"},
                      "cpu_baseline": {"value": val, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
                                       "sample": sample},
                      "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
          flush=True)


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, on the machine's host
    cores, each step a bounded sample of the workload sized so that the
    whole run ends in about two minutes."""
    rank, _, world = env_rank()
    if rank != 0:
        return
    import dlm_inputs as di

    spec = di.WORKLOADS[SUITE_HEADLINE if args.workload == SUITE else args.workload]
    if spec.kind == "decision":
        _decision_reference(args, spec, world)
        return
    need = oracle_host_bytes(spec, 1024)
    if need > 0.6 * __import__("psutil").virtual_memory().available:
        print(json.dumps({"impl": "reference",
                          "unavailable": f"the CPU oracle needs ~{need / 1e9:.0f} GB of host memory "
                                         "for this workload"}), flush=True)
        return
    rows = _calibrated_rows(spec, 100.0 / (args.steps + args.warmup))
    sub = sample_spec(spec, rows)
    case = di.make_case(sub, "cpu")
    oracle_inputs(sub, case)
    for i in range(args.warmup):
        oracle_step(sub, case, 10 + i, rows)
    t0 = time.perf_counter()
    scored = 0
    for i in range(args.steps):
        scored += oracle_step(sub, case, 1000 + i, rows)
    dt = time.perf_counter() - t0
    val = scored / dt
    cut, work = sample_words(spec, rows)
    sample = f"each step: the workload cut to {cut} (V = {spec.vocab}); the oracle's whole path ({work})"
    res = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic",
           "config": {"workload": spec.key, "description": spec.description,
                      "global_batch": spec.n_units, "seq_len": rows, "vocab": spec.vocab,
                      "parallelism": "cpu"},
           "cpu_baseline": {"value": val, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--keep-unscored", action="store_true",
                    help="loss workloads: the call does not write unscored rows (secondary figure)")
    ap.add_argument("--align", choices=["aligned", "shifted"], default="aligned",
                    help="fused-head workloads: targets aligned (row i scores token i) or shifted (token i+1)")
    ap.add_argument("--objective", choices=["plain", "rhine"], default="plain",
                    help="uniform-noise workloads: plain canvas mean, or the Rhine objective options")
    ap.add_argument("--slots", type=int, default=0,
                    help="typed-decision workloads: label slots per call (default: the workload's 128)")
    args = ap.parse_args()
    if args.slots < 0 or args.slots > 65535:
        raise SystemExit("--slots must be in 0..65535")
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
