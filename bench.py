#!/usr/bin/env python
"""Throughput of AM-OMP KV compaction on B200: KV-head compactions per second
and seconds per full-model compaction.

One step = one am_compact_heads call over a batch of synthetic heads already
resident in HBM: shift → Φ pass → OMP passes (correlation, selection, Gram,
NNLS, residual) → β, packing → value fit.  Workloads (the pages' settings,
with seeded synthetic heads in place of model activations):

  qwen3_4b_model      (default) the full Qwen3-4B-shaped model at 50×: 288 heads,
                      T = n = 8192, d = 128, bf16, log-normal budgets 8..1024,
                      top-k 4 with a refit every 2 rounds; one step compacts the
                      whole model, so s_per_model is the measured step time
  qwen3_4b_layer      one layer of it: 8 heads, t = 164
  llama31_8b_longctx  a Llama-3.1-8B-shaped 60000-token context at 10×: 32 × 8
                      sequences cut into 7 × 8192 + 2656-key chunks, 2048
                      chunk-heads with n = 8192, t = 819 / 266, top-k 8, R = 2;
                      the chunk-heads run in waves through one workspace
  online_rounds       six chained online compaction rounds of 288 heads
                      (cache 2048, keep 20, halve the rest)
  single_head_fp32    the small i.i.d. fp32 head

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--shard own|lpt] [--impl ours|reference]

N > 1 runs under torch.distributed.run, one rank per GPU.  --shard own (the
default): every rank compacts its own seeded copy of the workload (weak
scaling, no collective on the data path).  --shard lpt: the ranks split one
workload's heads by longest-processing-time on cost t·⌈t/(k·R)⌉ (strong
scaling).  The timed region is bracketed by a barrier and a device
synchronize; the step time is the max over ranks.

Timing: per-step CUDA events on the compute stream; a 256 MiB buffer is
written between timed steps to flush L2 (the inputs are larger than L2 as
well).  Stage times come from the library's own event brackets
(am_profile_*) on separate untimed steps, giving the live roofline of the
dominant stage (stages of different head groups overlap on the GPU, so
stage times can add up to more than a step).  `--impl reference` times the
float64 CPU oracle on a bounded sample of the same workload instead.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KV-head compactions/sec and seconds per full-model compaction, 1 B200"
LAYERS_QWEN3_4B = 36
WORKLOADS = ["qwen3_4b_model", "qwen3_4b_layer", "llama31_8b_longctx", "online_rounds", "single_head_fp32"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 20 for the model, 100 for the layer, 3 for the long context)")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen3_4b_model", choices=WORKLOADS)
    ap.add_argument("--shard", choices=["own", "lpt"], default="own",
                    help="multi-GPU: each rank its own workload copy (weak) or an LPT split of one (strong)")
    ap.add_argument("--heads", type=int, default=None,
                    help="heads per GPU for the layer workload (default 8); smaller for profiling")
    ap.add_argument("--sequences", type=int, default=None,
                    help="long-context workload: keep the first sequences only (default all 256)")
    ap.add_argument("--wave-heads", type=int, default=None,
                    help="heads per wave (default: as many as fit in 3/4 of the free device memory)")
    ap.add_argument("--corr", choices=["auto", "fp32", "bf16", "recompute", "bounded"], default="auto",
                    help="correlation pass: stored fp32 / stored bf16 copy / tensor-core recompute / "
                         "bounded (exact values for the keys a Cauchy-Schwarz bound cannot exclude)")
    ap.add_argument("--select", choices=["omp", "highest"], default="omp",
                    help="key selection: greedy OMP (the method) or the t keys of highest total attention")
    ap.add_argument("--consume", type=int, default=None, metavar="T_NEW",
                    help="instead of the compaction line, time attention of --queries queries per head over "
                         "each head's compacted segment plus T_NEW fresh keys (one GPU)")
    ap.add_argument("--queries", type=int, default=128)
    ap.add_argument("--cpu-seconds", type=float, default=20.0,
                    help="host time budget of the oracle sample behind cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = {"qwen3_4b_layer": 100, "llama31_8b_longctx": 3, "single_head_fp32": 100}.get(args.workload, 20)
    return args


def max_over_ranks(ms, dist, device):
    """The step time of the job: the slowest rank's (identity for one process)."""
    if dist is None:
        return float(ms)
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(heads_per_rank, world, ms):
    """Whole-job heads/s: every rank compacts its own heads in the same step time."""
    return heads_per_rank * world / (ms * 1e-3)


def _longctx_sequence(seed):
    from attention_matching_b200 import workloads as W
    return W.long_sequence_chunks(seed, 60000, 8192, 8192)


def longctx_workload(seed_base, sequences):
    """The long-context workload, its sequences drawn in parallel worker
    processes (started with 'spawn', before any CUDA use); the same heads as
    workloads.llama31_8b_longctx(seed_base, max_sequences=sequences)."""
    import concurrent.futures
    import multiprocessing as mp
    from attention_matching_b200 import workloads as W
    workers = max(1, min(16, (os.cpu_count() or 1), sequences))
    with concurrent.futures.ProcessPoolExecutor(workers, mp_context=mp.get_context("spawn")) as ex:
        chunks = list(ex.map(_longctx_sequence, [seed_base + q for q in range(sequences)]))
    heads = [c for seq in chunks for c in seq]
    budgets = [W.budget_for_ratio(h.T, 10.0) for h in heads]
    name = f"llama31_8b_longctx_{sequences}seq_T60000_chunk8192_n8192_d128_x10"
    return W.Workload(name, heads, budgets, 8, 2, "bf16", key_offsets=W.key_offsets_of(heads))


def build_workload(name, rank, heads=None, sequences=None, only=None):
    """The named workload; rank r draws its own seeds (weak scaling), `only`
    keeps a subset of the model's heads (an LPT shard)."""
    from attention_matching_b200 import workloads as W
    if name == "qwen3_4b_layer":
        return W.qwen3_4b_layer(num_heads=heads or 8, seed_base=2000 + 1000 * rank)
    if name == "qwen3_4b_model":
        return W.qwen3_4b_model(seed_base=4000 + 1000 * rank, only=only)
    if name == "llama31_8b_longctx":
        return longctx_workload(5000 + 1000 * rank, sequences or 256)
    return W.single_head_fp32(seed=1000 + rank)


def model_budgets(name, heads=None):
    """Budgets and picks per pass of the whole workload (for an LPT split)."""
    from attention_matching_b200 import workloads as W
    if name == "qwen3_4b_model":
        return W.lognormal_budgets(4000 + 999, 288, int(math.floor(8192 * 288 / 50 + 0.5))), 8
    raise ValueError(f"--shard lpt is defined for qwen3_4b_model, not {name}")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "sm_max_mhz": float(pk.get("sm_max_mhz", 1965.0)), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0, "source": "fallback"}


# ---------------------------------------------------------------- clocks ----
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
        if self.gpu_id is not None:
            cmd += ["-i", str(self.gpu_id)]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def wait_first(self, limit_s=10.0):
        """Block until nvidia-smi has printed its first sample (it takes a
        moment to start), so that the samples cover the timed region."""
        t0 = time.time()
        while self.proc is not None and not self.lines and time.time() - t0 < limit_s:
            time.sleep(0.01)
        self.lines.clear()

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) != 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for _, _, r in rows for k in range(4) if r[k].lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def gpu_smi_id(torch, dev):
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        first = vis.split(",")[0] if vis else str(dev)
        return first if first.isdigit() else None


# ------------------------------------------------------------ cpu oracle ----
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([x.get("num_threads", 1) for x in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(wl, seconds, order):
    """Time the float64 oracle head by head in `order` until `seconds` of host
    time are spent (at least one head); per-head wall times."""
    from oracle import am_oracle as O
    t0 = time.perf_counter()
    done, each = [], []
    for h in order:
        t1 = time.perf_counter()
        Q, K, V = wl.heads[h].f64()
        O.compact_head(Q, K, V, wl.budgets[h], wl.topk, wl.refit_every)
        done.append(h)
        each.append(time.perf_counter() - t1)
        if time.perf_counter() - t0 >= seconds:
            break
    return done, each, _blas_threads()


def cpu_baseline(wl, seconds):
    """The oracle (as it stands) on a bounded sample of the workload's heads:
    a seeded random order over the heads whose budget is at most the median
    and at most 300 (so that no single head exceeds the time budget; when no
    head qualifies, the smallest budgets).  The whole workload's
    oracle time is extrapolated with per-head time = a + b·cost_h, cost_h =
    t_h·⌈t_h/(k·R)⌉, a and b >= 0 fitted to the sampled heads by least squares
    (with one sampled head or one distinct cost: proportional to cost).  The
    oracle's cost grows faster than cost_h on the largest budgets, so the
    extrapolation is generous to it there."""
    import random
    import numpy as np
    from attention_matching_b200.sharding import head_cost
    kR = wl.topk * wl.refit_every
    cost = np.array([head_cost(t, kR) for t in wl.budgets], dtype=np.float64)
    cap = min(float(np.median(wl.budgets)), 300.0)
    order = [h for h in range(len(wl.heads)) if wl.budgets[h] <= cap]
    if not order:
        lo = min(wl.budgets)
        order = [h for h in range(len(wl.heads)) if wl.budgets[h] == lo]
    random.Random(12345).shuffle(order)
    done, each, cores = oracle_sample(wl, seconds, order)
    c, tm = cost[done], np.array(each)
    a, b = 0.0, float(tm.sum() / c.sum())
    if len(set(c.tolist())) >= 2:
        A = np.stack([np.ones_like(c), c], axis=1)
        (fa, fb), *_ = np.linalg.lstsq(A, tm, rcond=None)
        if fa >= 0 and fb >= 0:
            a, b = float(fa), float(fb)
    whole = float(len(cost) * a + b * cost.sum())
    dt = float(tm.sum())
    return {"value": len(wl.heads) / whole, "unit": "heads/s", "cores": cores, "kind": "oracle",
            "s_per_workload_extrapolated": whole,
            "sample": f"{len(done)} of {len(wl.heads)} heads of {wl.name} (seeded random order over budgets "
                      f"<= min(median, 300); sampled budgets {sorted(wl.budgets[h] for h in done)}), float64 "
                      f"NumPy/SciPy oracle, {dt:.1f} s wall; workload time extrapolated as "
                      f"sum(a + b*t*ceil(t/(k*R))) with a = {a:.3g} s, b = {b:.3g} s fitted to the sample"}


# -------------------------------------------------------------- roofline ----
HIGHEST_CHUNK = 8   # pre-selected keys the library appends per refit in highest-attention mode


def stage_models(wl, n, key_counts, d, ldn, corr_kind, rows_evaluated, tc=True):
    """Algorithmic work of one call (one step) per library stage: bytes that
    must cross HBM for the memory-bound stages, dense flops for the GEMM and
    the fp64 solver stages.  Summed over the stage's launches in the step.
    `key_counts` holds every head's T_h.  With the tensor-core feature pass
    the column norms are summed from its per-(query block, quarter) fp32
    partials instead of re-reading Φᵀ."""
    H = len(key_counts)
    sT = float(sum(key_counts))
    kR = HIGHEST_CHUNK if corr_kind == "highest" else wl.topk * wl.refit_every
    s1 = [min((p + 1) * kR, t) for t in wl.budgets for p in range((t + kR - 1) // kR)]
    row = ldn * 4                                   # one stored Φᵀ row (fp32)
    m = {
        "shift": {"bound": "tensor", "flops": 2.0 * n * sT * d},
        "phi": {"bound": "hbm", "bytes": sT * row + H * (n * d * 2 + n * d * 4 + ldn * 12) + sT * 2 * d * 2,
                "flops": 4.0 * n * sT * d},
        "target": {"bound": "hbm", "bytes": sT * row + sT * d * 4 + H * n * d * 4},
        "gram": {"bound": "hbm", "bytes": float(sum(s1)) * row},
        "resid": {"bound": "hbm", "bytes": float(sum(s1)) * row + len(s1) * ldn * 12},
        "nnls": {"bound": "hbm", "bytes": float(sum(2 * x * x * 8 for x in s1))},
        "design": {"bound": "hbm", "bytes": float(sum(wl.budgets)) * row * 2},
        # AᵀA and AᵀY as a dense GEMM (2·n·t·(t + d) flops): on the tensor cores for bf16
        # inputs with d in {64, 128} (six bf16 products per fp32 product), else fp64 FMA
        "normal": ({"bound": "tensor", "flops": float(sum(2 * n * t * (t + d) for t in wl.budgets))} if tc else
                   {"bound": "fp64", "flops": float(sum(n * t * (t + 1) + 2 * n * t * d for t in wl.budgets))}),
        "solve": {"bound": "fp64", "flops": float(sum(t ** 3 / 3 + 2 * t * t * d for t in wl.budgets))},
    }
    if corr_kind == "highest":
        # one fp64 pass over the stored features for the scores, then a per-head sort
        m["corr"] = {"bound": "hbm", "bytes": sT * row + H * ldn * 8}
    elif corr_kind == "recompute":
        passes = [sum(1 for _ in range((t + kR - 1) // kR)) for t in wl.budgets]
        work = float(sum(p * T for p, T in zip(passes, key_counts)))
        m["corr"] = {"bound": "tensor", "flops": 2.0 * work * n * d, "exps": work * n}
    elif corr_kind == "bounded":
        parts = 4 * ((n + 127) // 128)
        G = min((ldn // 4 + 31) // 32, 64)
        # partials in (or the stored features on the CUDA-core path), fp64 norms and the
        # per-group fp32 norms out
        norms_in = parts * 4 if tc else row
        m["norms"] = {"bound": "hbm", "bytes": sT * (norms_in + 8 + 64 * 4)}
        # per pass and head: every key's group norms read and its bound written, then the
        # evaluated rows of the stored features
        heads_passes = float(sum(((t + kR - 1) // kR) * T for t, T in zip(wl.budgets, key_counts)))
        m["rows"] = {"bound": "hbm", "bytes": float(rows_evaluated) * row + heads_passes * (G * 4 + 4 + 4)}
    else:
        passes = [(t + kR - 1) // kR for t in wl.budgets]
        b = 2 if corr_kind == "bf16" else 4
        m["corr"] = {"bound": "hbm", "bytes": float(sum(p * (T * ldn * b + row + T * 4)
                                                        for p, T in zip(passes, key_counts)))}
    return m


def stage_roofline(name, st, steps, model, peaks, clocks):
    """Achieved rate of one stage against its roofline: the stage's algorithmic
    work per step times the steps, over its measured device time."""
    secs = st["ms"] * 1e-3
    mhz = (clocks or {}).get("sm_mhz") or peaks["sm_max_mhz"]
    out = {"kernel": name, "avg_launch_ms": st["ms"] / st["launches"], "launches_per_step": st["launches"] / steps}
    if model is None:
        out.update({"bound": None, "achieved": None, "peak": None, "unit": None, "frac": None})
        return out
    if model["bound"] == "hbm":
        ach = model["bytes"] * steps / secs / 1e9
        out.update({"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": ach / peaks["hbm_gbs"], "peak_source": peaks["source"] + " hbm_gbs",
                    "algorithmic_bytes_per_step": model["bytes"]})
        if "flops" in model:
            tf = model["flops"] * steps / secs / 1e12
            out["tensor"] = {"achieved_tflops": tf, "frac_of_sustained_bf16": tf / peaks["bf16_tflops_sustained"]}
    elif model["bound"] == "tensor":
        ach = model["flops"] * steps / secs / 1e12
        pk = peaks["bf16_tflops_sustained"]
        out.update({"bound": "tensor", "achieved": ach, "peak": pk, "unit": "TFLOP/s", "frac": ach / pk,
                    "peak_source": peaks["source"] + " bf16_tflops_sustained",
                    "algorithmic_flops_per_step": model["flops"]})
        if "exps" in model:
            # one exponential per feature against the ex2 unit rate, 148 SMs x 16 per clock
            exp_peak = 148 * 16 * mhz * 1e6
            rate = model["exps"] * steps / secs
            out["exp_rate"] = {"achieved_per_s": rate, "peak_per_s": exp_peak, "frac": rate / exp_peak}
    else:
        # fp64 FMA pipes: 148 SMs x 64 lanes x 2 flops x SM clock
        peak = 148 * 64 * 2 * mhz * 1e6 / 1e12
        ach = model["flops"] * steps / secs / 1e12
        out.update({"bound": "alu", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                    "peak_source": "fp64 FMA: 148 SMs x 64 lanes x 2 x median SM clock",
                    "algorithmic_flops_per_step": model["flops"]})
    return out


def roofline(stages, steps, models, peaks, clocks, traffic_info):
    """The dominant stage's roofline (the JSON contract), plus every stage's."""
    per = {k: v for k, v in stages.items() if v["launches"] > 0}
    dom = max(per, key=lambda k: per[k]["ms"])
    out = stage_roofline(dom, per[dom], steps, models.get(dom), peaks, clocks)
    tr = traffic_info.get(dom)
    out["traffic"] = None if tr is None else tr["bytes_per_launch"]
    if tr is not None:
        out["traffic_source"] = tr["source"]
    out["all_stages"] = {k: {kk: vv for kk, vv in stage_roofline(k, v, steps, models.get(k), peaks, clocks).items()
                             if kk in ("bound", "achieved", "unit", "frac", "avg_launch_ms", "launches_per_step")}
                         for k, v in sorted(per.items(), key=lambda kv: -kv[1]["ms"])}
    return out


def committed_traffic(workload):
    """DRAM bytes per launch of a stage's kernel on this workload from the
    committed ncu summaries (profiles/traffic.json), used only while the
    profiled kernel's source region still hashes to what was profiled."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return {}
    out = {}
    for v in rec.values():
        if v.get("workload") != workload:
            continue
        try:
            src = open(os.path.join(ROOT, v["source"])).read()
            region = src[src.index(v["region_begin"]):src.index(v["region_end"])]
        except Exception:
            continue
        if hashlib.sha256(region.encode()).hexdigest()[:16] == v["region_sha256_16"]:
            out[v["stage"]] = {"bytes_per_launch": v["dram_bytes_per_launch"], "source": v["summary"]}
    return out


# ------------------------------------------------------------------ arms ----
def run_reference(args, rank, world):
    """The float64 oracle on the host's cores, on this arm's workload: each
    step a bounded sample of heads (--cpu-seconds), extrapolated to the whole
    workload by the cost weights; rank 0 only."""
    if rank != 0:
        return 0
    if args.workload == "online_rounds":
        print(json.dumps({"impl": "reference", "unavailable": "the oracle reference arm covers the one-call "
                          "workloads; online rounds chain the GPU's own outputs"}))
        return 0
    wl = build_workload(args.workload, 0, args.heads, sequences=min(args.sequences or 2, 2)
                        if args.workload == "llama31_8b_longctx" else None)
    vals, whole = [], []
    cb = None
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(wl, args.cpu_seconds)
        if i >= args.warmup:
            vals.append(cb["value"])
            whole.append(cb["s_per_workload_extrapolated"])
    value = statistics.mean(vals)
    ms = 1e3 * statistics.mean(whole)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "heads/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "sample": cb["sample"]},
        "cpu_baseline": dict(cb, value=value),
        "e2e": {"value": value, "unit": "heads/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def _inputs(wl, torch):
    """Host tensors of the workload: stacked [H][T][d], or packed [Σ T_h][d]
    with key offsets when the heads' key counts differ."""
    Qh = torch.stack([h.Q for h in wl.heads]).contiguous()
    if wl.key_offsets is None:
        Kh = torch.stack([h.K for h in wl.heads]).contiguous()
        Vh = torch.stack([h.V for h in wl.heads]).contiguous()
    else:
        Kh = torch.cat([h.K for h in wl.heads]).contiguous()
        Vh = torch.cat([h.V for h in wl.heads]).contiguous()
    return Qh, Kh, Vh


def run_ours(args, rank, world, local_rank):
    import torch
    import attention_matching_b200 as am
    from attention_matching_b200 import sharding
    # the long-context workload is drawn by a spawn pool before any CUDA use
    my_heads = None
    if args.shard == "lpt" and world > 1:
        budgets_all, kR = model_budgets(args.workload)
        parts = sharding.lpt_partition([sharding.head_cost(t, kR) for t in budgets_all], world)
        my_heads = parts[rank]
        wl = build_workload(args.workload, 0, only=my_heads)
    else:
        wl = build_workload(args.workload, rank, args.heads, args.sequences)
    dist = None
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    H = len(wl.heads)
    n, d = wl.heads[0].n, wl.heads[0].d
    key_counts = [h.T for h in wl.heads]
    T = max(key_counts)
    Qh, Kh, Vh = _inputs(wl, torch)
    Q, K, V = Qh.to(dev), Kh.to(dev), Vh.to(dev)
    corr_mode = {"auto": am.CORR_AUTO, "fp32": am.CORR_STORED_FP32, "bf16": am.CORR_STORED_BF16,
                 "recompute": am.CORR_RECOMPUTE, "bounded": am.CORR_BOUNDED}[args.corr]
    select_mode = am.SELECT_HIGHEST if args.select == "highest" else am.SELECT_OMP
    kw = dict(topk=wl.topk, refit_every=wl.refit_every, corr_mode=corr_mode, select_mode=select_mode,
              key_offsets=wl.key_offsets)
    opts = am.make_opts(am.BF16 if Q.dtype == torch.bfloat16 else am.FP32, wl.topk, wl.refit_every,
                        corr_mode=corr_mode, select_mode=select_mode)
    koffs_c = None
    if wl.key_offsets is not None:
        import ctypes
        koffs_c = (ctypes.c_int64 * (H + 1))(*wl.key_offsets)
        opts.key_offsets = ctypes.cast(koffs_c, ctypes.c_void_p)
    tc_ok = Q.dtype == torch.bfloat16 and d in (64, 128)
    corr_kind = "highest" if args.select == "highest" else {"auto": "bounded"}.get(args.corr, args.corr)
    full_ws = am.workspace_size(n, T, d, wl.budgets, opts)
    wave = args.wave_heads
    if wave is None:
        free, _ = torch.cuda.mem_get_info(dev)
        room = int(0.75 * free) - (1 << 30)
        wave = H
        while wave > 1 and am.workspace_size(n, T, d, wl.budgets, opts, wave_heads=wave) > room:
            wave = max(1, wave * 3 // 4)
    ws_bytes = am.workspace_size(n, T, d, wl.budgets, opts, wave_heads=wave)
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device=dev)

    first = am.compact_heads(Q, K, V, wl.budgets, workspace=ws, **kw)   # checks device status
    for _ in range(args.warmup):
        am.compact_heads(Q, K, V, wl.budgets, workspace=ws, check=False, **kw)
    torch.cuda.synchronize()

    clocks = ClockSampler(gpu_smi_id(torch, local_rank))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    clocks.wait_first()
    l0 = am.kernel_launches()
    evs = []
    for _ in range(args.steps):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        am.compact_heads(Q, K, V, wl.budgets, workspace=ws, check=False, **kw)
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    launches = am.kernel_launches() - l0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    # stage times from separate, untimed steps with the library's event brackets
    prof_steps = max(1, min(args.steps, 10))
    am.profile_enable(True)
    for _ in range(prof_steps):
        flush.fill_(1)
        am.compact_heads(Q, K, V, wl.budgets, workspace=ws, check=False, **kw)
    torch.cuda.synchronize()
    am.profile_enable(False)
    stages = am.profile_collect()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    ms = statistics.mean(step_ms)
    ms = max_over_ranks(ms, dist if world > 1 else None, dev)
    _, worst = am.get_status(ws, H)
    one_wave = ws_bytes >= full_ws
    # per-head statistics of the last call (kept in the workspace prefix, so
    # valid after a call of several waves too)
    cst = am.call_stats({"workspace": ws}, n, T, d, wl.budgets, wl.topk, wl.refit_every,
                        am.BF16 if Q.dtype == torch.bfloat16 else am.FP32, corr_mode, select_mode)
    rows_eval = int(cst["rows_evaluated"].sum().item()) if corr_kind == "bounded" else None
    refits = int(cst["nnls_refits"].sum().item())
    solves = int(cst["nnls_solves"].sum().item())

    # end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e:
        Qp, Kp, Vp = Qh.pin_memory(), Kh.pin_memory(), Vh.pin_memory()
        am.compact_heads(Qp, Kp, Vp, wl.budgets, workspace=ws, check=False, **kw)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ev2 = []
        d2h = 0
        for _ in range(args.steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            o = am.compact_heads(Qp, Kp, Vp, wl.budgets, workspace=ws, check=False, **kw)
            b.record(stream)
            ev2.append((a, b))
            d2h = sum(o[k].numel() * o[k].element_size() for k in ("C_k", "beta", "C_v", "indices"))
        torch.cuda.synchronize()
        e_ms = statistics.mean(a.elapsed_time(b) for a, b in ev2)
        e_ms = max_over_ranks(e_ms, dist if world > 1 else None, dev)
        e2e = {"value": job_throughput(H, world, e_ms) if my_heads is None else len(budgets_all) / (e_ms * 1e-3),
               "unit": "heads/s", "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in (Qh, Kh, Vh)),
               "d2h_bytes_per_step": d2h, "ms_per_step": e_ms}

    if world > 1:
        dist.barrier()
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    ldn = (n + 31) // 32 * 32
    peaks = load_peaks()
    models = stage_models(wl, n, key_counts, d, ldn, corr_kind, rows_eval or 0, tc_ok)
    rf = roofline(stages, prof_steps, models, peaks, clk, committed_traffic(wl.name))
    total_heads = H * world if my_heads is None else len(budgets_all)
    value = total_heads / (ms * 1e-3)
    per_step_stage = {k: round(v["ms"] / prof_steps, 4) for k, v in stages.items() if v["launches"]}
    cfg = {"workload": wl.name, "heads_per_gpu": H, "n": n, "T": T, "d": d,
           "budgets": wl.budgets if H <= 8 else f"{sum(wl.budgets)} total, min {min(wl.budgets)} max {max(wl.budgets)}",
           "topk": wl.topk, "refit_every": wl.refit_every,
           "selection": "greedy OMP with NNLS refits" if args.select == "omp" else
                        "the t keys of highest total attention, NNLS beta fit",
           "correlation": {"fp32": "streams stored fp32 Phi^T", "bf16": "streams a bf16 copy of Phi^T",
                           "highest": "fp64 total-attention score of every key, one pass over Phi^T",
                           "recompute": "recomputes Phi on the tensor cores each pass",
                           "bounded": "exact fp64 values for the keys whose Cauchy-Schwarz bound "
                                      "reaches the pass's top k*R"}[corr_kind],
           "l2": "256 MiB buffer written between timed steps; inputs larger than L2",
           "workspace_bytes": ws_bytes, "wave_heads": wave if not one_wave else H,
           "stage_ms_per_step": per_step_stage, "device_status": worst}
    if wl.key_offsets is not None:
        cfg["key_counts"] = f"{len(key_counts)} heads, {sorted(set(key_counts))}"
    if rows_eval:
        cfg["correlation_rows_evaluated_per_step"] = rows_eval
    if refits:
        cfg["nnls_refits_per_step"] = refits
        cfg["nnls_inner_solves_per_step"] = solves
    if my_heads is not None:
        cfg["sharding"] = f"LPT over {world} ranks of one workload's {len(budgets_all)} heads, cost t*ceil(t/(k*R))"
    if args.workload == "qwen3_4b_layer":
        cfg["s_per_model_extrapolated_x36_layers"] = LAYERS_QWEN3_4B * ms * 1e-3
    if args.workload == "qwen3_4b_model":
        cfg["s_per_model"] = ms * 1e-3
    if args.workload == "llama31_8b_longctx":
        cfg["s_per_context"] = ms * 1e-3
    line = {
        "metric": METRIC, "value": value, "unit": "heads/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak" if my_heads is None else "strong",
        "vs_baseline": None, "dtype": "bf16" if Q.dtype == torch.bfloat16 else "fp32",
        "data": "synthetic: seeded structured heads shaped like the pages' workloads (no datasets or weights)",
        "config": cfg, "roofline": rf, "gpu_launches": launches, "clocks": clk,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
    print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    del first
    return 0


def run_online(args, rank, world, local_rank):
    """Online compaction, Qwen3-4B shaped: 288 heads, cache 2048, six rounds that
    each halve all but the latest 20 keys (t = 1014 of 2028), n = 2048.  Every
    round's am_compact_heads runs on inputs already in HBM and is timed with
    CUDA events; the next round is assembled from this round's outputs on the
    host (outside the timed region).  e2e adds each round's host-to-device
    copy of its inputs and the copy back of its outputs."""
    import numpy as np
    import torch
    import attention_matching_b200 as am
    from attention_matching_b200 import workloads as W
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    H = args.heads or 288
    rounds = 6
    on = W.OnlineHeads(H, seed=3000 + 1000 * rank)
    stream = torch.cuda.current_stream(dev)
    ws = None
    compacted, times, e2e_times, stages_all, first_heads = None, [], [], {}, None
    h2d = d2h = 0
    clocks = ClockSampler(gpu_smi_id(torch, local_rank))
    launches = 0
    for rnd in range(rounds):
        heads = on.next_round(compacted)
        if first_heads is None:
            first_heads = heads
        Qh = torch.stack([h.Q for h in heads]).pin_memory()
        Kh = torch.stack([h.K for h in heads]).pin_memory()
        Vh = torch.stack([h.V for h in heads]).pin_memory()
        kbh = torch.tensor(np.stack([h.key_bias for h in heads])).pin_memory()
        budgets = [on.budget] * H
        if ws is None:
            opts = am.make_opts(am.BF16, 4, 2)
            ws = torch.empty((am.workspace_size(on.n, on.compact_len, on.d, budgets, opts),),
                             dtype=torch.uint8, device=dev)
            # untimed warm-up calls on the first round's inputs (they feed nothing forward)
            for _ in range(args.warmup):
                Qw, Kw, Vw, kbw = (x.to(dev, non_blocking=True) for x in (Qh, Kh, Vh, kbh))
                am.compact_heads(Qw, Kw, Vw, budgets, topk=4, refit_every=2, key_bias=kbw, workspace=ws,
                                 check=False)
            torch.cuda.synchronize()
            clocks.start()
            clocks.wait_first()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        Q, K, V, kb = (x.to(dev, non_blocking=True) for x in (Qh, Kh, Vh, kbh))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        l0 = am.kernel_launches()
        out = am.compact_heads(Q, K, V, budgets, topk=4, refit_every=2, key_bias=kb, workspace=ws, check=False)
        b.record(stream)
        host = {k: out[k].to("cpu", non_blocking=True) for k in ("C_k", "beta", "C_v", "indices")}
        e1 = torch.cuda.Event(enable_timing=True)
        e1.record(stream)
        torch.cuda.synchronize()
        launches += am.kernel_launches() - l0
        times.append(a.elapsed_time(b))
        e2e_times.append(e0.elapsed_time(e1))
        h2d = sum(x.numel() * x.element_size() for x in (Qh, Kh, Vh, kbh))
        d2h = sum(x.numel() * x.element_size() for x in host.values())
        cu = out["cu_t"].tolist()
        Ck, beta, Cv = host["C_k"].float().numpy(), host["beta"].numpy(), host["C_v"].numpy()
        compacted = [(Ck[cu[h]:cu[h + 1]], beta[cu[h]:cu[h + 1]], Cv[cu[h]:cu[h + 1]]) for h in range(H)]
    clk = clocks.stop()
    _, worst = am.get_status(ws, H)
    # stage times: the first round's inputs once more with the event brackets
    Q = torch.stack([h.Q for h in first_heads]).to(dev)
    K = torch.stack([h.K for h in first_heads]).to(dev)
    V = torch.stack([h.V for h in first_heads]).to(dev)
    kb = torch.tensor(np.stack([h.key_bias for h in first_heads]), device=dev)
    am.profile_enable(True)
    am.compact_heads(Q, K, V, [on.budget] * H, topk=4, refit_every=2, key_bias=kb, workspace=ws, check=False)
    torch.cuda.synchronize()
    am.profile_enable(False)
    stages = am.profile_collect()
    total_ms = sum(times)
    n, T, d, ldn = on.n, on.compact_len, on.d, (on.n + 31) // 32 * 32

    class _WL:
        topk, refit_every, budgets, name = 4, 2, [on.budget] * H, f"online_rounds_H{H}"
    models = stage_models(_WL, n, [T] * H, d, ldn, "bounded", 0, True)
    models.pop("rows", None)
    rf = roofline(stages, 1, models, load_peaks(), clk, {})
    line = {
        "metric": METRIC, "value": job_throughput(H * rounds, 1, total_ms), "unit": "heads/s", "n_gpus": 1,
        "steps": rounds, "warmup": args.warmup, "ms_per_step": total_ms / rounds, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded structured heads, online rounds chained on the GPU's own outputs",
        "config": {"workload": f"online_rounds_H{H}_cache2048_keep20_t{on.budget}_n2048_d128_x{rounds}",
                   "round_ms": times, "s_per_6_rounds": total_ms * 1e-3,
                   "stage_ms_round1": {k: round(v["ms"], 3) for k, v in stages.items() if v["launches"]},
                   "device_status": worst,
                   "l2": "each round's inputs (288 heads x 2028 keys) are larger than L2"},
        "roofline": rf, "gpu_launches": launches, "clocks": clk,
        "e2e": {"value": job_throughput(H * rounds, 1, sum(e2e_times)), "unit": "heads/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": sum(e2e_times) / rounds},
    }
    if not args.no_cpu_baseline:
        from attention_matching_b200.workloads import Workload
        line["cpu_baseline"] = cpu_baseline(Workload("online_round1", first_heads, [on.budget] * H, 4, 2, "bf16"),
                                            args.cpu_seconds)
        line["cpu_baseline"]["sample"] += " (round 1 only; key_bias ignored by this sample, all zeros in round 1)"
    print(json.dumps(line))
    return 0


def run_consume(args, local_rank):
    """Attention over a compacted cache (am_attend_packed): the workload's
    heads are compacted once, then each head's --queries reference queries
    attend over its compacted segment plus T_NEW fresh keys."""
    import torch
    import attention_matching_b200 as am
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = build_workload(args.workload, 0, args.heads)
    H, d = len(wl.heads), wl.heads[0].d
    Q = torch.stack([h.Q for h in wl.heads]).contiguous().to(dev)
    K = torch.stack([h.K for h in wl.heads]).contiguous().to(dev)
    V = torch.stack([h.V for h in wl.heads]).contiguous().to(dev)
    packed = am.compact_heads(Q, K, V, wl.budgets, topk=wl.topk, refit_every=wl.refit_every)
    g = torch.Generator(device="cpu").manual_seed(7)
    Tn, nq = args.consume, min(args.queries, wl.heads[0].n)
    Kn = torch.randn((H, Tn, d), generator=g).to(Q.dtype).to(dev)
    Vn = torch.randn((H, Tn, d), generator=g).to(Q.dtype).to(dev)
    Qd = Q[:, :nq].contiguous()
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        am.attend_packed(Qd, packed, Kn, Vn)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    clocks = ClockSampler(gpu_smi_id(torch, local_rank))
    clocks.start()
    clocks.wait_first()
    evs = []
    for _ in range(args.steps):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        am.attend_packed(Qd, packed, Kn, Vn)
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    esz = Q.element_size()
    t_sum = sum(wl.budgets)
    # every operand read once and the output written once
    algo = t_sum * (d * esz + 4 + d * 4) + H * (2 * Tn * d * esz + nq * d * esz + nq * d * 4)
    peaks = load_peaks()
    ach = algo / (ms * 1e-3) / 1e9
    line = {
        "metric": "attention over a compacted cache plus fresh keys", "value": H * nq / (ms * 1e-3),
        "unit": "queries/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if esz == 2 else "fp32", "data": "synthetic",
        "config": {"workload": wl.name, "heads": H, "budgets_total": t_sum, "fresh_keys": Tn,
                   "queries_per_head": nq, "d": d, "l2": "256 MiB buffer written between timed steps"},
        "roofline": {"kernel": "k_attend", "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": ach / peaks["hbm_gbs"], "algorithmic_bytes": algo,
                     "traffic": None},
        "gpu_launches": args.steps, "clocks": clk,
    }
    print(json.dumps(line))
    return 0


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.consume is not None:
        return run_consume(args, local_rank)
    if args.workload == "online_rounds":
        return run_online(args, rank, world, local_rank)
    return run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
