#!/usr/bin/env python
"""Benchmark: forward + backward of causal factorized sparse attention.

One step = sparse_attn_fwd + sparse_attn_bwd (through the C ABI) on every
workload of the step.  The default step holds both N = 12288 workloads, so
it runs every kernel of the hot path (natural, column and summary views):
  text-fixed      fixed pattern,   B=2 H=8  N=12288 D=64 l=128 c=32 block=64
  image64-strided strided pattern, B=1 H=16 N=12288 D=64 l=192      block=64
Metric: nonzero-block TFLOP/s, counted on the public block tables
(4 b^2 D per nonzero block forward, 10 b^2 D backward, per batch and head),
and tokens/s = B*N per workload / step time.  Inputs are seeded N(0,1)
bf16 tensors (synthetic; no dataset).

Timing: W untimed warm-up steps, then exactly K steps, each bracketed by
CUDA events on the launching stream, with a 256 MiB write between steps to
flush L2; barrier + synchronize around the timed loop; max over ranks.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from factorized_block_sparse_b200 import synth  # noqa: E402

METRIC = "fwd+bwd nonzero-block TFLOP/s (% of B200 BF16 peak) and tokens/s at N=12288"
STEPS = {
    "n12288": ["text-fixed", "image64-strided"],
    # the strided image64 pattern as two heads (row head + column head, own softmax each)
    "image64-two-head": ["image64-local", "image64-column"],
}
for _n in synth.WORKLOADS:
    STEPS[_n] = [_n]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(bf16=p["bf16_tflops"], bf16_sustained=p["bf16_tflops_sustained"], hbm=p["hbm_gbs"],
                    source="measured")
    return dict(bf16=1590.0, bf16_sustained=1400.0, hbm=6650.0, source="fallback")


# ----------------------------------------------------------------- flop counts
def block_counts(w, sa=None):
    """Nonzero public blocks per view of a workload (from the library's table)."""
    if sa is not None:
        lay = sa.Layout(w["mode"], w["N"], w["l"], w["c"], w["block"])
        views = {"strided": ("N", "T"), "fixed": ("N", "S"), "column": ("T",)}.get(w["mode"], ("N",))
        return {v: len(lay.export(v)["col_idx"]) for v in views}, lay
    raise ValueError("library needed")


def flops(w, counts):
    per = w["block"] ** 2 * w["D"] * w["B"] * w["H"]
    nnz = sum(counts.values())
    return 4 * per * nnz, 10 * per * nnz


def element_nnz(w):
    """(query, key) pairs per head in the workload's mask (element level)."""
    import numpy as np

    N, l, c, mode = w["N"], w["l"], w["c"], w["mode"]
    i = np.arange(N, dtype=np.int64)
    if mode == "all":
        return N * (N + 1) // 2
    if mode == "local":
        return int(np.minimum(i + 1, l).sum())
    if mode == "strided":  # window of l (diagonal included) + earlier positions of the column
        return int(np.minimum(i + 1, l).sum() + (i // l).sum())
    if mode == "fixed":  # own block (causal) + the last c offsets of every earlier block
        return int(((i % l) + 1).sum() + ((i // l) * c).sum())
    if mode == "column":  # earlier positions of the column and the position itself
        return int((i // l + 1).sum())
    if mode == "block":  # own block, causal
        return int(((i % l) + 1).sum())
    raise ValueError(mode)


def algorithmic_bytes(w):
    """Minimal HBM bytes of forward + backward: q, k, v read and o, lse written (forward); q, k, v, o,
    dO, lse read and dq, dk, dv written (backward); the strided merge re-reads and re-writes o, lse."""
    D, rows = w["D"], w["B"] * w["H"] * w["N"]
    b = rows * ((8 * D + 4) + (16 * D + 4))
    if w["mode"] == "strided":
        b += rows * (4 * D + 8)
    return b


def workload_lines(state, ktimes, pk):
    """Per-workload kernel time (sum of its kernels' mean launch times, CUDA events), throughput
    and fraction of the workload's own roofline max(flops / bf16 peak, algorithmic bytes / HBM peak)."""
    modes = [s["w"]["mode"] for s in state]
    if len(set(modes)) != len(modes):
        return None  # kernel times are kept per pattern
    out = {}
    for s in state:
        w, m = s["w"], s["w"]["mode"]
        t = {"fwd": 0.0, "bwd": 0.0}
        for name, (ms, c) in ktimes.items():
            if c and name.endswith("." + m):
                t["fwd" if name.startswith("sa_fwd") else "bwd"] += ms / c
        ms = t["fwd"] + t["bwd"]
        fl = s["flops"]
        el = element_nnz(w) * w["B"] * w["H"] * 14 * w["D"]  # 4D (QK^T, PV) + 10D (backward) per pair
        by = algorithmic_bytes(w)
        t_tc = fl / (pk["bf16"] * 1e12) * 1e3
        t_hbm = by / (pk["hbm"] * 1e9) * 1e3
        out[s["name"]] = {
            "fwd_ms": round(t["fwd"], 4), "bwd_ms": round(t["bwd"], 4),
            "nonzero_block_tflops": round(fl / (ms * 1e-3) / 1e12, 2),
            "element_tflops": round(el / (ms * 1e-3) / 1e12, 2),
            "tokens_per_s": round(w["B"] * w["N"] / (ms * 1e-3), 1),
            "roofline": {"bound": "tensor" if t_tc >= t_hbm else "hbm", "tensor_ms": round(t_tc, 4),
                         "hbm_ms": round(t_hbm, 4), "frac": round(max(t_tc, t_hbm) / ms, 4)},
        }
    return out


def kernel_units(w, counts):
    """Algorithmic work per launch of each kernel of a workload (flops or bytes)."""
    per = w["block"] ** 2 * w["D"] * w["B"] * w["H"]
    rows = w["B"] * w["H"] * w["N"]
    D = w["D"]
    m = w["mode"]
    sec = counts.get("T", 0) + counts.get("S", 0)
    fwd_main = counts.get("N", 0) + (counts.get("S", 0) if m == "fixed" else 0)
    out = {
        f"sa_bwd_preprocess.{m}": ("hbm", rows * (2 * D * 2 + 4)),
        f"sa_bwd_finalize_dq.{m}": ("hbm", rows * D * (4 + 2)),
    }
    if m == "fixed" and w.get("c"):  # the summary keys' dK, dV: two fp32 rows read, two bf16 rows written
        out[f"sa_bwd_finalize_summary_dkv.{m}"] = ("hbm", w["B"] * w["H"] * (w["N"] // w["l"]) * w["c"] * D * 12)
    if "N" in counts:
        out[f"sa_fwd_natural_view.{m}"] = ("tensor", 4 * per * fwd_main)
        out[f"sa_bwd_natural_view.{m}"] = ("tensor", 10 * per * counts["N"])
    if "T" in counts:
        out[f"sa_fwd_column_view.{m}"] = ("tensor", 4 * per * counts["T"])
    if sec:
        out[f"sa_bwd_secondary_view.{m}"] = ("tensor", 10 * per * sec)
    return out


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons, power = [], None, set(), []
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ----------------------------------------------------------------- distributed
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(value, world, device):
    """Max of a float over ranks (identity for one rank)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job(world, step_flops, step_tokens, local_ms_total, steps, device=None):
    """Whole-job throughput of a weak-scaled run: every rank does the same work
    on its own data; the time is the slowest rank's (max over ranks)."""
    ms_step = max_over_ranks(local_ms_total, world, device) / steps
    return world * step_flops / (ms_step * 1e-3) / 1e12, world * step_tokens / (ms_step * 1e-3), ms_step


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ----------------------------------------------------------------- CPU oracle
def oracle_nnz(w):
    """Nonzero public blocks per (batch, head) of a workload, from the oracle's tables."""
    from oracle import views as oviews

    return sum(oviews.block_nonzeros(w["mode"], w["N"], w["l"], w["c"], w["block"]).values())


def oracle_inputs(names):
    out = []
    for n in names:
        w = synth.WORKLOADS[n]
        # a [1, 1, N, D] draw equals slice (b=0, h=0) of the full workload's draw
        out.append((w, synth.inputs(1, 1, w["N"], w["D"]), oracle_nnz(w)))
    return out


def oracle_sample_step(ws, step_idx, rows_per=512):
    """Bounded oracle sample: query rows [r0, r0+rows_per) of slice (0, 0) of
    each workload; forward rows (O, lse) and dQ rows with the float64 oracle
    as it stands.  Returns (seconds, credited flops).  Credit: 10 b^2 D
    (QK^T, PV, the recomputed QK^T, dO V^T, dS K) per nonzero public block,
    times rows_per / N of the head's blocks (the chunk start rotates over the
    sequence from step to step)."""
    from oracle import attention

    total_s, total_f = 0.0, 0.0
    for w, x, nnz in ws:
        N, b, D = w["N"], w["block"], w["D"]
        n_chunks = N // rows_per
        r0 = (step_idx % n_chunks) * rows_per
        rows = list(range(r0, r0 + rows_per))
        q, k, v, dO = (synth.to_f64(x[n]) for n in ("q", "k", "v", "dO"))
        t0 = time.perf_counter()
        attention.forward_rows(q, k, v, w["mode"], w["l"], w["c"], rows)
        attention.dq_rows(q, k, v, dO, w["mode"], w["l"], w["c"], rows)
        total_s += time.perf_counter() - t0
        total_f += 10 * b * b * D * nnz * rows_per / N
    return total_s, total_f


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        info = threadpool_info()
        n = [i.get("num_threads") for i in info if i.get("user_api") == "blas"]
        return int(n[0]) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(names, seconds_budget=15.0):
    ws = oracle_inputs(names)
    oracle_sample_step(ws, 0, 128)  # first touch
    spent, fl, steps = 0.0, 0, 0
    while spent < seconds_budget and steps < 48:
        s, f = oracle_sample_step(ws, steps)
        spent += s
        fl += f
        steps += 1
    return {"value": fl / spent / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "seconds": round(spent, 2),
            "sample": f"{steps} chunks of 512 query rows of slice (b=0,h=0) of each of {names}: float64 "
                      "oracle forward rows + dQ rows; credited 10 b^2 D per nonzero block, pro rata of rows"}


def run_reference(args, names):
    world, rank, _ = dist_setup_cpu_only()
    if rank != 0:
        return 0
    ws = oracle_inputs(names)
    for i in range(args.warmup):
        oracle_sample_step(ws, i, 256)
    spent, fl = 0.0, 0
    for i in range(args.steps):
        s, f = oracle_sample_step(ws, i, 256)
        spent += s
        fl += f
    value = fl / spent / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * spent / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(names, args),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"per step: 256 query rows of slice (b=0,h=0) of each of {names}; float64 "
                                   "oracle forward rows + dQ rows; credited 10 b^2 D per nonzero block, pro rata of rows"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def dist_setup_cpu_only():
    return int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0


def config_dict(names, args):
    ws = [synth.WORKLOADS[n] for n in names]
    return {
        "workload": " + ".join(
            f"{n}({w['mode']}, B={w['B']}, H={w['H']}, N={w['N']}, D={w['D']}, l={w['l']}"
            + (f", c={w['c']}" if w["mode"] == "fixed" else "") + f", block={w['block']})"
            for n, w in zip(names, ws)) + ", fwd+bwd",
        "global_batch": sum(w["B"] for w in ws) * max(1, args.gpus),
        "seq_len": ws[0]["N"],
        "parallelism": f"replicas x{max(1, args.gpus)} (independent (batch, head) work per GPU, no collective)",
        "l2": "flushed between timed steps (256 MiB write outside the events)",
        "streams": getattr(args, "streams", 1),
    }


# ----------------------------------------------------------------- main arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="n12288", choices=sorted(STEPS))
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--configs", type=int, default=1, help="1: also time every other named configuration")
    ap.add_argument("--streams", type=int, default=2, help="streams the step's independent workloads use")
    ap.add_argument("--block", type=int, default=1, help="1: also time the Sparse Transformer block around the op")
    args = ap.parse_args()
    names = STEPS[args.workload]
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args, names)

    import torch

    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from factorized_block_sparse_b200 import sparse_attn as sa

    pk = peaks()
    # inputs resident in HBM
    state = []
    fl_fwd = fl_bwd = 0
    units = {}
    for n in names:
        w = synth.WORKLOADS[n]
        counts, lay = block_counts(w, sa)
        f0, f1 = flops(w, counts)
        fl_fwd += f0
        fl_bwd += f1
        units.update(kernel_units(w, counts))
        x = synth.inputs(w["B"], w["H"], w["N"], w["D"], seed_offset=rank)
        q, k, v, dO = (x[t].to(dev) for t in ("q", "k", "v", "dO"))
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = sa.workspace(w["B"], w["H"], w["N"], w["D"], lay, dev)
        lay.upload()
        state.append(dict(w=w, name=n, flops=f0 + f1, lay=lay, x=x, q=q, k=k, v=v, dO=dO, o=o, lse=lse, dq=dq,
                          dk=dk, dv=dv, ws=ws))
    stream = torch.cuda.current_stream()
    sptr = stream.cuda_stream
    # The step's workloads are independent problems: with --streams 2 the
    # second one is issued on its own stream (forked from and joined back to
    # the launching stream inside the step), so their kernels can overlap.
    streams = [stream] + [torch.cuda.Stream(device=dev) for _ in range(min(args.streams, len(state)) - 1)]

    def run_one(s, strm):
        p = strm.cuda_stream
        sa.sparse_attn_fwd(s["q"], s["k"], s["v"], s["o"], s["lse"], s["lay"], p)
        sa.sparse_attn_bwd(s["q"], s["k"], s["v"], s["o"], s["lse"], s["dO"], s["dq"], s["dk"], s["dv"],
                           s["lay"], s["ws"], p)

    def step(serial=False):
        if serial or len(streams) == 1:
            for s in state:
                run_one(s, stream)
            return
        fork = torch.cuda.Event()
        fork.record(stream)
        for strm in streams[1:]:
            strm.wait_event(fork)
        for i, s in enumerate(state):
            run_one(s, streams[i % len(streams)])
        for strm in streams[1:]:
            join = torch.cuda.Event()
            join.record(strm)
            stream.wait_event(join)

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = sa.sparse_attn_status()
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {sa.strerror(st)}")

    def timed(per_kernel):
        """K steps, each bracketed by CUDA events on the launching stream, L2
        flushed before each; with per_kernel the library also brackets every
        launch with events (which serialises the launches)."""
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        barrier(world)
        torch.cuda.synchronize()
        sa.timing_reset()
        sa.timing_enable(per_kernel)
        n0 = sa.launch_count()
        for i in range(args.steps):
            flush.zero_()
            evs[i][0].record(stream)
            step(serial=per_kernel)  # per-launch events: one stream, so each launch's events bracket it alone
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        n = sa.launch_count() - n0
        sa.timing_enable(False)
        kt = sa.kernel_times()
        st = sa.sparse_attn_status()
        if st != 0:
            raise RuntimeError(f"device status after timing: {sa.strerror(st)}")
        return sum(a.elapsed_time(b) for a, b in evs), n, kt

    # the headline: K steps with no per-launch events in between
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    local_ms, launches, _ = timed(False)
    clocks = sampler.stop()
    # the per-kernel breakdown and the roofline: K more steps with every launch bracketed by events
    kernel_pass_ms, _, ktimes = timed(True)
    step_flops = fl_fwd + fl_bwd
    value, tokens_per_s, ms_step = whole_job(world, step_flops, sum(s["w"]["B"] * s["w"]["N"] for s in state),
                                             local_ms, args.steps, dev)

    # dominant kernel of the timed region
    dom, dom_ms = None, -1.0
    for name, (ms, cnt) in ktimes.items():
        if cnt and name in units and ms > dom_ms:
            dom, dom_ms = name, ms
    cnt = ktimes[dom][1]
    bound, per_launch = units.get(dom, ("tensor", None))
    avg_ms = dom_ms / cnt
    if bound == "tensor":
        achieved = per_launch / (avg_ms * 1e-3) / 1e12
        peak, unit = pk["bf16"], "TFLOP/s"
    else:
        achieved = per_launch / (avg_ms * 1e-3) / 1e9
        peak, unit = pk["hbm"], "GB/s"
    traffic = read_traffic(dom)
    kernels = {n: {"ms_per_launch": round(ms / c, 4), "launches": c,
                   **({"achieved": round(units[n][1] / (ms / c * 1e-3) / (1e12 if units[n][0] == "tensor" else 1e9), 2),
                       "unit": "TFLOP/s" if units[n][0] == "tensor" else "GB/s"} if n in units else {})}
               for n, (ms, c) in ktimes.items() if c}

    # every other named configuration, one at a time (extra keys; the headline stays the step above)
    configs = None
    if args.configs and world == 1:
        configs = measure_configs(sa, [n for n in CONFIGS if n not in names], pk, dev, stream, flush)

    # the Sparse Transformer block around the op (extra key)
    block = None
    if args.block and world == 1:
        block = measure_block(sa, pk, dev, stream, flush)

    # end to end through the C ABI with pinned host buffers
    e2e = None
    if args.e2e_steps > 0:
        e2e = measure_e2e(sa, state, stream, args.e2e_steps, step_flops, world, dev)

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded iid N(0,1), rounded to bf16)",
        "config": config_dict(names, args),
        "tokens_per_s": round(tokens_per_s, 1),
        "pct_of_bf16_peak": round(100 * value / (world * pk["bf16"]), 2),
        "pct_of_bf16_sustained": round(100 * value / (world * pk["bf16_sustained"]), 2),
        "peak_source": pk["source"],
        "flops_per_step": {"fwd": fl_fwd, "bwd": fl_bwd},
        "roofline": {"kernel": dom, "bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_kind": "burst (of measured)" if pk["source"] == "measured" else "fallback"},
        "kernels": kernels,
        "kernel_pass": {"ms_per_step": round(max_over_ranks(kernel_pass_ms, world, dev) / args.steps, 4),
                        "note": "per-kernel events are taken in a second pass of K steps on one stream with "
                                "every launch bracketed by events; the headline steps run without them, the "
                                "step's workloads on their own streams"},
        "workloads": workload_lines(state, ktimes, pk),
        "configs": configs,
        "block": block,
        "gpu_launches": launches,
        "clocks": clocks,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(names, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


# The configurations the metric names besides the step's own (the tiny,
# image32, dense image64 and audio shapes) and the two longer sequences.
CONFIGS = ["tiny-strided", "image32-strided", "image64-all", "audio-strided", "long-strided-262144",
           "long-strided-1048576"]


def measure_configs(sa, names, pk, dev, stream, flush, steps=10, warmup=3):
    """fwd + bwd of each named workload alone: ms per step (CUDA events around
    each step, L2 flushed before it), nonzero-block TFLOP/s, tokens/s and the
    fraction of the workload's own roofline max(flops / bf16 peak, algorithmic
    bytes / HBM peak).  Inputs: seeded N(0, 1) drawn on the device."""
    import torch

    out = {}
    for n in names:
        w = synth.WORKLOADS[n]
        counts, lay = block_counts(w, sa)
        f0, f1 = flops(w, counts)
        gen = torch.Generator(device=dev)
        gen.manual_seed(1234)
        shape = (w["B"], w["H"], w["N"], w["D"])
        q, k, v, dO = (torch.randn(shape, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
                       for _ in range(4))
        o = torch.empty_like(q)
        lse = torch.empty(shape[:3], dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = sa.workspace(w["B"], w["H"], w["N"], w["D"], lay, dev)
        lay.upload()
        sptr = stream.cuda_stream

        def one():
            sa.sparse_attn_fwd(q, k, v, o, lse, lay, sptr)
            sa.sparse_attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, lay, ws, sptr)

        for _ in range(warmup):
            one()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            flush.zero_()
            evs[i][0].record(stream)
            one()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        st = sa.sparse_attn_status()
        if st != 0:
            raise RuntimeError(f"device status after {n}: {sa.strerror(st)}")
        ms = sum(a.elapsed_time(b) for a, b in evs) / steps
        t_tc = (f0 + f1) / (pk["bf16"] * 1e12) * 1e3
        t_hbm = algorithmic_bytes(w) / (pk["hbm"] * 1e9) * 1e3
        out[n] = {"workload": f"{w['mode']}, B={w['B']}, H={w['H']}, N={w['N']}, D={w['D']}, l={w['l']}"
                              + (f", c={w['c']}" if w["mode"] == "fixed" else "") + f", block={w['block']}",
                  "ms_per_step": round(ms, 4), "nonzero_block_tflops": round((f0 + f1) / (ms * 1e-3) / 1e12, 2),
                  "tokens_per_s": round(w["B"] * w["N"] / (ms * 1e-3), 1),
                  "roofline": {"bound": "tensor" if t_tc >= t_hbm else "hbm", "frac": round(max(t_tc, t_hbm) / ms, 4)}}
        del q, k, v, dO, o, lse, dq, dk, dv, ws
        lay.close()
        torch.cuda.empty_cache()
    return out


def block_flops(w, counts, C):
    """FLOPs of one forward + backward of the block (the backward recomputes
    the forward but for y): projections 2 M K Nn each, 24 M C^2 in the
    forward and 16 + 48 M C^2 in the backward; the attention's nonzero-block
    FLOPs forward, again in the backward's recomputation, and backward."""
    M = w["B"] * w["N"]
    fa, ba = flops(w, counts)
    return (24 + 64) * M * C * C + 2 * fa + ba, (24 + 64) * M * C * C


def measure_block(sa, pk, dev, stream, flush, steps=10, warmup=3):
    """forward + backward of the Sparse Transformer block at the text-fixed
    shape (B=2, N=12288, H=8, D=64: C=512, the fixed pattern), CUDA events
    around each step, L2 flushed before it; random-init parameters."""
    import torch

    from factorized_block_sparse_b200 import sparse_block as sb

    w = synth.WORKLOADS["text-fixed"]
    B, N, H, D = w["B"], w["N"], w["H"], w["D"]
    C = H * D
    counts, lay = block_counts(w, sa)
    fl, fl_gemm = block_flops(w, counts, C)
    xin = synth.block_inputs(B, N, C)
    x, dy = xin["x"].to(dev), xin["dy"].to(dev)
    p = {k: v.to(dev) for k, v in synth.block_params(C).items()}
    ws = sb.workspace(B, N, H, D, lay, dev)
    y = torch.empty_like(x)
    dx = torch.empty_like(x)
    g = {n: torch.empty(p[n].shape, dtype=torch.float32, device=dev) for n in sb.PARAMS}
    sptr = stream.cuda_stream

    def one():
        sb.sparse_block_fwd(x, p, y, H, lay, ws, sptr)
        sb.sparse_block_bwd(x, dy, p, dx, g, H, lay, ws, sptr)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        evs[i][0].record(stream)
        one()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    st = sa.sparse_attn_status()
    if st != 0:
        raise RuntimeError(f"device status after the block: {sa.strerror(st)}")
    ms = sum(a.elapsed_time(b) for a, b in evs) / steps
    achieved = fl / (ms * 1e-3) / 1e12
    out = {"workload": f"one block, fixed pattern, B={B}, N={N}, H={H}, D={D} (C={C}, hidden {4 * C}), l={w['l']}, "
                       f"c={w['c']}, block={w['block']}; bf16 activations, cuBLAS and cuBLASLt projections",
           "ms_per_step": round(ms, 4), "tflops": round(achieved, 2), "unit": "TFLOP/s",
           "flops_per_step": {"total": fl, "projections": fl_gemm},
           "tokens_per_s": round(B * N / (ms * 1e-3), 1),
           "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": pk["bf16"],
                        "frac": round(achieved / pk["bf16"], 4)}}
    del x, dy, p, ws, y, dx, g
    lay.close()
    torch.cuda.empty_cache()
    return out


def measure_e2e(sa, state, stream, steps, step_flops, world, dev):
    """The step through the public API from pinned host buffers: every step
    copies its inputs (q, k, v, dO) host->device and its results (o, lse, dq,
    dk, dv) device->host.  Steps are pipelined over two device buffer sets and
    three streams (host->device copies, compute, device->host copies), so one
    step's copies in each direction overlap the neighbouring steps' compute
    and opposite copies, as a training loop feeding the op from the host would
    run; the value is the time from the first copy to the last one over the
    steps."""
    import torch

    h2d = d2h = 0
    hin = []
    for s in state:
        t_in = {t: s["x"][t].pin_memory() for t in ("q", "k", "v", "dO")}
        h2d += sum(t.numel() * t.element_size() for t in t_in.values())
        hin.append(t_in)
    # two device sets (set 0 is the bench's own tensors) and a pinned output set per device set
    sets = [state, [dict(s, **{t: torch.empty_like(s[t]) for t in ("q", "k", "v", "dO", "o", "lse", "dq", "dk", "dv")},
                         ws=torch.empty_like(s["ws"])) for s in state]]
    hout = [[{t: torch.empty(s[t].shape, dtype=s[t].dtype, pin_memory=True) for t in ("o", "lse", "dq", "dk", "dv")}
             for s in state] for _ in range(2)]
    d2h = sum(t.numel() * t.element_size() for h in hout[0] for t in h.values())
    s_in, s_out, s_c = torch.cuda.Stream(dev), torch.cuda.Stream(dev), stream
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    cptr = s_c.cuda_stream

    def one(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_c[b])  # step i-2 has consumed this set's inputs
            for d, h in zip(sets[b], hin):
                for t in ("q", "k", "v", "dO"):
                    d[t].copy_(h[t], non_blocking=True)
            ev_in[b].record(s_in)
        s_c.wait_event(ev_in[b])
        if i >= 2:
            s_c.wait_event(ev_out[b])  # step i-2's results have left this set
        for d in sets[b]:
            sa.sparse_attn_fwd(d["q"], d["k"], d["v"], d["o"], d["lse"], d["lay"], cptr)
            sa.sparse_attn_bwd(d["q"], d["k"], d["v"], d["o"], d["lse"], d["dO"], d["dq"], d["dk"], d["dv"],
                               d["lay"], d["ws"], cptr)
        ev_c[b].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_c[b])
            for d, h in zip(sets[b], hout[b]):
                for t in ("o", "lse", "dq", "dk", "dv"):
                    h[t].copy_(d[t], non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record(s_in)
    for i in range(steps):
        one(i)
    s_out.wait_event(ev_c[(steps - 1) % 2])
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / steps
    return {"value": round(world * step_flops / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelined": "two device buffer sets; host->device copies, compute and device->host copies on "
                         "three streams"}


def read_traffic(kernel):
    """Per-launch DRAM bytes of `kernel` from profiles/dram_traffic.txt, if the
    recorded kernel source hash still matches the current sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    cur = source_hash()
    for line in open(path):
        parts = line.split()
        if len(parts) >= 3 and not line.startswith("#") and parts[0] == kernel and parts[1] == cur:
            return float(parts[2])
    return None


def source_hash():
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "factorized_block_sparse_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        if not fn.startswith("sa_"):  # the attention library's sources (not the block around it)
            continue
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


if __name__ == "__main__":
    sys.exit(main())
