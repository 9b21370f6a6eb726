#!/usr/bin/env python
"""Benchmark of the fused exact-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload llama] [--dtype bf16] [--passes fwd,bwd]

One step = one pass of the whole hot path over one batch of synthetic input:
the forward (and, with the backward built, the backward) of one Llama-3-8B
attention layer, B=1, H=32, Nq=Nk=8192, d_k=128, causal (the shapes of the
FlashAttention case-study slides, "The same computation at real size").

value    = algorithmic TFLOP/s of the step (4*B*H*Nq*Nk*D forward, halved for
           causal; 2.5x that for the backward), inputs resident in HBM, L2
           flushed between steps, timed with CUDA events on the launch stream.
e2e      = the same metric through the public binding with HOST buffers:
           pinned-host -> device copies of every step's inputs and the device
           -> host read of its outputs are inside the timed region (on copy
           streams, overlapped with the kernels of the neighbouring steps).
roofline = the dominant kernel's achieved TFLOP/s against the measured bf16
           tensor-core peak (MEASURED_PEAKS.json).
cpu_baseline = the float64 oracle on a bounded row sample, on host cores.

Under torchrun (N > 1) every rank runs the same per-GPU workload on its own
GPU (independent (batch, head) shards, no collective on the data path): weak
scaling; value = all ranks' FLOPs / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOP/s on 1 B200 and fraction of dense BF16/FP16 peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama")
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "f16", "e4m3"],
                    help="storage type of Q, K, V (e4m3: the FP8 forward, bf16 output)")
    ap.add_argument("--passes", default="fwd,bwd", help="comma list of fwd,bwd")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target oracle CPU time of the cpu_baseline sample")
    ap.add_argument("--flush-mib", type=int, default=512)
    ap.add_argument("--seq-len", type=int, default=None,
                    help="sweep workload only: Nq = Nk = N with B = max(1, 16384 // N)")
    ap.add_argument("--causal", type=int, choices=[0, 1], default=None,
                    help="override the workload's causal flag")
    ap.add_argument("--heads", type=int, default=None,
                    help="override the workload's head count (smaller profiling cases)")
    ap.add_argument("--splits", type=int, default=None,
                    help="forward through fa_fwd_splitkv with this many key ranges "
                         "(default: fa_splitkv_num_splits for the decode workload, else the "
                         "single-pass fa_fwd)")
    return ap.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_cfg(args):
    from exact_attention_112_b200 import inputs
    over = {"dtype": args.dtype}
    if args.seq_len is not None:
        if args.workload != "sweep":
            raise SystemExit("--seq-len applies to the sweep workload only")
        over["N"] = args.seq_len
    if args.causal is not None:
        over["causal"] = bool(args.causal)
    if args.heads is not None:
        over["H"] = args.heads
    w = inputs.workload(args.workload, **over)
    if args.seq_len is not None or args.causal is not None or args.heads is not None:
        # keeps stored ncu traffic (keyed by workload name) off modified shapes
        w["name"] = f"{w['name']}-H{w['H']}-N{w['Nq']}-{'causal' if w['causal'] else 'full'}"
    # stored ncu traffic is looked up by this key; 8-bit inputs move other byte
    # counts than the 16-bit captures
    w["traffic_key"] = w["name"] + ("-e4m3" if w["dtype"] == "e4m3" else "")
    if args.splits is not None:
        w["splits"] = args.splits
    elif args.workload == "decode":
        # the library's own choice for these sizes and this device's SM count
        import torch
        import exact_attention_112_b200 as fa
        sms = torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else 148
        w["splits"] = fa.fa_splitkv_num_splits(w["B"], w["H"], w["Nq"], w["Nk"], sms)
    else:
        w["splits"] = 1
    return w


def flops_of(w, passes):
    from exact_attention_112_b200 import metrics
    f = {}
    if "fwd" in passes:
        f["fwd"] = metrics.fwd_flops(w["B"], w["H"], w["Nq"], w["Nk"], w["D"], w["causal"])
    if "bwd" in passes:
        f["bwd"] = metrics.bwd_flops(w["B"], w["H"], w["Nq"], w["Nk"], w["D"], w["causal"])
    return f


WORKLOAD_TITLES = {"llama": "llama-3-8b layer attention", "bwd": "attention backward workload",
                   "tiny": "tiny attention", "stress": "numerical-stress attention",
                   "sweep": "sequence-sweep attention", "decode": "split-KV decode attention"}


# Algorithmic FLOPs of one launch of each kernel, as multiples of the forward's
# 4*B*H*Nq*Nk*D (halved for causal).  The backward's five tile products
# (S, dP, dV, dK, dQ) are split between the two recompute kernels: the dK/dV
# kernel does S^T, dP^T, dV, dK (4 of 5 = 2.0x forward); the dQ kernel does dQ
# (0.5x forward) plus a recomputation of S and dP that is not algorithmic work.
KERNEL_FWD_MULTIPLE = {"fa_fwd_kernel": 1.0, "fa_fwd_split_kernel": 1.0,
                       "fa_bwd_dkdv_kernel": 2.0, "fa_bwd_dq_kernel": 0.5}
# tile products each kernel executes, as multiples of the forward (2 products)
KERNEL_EXEC_MULTIPLE = {"fa_fwd_kernel": 1.0, "fa_fwd_split_kernel": 1.0,
                        "fa_bwd_dkdv_kernel": 2.0, "fa_bwd_dq_kernel": 1.5}


def max_over_ranks(x, world, device=None):
    """Maximum of a per-rank float over all ranks (identity for one rank)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world, step_flops, steps, t_max_ms):
    """Whole-job TFLOP/s: every rank did `steps` steps of `step_flops`; the job
    took as long as its slowest rank."""
    return world * step_flops * steps / (t_max_ms * 1e-3) / 1e12


def kernel_table(records, w):
    """Per-kernel totals of fa_profile_read() records over the timed steps, with
    each known kernel's algorithmic TFLOP/s and algorithmic HBM GB/s."""
    from exact_attention_112_b200 import metrics
    f1 = metrics.fwd_flops(w["B"], w["H"], w["Nq"], w["Nk"], w["D"], w["causal"])
    elem = 1 if w["dtype"] == "e4m3" else 2
    agg = {}
    for name, ms in records:
        a = agg.setdefault(name, [0, 0.0])
        a[0] += 1
        a[1] += ms
    total = sum(a[1] for a in agg.values()) or 1.0
    out = {}
    for name, (n, ms) in agg.items():
        e = {"launches": n, "ms_per_launch": ms / n, "share": ms / total}
        if name in KERNEL_FWD_MULTIPLE:
            e["algorithmic_tflops"] = KERNEL_FWD_MULTIPLE[name] * f1 / (ms / n * 1e-3) / 1e12
            e["executed_tflops"] = KERNEL_EXEC_MULTIPLE[name] * f1 / (ms / n * 1e-3) / 1e12
        nb = metrics.kernel_bytes(name, w["B"], w["H"], w["Nq"], w["Nk"], w["D"], elem=elem,
                                  bias=w.get("bias_frac", 0) > 0, splits=w.get("splits", 1))
        if nb is not None:
            e["algorithmic_bytes"] = nb
            e["algorithmic_gbs"] = nb / (ms / n * 1e-3) / 1e9
        out[name] = e
    return out


def pick_roofline(kd, peak_tflops, hbm_gbs):
    """The roofline that binds one kernel (a kernel_table entry): HBM when its
    algorithmic FLOP per byte is below the ridge (peak FLOP/s over peak
    bytes/s), else the tensor cores; achieved and peak in the bound's unit."""
    intensity = kd["algorithmic_tflops"] * 1e12 / (kd["algorithmic_gbs"] * 1e9)
    ridge = peak_tflops * 1e12 / (hbm_gbs * 1e9)
    if intensity < ridge:
        r = {"bound": "hbm", "achieved": kd["algorithmic_gbs"], "peak": hbm_gbs, "unit": "GB/s",
             "frac": kd["algorithmic_gbs"] / hbm_gbs}
    else:
        r = {"bound": "tensor", "achieved": kd["algorithmic_tflops"], "peak": peak_tflops, "unit": UNIT,
             "frac": kd["algorithmic_tflops"] / peak_tflops}
    r.update({"algorithmic_bytes_per_launch": kd["algorithmic_bytes"], "flop_per_byte": intensity,
              "ridge_flop_per_byte": ridge})
    return r


def workload_name(w, passes):
    return (f"{WORKLOAD_TITLES.get(w['name'], w['name'])} {'+'.join(passes)}: B={w['B']} H={w['H']} "
            f"Nq={w['Nq']} Nk={w['Nk']} D={w['D']} "
            f"{'causal' if w['causal'] else 'non-causal'} {w['dtype']}"
            + (f", keys in {w['splits']} split-KV ranges" if w.get("splits", 1) > 1 else ""))


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        self.dev = device_index

    def start(self):
        import tempfile
        self.path = tempfile.mktemp(suffix=".csv")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.dev)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[3:]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3])
                          if v.lower().startswith("active")})
        loaded = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(r[2] for r in rows)}


# --------------------------------------------------------------------------
# CPU oracle sample (cpu_baseline and the reference arm)
# --------------------------------------------------------------------------
def oracle_sample_setup(w, passes):
    """Host float64 inputs of the workload for the oracle."""
    from exact_attention_112_b200 import inputs
    inp = inputs.make_inputs(w["B"], w["H"], w["Nq"], w["Nk"], w["D"], dtype=w["dtype"],
                             seed=w["seed"], qk_std=w["qk_std"], v_dist=w["v_dist"],
                             bias_frac=w["bias_frac"], with_dO="bwd" in passes)
    f = inputs.to_f64
    return {k: f(inp[k]) for k in ("q", "k", "v", "key_bias", "do")}


def oracle_rows_time(arrs, w, rows, passes, outputs=None):
    """Run the oracle's passes on the query rows `rows` of every (b, h); return
    (seconds, algorithmic FLOPs of that share of the step).  If `outputs` is a
    dict, the oracle's results are stored in it: o, lse of those rows and the
    exact dQ of those rows (the row-sampled backward's dK, dV hold only the
    sampled rows' share and are not kept)."""
    import numpy as np
    import oracle
    scale = 1.0 / math.sqrt(w["D"])
    t0 = time.perf_counter()
    if "fwd" in passes:
        r = oracle.fwd(arrs["q"], arrs["k"], arrs["v"], arrs["key_bias"], w["causal"], scale,
                       rows=rows)
        if outputs is not None:
            outputs["o"], outputs["lse"] = r
    if "bwd" in passes:
        r = oracle.bwd(arrs["q"], arrs["k"], arrs["v"], arrs["do"], arrs["key_bias"], w["causal"],
                       scale, rows=rows)
        if outputs is not None:
            outputs["dq"] = r[0][:, rows]
    dt = time.perf_counter() - t0
    rows = np.asarray(rows)
    if w["causal"]:
        vis = np.clip(rows + (w["Nk"] - w["Nq"]) + 1, 0, w["Nk"])
    else:
        vis = np.full(rows.shape, w["Nk"])
    per_fwd = 4.0 * w["D"] * float(vis.sum()) * w["B"] * w["H"]
    fl = (per_fwd if "fwd" in passes else 0.0) + (2.5 * per_fwd if "bwd" in passes else 0.0)
    return dt, fl


def pick_rows(w, n, boundaries=False):
    """n evenly spaced query rows (plus, with `boundaries`, the first and last
    row of every 128-row tile), sorted and unique."""
    import numpy as np
    rows = np.linspace(0, w["Nq"] - 1, max(1, n)).round().astype(np.int64)
    if boundaries:
        t = np.arange(0, w["Nq"], 128)
        rows = np.concatenate([rows, t, np.minimum(t + 127, w["Nq"] - 1)])
    return np.unique(rows)


# Acceptance bar of the GPU results against the float64 oracle (the same
# figures the parity tests use): O max-abs error per storage type, LSE max-abs
# error, and gradients max|g - g_ref| / max|g_ref|.
TOL_O = {"f16": 1e-2, "bf16": 2e-2}
TOL_LSE = 1e-3
TOL_GRAD_REL = 5e-2


def parity_report(w, rows, ref, gpu):
    """Compare the GPU's outputs of the benchmarked configuration with the
    oracle's on the sampled rows (O, LSE, dQ: each row depends only on its own
    query and all keys, so the sample is exact for those rows), and check two
    identities that hold at any size for dK and dV (per (b, h) and d):
        sum_j dV_j = sum_i dO_i   over rows that see a key (sum_j P_ij = 1),
        sum_j dK_j = 0            (sum_j dS_ij = D_i - D_i = 0).
    Returns a dict with the errors and `ok`."""
    import numpy as np
    rep, ok = {"rows_per_head": int(len(rows)), "heads": w["B"] * w["H"]}, True
    if "o" in ref:
        o = gpu["o"][:, :, rows]
        lse = gpu["lse"][:, :, rows]
        fin = np.isfinite(ref["lse"])
        same_empty = bool(np.array_equal(np.isfinite(lse), fin))
        err_o = float(np.abs(o - ref["o"]).max())
        err_l = float(np.abs(lse[fin] - ref["lse"][fin]).max()) if fin.any() else 0.0
        rep.update(o_max_abs=err_o, lse_max_abs=err_l, empty_rows_match=same_empty)
        if w["dtype"] == "e4m3":
            # P is rounded to E4M3 (3 mantissa bits) before P.V: per element
            # |O - O_ref| <= 2^-4 A + 2^-8 |O_ref| + 2e-3, A = softmax(S) |V|
            excess = float((np.abs(o - ref["o"]) - (ref["o_absv"] / 16.0 + np.abs(ref["o"]) / 256.0
                                                     + 2e-3)).max())
            rep["o_excess_over_e4m3_bound"] = excess
            ok &= same_empty and excess <= 0.0 and err_l <= TOL_LSE
        else:
            ok &= same_empty and err_o <= TOL_O[w["dtype"]] and err_l <= TOL_LSE
    if "dq" in ref:
        g = gpu["dq"].reshape(w["B"] * w["H"], w["Nq"], w["D"])[:, rows]
        err = float(np.abs(g - ref["dq"]).max() / max(np.abs(ref["dq"]).max(), 1e-30))
        rep["dq_rel_to_max"] = err
        ok &= err <= TOL_GRAD_REL
        # identities for dK and dV (float64 sums of the 16-bit results)
        vis = np.ones(w["Nq"], dtype=bool)
        if w["causal"]:
            vis = np.arange(w["Nq"]) + (w["Nk"] - w["Nq"]) >= 0
        sum_do = gpu["do"][:, :, vis].sum(axis=2)
        sum_dv = gpu["dv"].sum(axis=2)
        e_dv = float(np.abs(sum_dv - sum_do).max() / max(np.abs(sum_do).max(), 1e-30))
        e_dk = float(np.abs(gpu["dk"].sum(axis=2)).max() /
                     max(np.abs(gpu["dk"]).sum(axis=2).max(), 1e-30))
        rep.update(sum_dv_rel=e_dv, sum_dk_rel=e_dk)
        ok &= e_dv <= 1e-2 and e_dk <= 1e-2
    rep["ok"] = bool(ok)
    return rep


def sample_text(w, rows, passes):
    return (f"float64 oracle {'+'.join(passes)} on {len(rows)} evenly spaced query rows of "
            f"each of the {w['B'] * w['H']} (b,h) pairs")


def cpu_baseline(w, target_s, passes, gpu=None):
    """Time the oracle on a bounded row sample of the workload.  With `gpu`
    (host copies of the GPU's outputs for the same inputs), its results on that
    sample are also the parity check of the benchmarked run; returns
    (baseline, parity report or None)."""
    import oracle
    arrs = oracle_sample_setup(w, passes)
    cores = oracle.max_threads()
    dt, fl = oracle_rows_time(arrs, w, pick_rows(w, 8), passes)          # calibration
    n = max(8, int(8 * target_s / max(dt, 1e-3)))
    rows = pick_rows(w, min(n, w["Nq"]), boundaries=gpu is not None)
    ref = {}
    dt, fl = oracle_rows_time(arrs, w, rows, passes, outputs=ref)
    if gpu is not None and w["dtype"] == "e4m3":
        # the E4M3 rounding bound needs softmax(S) |V| on the same rows (untimed)
        import numpy as np
        ref["o_absv"], _ = oracle.fwd(arrs["q"], arrs["k"], np.abs(arrs["v"]), arrs["key_bias"],
                                      w["causal"], 1.0 / math.sqrt(w["D"]), rows=rows)
    base = {"value": fl / dt / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": sample_text(w, rows, passes) + f" ({fl / 1e9:.1f} GFLOP algorithmic, {dt:.1f} s)",
            "seconds": dt,
            # query rows (of every (b, h)) per second, and the whole step's time
            # at the sample's FLOP rate
            "rows_per_s": len(rows) * w["B"] * w["H"] / dt,
            "full_step_s_extrapolated": sum(flops_of(w, passes).values()) / (fl / dt)}
    if w.get("name") == "tiny":
        # the single-thread figure beside the all-core one (the tiny workload
        # is small enough to time whole)
        oracle.set_threads(1)
        try:
            dt1, fl1 = oracle_rows_time(arrs, w, rows, passes)
        finally:
            oracle.set_threads(cores)
        base["one_thread"] = {"value": fl1 / dt1 / 1e12, "seconds": dt1}
    if gpu is None:
        return base, None
    gpu = dict(gpu)
    if "bwd" in passes:
        gpu["do"] = arrs["do"]
    return base, parity_report(w, rows, ref, gpu)


def run_reference(args):
    """The oracle as the reference arm: each step is a bounded row sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    w = workload_cfg(args)
    passes = [p for p in args.passes.split(",") if p]
    arrs = oracle_sample_setup(w, passes)
    cores = oracle.max_threads()
    dt, _ = oracle_rows_time(arrs, w, pick_rows(w, 4), passes)
    budget = 150.0 / max(1, args.steps + args.warmup)   # whole run within a few minutes
    n = max(2, int(4 * budget / max(dt, 1e-4)))
    rows = pick_rows(w, min(n, w["Nq"]))
    for _ in range(args.warmup):
        oracle_rows_time(arrs, w, rows, passes)
    tot_t, tot_f = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl = oracle_rows_time(arrs, w, rows, passes)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(w, passes), "B": w["B"], "H": w["H"],
                   "Nq": w["Nq"], "Nk": w["Nk"], "D": w["D"], "causal": w["causal"],
                   "passes": passes},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": "each step: " + sample_text(w, rows, passes)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
def run_ours(args):
    import torch
    import torch.distributed as dist

    import exact_attention_112_b200 as fa
    from exact_attention_112_b200 import inputs, metrics

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    passes = [p for p in args.passes.split(",") if p]
    w = workload_cfg(args)
    B, H, Nq, Nk, D, causal = w["B"], w["H"], w["Nq"], w["Nk"], w["D"], w["causal"]
    fp8 = w["dtype"] == "e4m3"
    if fp8 and passes != ["fwd"]:
        raise SystemExit("--dtype e4m3 is the FP8 forward: use --passes fwd")
    # every rank draws its own (b, h) shard of a larger batch: seed by rank
    inp = inputs.make_inputs(B, H, Nq, Nk, D, dtype=w["dtype"], seed=w["seed"] + 7 * rank,
                             qk_std=w["qk_std"], v_dist=w["v_dist"], bias_frac=w["bias_frac"],
                             with_dO="bwd" in passes)
    q, k, v = (inp[x].to(dev) for x in ("q", "k", "v"))
    bias = None if inp["key_bias"] is None else inp["key_bias"].to(dev)
    o = torch.empty(q.shape, dtype=torch.bfloat16 if fp8 else q.dtype, device=dev)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    if "bwd" in passes:
        dO = inp["do"].to(dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(fa.fa_bwd_workspace_bytes(B, H, Nq, Nk, D), dtype=torch.uint8, device=dev)
    flush = torch.empty(args.flush_mib * (1 << 20), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    splits = w["splits"]
    if splits > 1:
        ws_split = torch.empty(fa.fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, D, splits),
                               dtype=torch.uint8, device=dev)

    def forward(t=None):
        """The forward pass on the buffer set t (default: the timed buffers)."""
        t = t or {"q": q, "k": k, "v": v, "o": o, "lse": lse}
        if fp8:
            fa.fa_fwd_fp8(t["q"], t["k"], t["v"], t["o"], t["lse"], causal=causal, key_bias=bias,
                          stream=stream)
        elif splits > 1:
            fa.fa_fwd_splitkv(t["q"], t["k"], t["v"], t["o"], t["lse"], splits, ws_split,
                              causal=causal, key_bias=bias, stream=stream)
        else:
            fa.fa_fwd(t["q"], t["k"], t["v"], t["o"], t["lse"], causal=causal, key_bias=bias,
                      stream=stream)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        forward()
        if ev is not None:
            ev[1].record(stream)
        if "bwd" in passes:
            fa.fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, ws, causal=causal, key_bias=bias,
                      stream=stream)
            if ev is not None:
                ev[2].record(stream)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    assert fa.fa_device_status(stream) == fa.FA_OK

    # ---- before timing: the oracle on a row sample (the cpu_baseline leg),
    # whose results also check the outputs of the warm-up steps above
    cpu_line, parity = None, None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gpu_out = {"o": o.float().cpu().numpy(), "lse": lse.cpu().numpy()}
        if "bwd" in passes:
            gpu_out.update({n_: t_.float().cpu().numpy() for n_, t_ in
                            (("dq", dq), ("dk", dk), ("dv", dv))})
        cpu_line, parity = cpu_baseline(w, args.cpu_seconds, passes, gpu_out)
        if not parity["ok"]:
            print(json.dumps({"error": "parity check against the oracle failed",
                              "parity": parity}), file=sys.stderr, flush=True)
            return 1

    n_ev = 3 if "bwd" in passes else 2
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    sampler = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = fa.fa_launch_count()
    fa.fa_profile_read()                   # drop anything recorded before
    fa.fa_profile_enable(True)
    for s in range(args.steps):
        flush.zero_()                      # L2 flush outside the timed events
        step(evs[s])
    torch.cuda.synchronize(dev)
    fa.fa_profile_enable(False)
    launches = fa.fa_launch_count() - launches0
    kernels = kernel_table(fa.fa_profile_read(capacity=16 * args.steps + 64), w)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    st = fa.fa_device_status(stream)
    if st != fa.FA_OK:
        raise RuntimeError(f"device status after timing: {fa.fa_status_string(st)}")

    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    bwd_ms = [e[1].elapsed_time(e[2]) for e in evs] if "bwd" in passes else []
    step_ms = [f + b for f, b in zip(fwd_ms, bwd_ms or [0.0] * len(fwd_ms))]
    t_local = sum(step_ms)
    t_max = max_over_ranks(t_local, world, dev)
    fl = flops_of(w, passes)
    step_flops = sum(fl.values())
    value = weak_scaling_value(world, step_flops, args.steps, t_max)

    # ---- end to end through the public binding, host buffers.  Every step
    # copies its inputs from pinned host memory and reads its outputs back.
    # Two sets of device buffers alternate so that the upload of step i+1 and
    # the read-back of step i run on their own copy streams while the kernels
    # of step i run (the copy engines work beside the SMs).
    names_in = ["q", "k", "v"] + (["do"] if "bwd" in passes else [])
    names_out = ["o", "lse"] + (["dq", "dk", "dv"] if "bwd" in passes else [])
    host = {x: inp[x].pin_memory() for x in names_in}
    sets = [{"q": q, "k": k, "v": v, "o": o, "lse": lse}]
    if "bwd" in passes:
        sets[0].update(do=dO, dq=dq, dk=dk, dv=dv)
    sets.append({n_: torch.empty_like(t_) for n_, t_ in sets[0].items()})
    host_out = {n_: torch.empty(sets[0][n_].shape, dtype=sets[0][n_].dtype).pin_memory()
                for n_ in names_out}
    h2d = sum(t_.numel() * t_.element_size() for t_ in host.values())
    d2h = sum(t_.numel() * t_.element_size() for t_ in host_out.values())
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n, start_ev):
        up.wait_event(start_ev)
        down.wait_event(start_ev)
        for i in range(n):
            b = i % 2
            t = sets[b]
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(ev_done[b])          # step i-2 has read these inputs
                for x in names_in:
                    t[x].copy_(host[x], non_blocking=True)
                ev_in[b].record(up)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])           # step i-2's outputs are read back
            forward(t)
            if "bwd" in passes:
                fa.fa_bwd(t["q"], t["k"], t["v"], t["o"], t["lse"], t["do"], t["dq"], t["dk"],
                          t["dv"], ws, causal=causal, key_bias=bias, stream=stream)
            ev_done[b].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_done[b])
                for x in names_out:
                    host_out[x].copy_(t[x], non_blocking=True)
                ev_out[b].record(down)
        stream.wait_event(ev_out[(n - 1) % 2])
        if n >= 2:
            stream.wait_event(ev_out[(n - 2) % 2])

    warm = torch.cuda.Event()
    warm.record(stream)
    e2e_run(2, warm)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(args.e2e_steps, e0)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = weak_scaling_value(world, step_flops, args.e2e_steps, e2e_ms)

    # ---- roofline of the dominant kernel (largest share of the timed device time)
    peaks, peak_kind = load_peaks()
    kern_ms = {"fwd": statistics.mean(fwd_ms)}
    if bwd_ms:
        kern_ms["bwd"] = statistics.mean(bwd_ms)
    peak = float(peaks["bf16_tflops"])
    peak_source = (f"{peak_kind} bf16 burst (MEASURED_PEAKS.json)" if peak_kind == "measured"
                   else "fallback 1.59 PFLOP/s bf16")
    if fp8:
        # E4M3 tensor-core rate = bf16 rate x the nominal dense ratio 4.5 / 2.25
        peak *= 2.0
        peak_source += " x 2 (nominal FP8 / BF16 dense ratio)"
    dom = max((k for k in kernels if k in KERNEL_FWD_MULTIPLE), key=lambda k: kernels[k]["share"])
    hbm_peak = float(peaks["hbm_gbs"])
    roof = pick_roofline(kernels[dom], peak, hbm_peak)
    roof["peak_source"] = (peak_source if roof["bound"] == "tensor" else
                           f"{peak_kind} HBM copy bandwidth" +
                           (" (MEASURED_PEAKS.json)" if peak_kind == "measured" else " 6.65 TB/s"))
    roof.update({"traffic": load_traffic(dom, w), "kernel": dom})

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w["dtype"], "data": "synthetic",
        "config": {"workload": workload_name(w, passes), "B": B, "H": H, "Nq": Nq, "Nk": Nk,
                   "D": D, "causal": causal, "passes": passes, "kv_splits": splits,
                   "l2": f"flushed between steps ({args.flush_mib} MiB write, outside the events)",
                   "parallelism": "replicas" if world == 1 else f"{world} ranks, independent (b,h) shards"},
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
                "copies": "per step: pinned-host inputs uploaded and outputs read back on two "
                          "copy streams, overlapped with the neighbouring steps' kernels "
                          "(two device buffer sets)"},
        "gpu_launches": int(launches),
        "clocks": clocks,
        "per_pass": {p: {"ms": kern_ms[p], "tflops": fl[p] / (kern_ms[p] * 1e-3) / 1e12,
                         "frac_of_peak": fl[p] / (kern_ms[p] * 1e-3) / 1e12 / peak}
                     for p in kern_ms},
        "kernels": kernels,
    }
    if cpu_line is not None:
        line["cpu_baseline"] = cpu_line
        line["parity"] = parity
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def load_traffic(kernel, w):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary (profiles/), or None if none matches the current kernel build."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        d = json.load(open(path))
        ent = d.get(f"{kernel}:{w.get('traffic_key', w['name'])}")
        if ent and ent.get("kernel_rev") == kernel_rev(kernel):
            return ent["bytes_per_launch"]
    except (OSError, ValueError):
        pass
    return None


# The source file that defines each kernel; its revision also covers the
# device headers every kernel file includes.
KERNEL_SOURCE = {"fa_fwd_kernel": "fa_fwd.cu", "fa_fwd_split_kernel": "fa_fwd.cu",
                 "fa_fwd_combine_kernel": "fa_fwd.cu", "fa_bwd_dkdv_kernel": "fa_bwd.cu",
                 "fa_bwd_dq_kernel": "fa_bwd.cu", "fa_bwd_pre_kernel": "fa_bwd.cu"}
DEVICE_HEADERS = ("fa_ptx.cuh", "fa_internal.h")


def kernel_rev(kernel=None):
    """Content hash of the CUDA sources a kernel is built from (its own .cu file
    and the shared device headers; every source when the kernel is not known),
    so that ncu traffic taken from an older build is not reported."""
    import hashlib
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "exact_attention_112_b200", "csrc")
    names = sorted(os.listdir(csrc))
    if kernel in KERNEL_SOURCE:
        names = [n for n in names if n == KERNEL_SOURCE[kernel] or n in DEVICE_HEADERS]
    for f in names:
        h.update(f.encode())
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:12]


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
