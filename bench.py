"""Benchmark of the block-sparse decode step on B200 (one JSON line on stdout).

Workload (default): SAS-style GQA decode, bf16 -- batch 8, 32 query / 8 kv heads, d = 128,
context 32,768, blocks of 64, top-15 history blocks + the current block, keys with 16 planted
needle blocks per (batch, kv head).  One step = one pass of the decode hot path over the batch:
refresh the summary of the current block, score every history block, Top-K, sparse attention
(one fused kernel launch, replayed as a CUDA graph).  Each step reads a different one of 8
"layer" instances of the KV cache and summaries in turn, so the data a step touches is never in
the 126 MB L2; the steps are timed with CUDA events on the launching stream.

The same line carries the other rows of the hot path, each with a roofline block: the long
decode at 512K (same fused step, plus its score / Top-K / attention breakdown through the
separate calls), the summaries build (GB/s), the SAS gated prefill forward and gate gradient, and
the FreeSolo prefill (TFLOP/s on the gathered FLOPs).  ``cpu_baseline`` is the fp64 oracle run on
every host core (a process pool forked before the first GPU call), next to its one-thread figure.

``--impl reference`` times the fp64 CPU oracle on the same workload instead (a bounded sample of
the decode step per timed step, on every host core) and prints the same JSON line with
"impl": "reference".
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

import hashlib

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-attn decode tokens/s and HBM GB/s (% roofline); prefill TFLOP/s (% peak)"

WORKLOADS = {
    "sas_gqa_decode_32k": dict(B=8, Hq=32, Hk=8, d=128, n=32768, b=64, K=15, needles=16,
                               needle_layout="random", seed=2000),
    "long_decode_512k": dict(B=1, Hq=32, Hk=8, d=128, n=524288, b=64, K=31, needles=64,
                             needle_layout="stride", seed=3000),
}



# DRAM bytes (read + write) of one launch of the dominant kernel, from an ncu capture of the kernel
# built from the source whose hash is given (the capture command is recorded with the decode
# profile summary under profiles/).  Reported only while the source is unchanged.
# The hash covers the device code of the source: the file up to its first host function
# (`device_end`), so a change of the host-side launcher alone keeps the figure.
MEASURED_TRAFFIC = {
    ("sas_gqa_decode_32k", "decode_fused_kernel"): {
        "source": "block_sparse_attention_summaries_b200/csrc/decode_fused.cu",
        "device_end": "int pick_cluster(", "sha256_16": "18c12307660d9922",
        "bytes": 52_596_992 + 447_488},
    # two launches per step (chunk Top-K, then merge + attention): their sum
    ("long_decode_512k", "decode_fused_kernel"): {
        "source": "block_sparse_attention_summaries_b200/csrc/decode_fused.cu",
        "device_end": "int pick_cluster(", "sha256_16": "18c12307660d9922",
        "bytes": 33_624_064 + 16_127_232},
    # one launch each, full captures of the gated prefill forward and the gate gradient
    ("sas_gated_prefill_16k", "sas_fwd_tc_kernel"): {
        "source": "block_sparse_attention_summaries_b200/csrc/sas_fwd_tc.cu",
        "device_end": "bsa_status launch_sas(", "sha256_16": "6cb98727de799ac2",
        "bytes": 412_782_336 + 240_278_016},
    ("sas_gated_prefill_16k", "gate_grad_tc_kernel"): {
        "source": "block_sparse_attention_summaries_b200/csrc/prefill_tc.cu",
        "device_end": "bsa_status launch_tc(", "sha256_16": "09671dc7350d5094",
        "bytes": 940_605_952 + 4_610_304},
    ("freesolo_prefill_64k", "freesolo_select_tc_kernel"): {
        "source": "block_sparse_attention_summaries_b200/csrc/freesolo_tc.cu",
        "device_end": "size_t freesolo_select_tc_workspace(", "sha256_16": "79ef22b094ee8af3",
        "bytes": 142_674_432 + 14_409_472},
}


def device_source_hash(path: str, device_end: str) -> str:
    with open(path, "rb") as f:
        text = f.read()
    cut = text.find(device_end.encode())
    return hashlib.sha256(text[:cut] if cut >= 0 else text).hexdigest()[:16]


def measured_traffic(workload: str, kernel: str):
    rec = MEASURED_TRAFFIC.get((workload, kernel))
    if rec is None:
        return None
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), rec["source"])
    if device_source_hash(path, rec["device_end"]) != rec["sha256_16"]:
        return None
    return rec["bytes"]

def job_timing(total_ms: float, e2e_ms: float, world: int, device) -> tuple[float, float]:
    """The job's device times: the maximum over ranks (one all-reduce, taken by every rank in the
    same order; a single rank returns its own)."""
    if world <= 1:
        return total_ms, e2e_ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([total_ms, e2e_ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t[0]), float(t[1])


def job_throughput(tokens_per_rank_step: int, world: int, steps: int, ms: float) -> float:
    """Whole-job tokens/s: every rank decodes its own batch (weak scaling), so the tokens of all
    ranks count over the slowest rank's time."""
    return tokens_per_rank_step * world * steps / (ms / 1e3)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background (read-only queries)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int = 0, period_ms: int = 50):
        self.samples = []
        self.proc = None
        self.gpu = gpu_index
        self.period = period_ms
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", f"-lms={self.period}"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        for ts, line in self.samples:
            if self.t0 is not None and not (self.t0 - 0.05 <= ts <= (self.t1 or ts) + 0.05):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            rows.append(parts)
        if not rows:  # timed window shorter than the sampling period: use the whole run
            rows = [[p.strip() for p in line.split(",")] for _, line in self.samples]
            rows = [r for r in rows if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


def oracle_decode_sample(case, rows_b, summaries):
    """Time the oracle's decode of the listed batch rows (all heads) on one host thread;
    returns seconds."""
    from threadpoolctl import threadpool_limits

    from oracle import bsa_oracle as orc
    rows = [(bi, h) for bi in rows_b for h in range(case.Hq)]
    with threadpool_limits(limits=1):
        t = time.perf_counter()
        orc.decode_reference(case.q, case.k, case.v, case.seq_lens, case.b, case.K, rows=rows,
                             summaries=summaries)
        return time.perf_counter() - t


def oracle_summaries(case, rows_b):
    from oracle import bsa_oracle as orc
    out = {}
    for bi in rows_b:
        for kh in range(case.Hk):
            out[(bi, kh)] = orc.block_summaries(case.k[bi, kh, :case.seq_lens[bi]], case.b)
    return out


# The oracle pool: worker processes forked from the parent BEFORE its first CUDA call (a process
# forked after CUDA initialisation can hang), reading the case copy-on-write.  One task is one
# (batch row, kv head) group: its G query heads scored, selected and attended by the oracle.
_POOL_CASE = None


def _oracle_group(task):
    from threadpoolctl import threadpool_limits

    from oracle import bsa_oracle as orc
    bi, kh = task
    case, summ = _POOL_CASE
    G = case.Hq // case.Hk
    with threadpool_limits(limits=1):
        orc.decode_reference(case.q, case.k, case.v, case.seq_lens, case.b, case.K,
                             rows=[(bi, h) for h in range(kh * G, (kh + 1) * G)],
                             summaries={(bi, kh): summ[(bi, kh)]})
    return bi, kh


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


class OraclePool:
    """Whole decode steps of the oracle (every batch row, every head) spread over ``cores``
    forked worker processes, one single-threaded task per (batch row, kv head) group."""

    def __init__(self, case, summ, cores):
        import multiprocessing as mp
        global _POOL_CASE
        _POOL_CASE = (case, summ)
        self.case, self.cores = case, cores
        self.tasks = [(bi, kh) for bi in range(case.B) for kh in range(case.Hk)]
        self.pool = mp.get_context("fork").Pool(cores)
        self.pool.map(_oracle_group, self.tasks[:cores], chunksize=1)  # workers up and warm

    def step(self) -> float:
        """One decode step of the whole batch; returns seconds."""
        t = time.perf_counter()
        self.pool.map(_oracle_group, self.tasks, chunksize=1)
        return time.perf_counter() - t

    def close(self):
        self.pool.close()
        self.pool.join()


def cpu_baselines(case, seconds: float):
    """The oracle as it stands on the host: on every core (whole decode steps, as many as fit in
    about ``seconds``) and on one thread (batch rows, about ``seconds`` / 2).  Must run before the
    process makes its first CUDA call (the pool forks)."""
    summ = oracle_summaries(case, range(case.B))
    cores = host_cores()
    pool = OraclePool(case, summ, cores)
    total, steps = 0.0, 0
    while total < seconds or steps < 1:
        total += pool.step()
        steps += 1
    pool.close()
    multi = {"value": steps * case.B / total, "unit": "tokens/s", "cores": cores,
             "kind": "oracle",
             "sample": f"{steps} whole decode steps ({steps * case.B} tokens: every batch row, "
                       f"all {case.Hq} heads) of the same workload, one forked single-threaded "
                       "worker per core, one task per (batch row, kv head) group, summaries "
                       "precomputed"}
    tsec, done = 0.0, 0
    while tsec < seconds / 2 and done < 64:
        tsec += oracle_decode_sample(case, [done % case.B], summ)
        done += 1
    single = {"value": done / tsec, "unit": "tokens/s", "cores": 1, "kind": "oracle",
              "sample": f"{done} decode tokens (batch rows, all {case.Hq} heads), one thread"}
    return multi, single


def make_case(wl):
    from block_sparse_attention_summaries_b200 import inputs
    w = WORKLOADS[wl]
    return inputs.decode_case(w["seed"], B=w["B"], Hq=w["Hq"], Hk=w["Hk"], d=w["d"], n=w["n"],
                              b=w["b"], K=w["K"], needles=w["needles"],
                              needle_layout=w["needle_layout"])


def run_reference(args):
    """fp64 CPU oracle timed on the host cores: each timed step is one whole decode step of the
    workload (every batch row, all heads) spread over a forked process pool."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    case = make_case(args.workload)
    summ = oracle_summaries(case, range(case.B))
    cores = host_cores()
    pool = OraclePool(case, summ, cores)
    for _ in range(args.warmup):
        pool.step()
    total = sum(pool.step() for _ in range(args.steps))
    pool.close()
    ms = total / args.steps * 1e3
    value = args.steps * case.B / total
    w = WORKLOADS[args.workload]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1), bf16-rounded, planted needle blocks)",
        "config": {"workload": args.workload, **{k: w[k] for k in ("B", "Hq", "Hk", "d", "n",
                                                                   "b", "K")}},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step one whole decode step ({case.B} tokens, all "
                                   f"{case.Hq} heads) on {cores} forked single-threaded workers, "
                                   "summaries precomputed as on the GPU"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def roofline(bound, kernel, achieved, peak, unit, traffic=None, algorithmic=None,
             peak_source=""):
    """The roofline block of one row: achieved against the measured peak (frac), and the
    ncu-recorded DRAM traffic of one launch when a capture of the current kernel exists."""
    out = {"bound": bound, "kernel": kernel, "achieved": achieved, "peak": peak, "unit": unit,
           "frac": achieved / peak if peak else None, "traffic": traffic}
    if algorithmic is not None:
        out["algorithmic"] = algorithmic
    out["peak_source"] = peak_source
    return out


def time_cuda(fn, reps, stream):
    """Average milliseconds of fn() over reps launches (CUDA events on `stream`, one warm-up)."""
    import torch
    with torch.cuda.stream(stream):
        fn()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        ev[0].record(stream)
        for i in range(reps):
            fn()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
    return [ev[i].elapsed_time(ev[i + 1]) for i in range(reps)]


def run_prefill(dev, peaks, reps=5, rows=("sas", "freesolo", "fsl")):
    """Prefill rows: SAS gated training prefill (forward on tcgen05 + gate gradient) and FreeSolo
    two-branch prefill, each as TFLOP/s on the gathered FLOPs (4 d per attended query-key pair)."""
    import torch

    import block_sparse_attention_summaries_b200 as bsa
    from block_sparse_attention_summaries_b200 import inputs

    out = {}
    stream = torch.cuda.Stream(dev)
    bf = lambda x: torch.from_numpy(x).to(dev, torch.bfloat16)
    peak = peaks["bf16_tflops"]
    src = peaks["source"] + " bf16 (burst)"
    if "sas" in rows:
        pc = inputs.prefill_case(5000)
        q, k, v, do = bf(pc.q), bf(pc.k), bf(pc.v), bf(pc.dout)
        s = torch.from_numpy(pc.scores).to(dev)
        idx, cnt = bsa.topk_blocks(s, pc.K, units=pc.U, q_block=64, b=64)
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:-1], device=dev, dtype=torch.float32)
        dg = torch.empty(pc.B, pc.Hq, pc.U, pc.K, device=dev, dtype=torch.float32)
        cnt_h = cnt.cpu().numpy().astype(np.int64)  # [B, Hq, U]
        d = pc.d
        per_unit = cnt_h * 64 * 64 + 64 * 65 // 2  # attended pairs per unit (history + causal diag)
        fwd_flops = float(4 * d * per_unit.sum())
        grad_flops = float(4 * d * (cnt_h * 64 * 64).sum())
        fwd = lambda: bsa.sparse_attn_fwd(q, k, v, idx, 64, count=cnt, q_block=64, gate=True,
                                          norm="selected", scores=s, o=o, lse=lse)
        grad = lambda: bsa.gate_grad(q, k, v, o, lse, do, idx, 64, s, q_block=64, count=cnt,
                                     norm="selected", dg=dg)
        t_fwd = statistics.fmean(time_cuda(fwd, reps, stream))
        t_grad = statistics.fmean(time_cuda(grad, max(2, reps // 2), stream))
        n_cand = torch.arange(pc.U, dtype=torch.int32, device=dev).expand(pc.B, pc.Hq, pc.U).contiguous()
        ds = torch.empty_like(s)
        sgrad = lambda: bsa.selector_grad(s, n_cand, idx, cnt, dg, bsa.NORM_SELECTED, ds=ds)
        t_sgrad = statistics.fmean(time_cuda(sgrad, reps, stream))
        # selected normaliser: ds written over every candidate slot; idx, dg and the selected scores
        # read per slot; count and n_cand per unit
        sgrad_bytes = float(s.numel() * 4 + idx.numel() * 4 * 3 + cnt.numel() * 4 * 2)
        # the outer-gate variant (gate outside the softmax) on the CUDA-core row kernels
        o2 = torch.empty_like(q)
        lse2 = torch.empty_like(lse)
        dg2 = torch.empty_like(dg)
        ofwd = lambda: bsa.sparse_attn_fwd(q, k, v, idx, 64, count=cnt, q_block=64, gate="outer",
                                           norm="selected", scores=s, o=o2, lse=lse2)
        ograd = lambda: bsa.gate_grad(q, k, v, o2, lse2, do, idx, 64, s, q_block=64, count=cnt,
                                      norm="selected", dg=dg2, outer=True)
        t_ofwd = statistics.fmean(time_cuda(ofwd, max(2, reps // 2), stream))
        t_ograd = statistics.fmean(time_cuda(ograd, max(2, reps // 2), stream))
        out["sas_gated_prefill_16k"] = {
            "config": {"B": pc.B, "Hq": pc.Hq, "Hk": pc.Hk, "d": d, "n": pc.n, "b": 64,
                       "q_block": 64, "K": pc.K, "gate": "log-softmax over the selected blocks"},
            "forward": {"kernel": "sas_fwd_tc_kernel (tcgen05, two softmax warpgroups)", "ms": t_fwd,
                        "gathered_gflop": fwd_flops / 1e9, "tflops": fwd_flops / t_fwd / 1e9,
                        "roofline": roofline("tensor", "sas_fwd_tc_kernel", fwd_flops / t_fwd / 1e9,
                                             peak, "TFLOP/s", peak_source=src,
                                             traffic=measured_traffic("sas_gated_prefill_16k",
                                                                      "sas_fwd_tc_kernel"))},
            "gate_grad": {"kernel": "gate_grad_tc_kernel (tcgen05)", "ms": t_grad,
                          "gathered_gflop": grad_flops / 1e9, "tflops": grad_flops / t_grad / 1e9,
                          "roofline": roofline("tensor", "gate_grad_tc_kernel",
                                               grad_flops / t_grad / 1e9, peak, "TFLOP/s",
                                               peak_source=src,
                                               traffic=measured_traffic("sas_gated_prefill_16k",
                                                                        "gate_grad_tc_kernel"))},
            "selector_grad": {"kernel": "selector_grad_kernel", "ms": t_sgrad,
                              "bytes": sgrad_bytes, "gbs": sgrad_bytes / t_sgrad / 1e6,
                              "roofline": roofline("hbm", "selector_grad_kernel",
                                                   sgrad_bytes / t_sgrad / 1e6, peaks["hbm_gbs"],
                                                   "GB/s", algorithmic=sgrad_bytes,
                                                   peak_source=peaks["source"] + " (burst copy)")},
            "outer_gate": {"kernels": "sas_fwd_tc_kernel, gate_grad_tc_kernel (tcgen05)",
                           "forward_ms": t_ofwd, "forward_tflops": fwd_flops / t_ofwd / 1e9,
                           "grad_ms": t_ograd, "grad_tflops": grad_flops / t_ograd / 1e9,
                           "roofline": roofline("tensor", "sas_fwd_tc_kernel (outer gate)",
                                                fwd_flops / t_ofwd / 1e9, peak, "TFLOP/s",
                                                peak_source=src)},
        }
        del q, k, v, do, o, s, idx, cnt, lse, dg, o2, lse2, dg2
        torch.cuda.empty_cache()
    if "freesolo" in rows:
        fc = inputs.freesolo_case(4000)
        q, k, v = bf(fc.q), bf(fc.k), bf(fc.v)
        lam, sig, alpha = (torch.from_numpy(x).to(dev) for x in (fc.lam, fc.sigma, fc.alpha))
        mk, mx, ce = bsa.build_block_summaries(k, fc.cell)
        idx, cnt = bsa.freesolo_select(q, mk, mx, ce, lam, sig, fc.cell, fc.q_block, fc.K)
        o = torch.empty_like(q)
        ws = torch.zeros(int(bsa.lib().bsa_freesolo_workspace_bytes(bsa.BSA_BF16, fc.B, fc.H, fc.n,
                                                                      fc.d, fc.cell, fc.K)),
                         dtype=torch.uint8, device=dev)
        sws = torch.zeros(max(1, int(bsa.lib().bsa_freesolo_select_workspace_bytes(
            bsa.BSA_BF16, fc.B, fc.H, fc.n, fc.d, fc.cell, fc.q_block, fc.K))), dtype=torch.uint8,
            device=dev)
        sel = lambda: bsa.freesolo_select(q, mk, mx, ce, lam, sig, fc.cell, fc.q_block, fc.K,
                                          idx=idx, count=cnt, ws=sws)
        att = lambda: bsa.freesolo_attn(q, k, v, alpha, idx, cnt, fc.cell, fc.window, fc.rope_theta,
                                        o=o, ws=ws)
        t_sel = statistics.fmean(time_cuda(sel, 2, stream))
        t_att = statistics.fmean(time_cuda(att, 2, stream))
        cnt_h = cnt.cpu().numpy().astype(np.int64)
        pos = np.arange(fc.n)
        win = np.minimum(pos + 1, fc.window).sum() * fc.B * fc.H
        att_flops = float(4 * fc.d * (win + (cnt_h * fc.cell).sum()))
        ncand = ((pos // fc.q_block) * fc.q_block) // fc.cell
        score_flops = float(2 * fc.d * ncand.sum() * fc.B * fc.H)
        out["freesolo_prefill_64k"] = {
            "config": {"B": fc.B, "H": fc.H, "d": fc.d, "n": fc.n, "cell": fc.cell,
                       "q_block": fc.q_block, "K": fc.K, "window": fc.window},
            "select": {"kernel": "split_hi_lo + freesolo_select_tc_kernel (tcgen05)", "ms": t_sel,
                       "score_gflop": score_flops / 1e9, "tflops": score_flops / t_sel / 1e9,
                       "roofline": roofline("tensor", "freesolo_select_tc_kernel",
                                            score_flops / t_sel / 1e9, peak, "TFLOP/s",
                                            peak_source=src,
                                            traffic=measured_traffic("freesolo_prefill_64k",
                                                                     "freesolo_select_tc_kernel"))},
            "attention": {"kernel": "rope (q, k) + window_tc_kernel (persistent 128-query tiles) + "
                                    "cell-major long branch (fs_long_* kernels, tcgen05 tiles) + "
                                    "combine", "ms": t_att,
                          "gathered_gflop": att_flops / 1e9, "tflops": att_flops / t_att / 1e9,
                          "roofline": roofline("tensor", "freesolo attention (all launches)",
                                               att_flops / t_att / 1e9, peak, "TFLOP/s",
                                               peak_source=src)},
            "tokens_per_s": fc.n * fc.B / ((t_sel + t_att) / 1e3),
        }
        del q, k, v, o, ws, sws, idx, cnt
        torch.cuda.empty_cache()
    if "fsl" in rows:
        # FS-L / FS-B decode at 256K, batch 1 ([FreeSolo] "How it differs": FS-L keeps W + P cells
        # per head in a fixed-size state, FS-B searches two forests): the kept-cell selection against
        # full O(C) scoring, the FS-L state update per query block, the decode call (window + long
        # branch + mix) and the FS-B build and search.  Each call of a timed graph decodes its own
        # position (positions 600 tokens apart, so no call finds another's window in L2).
        H, d, n, cell, K, W, P, window, width = 16, 64, 262144, 32, 4, 8, 64, 512, 16
        g = torch.Generator(device=dev).manual_seed(4200)
        kf = torch.randn(1, H, n, d, device=dev, generator=g).to(torch.bfloat16)
        vf = torch.randn(1, H, n, d, device=dev, generator=g).to(torch.bfloat16)
        qf = torch.randn(1, H, d, device=dev, generator=g).to(torch.bfloat16)
        mk, mx, ce = bsa.build_block_summaries(kf, cell)
        C = mk.shape[2]
        lam = torch.full((H,), 0.5, device=dev)
        sig = torch.full((H,), 4096.0, device=dev)
        alpha = torch.rand(H, device=dev, generator=g)
        iters = 20
        positions = [n - 1 - 600 * r for r in range(iters)]
        pos_t = [torch.full((1,), p_, dtype=torch.int32, device=dev) for p_ in positions]
        ncell_t = [torch.full((H,), (p_ // 128) * 128 // cell, dtype=torch.int32, device=dev)
                   for p_ in positions]
        states = []
        for r in range(iters):  # a state per position, grown from empty
            st = bsa.FslState(H, W, P, dev)
            st.update(mx.view(H, C), ncell_t[r])
            states.append(st)
        seq = torch.full((1,), n, dtype=torch.int32, device=dev)
        sc = torch.empty(1, H, C, device=dev)
        ncnd = torch.empty(H, device=dev, dtype=torch.int32)
        o_f = torch.empty(1, H, d, device=dev, dtype=torch.bfloat16)
        idx_f = torch.empty(1, H, K, device=dev, dtype=torch.int32)
        cnt_f = torch.empty(1, H, device=dev, dtype=torch.int32)
        stat_f = torch.zeros(1, dtype=torch.int32, device=dev)

        def graph_ms(fns):
            """Device time per call: the calls captured in one CUDA graph (these calls are a few
            microseconds each, far below the cost of launching them one by one from Python)."""
            with torch.cuda.stream(stream):
                for fn in fns:
                    fn()
            torch.cuda.synchronize(dev)
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                for fn in fns:
                    fn()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                gr.replay()
                e0.record(stream)
                for _ in range(reps):
                    gr.replay()
                e1.record(stream)
            e1.synchronize()
            del gr
            return e0.elapsed_time(e1) / (reps * len(fns))

        seqs = [p_ + 1 for p_ in pos_t]
        full = [lambda r=r: bsa.topk_blocks(bsa.score_blocks(
            qf, mk, n, cell, seq_lens=seqs[r], max_norm=mx, centre=ce, lambda_h=lam, sigma_h=sig,
            prefix_block=128, scores=sc, n_cand=ncnd)[0], K, n_cand=ncnd) for r in range(iters)]
        fsl_sel = [lambda r=r: bsa.fsl_select(qf, pos_t[r], mk, mx, ce, lam, sig,
                                              states[r].cand.view(1, H, -1),
                                              states[r].cand_count.view(1, H), K)
                   for r in range(iters)]
        fsl_dec = [lambda r=r: bsa.fsl_decode(qf, kf, vf, pos_t[r], cell, mk, mx, ce, lam, sig, alpha,
                                              states[r].cand.view(1, H, -1),
                                              states[r].cand_count.view(1, H), K, window=window,
                                              o=o_f, idx=idx_f, count=cnt_f, status=stat_f)
                   for r in range(iters)]
        t_full = graph_ms(full)
        t_fsl_sel = graph_ms(fsl_sel)
        t_fsl_dec = graph_ms(fsl_dec)
        # the state update at a query-block boundary: 4 new cells per head (the state is reset to
        # its previous prefix inside the graph, three small copies)
        saved = [(st.older.clone(), st.older_count.clone(), st.state_cells.clone()) for st in states]
        prev = [c - 4 for c in ncell_t]
        for st, p_ in zip(states, prev):  # states one query block earlier
            st.older.fill_(-1)
            st.older_count.zero_()
            st.state_cells.zero_()
            st.update(mx.view(H, C), p_)
        base = [(st.older.clone(), st.older_count.clone(), st.state_cells.clone()) for st in states]

        def upd(r):
            st = states[r]
            st.older.copy_(base[r][0])
            st.older_count.copy_(base[r][1])
            st.state_cells.copy_(base[r][2])
            st.update(mx.view(H, C), ncell_t[r])
        t_reset = graph_ms([lambda r=r: (states[r].older.copy_(base[r][0]),
                                         states[r].older_count.copy_(base[r][1]),
                                         states[r].state_cells.copy_(base[r][2]))
                            for r in range(iters)])
        t_upd = graph_ms([lambda r=r: upd(r) for r in range(iters)]) - t_reset
        for st, sv in zip(states, saved):
            assert torch.equal(st.older_count, sv[1]) and torch.equal(st.older, sv[0])
        # FS-B: forests built for the query block's prefix, then beam search + re-rank + decode
        forests = [bsa.fsb_build(mk, mx, ce, ncell_t[r]) for r in range(iters)]
        fidx = torch.empty(1, H, K, device=dev, dtype=torch.int32)
        fcnt = torch.empty(1, H, device=dev, dtype=torch.int32)
        flse = torch.empty(1, H, K, device=dev)
        t_fsb_build = graph_ms([lambda r=r: bsa.fsb_build(mk, mx, ce, ncell_t[r], forest=forests[r])
                                for r in range(4)])
        t_fsb_sel = graph_ms([lambda r=r: bsa.fsb_select(qf, kf, pos_t[r], cell, forests[r], lam,
                                                         sig, width, K, idx=fidx, count=fcnt,
                                                         lse=flse)
                              for r in range(iters)])
        del forests
        # algorithmic bytes of one FS-L decode call: the window's K and V, the K selected cells' K
        # and V, the kept cells' summaries, q and o
        win = min(window, positions[0] + 1)
        dec_bytes = H * (win * d * 2 * 2 + K * cell * d * 2 * 2 + (W + P) * (d + 2) * 4 + 2 * d * 2)
        gbs = dec_bytes / (t_fsl_dec / 1e3) / 1e9
        out["fsl_decode_256k"] = {
            "config": {"B": 1, "H": H, "d": d, "n": n, "cell": cell, "K": K, "W": W, "P": P,
                       "window": window, "cells": C, "fsb_beam": width},
            "full_select_ms": t_full, "fsl_select_ms": t_fsl_sel,
            "fsl_state_update_ms": t_upd, "fsl_decode_ms": t_fsl_dec,
            "fsl_step_ms": t_fsl_dec + t_upd / 128.0,
            "fsl_tokens_per_s": 1.0 / ((t_fsl_dec + t_upd / 128.0) / 1e3),
            "fsb_build_ms": t_fsb_build, "fsb_select_ms": t_fsb_sel,
            "fsb_step_ms": t_fsb_sel + t_fsl_dec + t_fsb_build / 128.0,
            "decode_bytes": dec_bytes,
            "roofline": roofline("hbm", "fsl_decode_kernel", gbs, peaks["hbm_gbs"], "GB/s",
                                 algorithmic=dec_bytes,
                                 peak_source=peaks["source"] + " (burst copy)"),
            "kernels": "full: score_decode_kernel + topk_kernel over every cell; FS-L: "
                       "fsl_select_kernel over the W + P kept cells; fsl_state_update_kernel (4 new "
                       "cells per 128-token query block, amortised over its 128 steps); "
                       "fsl_decode_kernel (4-CTA cluster per head); FS-B: topk_kernel (upper half) + "
                       "fsb_build_levels/radius_kernel per query block (amortised over 128 steps), "
                       "fsb_search_kernel per step",
        }
        del kf, vf
        torch.cuda.empty_cache()
    return out


def build_layers(dev, case, w, R):
    """R "layers": the seeded case and R-1 copies with the kv heads (and their query heads)
    rotated, so that each step reads memory the previous steps did not leave in L2."""
    import torch

    import block_sparse_attention_summaries_b200 as bsa
    B, Hq, Hk, d, b, K = (w[x] for x in ("B", "Hq", "Hk", "d", "b", "K"))
    G = Hq // Hk
    q0 = torch.from_numpy(case.q).to(dev, torch.bfloat16)
    k0 = torch.from_numpy(case.k).to(dev, torch.bfloat16)
    v0 = torch.from_numpy(case.v).to(dev, torch.bfloat16)
    layers = []
    for r in range(R):
        kk = torch.roll(k0, shifts=r, dims=1).contiguous() if r else k0
        vv = torch.roll(v0, shifts=r, dims=1).contiguous() if r else v0
        qq = torch.roll(q0, shifts=r * G, dims=1).contiguous() if r else q0
        mk, mx, ce = bsa.build_block_summaries(kk, b)  # prefill-time state
        layers.append(dict(q=qq, k=kk, v=vv, mean_k=mk, max_norm=mx, centre=ce,
                           o=torch.empty(B, Hq, d, device=dev, dtype=torch.bfloat16),
                           lse=torch.empty(B, Hq, device=dev, dtype=torch.float32),
                           idx=torch.empty(B, Hq, K, device=dev, dtype=torch.int32),
                           count=torch.empty(B, Hq, device=dev, dtype=torch.int32)))
    return layers


def capture_fused(dev, layers, w, status, stream, ws=None):
    """CUDA graphs of the fused decode step (one kernel launch per step; with a workspace ``ws``,
    long histories take the two-launch path of bsa_decode_step_ws): one graph per layer, and one
    graph of a whole decode iteration (every layer's step in order, as a model replays one graph
    per generated token). Returns (per-layer graphs, iteration graph)."""
    import torch

    import block_sparse_attention_summaries_b200 as bsa
    b, K = w["b"], w["K"]

    def fused(L):
        if ws is not None:
            bsa.decode_step_ws(L["q"], L["k"], L["v"], L["mean_k"], b, K, ws=ws, append=True,
                               max_norm=L["max_norm"], centre=L["centre"], o=L["o"],
                               lse=L["lse"], idx=L["idx"], count=L["count"], status=status)
            return
        bsa.decode_step_fused(L["q"], L["k"], L["v"], L["mean_k"], b, K, append=True,
                              max_norm=L["max_norm"], centre=L["centre"], o=L["o"], lse=L["lse"],
                              idx=L["idx"], count=L["count"], status=status)

    return capture_steps(dev, layers, fused, stream)


def capture_steps(dev, layers, step, stream):
    """``step(L)`` captured once per layer and once as a whole iteration over the layers."""
    import torch
    graphs = []
    with torch.cuda.stream(stream):
        for L in layers:
            step(L)
        torch.cuda.synchronize(dev)
        for L in layers:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step(L)
            graphs.append(g)
        cycle = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cycle, stream=stream):
            for L in layers:
                step(L)
    torch.cuda.synchronize(dev)
    return graphs, cycle


def replay_steps(graphs, steps):
    """``steps`` decode steps: whole iterations over the layers, then single layers for the
    remainder (graphs as returned by capture_steps)."""
    per_layer, cycle = graphs
    R = len(per_layer)
    for _ in range(steps // R):
        cycle.replay()
    for i in range(steps % R):
        per_layer[i].replay()


def time_graph_cycle(dev, graphs, steps, warmup, stream):
    """Milliseconds of ``steps`` decode steps (layer i % R in turn) between two events on the
    stream (an event recorded between two steps would cost the step about 2 us: it ends the
    overlap of one launch's tail with the next one's start)."""
    import torch
    with torch.cuda.stream(stream):
        replay_steps(graphs, warmup)
        torch.cuda.synchronize(dev)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record(stream)
        replay_steps(graphs, steps)
        ev[1].record(stream)
        torch.cuda.synchronize(dev)
    return ev[0].elapsed_time(ev[1])


def decode_accounting(case, w, idx_h):
    """Algorithmic bytes of one decode step and the needle recall of its selection: summaries
    scored (every history block of every kv head, fp32) + the union over each GQA group of the
    selected K/V blocks (each crosses HBM once) + the current block; q, o, the indices and the
    appended summary as I/O."""
    B, Hq, Hk, d, n, b, K = (w[x] for x in ("B", "Hq", "Hk", "d", "n", "b", "K"))
    G = Hq // Hk
    cur = (n - 1) // b
    union_blocks = per_head_blocks = 0
    for bi in range(B):
        for kh in range(Hk):
            sel = set(int(x) for x in idx_h[bi, kh * G:(kh + 1) * G].ravel() if x >= 0)
            union_blocks += len(sel) + 1
            per_head_blocks += int((idx_h[bi, kh * G:(kh + 1) * G] >= 0).sum()) + G
    cur_tokens = n - cur * b
    kv_bytes = (union_blocks - B * Hk) * b * d * 2 * 2 + B * Hk * cur_tokens * d * 2 * 2
    summary_bytes = B * Hk * cur * d * 4
    io_bytes = B * Hq * d * 2 * 2 + B * Hq * (K * 4 + 8) + B * Hk * (d + 2) * 4
    hits = tot = 0
    for (bi, kh), blocks in case.needles.items():
        sel = set(int(x) for x in idx_h[bi, kh * G:(kh + 1) * G].ravel() if x >= 0)
        hits += len(sel & set(int(c) for c in blocks))
        tot += len(blocks)
    return {"union_blocks": union_blocks, "per_head_blocks": per_head_blocks,
            "kv_bytes": kv_bytes, "summary_bytes": summary_bytes, "io_bytes": io_bytes,
            "needle_recall": hits / max(1, tot), "cur_tokens": cur_tokens}


def separate_calls(dev, layers, w, warmup, nsep, stream):
    """The same step through the separate C-ABI calls (summary append + scores, Top-K, split-K
    attention), each captured in its own graph: the per-stage breakdown in microseconds."""
    import torch

    import block_sparse_attention_summaries_b200 as bsa
    B, Hq, Hk, d, n, b, K = (w[x] for x in ("B", "Hq", "Hk", "d", "n", "b", "K"))
    C = (n + b - 1) // b
    R = len(layers)
    sep = []
    with torch.cuda.stream(stream):
        scores = torch.empty(B, Hq, C, device=dev, dtype=torch.float32)
        n_cand = torch.empty(B * Hq, device=dev, dtype=torch.int32)
        ws = torch.zeros(bsa.sparse_attn_workspace_bytes(B, Hq, Hk, 1, n, d, b, K),
                         dtype=torch.uint8, device=dev)
        stage_graphs = []
        for L in layers:
            fns = [lambda L=L: (bsa.build_block_summaries(L["k"], b, None, -1, 1, L["mean_k"],
                                                          L["max_norm"], L["centre"]),
                                bsa.score_blocks(L["q"], L["mean_k"], n, b, scores=scores,
                                                 n_cand=n_cand)),
                   lambda L=L: bsa.topk_blocks(scores, K, n_cand=n_cand, idx=L["idx"],
                                               count=L["count"]),
                   lambda L=L: bsa.sparse_attn_fwd(L["q"], L["k"], L["v"], L["idx"], b,
                                                   count=L["count"], o=L["o"], lse=L["lse"],
                                                   ws=ws)]
            gs = []
            for fn in fns:
                fn()
                torch.cuda.synchronize(dev)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    fn()
                gs.append(g)
            stage_graphs.append(gs)
        for i in range(warmup):
            for g in stage_graphs[i % R]:
                g.replay()
        torch.cuda.synchronize(dev)
        for i in range(nsep):
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            gs = stage_graphs[i % R]
            e[0].record(stream)
            gs[0].replay()
            e[1].record(stream)
            gs[1].replay()
            e[2].record(stream)
            gs[2].replay()
            e[3].record(stream)
            sep.append(e)
        torch.cuda.synchronize(dev)
    out = {"append+score": statistics.fmean(e[0].elapsed_time(e[1]) for e in sep) * 1e3,
           "topk": statistics.fmean(e[1].elapsed_time(e[2]) for e in sep) * 1e3,
           "attention": statistics.fmean(e[2].elapsed_time(e[3]) for e in sep) * 1e3,
           "step": statistics.fmean(e[0].elapsed_time(e[3]) for e in sep) * 1e3}
    out["selection_share"] = (out["append+score"] + out["topk"]) / max(out["step"], 1e-9)
    del stage_graphs  # graphs before the buffers they replay into
    return out


def run_long_decode(dev, peaks, args, stream):
    """The long-context decode row: 512K context, batch 1, K = 31 (the context of the SAS
    review's headline decode figure, "Decoding efficiency", Fig. 7a/7c): the fused step timed
    as the headline is, its roofline, the separate-call breakdown and the needle recall."""
    import torch
    wl = "long_decode_512k"
    w = WORKLOADS[wl]
    case = make_case(wl)
    R = max(2, min(args.layers, 4))  # 4 x (33.5 MB summaries + union K/V) per cycle > 126 MB L2
    layers = build_layers(dev, case, w, R)
    status = torch.zeros(4, dtype=torch.int32, device=dev)
    import block_sparse_attention_summaries_b200 as bsa
    ws_bytes = bsa.decode_step_workspace_bytes(w["B"], w["Hq"], w["Hk"], w["n"], w["d"], w["b"],
                                               w["K"])
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    graphs = capture_fused(dev, layers, w, status, stream, ws=ws)
    steps = max(50, min(args.steps, 400))
    ms = time_graph_cycle(dev, graphs, steps, args.warmup, stream) / steps
    acc = decode_accounting(case, w, layers[0]["idx"].cpu().numpy())
    sep = separate_calls(dev, layers, w, args.warmup, max(20, min(args.steps, 100)), stream)
    algo = acc["kv_bytes"] + acc["summary_bytes"] + acc["io_bytes"]
    gbs = algo / (ms / 1e3) / 1e9
    out = {"config": {"workload": wl, **{x: w[x] for x in ("B", "Hq", "Hk", "d", "n", "b", "K")},
                      "l2": f"{R} rotated layer instances"},
           "us_per_step": ms * 1e3, "tokens_per_s": w["B"] / (ms / 1e3),
           "algorithmic_bytes": algo, "gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"],
           "union_blocks": acc["union_blocks"], "needle_recall": acc["needle_recall"],
           "status_word": int(status.max().item()),
           "launches_per_step": 2 if ws_bytes > 0 else 1, "workspace_bytes": ws_bytes,
           "separate_calls_us": sep,
           "roofline": roofline("hbm", "decode_fused_kernel", gbs, peaks["hbm_gbs"], "GB/s",
                                traffic=measured_traffic(wl, "decode_fused_kernel"),
                                algorithmic=algo,
                                peak_source=peaks["source"] + " (burst copy)")}
    del graphs
    del layers
    torch.cuda.empty_cache()
    return out


def run_summaries_build(dev, peaks, layers, w, stream):
    """The summaries build over the whole cache of each layer (prefill-time state): one HBM read
    of K and the write of mean key, max norm and centre per block, as GB/s of those bytes."""
    import torch

    import block_sparse_attention_summaries_b200 as bsa
    B, Hk, d, n, b = (w[x] for x in ("B", "Hk", "d", "n", "b"))
    C = (n + b - 1) // b
    L0 = layers[0]
    mk, mx, ce = (torch.empty_like(L0[x]) for x in ("mean_k", "max_norm", "centre"))
    R = len(layers)
    fns = [lambda L=L: bsa.build_block_summaries(L["k"], b, None, 0, -1, mk, mx, ce)
           for L in layers]
    ts = []
    with torch.cuda.stream(stream):
        for f in fns:
            f()
        torch.cuda.synchronize(dev)
        for i in range(3 * R):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fns[i % R]()
            e1.record(stream)
            ts.append((e0, e1))
        torch.cuda.synchronize(dev)
    ms = statistics.fmean(a.elapsed_time(z) for a, z in ts)
    nbytes = B * Hk * n * d * 2 + B * Hk * C * (d + 2) * 4
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"kernel": "summaries_kernel", "ms": ms, "bytes": nbytes, "gbs": gbs,
            "roofline": roofline("hbm", "summaries_kernel", gbs, peaks["hbm_gbs"], "GB/s",
                                 algorithmic=nbytes,
                                 peak_source=peaks["source"] + " (burst copy)")}


def flat_rows(rows):
    """Scalar summary of the secondary rows (time, throughput, roofline fraction per row)."""
    out = {}
    sas = rows.get("sas_gated_prefill_16k")
    if sas:
        for key, name in (("forward", "sas_fwd"), ("gate_grad", "sas_gate_grad")):
            out[f"{name}_ms"] = sas[key]["ms"]
            out[f"{name}_tflops"] = sas[key]["tflops"]
            out[f"{name}_frac"] = sas[key]["roofline"]["frac"]
        out["sas_outer_fwd_frac"] = sas["outer_gate"]["roofline"]["frac"]
    fs = rows.get("freesolo_prefill_64k")
    if fs:
        for key, name in (("select", "freesolo_select"), ("attention", "freesolo_attn")):
            out[f"{name}_ms"] = fs[key]["ms"]
            out[f"{name}_tflops"] = fs[key]["tflops"]
            out[f"{name}_frac"] = fs[key]["roofline"]["frac"]
    ld = rows.get("long_decode_512k")
    if ld:
        out["long_decode_512k_us"] = ld["us_per_step"]
        out["long_decode_512k_tokens_per_s"] = ld["tokens_per_s"]
        out["long_decode_512k_frac"] = ld["roofline"]["frac"]
        out["long_decode_512k_selection_share"] = ld["separate_calls_us"]["selection_share"]
    fl = rows.get("fsl_decode_256k")
    if fl:
        out["fsl_decode_256k_us"] = fl["fsl_decode_ms"] * 1e3
        out["fsl_decode_256k_frac"] = fl["roofline"]["frac"]
        out["fsl_state_update_us"] = fl["fsl_state_update_ms"] * 1e3
        out["fsb_select_256k_us"] = fl["fsb_select_ms"] * 1e3
    sb = rows.get("summaries_build_32k")
    if sb:
        out["summaries_build_gbs"] = sb["gbs"]
        out["summaries_build_frac"] = sb["roofline"]["frac"]
    return out


def run_gpu(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = WORKLOADS[args.workload]
    case = make_case(args.workload)
    cpu_multi = cpu_single = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.prefill_only:
        # the oracle pool forks: before this process makes its first CUDA call
        cpu_multi, cpu_single = cpu_baselines(case, args.cpu_seconds)

    import torch
    import torch.distributed as dist

    import block_sparse_attention_summaries_b200 as bsa

    if args.prefill_only:
        torch.cuda.set_device(0)
        bsa.lib()
        rows = tuple(x for x in args.prefill_rows.split(",") if x)
        print(json.dumps({"prefill": run_prefill(torch.device("cuda", 0), load_peaks(),
                                                 rows=rows)}), flush=True)
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev)
    bsa.lib()
    peaks = load_peaks()

    B, Hq, Hk, d, n, b, K = (w[x] for x in ("B", "Hq", "Hk", "d", "n", "b", "K"))
    R = args.layers
    layers = build_layers(dev, case, w, R)
    status = torch.zeros(4, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(dev)
    # long histories take the two-launch path (bsa_decode_step_ws) through a workspace
    ws_bytes = bsa.decode_step_workspace_bytes(B, Hq, Hk, n, d, b, K)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes > 0 else None
    graphs = capture_fused(dev, layers, w, status, stream, ws=ws)
    launches_per_step = 2 if ws is not None else 1
    idx_h = layers[0]["idx"].cpu().numpy()
    acc = decode_accounting(case, w, idx_h)
    step_bytes = acc["kv_bytes"] + acc["summary_bytes"]  # selected K/V + summaries
    io_bytes = acc["io_bytes"]

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    with torch.cuda.stream(stream):
        replay_steps(graphs, args.warmup)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        sampler.mark("t0")
        # events bracket the K steps only: an event recorded between two steps costs the step
        # about 2 us (it ends the overlap of one launch's tail with the next one's start)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record(stream)
        replay_steps(graphs, args.steps)
        ev[1].record(stream)
        torch.cuda.synchronize(dev)
        sampler.mark("t1")
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
    total_ms = ev[0].elapsed_time(ev[1])

    sep = separate_calls(dev, layers, w, args.warmup, max(50, min(args.steps, 400)), stream)

    # GQA-shared selection and bf16 summaries (bsa_decode_step_ex flags): time per step on the same
    # rotated layers, algorithmic bytes, and how far the selection moves from the per-head fp32 one
    variants = {}
    G = Hq // Hk
    cur = (n - 1) // b
    ref_sets = [set(int(x) for x in row if x >= 0) for row in idx_h.reshape(-1, K)]
    for name, flags in (("bf16_summaries", bsa.DECODE_BF16_SUMMARIES),
                        ("per_head_fp32_control", 0),
                        ("shared_selection", bsa.DECODE_SHARED_SELECTION),
                        ("shared_bf16", bsa.DECODE_SHARED_SELECTION | bsa.DECODE_BF16_SUMMARIES)):
        bf16_sum = bool(flags & bsa.DECODE_BF16_SUMMARIES)
        # every buffer a captured graph uses stays referenced as long as the graphs live:
        # entering a capture empties the allocator's cache, so a buffer kept alive only by a
        # replaced closure would go back to the driver and its graph would replay into freed memory
        vbufs = []
        with torch.cuda.stream(stream):
            for L in layers:
                mk = bsa.round_summaries_bf16(L["mean_k"]) if bf16_sum else L["mean_k"].clone()
                vbufs.append(dict(L, mean_k=mk, idx=torch.empty(B, Hq, K, device=dev,
                                                               dtype=torch.int32)))

        def vstep(L, flags=flags):
            bsa.decode_step_ex(L["q"], L["k"], L["v"], L["mean_k"], b, K, flags, append=True,
                               max_norm=L["max_norm"], centre=L["centre"], o=L["o"],
                               lse=L["lse"], idx=L["idx"], count=L["count"], status=status)
        vgraphs = capture_steps(dev, vbufs, vstep, stream)
        vidx = vbufs[0]["idx"].cpu().numpy()
        nv = max(50, min(args.steps, 400))
        v_us = time_graph_cycle(dev, vgraphs, nv, args.warmup, stream) / nv * 1e3
        del vgraphs  # graphs first, then the buffers they replay into
        del vbufs
        v_union = v_hits = tot = 0
        for bi in range(B):
            for kh in range(Hk):
                sel = set(int(x) for x in vidx[bi, kh * G:(kh + 1) * G].ravel() if x >= 0)
                v_union += len(sel) + 1
                blocks = case.needles.get((bi, kh), [])
                v_hits += len(sel & set(int(c) for c in blocks))
                tot += len(blocks)
        v_kv = (v_union - B * Hk) * b * d * 2 * 2 + B * Hk * acc["cur_tokens"] * d * 2 * 2
        v_sum = B * Hk * cur * d * (2 if bf16_sum else 4)
        v_bytes = v_kv + v_sum + io_bytes
        agree = statistics.fmean(
            len(ref & set(int(x) for x in row if x >= 0)) / max(1, len(ref))
            for ref, row in zip(ref_sets, vidx.reshape(-1, K)))
        variants[name] = {"us_per_step": v_us, "tokens_per_s": B / (v_us / 1e6),
                          "algorithmic_bytes": v_bytes, "gbs": v_bytes / (v_us / 1e6) / 1e9,
                          "frac_of_hbm": v_bytes / (v_us / 1e6) / 1e9 / peaks["hbm_gbs"],
                          "union_blocks": v_union, "needle_recall": v_hits / max(1, tot),
                          "index_agreement_vs_per_head_fp32": agree}

    # end to end through the public API with host buffers: a prepared binding call per step
    # (bsa.DecodeStep -> bsa_decode_step_ws with DECODE_HOST_IO, no graph) whose q is page-locked
    # host memory that the step moves to the device itself and whose o it writes back to
    # page-locked host memory
    q_host = [torch.from_numpy(np.ascontiguousarray(L["q"].float().cpu().numpy()))
              .to(torch.bfloat16).pin_memory() for L in layers]
    o_host = torch.empty(B, Hq, d, dtype=torch.bfloat16).pin_memory()
    ws_io = torch.empty(bsa.decode_step_workspace_bytes(B, Hq, Hk, n, d, b, K,
                                                        bsa.DECODE_HOST_IO),
                        dtype=torch.uint8, device=dev)
    plans = [bsa.DecodeStep(q_host[r], L["k"], L["v"], L["mean_k"], b, K,
                            flags=bsa.DECODE_HOST_IO, append=True, max_norm=L["max_norm"],
                            centre=L["centre"], o=o_host, lse=L["lse"], idx=L["idx"],
                            count=L["count"], status=status, ws=ws_io)
             for r, L in enumerate(layers)]
    # two events bracket the timed steps, as for the device-only figure (an event between two
    # steps would add its own cost to every step)
    with torch.cuda.stream(stream):
        for i in range(args.warmup + args.steps):
            if i == args.warmup:
                torch.cuda.synchronize(dev)
                e0 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            plans[i % R](stream)
        e1 = torch.cuda.Event(enable_timing=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    e2e_total = e0.elapsed_time(e1)
    sampler.stop()
    clocks = sampler.summary()
    st_word = int(status.max().item())

    mx_total, e2e_total = job_timing(total_ms, e2e_total, world, dev)
    ms_per_step = mx_total / args.steps
    value = job_throughput(B, world, args.steps, mx_total)
    e2e_value = job_throughput(B, world, args.steps, e2e_total)

    avg_ms = total_ms / args.steps  # one fused kernel per step
    achieved = (step_bytes + io_bytes) / (avg_ms / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1), bf16-rounded, planted needle blocks)",
        "config": {"workload": args.workload, **{x: w[x] for x in ("B", "Hq", "Hk", "d", "n", "b",
                                                                   "K")},
                   "parallelism": f"replicas{world}",
                   "l2": f"inputs larger than L2: {R} rotated layer instances of the KV cache and "
                         "summaries (one step per instance in turn)",
                   "graphs": "one CUDA graph per decode iteration over the layers (one fused "
                             "kernel per layer step, programmatic dependent launch)"},
        "roofline": {"bound": "hbm", "kernel": "decode_fused_kernel",
                     "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"],
                     "traffic": measured_traffic(args.workload, "decode_fused_kernel"),
                     "algorithmic_bytes": step_bytes + io_bytes,
                     "peak_source": peaks["source"] + " (burst copy)"},
        "hbm": {"selected_kv_plus_summary_bytes": step_bytes,
                "gbs": step_bytes / (avg_ms / 1e3) / 1e9,
                "frac": step_bytes / (avg_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                "what": "selected K/V (union per GQA group) + summaries, per step time"},
        "separate_calls_us": sep,
        "variants": variants,
        "union_blocks": acc["union_blocks"], "per_head_blocks": acc["per_head_blocks"],
        "needle_recall": acc["needle_recall"], "status_word": st_word,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": B * Hq * d * 2,
                "d2h_bytes_per_step": B * Hq * d * 2,
                "what": "per step one prepared binding call (bsa.DecodeStep) into the C ABI "
                        "(bsa_decode_step_ws, DECODE_HOST_IO; no graph): q read from pinned "
                        "host memory into the device by the step's staging kernel, the fused "
                        "step, o written by it to pinned host memory; two CUDA events bracket "
                        "the timed steps"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": {k2: clocks[k2] for k2 in ("sm_mhz", "sm_max_mhz", "reasons")},
        "clock_samples": clocks["samples"],
    }
    rows = {}
    rows["summaries_build_32k"] = run_summaries_build(dev, peaks, layers, w, stream)
    del graphs, plans, layers
    torch.cuda.empty_cache()
    if not args.no_long and args.workload != "long_decode_512k":
        rows["long_decode_512k"] = run_long_decode(dev, peaks, args, stream)
    if not args.no_prefill:
        rows.update(run_prefill(dev, peaks))
    line["prefill"] = flat_rows(rows)
    line["rows"] = rows
    if cpu_multi is not None:
        line["cpu_baseline"] = cpu_multi
        line["cpu_baseline_one_thread"] = cpu_single
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="sas_gqa_decode_32k", choices=sorted(WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=8.0)
    ap.add_argument("--layers", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-long", action="store_true", help="skip the 512K long-decode row")
    ap.add_argument("--prefill-only", action="store_true",
                    help="time only the prefill rows (profiling the prefill kernels)")
    ap.add_argument("--prefill-rows", default="sas,freesolo,fsl",
                    help="with --prefill-only: which rows (sas, freesolo, fsl)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
