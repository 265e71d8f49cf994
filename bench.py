#!/usr/bin/env python3
"""Benchmark of the online-softmax attention hot path on B200 (one JSON line on stdout, rank 0).

One step = one pass over every step of the path on synthetic data already resident in HBM:
  * GQA causal prefill forward + backward, B=1, Hq=32, Hkv=8, S=4096, D=128, bf16
    (attn_fwd then attn_bwd), and
  * split-KV decode of 48 streams, Hq=32, Hkv=8, D=128, cache lengths uniform in [1024, 4096]
    (attn_decode_splitkv: split kernel + combine kernel).
`value` is the step's algorithmic attention FLOPs (forward 4*D per visible query/key pair per query
head, backward 2.5x that, decode 4*D per cached key per query head) divided by the device time of
the step, in TFLOP/s; `components` gives each part alone with its own roofline fraction (prefill
against the bf16 tensor peak, decode in KV GB/s against HBM bandwidth). The 44032-token causal
prefill forward and the sequence-512 transformer-block attention are measured as extra components.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events on the launch stream;
L2 is flushed between steps (a 512 MiB device write outside the events). The step time is the
median of the K steps (the mean is reported beside it). Nothing else is recorded inside that loop:
the per-kernel split (`kernels`, `roofline`) comes from a second, separate pass with CUDA events
around every launch. Multi-GPU: one process per GPU, every rank runs the same replica workload
(weak scaling; no data-path collective), the time is the max over ranks (an all-reduce of the
timing scalar only). `python bench.py --gpus N` without a process group starts the N ranks itself
(torchrun, rendezvous on 127.0.0.1); under an existing group --gpus must equal its size.

`--impl reference` times the fp64 CPU oracle (the only other implementation of this path) on a
bounded sample of the same workload (one query head of the prefill, two decode streams) and reports
the same metric over the sample's own work and measured seconds; the extrapolation to a whole step
is a labelled extra field. Under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention TFLOP/s fwd/bwd and decode KV GB/s on 1 B200, % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CSRC = os.path.join(ROOT, "online_softmax_attention_fwd_b200", "csrc")
# kernel family -> source file whose contents identify the kernel revision (for ncu traffic)
KERNEL_SOURCES = {"fwd_sm100": "fwd_sm100.cu", "bwd_sm100": "bwd_sm100.cu", "decode_split": "decode.cu",
                  "merge": "merge.cu", "fwd_sm100_fp8": "fwd_sm100.cu", "bwd_dkv_convert": "bwd_sm100.cu",
                  "decode_combine": "decode.cu", "bwd_simt_dq": "simt.cu", "bwd_simt_dkdv": "simt.cu",
                  "bwd_simt_delta": "simt.cu", "bwd_prep": "bwd_sm100.cu", "bwd_dq_convert": "bwd_sm100.cu"}


# ------------------------------------------------------------------------------------------------
# work accounting
# ------------------------------------------------------------------------------------------------

def visible_pairs(Sq: int, Sk: int, causal: bool) -> int:
    """Number of (query, key) pairs that are not masked (bottom-right aligned causal mask)."""
    if not causal:
        return Sq * Sk
    total = 0
    # row i sees keys 0 .. min(Sk-1, i + Sk - Sq)
    for i in range(Sq):
        total += max(0, min(Sk, i + Sk - Sq + 1))
    return total


def prefill_fwd_flops(B, Hq, Sq, Sk, D, causal) -> float:
    return 4.0 * D * Hq * B * visible_pairs(Sq, Sk, causal)


def decode_flops(lengths, Hq, D) -> float:
    return 4.0 * D * Hq * float(sum(int(x) for x in lengths))


def decode_bytes(lengths, Hq, Hkv, D) -> float:
    """Algorithmic decode bytes: K and V read once, Q read, O (bf16) and lse (fp32) written."""
    T = float(sum(int(x) for x in lengths))
    N = len(lengths)
    return 2.0 * T * Hkv * D * 2 + N * Hq * D * 2 * 2 + N * Hq * 4


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(family: str):
    src = KERNEL_SOURCES.get(family)
    if not src or not os.path.exists(os.path.join(CSRC, src)):
        return None
    h = hashlib.sha256()
    for f in (src, "common.cuh"):
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(family: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this kernel revision."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{family}:{workload}")
    if not e or e.get("source_hash") != kernel_source_hash(family):
        return None
    return float(e["dram_bytes_per_launch"])


# ------------------------------------------------------------------------------------------------
# clocks
# ------------------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 50):
        self.path = tempfile.mktemp(suffix=".csv")
        self.proc = None
        self.gpu = gpu_index
        self.period = period_ms

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", f"-lms={self.period}"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for r in csv.reader(f):
                if len(r) >= 9:
                    rows.append([x.strip() for x in r])
        os.unlink(self.path)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        sm = []
        smax = None
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
            except ValueError:
                continue
            for i, n in enumerate(names):
                if r[5 + i].lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# distributed helpers (also exercised by tests/test_multirank.py with gloo on CPU)
# ------------------------------------------------------------------------------------------------

def roofline_entry(prof: dict, work: dict, peaks: dict, peak_src: str, traffic_fn=None):
    """The `roofline` object for the kernel with the most live device time.

    prof: kernel family -> (total ms, launches) from the CUDA events; work: family -> (bound,
    algorithmic FLOPs or bytes per launch, or None when the kernel's work is not counted).
    achieved = work per launch / mean launch time, frac = achieved / the measured peak. A dominant
    kernel without a work figure (a CUDA-core kernel, or the decode combine, which comes out on top
    only under a profiler's serialised timing) gets no achieved figure and no fraction.
    """
    if not prof:
        return None
    traffic_fn = traffic_fn or ncu_traffic
    dom = max(prof.items(), key=lambda kv: kv[1][0])[0]
    ms, nl = prof[dom]
    per_launch_s = ms / 1e3 / nl
    bound, wk = work.get(dom, ("unknown", None))
    traffic = traffic_fn(dom, "gqa4k" if dom.startswith(("fwd", "bwd")) else "decode48")
    if bound == "tensor" and wk is not None:
        ach = wk / per_launch_s / 1e12
        return {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"],
                "frac_of_sustained": ach / peaks["bf16_tflops_sustained"], "traffic": traffic,
                "peak_source": f"{peak_src} (burst bf16)", "launch_ms": per_launch_s * 1e3}
    if bound == "hbm" and wk is not None:
        ach = wk / per_launch_s / 1e9
        return {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "traffic": traffic, "peak_source": peak_src,
                "launch_ms": per_launch_s * 1e3}
    return {"kernel": dom, "bound": "alu" if bound in ("alu", "unknown") else bound, "achieved": None,
            "peak": None, "unit": None, "frac": None, "traffic": traffic, "launch_ms": per_launch_s * 1e3,
            "note": "no algorithmic work figure for this kernel; no roofline fraction is claimed"}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(value: float, device=None) -> float:
    """Max of a scalar over all ranks (identity when no process group is initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(work_per_step_per_rank: float, steps: int, world: int, max_seconds: float) -> float:
    """Aggregate throughput: every rank's work over the slowest rank's time."""
    return work_per_step_per_rank * steps * world / max_seconds


# ------------------------------------------------------------------------------------------------
# CPU oracle baseline (rank 0, bounded sample)
# ------------------------------------------------------------------------------------------------

def oracle_sample(prefill, dec, n_heads: int, n_streams: int):
    """Runs the fp64 oracle on `n_heads` query heads of the prefill (forward + backward) and on
    `n_streams` decode streams; returns (seconds, extrapolated seconds for the whole step, cores)."""
    import numpy as np
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max([int(i.get("num_threads", 1)) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count() or 1
    f64 = lambda t: t.to("cpu").double().numpy()
    Hq = prefill.q.shape[2]
    G = Hq // prefill.k.shape[2]
    q, k, v, do = f64(prefill.q[:, :, :n_heads]), f64(prefill.k[:, :, : max(1, n_heads // G)]), \
        f64(prefill.v[:, :, : max(1, n_heads // G)]), f64(prefill.do[:, :, :n_heads])
    t0 = time.perf_counter()
    oracle.attention_fwd(q, k, v, prefill.causal, prefill.scale)
    oracle.attention_bwd(q, k, v, do, prefill.causal, prefill.scale)
    t1 = time.perf_counter()
    off = dec.offsets.numpy()
    sel = list(range(n_streams))
    qd = f64(dec.q[sel])
    lo, hi = int(off[0]), int(off[n_streams])
    kd, vd = f64(dec.k[lo:hi]), f64(dec.v[lo:hi])
    oracle.decode_attention(qd, kd, vd, off[: n_streams + 1] - lo, dec.scale)
    t2 = time.perf_counter()
    N = dec.q.shape[0]
    lengths = dec.meta["lengths"].numpy()
    frac_streams = float(lengths[:n_streams].sum()) / float(lengths.sum())
    extrap = (t1 - t0) * (Hq / n_heads) + (t2 - t1) / frac_streams
    return t2 - t0, extrap, cores


# ------------------------------------------------------------------------------------------------
# main benchmark
# ------------------------------------------------------------------------------------------------

def oracle_sample_flops(prefill, dec, n_heads: int, n_streams: int) -> float:
    """Algorithmic FLOPs of the work ``oracle_sample`` does (same convention as the GPU step)."""
    B, Sq, Hq, D = prefill.q.shape
    f = 3.5 * prefill_fwd_flops(B, n_heads, Sq, prefill.k.shape[1], D, prefill.causal)
    return f + decode_flops(dec.meta["lengths"][:n_streams], 1, D) * Hq


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import torch
    from online_softmax_attention_fwd_b200 import workloads as W
    torch.set_num_threads(os.cpu_count() or 1)
    pre = W.gqa_prefill_4k("A")
    dec = W.decode48()
    n_heads, n_streams = 1, 2
    sample_flops = oracle_sample_flops(pre, dec, n_heads, n_streams)
    for _ in range(args.warmup):
        oracle_sample(pre, dec, n_heads, n_streams)
    secs, extrap = [], []
    cores = 1
    for _ in range(args.steps):
        s, e, cores = oracle_sample(pre, dec, n_heads, n_streams)
        secs.append(s)
        extrap.append(e)
    t = statistics.median(secs)
    value = sample_flops / t / 1e12
    sample = ("per step: fp64 oracle forward+backward on 1 of 32 query heads of the 4k GQA prefill and "
              "decode of 2 of 48 streams; value = that sample's algorithmic FLOPs / its measured seconds")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample, "sample_seconds_per_step": t,
                             "extrapolated_full_step_seconds": statistics.median(extrap)},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_block():
    return {"workload": "gqa_causal_prefill_b1_hq32_hkv8_s4096_d128_fwd_bwd + decode_n48_hq32_hkv8_d128_len1024-4096",
            "global_batch": 1, "seq_len": 4096, "decode_streams": 48, "heads_q": 32, "heads_kv": 8,
            "head_dim": 128, "causal": True, "parallelism": "replicas (weak scaling)",
            "l2": "flushed between timed steps (512 MiB device write outside the step events)"}


def run_ours(args):
    import torch
    import torch.distributed as dist

    import online_softmax_attention_fwd_b200 as attn
    from online_softmax_attention_fwd_b200 import workloads as W

    ws, rank, local = dist_env()
    if ws > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    attn.lib()
    peaks, peak_src = load_peaks()

    pre = W.gqa_prefill_4k("A")
    dec = W.decode48()
    B, Sq, Hq, D = pre.q.shape
    Hkv = pre.k.shape[2]
    q, k, v, do = (t.to(dev) for t in (pre.q, pre.k, pre.v, pre.do))
    o, lse = torch.empty_like(q), torch.empty(B, Hq, Sq, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsb = torch.empty(attn.bwd_workspace_size(B, Hq, Hkv, Sq, Sq, D), dtype=torch.uint8, device=dev)
    qd, kd, vd, off = (t.to(dev) for t in (dec.q, dec.k, dec.v, dec.offsets))
    od, lsed = torch.empty_like(qd), torch.empty(qd.shape[0], Hq, dtype=torch.float32, device=dev)
    wsd = torch.empty(attn.decode_workspace_size(qd.shape[0], Hq, D, 16), dtype=torch.uint8, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    f_fwd = prefill_fwd_flops(B, Hq, Sq, Sq, D, True)
    f_bwd = 2.5 * f_fwd
    lengths = dec.meta["lengths"]
    f_dec = decode_flops(lengths, Hq, D)
    b_dec = decode_bytes(lengths, Hq, Hkv, D)
    step_flops = f_fwd + f_bwd + f_dec

    def part_fwd():
        attn.fwd(q, k, v, causal=True, scale=pre.scale, out=o, lse=lse)

    def part_bwd():
        attn.bwd(q, k, v, o, lse, do, causal=True, scale=pre.scale, workspace=wsb, out=(dq, dk, dv))

    def part_dec():
        attn.decode(qd, kd, vd, off, max_splits=16, scale=dec.scale, out=od, lse=lsed, workspace=wsd)

    def step():
        part_fwd()
        part_bwd()
        part_dec()

    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    # ---------------- timed region: K steps, per-step events, L2 flushed between steps (the flush
    # runs outside the events); no per-launch profiling events inside this loop
    sampler = ClockSampler(local)
    sampler.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = attn.launch_count()
    t_wall0 = time.perf_counter()
    for i in range(args.steps):
        flush.zero_()
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall0
    launches = attn.launch_count() - launches0
    if ws > 1:
        dist.barrier()
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    med_s = reduce_max(statistics.median(step_ms) / 1e3, dev)
    mean_s = reduce_max(statistics.mean(step_ms) / 1e3, dev)
    value = whole_job_rate(step_flops, 1, ws, med_s) / 1e12
    status = attn.device_status()

    # ---------------- per-kernel split: a second, separate pass with CUDA events around every launch
    prof_steps = max(3, min(args.steps, 20))
    for _ in range(2):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    attn.profile_start()
    for _ in range(prof_steps):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    prof = attn.profile_stop()

    # ---------------- per-part timing (each part alone, same hygiene) for the components
    def time_part(fn, iters):
        es = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
        for _ in range(2):
            flush.zero_()
            fn()
        for a, b in es:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in es) / 1e3

    iters = max(5, min(args.steps, 30))
    t_fwd, t_bwd, t_dec = time_part(part_fwd, iters), time_part(part_bwd, iters), time_part(part_dec, iters)
    components = {
        "gqa4k_fwd": {"ms": t_fwd * 1e3, "tflops": f_fwd / t_fwd / 1e12,
                      "frac_of_bf16_peak": f_fwd / t_fwd / 1e12 / peaks["bf16_tflops"]},
        "gqa4k_bwd": {"ms": t_bwd * 1e3, "tflops": f_bwd / t_bwd / 1e12,
                      "frac_of_bf16_peak": f_bwd / t_bwd / 1e12 / peaks["bf16_tflops"],
                      "tflops_2x_convention": 2.0 * f_fwd / t_bwd / 1e12},
        "decode48": {"ms": t_dec * 1e3, "kv_gbs": b_dec / t_dec / 1e9,
                     "frac_of_hbm": b_dec / t_dec / 1e9 / peaks["hbm_gbs"]},
    }
    if not args.no_extras:
        for causal in (False, True):
            wb = W.block512(causal)
            qb, kb, vb, dob = (t.to(dev) for t in (wb.q, wb.k, wb.v, wb.do))
            ob, lb = attn.fwd(qb, kb, vb, causal=causal, scale=wb.scale)
            fb = prefill_fwd_flops(4, 16, 512, 512, 64, causal)
            tf = time_part(lambda: attn.fwd(qb, kb, vb, causal=causal, scale=wb.scale, out=ob, lse=lb), iters)
            tb = time_part(lambda: attn.bwd(qb, kb, vb, ob, lb, dob, causal=causal, scale=wb.scale), iters)
            components[f"block512_{'causal' if causal else 'full'}"] = {
                "fwd_ms": tf * 1e3, "fwd_tflops": fb / tf / 1e12, "bwd_ms": tb * 1e3,
                "bwd_tflops": 2.5 * fb / tb / 1e12}
            del qb, kb, vb, dob, ob, lb
        # the same 48 decode streams read from a paged cache (64-key pages, shuffled pool)
        pc = W.paged_from_packed(dec, 64, seed=0)
        kp, vp, bt, sl = (t.to(dev) for t in (pc.k_pages, pc.v_pages, pc.block_table, pc.seq_lens))
        t_pg = time_part(lambda: attn.decode_paged(qd, kp, vp, bt, sl, max_splits=16, scale=dec.scale, out=od,
                                                   lse=lsed, workspace=wsd), iters)
        components["decode48_paged64"] = {"ms": t_pg * 1e3, "kv_gbs": b_dec / t_pg / 1e9,
                                          "frac_of_hbm": b_dec / t_pg / 1e9 / peaks["hbm_gbs"]}
        del kp, vp, bt, sl, pc
        # the same 48 streams with four query tokens each (a speculative step): same keys read once
        wq = W.random_decode(48, 32, 8, 128, lengths.tolist(), seed=0, q_len=4)
        qd4 = wq.q.to(dev)
        od4 = torch.empty_like(qd4)
        l4 = torch.empty(48, 32, 4, dtype=torch.float32, device=dev)
        ws4 = torch.empty(attn.decode_workspace_size(48 * 4, Hq, D, 16), dtype=torch.uint8, device=dev)
        t_d4 = time_part(lambda: attn.decode(qd4, kd, vd, off, max_splits=16, scale=dec.scale, out=od4, lse=l4,
                                             workspace=ws4), iters)
        b_d4 = decode_bytes(lengths, Hq * 4, Hkv, D)
        components["decode48_qlen4"] = {"ms": t_d4 * 1e3, "kv_gbs": b_d4 / t_d4 / 1e9,
                                        "frac_of_hbm": b_d4 / t_d4 / 1e9 / peaks["hbm_gbs"],
                                        "tflops": 4 * f_dec / t_d4 / 1e12}
        del qd4, od4, l4, ws4
        # packed variable-length prefill: 8 causal prompts of 512-4096 tokens, forward and backward
        wv = W.varlen_prefill_8x()
        qv, kv_, vv, dov, cqv, ckv = (t.to(dev) for t in (wv.q, wv.k, wv.v, wv.do, wv.cu_q, wv.cu_k))
        lv = wv.meta["lengths_q"].tolist()
        mv = max(lv)
        fv = sum(prefill_fwd_flops(1, 32, L, L, 128, True) for L in lv)
        ov, lsev = attn.fwd_varlen(qv, kv_, vv, cqv, ckv, mv, mv, causal=True, scale=wv.scale)
        wsv = torch.empty(attn.lib().attn_bwd_varlen_workspace_size(8, 32, 8, mv, mv, 128), dtype=torch.uint8, device=dev)
        gv = tuple(torch.empty_like(t) for t in (qv, kv_, vv))
        t_vf = time_part(lambda: attn.fwd_varlen(qv, kv_, vv, cqv, ckv, mv, mv, causal=True, scale=wv.scale,
                                                 out=ov, lse=lsev), iters)
        t_vb = time_part(lambda: attn.bwd_varlen(qv, kv_, vv, ov, lsev, dov, cqv, ckv, mv, mv, causal=True,
                                                 scale=wv.scale, workspace=wsv, out=gv), iters)
        components["varlen8x_fwd"] = {"ms": t_vf * 1e3, "tflops": fv / t_vf / 1e12,
                                      "frac_of_bf16_peak": fv / t_vf / 1e12 / peaks["bf16_tflops"],
                                      "tokens": sum(lv)}
        components["varlen8x_bwd"] = {"ms": t_vb * 1e3, "tflops": 2.5 * fv / t_vb / 1e12,
                                      "frac_of_bf16_peak": 2.5 * fv / t_vb / 1e12 / peaks["bf16_tflops"]}
        del qv, kv_, vv, dov, ov, lsev, wsv, gv
        # FP8 (e4m3) forward at the 4k GQA shape, against the fp8 dense peak (2x the measured bf16)
        w8 = W.fp8_prefill(1, 4096, 4096, 32, 8, 128, True, seed=0)
        q8, k8, v8 = (t.to(dev) for t in (w8.q, w8.k, w8.v))
        o8, l8 = attn.fwd_fp8(q8, k8, v8, w8.q_scale, w8.k_scale, w8.v_scale, causal=True, scale=w8.scale)
        t8 = time_part(lambda: attn.fwd_fp8(q8, k8, v8, w8.q_scale, w8.k_scale, w8.v_scale, causal=True,
                                            scale=w8.scale, out=o8, lse=l8), iters)
        components["fp8_gqa4k_fwd"] = {"ms": t8 * 1e3, "tflops": f_fwd / t8 / 1e12,
                                       "frac_of_fp8_peak": f_fwd / t8 / 1e12 / (2.0 * peaks["bf16_tflops"]),
                                       "fp8_peak_note": "2 x measured bf16 (nominal fp8 / bf16 dense ratio 4.5 / 2.25)"}
        del q8, k8, v8, o8, l8
        # monoid merge of two partial attentions of the 4k prefill's shape (a context-parallel step)
        o_acc = torch.zeros(B, Sq, Hq, D, dtype=torch.float32, device=dev)
        l_acc = torch.zeros(B, Hq, Sq, dtype=torch.float32, device=dev)
        o_mo = torch.empty_like(o)
        t_m = time_part(lambda: attn.merge(o_acc, l_acc, o, lse, o_mo), iters)
        b_m = B * Sq * Hq * D * (4 + 4 + 2 + 2) + B * Hq * Sq * 4 * 3
        components["merge_gqa4k"] = {"ms": t_m * 1e3, "gbs": b_m / t_m / 1e9,
                                     "frac_of_hbm": b_m / t_m / 1e9 / peaks["hbm_gbs"]}
        del o_acc, l_acc, o_mo
        w5 = W.long_prefill_44k()
        q5, k5, v5 = (t.to(dev) for t in (w5.q, w5.k, w5.v))
        o5, l5 = attn.fwd(q5, k5, v5, causal=True, scale=w5.scale)
        f5 = prefill_fwd_flops(1, 32, 44032, 44032, 128, True)
        t5 = time_part(lambda: attn.fwd(q5, k5, v5, causal=True, scale=w5.scale, out=o5, lse=l5), 3)
        components["long44k_fwd"] = {"ms": t5 * 1e3, "tflops": f5 / t5 / 1e12,
                                     "frac_of_bf16_peak": f5 / t5 / 1e12 / peaks["bf16_tflops"]}
        del q5, k5, v5, o5, l5

    # ---------------- roofline of the dominant kernel (live CUDA events around each launch)
    work = {"fwd_sm100": ("tensor", f_fwd), "bwd_sm100": ("tensor", f_bwd), "merge": ("hbm", None),
            "bwd_simt_dq": ("alu", None), "bwd_simt_dkdv": ("alu", None),
            "decode_split": ("hbm", b_dec), "decode_combine": ("hbm", None)}
    roofline = roofline_entry(prof, work, peaks, peak_src)
    kernels = {n: {"total_ms": ms, "launches": nl, "share": ms / max(1e-12, sum(x[0] for x in prof.values()))}
               for n, (ms, nl) in prof.items()}

    # ---------------- end to end through the C ABI with host buffers
    pin = lambda t: t.to("cpu").pin_memory()
    h_in = [pin(t) for t in (pre.q, pre.k, pre.v, pre.do, dec.q, dec.k, dec.v, dec.offsets)]
    d_in = [q, k, v, do, qd, kd, vd, off]
    d_out = [o, lse, dq, dk, dv, od, lsed]
    h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in d_out]
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = sum(t.numel() * t.element_size() for t in h_out)
    e2e_iters = max(3, min(args.steps, 10))
    es = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_iters + 1)]
    for i, (a, b) in enumerate(es):
        flush.zero_()
        a.record(stream)
        for hsrc, ddst in zip(h_in, d_in):
            ddst.copy_(hsrc, non_blocking=True)
        step()
        for dsrc, hdst in zip(d_out, h_out):
            hdst.copy_(dsrc, non_blocking=True)
        b.record(stream)
    torch.cuda.synchronize()
    e2e_s = statistics.mean(a.elapsed_time(b) for a, b in es[1:]) / 1e3
    e2e_value = whole_job_rate(step_flops, 1, ws, reduce_max(e2e_s, dev)) / 1e12

    # ---------------- CPU baseline: the oracle on a bounded sample (rank 0, N = 1)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        secs, extrap, cores = oracle_sample(pre, dec, 4, 8)
        cpu = {"value": step_flops / extrap / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": ("fp64 oracle forward+backward on 4 of 32 query heads (one GQA group) of the 4k "
                          "prefill and decode of 8 of 48 streams, extrapolated by head and cached-key "
                          f"count; {secs:.1f} s of CPU"),
               "extrapolated_step_seconds": extrap}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": med_s * 1e3, "ms_per_step_mean": mean_s * 1e3,
                "step_statistic": "median over the K timed steps, max over ranks", "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": config_block(), "clocks": clocks,
                "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h, "ms_per_step": e2e_s * 1e3},
                "gpu_launches": launches, "roofline": roofline, "cpu_baseline": cpu,
                "components": components, "kernels": kernels,
                "kernels_note": f"per-kernel CUDA events from a separate {prof_steps}-step pass after the timed region",
                "wall_s_timed_region": t_wall, "device_status": status,
                "peaks": {**peaks, "source": peak_src}}
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0 if status == 0 else 1


def run_case(name):
    """One launch of each kernel of a workload and nothing else (a small command for ncu captures):
    `prefill` = the 4k GQA causal forward and backward, `decode` = the 48-stream split-KV decode,
    `decode_paged` = the same 48 streams read from a cache of 64-key pages, `decode_qlen` = the 48
    streams with four query tokens each, `varlen` = the packed 8-prompt prefill forward and backward,
    `fp8` = the FP8 forward at the 4k GQA shape,
    `long` = the forward of the long-prefill workload at S = 16384 (the 44k workload's construction
    and kernel at a size that a full ncu capture handles; about 0.4 GB on the device)."""
    import torch
    import online_softmax_attention_fwd_b200 as attn
    from online_softmax_attention_fwd_b200 import workloads as W
    dev = torch.device("cuda")
    if name == "long":
        w = W.long_prefill_44k(S=16384)
        q, k, v = (t.to(dev) for t in (w.q, w.k, w.v))
        attn.fwd(q, k, v, causal=True, scale=w.scale)
    elif name == "prefill":
        w = W.gqa_prefill_4k("A")
        q, k, v, do = (t.to(dev) for t in (w.q, w.k, w.v, w.do))
        o, lse = attn.fwd(q, k, v, causal=True, scale=w.scale)
        attn.bwd(q, k, v, o, lse, do, causal=True, scale=w.scale)
    elif name == "decode_qlen":
        wd = W.decode48()
        wq = W.random_decode(48, 32, 8, 128, wd.meta["lengths"].tolist(), seed=0, q_len=4)
        q, k, v, off = (t.to(dev) for t in (wq.q, wd.k, wd.v, wd.offsets))
        attn.decode(q, k, v, off, scale=wd.scale)
    elif name == "varlen":
        w = W.varlen_prefill_8x()
        q, k, v, do, cq, ck = (t.to(dev) for t in (w.q, w.k, w.v, w.do, w.cu_q, w.cu_k))
        m = int(w.meta["lengths_q"].max())
        o, lse = attn.fwd_varlen(q, k, v, cq, ck, m, m, causal=True, scale=w.scale)
        attn.bwd_varlen(q, k, v, o, lse, do, cq, ck, m, m, causal=True, scale=w.scale)
    elif name == "fp8":
        w = W.fp8_prefill(1, 4096, 4096, 32, 8, 128, True, seed=0)
        q, k, v = (t.to(dev) for t in (w.q, w.k, w.v))
        attn.fwd_fp8(q, k, v, w.q_scale, w.k_scale, w.v_scale, causal=True, scale=w.scale)
    elif name == "decode_paged":
        wd = W.decode48()
        pc = W.paged_from_packed(wd, 64, seed=0)
        q, kp, vp, bt, sl = (t.to(dev) for t in (wd.q, pc.k_pages, pc.v_pages, pc.block_table, pc.seq_lens))
        attn.decode_paged(q, kp, vp, bt, sl, scale=wd.scale)
    else:
        wd = W.decode48()
        q, k, v, off = (t.to(dev) for t in (wd.q, wd.k, wd.v, wd.offsets))
        attn.decode(q, k, v, off, scale=wd.scale)
    torch.cuda.synchronize()
    status = attn.device_status()
    print(json.dumps({"case": name, "device_status": status}))
    return 0 if status == 0 else 1


def launch_ranks(n: int, script: str, argv, port: int = 0, timeout_s: float = 1800.0) -> int:
    """Runs ``script argv`` as ``n`` ranks of one node under torchrun (rendezvous on 127.0.0.1),
    passing through what the ranks print; returns torchrun's exit code. ``bench.py --gpus N`` uses it
    when it is started without a process group (no WORLD_SIZE in the environment)."""
    if port == 0:
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", script] + list(argv)
    r = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=sys.stderr, text=True, timeout=timeout_s)
    sys.stdout.write(r.stdout)
    sys.stdout.flush()
    return r.returncode


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--case", choices=["prefill", "decode", "long", "decode_paged", "decode_qlen", "varlen", "fp8"],
                    help="run one launch of each kernel of this workload and exit (for profilers)")
    args = ap.parse_args()
    if args.case:
        return run_case(args.case)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    ws = int(os.environ.get("WORLD_SIZE", "0"))
    if ws == 0 and args.gpus > 1:
        # no process group yet: start one rank per GPU and let them run this same command
        return launch_ranks(args.gpus, os.path.abspath(__file__), sys.argv[1:])
    if ws and ws != args.gpus:
        ap.error(f"--gpus {args.gpus} does not match the {ws} ranks of this process group")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
