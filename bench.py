#!/usr/bin/env python
"""Benchmark of one absorbed-MLA decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long] [--impl reference]

A step is one pass of the whole path over one batch: append the batch's new
cache rows, absorb the queries, split-KV attention, combine, up-project.  The
default workload is the long-context one (8 sequences x 131072 cached rows,
128 heads, bf16 paged cache, 64 splits of 2048 rows); its 1.21 GB cache is
larger than L2, so successive steps stream it from HBM.

Rank 0 prints one JSON line.  Under torchrun each rank runs the same workload
on its own GPU (independent sequences, no data-path collective: weak scaling);
time is the max over ranks.  `--impl reference` times the CPU fp64 oracle
instead, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "MLA decode tokens/s, latent-cache HBM GB/s and % of B200 roofline"
CACHE_BYTES = {"f32": 2304, "bf16": 1152, "e4m3": 580}   # per cached row: 576 numbers (+ fp32 scale)
DECODE_SRC = ["latent_attention_decode_absorbed_b200/csrc/decode_pair.cu",
              "latent_attention_decode_absorbed_b200/csrc/decode_tc.cu",
              "latent_attention_decode_absorbed_b200/csrc/sm100.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_traffic.json")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def tensor_peak(pk, mma):
    """Dense tensor peak for the decode's MMA operand type: the measured bf16
    figure (also the f16 one), or for e4m3 operands that figure times the
    nominal dense ratio 2 (4.5 against 2.25 PFLOP/s)."""
    return pk["bf16_tflops"] * (2.0 if mma == "e4m3" else 1.0)


def binding_roofline(alg_bytes, alg_flops, launch_ms, pk, traffic, mma="bf16"):
    """The decode launch against its binding roofline: the cache bytes at the
    HBM peak or the contraction FLOPs at the tensor peak of its MMA operand
    type (bf16; f16 for the widened e4m3 cache; e4m3 for the 8-bit form),
    whichever takes longer."""
    s = launch_ms / 1e3
    tpk = tensor_peak(pk, mma)
    if alg_flops / (tpk * 1e12) > alg_bytes / (pk["hbm_gbs"] * 1e9):
        achieved = alg_flops / s / 1e12
        r = {"bound": "tensor", "achieved": achieved, "peak": tpk, "unit": "TFLOP/s",
             "frac": achieved / tpk, "traffic": traffic, "mma": mma,
             "frac_of_bf16_peak": achieved / pk["bf16_tflops"]}
    else:
        achieved = alg_bytes / s / 1e9
        r = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
             "frac": achieved / pk["hbm_gbs"], "traffic": traffic}
    r.update({"kernel": "mla_decode_fwd", "peak_source": pk["source"], "algorithmic_bytes_per_launch": alg_bytes,
              "algorithmic_flops_per_launch": alg_flops, "launch_ms": launch_ms})
    return r


def mma_type(step):
    """Operand type of the decode's MMAs for a DecodeStep."""
    if getattr(step, "q8", False):
        return "e4m3"
    return "f16" if step.cache_dtype == 2 else "bf16"


def decode_src_hash():
    h = hashlib.sha256()
    for f in DECODE_SRC:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per decode launch measured by ncu (profiles/decode_traffic.json),
    if the entry was taken on the current decode kernel source for this workload."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    src = decode_src_hash()
    for e in json.load(open(TRAFFIC_FILE)).get("entries", []):
        if e.get("workload") == workload and e.get("src") == src:
            return int(e["bytes"])
    return None


def max_over_ranks(values, world, device=None):
    """Element-wise max of per-rank timings (list of floats) over all ranks.

    Multi-GPU numbers are the slowest rank's: every rank times the same K
    steps between barriers, and the job is done when the last one is."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world, tokens_per_step, steps, elapsed_ms):
    """Whole-job tokens/s: every rank completes `tokens_per_step` query tokens
    per step (independent sequences per GPU, weak scaling)."""
    return world * tokens_per_step * steps / (elapsed_ms / 1e3)


def algorithmic(w, lens):
    rows = int(lens.sum())
    bytes_ = rows * CACHE_BYTES[w.cache_dtype]
    vis = sum(int(L) - w.q_len + t + 1 for L in lens for t in range(w.q_len))  # rows seen, all queries
    flops = 2.0 * w.n_heads * vis * (576 + 512)
    return bytes_, flops


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = os.path.join("/tmp", f"mla_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0])); smax = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_smi_id(dev_index):
    import torch
    try:
        p = torch.cuda.get_device_properties(dev_index)
        return f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
    except Exception:
        return dev_index


# ------------------------------------------------------------------ CPU oracle timing
def time_oracle(w, heads, budget_s, min_reps=1):
    """Time the fp64 oracle's absorbed step for sequence 0's query rows over
    its full cache, restricted to `heads` heads; repeat up to budget_s.
    The cache (RMSNorm/RoPE of every row) is state built before timing, as on
    the GPU.  Returns (query tokens per second, reps, seconds, cores)."""
    import oracle
    kv = W.kv_rows(w, 0)
    c_hat, k_r = oracle.sequence_cache(kv, w.cache_dtype, None, w.eps, w.theta)
    qn, qp = W.queries(w)
    wuk, wuv = W.weights(w)
    hs = slice(0, heads)
    qn, qp = qn[:w.q_len, hs], qp[:w.q_len, hs]
    wuk, wuv = wuk[hs], wuv[hs]
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.attention_absorbed(qn, qp, wuk, wuv, c_hat, k_r)
        reps += 1
        el = time.perf_counter() - t0
        if reps >= min_reps and el >= budget_s:
            break
        if reps >= min_reps and el * (reps + 1) / reps > 3 * budget_s:
            break
    tokens = reps * w.q_len * heads / w.n_heads
    cores = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        cores = max(i.get("num_threads", 1) for i in threadpool_info()) or cores
    except Exception:
        pass
    return tokens / el, reps, el, cores


def run_reference(args, w, rank, world):
    if rank != 0:
        return 0
    lens = W.seq_lens(w)
    heads = min(16, w.n_heads)
    # one "step" = sequence 0's query rows over its whole cache for `heads` heads
    import oracle
    kv = W.kv_rows(w, 0)
    c_hat, k_r = oracle.sequence_cache(kv, w.cache_dtype, None, w.eps, w.theta)
    qn, qp = W.queries(w)
    wuk, wuv = W.weights(w)
    qn, qp, wuk, wuv = qn[:w.q_len, :heads], qp[:w.q_len, :heads], wuk[:heads], wuv[:heads]
    for _ in range(args.warmup):
        oracle.attention_absorbed(qn, qp, wuk, wuv, c_hat, k_r)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.attention_absorbed(qn, qp, wuk, wuv, c_hat, k_r)
    el = time.perf_counter() - t0
    tokens = args.steps * w.q_len * heads / w.n_heads
    value = tokens / el
    cores = os.cpu_count()
    sample = (f"sequence 0 of {w.batch}: {w.q_len} query row(s) x {heads} of {w.n_heads} heads over all "
              f"{int(lens[0])} cached rows per step (= {heads / w.n_heads:.4f} query tokens); absorbed fp64 "
              f"oracle, cache built before timing")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, lens),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, lens):
    return {"workload": w.name, "batch": w.batch, "q_len": w.q_len, "n_heads": w.n_heads,
            "seq_len": int(lens.max()) if w.seq_len else f"U[{w.len_range[0]},{w.len_range[1]}]",
            "cached_rows": int(lens.sum()), "cache_dtype": w.cache_dtype, "qw_dtype": w.dtype,
            "paged": w.paged, "page_size": 64, "split_tokens": w.split_tokens,
            "dims": "d_c=512 d_rope=64 d_nope=128 d_v=128", "parallelism": "replicas (independent sequences per GPU)",
            "l2": "no flush: the cache is larger than L2" if int(lens.sum()) * CACHE_BYTES[w.cache_dtype] > 256e6
            else "L2 flushed before every step (256 MB write)"}


# ------------------------------------------------------------------ GPU arm
def _timed_steps(torch, step_fn, steps, stream, flush, barrier, decode_events=True):
    """Time `steps` calls of step_fn(ev) on the device.  Without an L2 flush
    the steps run back to back between two events; with one, the flush runs
    before each step, outside that step's own pair of events, and the step
    time is the sum of the per-step intervals.  Returns (total ms of the
    timed steps, per-step decode-launch ms list)."""
    dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) if decode_events else None
           for _ in range(steps)]
    barrier(); torch.cuda.synchronize()
    if flush is None:
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(steps):
            step_fn(dec[i])
        t1.record(stream)
        torch.cuda.synchronize(); barrier()
        total = t0.elapsed_time(t1)
    else:
        se = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            flush.fill_(1.0)
            se[i][0].record(stream)
            step_fn(dec[i])
            se[i][1].record(stream)
        torch.cuda.synchronize(); barrier()
        total = sum(a.elapsed_time(b) for a, b in se)
    return total, [e[0].elapsed_time(e[1]) for e in dec] if decode_events else []


def _decode_summary(alg_bytes, alg_flops, dec_ms, step_ms, pk, mma="bf16"):
    tpk = tensor_peak(pk, mma)
    roof_ms = 1e3 * max(alg_bytes / (pk["hbm_gbs"] * 1e9), alg_flops / (tpk * 1e12))
    return {"cache_gbs": alg_bytes / (dec_ms / 1e3) / 1e9, "tflops": alg_flops / (dec_ms / 1e3) / 1e12,
            "tensor_frac_burst": alg_flops / (dec_ms / 1e3) / 1e12 / tpk,
            "roofline_ms": roof_ms, "roofline_frac": roof_ms / dec_ms, "share_of_step": dec_ms / step_ms}


def run_gpu(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from workloads.device import DeviceWorkload
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dw = DeviceWorkload(w, device=dev, q8=False if args.f16_operands else None)
    step = dw.step
    lens = dw.lens
    stream = torch.cuda.current_stream(dev)
    alg_bytes, alg_flops = algorithmic(w, lens)
    # workloads whose cache would stay in L2 get a 256 MB write before every
    # step, outside the step's timed interval
    flush = None
    if alg_bytes <= 256e6:
        flush = torch.empty(int(256e6) // 4, dtype=torch.float32, device=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    # the step's five launches, recorded once as CUDA graphs (pre, attend,
    # post) and replayed: small steps are otherwise bound by host-side calls
    graphs = step.capture(dw.kv_new, dw.seq_ids, dw.positions, dw.q_nope, dw.q_pe, dw.w_uk, dw.w_uv)

    def one_step(ev=None):
        graphs.pre.replay()
        if ev is not None:
            ev[0].record(stream)
        graphs.attend.replay()
        if ev is not None:
            ev[1].record(stream)
        graphs.post.replay()

    for _ in range(args.warmup):
        if flush is not None:
            flush.fill_(1.0)
        one_step()
    torch.cuda.synchronize()
    assert int(step.err.item()) == 0, "device error flag set"
    with ClockSampler(gpu_smi_id(local_rank)) as clk:
        elapsed_ms, decode_ms = _timed_steps(torch, one_step, args.steps, stream, flush, barrier)
    clocks = clk.summary()
    # end-to-end through the public API: pinned host inputs in, host output back, every step
    h_kv = dw.kv_new.cpu().pin_memory()
    h_qn, h_qp = dw.q_nope.cpu().pin_memory(), dw.q_pe.cpu().pin_memory()
    h_out = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    h2d = h_kv.numel() * h_kv.element_size() + h_qn.numel() * h_qn.element_size() + h_qp.numel() * h_qp.element_size()
    d2h = h_out.numel() * h_out.element_size()

    # the same step with the inputs copied in from pinned host memory and the
    # output copied back, recorded as graphs through DecodeStep.capture
    e2e_graphs = step.capture(dw.kv_new, dw.seq_ids, dw.positions, dw.q_nope, dw.q_pe, dw.w_uk, dw.w_uv,
                              host_in=[(dw.kv_new, h_kv), (dw.q_nope, h_qn), (dw.q_pe, h_qp)], host_out=h_out)

    def e2e_step(ev=None):
        e2e_graphs.replay()

    for _ in range(max(3, args.warmup)):
        if flush is not None:
            flush.fill_(1.0)
        e2e_step()
    e2e_ms, _ = _timed_steps(torch, e2e_step, args.steps, stream, flush, barrier, decode_events=False)
    assert int(step.err.item()) == 0, "device error flag set"

    # max over ranks
    elapsed_ms, e2e_ms, dec_ms = max_over_ranks([elapsed_ms, e2e_ms, float(np.mean(decode_ms))], world, dev)
    extra = level2 = None
    if world == 1 and not args.no_extra and w.name == "long":
        extra = time_extra(args, "fp8_mtp", dev, stream)
        level2 = time_level2(args, dev, stream)
    if rank != 0:
        return 0
    tokens_per_step = w.batch * w.q_len
    value = job_throughput(world, tokens_per_step, args.steps, elapsed_ms)
    e2e_value = job_throughput(world, tokens_per_step, args.steps, e2e_ms)
    pk = peaks()
    traffic = recorded_traffic(w.name)
    roofline = binding_roofline(alg_bytes, alg_flops, dec_ms, pk, traffic, mma_type(step))
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic", "config": workload_config(w, lens),
        "roofline": roofline,
        "decode": _decode_summary(alg_bytes, alg_flops, dec_ms, elapsed_ms / args.steps, pk, mma_type(step)),
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": step.launches_per_step * args.steps,
        "clocks": clocks,
    }
    if extra is not None:
        line["fp8_mtp"] = extra
    if level2 is not None:
        line["level2_comparison"] = level2
    if not args.no_cpu_baseline and world == 1:
        v, reps, el, cores = time_oracle(w, heads=w.n_heads, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": f"{reps} x sequence 0's {w.q_len} query row(s), all {w.n_heads} heads, "
                                          f"over {int(lens[0])} cached rows ({el:.1f} s); absorbed fp64 oracle, "
                                          f"cache built before timing"}
    print(json.dumps(line), flush=True)
    return 0


def time_level2(args, dev, stream):
    """The non-absorbed ("level 2") decode next to the absorbed one on the
    one-sequence workload (v3_b1): per-head keys and values decompressed from
    the latents (mla_decompress_kv) and standard attention over them
    (mla_attend_naive), against absorb_q + decode + combine + out_uv, both
    producing the per-head outputs.  Each timed after a 256 MB L2 flush."""
    import torch
    import latent_attention_decode_absorbed_b200 as mla
    from workloads.device import DeviceWorkload
    w = W.WORKLOADS["v3_b1"]
    dw = DeviceWorkload(w, device=dev)
    st = dw.step
    H = w.n_heads
    k_c = torch.empty((st.num_pages, 64, H, 128), dtype=torch.bfloat16, device=dev)
    v_c = torch.empty_like(k_c)
    out = torch.empty(st.out.shape, dtype=st.out.dtype, device=dev)
    flush = torch.empty(int(256e6) // 4, dtype=torch.float32, device=dev)

    def level2():
        mla.mla_decompress_kv(st.cache, mla.MLA_BF16, st.num_pages, 64, dw.w_uk, dw.w_uv, H, k_c, v_c, st.err)
        mla.mla_attend_naive(dw.q_nope, dw.q_pe, st.cache, mla.MLA_BF16, k_c, v_c, st.num_pages, st.block_table,
                             st.max_pages, 64, st.seq_lens, w.batch, w.q_len, H, st.softmax_scale, out, None, st.err)

    def absorbed():
        st.absorb(dw.q_nope, dw.q_pe, dw.w_uk)
        st.attend()
        st.finish(dw.w_uv)

    res = {}
    for name, fn in (("level2", level2), ("absorbed", absorbed)):
        for _ in range(max(3, args.warmup)):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for e in ev:
            flush.fill_(1.0)
            e[0].record(stream)
            fn()
            e[1].record(stream)
        torch.cuda.synchronize()
        res[name] = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    assert int(st.err.item()) == 0, "device error flag set"
    kv_bytes = 2 * k_c.numel() * k_c.element_size()
    line = {"config": workload_config(w, dw.lens), "steps": args.steps,
            "level2_ms": res["level2"], "absorbed_ms": res["absorbed"],
            "absorbed_speedup": res["level2"] / res["absorbed"],
            "level2_kv_bytes": kv_bytes,
            "note": "per-head outputs of one decode step; level2 = mla_decompress_kv + mla_attend_naive, "
                    "absorbed = absorb_q + decode + combine + out_uv (one launch for the last two at this size); CUDA events, L2 flushed before each"}
    del dw, st, k_c, v_c, flush
    torch.cuda.empty_cache()
    return line


def time_extra(args, name, dev, stream):
    """The same step on a second workload in the same process (the e4m3
    two-token workload next to the long one): its decode launch against its
    binding roofline, which for that workload is the tensor pipe."""
    import torch
    from workloads.device import DeviceWorkload
    w = W.WORKLOADS[name]
    dw = DeviceWorkload(w, device=dev, q8=False if args.f16_operands else None)
    step = dw.step
    alg_bytes, alg_flops = algorithmic(w, dw.lens)
    flush = torch.empty(int(256e6) // 4, dtype=torch.float32, device=dev) if alg_bytes <= 256e6 else None

    # the step's five launches, recorded once as CUDA graphs (pre, attend,
    # post) and replayed: small steps are otherwise bound by host-side calls
    graphs = step.capture(dw.kv_new, dw.seq_ids, dw.positions, dw.q_nope, dw.q_pe, dw.w_uk, dw.w_uv)

    def one_step(ev=None):
        graphs.pre.replay()
        if ev is not None:
            ev[0].record(stream)
        graphs.attend.replay()
        if ev is not None:
            ev[1].record(stream)
        graphs.post.replay()

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    assert int(step.err.item()) == 0, "device error flag set"
    with ClockSampler(gpu_smi_id(dev.index or 0)) as clk:
        total_ms, dec = _timed_steps(torch, one_step, args.steps, stream, flush, lambda: None)
    pk = peaks()
    dec_ms = float(np.mean(dec))
    out = {"config": workload_config(w, dw.lens), "steps": args.steps,
           "value": w.batch * w.q_len * args.steps / (total_ms / 1e3), "unit": "tokens/s",
           "ms_per_step": total_ms / args.steps,
           "roofline": binding_roofline(alg_bytes, alg_flops, dec_ms, pk, recorded_traffic(name), mma_type(step)),
           "decode": _decode_summary(alg_bytes, alg_flops, dec_ms, total_ms / args.steps, pk, mma_type(step)),
           "clocks": clk.summary()}
    del graphs, dw, step
    torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long", choices=W.WORKLOAD_ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the e4m3 two-token line and the level-2 comparison (long workload only)")
    # smaller cases of a workload's shape, for profiler captures (not bench lines)
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch (profiling)")
    ap.add_argument("--seq-len", type=int, default=None, help="override the workload's fixed length (profiling)")
    ap.add_argument("--split-tokens", type=int, default=None, help="override the split length (profiling)")
    ap.add_argument("--f16-operands", action="store_true",
                    help="e4m3 cache: the widened f16-operand decode (mla_decode_fwd) instead of the 8-bit MMAs (profiling)")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    w = W.WORKLOADS[args.workload]
    over = {k: v for k, v in (("batch", args.batch), ("seq_len", args.seq_len),
                              ("split_tokens", args.split_tokens)) if v is not None}
    if over:
        w = W.with_overrides(w, name=w.name + "-profile-case", **over)
    if args.impl == "reference":
        return run_reference(args, w, rank, world)
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        return run_gpu(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
