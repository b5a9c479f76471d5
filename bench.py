"""Benchmark: mixed-head decode attention, one layer-step = KV append of the
new token + decode attention for every sequence and query head, on the
GQA 128K workload (Llama-3-8B attention shape: 32 query / 8 KV heads,
d=128, batch 8 with ragged lengths U[16K, 128K], 4 of 8 KV heads retrieval,
sink 64 + window 256, 32 distinct decode steps cycled).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Prints one JSON line (rank 0).  Multi-GPU: one process per GPU (torchrun),
each rank decodes its own 8 sequences of a global batch of 8N (weak scaling,
no collective on the data path); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import duo_workloads as W  # noqa: E402

METRIC = "mixed-head decode attn: µs/layer-step, achieved HBM GB/s (% of B200 peak)"
WORKLOAD = "gqa128k"
FALLBACK_HBM_GBS = 6650.0
# DRAM read + write bytes per launch of decode_tc_kernel<4> on this workload,
# from the ncu capture summarised in profiles/decode_tc_kernel_gqa128k.md.  Must be
# reset to None whenever the decode kernel changes.
DECODE_TRAFFIC_BYTES = 1123966208 + 3172096
# The same for decode_tc_kernel<4, FP8> on the FP8 cache of this workload
# (profiles/decode_tc_kernel_fp8_gqa128k.md); None once that kernel changes.
DECODE_FP8_TRAFFIC_BYTES = 562046464 + 5267968
# The same for the INT4 instantiation (profiles/decode_tc_kernel_int4_gqa128k.md).
DECODE_INT4_TRAFFIC_BYTES = 281096192 + 3445248
# Paged cache, the two slice launches of the sequence split, and the gated
# forward's full-attention launch (profiles/decode_tc_kernel_variants_gqa128k.md).
DECODE_PAGED_TRAFFIC_BYTES = 1120185344 + 2994432
DECODE_SEQSPLIT_TRAFFIC_BYTES = 838149120 + 3019264 + 291843840 + 142336
DECODE_GATED_TRAFFIC_BYTES = 2231668992 + 3008256
# decode_tc_kernel<1> on one copy of the MHA-32K cache, and decode_tc_kernel<4>
# on one layer of the million-token cache (profiles/decode_tc_kernel_mha32k_mtok.md).
MHA32K_DECODE_TRAFFIC_BYTES = 139653376 + 3044352
MTOK_DECODE_TRAFFIC_BYTES = 1085167360 + 3202048


# ---------------------------------------------------------------- helpers
def kv_bytes(lens_after, mask, d, S, Wn, cap):
    """Algorithmic KV bytes of one layer-step: full K and V rows of every
    retrieval head, the min(T, S+W) filled ring slots of every streaming head."""
    n_r = int(mask.sum())
    n_s = len(mask) - n_r
    tot = 0
    for T in lens_after:
        tot += n_r * 4 * d * min(int(T), cap) + n_s * 4 * d * min(int(T), S + Wn)
    return tot


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx or None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def max_over_ranks(x: float, world: int, dev) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_workload(rank: int, world: int):
    """Rank r decodes sequences 8r .. 8r+7 of a global batch of 8 * world."""
    base = W.WORKLOADS[WORKLOAD]
    g = W.scaled(base, batch=base.batch * world)
    lens = W.context_lengths(g)[rank * base.batch:(rank + 1) * base.batch]
    return base, g, lens


# ---------------------------------------------------------------- our arm
def fill_rank(cache, gw, lens0, first_b, dev, slab=16384):
    """Bulk-append the seeded history of this rank's sequences."""
    fill_targets([(cache, None)], gw, lens0, first_b, dev, slab)


def fill_targets(targets, gw, lens0, first_b, dev, slab=16384):
    """Bulk-append the seeded history into every (cache, rows) target; rows =
    None appends whole sequences, rows = (lo, hi) (int32 [B] on the device)
    keeps retrieval positions [lo, hi) (a slice of a sequence-split cache)."""
    B = len(lens0)
    top = int(lens0.max())
    for p0 in range(0, top, slab):
        n = min(slab, top - p0)
        k = torch.zeros(B, gw.n_kv, n, gw.d, dtype=torch.bfloat16)
        v = torch.zeros_like(k)
        cnt = np.clip(lens0 - p0, 0, n).astype(np.int32)
        for b in range(B):
            c = int(cnt[b])
            for g in range(gw.n_kv):
                if c:
                    k[b, g, :c] = W.tokens(gw, 0, first_b + b, g, W.TENSOR_K, p0, p0 + c)
                    v[b, g, :c] = W.tokens(gw, 0, first_b + b, g, W.TENSOR_V, p0, p0 + c)
        kd, vd = k.to(dev), v.to(dev)
        lb = torch.from_numpy(np.minimum(lens0, p0).astype(np.int32)).to(dev)
        cd = torch.from_numpy(cnt).to(dev)
        for cache, rows in targets:
            if rows is None:
                cache.append(0, kd, vd, lb, cd)
            else:
                cache.append_rows(0, kd, vd, lb, rows[0], rows[1], cd)


def step_inputs(gw, lens0, first_b, steps):
    """Per decode step s: q [B][Hq][d], k/v [B][n_kv][1][d] (CPU bf16)."""
    B = len(lens0)
    q = torch.empty(steps, B, gw.hq, gw.d, dtype=torch.bfloat16)
    k = torch.empty(steps, B, gw.n_kv, 1, gw.d, dtype=torch.bfloat16)
    v = torch.empty_like(k)
    for b in range(B):
        p = int(lens0[b])
        for h in range(gw.hq):
            q[:, b, h] = W.tokens(gw, 0, first_b + b, h, W.TENSOR_Q, p, p + steps)
        for g in range(gw.n_kv):
            k[:, b, g, 0] = W.tokens(gw, 0, first_b + b, g, W.TENSOR_K, p, p + steps)
            v[:, b, g, 0] = W.tokens(gw, 0, first_b + b, g, W.TENSOR_V, p, p + steps)
    return ([q[s].contiguous() for s in range(steps)], [k[s].contiguous() for s in range(steps)],
            [v[s].contiguous() for s in range(steps)])


def back_to_back_us(launch, n):
    """Mean duration (µs) of n launches issued back to back on the current
    stream, CUDA events only at the two ends of the run: the live duration of
    a kernel in a decode loop, where each programmatic launch overlaps its
    set-up with the previous launch's tail (events between launches would
    keep it from doing so and add a launch gap to every launch)."""
    stream = torch.cuda.current_stream()
    for i in range(3):
        launch(i)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(n):
        launch(i)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / n


B2B_TIMING = ("decode launches back to back over the cycled steps (no appends between), CUDA events at the "
              "two ends of the run")


def run_ours(args, rank, world, local):
    from head_wise_kv_b200 import DuoKVCache
    from head_wise_kv_b200 import _lib as L

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    base, gw, lens0 = rank_workload(rank, world)
    first_b = rank * base.batch
    mask = W.retrieval_mask(gw, 0)
    steps = base.steps
    cap = int(lens0.max()) + steps
    B = base.batch
    cache = DuoKVCache(1, B, base.hq, base.n_kv, base.d, base.sink, base.window, cap, mask[None], device=dev)
    fill_rank(cache, gw, lens0, first_b, dev)
    qs, ks, vs = step_inputs(gw, lens0, first_b, steps)
    dq = [q.to(dev) for q in qs]
    dk = [k.to(dev) for k in ks]
    dv = [v.to(dev) for v in vs]
    lb = [torch.from_numpy((lens0 + s).astype(np.int32)).to(dev) for s in range(steps)]
    la = [torch.from_numpy((lens0 + s + 1).astype(np.int32)).to(dev) for s in range(steps)]
    out = torch.empty(B, base.hq, base.d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    scale = base.scale

    def one(i):
        s = i % steps
        cache.step(0, dq[s], dk[s], dv[s], lb[s], la[s], scale, out=out)   # append + decode

    for i in range(args.warmup):
        one(i)
    torch.cuda.synchronize()
    assert cache.status() == 0, "device status set during warm-up"

    K = args.steps
    # The timed region: K layer-steps with events only at its two ends (an
    # event between the append and the decode would keep the decode's
    # programmatic launch from overlapping the append, which a real step has).
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        e_start.record(stream)
        for i in range(K):
            one(i)
        e_end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    total_ms = e_start.elapsed_time(e_end)
    assert cache.status() == 0, "device status set during the timed region"
    total_ms = max_over_ranks(total_ms, world, dev)
    us_per_step = total_ms * 1e3 / K

    # Launch durations for the roofline: the same steps again with events
    # around each launch (per-launch times, conservative: each includes its
    # launch gap, without the overlap with the append).
    KR = min(K, 1024)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(KR)]
    for i in range(KR):
        s = i % steps
        ev[i][0].record(stream)
        cache.append(0, dk[s], dv[s], lb[s])
        ev[i][1].record(stream)
        cache.decode(0, dq[s], la[s], scale, out=out)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    dec_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(KR)]
    app_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(KR)]
    each_ms = [ev[i][0].elapsed_time(ev[i][2]) for i in range(KR)]

    # algorithmic bytes of the decode launch, averaged over the steps timed
    bytes_steps = [kv_bytes(lens0 + (i % steps) + 1, mask, base.d, base.sink, base.window, cap) for i in range(KR)]
    avg_bytes = sum(bytes_steps) / KR
    dec_avg_ms = sum(dec_ms) / KR
    dec_b2b_us = back_to_back_us(lambda i: cache.decode(0, dq[i % steps], la[i % steps], scale, out=out), KR)
    hbm_peak, peak_kind = peaks()
    achieved = avg_bytes / (dec_b2b_us * 1e-6) / 1e9
    step_gbs = avg_bytes / (us_per_step * 1e-6) / 1e9

    # ---------------- e2e: host buffers in, host result out, copies timed.
    # A serving loop's shape: each step's inputs (q, k, v, lengths) packed in
    # one pinned host buffer and copied in with one H2D copy, the fp32 output
    # copied back to pinned host memory; the copies run on a second stream,
    # double-buffered, so step i+1's inputs and step i-1's output move while
    # step i computes.  Timed from the first copy in to the last copy out.
    def sec(nbytes):
        return (nbytes + 255) // 256 * 256
    n_q, n_k, n_l = dq[0].numel() * 2, dk[0].numel() * 2, lb[0].numel() * 4
    offs = np.cumsum([0, sec(n_q), sec(n_k), sec(n_k), sec(n_l), sec(n_l)])
    packed = []
    for s in range(steps):
        hbuf = torch.empty(int(offs[-1]), dtype=torch.uint8).pin_memory()
        for t, o in ((qs[s], offs[0]), (ks[s], offs[1]), (vs[s], offs[2])):
            nb = t.numel() * 2
            hbuf[o:o + nb].copy_(t.contiguous().view(torch.uint8).view(-1))
        for t, o in ((lb[s].cpu(), offs[3]), (la[s].cpu(), offs[4])):
            hbuf[o:o + n_l].copy_(t.view(torch.uint8).view(-1))
        packed.append(hbuf)
    dev_in = [torch.empty(int(offs[-1]), dtype=torch.uint8, device=dev) for _ in range(2)]
    outs2 = [torch.empty(B, base.hq, base.d, dtype=torch.float32, device=dev) for _ in range(2)]
    host_out = [torch.empty(B, base.hq, base.d, dtype=torch.float32).pin_memory() for _ in range(2)]
    views = []
    for buf in dev_in:
        views.append((buf[offs[0]:offs[0] + n_q].view(torch.bfloat16).view(dq[0].shape),
                      buf[offs[1]:offs[1] + n_k].view(torch.bfloat16).view(dk[0].shape),
                      buf[offs[2]:offs[2] + n_k].view(torch.bfloat16).view(dv[0].shape),
                      buf[offs[3]:offs[3] + n_l].view(torch.int32), buf[offs[4]:offs[4] + n_l].view(torch.int32)))
    cs = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def h2d(i):
        k = i % 2
        with torch.cuda.stream(cs):
            if i >= 2:
                cs.wait_event(ev_comp[k])              # step i-2 is done with this input set
            dev_in[k].copy_(packed[i % steps], non_blocking=True)
            ev_in[k].record(cs)

    def compute(i):
        k = i % 2
        stream.wait_event(ev_in[k])
        if i >= 2:
            stream.wait_event(ev_out[k])               # step i-2's output has been copied out
        q_, k_, v_, lb_, la_ = views[k]
        cache.step(0, q_, k_, v_, lb_, la_, scale, out=outs2[k])
        ev_comp[k].record(stream)

    def d2h(i):
        k = i % 2
        with torch.cuda.stream(cs):
            cs.wait_event(ev_comp[k])
            host_out[k].copy_(outs2[k], non_blocking=True)
            ev_out[k].record(cs)

    def run_e2e(n):
        h2d(0)
        for i in range(n):
            compute(i)
            if i + 1 < n:
                h2d(i + 1)
            d2h(i)

    run_e2e(args.warmup)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cs)
    run_e2e(K)
    e1.record(cs)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    # the pipelined loop computed what the device-side loop computes
    s_last = (K - 1) % steps
    ref_out = cache.decode(0, dq[s_last], la[s_last], scale)
    assert torch.equal(host_out[(K - 1) % 2], ref_out.cpu()), "e2e output differs from the device-side decode"
    h2d_bytes = int(offs[-1])
    d2h_bytes = host_out[0].numel() * 4

    res = {
        "metric": METRIC,
        "value": round(us_per_step, 3),
        "unit": "us/layer-step",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / K, 6),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": "gqa128k: GQA 32q/8kv d=128, B=8/GPU ragged T~U[16384,131072], 4/8 KV heads "
                        "retrieval, S=64 W=256, append+decode per layer-step (duo_decode_step), 32 distinct steps cycled",
            "global_batch": B * world,
            "seq_len": [int(x) for x in lens0],
            "kv_bytes_per_layer_step": int(avg_bytes),
            "l2": "not flushed: the KV read per step (~1.2 GB) is larger than L2 (126 MB)",
            "parallelism": f"replicas/dp{world} (independent sequences per GPU)",
        },
        "hbm_gbs_step": round(step_gbs * world, 1),
        "value_stats": {"timing": "value: mean over the timed region (events at its two ends); "
                                  "layer_step_us_each: each layer-step timed alone in a second pass",
                        "layer_step_us_each": _stats_us(each_ms)},
        "append_us": round(1e3 * sum(app_ms) / KR, 3),
        "decode_us": round(1e3 * dec_avg_ms, 3),
        "decode_us_median": round(1e3 * statistics.median(dec_ms), 3),
        "decode_us_timing": "CUDA events around each decode launch (after its append), 1024 steps after the "
                            "timed region: each includes a launch gap",
        "decode_us_back_to_back": round(dec_b2b_us, 3),
        "roofline": {
            "bound": "hbm",
            "kernel": "decode_tc_kernel (split-K tcgen05 attention with the log-sum-exp merge in-kernel)",
            "launch_timing": B2B_TIMING + f", {KR} launches",
            "achieved": round(achieved, 1),
            "peak": hbm_peak,
            "peak_kind": peak_kind,
            "unit": "GB/s",
            "frac": round(achieved / hbm_peak, 4),
            "traffic": DECODE_TRAFFIC_BYTES,
            "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum, one launch",
        },
        "e2e": {"value": round(e2e_ms * 1e3 / K, 3), "unit": "us/layer-step",
                "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
                "copies": "one packed H2D + one D2H per step on a second stream, double-buffered, "
                          "overlapping the neighbouring steps' compute"},
        "gpu_launches": 2 * K,          # append + decode per layer-step
        "clocks": clk.summary(),
    }
    cache.close()
    return res, (gw, lens0, mask, first_b)


# ---------------------------------------------------------------- FP8 decode
def run_variant_decode(local, kv_dtype="fp8", paged=False, steps=512, warmup=16):
    """The same layer-step (append of the new token + decode) on another
    cache of the same workload: FP8 E4M3 (scales 1.0: the N(0,1) data sits
    well inside E4M3's range; roofline at one byte per cached element), INT4
    (scales 0.5: about the largest |value| / 7 of the data; roofline at half a
    byte per element), or a paged cache (256-token pages handed out in a
    shuffled order)."""
    from head_wise_kv_b200 import DuoKVCache
    dev = torch.device("cuda", local)
    base, gw, lens0 = rank_workload(0, 1)
    mask = W.retrieval_mask(gw, 0)
    cap = int(lens0.max()) + base.steps
    B = base.batch
    page = 256
    per_seq = (cap + page - 1) // page
    sc = np.full((1, base.n_kv), 0.5, np.float32) if kv_dtype == "int4" else None
    cache = DuoKVCache(1, B, base.hq, base.n_kv, base.d, base.sink, base.window, cap, mask[None], device=dev,
                       kv_dtype=kv_dtype, k_scale=sc, v_scale=sc, page_tokens=page if paged else 0,
                       num_pages=B * per_seq if paged else 0)
    if paged:
        perm = np.random.default_rng(0).permutation(B * per_seq).astype(np.int32).reshape(B, per_seq)
        table = torch.from_numpy(perm).to(dev)
        cache.set_page_table(table)
    fill_rank(cache, gw, lens0, 0, dev)
    qs, ks, vs = step_inputs(gw, lens0, 0, base.steps)
    dq = [q.to(dev) for q in qs]
    dk = [k.to(dev) for k in ks]
    dv = [v.to(dev) for v in vs]
    lb = [torch.from_numpy((lens0 + s).astype(np.int32)).to(dev) for s in range(base.steps)]
    la = [torch.from_numpy((lens0 + s + 1).astype(np.int32)).to(dev) for s in range(base.steps)]
    out = torch.empty(B, base.hq, base.d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for i in range(warmup):
        s = i % base.steps
        cache.step(0, dq[s], dk[s], dv[s], lb[s], la[s], base.scale, out=out)
    torch.cuda.synchronize()
    assert cache.status() == 0, "device status set during the warm-up"
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):                   # layer-steps, events only at the ends
        s = i % base.steps
        cache.step(0, dq[s], dk[s], dv[s], lb[s], la[s], base.scale, out=out)
    e1.record(stream)
    torch.cuda.synchronize()
    step_ms = e0.elapsed_time(e1) / steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):                   # per-launch decode times for the roofline
        s = i % base.steps
        cache.append(0, dk[s], dv[s], lb[s])
        ev[i][0].record(stream)
        cache.decode(0, dq[s], la[s], base.scale, out=out)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    assert cache.status() == 0, "device status set during the timed region"
    dec_ms = sum(ev[i][0].elapsed_time(ev[i][1]) for i in range(steps)) / steps
    b2b_us = back_to_back_us(lambda i: cache.decode(0, dq[i % base.steps], la[i % base.steps], base.scale, out=out),
                             steps)
    elem = {"fp8": 1, "int4": 0.5, "bf16": 2}[kv_dtype]
    nbytes = sum(kv_bytes(lens0 + (i % base.steps) + 1, mask, base.d, base.sink, base.window, cap)
                 for i in range(steps)) / steps * elem / 2
    hbm_peak, peak_kind = peaks()
    achieved = nbytes / (b2b_us * 1e-6) / 1e9
    cache.close()
    what = {"fp8": "an FP8 E4M3 cache (retrieval and streaming heads)",
            "int4": "an INT4 cache (retrieval and streaming heads, scales 0.5)", "bf16": "a bf16 cache"}[kv_dtype] + \
        (", retrieval heads paged (256-token pages, shuffled)" if paged else "")
    return {
        "workload": f"gqa128k with {what}, append + decode per layer-step, 32 distinct steps cycled",
        "steps": steps, "warmup": warmup,
        "layer_step_us": round(step_ms * 1e3, 3),
        "decode_us": round(dec_ms * 1e3, 3),
        "decode_us_timing": "CUDA events around each decode launch (after its append): each includes a launch gap",
        "decode_us_back_to_back": round(b2b_us, 3),
        "kv_bytes_per_layer_step": int(nbytes),
        "roofline": {"bound": "hbm", "kernel": f"decode_tc_kernel {kv_dtype}{' paged' if paged else ''}",
                     "launch_timing": B2B_TIMING + f", {steps} launches",
                     "achieved": round(achieved, 1), "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4),
                     "traffic": DECODE_PAGED_TRAFFIC_BYTES if paged and kv_dtype == "bf16" else
                     None if paged else {"fp8": DECODE_FP8_TRAFFIC_BYTES, "int4": DECODE_INT4_TRAFFIC_BYTES}.get(kv_dtype),
                     "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum, one launch"},
        "gpu_launches": 2 * steps,
    }


def _step_tensors(gw, base, lens0, dev):
    qs, ks, vs = step_inputs(gw, lens0, 0, base.steps)
    dq = [q.to(dev) for q in qs]
    dk = [k.to(dev) for k in ks]
    dv = [v.to(dev) for v in vs]
    lb = [torch.from_numpy((lens0 + s).astype(np.int32)).to(dev) for s in range(base.steps)]
    la = [torch.from_numpy((lens0 + s + 1).astype(np.int32)).to(dev) for s in range(base.steps)]
    return dq, dk, dv, lb, la


def run_seqsplit(local, R=2, steps=256, warmup=16):
    """Sequence-split decode (f4): every sequence's retrieval positions cut
    into R contiguous slices, as R GPUs would hold them.  Here the R slices
    are R independent caches on one GPU, run one after another (none waits on
    another).  Per layer-step: each slice appends the new token
    (append_rows), decodes its rows (decode_rows; the last slice also the
    streaming heads), and lse_merge combines the R partial (out, lse) -- the
    exchange between GPUs (an all-gather of 16.5 KB per sequence and layer)
    is the one step not run here."""
    from head_wise_kv_b200 import DuoKVCache, seqsplit
    from head_wise_kv_b200.cache import lse_merge
    dev = torch.device("cuda", local)
    base, gw, lens0 = rank_workload(0, 1)
    mask = W.retrieval_mask(gw, 0)
    B = base.batch
    total = int(lens0.max()) + base.steps
    cap = (total + R - 1) // R
    caches = [DuoKVCache(1, B, base.hq, base.n_kv, base.d, base.sink, base.window, cap, mask[None], device=dev)
              for _ in range(R)]
    bounds = []
    for r in range(R):
        lo, hi = seqsplit.slice_bounds(cap, r)
        bounds.append((torch.full((B,), lo, dtype=torch.int32, device=dev),
                       torch.full((B,), hi, dtype=torch.int32, device=dev)))
    fill_targets(list(zip(caches, bounds)), gw, lens0, 0, dev)
    dq, dk, dv, lb, la = _step_tensors(gw, base, lens0, dev)
    rows = [[seqsplit.local_rows(la[s], cap, r) for s in range(base.steps)] for r in range(R)]
    zero = torch.zeros(B, dtype=torch.int32, device=dev)
    po = torch.empty(R, B, base.hq, base.d, dtype=torch.float32, device=dev)
    pl = torch.empty(R, B, base.hq, dtype=torch.float32, device=dev)
    out = torch.empty(B, base.hq, base.d, dtype=torch.float32, device=dev)
    lse = torch.empty(B, base.hq, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i, ev=None):
        s = i % base.steps
        for r, c in enumerate(caches):
            c.append_rows(0, dk[s], dv[s], lb[s], bounds[r][0], bounds[r][1])
        for r, c in enumerate(caches):
            if ev is not None:
                ev[r][0].record(stream)
            c.decode_rows(0, dq[s], rows[r][s], base.scale, s_len=la[s] if r == R - 1 else zero, out=po[r],
                          lse=pl[r])
            if ev is not None:
                ev[r][1].record(stream)
        lse_merge(po, pl, out=out, lse=lse)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    assert all(c.status() == 0 for c in caches), "device status set during the warm-up"
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    step_ms = e0.elapsed_time(e1) / steps
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(R)]
           for _ in range(steps)]
    for i in range(steps):
        step(i, evs[i])
    torch.cuda.synchronize()
    assert all(c.status() == 0 for c in caches), "device status set during the timed region"
    slice_ms = [sum(evs[i][r][0].elapsed_time(evs[i][r][1]) for i in range(steps)) / steps for r in range(R)]
    nbytes = sum(kv_bytes(lens0 + (i % base.steps) + 1, mask, base.d, base.sink, base.window, total)
                 for i in range(steps)) / steps
    hbm_peak, peak_kind = peaks()
    achieved = nbytes / (sum(slice_ms) * 1e-3) / 1e9
    for c in caches:
        c.close()
    return {
        "workload": f"gqa128k, every sequence's retrieval positions split into {R} slices of {cap} rows "
                    f"(R caches on one GPU, run one after another), append_rows + decode_rows per slice + "
                    f"lse_merge per layer-step, 32 distinct steps cycled",
        "steps": steps, "warmup": warmup,
        "layer_step_us": round(step_ms * 1e3, 3),
        "slice_decode_us": [round(x * 1e3, 3) for x in slice_ms],
        "kv_bytes_per_layer_step": int(nbytes),
        "roofline": {"bound": "hbm", "kernel": "decode_tc_kernel over row ranges (all slices)",
                     "achieved": round(achieved, 1), "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4),
                     "traffic": DECODE_SEQSPLIT_TRAFFIC_BYTES if R == 2 else None,
                     "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum, both slice launches"},
        "gpu_launches": (2 * R + 1) * steps,
    }


def run_gated(local, steps=256, warmup=16):
    """Gated (alpha-blended) decode (f3) on the gqa128k shape with every KV
    head keeping its whole history (the setting of the identification pass):
    per layer-step the append, full attention for every head, streaming
    attention as two row ranges (the sinks and the recent window) merged by
    log-sum-exp, and out = alpha_h full + (1 - alpha_h) streaming per query
    head (alpha seeded uniform in [0, 1))."""
    from head_wise_kv_b200 import DuoKVCache
    from head_wise_kv_b200.cache import alpha_blend, lse_merge
    dev = torch.device("cuda", local)
    base, gw, lens0 = rank_workload(0, 1)
    B, S, Wn = base.batch, base.sink, base.window
    full_mask = np.ones(base.n_kv, np.uint8)
    cap = int(lens0.max()) + base.steps
    cache = DuoKVCache(1, B, base.hq, base.n_kv, base.d, S, Wn, cap, full_mask[None], device=dev)
    fill_rank(cache, gw, lens0, 0, dev)
    dq, dk, dv, lb, la = _step_tensors(gw, base, lens0, dev)
    sink_end = [torch.clamp(x, max=S) for x in la]
    win_begin = [torch.clamp(x - Wn, min=S) for x in la]
    alpha = torch.from_numpy(np.random.default_rng(3).uniform(0, 1, base.hq).astype(np.float32)).to(dev)
    full = torch.empty(B, base.hq, base.d, dtype=torch.float32, device=dev)
    po = torch.empty(2, B, base.hq, base.d, dtype=torch.float32, device=dev)
    pl = torch.empty(2, B, base.hq, dtype=torch.float32, device=dev)
    strm = torch.empty(B, base.hq, base.d, dtype=torch.float32, device=dev)
    slse = torch.empty(B, base.hq, dtype=torch.float32, device=dev)
    out = torch.empty_like(full)
    stream = torch.cuda.current_stream(dev)

    def step(i, ev=None):
        s = i % base.steps
        cache.append(0, dk[s], dv[s], lb[s])
        if ev is not None:
            ev[0].record(stream)
        cache.decode(0, dq[s], la[s], base.scale, out=full)
        if ev is not None:
            ev[1].record(stream)
        cache.decode_rows(0, dq[s], sink_end[s], base.scale, out=po[0], lse=pl[0])
        cache.decode_rows(0, dq[s], la[s], base.scale, r_begin=win_begin[s], out=po[1], lse=pl[1])
        lse_merge(po, pl, out=strm, lse=slse)
        alpha_blend(alpha, full, strm, out=out)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    assert cache.status() == 0, "device status set during the warm-up"
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    step_ms = e0.elapsed_time(e1) / steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        step(i, evs[i])
    torch.cuda.synchronize()
    assert cache.status() == 0, "device status set during the timed region"
    full_ms = sum(evs[i][0].elapsed_time(evs[i][1]) for i in range(steps)) / steps
    n_kv, row = base.n_kv, 4 * base.d
    fb = sb = 0
    for i in range(steps):
        for T in lens0 + (i % base.steps) + 1:
            T = int(T)
            fb += n_kv * row * T
            sb += n_kv * row * (min(T, S) + max(0, T - max(T - Wn, S)))
    fb, sb = fb / steps, sb / steps
    hbm_peak, peak_kind = peaks()
    achieved = fb / (full_ms * 1e-3) / 1e9
    cache.close()
    return {
        "workload": "gqa128k shape, all 8 KV heads keep their whole history; append + full decode + streaming "
                    "decode (sink rows and window rows, lse-merged) + per-head alpha blend per layer-step, "
                    "32 distinct steps cycled",
        "steps": steps, "warmup": warmup,
        "layer_step_us": round(step_ms * 1e3, 3),
        "full_decode_us": round(full_ms * 1e3, 3),
        "kv_bytes_per_layer_step": {"full": int(fb), "streaming": int(sb)},
        "roofline": {"bound": "hbm", "kernel": "decode_tc_kernel (full attention of every head)",
                     "achieved": round(achieved, 1), "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4), "traffic": DECODE_GATED_TRAFFIC_BYTES,
                     "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum, one launch"},
        "gpu_launches": 6 * steps,
    }


# ---------------------------------------------------------------- the other decode workloads
def _l2_flush_buffer(dev):
    """A buffer twice the device's L2: writing it evicts whatever a step left
    in L2."""
    l2 = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0) or (126 << 20))
    return torch.empty(2 * l2, dtype=torch.uint8, device=dev)


def _stats_us(ms):
    return {"median": round(statistics.median(ms) * 1e3, 3), "mean": round(sum(ms) / len(ms) * 1e3, 3)}


def run_tiny(local, steps=512, warmup=16):
    """Tiny workload (1 layer, MHA 4 heads, d=64, B=1, T0=512, 16 decode
    steps cycled, heads {0,2} retrieval, S=16, W=64): the latency floor of a
    layer-step.  L2 is flushed before every step (a write of twice its size),
    and each step is timed on its own with CUDA events; median reported."""
    from head_wise_kv_b200 import DuoKVCache
    dev = torch.device("cuda", local)
    w = W.WORKLOADS["tiny"]
    mask = W.retrieval_mask(w, 0)
    lens0 = W.context_lengths(w)
    cap = int(lens0.max()) + w.steps
    cache = DuoKVCache(1, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap, mask[None], device=dev)
    fill_rank(cache, w, lens0, 0, dev)
    dq, dk, dv, lb, la = _step_tensors(w, w, lens0, dev)
    out = torch.empty(w.batch, w.hq, w.d, dtype=torch.float32, device=dev)
    flush = _l2_flush_buffer(dev)
    stream = torch.cuda.current_stream(dev)
    n = warmup + steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i in range(n):
        s = i % w.steps
        flush.zero_()
        ev[i][0].record(stream)
        cache.step(0, dq[s], dk[s], dv[s], lb[s], la[s], w.scale, out=out)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    assert cache.status() == 0, "device status set during the tiny benchmark"
    ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(warmup, n)]
    nbytes = sum(kv_bytes(lens0 + (i % w.steps) + 1, mask, w.d, w.sink, w.window, cap) for i in range(steps)) / steps
    med = statistics.median(ms)
    hbm_peak, peak_kind = peaks()
    achieved = nbytes / (med * 1e-3) / 1e9
    cache.close()
    return {
        "workload": "tiny: 1 layer, MHA 4 heads, d=64, B=1, T0=512, 16 decode steps cycled, heads {0,2} "
                    "retrieval, S=16, W=64, K and q RoPE'd",
        "steps": steps, "warmup": warmup,
        "layer_step_us": _stats_us(ms),
        "kv_bytes_per_layer_step": int(nbytes),
        "l2": "flushed before every step (write of 2x L2); each step timed alone with CUDA events",
        "roofline": {"bound": "latency", "kernel": "append_kernel + decode_kernel + merge_kernel (d=64)",
                     "achieved": round(achieved, 1), "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 6), "traffic": None,
                     "note": "0.3 MB per step: three launches' latency, not bandwidth, sets the time"},
        "gpu_launches": 3 * steps,
    }


def run_mha32k(local, steps=1024, warmup=32, copies=4):
    """MHA-32K workload (Llama-2-7B attention: 32 = 32 heads, d=128, B=1,
    T0=32768, 64 decode steps with append/evict, 8 retrieval heads, S=64,
    W=256, key rows 0..3 x4).  One step reads ~138 MB, about L2's size, so
    `copies` caches with the same history are used in rotation (step i on
    copy i mod copies): between two uses of a copy the other copies stream
    ~3x L2, so every step reads its keys from HBM."""
    from head_wise_kv_b200 import DuoKVCache
    dev = torch.device("cuda", local)
    w = W.WORKLOADS["mha32k"]
    mask = W.retrieval_mask(w, 0)
    lens0 = W.context_lengths(w)
    cap = int(lens0.max()) + w.steps
    caches = [DuoKVCache(1, w.batch, w.hq, w.n_kv, w.d, w.sink, w.window, cap, mask[None], device=dev)
              for _ in range(copies)]
    fill_targets([(c, None) for c in caches], w, lens0, 0, dev)
    dq, dk, dv, lb, la = _step_tensors(w, w, lens0, dev)
    out = torch.empty(w.batch, w.hq, w.d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def which(i):
        return caches[i % copies], (i // copies) % w.steps

    for i in range(warmup):
        c, s = which(i)
        c.step(0, dq[s], dk[s], dv[s], lb[s], la[s], w.scale, out=out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):                   # events only at the ends
        c, s = which(i)
        c.step(0, dq[s], dk[s], dv[s], lb[s], la[s], w.scale, out=out)
    e1.record(stream)
    torch.cuda.synchronize()
    step_ms = e0.elapsed_time(e1) / steps
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(steps)]
    for i in range(steps):                   # per-step and per-launch times
        c, s = which(i)
        ev[i][0].record(stream)
        c.append(0, dk[s], dv[s], lb[s])
        ev[i][1].record(stream)
        c.decode(0, dq[s], la[s], w.scale, out=out)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    assert all(c.status() == 0 for c in caches), "device status set during the MHA-32K benchmark"
    step_each = [ev[i][0].elapsed_time(ev[i][2]) for i in range(steps)]
    dec_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(steps)]
    nbytes = sum(kv_bytes(lens0 + ((i // copies) % w.steps) + 1, mask, w.d, w.sink, w.window, cap)
                 for i in range(steps)) / steps
    hbm_peak, peak_kind = peaks()

    def dec_only(i):
        c, s = which(i)
        c.decode(0, dq[s], la[s], w.scale, out=out)
    b2b_us = back_to_back_us(dec_only, steps)
    achieved = nbytes / (b2b_us * 1e-6) / 1e9
    for c in caches:
        c.close()
    return {
        "workload": "mha32k: Llama-2-7B attention, MHA 32 heads, d=128, B=1, T0=32768, 8 retrieval heads, "
                    "S=64, W=256, key rows 0-3 x4, append + decode per layer-step, 64 distinct steps cycled",
        "steps": steps, "warmup": warmup,
        "layer_step_us": round(step_ms * 1e3, 3),
        "layer_step_us_each": _stats_us(step_each),
        "decode_us": _stats_us(dec_ms),
        "decode_us_timing": "CUDA events around each decode launch (after its append): each includes a launch gap",
        "decode_us_back_to_back": round(b2b_us, 3),
        "kv_bytes_per_layer_step": int(nbytes),
        "hbm_gbs_step": round(nbytes / (step_ms * 1e-3) / 1e9, 1),
        "l2": f"{copies} cache copies in rotation ({copies} x {nbytes / 1e6:.0f} MB > 3x L2): every step "
              f"reads its keys from HBM",
        "roofline": {"bound": "hbm", "kernel": "decode_tc_kernel (G=1)",
                     "launch_timing": B2B_TIMING + f", copies in rotation, {steps} launches",
                     "achieved": round(achieved, 1),
                     "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                     "traffic": MHA32K_DECODE_TRAFFIC_BYTES,
                     "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum, one launch"},
        "gpu_launches": 2 * steps,
    }


def run_mtok(local, steps=10, warmup=3, slab=65536, layers=None):
    """Million-token workload: 32 layers of GQA 32q/8kv, d=128, B=1,
    T=1,048,576, 2 of 8 KV heads retrieval per layer, S=64, W=1024.  The
    caches are filled by bulk appends of N(0,1) bf16 keys and values drawn
    on the device (a seeded torch generator; 34 GB of history, which host
    draws would take minutes to produce; the timing does not depend on the
    values).  One step = append + decode in each of the 32 layers in turn;
    the steps re-append position T (the same bytes)."""
    from head_wise_kv_b200 import DuoKVCache
    dev = torch.device("cuda", local)
    w = W.WORKLOADS["mtok"]
    if layers is not None:        # profiling: the first `layers` layers (the same launch per layer)
        w = W.scaled(w, layers=layers)
    masks = W.retrieval_masks(w)
    T0 = w.t0
    cache = DuoKVCache(w.layers, 1, w.hq, w.n_kv, w.d, w.sink, w.window, T0 + 1, masks, device=dev)
    gen = torch.Generator(device=dev).manual_seed(W.WORKLOADS["mtok"].seed)
    for layer in range(w.layers):
        for p0 in range(0, T0, slab):
            n = min(slab, T0 - p0)
            k = torch.randn(1, w.n_kv, n, w.d, generator=gen, device=dev).to(torch.bfloat16)
            v = torch.randn(1, w.n_kv, n, w.d, generator=gen, device=dev).to(torch.bfloat16)
            cache.append(layer, k, v, torch.tensor([p0], dtype=torch.int32, device=dev))
            del k, v
    torch.cuda.synchronize()
    assert cache.status() == 0, "device status set while filling the million-token cache"
    qs = [torch.randn(1, w.hq, w.d, generator=gen, device=dev).to(torch.bfloat16) for _ in range(w.layers)]
    ks = [torch.randn(1, w.n_kv, 1, w.d, generator=gen, device=dev).to(torch.bfloat16) for _ in range(w.layers)]
    vs = [torch.randn(1, w.n_kv, 1, w.d, generator=gen, device=dev).to(torch.bfloat16) for _ in range(w.layers)]
    lb = torch.tensor([T0], dtype=torch.int32, device=dev)
    la = torch.tensor([T0 + 1], dtype=torch.int32, device=dev)
    out = torch.empty(1, w.hq, w.d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        for layer in range(w.layers):
            if ev is None:
                cache.step(layer, qs[layer], ks[layer], vs[layer], lb, la, w.scale, out=out)
                continue
            cache.append(layer, ks[layer], vs[layer], lb)      # per-launch times: the two calls apart
            ev[layer][0].record(stream)
            cache.decode(layer, qs[layer], la, w.scale, out=out)
            ev[layer][1].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    step_ms = e0.elapsed_time(e1) / steps
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(w.layers)]
           for _ in range(steps)]
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize()
    assert cache.status() == 0, "device status set during the million-token benchmark"
    dec_ms = [evs[i][l][0].elapsed_time(evs[i][l][1]) for i in range(steps) for l in range(w.layers)]
    layer_bytes = [kv_bytes([T0 + 1], masks[l], w.d, w.sink, w.window, T0 + 1) for l in range(w.layers)]
    step_bytes = sum(layer_bytes)
    hbm_peak, peak_kind = peaks()
    b2b_us = back_to_back_us(lambda i: cache.decode(i % w.layers, qs[i % w.layers], la, w.scale, out=out),
                             w.layers * steps)
    achieved = (step_bytes / w.layers) / (b2b_us * 1e-6) / 1e9
    cache.close()
    return {
        "workload": f"mtok: {w.layers} layers GQA 32q/8kv, d=128, B=1, T=1048576, 2/8 KV heads retrieval per "
                    f"layer, S=64, W=1024; one step = append + decode in each layer in turn",
        "steps": steps, "warmup": warmup,
        "ms_per_step": round(step_ms, 4),
        "layer_step_us": round(step_ms * 1e3 / w.layers, 3),
        "decode_us": _stats_us(dec_ms),
        "decode_us_timing": "CUDA events around each decode launch (after its append): each includes a launch gap",
        "decode_us_back_to_back": round(b2b_us, 3),
        "kv_bytes_per_step": int(step_bytes),
        "hbm_gbs_step": round(step_bytes / (step_ms * 1e-3) / 1e9, 1),
        "l2": "not flushed: each layer reads ~1.08 GB (> L2)",
        "roofline": {"bound": "hbm", "kernel": "decode_tc_kernel (G=4), one launch per layer",
                     "launch_timing": B2B_TIMING + f", layers in turn, {w.layers * steps} launches",
                     "achieved": round(achieved, 1), "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4), "traffic": MTOK_DECODE_TRAFFIC_BYTES,
                     "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum, one launch (one layer)"},
        "gpu_launches": 2 * w.layers * steps,
    }


# ---------------------------------------------------------------- chunked prefill
def prefill_pairs(prompt, chunk, n_r_q, n_s_q, S, Wn):
    """Mask-valid (query, key) pairs of a chunked prefill: retrieval query heads
    see every key j <= t, streaming query heads min(t+1, S+W) keys."""
    pairs = 0
    for P in range(0, prompt, chunk):
        C = min(chunk, prompt - P)
        pairs += n_r_q * (P * C + C * (C + 1) // 2)
        t = np.arange(P, P + C, dtype=np.int64)
        pairs += n_s_q * int(np.minimum(t + 1, S + Wn).sum())
    return pairs


def bf16_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["bf16_tflops"]), float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), "measured"
    return 1590.0, 1400.0, "fallback"


def run_prefill(local, reps=3):
    """The 64K-token prompt in 16 chunks of 4096, attention then append per
    chunk (one layer, GQA 32q/8kv, 4 retrieval KV heads, S=64, W=1024)."""
    from head_wise_kv_b200 import DuoKVCache

    dev = torch.device("cuda", local)
    w = W.WORKLOADS["prefill64k"]
    mask = W.retrieval_mask(w, 0)
    G = w.hq // w.n_kv
    C, n_chunks = w.chunk, w.prompt // w.chunk
    cache = DuoKVCache(1, 1, w.hq, w.n_kv, w.d, w.sink, w.window, w.prompt, mask[None], device=dev)
    q = torch.empty(w.hq, w.prompt, w.d, dtype=torch.bfloat16)
    k = torch.empty(w.n_kv, w.prompt, w.d, dtype=torch.bfloat16)
    v = torch.empty_like(k)
    for h in range(w.hq):
        q[h] = W.tokens(w, 0, 0, h, W.TENSOR_Q, 0, w.prompt)
    for g in range(w.n_kv):
        k[g] = W.tokens(w, 0, 0, g, W.TENSOR_K, 0, w.prompt)
        v[g] = W.tokens(w, 0, 0, g, W.TENSOR_V, 0, w.prompt)
    dq = [q[:, c * C:(c + 1) * C].contiguous()[None].to(dev) for c in range(n_chunks)]
    dk = [k[:, c * C:(c + 1) * C].contiguous()[None].to(dev) for c in range(n_chunks)]
    dv = [v[:, c * C:(c + 1) * C].contiguous()[None].to(dev) for c in range(n_chunks)]
    pre = [torch.tensor([c * C], dtype=torch.int32, device=dev) for c in range(n_chunks)]
    out = torch.empty(1, w.hq, C, w.d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * n_chunks + 1)] for _ in range(reps + 1)]
    for r in range(reps + 1):     # repetition 0 is the warm-up
        e = ev[r]
        e[0].record(stream)
        for c in range(n_chunks):
            cache.prefill(0, dq[c], dk[c], dv[c], pre[c], w.scale, out=out)
            e[2 * c + 1].record(stream)
            cache.append(0, dk[c], dv[c], pre[c])
            e[2 * c + 2].record(stream)
    torch.cuda.synchronize()
    assert cache.status() == 0, "device status set during the prefill benchmark"
    attn_ms, total_ms = [], []
    for r in range(1, reps + 1):
        e = ev[r]
        attn_ms.append(sum(e[2 * c].elapsed_time(e[2 * c + 1]) for c in range(n_chunks)))
        total_ms.append(e[0].elapsed_time(e[-1]))
    n_r_q = int(mask.sum()) * G
    pairs = prefill_pairs(w.prompt, C, n_r_q, w.hq - n_r_q, w.sink, w.window)
    flops = 4 * w.d * pairs
    a_ms = statistics.median(attn_ms)
    tflops = flops / (a_ms * 1e-3) / 1e12
    burst, sustained, kind = bf16_peaks()
    cache.close()
    return {
        "workload": "prefill64k: 65536-token prompt in 16 chunks of 4096, GQA 32q/8kv d=128, 4/8 KV heads "
                    "retrieval (causal), 4 streaming (sink 64 + window 1024)",
        "attn_ms": round(a_ms, 3),
        "total_ms_with_append": round(statistics.median(total_ms), 3),
        "useful_flops": int(flops),
        "useful_tflops": round(tflops, 1),
        "roofline": {"bound": "tensor", "kernel": "prefill_kernel (tcgen05)", "achieved": round(tflops, 1),
                     "peak": sustained, "peak_kind": f"{kind} sustained bf16", "unit": "TFLOP/s",
                     "frac": round(tflops / sustained, 4), "frac_of_burst": round(tflops / burst, 4),
                     "traffic": None},
        "gpu_launches": 4 * n_chunks * reps,   # per chunk: V conversion, attention, split merge, append
    }


# ---------------------------------------------------------------- oracle timing
def oracle_step_sample(gw, lens0, mask, first_b, seqs, min_seconds=10.0, max_reps=16):
    """Time the fp64 oracle on one full layer-step of the given sequences
    (every query head), repeated until about `min_seconds` of CPU time;
    returns (seconds per layer-step, KV bytes covered, repetitions)."""
    from oracle import duo_oracle as O
    base = W.WORKLOADS[WORKLOAD]
    hists = []
    nbytes = 0
    for b in seqs:
        T = int(lens0[b]) + 1
        hist_k = {g: W.tokens(gw, 0, first_b + b, g, W.TENSOR_K, 0, T).float().numpy() for g in range(gw.n_kv)}
        hist_v = {g: W.tokens(gw, 0, first_b + b, g, W.TENSOR_V, 0, T).float().numpy() for g in range(gw.n_kv)}
        q = torch.stack([W.tokens(gw, 0, first_b + b, h, W.TENSOR_Q, T - 1, T)[0] for h in range(gw.hq)])
        hists.append((T, hist_k, hist_v, q[None].double().numpy()))
        nbytes += kv_bytes([T], mask, base.d, base.sink, base.window, 1 << 40)
    reps, secs = 0, 0.0
    while reps < max_reps and (reps == 0 or secs < min_seconds):
        t0 = time.perf_counter()
        for T, hk, hv, q in hists:
            O.decode_attention(q, lambda _b, g, hk=hk: hk[g], lambda _b, g, hv=hv: hv[g], [T], mask, gw.sink,
                               gw.window, gw.scale)
        secs += time.perf_counter() - t0
        reps += 1
    return secs / reps, nbytes, reps


def cpu_baseline(ctx):
    gw, lens0, mask, first_b = ctx
    cores = len(os.sched_getaffinity(0))
    secs, nbytes, reps = oracle_step_sample(gw, lens0, mask, first_b, range(len(lens0)))
    total = kv_bytes(lens0 + 1, mask, gw.d, gw.sink, gw.window, 1 << 40)
    return {"value": round(secs * 1e6 * total / nbytes, 1), "unit": "us/layer-step", "cores": cores,
            "kind": "oracle",
            "sample": f"numpy fp64 oracle on one full layer-step (all {len(lens0)} sequences, all 32 query "
                      f"heads, first decode step), mean of {reps} repetitions, {secs:.2f} s each"}


def cpu_baseline_prefill(sample_rows=256, chunks=(15, 7)):
    """The fp64 oracle's chunked prefill on a bounded sample of the 64K
    prompt: the first `sample_rows` query rows of the given chunks, every
    query head, timed; its useful FLOP rate scales it to the whole prompt."""
    from oracle import duo_oracle as O
    w = W.WORKLOADS["prefill64k"]
    mask = W.retrieval_mask(w, 0)
    G = w.hq // w.n_kv
    C = w.chunk
    top = (max(chunks) + 1) * C
    K = {g: W.tokens(w, 0, 0, g, W.TENSOR_K, 0, top).float().numpy() for g in range(w.n_kv)}
    V = {g: W.tokens(w, 0, 0, g, W.TENSOR_V, 0, top).float().numpy() for g in range(w.n_kv)}
    rows = np.arange(sample_rows)
    secs, pairs = 0.0, 0
    for c in chunks:
        P = c * C
        q = torch.stack([W.tokens(w, 0, 0, h, W.TENSOR_Q, P, P + C) for h in range(w.hq)])[None]
        q = q.double().numpy()
        t0 = time.perf_counter()
        O.prefill_attention(q, lambda _b, g: K[g], lambda _b, g: V[g], np.array([P]), mask, w.sink, w.window,
                            w.scale, rows=rows)
        secs += time.perf_counter() - t0
        t = P + rows
        n_r_q = int(mask.sum()) * G
        pairs += n_r_q * int((t + 1).sum()) + (w.hq - n_r_q) * int(np.minimum(t + 1, w.sink + w.window).sum())
    rate = 4 * w.d * pairs / secs                  # useful FLOP/s
    n_r_q = int(mask.sum()) * G
    total = 4 * w.d * prefill_pairs(w.prompt, C, n_r_q, w.hq - n_r_q, w.sink, w.window)
    return {"value": round(total / rate * 1e3, 1), "unit": "ms per 64K-token prompt (attention)",
            "useful_tflops": round(rate / 1e12, 4), "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"numpy fp64 oracle prefill of query rows 0..{sample_rows - 1} of chunks "
                      f"{list(chunks)} (P = {[c * C for c in chunks]}), all 32 query heads, {secs:.2f} s; "
                      f"scaled to the whole prompt by useful FLOPs"}


def cpu_baseline_mtok(min_seconds=10.0, max_layers=4):
    """The fp64 oracle's decode of whole layers of the million-token step
    (layers 0, 1, ... until about `min_seconds` of CPU time): seconds per
    layer measured, per 32-layer step = 32 x that."""
    from oracle import duo_oracle as O
    w = W.WORKLOADS["mtok"]
    T = w.t0 + 1
    secs, layers = 0.0, 0
    while layers < max_layers and (layers == 0 or secs < min_seconds):
        mask = W.retrieval_mask(w, layers)
        keep = O.keep_set(T - 1, w.sink, w.window)
        hk, hv = {}, {}
        for g in range(w.n_kv):
            if mask[g]:
                hk[g] = W.tokens(w, layers, 0, g, W.TENSOR_K, 0, T).float().numpy()
                hv[g] = W.tokens(w, layers, 0, g, W.TENSOR_V, 0, T).float().numpy()
            else:   # a streaming head's history is read only at its kept positions
                hk[g] = np.zeros((T, w.d), np.float32)
                hv[g] = np.zeros((T, w.d), np.float32)
                for a, e in [(0, w.sink), (T - w.window, T)]:
                    hk[g][a:e] = W.tokens(w, layers, 0, g, W.TENSOR_K, a, e).float().numpy()
                    hv[g][a:e] = W.tokens(w, layers, 0, g, W.TENSOR_V, a, e).float().numpy()
        assert len(keep) == w.sink + w.window
        q = torch.stack([W.tokens(w, layers, 0, h, W.TENSOR_Q, T - 1, T)[0] for h in range(w.hq)])[None]
        q = q.double().numpy()
        t0 = time.perf_counter()
        O.decode_attention(q, lambda _b, g: hk[g], lambda _b, g: hv[g], [T], mask, w.sink, w.window, w.scale)
        secs += time.perf_counter() - t0
        layers += 1
        del hk, hv
    per_layer = secs / layers
    return {"value": round(per_layer * 1e6, 1), "unit": "us/layer-step",
            "ms_per_step": round(per_layer * 1e3 * w.layers, 1), "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle",
            "sample": f"numpy fp64 oracle decode of {layers} whole layer(s) of the million-token step (all 32 "
                      f"query heads), {secs:.2f} s; ms_per_step = 32 x the per-layer mean"}


def run_reference(args, rank, world):
    """The oracle as the reference arm: every step is one full layer-step of
    the GQA-128K workload (all 8 sequences, all 32 query heads), the same
    decode steps the GPU arm cycles through, timed on the host cores."""
    if rank != 0:
        return None
    from oracle import duo_oracle as O
    base, gw, lens0 = rank_workload(0, 1)
    mask = W.retrieval_mask(gw, 0)
    n_steps = base.steps
    hk, hv, qs = [], [], []
    for b in range(base.batch):
        Tmax = int(lens0[b]) + n_steps
        hk.append({g: W.tokens(gw, 0, b, g, W.TENSOR_K, 0, Tmax).float().numpy() for g in range(gw.n_kv)})
        hv.append({g: W.tokens(gw, 0, b, g, W.TENSOR_V, 0, Tmax).float().numpy() for g in range(gw.n_kv)})
        p = int(lens0[b])
        qs.append(torch.stack([W.tokens(gw, 0, b, h, W.TENSOR_Q, p, p + n_steps) for h in range(gw.hq)], 1))

    def one(i):
        s = i % n_steps
        for b in range(base.batch):
            T = int(lens0[b]) + s + 1
            q = qs[b][s][None].double().numpy()
            O.decode_attention(q, lambda _b, g: hk[b][g], lambda _b, g: hv[b][g], [T], mask, gw.sink,
                               gw.window, gw.scale)

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one(i)
    secs = (time.perf_counter() - t0) / args.steps
    val = secs * 1e6
    cores = len(os.sched_getaffinity(0))
    sample = (f"per step: the fp64 oracle's decode of one full layer-step (all {base.batch} sequences, all "
              f"{gw.hq} query heads, history as float32 arrays in host memory), decode steps cycled as on the GPU")
    return {
        "impl": "reference", "metric": METRIC, "value": round(val, 1), "unit": "us/layer-step",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(val / 1e3, 4),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "gqa128k: GQA 32q/8kv d=128, B=8 ragged T~U[16384,131072], 4/8 KV heads "
                               "retrieval, S=64 W=256, one full layer-step per step (fp64 oracle)",
                   "global_batch": base.batch, "seq_len": [int(x) for x in lens0],
                   "parallelism": "rank 0 only"},
        "cpu_baseline": {"value": round(val, 1), "unit": "us/layer-step", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(val, 1), "unit": "us/layer-step", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 2048; 20 for --impl reference, whose steps take ~1.5 s)")
    ap.add_argument("--warmup", type=int, default=None, help="warm-up steps (default 64; 3 for --impl reference)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the chunked-prefill measurement")
    ap.add_argument("--only", choices=["decode", "prefill", "fp8", "int4", "paged", "seqsplit", "gated", "tiny",
                                       "mha32k", "mtok"],
                    default=None,
                    help="measure one path only (profiling runs)")
    ap.add_argument("--no-fp8", action="store_true",
                    help="skip the FP8-, INT4-, paged-cache, sequence-split and gated decode measurements")
    ap.add_argument("--mtok-layers", type=int, default=None,
                    help="with --only mtok: run only the first N layers (profiling a smaller case)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the tiny, MHA-32K and million-token decode measurements")
    args = ap.parse_args(argv)
    if args.steps is None:
        args.steps = 20 if args.impl == "reference" else 2048
    if args.warmup is None:
        args.warmup = 3 if args.impl == "reference" else 64
    args.warmup = max(args.warmup, 3)
    rank, world, local = dist_init()
    try:
        if args.impl == "reference":
            res = run_reference(args, rank, world)
        elif args.only == "prefill":
            res = {"metric": "chunked prefill attention", "prefill": run_prefill(local)} if rank == 0 else None
        elif args.only == "fp8":
            res = ({"metric": "FP8-cache decode",
                    "decode_fp8": run_variant_decode(local, "fp8", False, args.steps, args.warmup)}
                   if rank == 0 else None)
        elif args.only == "int4":
            res = ({"metric": "INT4-cache decode",
                    "decode_int4": run_variant_decode(local, "int4", False, args.steps, args.warmup)}
                   if rank == 0 else None)
        elif args.only == "seqsplit":
            res = ({"metric": "sequence-split decode",
                    "decode_seqsplit": run_seqsplit(local, 2, min(args.steps, 256), args.warmup)}
                   if rank == 0 else None)
        elif args.only == "gated":
            res = ({"metric": "gated (alpha-blended) decode",
                    "decode_gated": run_gated(local, min(args.steps, 256), args.warmup)}
                   if rank == 0 else None)
        elif args.only == "tiny":
            res = {"metric": "tiny decode", "decode_tiny": run_tiny(local)} if rank == 0 else None
        elif args.only == "mha32k":
            res = ({"metric": "MHA-32K decode", "decode_mha32k": run_mha32k(local, min(args.steps, 1024))}
                   if rank == 0 else None)
        elif args.only == "mtok":
            res = ({"metric": "million-token decode",
                    "decode_mtok": run_mtok(local, min(args.steps, 10), layers=args.mtok_layers)}
                   if rank == 0 else None)
        elif args.only == "paged":
            res = ({"metric": "paged-cache decode",
                    "decode_paged": run_variant_decode(local, "bf16", True, args.steps, args.warmup)}
                   if rank == 0 else None)
        else:
            res, ctx = run_ours(args, rank, world, local)
            if world == 1 and not args.no_prefill and args.only != "decode":
                res["prefill"] = run_prefill(local)
            if world == 1 and not args.no_fp8 and args.only != "decode":
                res["decode_fp8"] = run_variant_decode(local, "fp8")
                res["decode_int4"] = run_variant_decode(local, "int4")
                res["decode_paged"] = run_variant_decode(local, "bf16", True)
                res["decode_seqsplit"] = run_seqsplit(local)
                res["decode_gated"] = run_gated(local)
            if world == 1 and not args.no_workloads and args.only != "decode":
                res["decode_tiny"] = run_tiny(local)
                res["decode_mha32k"] = run_mha32k(local)
                res["decode_mtok"] = run_mtok(local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline(ctx)
                if "prefill" in res:
                    res["prefill"]["cpu_baseline"] = cpu_baseline_prefill()
                if "decode_mtok" in res:
                    res["decode_mtok"]["cpu_baseline"] = cpu_baseline_mtok()
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
