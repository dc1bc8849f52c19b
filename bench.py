"""Benchmark of the quantized KV-cache hot path: one step = append one new bf16
K/V token per sequence (quantize, residual window, flush when a key group
fills) + decode attention for every sequence over the packed paged cache.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 3] [--impl kvq|reference]
    python bench.py --floor            # the HBM read floor of one decode pass (own JSON)

Prints ONE JSON line (rank 0).  `value` is decode-attention KV GB/s of the
headline workload (--workload, default 3: the INT4 KIVI-style cache): the
algorithmic bytes of the decode call (codes, scales, zero-points, BF16 window
rows, q, out, block-table entries) over its device time, summed over ranks and
divided by the max over ranks.  The decode call is two launches (attention,
then the split-K merge); `roofline.achieved` is the same bytes over the
attention kernel alone (an event recorded between the two).  Inputs live in HBM before the timed region; L2 is flushed before
every timed step (untimed): a 256 MB write, then a read of another 256 MB so
that the write's dirty lines are written back before the timed region and the
timed kernels start on a cold, clean L2.  `e2e` is the same metric through the
C ABI with host buffers: one kvq_step_host call per step (one page-locked
host-to-device copy of the step's k | v | q, append, decode, the attention
output written into page-locked host memory) inside the timed region,
synchronised every step.  With N > 1 every rank runs its own replica
(sequences shard across GPUs; no collective is on the data path; the only
collectives are the barrier and the max-over-ranks timing).  `--impl
reference` times the CPU oracle (test infrastructure) on the same K steps
after W warm-up steps, each decoding a sample of the sequences sized so that
the run stays within a few minutes.

Beside the headline (skipped with --no-workloads): `workloads` gives the same
measurement for the other four workloads with min(K, 20) steps each.  On one
GPU (skipped with --no-control): `bulk_append` times the headline workload's
bulk prefill append; `bf16_control` times decode alone over the same draws for
the quantized, BF16 and FP8 caches; and `next_rows` measures prefix sharing
(pool blocks and decode time against unshared copies) and chunked prefill (a
256-token chunk over an 8192-token context through the prefill kernel).
NVTX ranges mark every append, decode and step_host call.
"""
import argparse
import gc
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from quantized_kv_cache_14_b200.workloads import Draws, workload  # noqa: E402

D = 128
L2_FLUSH_BYTES = 256 << 20
REF_BUDGET_S = 90.0   # oracle decode seconds of the reference arm's warm-up and timed steps


# ---------------------------------------------------------------------------
# algorithmic bytes
# ---------------------------------------------------------------------------

def decode_bytes(w, lengths):
    """Bytes a decode call must move: codes + scales (+ zero-points) of the
    quantized tokens, BF16 rows of the residual window, q, out and one
    block-table entry per page read."""
    f = w.fmt
    es = 4 if f.scale_fp32 else 2
    meta = 0 if (f.bits == 16 or f.fp8) else es * (1 + f.asym)   # BF16 control and FP8: no metadata
    per_tok_q = w.h_kv * (2 * D * f.bits // 8 + D * meta // f.g_k + D * meta // f.g_v)
    per_tok_r = w.h_kv * 2 * D * 2
    total = 0
    for L in lengths:
        Lq = (L // f.residual) * f.residual if f.residual else L
        total += Lq * per_tok_q + (L - Lq) * per_tok_r + ((Lq + f.page - 1) // f.page) * 4
    total += len(lengths) * w.h_q * D * (2 + 4)
    return total


def append_bytes(w, lengths_before, n_new_per_seq=1):
    """Bytes an append of one token per sequence must move: the new bf16 K/V
    rows read, residual slots written, and for every key group that fills, its
    residual rows re-read plus the codes and scales written."""
    f = w.fmt
    es = 4 if f.scale_fp32 else 2
    meta = es * (1 + f.asym)
    row = w.h_kv * D * 2
    total = 0
    for L in lengths_before:
        total += 2 * row                                # new K and V rows read
        if f.residual == 0:
            total += w.h_kv * (2 * D * f.bits // 8 + D * meta // f.g_k + D * meta // f.g_v)
        elif (L + 1) % f.residual == 0:
            R = f.residual
            total += 2 * row * (R - 1)                  # window rows re-read
            total += R * w.h_kv * (2 * D * f.bits // 8 + D * meta // f.g_v) + w.h_kv * D * meta
        else:
            total += 2 * row                            # written to the window
    return total


def pool_blocks(lengths, growth, page):
    return int(sum((L + growth + page - 1) // page for L in lengths)) + 64


# ---------------------------------------------------------------------------
# environment: ranks, clocks, peaks
# ---------------------------------------------------------------------------

def dist_setup(n_gpus):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws == 1:
        return 0, 1, None
    import datetime
    import torch
    import torch.distributed as dist
    backend = os.environ.get("KVQ_BENCH_BACKEND", "nccl" if torch.cuda.is_available() else "gloo")
    rank = int(os.environ["RANK"])
    if backend == "nccl":
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", rank)))
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, ws, dist


def barrier(dist):
    if dist is not None:
        dist.barrier()


def max_over_ranks(dist, values):
    """Elementwise max of a list of floats over ranks."""
    if dist is None:
        return list(values)
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(values, dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def sum_over_ranks(dist, values):
    if dist is None:
        return list(values)
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(values, dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.cpu().tolist()


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while timing."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index, enabled=True, period_ms=50):
        self.proc = None
        self.device_index = device_index
        if not enabled:
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={device_index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", f"-lms={period_ms}"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)),
                "reasons": sorted(reasons), "samples": len(sm)}


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_sha():
    h = hashlib.sha256()
    for f in ("kvq_decode.cu", "kvq_device.cuh", "kvq_tiles.cuh", "kvq_internal.h"):
        with open(os.path.join(ROOT, "quantized_kv_cache_14_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def committed_traffic(workload_name, algorithmic_bytes):
    """Per-launch DRAM bytes of the attention kernel from the committed ncu
    record, scaled from the captured launch to a launch moving
    `algorithmic_bytes` (traffic grows with the units processed), if the record
    was taken from the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    if rec.get("kernel_source_sha") != kernel_source_sha():
        return None
    t = rec.get("traffic_bytes_per_launch", {}).get(workload_name)
    a = rec.get("algorithmic_bytes_per_launch", {}).get(workload_name)
    if t is None or not a:
        return None
    return t * algorithmic_bytes / a


# ---------------------------------------------------------------------------
# the CUDA arm
# ---------------------------------------------------------------------------

def bulk_append_bytes(w, lengths):
    """Bytes a bulk prefill append must move: every new bf16 K/V row read once,
    codes and scales (+ zero-points) of the tokens that land in quantized
    groups written, and the BF16 window rows written (groups that complete
    within the call are quantized from the input rows)."""
    f = w.fmt
    es = 4 if f.scale_fp32 else 2
    meta = 0 if (f.bits == 16 or f.fp8) else es * (1 + f.asym)
    row = w.h_kv * D * 2
    per_tok_q = w.h_kv * (2 * D * f.bits // 8 + D * meta // f.g_k + D * meta // f.g_v)
    total = 0
    for L in lengths:
        Lq = (L // f.residual) * f.residual if f.residual else L
        total += 2 * row * L + per_tok_q * Lq + 2 * row * (L - Lq)
    return total


def nvtx(name):
    import torch
    torch.cuda.nvtx.range_push(name)


def nvtx_pop():
    import torch
    torch.cuda.nvtx.range_pop()


def time_bulk_append(w, new_cache, k_all, v_all, dr, calls):
    """The bulk prefill append alone, on one cache whose sequences are freed
    between calls; the first calls grow the library's plan buffer and
    page-locked plan slots (four of them), so they are not timed.  The GPU is
    held by a sleep while the host plans, so the events see device time only."""
    import torch
    c = new_cache()
    ts = []
    for it in range(calls + 4):
        for sq in range(w.batch):
            c.free_seq(sq)
        torch.cuda.synchronize()
        torch.cuda._sleep(60_000_000)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        c.append(k_all, v_all, dr.seq_ids)
        e1.record()
        torch.cuda.synchronize()
        assert c.sync_status() == 0
        if it >= 4:
            ts.append(e0.elapsed_time(e1) * 1e3)
    c.close()
    us = float(np.median(ts))
    nbytes = bulk_append_bytes(w, dr.lengths)
    return {"us": us, "bytes": nbytes, "gbs": nbytes / (us * 1e-6) / 1e9, "tokens": int(sum(dr.lengths)),
            "calls": calls, "what": "bulk prefill append of every prefill token, device time"}


def run_bulk_only(args):
    """The workload's bulk prefill append alone (every prefill token of its
    sequences through one kvq_append call): device time per call."""
    import torch
    from quantized_kv_cache_14_b200 import kvq
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = workload(args.workload)
    dr = Draws(w, steps=1)
    f = w.fmt
    nb = pool_blocks(dr.lengths, 4, f.page)
    mbps = max((L + 4) // f.page + 2 for L in dr.lengths)
    fmt = kvq.Format(f.bits, f.asym, f.k_axis, f.g_k, f.g_v, f.scale_fp32, f.residual, f.page)

    def new_cache():
        return kvq.KVCache(fmt, w.h_q, w.h_kv, max_seqs=w.batch, num_blocks=nb, max_blocks_per_seq=mbps,
                           seed=w.seed, device=0)

    def bf16_dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    bulk = time_bulk_append(w, new_cache, bf16_dev(dr.k), bf16_dev(dr.v), dr, max(1, min(args.steps, 10)))
    bulk["workload"] = w.name
    return bulk


def run_gpu(args, rank, ws, dist, widx, steps, warmup, bulk_calls=0):
    """One workload: prefill (bulk append, untimed), then `warmup` steps and
    three timed passes of `steps` steps each -- device-resident inputs (the
    append + decode calls as a user makes them) for `value`; the same with an
    event recorded between the attention kernel and the split-K merge, for
    `roofline` (the attention kernel alone); and host inputs through
    kvq_step_host for `e2e`.  With bulk_calls > 0 it also times the bulk
    prefill append itself (a fresh cache each call)."""
    import torch
    from quantized_kv_cache_14_b200 import kvq

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", rank)) if ws > 1 else 0)
    dev = torch.device("cuda", torch.cuda.current_device())
    w = workload(widx)
    w.seed = w.seed + 1000 * rank        # each replica draws its own inputs
    total_steps = warmup + 3 * steps + 1   # warm-up, device pass, attention pass, e2e warm-up + pass
    dr = Draws(w, steps=total_steps)
    f = w.fmt
    nb = pool_blocks(dr.lengths, total_steps + 2, f.page)
    mbps = max((L + total_steps + 2) // f.page + 2 for L in dr.lengths)
    fmt = kvq.Format(f.bits, f.asym, f.k_axis, f.g_k, f.g_v, f.scale_fp32, f.residual, f.page)

    def new_cache():
        return kvq.KVCache(fmt, w.h_q, w.h_kv, max_seqs=w.batch, num_blocks=nb, max_blocks_per_seq=mbps,
                           seed=w.seed, device=torch.cuda.current_device())

    def bf16_dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    k_all, v_all = bf16_dev(dr.k), bf16_dev(dr.v)
    bulk = time_bulk_append(w, new_cache, k_all, v_all, dr, bulk_calls) if bulk_calls > 0 else None
    cache = new_cache()
    cache.append(k_all, v_all, dr.seq_ids)      # prefill, untimed
    del k_all, v_all
    lens = list(dr.lengths)
    B = w.batch
    ids = np.arange(B, dtype=np.int32)
    steps_in = [dr.step() for _ in range(total_steps)]
    dev_in = [(bf16_dev(k), bf16_dev(v), bf16_dev(q)) for k, v, q in steps_in]
    # host inputs of a step in one page-locked buffer, k | v | q back to back,
    # so kvq_step_host issues one host-to-device copy
    host_in = []
    for k, v, q in steps_in:
        flat = np.concatenate([k.ravel(), v.ravel(), q.ravel()]).view(np.int16)
        buf = torch.from_numpy(flat).view(torch.bfloat16).pin_memory()
        nk = k.size
        host_in.append((buf[:nk].view(k.shape), buf[nk:2 * nk].view(v.shape), buf[2 * nk:].view(q.shape)))
    del dr
    out = torch.empty((B, w.h_q, D), dtype=torch.float32, device=dev)
    out_host = torch.empty_like(out, device="cpu").pin_memory()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    assert cache.sync_status() == 0

    def one_step(s, e2e, evs):
        nonlocal lens
        ev0, ev1, ev2 = evs
        flush.zero_()                                   # untimed: evicts L2 ...
        flush_rd.sum()                                  # ... and writes the dirty lines back
        ev0.record()
        lens = [L + 1 for L in lens]
        if e2e:
            # one C-ABI call from page-locked host buffers: one H2D copy of
            # k | v | q, append, decode over the stored lengths, output written
            # into page-locked host memory
            kh, vh, qh = host_in[s]
            nvtx("step_host")
            cache.step_host(kh, vh, ids, qh, out_host)
            nvtx_pop()
            ev1.record()
            ev2.record()
            return
        k, v, q = dev_in[s]
        nvtx("append")
        cache.append(k, v, ids)
        nvtx_pop()
        ev1.record()
        nvtx("decode")
        cache.decode(q, None, out)              # attends over the stored lengths
        nvtx_pop()
        ev2.record()

    for s in range(warmup):
        one_step(s, False, [torch.cuda.Event(enable_timing=True) for _ in range(3)])
    torch.cuda.synchronize()
    assert cache.sync_status() == 0

    # timed: device-resident inputs, the calls as a user makes them.  The
    # host enqueues every step before waiting (as a serving loop runs ahead of
    # the GPU), so the events see device time, not host launch gaps.
    gc.collect()
    gc.disable()   # no collector pause inside a timed region (enabled again below)
    st0 = cache.stats()["kernel_launches"]
    sampler = ClockSampler(torch.cuda.current_device(), enabled=not args.no_clocks)
    time.sleep(0.15 if sampler.proc else 0)
    barrier(dist)
    torch.cuda.synchronize()
    kv_bytes, app_bytes, seq_tokens = 0, 0, 0
    s0 = warmup
    step_evs = []
    for s in range(s0, s0 + steps):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        before = list(lens)
        one_step(s, False, evs)
        step_evs.append(evs)
        kv_bytes += decode_bytes(w, lens)
        app_bytes += append_bytes(w, before)
        seq_tokens += sum(lens)
    torch.cuda.synchronize()
    recs = [(e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2])) for e in step_evs]
    barrier(dist)
    launches = cache.stats()["kernel_launches"] - st0
    clocks = sampler.stop()
    assert cache.sync_status() == 0

    # timed: the attention kernel alone -- the library records an event between
    # it and the merge (which then runs as a plain launch); one event per step
    barrier(dist)
    torch.cuda.synchronize()
    attn_bytes = 0
    s0 += steps
    attn_evs = []
    for s in range(s0, s0 + steps):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        mid = torch.cuda.Event(enable_timing=True)
        mid.record()              # creates the CUDA event; the library records it again
        cache.set_decode_event(mid)
        one_step(s, False, evs)
        attn_evs.append((evs, mid))
        attn_bytes += decode_bytes(w, lens)
    torch.cuda.synchronize()
    t_attn = sum(e[1].elapsed_time(mid) for e, mid in attn_evs)
    barrier(dist)
    cache.set_decode_event(None)
    assert cache.sync_status() == 0

    # timed: end to end through the C ABI with host buffers, after one untimed
    # step through the same call (its first use grows the library's host-step
    # buffers: a device synchronize and an allocation)
    s0 += steps
    one_step(s0, True, [torch.cuda.Event(enable_timing=True) for _ in range(3)])
    s0 += 1
    barrier(dist)
    torch.cuda.synchronize()
    e2e_ms, e2e_bytes = 0.0, 0
    for s in range(s0, s0 + steps):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        one_step(s, True, evs)
        evs[2].synchronize()
        e2e_ms += evs[0].elapsed_time(evs[2])
        e2e_bytes += decode_bytes(w, lens)
    torch.cuda.synchronize()
    gc.enable()
    barrier(dist)
    assert cache.sync_status() == 0
    cache.close()

    t_app = sum(r[0] for r in recs)
    t_dec = sum(r[1] for r in recs)
    step_ms = t_app + t_dec
    mx = max_over_ranks(dist, [t_app, t_dec, step_ms, e2e_ms])
    tot = sum_over_ranks(dist, [kv_bytes, app_bytes, seq_tokens, e2e_bytes])
    K = steps
    return {
        "w": w, "K": K, "ws": ws, "launches": launches, "clocks": clocks,
        "kv_gbs": tot[0] / (mx[1] * 1e-3) / 1e9,
        "attn_gbs": (attn_bytes / K) / (t_attn / K * 1e-3) / 1e9,
        "attn_bytes_per_launch": attn_bytes / K,
        "attn_us": t_attn / K * 1e3,
        "decode_us": t_dec / K * 1e3,
        "append_us": t_app / K * 1e3,
        "append_gbs": tot[1] / (mx[0] * 1e-3) / 1e9,
        "seq_tok_s": tot[2] / (mx[2] * 1e-3),
        "ms_per_step": mx[2] / K,
        "e2e_gbs": tot[3] / (mx[3] * 1e-3) / 1e9,
        "kv_bytes_per_step": kv_bytes / K,
        "lens_final": lens,
        "h2d": B * w.h_kv * D * 2 * 2 + B * w.h_q * D * 2,
        "d2h": B * w.h_q * D * 4,
        "bulk": bulk,
    }


def run_control(args):
    """The pages' trade-off, saved traffic versus dequantization work, on this
    workload: decode alone (no appends) over the quantized cache and over the
    BF16 control cache (same paged path, bf16 rows, no dequantization), both
    filled from the same draws; L2 flushed clean before every call."""
    import dataclasses
    import torch
    from quantized_kv_cache_14_b200 import kvq
    from quantized_kv_cache_14_b200.workloads import CacheFormat
    dev = torch.device("cuda", torch.cuda.current_device())
    w = workload(args.workload)
    K = max(5, min(args.steps, 50))
    dr = Draws(w, steps=1)
    k, v, q = dr.step()
    lens = [L + 1 for L in dr.lengths]
    bf = dataclasses.replace(w, fmt=CacheFormat(16, 0, 0, 128, 128, 0, 0, w.fmt.page))
    f8 = dataclasses.replace(w, fmt=CacheFormat(8, 0, 0, 128, 128, 0, 0, w.fmt.page, fp8=1))
    # FP8 scales per kv head: amax of the prefill / 448 (no calibration)
    kf = np.abs((dr.k.view(np.uint16).astype(np.uint32) << 16).view(np.float32))
    vf = np.abs((dr.v.view(np.uint16).astype(np.uint32) << 16).view(np.float32))
    f8_scales = ((np.maximum(kf.max(axis=(0, 2)), 1e-6) / 448.0).astype(np.float32),
                 (np.maximum(vf.max(axis=(0, 2)), 1e-6) / 448.0).astype(np.float32))
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    out = {}
    for tag, ww in (("quantized", w), ("bf16", bf), ("fp8", f8)):
        f = ww.fmt
        nb = pool_blocks(lens, 2, f.page)
        mbps = max((L + 2) // f.page + 2 for L in lens)
        cache = kvq.KVCache(kvq.Format(f.bits, f.asym, f.k_axis, f.g_k, f.g_v, f.scale_fp32, f.residual,
                                       f.page, f.fp8), ww.h_q, ww.h_kv, max_seqs=ww.batch, num_blocks=nb,
                            max_blocks_per_seq=mbps, seed=ww.seed, device=torch.cuda.current_device())
        if f.fp8:
            cache.set_fp8_scales(*f8_scales)

        def dbf(a):
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        cache.append(dbf(dr.k), dbf(dr.v), dr.seq_ids)
        cache.append(dbf(k), dbf(v), np.arange(ww.batch, dtype=np.int32))
        qd = dbf(q)
        sl = torch.tensor(lens, dtype=torch.int32, device=dev)
        o = torch.empty((ww.batch, ww.h_q, D), dtype=torch.float32, device=dev)
        evs = []
        for it in range(K + 3):
            flush.zero_()
            flush_rd.sum()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            cache.decode(qd, sl, o)
            e1.record()
            if it >= 3:
                evs.append((e0, e1))
        torch.cuda.synchronize()
        assert cache.sync_status() == 0
        us = float(np.median([a.elapsed_time(b) for a, b in evs])) * 1e3
        nbytes = decode_bytes(ww, lens)
        out[tag] = {"decode_us": us, "kv_bytes": nbytes, "gbs": nbytes / (us * 1e-6) / 1e9}
        cache.close()
    return {"format": "BF16 control: the same paged path over bf16 rows, no dequantization; FP8: E4M3 "
                      "with one scale per kv head (amax / 448 of the prefill)",
            "calls": K, "quantized": out["quantized"], "bf16": out["bf16"], "fp8": out["fp8"],
            "speedup_quantized_over_bf16": out["bf16"]["decode_us"] / out["quantized"]["decode_us"],
            "speedup_fp8_over_bf16": out["bf16"]["decode_us"] / out["fp8"]["decode_us"]}


def _timed_calls(fn, K, flush, flush_rd):
    """Median device time (µs) of fn() over K calls after 3 warm-up calls,
    with a clean L2 flush before each."""
    import torch
    evs = []
    for it in range(K + 3):
        flush.zero_()
        flush_rd.sum()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        if it >= 3:
            evs.append((e0, e1))
    torch.cuda.synchronize()
    return float(np.median([a.elapsed_time(b) for a, b in evs])) * 1e3


def run_next_rows(args):
    """The widened rows on the workload's format:
    prefix sharing -- 16 sequences over one 8192-token prefix (whole key
    groups) plus 64 tokens of their own, the prefix held once through
    kvq_share_prefix, against 16 unshared copies of the same tokens: pool
    blocks and decode time (outputs must agree bit for bit);
    chunked prefill -- run_chunked_prefill."""
    import torch
    from quantized_kv_cache_14_b200 import kvq
    from quantized_kv_cache_14_b200.workloads import random_bf16
    dev = torch.device("cuda", torch.cuda.current_device())
    w = workload(args.workload)
    f = w.fmt
    K = max(5, min(args.steps, 30))
    rng = np.random.default_rng(w.seed + 77)
    fmt = kvq.Format(f.bits, f.asym, f.k_axis, f.g_k, f.g_v, f.scale_fp32, f.residual, f.page, f.fp8)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def dbf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    B, Lp, Ls = w.batch, 8192, 64
    kp, vp = random_bf16(rng, (Lp, w.h_kv, D)), random_bf16(rng, (Lp, w.h_kv, D))
    ks, vs = random_bf16(rng, (B * Ls, w.h_kv, D)), random_bf16(rng, (B * Ls, w.h_kv, D))
    sid = np.repeat(np.arange(B, dtype=np.int32), Ls)
    q = dbf(random_bf16(rng, (B, w.h_q, D)))
    lens = [Lp + Ls] * B
    mbps = (Lp + Ls) // f.page + 4
    share = {}
    outs = {}
    for tag in ("shared", "unshared"):
        nb = (B if tag == "unshared" else 1) * (Lp // f.page) + B * (Ls // f.page + 2) + 64
        c = kvq.KVCache(fmt, w.h_q, w.h_kv, max_seqs=B, num_blocks=nb, max_blocks_per_seq=mbps,
                        seed=w.seed, device=torch.cuda.current_device())
        if tag == "shared":
            c.append(dbf(kp), dbf(vp), np.zeros(Lp, np.int32))
            for s in range(1, B):
                c.share_prefix(0, s, Lp)
        else:
            c.append(dbf(np.tile(kp, (B, 1, 1))), dbf(np.tile(vp, (B, 1, 1))),
                     np.repeat(np.arange(B, dtype=np.int32), Lp))
        c.append(dbf(ks), dbf(vs), sid)
        o = torch.empty((B, w.h_q, D), dtype=torch.float32, device=dev)
        us = _timed_calls(lambda: c.decode(q, None, o), K, flush, flush_rd)
        assert c.sync_status() == 0
        outs[tag] = o.cpu()
        st = c.stats()
        share[tag] = {"decode_us": us, "blocks_used": int(st["blocks_used"]),
                      "pool_bytes_used": int(st["blocks_used"]) * c.layout["block_bytes"]}
        c.close()
    share["outputs_equal"] = bool(torch.equal(outs["shared"], outs["unshared"]))
    share["memory_ratio"] = share["unshared"]["blocks_used"] / share["shared"]["blocks_used"]
    share["speedup"] = share["unshared"]["decode_us"] / share["shared"]["decode_us"]
    share["workload"] = f"{B} sequences x ({Lp} shared + {Ls} own) tokens"

    return {"calls": K, "prefix_sharing": share, "chunked_prefill": run_chunked_prefill(args)}


def run_chunked_prefill(args):
    """Chunked prefill on the workload's format: one sequence with an
    8192-token context and a new chunk of 256 tokens, each chunk token
    attending its causal prefix through kvq_prefill_attn (a user's call:
    host planning, plan upload, attention and split merge inside the timed
    region): time per chunk, query tokens per second and attention TFLOP/s."""
    import torch
    from quantized_kv_cache_14_b200 import kvq
    from quantized_kv_cache_14_b200.workloads import random_bf16
    dev = torch.device("cuda", torch.cuda.current_device())
    w = workload(args.workload)
    f = w.fmt
    K = max(5, min(args.steps, 30))
    rng = np.random.default_rng(w.seed + 78)
    fmt = kvq.Format(f.bits, f.asym, f.k_axis, f.g_k, f.g_v, f.scale_fp32, f.residual, f.page, f.fp8)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def dbf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    Lc, C = 8192, 256
    c = kvq.KVCache(fmt, w.h_q, w.h_kv, max_seqs=C, num_blocks=(Lc + C) // f.page + 64,
                    max_blocks_per_seq=(Lc + C) // f.page + 4, seed=w.seed, device=torch.cuda.current_device())
    c.append(dbf(random_bf16(rng, (Lc + C, w.h_kv, D))), dbf(random_bf16(rng, (Lc + C, w.h_kv, D))),
             np.zeros(Lc + C, np.int32))
    qc = dbf(random_bf16(rng, (C, w.h_q, D)))
    oc = torch.empty((C, w.h_q, D), dtype=torch.float32, device=dev)
    ids = np.zeros(C, np.int32)
    pos = np.arange(Lc, Lc + C, dtype=np.int32)
    us = _timed_calls(lambda: c.prefill_attn(qc, ids, pos, oc), K, flush, flush_rd)
    assert c.sync_status() == 0
    c.close()
    row_bytes = decode_bytes(w, [int(p) + 1 for p in pos])
    flops = 4.0 * w.h_q * D * float(sum(int(p) + 1 for p in pos))   # QK^T and PV, 2 flops per MAC
    prefill = {"workload": f"one sequence, {Lc}-token context, chunk of {C} new tokens",
               "chunk_us": us, "query_tokens_per_s": C / (us * 1e-6),
               "attention_tflops": flops / (us * 1e-6) / 1e12,
               "row_bytes": row_bytes, "row_gbs": row_bytes / (us * 1e-6) / 1e9,
               "note": "a block of query tokens (32 x 4 heads = 128 rows of the tcgen05 M dimension on "
                       "the tensor-core path, 64 / g tokens on the mma.sync path) shares every staged "
                       "tile, key range split over CTAs; row_gbs counts the bytes each row would read "
                       "on its own"}
    prefill["calls"] = K
    return prefill


def chunk_used_bytes(w, layout):
    """Bytes a decode stage copies per page chunk: codes and metadata, without
    the chunk's tail padding."""
    f = w.fmt
    es = 4 if f.scale_fp32 else 2
    if f.bits == 16 or f.fp8:
        meta = 0
    elif f.k_axis:
        meta = layout["kslice"] * es * (1 + f.asym)
    else:
        meta = f.page * (D // f.g_k) * es * (1 + f.asym)
    return layout["off_kmeta"] + (meta + 15) // 16 * 16


def run_floor(args):
    """HBM read floor of one decode pass (kvq_read_floor): the time a single
    launch needs just to read bytes, with no compute.  Three byte sets:
    `paged`, the page chunks a decode call of the workload stages, in decode
    order, at their block-table addresses (the same bytes as the decode call's
    quantized part); `linear`, the same number of chunks back to back; and
    contiguous buffers of 1 and 2 GB.  Two ways of reading: `bulk`, the decode
    kernel's scheme (cp.async.bulk into per-warp stages, persistent grid of
    four-warp CTAs) over a sweep of CTAs per SM, stages per warp and chunks
    per unit; `stream`, 128-bit loads by every thread.  Median and best of
    `calls` launches, L2 flushed clean before each."""
    import torch
    from quantized_kv_cache_14_b200 import kvq
    dev = torch.device("cuda", torch.cuda.current_device())
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    w = workload(args.workload)
    f = w.fmt
    dr = Draws(w, steps=1)
    nb = pool_blocks(dr.lengths, 2, f.page)
    mbps = max((L + 2) // f.page + 2 for L in dr.lengths)
    cache = kvq.KVCache(kvq.Format(f.bits, f.asym, f.k_axis, f.g_k, f.g_v, f.scale_fp32, f.residual, f.page),
                        w.h_q, w.h_kv, max_seqs=w.batch, num_blocks=nb, max_blocks_per_seq=mbps, seed=w.seed,
                        device=torch.cuda.current_device())

    def dbf(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    cache.append(dbf(dr.k), dbf(dr.v), dr.seq_ids)
    torch.cuda.synchronize()
    lay = cache.layout
    chunk = chunk_used_bytes(w, lay)
    offs = []
    for i, L in enumerate(dr.lengths):
        Lq = (L // f.residual) * f.residual if f.residual else L
        npg = (Lq + f.page - 1) // f.page
        tab = cache.block_table_host(i)[:npg].astype(np.int64)
        for h in range(w.h_kv):
            offs.append(tab * lay["block_bytes"] + h * lay["chunk_bytes"])
    offs = torch.from_numpy(np.concatenate(offs)).to(dev)
    n = int(offs.numel())
    pool_ptr, pool_bytes = cache.pool_device()
    sink = torch.zeros(2, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    K = max(10, min(args.steps, 50))
    smem_per_sm = torch.cuda.get_device_properties(dev).shared_memory_per_multiprocessor

    def timed(fn):
        evs = []
        for it in range(K + 3):
            flush.zero_()
            flush_rd.sum()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            if it >= 3:
                evs.append((e0, e1))
        torch.cuda.synchronize()
        t = [a.elapsed_time(b) * 1e3 for a, b in evs]
        return float(np.median(t)), float(min(t))

    peak, peak_kind = measured_peak()
    rows = []

    def record(kind, nbytes, mode, ctas, stages, per_unit, fn):
        med, best = timed(fn)
        rows.append({"bytes": kind, "nbytes": nbytes, "mode": mode, "ctas": ctas,
                     "ctas_per_sm": ctas / sms, "stages": stages, "per_unit": per_unit,
                     "us_median": med, "us_best": best, "gbs_median": nbytes / med / 1e3,
                     "frac_median": nbytes / med / 1e3 / peak})

    sweep = [(3, 2, 4), (3, 1, 8), (2, 3, 4), (2, 2, 8), (1, 6, 4), (1, 4, 8), (4, 1, 4), (2, 2, 4), (1, 2, 4)]
    lin = torch.empty(n * chunk + 16, dtype=torch.uint8, device=dev)
    lin.random_(0, 255)
    for per_sm, S, U in sweep:
        smem = 4 * S * ((U * chunk + 127) // 128 * 128 + 8)
        if per_sm * (smem + 1024) > smem_per_sm:
            continue
        ctas = per_sm * sms
        record("paged", n * chunk, "bulk", ctas, S, U, lambda: kvq.kvq_read_floor(
            pool_ptr, offs.data_ptr(), n, pool_bytes, chunk, 0, ctas, S, U, sink.data_ptr(),
            torch.cuda.current_stream().cuda_stream))
        record("linear", n * chunk, "bulk", ctas, S, U, lambda: kvq.kvq_read_floor(
            lin.data_ptr(), 0, n, lin.numel() // 16 * 16, chunk, 0, ctas, S, U, sink.data_ptr(),
            torch.cuda.current_stream().cuda_stream))
    span_lin = n * chunk // 16 * 16
    for mult in (2, 4, 8, 16):
        ctas = mult * sms
        record("linear", span_lin, "stream", ctas, 0, 0, lambda: kvq.kvq_read_floor(
            lin.data_ptr(), 0, 0, span_lin, 16, 1, ctas, 1, 1, sink.data_ptr(),
            torch.cuda.current_stream().cuda_stream))
    del lin
    for gb in (1, 2):
        big = torch.empty(gb << 30, dtype=torch.uint8, device=dev)
        big.random_(0, 255)
        nbig = big.numel() // chunk
        for per_sm, S, U in ((3, 2, 4), (1, 6, 4)):
            ctas = per_sm * sms
            record(f"{gb}GB", nbig * chunk, "bulk", ctas, S, U, lambda: kvq.kvq_read_floor(
                big.data_ptr(), 0, nbig, big.numel(), chunk, 0, ctas, S, U, sink.data_ptr(),
                torch.cuda.current_stream().cuda_stream))
        for mult in (4, 8):
            ctas = mult * sms
            record(f"{gb}GB", big.numel(), "stream", ctas, 0, 0, lambda: kvq.kvq_read_floor(
                big.data_ptr(), 0, 0, big.numel(), 16, 1, ctas, 1, 1, sink.data_ptr(),
                torch.cuda.current_stream().cuda_stream))
        del big
    torch.cuda.synchronize()
    err = int(sink[1].item())
    cache.close()
    return {"floor": rows, "workload": w.name, "chunk_bytes": chunk, "chunks": n, "sms": sms,
            "peak": peak, "peak_kind": peak_kind, "calls": K, "error_flags": err,
            "l2": "flushed before every call (256 MB write then 256 MB read, untimed)"}


# ---------------------------------------------------------------------------
# the CPU oracle (baseline / reference arm)
# ---------------------------------------------------------------------------

def oracle_cache_for(w, dr, growth):
    from oracle import oracle as O
    f = w.fmt
    nb = pool_blocks(dr.lengths, growth, f.page)
    mbps = max((L + growth) // f.page + 2 for L in dr.lengths)
    oc = O.OracleCache(bits=f.bits, asym=f.asym, k_axis=f.k_axis, g_k=f.g_k, g_v=f.g_v,
                       scale_fp32=f.scale_fp32, residual=f.residual, page=f.page, h_q=w.h_q,
                       h_kv=w.h_kv, d_h=D, max_seqs=w.batch, num_blocks=nb,
                       max_blocks_per_seq=mbps, seed=w.seed, fail_alloc_after=-1)
    assert oc.append(dr.k, dr.v, dr.seq_ids) == 0
    return oc


def run_oracle_sample(w, steps, warmup, rows, threads, budget_s=None):
    """Oracle steps (append one token per sequence + decode of `rows`
    sequences); returns (decode GB/s, seconds timed, bytes, final lengths,
    rows decoded per step).  With `budget_s`, one untimed decode of all `rows`
    on the prefilled cache first measures the cost of a wave of (row, kv
    head) items on `threads` threads, and the rows per step drop (to 1 at
    least) until warmup + steps decodes fit the budget."""
    dr = Draws(w, steps=steps + warmup)
    oc = oracle_cache_for(w, dr, steps + warmup + 2)
    lens = list(dr.lengths)
    ids = np.arange(w.batch, dtype=np.int32)
    if budget_s is not None:
        sub = np.arange(rows, dtype=np.int32)
        q0 = np.zeros((rows, w.h_q, D), np.uint16)   # the decode's cost does not depend on q
        t0 = time.perf_counter()
        oc.decode(q0, [lens[i] for i in sub], seq_ids=sub, nthreads=threads)
        waves = -(-rows * w.h_kv // threads)
        t_wave = (time.perf_counter() - t0) / waves
        while rows > 1 and (steps + warmup) * t_wave * -(-rows * w.h_kv // threads) > budget_s:
            rows -= 1
    t_dec, nbytes = 0.0, 0
    for s in range(warmup + steps):
        k, v, q = dr.step()
        assert oc.append(k, v, ids) == 0
        lens = [L + 1 for L in lens]
        sub = np.arange(rows, dtype=np.int32)
        t0 = time.perf_counter()
        oc.decode(q[:rows], [lens[i] for i in sub], seq_ids=sub, nthreads=threads)
        dt = time.perf_counter() - t0
        if s >= warmup:
            t_dec += dt
            nbytes += decode_bytes(w, [lens[i] for i in sub])
    oc.close()
    return nbytes / t_dec / 1e9, t_dec, nbytes, lens, rows


def workload_config(w, lens):
    f = w.fmt
    kind = {(8, 0): "INT8 sym", (4, 0): "INT4 sym", (2, 1): "INT2 asym", (2, 0): "INT2 sym",
            (4, 1): "INT4 asym", (8, 1): "INT8 asym"}[(f.bits, f.asym)]
    axis = "per-channel" if f.k_axis else "per-token"
    return {
        "workload": f"{w.name}: {w.note}",
        "format": f"{kind}, keys {axis} G={f.g_k}, values per-token G={f.g_v}, "
                  f"{'fp32' if f.scale_fp32 else 'fp16'} scales, page {f.page}, BF16 window {f.residual}",
        "batch": w.batch, "h_q": w.h_q, "h_kv": w.h_kv, "d_h": D,
        "seq_len_min": int(min(lens)), "seq_len_max": int(max(lens)),
        "l2": "flushed before every timed step (256 MB write then 256 MB read, untimed)",
        "step": "append 1 token per sequence (quantize/window/flush) + decode attention",
        "parallelism": "replicas",
    }


def attention_kernel_name(w):
    """The decode attention kernel the library picks for the workload's format
    (the warp-specialised kernel's three specs, else the generic kernel)."""
    f = w.fmt
    if (w.h_q // w.h_kv == 4 and f.page == 16 and not f.scale_fp32 and not f.fp8 and
            (f.bits, f.asym, f.k_axis, f.g_k, f.g_v, f.residual) in
            ((4, 0, 1, 64, 64, 64), (2, 1, 1, 32, 32, 32), (8, 0, 0, 128, 128, 0))):
        spec = {4: "SpecInt4Kivi", 2: "SpecInt2Kivi", 8: "SpecInt8Tok"}[f.bits]
        return f"decode_ws_kernel<{spec}>"
    return "decode_kernel"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", type=int, default=3, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=0, help="rows of the CPU oracle sample")
    ap.add_argument("--no-control", action="store_true", help="skip the BF16 / FP8 comparison and the prefix-sharing and chunked-prefill measurements")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time only --workload (skip the other four workloads' lines)")
    ap.add_argument("--only", choices=["prefill", "bulk"],
                    help="measure one row alone and print its own JSON: prefill = chunked prefill, "
                         "bulk = the workload's bulk prefill append")
    ap.add_argument("--floor", action="store_true",
                    help="measure the HBM read floor of one decode pass instead (one GPU; prints its own JSON)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.floor:
        print(json.dumps(run_floor(args)))
        return
    if args.only == "prefill":
        print(json.dumps(run_chunked_prefill(args)))
        return
    if args.only == "bulk":
        print(json.dumps(run_bulk_only(args)))
        return

    rank, ws, dist = dist_setup(args.gpus)
    w = workload(args.workload)
    threads = os.cpu_count() or 1
    rows = args.cpu_rows or min(w.batch, 16)

    if args.impl == "reference":
        if rank != 0:
            return
        # the same K timed steps after W warm-up steps as the CUDA arm, each
        # step a sample of the workload: rows per step sized so that the
        # oracle's decodes take about REF_BUDGET_S in all
        steps, warm = args.steps, args.warmup
        gbs, secs, nbytes, lens, rows = run_oracle_sample(w, steps, warm, rows, threads, budget_s=REF_BUDGET_S)
        line = {
            "metric": "decode-attn KV GB/s", "value": gbs, "unit": "GB/s", "impl": "reference",
            "n_gpus": 0, "steps": steps, "warmup": warm,
            "ms_per_step": secs / steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, lens),
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": f"{steps} steps after {warm} warm-up: append 1 token to each of "
                                       f"{w.batch} sequences, decode {rows} of them, fp64 C++ oracle"},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line))
        return

    res = run_gpu(args, rank, ws, dist, args.workload, args.steps, args.warmup,
                  bulk_calls=0 if args.no_control else 5)
    others = {}
    if not args.no_workloads:
        for widx in (1, 2, 3, 4, 5):
            if widx == args.workload:
                continue
            r = run_gpu(args, rank, ws, dist, widx, max(5, min(args.steps, 20)), args.warmup)
            others[workload(widx).name] = r
    if rank != 0:
        return
    peak, peak_kind = measured_peak()
    cpu = None
    if ws == 1 and not args.no_cpu_baseline:
        n_cpu = 24   # about 10 s of oracle decode on the machine's host cores
        gbs, secs, _, _, _ = run_oracle_sample(w, n_cpu, 0, rows, threads)
        cpu = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"{n_cpu} steps of {rows}/{w.batch} sequences (append + fp64 decode), "
                         f"{secs:.1f} s timed"}
    traffic = committed_traffic(w.name, res["attn_bytes_per_launch"])
    control = run_control(args) if (ws == 1 and not args.no_control) else None
    next_rows = run_next_rows(args) if (ws == 1 and not args.no_control) else None
    per_workload = {}
    for name, r in others.items():
        per_workload[name] = {
            "steps": r["K"], "attn_us": r["attn_us"], "decode_us": r["decode_us"], "kv_gbs": r["kv_gbs"],
            "frac": r["attn_gbs"] / peak, "kv_bytes_per_step": r["kv_bytes_per_step"],
            "e2e_gbs": r["e2e_gbs"], "append_us": r["append_us"], "append_gbs": r["append_gbs"],
            "seq_tokens_per_s": r["seq_tok_s"], "clocks": r["clocks"],
            "config": workload_config(r["w"], r["lens_final"])["workload"],
        }
    bulk = res["bulk"]
    if bulk is not None:
        bulk["frac"] = bulk["gbs"] / peak
    line = {
        "metric": "decode-attn KV GB/s", "value": res["kv_gbs"], "unit": "GB/s",
        "n_gpus": ws, "steps": res["K"], "warmup": args.warmup,
        "ms_per_step": res["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        # the arithmetic: bf16 rows in, codes quantized in fp32, attention on
        # fp16 tensor-core operands (hi + lo parts) accumulated in fp32, fp32
        # softmax and output
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, res["lens_final"]),
        "roofline": {"bound": "hbm", "achieved": res["attn_gbs"], "peak": peak, "unit": "GB/s",
                     "frac": res["attn_gbs"] / peak, "traffic": traffic,
                     "peak_kind": peak_kind,
                     "kernel": attention_kernel_name(w) + " (attention, without the merge)"},
        "cpu_baseline": cpu,
        "e2e": {"value": res["e2e_gbs"], "unit": "GB/s", "h2d_bytes_per_step": res["h2d"],
                "d2h_bytes_per_step": res["d2h"]},
        "gpu_launches": res["launches"],
        "clocks": res["clocks"],
        "seq_tokens_per_s": res["seq_tok_s"],
        "append_gbs": res["append_gbs"],
        "bulk_append": bulk,
        "attn_us": res["attn_us"], "decode_us": res["decode_us"], "append_us": res["append_us"],
        "kv_bytes_per_step": res["kv_bytes_per_step"],
        "frac_of_8TBps": res["kv_gbs"] / 8000.0,
        "frac_of_peak": res["kv_gbs"] / peak,
        "workloads": per_workload,
        "bf16_control": control,
        "next_rows": next_rows,
    }
    print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
