#!/usr/bin/env python
"""Decode-step benchmark of the ragged paged decode library on B200.

One step = one decode step of one layer over the whole batch: the split-K decode kernel plus
the log-sum-exp merge, through the C ABI (tg_ragged_paged_decode / tg_tiered_decode). The
batch's KV cache, page tables and plan are resident in HBM before timing (admission happens
once, as in serving); the step's inputs are the queries.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--layers L]
                    [--impl ours|reference]
    python bench.py --path sink|h2o|ttkv|ttkv-host|splitzip ...   (one GPU, other lines)

The default workload is the multi-turn serving step (config 3): its 32 layers are made resident
one at a time (all 32 layers' pools exceed one GPU) and each layer's step is timed; the line
reports all layers' K/V bytes over the summed step time, per-layer figures and the worst layer.
Per layer: W warm-up steps, K timed steps with nothing instrumented, then a separate pass with
the library's kernel events on (per-kernel times for the roofline), then K end-to-end steps
through the host-buffer call.

N > 1 runs under torch.distributed.run, one rank per GPU. The batch is sharded by sequence with
the library's ahead-of-time placement (per-GPU work fixed: weak scaling); the decode has no
data-path collective, the ranks only agree on timing (barrier + max over ranks).

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "ragged paged decode attn: KV-read GB/s vs HBM peak; decode tokens/s per layer"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2**20

WORKLOAD_NAMES = {
    1: "tiny ragged MHA decode: 1 seq, 8/8 heads, d 64, retained U[16,256] per head, page 16",
    2: "GQA decode layer, ragged budgets: batch 64/GPU, 32 q / 8 KV heads, d 128, context "
       "U[2048,8192], retention ratio ranked onto [0.1,0.9] +-0.05 per (seq, KV head), "
       "4 budget groups, page 16, pool 90% occupied, shuffled",
    3: "multi-turn serving step, one layer: batch 256/GPU, 32 q / 8 KV heads, d 128, context "
       "U[4096,32768], ratios [0.05,0.5] over 256 (layer, head) ranks, 8 budget groups",
    4: "prefix-shared decode: 512 seqs/GPU, 32 q / 8 KV heads, d 128, 2000-token system prefix "
       "+ 1 of 8 500-token docs + private 80-100 tokens, full retention",
    5: "tiered long-context decode: batch 4/GPU, context 131072, 32 q / 8 KV heads, d 128, last "
       "8192 tokens bf16, older INT8 per token per head, >= 64 chunks per head",
}


def _env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def _plan_kw(cfg):
    """Plan options per workload (chosen by measurement on B200; see workload.timed_plan_options)."""
    from non_uniform_paged_flash_b200 import workload
    return workload.timed_plan_options(cfg)


SLOW_BITS = 8   # code width of the tiered workloads' slow tier (--slow-bits)
NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e nominal bandwidth (context beside the measured peak)


def _workload_name(cfg, sp):
    """The workload's name, with the slow tier's code width where it is not the named INT8."""
    name = WORKLOAD_NAMES[cfg]
    if sp.kind == "tiered" and sp.slow_bits == 4:
        name = name.replace("older INT8", "older INT4") if "older INT8" in name else name + " (INT4 slow tier)"
    return name


def _preset(cfg):
    """The named workload; tiered ones with the slow tier at SLOW_BITS."""
    from dataclasses import replace
    sp = synth.preset(cfg)
    return replace(sp, slow_bits=SLOW_BITS) if sp.kind == "tiered" else sp


def _global_spec(cfg, world):
    sp = _preset(cfg)
    if world > 1:
        from dataclasses import replace
        sp = replace(sp, B=sp.B * world)
    return sp


def _my_sequences(sp, rank, world, kv_len, fast_len):
    """Ahead-of-time placement of sequences on ranks by retained K/V bytes."""
    if world == 1:
        return None
    import non_uniform_paged_flash_b200 as tg
    if fast_len is None:
        per_seq = kv_len.astype(np.int64).sum(1) * 2 * sp.D * 2
    else:
        f = np.minimum(fast_len, kv_len).astype(np.int64)
        slow_row = sp.D if sp.slow_bits == 8 else sp.D // 2     # code bytes per slow token-head
        per_seq = ((kv_len - f) * 2 * (slow_row + 4) + f * 2 * sp.D * 2).sum(1)
    gpu = tg.tg_place_sequences(per_seq, world)
    return np.nonzero(gpu == rank)[0]


def _over_ranks(dist, vals, n_max):
    """The first n_max entries of vals (times, error flags) as their maximum over ranks, the
    rest (work done) as their sum; vals is a float64 tensor on the process group's device."""
    if dist is None:
        return vals.tolist()
    mx, sm = vals.clone(), vals.clone()
    dist.all_reduce(mx, op=dist.ReduceOp.MAX)
    dist.all_reduce(sm, op=dist.ReduceOp.SUM)
    return mx[:n_max].tolist() + sm[n_max:].tolist()


def _measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _traffic(cfg, alg_per_launch=None):
    """DRAM bytes per launch of the decode kernel from a committed ncu capture, if the kernel
    source is unchanged since the capture; else None. A capture of one layer of a multi-layer
    workload is stored as its traffic / algorithmic-bytes ratio and scaled to alg_per_launch
    (the traffic grows with the pages a launch reads). A tiered workload with the INT4 slow tier
    has its own entry."""
    src = os.path.join(ROOT, "non_uniform_paged_flash_b200", "csrc", "tg_kernels.cu")
    path = os.path.join(ROOT, "profiles", "decode_kernel_traffic.json")
    try:
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
        with open(path) as f:
            j = json.load(f)
        int4 = synth.preset(cfg).kind == "tiered" and SLOW_BITS == 4
        e = j.get(f"config{cfg}" + ("_int4" if int4 else ""))  # the INT4 slow tier moves other bytes
        if e and e.get("kernel_sha") == sha:
            if "traffic_over_algorithmic" in e and alg_per_launch is not None:
                return float(e["traffic_over_algorithmic"]) * float(alg_per_launch)
            if "traffic_bytes_per_launch" in e:
                return float(e["traffic_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed regions run."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "utilization.gpu")

    def __init__(self, gpu_index):
        self.gpu = str(gpu_index)
        self.proc = None
        self.lines = []
        self.reader = None

    def start(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        # the samples are kept in memory, read from the pipe by a thread
        self.reader = threading.Thread(target=lambda: self.lines.extend(self.proc.stdout), daemon=True)
        self.reader.start()

    @staticmethod
    def _when(stamp):
        """nvidia-smi's local timestamp ("YYYY/MM/DD HH:MM:SS.mmm") as seconds since the epoch."""
        import datetime
        try:
            return datetime.datetime.strptime(stamp.strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def stop(self, windows=()):
        """Summary of the samples. With windows [(t0, t1), ...] (time.time() around the timed
        regions), the SM clock median is taken over the samples inside them, else over the
        samples that saw the GPU busy, else over all; throttle reasons over the same set."""
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.reader is not None:
            self.reader.join(timeout=5)
        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in list(self.lines):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 11:
                continue
            try:
                rows.append({"t": self._when(parts[0]), "sm": float(parts[2]), "max": float(parts[3]),
                             "reasons": {n for n, v in zip(names, parts[6:10]) if v.lower() == "active"},
                             "util": float(parts[10]) if parts[10].replace(".", "", 1).isdigit() else 0.0})
            except ValueError:
                continue
        if not rows:
            return None
        inside = [r for r in rows if r["t"] is not None and
                  any(t0 - 0.05 <= r["t"] <= t1 + 0.05 for t0, t1 in windows)]
        busy = [r for r in rows if r["util"] >= 50.0]
        used, basis = (inside, "samples inside the timed regions") if inside else (
            (busy, "samples with the GPU busy") if busy else (rows, "all samples"))
        reasons = set().union(*(r["reasons"] for r in used))
        return {"sm_mhz": statistics.median(r["sm"] for r in used), "sm_max_mhz": rows[-1]["max"],
                "reasons": sorted(reasons), "samples": len(used), "samples_total": len(rows),
                "basis": basis}


# ------------------------------------------------------------------------------------------
# Reference arm: the CPU oracle, as it stands, on bounded samples of the same workload.
# ------------------------------------------------------------------------------------------

def run_reference(args):
    rank = _env_int("RANK", 0)
    if rank != 0:
        return 0
    import oracle
    from oracle import workload as ow
    cfg = args.config
    sp = _preset(cfg)
    o = ow.layout(sp, 0)
    q = ow.q_bits(sp)
    G = sp.Hq // sp.Hkv
    # Each step: the query rows of one sequence (round-robin over the batch).
    if o.fast_len is None:
        k = synth.pool_bits(sp, "k", o.num_pages)
        v = synth.pool_bits(sp, "v", o.num_pages)

        def step(b):
            sel = np.arange(b * sp.Hq, (b + 1) * sp.Hq)
            oracle.decode(q, k, v, o.table, o.head_off, o.kv_len, sp.scale, sel=sel)
            return int(o.kv_len[b].astype(np.int64).sum()) * 2 * sp.D * 2
    else:
        k = synth.pool_bits(sp, "k", o.num_pages)
        v = synth.pool_bits(sp, "v", o.num_pages)
        kq, ks, vq, vs = ow.slow_tier(sp, o)            # INT8, or INT4 codes widened to int8
        cb = sp.D // 2 if sp.slow_bits == 4 else sp.D  # stored code bytes per slow token-head

        def step(b):
            # one KV head of one sequence per step (bounded: the heads are 131072 tokens)
            h = b % sp.Hkv
            bb = (b // sp.Hkv) % sp.B
            sel = np.arange(bb * sp.Hq + h * G, bb * sp.Hq + (h + 1) * G)
            oracle.tiered_decode(q, kq, vq, ks, vs, o.slow_table, o.slow_off, k, v, o.table,
                                 o.head_off, o.kv_len, o.fast_len, sp.scale, sel=sel)
            n = int(o.kv_len[bb, h])
            f = min(int(o.fast_len[bb, h]), n)
            return (n - f) * 2 * (cb + 4) + f * 2 * sp.D * 2
    for i in range(args.warmup):
        step(i % sp.B)
    t0 = time.perf_counter()
    nbytes = 0
    for i in range(args.steps):
        nbytes += step(i % sp.B)
    dt = time.perf_counter() - t0
    value = nbytes / dt / 1e9
    cores = oracle.num_threads()
    sample = ("per step: all query rows of one sequence" if o.fast_len is None else
              "per step: the query rows of one (sequence, KV head)") + \
        (" of layer 0" if sp.layers > 1 else "") + f"; fp64 oracle over {cores} threads"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(cfg, _global_spec(cfg, _env_int("WORLD_SIZE", 1)),
                              _env_int("WORLD_SIZE", 1), min(args.layers, sp.layers)),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------
# Our arm
# ------------------------------------------------------------------------------------------

def cpu_baseline(cfg, budget_s=20.0, min_s=10.0, sample=None):
    """The oracle as it stands on a bounded sample of this workload (rank 0, N = 1). With a
    list `sample`, the first chunk's (row ids, (out, lse)) is appended to it, for the parity
    check of the bench line."""
    import oracle
    from oracle import workload as ow
    sp = _preset(cfg)
    o = ow.layout(sp, 0)
    q = ow.q_bits(sp)
    cores = oracle.num_threads()
    k = synth.pool_bits(sp, "k", o.num_pages)
    v = synth.pool_bits(sp, "v", o.num_pages)
    kv = o.kv_len.astype(np.int64)
    if o.fast_len is None:
        row_bytes = kv * 2 * sp.D * 2

        def rows(sel):
            return oracle.decode(q, k, v, o.table, o.head_off, o.kv_len, sp.scale, sel=sel)
    else:
        kq, ks, vq, vs = ow.slow_tier(sp, o)
        st = o.slow_table if o.slow_table.size else np.zeros(1, np.int32)
        f = np.minimum(o.fast_len.astype(np.int64), kv)
        cb = sp.D // 2 if sp.slow_bits == 4 else sp.D
        row_bytes = (kv - f) * 2 * (cb + 4) + f * 2 * sp.D * 2

        def rows(sel):
            return oracle.tiered_decode(q, kq, vq, ks, vs, st, o.slow_off, k, v, o.table,
                                        o.head_off, o.kv_len, o.fast_len, sp.scale, sel=sel)
    # passes over the batch, a few sequences at a time, until min_s of oracle time (or the
    # budget) is spent
    done, nbytes, t_used, passes = 0, 0, 0.0, 0
    chunk = max(1, sp.B // 16)
    while t_used < min_s and t_used < budget_s:
        b1 = min(sp.B, done + chunk)
        sel = np.arange(done * sp.Hq, b1 * sp.Hq)
        t0 = time.perf_counter()
        res = rows(sel)
        t_used += time.perf_counter() - t0
        if sample is not None and not sample:
            sample.append((sel, res))
        nbytes += int(row_bytes[done:b1].sum())
        done = b1
        if done == sp.B:
            done, passes = 0, passes + 1
    seqs = f"{passes} passes over all {sp.B} sequences" + (f" + sequences 0..{done - 1}" if done else "")
    return {"value": nbytes / t_used / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{seqs} (all their query rows), {t_used:.1f} s of fp64 oracle time on "
                      f"{cores} host threads"}


def _parity_sample(first, out, lse):
    """Max-abs differences of the timed step's outputs (layer 0; host copies out [rows, D],
    lse [rows]) from the fp64 oracle on the rows the CPU baseline computed (its first chunk of
    sequences, every query row of them)."""
    try:
        sel, (o_ref, l_ref) = first[0]
        out, lse = out[sel], lse[sel]
        fin = np.isfinite(l_ref)
        assert np.array_equal(fin, np.isfinite(lse)), "empty heads differ"
        return {"rows": int(len(sel)), "max_abs_out": float(np.abs(out - o_ref).max()),
                "max_abs_lse": float(np.abs(lse[fin] - l_ref[fin]).max()) if fin.any() else 0.0,
                "tolerance": {"out": 2e-2, "lse": 1e-3}}
    except Exception as e:   # the line is still printed; the failure is recorded in it
        return {"error": (type(e).__name__ + ": " + str(e))[:200]}


def _config(cfg, sp, world, n_layers):
    """The line's config dict (the same for both arms); sp is the global spec."""
    name = _workload_name(cfg, sp)
    c = {"workload": name, "config_id": cfg, "global_batch": int(sp.B),
         "parallelism": "sequence shards by AOT byte placement, no collective" if world > 1
         else "single GPU",
         "l2": "L2 flushed (252 MB written) between steps, outside the timed step" if cfg in (1, 4)
         else "inputs larger than L2 (K/V per step > 0.5 GB vs 126 MB L2); no flush"}
    if sp.layers > 1:
        c["workload"] = name + "; layers %d of %d, one resident at a time" % (n_layers, sp.layers)
        c["layers"] = n_layers
    return c


def _unique_kv_bytes(sp, lay):
    """K/V bytes of the distinct pages one step reads: a page referenced from r rows (a shared
    prefix page; always full) counts once instead of r times."""
    t = lay.table[lay.table >= 0]
    _, cnt = np.unique(t, return_counts=True)
    dup_tokens = int((cnt[cnt > 1].astype(np.int64) - 1).sum()) * sp.page
    return (int(lay.kv_len.astype(np.int64).sum()) - dup_tokens) * 2 * sp.D * 2


def _l2_profile(cfg):
    """L2 hit rate of the cascade kernel from a committed ncu capture, while the kernel source
    is unchanged since the capture; else None."""
    src = os.path.join(ROOT, "non_uniform_paged_flash_b200", "csrc", "tg_kernels.cu")
    path = os.path.join(ROOT, "profiles", "decode_kernel_traffic.json")
    try:
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
        with open(path) as f:
            e = json.load(f).get(f"config{cfg}")
        if e and e.get("kernel_sha") == sha and "l2_hit_rate" in e:
            return float(e["l2_hit_rate"])
    except Exception:
        pass
    return None


def _measure_layer(args, cfg, sp, layer, rank, world, dist, local, stream, pools, keep):
    """One layer of the workload made resident and measured: warm-up, then the timed steps
    (nothing instrumented), then a separate pass with the library's kernel events on (the
    per-kernel times of the roofline), then the end-to-end steps through the host-buffer call.
    Returns the layer's figures (host numbers only; device memory is released)."""
    import torch
    import non_uniform_paged_flash_b200 as tg
    from non_uniform_paged_flash_b200 import workload

    kv_all, fast_all = workload.retained(sp, layer)
    seqs = _my_sequences(sp, rank, world, kv_all, fast_all)
    lay = workload.layout(sp, layer, seqs)
    db = workload.to_device(sp, lay, layer, device=f"cuda:{local}", seqs=seqs, pools=pools,
                            **_plan_kw(cfg))
    info = tg.tg_plan_get_info(db.plan)
    alg = workload.algorithmic_bytes(sp, lay)

    # L2: inputs larger than twice L2 need no flush; smaller ones get a flush between steps.
    # Shared prefix pages count once (the K/V bytes of distinct pages): a step may reuse a page
    # in L2 across its readers, never across steps.
    uniq = _unique_kv_bytes(sp, lay)
    flush = None
    if uniq < 2 * L2_BYTES:
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=f"cuda:{local}")

    def barrier():
        if dist is not None:
            dist.barrier()

    def timed_steps(n, one):
        """Device time (ms) of n steps `one()` on the stream; with a flush, each step has its
        own event pair and the flush runs outside it."""
        if flush is None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n):
                one()
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for e0, e1 in evs:
            flush.zero_()
            e0.record(stream)
            one()
            e1.record(stream)
        torch.cuda.synchronize()
        return sum(e0.elapsed_time(e1) for e0, e1 in evs)

    for _ in range(args.warmup):
        if flush is not None:
            flush.zero_()
        db.run(stream)
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_OK, "device error word set during warm-up"

    # 1. the timed steps: the product path, nothing recorded inside it
    barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    ms_total = timed_steps(args.steps, lambda: db.run(stream))
    window = (t0, time.time())
    barrier()

    # 2. per-kernel times: the library's own events around the decode and merge launches, in a
    # separate pass (a recorded call gives up the merge kernel's launch overlap)
    n_ev = min(args.steps, 256)
    tg.tg_plan_timing_enable(db.plan, n_ev)
    for _ in range(n_ev):
        if flush is not None:
            flush.zero_()
        db.run(stream)
    n_rec, dec_ms, mrg_ms = tg.tg_plan_timing_read(db.plan)
    tg.tg_plan_timing_enable(db.plan, 0)
    status = tg.tg_plan_status(db.plan)

    # 3. end to end through the C-ABI host-buffer call: every step copies its pinned host q in
    # and its out + lse back to pinned host memory. The library's pipe double-buffers the device
    # staging, so a step's copies overlap its neighbours' decodes; the timed region runs from
    # before the first input copy to after the last output copy.
    q_host = db.q.cpu().pin_memory()
    out_host = torch.empty(db.out.shape, dtype=db.out.dtype).pin_memory()
    lse_host = torch.empty(db.lse.shape, dtype=db.lse.dtype).pin_memory()
    pipe = tg.HostPipe(db.plan)
    for _ in range(args.warmup):
        if flush is not None:
            flush.zero_()
        db.run_host(pipe, q_host, out_host, lse_host, stream)
    pipe.wait()
    barrier()
    torch.cuda.synchronize()

    def e2e_one():
        pipe.after(stream)
        db.run_host(pipe, q_host, out_host, lse_host, stream)
        pipe.join(stream)
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        pipe.after(stream)
        for _ in range(args.steps):
            db.run_host(pipe, q_host, out_host, lse_host, stream)
        pipe.join(stream)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
    else:
        e2e_ms = timed_steps(args.steps, e2e_one)   # no overlap: the flush sits between steps
    pipe.wait()
    assert torch.equal(out_host, db.out.cpu()), "host-buffer call differs from the device call"
    pipe.destroy()
    barrier()

    r = {"layer": layer, "ms_per_step": ms_total / args.steps, "e2e_ms_per_step": e2e_ms / args.steps,
         "decode_avg_ms": dec_ms / max(n_rec, 1), "merge_avg_ms": mrg_ms / max(n_rec, 1),
         "launches_timed": n_rec, "ok": status == tg.TG_OK, "kv_bytes": int(alg["kv"]),
         "algorithmic_bytes": int(alg["total"]), "batch": int(lay.kv_len.shape[0]),
         "launches_per_step": 1 + (1 if info["n_merge"] > 0 else 0) + (1 if info["n_cascade"] > 0 else 0),
         "plan": {k: info[k] for k in ("n_items", "n_partials", "n_merge", "n_workers", "grid",
                                       "stages", "smem_bytes", "n_cascade")},
         "h2d_bytes": int(db.q.numel() * db.q.element_size()),
         "d2h_bytes": int(db.out.numel() * db.out.element_size() + db.lse.numel() * db.lse.element_size()),
         "window": window}
    r["flushed"] = flush is not None
    if info["n_cascade"] > 0:
        r["unique_kv_bytes"] = uniq
    if keep:
        r["out"] = db.out.float().reshape(-1, sp.D).cpu().numpy()
        r["lse"] = db.lse.reshape(-1).cpu().numpy()
    if keep and cfg == 1:
        r["db"] = db        # the tiny workload also replays a CUDA graph of many copies
    else:
        db.plan.destroy()
        del db
        torch.cuda.empty_cache()
    return r


def run_ours(args):
    import torch
    from non_uniform_paged_flash_b200 import workload

    rank, world = _env_int("RANK", 0), _env_int("WORLD_SIZE", 1)
    local = _env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    cfg = args.config
    sp = _global_spec(cfg, world)
    n_layers = min(args.layers, sp.layers)
    stream = torch.cuda.current_stream()

    # A multi-layer workload keeps one pair of bf16 pools for all its layers (the pool bytes do
    # not depend on the layer; each layer's own tables decide what its heads read): sized for the
    # largest layer, uploaded once, outside any timed region.
    pools = None
    if n_layers > 1:
        most = 0
        for layer in range(n_layers):
            kv_all, fast_all = workload.retained(sp, layer)
            seqs = _my_sequences(sp, rank, world, kv_all, fast_all)
            most = max(most, workload.layout(sp, layer, seqs).num_pages)
        pools = workload.pools_to_device(sp, most, device=f"cuda:{local}")

    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    layers = [_measure_layer(args, cfg, sp, layer, rank, world, dist, local, stream, pools,
                             keep=(layer == 0 and rank == 0))
              for layer in range(n_layers)]
    clocks = sampler.stop([r["window"] for r in layers]) if sampler else None
    del pools

    # Max over ranks (times, error flag) and sums (work), per layer.
    vals = []
    for r in layers:
        vals += [r["ms_per_step"], r["e2e_ms_per_step"], r["decode_avg_ms"], r["merge_avg_ms"],
                 float(not r["ok"])]
    n_max = len(vals)
    for r in layers:
        vals += [float(r["kv_bytes"]), float(r["algorithmic_bytes"]), float(r["batch"])]
    vals = torch.tensor(vals, dtype=torch.float64, device=f"cuda:{local}")
    red = _over_ranks(dist, vals, n_max)
    mx, sm = red[:n_max], red[n_max:]
    per_layer = []
    for i, r in enumerate(layers):
        ms, e2e, dec, mrg, bad = mx[5 * i:5 * i + 5]
        kv, algb, b = sm[3 * i:3 * i + 3]
        per_layer.append({"layer": r["layer"], "ms_per_step": ms, "e2e_ms_per_step": e2e,
                          "decode_avg_ms": dec, "merge_avg_ms": mrg, "bad": bad > 0,
                          "kv_bytes": kv, "algorithmic_bytes": algb, "batch": b,
                          "frac_of_peak": None})

    if rank == 0:
        peak, peak_kind = _measured_peak()
        ms_sum = sum(r["ms_per_step"] for r in per_layer)
        e2e_sum = sum(r["e2e_ms_per_step"] for r in per_layer)
        kv_sum = sum(r["kv_bytes"] for r in per_layer)
        alg_sum = sum(r["algorithmic_bytes"] for r in per_layer)
        dec_sum = sum(r["decode_avg_ms"] for r in per_layer)
        for r in per_layer:
            r["frac_of_peak"] = r["algorithmic_bytes"] / (r["decode_avg_ms"] * 1e-3) / 1e9 / peak
        worst = min(per_layer, key=lambda r: r["frac_of_peak"])
        ms_step = ms_sum / n_layers
        achieved = alg_sum / (dec_sum * 1e-3) / 1e9
        b_total = per_layer[0]["batch"]
        first = layers[0]
        cascade = first["plan"]["n_cascade"] > 0
        launches = sum(args.steps * r["launches_per_step"] for r in layers)
        line = {
            "metric": METRIC, "value": kv_sum / (ms_sum * 1e-3) / 1e9, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if sp.kind != "tiered" else "bf16+int%d" % sp.slow_bits,
            "data": "synthetic",
            "config": _config(cfg, sp, world, n_layers),
            "tokens_per_s_per_layer": b_total / (ms_step * 1e-3),
            "kv_bytes_per_step": int(kv_sum / n_layers),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak,
                         "traffic": (_traffic(cfg, alg_sum / n_layers) if world == 1 else None),
                         "peak_kind": peak_kind,
                         "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                         "nominal_gbs": NOMINAL_HBM_GBS,
                         "kernel": "cascade_kernel + decode_kernel" if cascade else "decode_kernel",
                         "algorithmic_bytes_per_launch": alg_sum / n_layers,
                         "avg_launch_ms": dec_sum / n_layers,
                         "merge_avg_ms": sum(r["merge_avg_ms"] for r in per_layer) / n_layers,
                         "launches_timed": first["launches_timed"],
                         "timing": "decode-kernel events in a separate pass after the timed steps"},
            "e2e": {"value": kv_sum / (e2e_sum * 1e-3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": first["h2d_bytes"] * world,
                    "d2h_bytes_per_step": first["d2h_bytes"] * world,
                    "steps": args.steps,
                    "call": "tg_ragged_paged_decode_host" if sp.kind != "tiered"
                    else "tg_tiered_decode_host",
                    "overlap": "double-buffered staging; copies of neighbouring steps overlap"
                    if not first["flushed"] else "none (L2 flush between steps)"},
            "gpu_launches": launches,
            "plan": first["plan"],
            "device_status": "ok" if not any(r["bad"] for r in per_layer) else "error word set",
            "clocks": clocks,
        }
        if n_layers > 1:
            line["roofline"]["worst_layer"] = {"layer": worst["layer"], "frac": worst["frac_of_peak"]}
            line["per_layer"] = [{k: (round(v, 6) if isinstance(v, float) else v)
                                  for k, v in r.items() if k != "bad"} for r in per_layer]
        if cascade:
            uniq = first["unique_kv_bytes"] * world
            line["roofline"]["unique_kv_bytes_per_step"] = uniq
            line["roofline"]["frac_unique"] = uniq / (ms_step * 1e-3) / 1e9 / peak
            line["roofline"]["frac_logical"] = kv_sum / (ms_sum * 1e-3) / 1e9 / peak
            line["roofline"]["l2_hit_rate"] = _l2_profile(cfg)
        if world == 1 and cfg == 1:
            line["graph_replay"] = graph_replay(first["db"], workload.algorithmic_bytes(sp, first["db"].lay))
        if world == 1 and not args.no_cpu_baseline:
            sample = []
            line["cpu_baseline"] = cpu_baseline(cfg, sample=sample)
            line["parity_sample"] = _parity_sample(sample, first["out"], first["lse"])
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def graph_replay(db, alg, copies=1024, reps=5):
    """The tiny ragged MHA step is launch-bound and L2-resident on its own. Here `copies`
    distinct copies of its inputs (q, K and V pools, outputs; together above L2) are decoded by
    one CUDA graph of `copies` decode calls on the same plan, replayed `reps` times; the
    figure is K/V bytes of all copies / replay time."""
    import torch
    import non_uniform_paged_flash_b200 as tg
    dev = db.q.device
    k = db.k.unsqueeze(0).repeat(copies, *([1] * db.k.dim()))
    v = db.v.unsqueeze(0).repeat(copies, *([1] * db.v.dim()))
    q = db.q.unsqueeze(0).repeat(copies, *([1] * db.q.dim()))
    out = torch.empty((copies,) + tuple(db.out.shape), dtype=db.out.dtype, device=dev)
    lse = torch.empty((copies,) + tuple(db.lse.shape), dtype=db.lse.dtype, device=dev)
    held = (k.numel() + v.numel() + q.numel() + out.numel()) * 2 + lse.numel() * 4
    s = torch.cuda.Stream(device=dev)

    def calls():
        for i in range(copies):
            tg.tg_ragged_paged_decode(db.plan, q[i], k[i], v[i], db.table, db.head_off, db.kv_len,
                                      db.group_of_head, db.spec.scale, out[i], lse[i], s)
    try:
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            calls()
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            calls()
        for _ in range(2):
            g.replay()
        s.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):
            e0.record(s)
            for _ in range(reps):
                g.replay()
            e1.record(s)
        s.synchronize()
        ms = e0.elapsed_time(e1) / (reps * copies)
        db.run()
        torch.cuda.synchronize()
        same = bool(torch.equal(out[0], db.out) and torch.equal(out[copies - 1], db.out))
        del g
    except Exception as e:   # reported, never silently replaced by another number
        return {"error": str(e).splitlines()[0][:200]}
    return {"copies": copies, "replays": reps, "bytes_held": int(held),
            "us_per_step": ms * 1e3, "kv_gbs": alg["kv"] / (ms * 1e-3) / 1e9,
            "launches_per_step": 1 + (1 if tg.tg_plan_get_info(db.plan)["n_merge"] > 0 else 0),
            "outputs_equal_single_call": same}


def run_write_path(args):
    """Decode step with the write path on one GPU: append one token per (sequence, KV head)
    into the full, fixed-budget heads, then the decode (+ merge); with --path h2o the decode
    also writes the token scores and the H2O update accumulates them and picks the next step's
    victims. Prints one JSON line with the step time and each kernel's time and bytes."""
    import torch
    import non_uniform_paged_flash_b200 as tg
    from non_uniform_paged_flash_b200 import workload

    if args.path == "ttkv":
        return run_tier_path(args)
    cfg = args.config
    sp = synth.preset(cfg)
    if sp.kind == "tiered":
        raise SystemExit("--path sink|h2o is built for the bf16 tier; use --path ttkv")
    lay = workload.layout(sp, 0)
    db = workload.to_device(sp, lay, 0, **_plan_kw(cfg))
    B, Hkv = lay.kv_len.shape
    G = sp.Hq // sp.Hkv
    dev = db.q.device
    stream = torch.cuda.current_stream()
    shape = tg.make_shape(B, sp.Hq, sp.Hkv, sp.D, lay.num_pages)
    it = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a, dtype=dt)).to(dev)
    budget = it(lay.kv_len, np.int32)
    k_new = workload._bf16_tensor(synth.new_kv_bits(sp, 0, "k"), dev)
    v_new = workload._bf16_tensor(synth.new_kv_bits(sp, 0, "v"), dev)
    slot_out = torch.empty(B * Hkv, dtype=torch.int32, device=dev)
    cursor = torch.zeros(B * Hkv, dtype=torch.int32, device=dev)
    slots = lay.table.size * 16
    L = synth.full_lengths(sp).astype(np.int64)
    recent = 64
    h2o = args.path == "h2o"
    if h2o:
        pos = np.full(slots, -1, np.int32)
        for bh, pp in enumerate(synth.retained_positions(sp, lay.kv_len, np.repeat(L, Hkv), recent)):
            o = int(lay.head_off.reshape(-1)[bh]) * 16
            pos[o:o + pp.size] = pp
        slot_pos = it(pos, np.int32)
        slot_score = it(synth.init_scores(sp, slots), np.float32)
        ts = torch.zeros((slots, G), dtype=torch.float32, device=dev)
        victim = torch.empty(B * Hkv, dtype=torch.int32, device=dev)
        n_pos = args.warmup + args.steps + 1
        positions = it(L[None, :] + np.arange(n_pos)[:, None], np.int32)  # [step][B]
        tg.tg_h2o_update(shape, recent, None, None, db.head_off, budget, db.kv_len, slot_pos,
                         slot_score, positions[0], victim)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    n_ev = min(args.steps, 256)
    marks = [[ev() for _ in range(5)] for _ in range(n_ev)]

    def step(i, m=None):
        if m: m[0].record(stream)
        if h2o:
            tg.tg_append_h2o(shape, k_new, v_new, db.k, db.v, db.table, db.head_off, budget,
                             db.kv_len, victim, slot_pos, slot_score, positions[i], slot_out, stream)
        else:
            tg.tg_append_sink_recent(shape, 4, k_new, v_new, db.k, db.v, db.table, db.head_off,
                                     budget, db.kv_len, cursor, slot_out, stream)
        if m: m[1].record(stream)
        if h2o:
            tg.tg_ragged_paged_decode_scores(db.plan, db.q, db.k, db.v, db.table, db.head_off,
                                             db.kv_len, db.group_of_head, sp.scale, db.out,
                                             db.lse, ts, stream)
        else:
            db.run(stream)
        if m: m[2].record(stream)
        if h2o:
            tg.tg_h2o_update(shape, recent, ts, db.lse, db.head_off, budget, db.kv_len, slot_pos,
                             slot_score, positions[i + 1], victim, stream)
        if m: m[3].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_OK
    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    e0, e1 = ev(), ev()
    e0.record(stream)
    for i in range(args.steps):
        step(args.warmup + i)
    e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms_step = e0.elapsed_time(e1) / args.steps
    for i in range(n_ev):                       # per-kernel times, separate (marked) steps
        step(args.warmup + i, marks[i])
    torch.cuda.synchronize()
    assert tg.tg_plan_status(db.plan) == tg.TG_OK
    avg = lambda a, b: statistics.mean(m[a].elapsed_time(m[b]) for m in marks)
    t_app, t_dec, t_upd = avg(0, 1), avg(1, 2), avg(2, 3)
    alg = workload.algorithmic_bytes(sp, lay)
    tokens = int(lay.kv_len.sum())
    app_bytes = B * Hkv * (4 * sp.D * 2 + 12 + (8 if h2o else 4))
    upd_bytes = tokens * (4 * G + 12) + B * Hkv * 16 if h2o else 0
    dec_bytes = alg["total"] + (tokens * 4 * G if h2o else 0)
    peak, peak_kind = _measured_peak()
    line = {
        "metric": "decode step with %s write path: step time" % ("H2O" if h2o else "sink+recent"),
        "value": ms_step * 1e3, "unit": "us", "higher_is_better": False, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup,
        "config": {"workload": WORKLOAD_NAMES[cfg], "config_id": cfg, "recent": recent if h2o else None,
                   "sink": None if h2o else 4},
        "kernels_us": {"append": t_app * 1e3, "decode+merge": t_dec * 1e3,
                       "h2o_update": t_upd * 1e3 if h2o else None},
        "bytes": {"append": app_bytes, "decode": dec_bytes, "h2o_update": upd_bytes},
        "achieved_gbs": {"append": app_bytes / (t_app * 1e-3) / 1e9,
                         "h2o_update": upd_bytes / (t_upd * 1e-3) / 1e9 if h2o else None},
        "peak_gbs": peak, "peak_kind": peak_kind, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_tier_path(args):
    """Tiered decode step with the tier write path on one GPU (config 5 shape): every step
    appends one token per (sequence, KV head) to the fast window, which moves its oldest token
    into the INT8 tier (quantised in the same launch), then the tiered decode (+ merge) runs
    from one capacity plan made for the reserved sizes. Prints one JSON line."""
    import torch
    import non_uniform_paged_flash_b200 as tg
    from non_uniform_paged_flash_b200 import workload

    cfg = 5
    sp = _preset(cfg)
    lay = workload.layout(sp, 0)
    kw = _plan_kw(cfg)
    db = workload.to_device(sp, lay, 0, **kw)
    B, Hkv = lay.kv_len.shape
    BH = B * Hkv
    dev = db.q.device
    stream = torch.cuda.current_stream()
    n0 = lay.kv_len.reshape(-1).astype(np.int64)
    f0 = lay.fast_len.reshape(-1).astype(np.int64)
    n_ev = min(args.steps, 256)
    extra = args.warmup + args.steps + n_ev + 1           # tokens every head gains in this run
    # INT8 tier with room to grow: each head's row keeps its pages and gets hp new ones
    old_rows = -(-(n0 - f0) // 16)
    hp = -(-int(((n0 - f0) % 16).max() + extra) // 16) + 1
    P_old = lay.num_slow_pages
    table, off = [], np.zeros(BH, np.int64)
    for bh in range(BH):
        o = int(lay.slow_off.reshape(-1)[bh])
        off[bh] = len(table)
        table += lay.slow_table[o:o + int(old_rows[bh])].tolist()
        table += list(range(P_old + bh * hp, P_old + (bh + 1) * hp))
    P_new = P_old + BH * hp
    it = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a, dtype=dt)).to(dev)
    stab, soff = it(table, np.int32), it(off.reshape(B, Hkv), np.int64)

    def grow(t, tail):
        g = torch.zeros((P_new,) + tuple(t.shape[1:]), dtype=t.dtype, device=dev)
        g[:P_old].copy_(t)
        return g
    kq, vq = grow(db.k_q8, 16), grow(db.v_q8, 16)
    ks, vs = grow(db.k_scale, 16), grow(db.v_scale, 16)
    db.k_q8 = db.v_q8 = db.k_scale = db.v_scale = None
    S = (old_rows + hp) * 16                               # reserved INT8 slots per head
    shape = tg.make_shape(B, sp.Hq, sp.Hkv, sp.D, lay.num_pages, P_new)
    plan = tg.tg_plan_create(shape, (f0 + S).reshape(B, Hkv), lay.group_of_head, lay.group_off,
                             fast_len=f0.reshape(B, Hkv), slow_table_len=len(table),
                             capacity=True, slow_bits=sp.slow_bits, **kw)
    append = tg.tg_tiered_append_int4 if sp.slow_bits == 4 else tg.tg_tiered_append
    fcap = it(f0, np.int32)
    scap = it(S, np.int32)
    kv_dev, fl_dev = it(n0, np.int32), it(f0, np.int32)
    moved = torch.empty(BH, dtype=torch.int32, device=dev)
    slot = torch.empty(BH, dtype=torch.int32, device=dev)
    k_new = workload._bf16_tensor(synth.new_kv_bits(sp, 0, "k"), dev)
    v_new = workload._bf16_tensor(synth.new_kv_bits(sp, 0, "v"), dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    marks = [[ev() for _ in range(3)] for _ in range(n_ev)]

    def step(m=None):
        if m: m[0].record(stream)
        append(shape, k_new, v_new, db.k, db.v, db.table, db.head_off, fcap, kq, vq,
               ks, vs, stab, soff, scap, kv_dev, fl_dev, moved, slot, stream)
        if m: m[1].record(stream)
        tg.tg_tiered_decode(plan, db.q, kq, vq, ks, vs, stab, soff, db.k, db.v, db.table,
                            db.head_off, kv_dev, fl_dev, sp.scale, db.out, db.lse, stream)
        if m: m[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert tg.tg_plan_status(plan) == tg.TG_OK
    assert (slot.cpu().numpy() >= 0).all() and (moved.cpu().numpy() >= 0).all()
    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    e0, e1 = ev(), ev()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms_step = e0.elapsed_time(e1) / args.steps
    for m in marks:
        step(m)
    torch.cuda.synchronize()
    assert tg.tg_plan_status(plan) == tg.TG_OK
    assert (moved.cpu().numpy() >= 0).all()
    t_app = statistics.mean(m[0].elapsed_time(m[1]) for m in marks)
    t_dec = statistics.mean(m[1].elapsed_time(m[2]) for m in marks)
    row = sp.D // 2 if sp.slow_bits == 4 else sp.D      # code bytes per slow token and tensor
    kv_bytes = float(((kv_dev.cpu().numpy() - fl_dev.cpu().numpy()).astype(np.int64) * 2 * (row + 4)).sum()
                     + fl_dev.cpu().numpy().astype(np.int64).sum() * 2 * sp.D * 2)
    peak, peak_kind = _measured_peak()
    line = {
        "metric": "tiered decode step with tier migration: step time", "value": ms_step * 1e3,
        "unit": "us", "higher_is_better": False, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup,
        "config": {"workload": _workload_name(cfg, sp), "config_id": cfg, "plan": "capacity",
                   "slow_tier": "INT%d" % sp.slow_bits},
        "dtype": "bf16+int%d" % sp.slow_bits, "data": "synthetic",
        "kernels_us": {"tier_append": t_app * 1e3, "decode+merge": t_dec * 1e3},
        "kv_bytes_per_step": int(kv_bytes),
        "step_kv_gbs": kv_bytes / (ms_step * 1e-3) / 1e9, "peak_gbs": peak, "peak_kind": peak_kind,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_tier_host(args):
    """Tiered decode step with the INT8 tier in page-locked host memory (config 5 shape),
    streamed block-wise into an HBM ring while earlier blocks are decoded (TTKV's DRAM slow
    tier). The bound is the host link: the figure is INT8-tier bytes per step / step time,
    against a plain pinned host-to-device copy of the same size measured in the same run.
    Prints one JSON line."""
    import torch
    import non_uniform_paged_flash_b200 as tg
    from non_uniform_paged_flash_b200 import workload

    cfg = 5
    sp = _preset(cfg)
    lay = workload.layout(sp, 0)
    kw = _plan_kw(cfg)
    db = workload.to_device(sp, lay, 0, **kw)
    stream = torch.cuda.current_stream()
    db.run(stream)
    torch.cuda.synchronize()
    ref_out, ref_lse = db.out.clone(), db.lse.clone()
    host = db.host_slow_tier()
    slow_bytes = sum(t.numel() * t.element_size() for t in host)
    block_pages = args.block_pages
    ss = db.slow_stream(block_pages, 3, **{k: v for k, v in kw.items() if k != "early_prologue"})
    n_blocks = len(ss.blocks()[0])
    for _ in range(args.warmup):
        db.run_streamed(ss, host, stream)
    torch.cuda.synchronize()
    assert ss.status() == tg.TG_OK
    e_out = (db.out.float() - ref_out.float()).abs().max().item()
    e_lse = (db.lse - ref_lse).abs().max().item()
    # the host link alone: one pinned copy of the same bytes
    dst = torch.empty(slow_bytes, dtype=torch.uint8, device=db.q.device)
    src = torch.empty(slow_bytes, dtype=torch.uint8).pin_memory()
    link = []
    for _ in range(3):
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(stream)
        dst.copy_(src, non_blocking=True)
        b_.record(stream)
        torch.cuda.synchronize()
        link.append(slow_bytes / (a_.elapsed_time(b_) * 1e-3) / 1e9)
    del dst, src
    reps = max(1, min(args.steps, 20))
    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        db.run_streamed(ss, host, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / reps
    peak_link = max(link)
    achieved = slow_bytes / (ms * 1e-3) / 1e9
    alg = workload.algorithmic_bytes(sp, lay)
    line = {
        "metric": "tiered decode step, slow tier streamed from host memory (GB/s of slow tier)",
        "value": achieved, "unit": "GB/s", "higher_is_better": True, "n_gpus": 1, "steps": reps,
        "warmup": args.warmup, "ms_per_step": ms, "dtype": "bf16+int%d" % sp.slow_bits,
        "data": "synthetic",
        "config": {"workload": _workload_name(cfg, sp) + "; INT%d tier in pinned host memory" % sp.slow_bits,
                   "block_pages": block_pages, "ring_blocks": 3, "blocks_per_step": n_blocks},
        "host_tier_bytes_per_step": slow_bytes, "kv_bytes_per_step": int(alg["kv"]),
        "roofline": {"bound": "host link", "achieved": achieved, "peak": peak_link,
                     "unit": "GB/s", "frac": achieved / peak_link,
                     "peak_kind": "pinned host-to-device copy of the same bytes, this run"},
        "vs_hbm_tiered_step": {"max_abs_out": e_out, "max_abs_lse": e_lse},
        "gpu_launches": reps * (n_blocks * 2 + 3), "vs_baseline": None, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    ss.destroy()
    return 0


def run_splitzip(args):
    """SplitZip codec throughput on one GPU: the K and V pools of the GQA decode workload
    (config 2 shape, bf16) encoded and decoded back, each timed with CUDA events over
    args.steps repetitions (the pools are larger than L2). Prints one JSON line."""
    import torch
    import non_uniform_paged_flash_b200 as tg
    from non_uniform_paged_flash_b200 import workload

    cfg = 2
    sp = synth.preset(cfg)
    lay = workload.layout(sp, 0)
    dev = torch.device("cuda:0")
    src = torch.cat([workload._pool_to_device(sp, w, lay.num_pages, dev).view(torch.int16).reshape(-1)
                     for w in ("k", "v")])
    n = src.numel()
    cb = torch.empty(16, dtype=torch.uint8, device=dev)
    sm = torch.empty(n, dtype=torch.uint8, device=dev)
    codes = torch.empty((n + 1) // 2, dtype=torch.uint8, device=dev)
    cap = n // 16
    pos = torch.empty(cap, dtype=torch.int64, device=dev)
    exp = torch.empty(cap, dtype=torch.uint8, device=dev)
    n_esc = torch.zeros(1, dtype=torch.int64, device=dev)
    ws = torch.empty(tg.tg_splitzip_workspace_bytes(n), dtype=torch.uint8, device=dev)
    dst = torch.empty_like(src)
    enc = lambda: tg.tg_splitzip_encode(n, src, cb, sm, codes, pos, exp, n_esc, ws)
    dec = lambda: tg.tg_splitzip_decode(n, cb, sm, codes, pos, exp, n_esc, dst)
    for _ in range(args.warmup):
        enc()
        dec()
    torch.cuda.synchronize()
    assert torch.equal(dst, src), "round trip"
    k = int(n_esc.item())
    reps = min(args.steps, 200)
    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.3)

    def timed(fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps
    t_enc, t_dec = timed(enc), timed(dec)
    clocks = sampler.stop()
    assert torch.equal(dst, src)
    peak, peak_kind = _measured_peak()
    in_bytes = 2 * n
    stream_bytes = 16 + n + (n + 1) // 2 + 9 * k
    line = {
        "metric": "SplitZip bf16 codec throughput (GB/s of bf16 input)", "value": in_bytes / (t_enc * 1e-3) / 1e9,
        "unit": "GB/s", "higher_is_better": True, "n_gpus": 1, "steps": reps, "warmup": args.warmup,
        "config": {"workload": "K and V pools of: " + WORKLOAD_NAMES[cfg], "elements": n},
        "encode_gbs": in_bytes / (t_enc * 1e-3) / 1e9, "decode_gbs": in_bytes / (t_dec * 1e-3) / 1e9,
        "encode_us": t_enc * 1e3, "decode_us": t_dec * 1e3, "escapes": k,
        "compression_ratio": in_bytes / stream_bytes,
        "hbm_bytes_per_element": {"encode": 5.5, "decode": 3.5},
        "hbm_achieved_gbs": {"encode": 5.5 * n / (t_enc * 1e-3) / 1e9, "decode": 3.5 * n / (t_dec * 1e-3) / 1e9},
        "peak_gbs": peak, "peak_kind": peak_kind, "clocks": clocks,
        "dtype": "bf16 bits", "data": "synthetic", "vs_baseline": None,
        # the explainer's own figures, on a GPU it does not name: context, not a target
        "pages_gbs": {"encode": 613, "decode": 2181},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=3, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--slow-bits", type=int, default=8, choices=[8, 4],
                    help="code width of the tiered workloads' slow tier (config 5, ttkv-host)")
    ap.add_argument("--block-pages", type=int, default=8192,
                    help="--path ttkv-host: INT8-tier pages per streamed block")
    ap.add_argument("--layers", type=int, default=32,
                    help="multi-layer workload (config 3): how many of its layers to measure, "
                         "each made resident in turn (default: all 32)")
    ap.add_argument("--path", default="decode",
                    choices=["decode", "sink", "h2o", "ttkv", "ttkv-host", "splitzip"],
                    help="decode: the decode step (default); sink / h2o: the decode step with "
                         "the write path; ttkv: the tiered step with tier migration (config 5); "
                         "ttkv-host: the tiered step with the INT8 tier streamed from host "
                         "memory (config 5); splitzip: the KV codec; one GPU, separate JSON line")
    args = ap.parse_args()
    global SLOW_BITS
    SLOW_BITS = args.slow_bits
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.path == "splitzip":
        return run_splitzip(args)
    if args.path == "ttkv-host":
        return run_tier_host(args)
    if args.layers < 1:
        ap.error("--layers must be >= 1")
    if args.path != "decode":
        return run_write_path(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
