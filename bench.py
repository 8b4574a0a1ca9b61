#!/usr/bin/env python
"""Decode-step benchmark: compact-KV decode attention on B200.

One step = for every layer: append one token per sequence with its keep bits
(fdms_append_evict: ring write, eviction, compaction) and run decode attention
for all query heads (fdms_decode_attn: one kernel of per-head CTA clusters for
calls with few heads, else a split kernel and a combine kernel). Inputs
are the seeded synthetic workloads of ``workloads`` (shapes of the FastDMS
announcement's benchmark: ctx 8192, Llama-3.2-1B / Qwen3-8B shapes, c = 1 or 8).

Metric: compact KV bytes read by decode per second over whole steps (GB/s),
with µs per step beside it. Bytes are exact: the cache counts the slots every
decode call reads (a K row and a V row each).

Timing: the W warm-up steps run eagerly; the K timed steps are one CUDA graph,
captured once and replayed once between a barrier + synchronize on both sides,
timed with CUDA events on the launching stream (max over ranks). A second graph
holds K rounds of the decode calls of every layer alone (decode changes nothing
in the cache); its event-timed duration over the number of calls is the
per-launch duration of the roofline. Every step (and every round) reads more
compact KV than the 126 MB L2 holds, so nothing is found in L2 from before.

N > 1 (torchrun): every rank runs its own sequences (the path shards by
sequence with no exchange); value = bytes of all ranks / max time.

--impl reference: the fp64 CPU oracle timed on this host's cores on a bounded
sample of the same workload (one layer, all sequences), same metric and unit.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wk  # noqa: E402

METRIC = "decode-attn µs/step and achieved HBM GB/s on compact KV (% of B200 peak)"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama1b_c8", choices=sorted(wk.WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="budget of the oracle's timed sample")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-ctas", type=int, default=0)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other workloads' decode calls in the default run")
    ap.add_argument("--layers", type=int, default=0,
                    help="run only the workload's first N layers (a smaller case for "
                         "profiling: one decode call's bytes do not depend on it)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "MEASURED_PEAKS.json hbm_gbs (measured)"
    return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (no MEASURED_PEAKS.json)"


def code_hash(path):
    """First 16 hex digits of the sha256 of a source file's code: // comments,
    trailing blanks and empty lines removed, so that comment edits keep it."""
    import hashlib
    import re
    lines = []
    for line in open(path, encoding="utf-8"):
        line = re.sub(r"//.*$", "", line.rstrip("\n")).rstrip()
        if line:
            lines.append(line)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()[:16]


def load_traffic(workload):
    """DRAM bytes of one decode call from the committed ncu summary, if it was
    taken on the decode sources as they are now; else None."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.txt")
    if not os.path.exists(p):
        return None, "no capture"
    src = os.path.join(ROOT, "compressed_decode_attention_fdms_b200", "csrc")
    now = [code_hash(os.path.join(src, f)) for f in ("fdms_decode.cu", "fdms_internal.cuh")]
    for line in open(p):
        f = line.split()
        if not f or f[0].startswith("#") or f[0] != workload:
            continue
        if f[2:4] == now:
            return float(f[1]), "ncu dram__bytes_read.sum + dram__bytes_write.sum per " \
                                "decode call, mean over the calls of two full steps of " \
                                "this workload, one-pass capture on these decode sources"
        return None, "decode kernels changed since the ncu capture"
    return None, "no capture for this workload"


def rank_workload(wl, rank, world):
    """The workload a rank runs: every rank its own sequences (replicas; the
    path has no exchange step), so rank r draws from seed + 7919 r."""
    return wk.scaled(wl, seed=wl.seed + 7919 * rank) if world > 1 else wl


def over_ranks(t_ms, nbytes, world, device):
    """Whole-job figures: the longest time over ranks and the bytes of all of
    them (every rank takes the same two collective steps, in the same order)."""
    if world <= 1:
        return float(t_ms), float(nbytes)
    import torch.distributed as dist
    t = torch.tensor([float(t_ms)], dtype=torch.float64, device=device)
    b = torch.tensor([float(nbytes)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    return float(t.item()), float(b.item())


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def config_dict(wl):
    return {
        "workload": wl.name, "batch": wl.batch, "layers": wl.layers, "q_heads": wl.q_heads,
        "kv_heads": wl.kv_heads, "head_dim": wl.head_dim, "kv_dtype": wl.kv_dtype,
        "ctx": list(wl.ctx_range) if wl.ctx_range else wl.ctx, "window": wl.window,
        "period": wl.period, "keep_rate": wl.rate if wl.rate is not None else list(wl.rate_range),
    }


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device: int, period_s=0.002):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[device]) if vis else device
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception as e:  # no NVML: report that, keep going
            self.error = str(e)
        self.period = period_s

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "note": "NVML unavailable: " + getattr(self, "error", "")}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples),
                "source": "NVML polled every 2 ms during the timed region"}


# ----------------------------------------------------------------- oracle leg
def to_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 CPU tensor -> uint16 bit patterns (what the oracle reads)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_decode_bytes(oc, wl, b, row):
    """K/V bytes a decode of sequence b of the oracle cache's layer 0 reads:
    store and ring slots, one K row and one V row each (per-block FP8: sealed
    slots in E4M3, the staged and ring slots in bf16, twice the row)."""
    r, n = int(oc.r[0, b]), int(oc.n[0, b])
    lens = np.count_nonzero(oc.keep[0, b, :r], axis=0)          # [Hkv]
    if wl.kv_dtype != "fp8_e4m3_block":
        return int(np.sum(lens) + (n - r) * wl.kv_heads) * row
    sealed = lens // 64 * 64
    return int(np.sum(sealed) * row + (np.sum(lens - sealed) + (n - r) * wl.kv_heads) * 2 * row)


def oracle_sample(wl, budget_s: float, min_steps=1, max_steps=None, warmup=0):
    """Time the fp64 oracle on one layer of the workload, all sequences.

    Returns (bytes per second, per-step seconds list, description). Bytes are the
    compact slots the oracle's decode reads (store + ring, K and V rows).
    """
    from threadpoolctl import threadpool_limits
    from oracle.cache import OracleCache

    layer = 0
    ctx = wk.context_lengths(wl)
    n_steps = max_steps if max_steps is not None else wl.steps
    oc = OracleCache(1, wl.batch, wl.q_heads, wl.kv_heads, wl.head_dim, wl.window, wl.period,
                     wl.kv_dtype, capacity=int(ctx.max()) + n_steps + warmup + 1)
    pre = wk.prefill_inputs(wl, layer)
    elt = 1 if wl.kv_dtype.startswith("fp8") else 2
    row = 2 * wl.head_dim * elt
    times, bytes_ = [], 0
    with threadpool_limits(limits=1):
        oc.append(0, pre["n_new"].numpy(), to_bits(pre["k"]), to_bits(pre["v"]),
                  pre["keep"].numpy())
        total_t = 0.0
        for step in range(warmup + n_steps):
            inp = wk.decode_inputs(wl, layer, step)
            q = to_bits(wk.decode_query(wl, layer, step))
            kb, vb, keep = to_bits(inp["k"]), to_bits(inp["v"]), inp["keep"].numpy()
            t0 = time.perf_counter()
            oc.append(0, inp["n_new"].numpy(), kb, vb, keep)
            for b in range(wl.batch):
                oc.attention(0, b, q[b])
            dt = time.perf_counter() - t0
            if step < warmup:
                continue
            bytes_ += sum(oracle_decode_bytes(oc, wl, b, row) for b in range(wl.batch))
            times.append(dt)
            total_t += dt
            if len(times) >= min_steps and total_t >= budget_s:
                break
    desc = (f"fp64 numpy oracle, layer 0 of {wl.layers}, all {wl.batch} sequences x "
            f"{wl.kv_heads} kv heads, {len(times)} decode steps (append + attention) "
            f"after a {int(ctx.max())}-token prefill; 1 thread")
    return bytes_ / sum(times), times, desc


def oracle_seq_worker(job):
    """Time the fp64 oracle on some sequences of layer 0, in a process of its
    own (one thread): prefill, then decode steps (append + attention) until
    the time budget is spent or `steps` are done. Returns (bytes, seconds,
    steps) of the timed steps."""
    name, seqs, steps, budget_s = job
    from threadpoolctl import threadpool_limits
    from oracle.cache import OracleCache
    torch.set_num_threads(1)
    wl = wk.get(name)
    ctx = wk.context_lengths(wl)
    elt = 1 if wl.kv_dtype.startswith("fp8") else 2
    row = 2 * wl.head_dim * elt
    with threadpool_limits(limits=1):
        ocs = {}
        for b in seqs:
            pre = wk.prefill_inputs(wl, 0, seqs=[b])
            oc = OracleCache(1, 1, wl.q_heads, wl.kv_heads, wl.head_dim, wl.window, wl.period,
                             wl.kv_dtype, capacity=int(ctx[b]) + steps + 1)
            n = int(ctx[b])
            oc.append(0, np.array([n]), to_bits(pre["k"][b:b + 1, :n]),
                      to_bits(pre["v"][b:b + 1, :n]), pre["keep"][b:b + 1, :n].numpy())
            ocs[b] = oc
        total, nbytes, done = 0.0, 0, 0
        for step in range(steps):
            inp = wk.decode_inputs(wl, 0, step)
            q = to_bits(wk.decode_query(wl, 0, step))
            kb, vb, keep = to_bits(inp["k"]), to_bits(inp["v"]), inp["keep"].numpy()
            t0 = time.perf_counter()
            for b in seqs:
                ocs[b].append(0, np.array([1]), kb[b:b + 1], vb[b:b + 1], keep[b:b + 1])
                ocs[b].attention(0, 0, q[b])
            total += time.perf_counter() - t0
            done += 1
            for b in seqs:
                oc = ocs[b]
                nbytes += oracle_decode_bytes(oc, wl, 0, row)
            if total >= budget_s:
                break
    return nbytes, total, done


def oracle_parallel(wl, budget_s, steps=None):
    """The fp64 oracle on this host's cores: one spawned process per group of
    sequences of layer 0 (as many processes as cores, at most one per
    sequence), all running at once; bytes of every process / the longest
    process time. Spawned, not forked: this process has a CUDA context."""
    import multiprocessing as mp
    cores = max(1, min(os.cpu_count() or 1, wl.batch))
    groups = [list(range(i, wl.batch, cores)) for i in range(cores)]
    n_steps = steps if steps is not None else wl.steps
    jobs = [(wl.name, g, n_steps, budget_s) for g in groups]
    with mp.get_context("spawn").Pool(cores) as pool:
        res = pool.map(oracle_seq_worker, jobs)
    nbytes = sum(r[0] for r in res)
    t = max(r[1] for r in res)
    done = min(r[2] for r in res)
    desc = (f"fp64 numpy oracle, layer 0 of {wl.layers}, all {wl.batch} sequences x "
            f"{wl.kv_heads} kv heads, {done}+ decode steps (append + attention) after the "
            f"prefill; {cores} processes of one thread each (host has {os.cpu_count()} cores)")
    return {"value": nbytes / t / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": desc, "seconds": t}


def run_reference(args, wl):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    cb = oracle_parallel(wl, budget_s=1e9, steps=args.warmup + args.steps)
    gbs = cb["value"]
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * cb["seconds"] / max(1, args.warmup + args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {**config_dict(wl), "step": "one layer, all sequences"},
        "cpu_baseline": cb,
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- native leg
def pool_blocks(wl, steps_total):
    """Blocks for the pool: worst case when it fits in 40 GB, else a bound
    from the keep rates with a 6-sigma margin per head."""
    ctx = wk.context_lengths(wl)
    elt = 1 if wl.kv_dtype.startswith("fp8") else 2
    block_bytes = 2 * 64 * wl.head_dim * elt
    n = ctx[None, :, None] + steps_total
    worst = int(np.sum(np.ceil(np.broadcast_to(n, (wl.layers, wl.batch, wl.kv_heads)) / 64)))
    if worst * block_bytes <= 40e9:
        return 0
    p = wk.keep_rates(wl)
    mean = n * p
    sd = np.sqrt(n * p * (1 - p))
    return int(np.sum(np.ceil(np.minimum(n, mean + 6 * sd + 64) / 64) + 1))


def measure(fd, args, wl, dev, local, world, K, W, KE, WE):
    """One workload on this rank: prefill, W warm-up steps, K timed steps (one
    CUDA graph), K rounds of decode calls alone (the per-launch duration), and
    KE end-to-end steps. Returns the figures (whole-job bytes over ranks)."""
    steps_total = W + K + WE + KE
    cfg = fd.make_config(wl.layers, wl.batch, wl.q_heads, wl.kv_heads, wl.head_dim, wl.window,
                         wl.period, wl.max_ctx + steps_total, pool_blocks(wl, steps_total),
                         wl.kv_dtype, 0.0, args.decode_ctas)
    stream = torch.cuda.Stream(dev)
    cache = fd.fdms_cache_create(cfg, local, stream)
    L, B = wl.layers, wl.batch
    elt = 1 if wl.kv_dtype.startswith("fp8") else 2
    row = 2 * wl.head_dim * elt
    qo_bytes = 2 * B * wl.q_heads * wl.head_dim * 2      # q read + out written, bf16

    # prefill, timed on the device, with the bytes the appends must move: keep
    # bits, the input rows they read (all of them for the FP8 scale pass of a
    # first append, else survivors and ring rows) and the rows, positions and
    # keep bytes they write
    def prefill_bytes(inp):
        n = inp["n_new"].to(torch.int64)
        res = torch.where(n - wl.window >= wl.period, n - wl.window, torch.zeros_like(n))
        pos = torch.arange(inp["max_new"], device=dev).view(1, -1, 1)
        surv = int(((inp["keep"] != 0) & (pos < res.view(-1, 1, 1))).sum())
        ring_rows = int((n - res).sum()) * wl.kv_heads
        in_row = 2 * wl.head_dim * 2                      # K + V, bf16
        read_rows = int(n.sum()) * wl.kv_heads if elt == 1 else surv + ring_rows
        return (int(n.sum()) * wl.kv_heads + read_rows * in_row
                + (surv + ring_rows) * row + surv * 4 + ring_rows)

    in_bytes = 2 * B * wl.max_ctx * wl.kv_heads * wl.head_dim * 2 * L
    pre_bytes, pre_ms = 0.0, 0.0
    if in_bytes <= 24e9:   # all layers' inputs fit: one graph, no launch gaps
        pre_how = "CUDA events around one graph of every layer's fdms_append_evict"
        with torch.cuda.stream(stream):
            pre_in = [wk.prefill_inputs(wl, layer, device=dev) for layer in range(L)]
            pre_bytes = float(sum(prefill_bytes(inp) for inp in pre_in))
        stream.synchronize()
        graph_pre = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(graph_pre, stream=stream):
                for layer, inp in enumerate(pre_in):
                    fd.fdms_append_evict(cache, layer, B, inp["n_new"], inp["max_new"], inp["k"],
                                         inp["v"], inp["keep"], stream=stream)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            graph_pre.replay()
            e1.record(stream)
        stream.synchronize()
        pre_ms = e0.elapsed_time(e1)
        del graph_pre, pre_in
    else:                  # one layer's inputs at a time, each append between events
        pre_how = "CUDA events around each layer's fdms_append_evict, inputs made between"
        for layer in range(L):
            with torch.cuda.stream(stream):
                inp = wk.prefill_inputs(wl, layer, device=dev)
                pre_bytes += prefill_bytes(inp)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fd.fdms_append_evict(cache, layer, B, inp["n_new"], inp["max_new"], inp["k"],
                                     inp["v"], inp["keep"], stream=stream)
                e1.record(stream)
            stream.synchronize()
            pre_ms += e0.elapsed_time(e1)
            del inp
    with torch.cuda.stream(stream):
        # decode inputs of the device-timed steps, resident in HBM before timing
        steps_in = [[wk.decode_inputs(wl, l, s, device=dev) for l in range(L)]
                    for s in range(W + K)]
        qs = [[wk.decode_query(wl, l, s, device=dev) for l in range(L)] for s in range(W + K)]
        outs = [torch.empty((B, wl.q_heads, wl.head_dim), dtype=torch.bfloat16, device=dev)
                for _ in range(L)]
    stream.synchronize()

    def step(s):
        for layer in range(L):
            inp = steps_in[s][layer]
            fd.fdms_append_evict(cache, layer, B, inp["n_new"], 1, inp["k"], inp["v"],
                                 inp["keep"], stream=stream)
            fd.fdms_decode_attn(cache, layer, B, qs[s][layer], outs[layer], stream=stream)

    with torch.cuda.stream(stream):
        for s in range(W):
            step(s)
    stream.synchronize()

    # (1) the K timed steps as one graph
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream, capture_error_mode="thread_local"):
        for s in range(K):
            step(W + s)
    # (2) decode launches alone (decode reads the cache and changes nothing in
    # it), K rounds over all layers: the per-launch duration of the roofline
    graph_dec = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_dec, stream=stream, capture_error_mode="thread_local"):
        for s in range(K):
            for layer in range(L):
                fd.fdms_decode_attn(cache, layer, B, qs[W + s][layer], outs[layer], stream=stream)

    def timed(g):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        st_a = fd.fdms_cache_stats(cache, stream)
        with torch.cuda.stream(stream):       # replay on the stream the events see
            a.record(stream)
            g.replay()
            b.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        st_b = fd.fdms_cache_stats(cache, stream)
        if st_b["error"]:
            raise RuntimeError(f"device error latched: {fd.status_string(st_b['error'])}")
        return (a.elapsed_time(b), st_b["bytes_decoded"] - st_a["bytes_decoded"],
                st_b["decode_calls"] - st_a["decode_calls"])

    with ClockSampler(local) as clk:
        elapsed_ms, kv_bytes, calls = timed(graph)
    assert calls == K * L, (calls, K * L)
    dec_ms_total, dec_bytes, dec_calls = timed(graph_dec)
    assert dec_calls == K * L
    dec_avg_ms = dec_ms_total / dec_calls
    per_launch_bytes = dec_bytes / dec_calls + qo_bytes

    # whole-job numbers: max time over ranks, bytes summed over ranks
    t_max, bytes_all = over_ranks(elapsed_ms, kv_bytes, world, dev)
    value = bytes_all / (t_max * 1e-3) / 1e9

    # ---- KV memory after prefill and every step so far (the pages' memory
    # table: compact store + ring against a dense cache of the same tokens)
    st = fd.fdms_cache_stats(cache, stream)
    dense_bf16 = st["tokens_appended"] * wl.kv_heads * 2 * wl.head_dim * 2
    memory = {"compact_gib": st["bytes_compact"] / 2**30,
              "dense_same_dtype_gib": st["bytes_dense_equiv"] / 2**30,
              "dense_bf16_gib": dense_bf16 / 2**30,
              "compression_same_dtype": st["bytes_dense_equiv"] / max(1, st["bytes_compact"]),
              "compression_vs_bf16": dense_bf16 / max(1, st["bytes_compact"]),
              "reserved_gib": st["bytes_reserved"] / 2**30,
              "tokens_per_seq": st["tokens_appended"] // max(1, wl.layers * wl.batch)}

    # ---- end to end through the public API with pinned host buffers
    e2e = None
    if KE > 0:
        e2e = run_e2e(fd, cache, wl, stream, dev, W + K, WE, KE, row)
        e2e["ms"], e2e["bytes"] = over_ranks(e2e["ms"], e2e["bytes"], world, dev)

    peak, peak_src = load_peaks()
    traffic, traffic_src = load_traffic(wl.name)
    achieved = per_launch_bytes / (dec_avg_ms * 1e-3) / 1e9
    res = {
        "value": value, "t_max": t_max, "kv_bytes": kv_bytes, "elapsed_ms": elapsed_ms,
        "clocks": clk.summary(), "memory": memory, "e2e": e2e, "cs": fd.decode_cluster_size(cache, B),
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "traffic": traffic, "traffic_source": traffic_src,
            "per_launch_bytes": per_launch_bytes, "launch_us": dec_avg_ms * 1e3,
            "launch_timing": f"CUDA events around one graph of {K * L} back-to-back "
                             "decode calls (all layers, K rounds); duration / calls",
            "peak_source": peak_src,
        },
        "prefill": {"tokens_per_seq": int(wl.max_ctx), "layers": L,
                    "us_per_layer": 1e3 * pre_ms / L, "gb_per_layer": pre_bytes / L / 1e9,
                    "achieved_gbs": pre_bytes / (pre_ms * 1e-3) / 1e9,
                    "frac": pre_bytes / (pre_ms * 1e-3) / 1e9 / peak,
                    "timing": pre_how + (" (1 launch per layer: a CTA per head)"
                                         if wl.kv_dtype == "fp8_e4m3_block"
                                         else " (4 launches per layer)")},
        "decode_share_of_step": dec_avg_ms * L * K / elapsed_ms,
    }
    del graph, graph_dec
    fd.fdms_cache_destroy(cache)
    return res


def decode_kernel_desc(cs):
    return (f"fdms_decode_attn (k_decode_split: one cluster of {cs} CTAs per (seq, kv head), "
            "merged through distributed shared memory)" if cs else
            "fdms_decode_attn (k_decode_plan: one tile plan over the grid, each shared head "
            "merged by the warp holding its last tile)")


# workloads reported next to the headline one in the default run (their decode
# call and step at a shorter run): the pages' other single-GPU workloads, the
# Qwen3-8B one under both FP8 scale readings (one scale pair per head; one per
# sealed 64-slot block)
EXTRA_WORKLOADS = ("qwen8b_c8_fp8", "qwen8b_c8_fp8_block", "llama1b_c1")


def run_native(args, wl):
    import compressed_decode_attention_fdms_b200 as fd

    world, rank, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = rank_workload(wl, rank, world)
    W, K = args.warmup, args.steps
    KE = 0 if args.no_e2e else args.e2e_steps
    WE = 0 if args.no_e2e else 3
    m = measure(fd, args, wl, dev, local, world, K, W, KE, WE)
    extras = {}
    if world == 1 and not args.no_extras and args.workload == "llama1b_c8":
        for name in EXTRA_WORKLOADS:
            x = measure(fd, args, wk.get(name), dev, local, world, min(K, 20), W, 0, 0)
            extras[name] = {
                "config": config_dict(wk.get(name)), "value": x["value"], "unit": "GB/s",
                "us_per_step": 1e3 * x["t_max"] / min(K, 20), "roofline": x["roofline"],
                "kernel": decode_kernel_desc(x["cs"]), "clocks": x["clocks"],
                "memory": x["memory"], "kv_gb_per_step": x["kv_bytes"] / min(K, 20) / 1e9}
    result = None
    if rank == 0:
        roof = dict(m["roofline"])
        roof["kernel"] = decode_kernel_desc(m["cs"])
        result = {
            "metric": METRIC, "value": m["value"], "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": m["t_max"] / K, "us_per_step": 1e3 * m["t_max"] / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {**config_dict(wl), "parallelism": f"replicas{world}" if world > 1 else "1gpu",
                       "l2": "inputs larger than L2: every step reads "
                             f"{m['kv_bytes'] / K / 1e6:.0f} MB of compact KV (L2 126 MB)",
                       "timing": "K steps in one CUDA graph; events around each decode call"},
            "roofline": roof,
            "clocks": m["clocks"],
            # per layer and step: the append kernel and the decode kernel
            "gpu_launches": K * wl.layers * 2,
            "prefill": m["prefill"],
            "kv_gb_per_step": m["kv_bytes"] / K / 1e9,
            "memory": m["memory"],
            "decode_share_of_step": m["decode_share_of_step"],
        }
        if extras:
            result["workloads"] = extras
        e2e = m["e2e"]
        if e2e:
            result["e2e"] = {"value": e2e["bytes"] / (e2e["ms"] * 1e-3) / 1e9, "unit": "GB/s",
                             "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                             "us_per_step": 1e3 * e2e["ms"] / KE, "steps": KE,
                             "path": "Python binding -> C ABI, eager calls per layer; one packed "
                                     "H2D of the step's inputs and one D2H of all outputs per "
                                     "step, on two copy streams with double-buffered device "
                                     "memory (the next step's inputs go up and the last step's "
                                     "outputs come down while a step computes)"}
        if not args.no_cpu_baseline and world == 1:
            # decode steps past the workload's own count so that the budget,
            # not the step count, ends the sample
            cb = oracle_parallel(wl, args.cpu_seconds, steps=4096)
            cb1 = oracle_sample(wl, args.cpu_seconds / 2)
            result["cpu_baseline"] = cb
            result["cpu_baseline_1thread"] = {"value": cb1[0] / 1e9, "unit": "GB/s", "cores": 1,
                                              "kind": "oracle", "sample": cb1[2]}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if result is not None:
        print(json.dumps(result), flush=True)
    return 0


def run_e2e(fd, cache, wl, stream, dev, s0, warm, steps, row):
    """Steps through the public API with host buffers: every step, one copy of
    all its inputs (every layer's new token, keep bits and query, packed in
    one pinned buffer) to the device, every layer's fdms_append_evict +
    fdms_decode_attn on views of that buffer, and one copy of every layer's
    output back to pinned host memory. The copies run on two copy streams into
    double-buffered device memory, so that step s + 1's inputs go up and step
    s's outputs come down while the compute stream runs a step (events order
    every buffer's reuse)."""
    L, B = wl.layers, wl.batch
    # packed layout of one step: per layer n_new, k, v, keep, q, 16-byte aligned
    shapes = [("n_new", torch.int32, (B,)),
              ("k", torch.bfloat16, (B, 1, wl.kv_heads, wl.head_dim)),
              ("v", torch.bfloat16, (B, 1, wl.kv_heads, wl.head_dim)),
              ("keep", torch.uint8, (B, 1, wl.kv_heads)),
              ("q", torch.bfloat16, (B, wl.q_heads, wl.head_dim))]
    layout, off = [], 0
    for layer in range(L):
        per = {}
        for name, dt, shp in shapes:
            n = int(np.prod(shp)) * torch.tensor([], dtype=dt).element_size()
            per[name] = (off, n, dt, shp)
            off += (n + 15) // 16 * 16
        layout.append(per)
    step_bytes = off
    host = []
    for s in range(s0, s0 + warm + steps):
        buf = torch.empty(step_bytes, dtype=torch.uint8).pin_memory()
        for layer in range(L):
            inp = wk.decode_inputs(wl, layer, s)
            src = {"n_new": inp["n_new"], "k": inp["k"], "v": inp["v"], "keep": inp["keep"],
                   "q": wk.decode_query(wl, layer, s)}
            for name, (o, n, dt, shp) in layout[layer].items():
                buf[o:o + n].view(dt).view(shp).copy_(src[name])
        host.append(buf)
    NB = 2   # device input and output buffers in flight
    dbufs = [torch.empty(step_bytes, dtype=torch.uint8, device=dev) for _ in range(NB)]
    views = [[{name: dbuf[o:o + n].view(dt).view(shp) for name, (o, n, dt, shp) in per.items()}
              for per in layout] for dbuf in dbufs]
    douts = [torch.empty((L, B, wl.q_heads, wl.head_dim), dtype=torch.bfloat16, device=dev)
             for _ in range(NB)]
    houts = [torch.empty_like(douts[0], device="cpu").pin_memory() for _ in range(NB)]
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    in_ready = [torch.cuda.Event() for _ in range(NB)]
    computed = [torch.cuda.Event() for _ in range(NB)]
    out_read = [torch.cuda.Event() for _ in range(NB)]

    def one(s):
        i = s % NB
        up.wait_event(computed[i])          # the step that last read dbufs[i] is done
        with torch.cuda.stream(up):
            dbufs[i].copy_(host[s], non_blocking=True)
        in_ready[i].record(up)
        stream.wait_event(in_ready[i])
        stream.wait_event(out_read[i])      # douts[i]'s last contents are on the host
        for layer in range(L):
            d = views[i][layer]
            fd.fdms_append_evict(cache, layer, B, d["n_new"], 1, d["k"], d["v"], d["keep"],
                                 stream=stream)
            fd.fdms_decode_attn(cache, layer, B, d["q"], douts[i][layer], stream=stream)
        computed[i].record(stream)
        down.wait_event(computed[i])
        with torch.cuda.stream(down):
            houts[i].copy_(douts[i], non_blocking=True)
        out_read[i].record(down)

    with torch.cuda.stream(stream):
        for s in range(warm):
            one(s)
    stream.synchronize()
    st0 = fd.fdms_cache_stats(cache, stream)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        t0.record(stream)
        up.wait_event(t0)
        for s in range(warm, warm + steps):
            one(s)
        for i in range(NB):
            stream.wait_event(out_read[i])   # the last outputs are on the host
        t1.record(stream)
    torch.cuda.synchronize()
    st1 = fd.fdms_cache_stats(cache, stream)
    return {"ms": t0.elapsed_time(t1), "bytes": st1["bytes_decoded"] - st0["bytes_decoded"],
            "h2d": step_bytes, "d2h": douts[0].numel() * douts[0].element_size()}


def main():
    args = parse_args()
    wl = wk.get(args.workload)
    if args.layers > 0:
        wl = wk.scaled(wl, layers=min(args.layers, wl.layers))
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_native(args, wl)


if __name__ == "__main__":
    sys.exit(main())
