"""Benchmark: sparse FP4-KV decode query-tokens/s and achieved HBM GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one decode token for every sequence of the batch through the whole
hot path: pack of the token pair that completes at this step (2:1 gated
compression, FP4 group quantisation, indexer-key append), then the CSA2
layer group (indexer scan + exact top-K on every Full/Reindex layer, sparse
attention over top-K + window on every layer).  The K timed steps are
captured into one CUDA graph and replayed once between barriers; the time is
taken with CUDA events on the launching stream, max over ranks.  Inputs are
seeded synthetic tensors shaped like the pages' workloads (no weights, no
datasets).  With N > 1 (torchrun) each rank decodes its own batch of
sequences (independent problems, no collective on the data path: weak
scaling).

--impl reference times the CPU oracle on the same workload and metric
(bounded per-step sample: one sequence) on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse FP4-KV decode query-tokens/s; achieved HBM GB/s vs 8 TB/s"
UNIT = "query-tokens/s"
FALLBACK_HBM_GBS = 6650.0
KERNELS = ("pack", "pack_commit", "index_scan", "index_scan_tc", "topk_select", "block_max",
           "copy_topk", "attn_t128", "attn_simt", "attn_merge")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--config", default="batch32x128k")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-clocks", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--hier", type=int, default=0,
                   help="hierarchical indexer: blocks kept (0 = off; the pages use 2048 of 8)")
    p.add_argument("--hier-block", type=int, default=8)
    p.add_argument("--no-extra", action="store_true",
                   help="skip the hierarchical-indexer side measurement")
    return p.parse_args()


def time_group(w, steps, warmup, hier_blocks, hier_block, dev):
    """Device ms per decode step of workload w's layer groups (no pack), K
    steps in one CUDA graph, a new query set per step: the 18-layer encoder
    stack (3 groups, each with its own cache)."""
    import torch
    from fp4_compressed_kv_b200 import kvc, synth
    cfg = kvc.config_for(w)
    L, B, H = w.layers, w.batch, w.heads
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    groups = []
    for gi in range(w.groups):
        inp = synth.make_inputs(w.scaled(seed=w.seed + 100 * gi), dev)
        cache = kvc.Cache(cfg, w.batch, w.entries, device=dev)
        kvc.pack(cfg, inp["tokens"], inp["gate"], inp["idx_k"], cache, status=st)
        del inp["tokens"]
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        groups.append((inp, cache))
    out = torch.empty(L, B, H, w.latent, device=dev)
    lse = torch.empty(L, B, H, device=dev)
    tk = torch.empty(L, B, w.topk, dtype=torch.int32, device=dev)
    ws = kvc.workspace(cfg, B, w.entries, device=dev, hier_blocks=hier_blocks,
                       hier_block=hier_block)
    # a new query set per step and group
    sets = [synth.make_step_inputs(w.scaled(seed=w.seed + 100 * gi), warmup + steps, dev)
            for gi in range(w.groups)]

    def step(s):
        for gi, (inp, cache) in enumerate(groups):
            x = sets[gi][s]
            kvc.layer_group_step(cfg, list(w.modes), x["q"], x["idx_q"], x["windows"],
                                 w.window, cache, out, tk, ws, lse=lse, status=st,
                                 hier_blocks=hier_blocks, hier_block=hier_block)

    for s in range(warmup):
        step(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for s in range(warmup, warmup + steps):
            step(s)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g.replay()  # untimed first launch (uploads the graph)
    torch.cuda.synchronize()
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    assert st.item() == 0
    ms = e0.elapsed_time(e1) / steps
    del g
    return ms


def time_index_fp4(w, steps, warmup, dev):
    """Device ms of one top-K call of workload w's shape with FP4 indexer keys
    (72-byte rows: seeded random E2M1 codes, UE4M3 scales between 2^-8 and 2^1)
    against the same call with int8 keys (random values)."""
    import torch
    from fp4_compressed_kv_b200 import kvc, synth
    g = synth.generator(dev, w.seed + 7)
    res = {}
    for fmt in (0, 1):
        cfg = kvc.config_for(w.scaled(idx_fmt=fmt))
        cache = kvc.Cache(cfg, w.batch, w.entries, device=dev)
        if fmt == 1:
            half = w.idx_dim // 2
            cache.idx_k[..., :half] = torch.randint(0, 256, cache.idx_k[..., :half].shape,
                                                    generator=g, device=dev, dtype=torch.uint8)
            cache.idx_k[..., half:] = torch.randint(0x20, 0x40, cache.idx_k[..., half:].shape,
                                                    generator=g, device=dev, dtype=torch.uint8)
        else:
            cache.idx_k.copy_(torch.randint(-127, 128, cache.idx_k.shape, generator=g,
                                            device=dev, dtype=torch.int8))
        cache.n_entries.fill_(w.entries)
        q = torch.randint(-127, 128, (w.batch, w.idx_dim), generator=g, device=dev,
                          dtype=torch.int8)
        tk = torch.empty(w.batch, w.topk, dtype=torch.int32, device=dev)
        ws = kvc.workspace(cfg, w.batch, w.entries, device=dev)
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        for _ in range(warmup):
            kvc.index_topk(cfg, q, cache, tk, ws, status=st)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            for _ in range(steps):
                kvc.index_topk(cfg, q, cache, tk, ws, status=st)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        gr.replay()  # untimed first launch (uploads the graph)
        torch.cuda.synchronize()
        e0.record()
        gr.replay()
        e1.record()
        torch.cuda.synchronize()
        del gr
        assert st.item() == 0, st.item()
        res["fp4_keys" if fmt else "int8_keys"] = round(e0.elapsed_time(e1) / steps, 4)
        del cache, ws
        torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------------------------- bytes
def record_unpadded(w):
    n_groups = -(-w.latent // w.group) + -(-w.rope // w.group)
    return w.dim // 2 + n_groups * (1 if w.scale_fmt == 1 else 4)


def act_bytes(w):
    return 2 if w.act == "bf16" else 4


def scan_bytes(w, n):
    """Algorithmic bytes of one indexer scan over n entries, one sequence."""
    return n * w.idx_dim + w.idx_dim


def attn_bytes(w):
    """Algorithmic bytes of one attention problem (one sequence, one layer)."""
    a = act_bytes(w)
    return (w.topk * record_unpadded(w) + w.window * w.dim * a + w.heads * w.dim * a
            + w.heads * w.latent * 4 + w.topk * 4)


def pack_bytes(w, entries):
    """Algorithmic bytes of packing `entries` entries (2 raw tokens each)."""
    return entries * (2 * w.dim * act_bytes(w) + record_unpadded(w) + 2 * w.idx_dim)


def step_bytes(w, n):
    heads = sum(1 for m in w.modes if m != 2)
    return w.batch * (pack_bytes(w, 1) + heads * scan_bytes(w, n) + w.layers * attn_bytes(w))


# ----------------------------------------------------------------------------- peaks / clocks
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, enabled=True):
        self.proc = None
        self.out = os.path.join("/tmp", f"kvc_clocks_{os.getpid()}.csv")
        self.gpu = gpu_index
        if enabled:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=open(self.out, "w"), stderr=subprocess.DEVNULL)
            except Exception:
                self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.out):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return None
        sm = sorted(r[0] for r in rows)
        loaded = [r for r in rows if r[0] >= 0.5 * max(sm)]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2]) if v == "Active"})
        med = float(np.median([r[0] for r in loaded]))
        return {"sm_mhz": med, "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


def traffic_for(kernel):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on
    the kernel source as it is now (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_traffic.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    for line in open(path):
        if "=" in line and not line.startswith("#"):
            k, v = line.split("=", 1)
            kv[k.strip()] = v.strip()
    src = os.path.join(ROOT, "fp4_compressed_kv_b200", "csrc", kv.get("source", ""))
    if not os.path.exists(src):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if h != kv.get("source_sha256_16"):
        return None
    return kv


def time_scoring(w, steps, warmup, batched, dev):
    """Device ms to score and select every Full/Reindex layer of workload w
    (their indexer queries known up front): one batched tensor-core pass, or
    one scan per layer."""
    import torch
    from fp4_compressed_kv_b200 import kvc, synth
    cfg = kvc.config_for(w)
    heads = [i for i, m in enumerate(w.modes) if m != synth.REUSE]
    g = synth.generator(dev, w.seed)
    cache = kvc.Cache(cfg, w.batch, w.entries, device=dev)
    cache.idx_k.copy_(torch.randint(-127, 128, cache.idx_k.shape, generator=g, device=dev,
                                    dtype=torch.int8))
    cache.n_entries.fill_(w.entries)
    q = torch.randint(-127, 128, (len(heads), w.batch, w.idx_dim), generator=g, device=dev,
                      dtype=torch.int8)
    tk = torch.empty(len(heads), w.batch, w.topk, dtype=torch.int32, device=dev)
    if batched:
        ws = kvc.workspace_batched(cfg, len(heads), w.batch, w.entries, device=dev)

        def step():
            kvc.index_topk_batched(cfg, q, cache, tk, ws)
    else:
        ws = kvc.workspace(cfg, w.batch, w.entries, device=dev)

        def step():
            for i in range(len(heads)):
                kvc.index_topk(cfg, q[i], cache, tk[i], ws)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        for _ in range(steps):
            step()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gr.replay()  # untimed first launch (uploads the graph)
    torch.cuda.synchronize()
    e0.record()
    gr.replay()
    e1.record()
    torch.cuda.synchronize()
    del gr
    return e0.elapsed_time(e1) / steps


def time_attention_window(w, steps, warmup, fp8, dev):
    """Device ms of one attention call of workload w's shape (every sequence,
    one layer) with the window in bf16 or in FP8."""
    import torch
    from fp4_compressed_kv_b200 import kvc, synth
    wx = w.scaled(context=2 * 32768)  # 32 x 32768 records: 318 MB, beyond L2
    cfg = kvc.config_for(wx)
    g = synth.generator(dev, 17)
    B, N = wx.batch, wx.entries
    cache = kvc.Cache(cfg, B, N, device=dev)
    gate = (torch.randn(wx.dim, generator=g, device=dev) / wx.dim ** 0.5).float()
    nt = synth.make_new_tokens(wx, 2 * N, dev)
    kvc.pack(cfg, nt["tokens"], gate, nt["idx_k"], cache)
    del nt
    out = torch.empty(B, wx.heads, wx.latent, device=dev)
    ws = kvc.workspace(cfg, B, N, device=dev)
    sets = []
    for _ in range(8):  # rotated: every call gathers a new selection
        tk = torch.sort(torch.stack([torch.randperm(N, generator=g, device=dev)[: wx.topk]
                                     for _ in range(B)]), 1).values.int().contiguous()
        q = torch.randn(B, wx.heads, wx.dim, generator=g, device=dev).to(wx.torch_dtype)
        win = torch.randn(B, wx.window, wx.dim, generator=g, device=dev).to(wx.torch_dtype)
        codes = torch.empty(win.shape, dtype=torch.uint8, device=dev)
        scales = torch.empty(win.shape[:-1], dtype=torch.float32, device=dev)
        kvc.pack_window_fp8(cfg, win, codes, scales)
        sets.append((tk, q, win, codes, scales))

    def step(s):
        tk, q, win, codes, scales = sets[s % len(sets)]
        if fp8:
            kvc.sparse_decode_attn_fp8win(cfg, q, cache, tk, codes, scales, wx.window, out, ws)
        else:
            kvc.sparse_decode_attn(cfg, q, cache, tk, win, wx.window, out, ws)
    for s in range(warmup):
        step(s)
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        for s in range(steps):
            step(s)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gr.replay()  # untimed first launch (uploads the graph)
    torch.cuda.synchronize()
    e0.record()
    gr.replay()
    e1.record()
    torch.cuda.synchronize()
    del gr
    return e0.elapsed_time(e1) / steps


# ----------------------------------------------------------------------------- oracle leg
def oracle_decode_sample(w, seconds, seed_shift=0):
    """Time the CPU oracle on single-sequence decode steps of workload w.
    Returns (steps, elapsed_s, description).  Setup (packing the prefix with the
    oracle) is not timed; each timed step packs one pair, then runs the layer
    group (scan + top-K per Full/Reindex layer, attention per layer)."""
    import torch

    import oracle
    from fp4_compressed_kv_b200 import synth
    ws = w.scaled(batch=1, seed=w.seed + seed_shift)
    T = ws.context
    inp = synth.make_inputs(ws, "cpu", with_tokens=False)
    cfg = oracle.make_cfg(ws.latent, ws.rope, ws.group, ws.scale_fmt, ws.idx_dim, ws.topk,
                          ws.window, ws.heads, ws.sm_scale)
    N = ws.entries
    cap = N + 4096
    rb = oracle.record_bytes(cfg)
    rec = np.zeros((1, cap, rb), np.uint8)
    ic = np.zeros((1, cap, ws.idx_dim), np.int8)
    ic[0, :N] = inp["idx_k"][0].numpy()
    # records: the oracle packs its own entries; only the ones a step can select
    # matter, but the sample packs a full contiguous prefix block so any index
    # is valid (entries beyond the packed block are packed lazily below).
    n = np.array([N], np.int32)
    g = torch.Generator().manual_seed(ws.seed + 99)
    gate = inp["gate"].numpy()
    q = inp["q"].float().numpy()
    iq = inp["idx_q"].numpy()
    win = inp["windows"].float().numpy()
    packed = np.zeros(cap, bool)

    def ensure(idx_rows):
        need = [int(j) for j in idx_rows if j >= 0 and not packed[j]]
        if not need:
            return
        toks = (torch.randn(len(need), 2, ws.dim, generator=g) ).to(ws.torch_dtype).float().numpy()
        for t, j in zip(toks, need):
            e = oracle.compress_pair(t[0], t[1], gate)
            rec[0, j] = oracle.quantize_entry(cfg, e)[0]
            packed[j] = True

    steps = 0
    t_start = time.perf_counter()
    timed = 0.0
    while timed < seconds or steps == 0:
        # one decode step: pack the completed pair, then the layer group
        t0 = time.perf_counter()
        newt = torch.randn(1, 2, ws.dim, generator=g).to(ws.torch_dtype).float().numpy()
        newk = torch.randint(-127, 128, (1, 1, ws.idx_dim), generator=g, dtype=torch.int8).numpy()
        if n[0] >= cap:
            n[0] = N
        oracle.pack(cfg, newt, gate, newk, rec, ic, n)
        packed[n[0] - 1] = True
        t1 = time.perf_counter()
        # the records a step may select must exist: pack them (untimed)
        tk_all = [oracle.index_topk(cfg, iq[l], ic, n) for l in range(ws.layers)
                  if ws.modes[l] != 2]
        for tk in tk_all:
            ensure(tk[0])
        t2 = time.perf_counter()
        oracle.group_step(cfg, list(ws.modes), q, iq, win, ws.window, rec, ic, n)
        t3 = time.perf_counter()
        timed += (t1 - t0) + (t3 - t2)
        steps += 1
        if time.perf_counter() - t_start > 10 * seconds:
            break
    desc = (f"{steps} single-sequence decode steps of {w.name} (N={N} entries, "
            f"{ws.layers} layer(s), 1 core, oracle C code)")
    return steps, timed, desc


def _oracle_worker(job):
    """One spawned process: single-sequence oracle decode steps of workload
    `name` for about `seconds` of timed work, on its own sequence draw."""
    name, seconds, shift = job
    os.environ.setdefault("OMP_NUM_THREADS", "1")
    import torch
    torch.set_num_threads(1)
    from fp4_compressed_kv_b200 import synth
    steps, secs, _ = oracle_decode_sample(synth.WORKLOADS[name], seconds, seed_shift=shift)
    return steps, secs


def oracle_multicore(w, seconds, procs):
    """The oracle on `procs` host cores at once: one spawned process per core,
    each decoding its own sequences (the sequences of a batch are
    independent), all running concurrently.  Returns the summed query-tokens/s
    and the per-process results."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")  # CUDA is live in this process: never fork
    with ctx.Pool(procs) as pool:
        res = pool.map(_oracle_worker, [(w.name, seconds, 1 + i) for i in range(procs)])
    rate = sum(s / t for s, t in res if t > 0)
    return rate, res


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- ours
def measure_decode(w, steps, warmup, dev, stream, hier=0, hier_block=8, clocks_gpu=None):
    """Decode steps of workload w on this rank: the context is packed on the
    device (untimed), then K steps -- each packs the token pair completed at
    that step and runs the layer group on that step's own queries, indexer
    queries and windows -- are captured into one CUDA graph and replayed
    once between barriers (CUDA events on the launching stream, max over
    ranks).  A second capture of the same steps with an event pair around
    every library launch gives per-kernel durations.  Returns the numbers
    and the state the end-to-end leg reuses."""
    import torch

    from fp4_compressed_kv_b200 import kvc, synth
    from fp4_compressed_kv_b200 import dist as kd
    cfg = kvc.config_for(w)
    B, L, H = w.batch, w.layers, w.heads
    N0 = w.entries
    cap = N0 + warmup + steps + 64
    inp = synth.make_inputs(w, dev)
    cache = kvc.Cache(cfg, B, cap, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    kvc.pack(cfg, inp["tokens"], inp["gate"], inp["idx_k"], cache, status=status)
    torch.cuda.synchronize()
    del inp["tokens"], inp["idx_k"]
    torch.cuda.empty_cache()
    gate = inp["gate"]
    nsteps = warmup + steps
    # every step decodes new queries (so a new top-K set) and new windows
    sets = synth.make_step_inputs(w, nsteps, dev)
    ws = kvc.workspace(cfg, B, cap, device=dev, hier_blocks=hier, hier_block=hier_block)
    out = torch.empty(L, B, H, w.latent, device=dev)
    lse = torch.empty(L, B, H, device=dev)
    topk = torch.empty(L, B, w.topk, dtype=torch.int32, device=dev)
    newp = synth.make_new_tokens(w, 2 * nsteps, dev)
    pair_tok = [newp["tokens"][:, 2 * s:2 * s + 2].contiguous() for s in range(nsteps)]
    pair_idx = [newp["idx_k"][:, s:s + 1].contiguous() for s in range(nsteps)]
    modes = list(w.modes)

    def step(s):
        x = sets[s]
        kvc.pack(cfg, pair_tok[s], gate, pair_idx[s], cache, status=status)
        kvc.layer_group_step(cfg, modes, x["q"], x["idx_q"], x["windows"], w.window, cache, out,
                             topk, ws, lse=lse, status=status, hier_blocks=hier,
                             hier_block=hier_block)

    for s in range(warmup):
        step(s)
    torch.cuda.synchronize()

    # ---- capture the K timed steps into one graph and replay it once
    launches0 = kvc.launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for s in range(warmup, nsteps):
            step(s)
    launches = kvc.launch_count() - launches0
    n_before = cache.n_entries.clone()
    # one untimed replay first (the graph's first launch also uploads it);
    # the timed replay then starts again from the same context lengths
    graph.replay()
    torch.cuda.synchronize()
    cache.n_entries.copy_(n_before)

    clocks = Clocks(clocks_gpu, enabled=clocks_gpu is not None)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    kd.barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    kd.barrier()
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1)
    assert status.item() == 0, f"device status {status.item()}"
    n_after = cache.n_entries.clone()
    assert torch.all(n_after - n_before == steps)
    del graph
    ms_max = kd.max_over_ranks(ms, device=dev)

    # ---- the same K steps again, from the same starting length, captured with
    # a pair of event nodes around every library kernel: per-kernel durations
    # (the event nodes themselves add time, so this replay is not the headline)
    cache.n_entries.copy_(n_before)
    kvc.trace_begin(16 * steps * max(1, L) + 16)
    graph2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph2, stream=stream):
        for s in range(warmup, nsteps):
            step(s)
    kvc.trace_end()
    cache.n_entries.copy_(n_before)
    graph2.replay()  # untimed: uploads the graph (its event nodes record again below)
    torch.cuda.synchronize()
    cache.n_entries.copy_(n_before)
    kd.barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    graph2.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    ms_traced = kd.max_over_ranks(ev0.elapsed_time(ev1), device=dev)
    del graph2

    kernels = {}
    for name in KERNELS:
        cnt, tot = kvc.trace_kernel(name)
        if cnt:
            kernels[name] = {"launches": cnt, "ms_total": round(tot, 4),
                             "us_avg": round(1e3 * tot / cnt, 2)}
    n_mean = N0 + warmup + (steps + 1) / 2.0  # entries visible during the timed steps
    return {"cfg": cfg, "cache": cache, "status": status, "ws": ws, "out": out, "lse": lse,
            "topk": topk, "gate": gate, "sets": sets, "newp": newp, "n_before": n_before,
            "ms_max": ms_max, "ms_traced": ms_traced, "kernels": kernels, "launches": launches,
            "clocks": clk, "n_mean": n_mean}


def kernel_bytes(w, n_mean):
    """Algorithmic bytes per launch of the kernels whose work has a byte count."""
    return {"index_scan": w.batch * scan_bytes(w, n_mean),
            "attn_t128": w.batch * attn_bytes(w),
            "attn_simt": w.batch * attn_bytes(w),
            "pack": w.batch * pack_bytes(w, 1)}


def rooflines(w, m, peak, peak_kind):
    """Per-kernel achieved GB/s and fraction of the peak, and the roofline
    object of the dominant kernel (largest total time)."""
    kernels = m["kernels"]
    per_launch = kernel_bytes(w, m["n_mean"])
    for name, k in kernels.items():
        if name in per_launch:
            gbs = per_launch[name] / (k["us_avg"] * 1e-6) / 1e9
            k["gbs"] = round(gbs, 1)
            k["frac"] = round(gbs / peak, 4)
    dominant = max(kernels, key=lambda k: kernels[k]["ms_total"])
    dom = kernels[dominant]
    achieved = per_launch.get(dominant, 0) / (dom["us_avg"] * 1e-6) / 1e9
    traffic = traffic_for(dominant)
    return {"kernel": dominant, "bound": "hbm", "achieved": round(achieved, 1),
            "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
            "peak_source": f"{peak_kind} hbm_gbs",
            "bytes_per_launch": int(per_launch.get(dominant, 0)),
            "traffic": (int(float(traffic["dram_bytes_per_launch"])) if traffic else None)}


def workload_line(w, m, steps, world, peak, peak_kind):
    """The measurement of one workload: throughput, step bandwidth, the
    dominant kernel's roofline, per-kernel times and the bytes resident per
    token of its cache."""
    from fp4_compressed_kv_b200 import dist as kd
    from fp4_compressed_kv_b200 import kvc
    ms_step = m["ms_max"] / steps
    sb = step_bytes(w, m["n_mean"])
    step_gbs = sb / (ms_step * 1e-3) / 1e9
    roof = rooflines(w, m, peak, peak_kind)
    cfg = m["cfg"]
    return {"value": round(kd.job_throughput(steps, w.batch, world, m["ms_max"]), 1),
            "unit": UNIT, "ms_per_step": round(ms_step, 4),
            "ms_per_step_traced": round(m["ms_traced"] / steps, 4),
            "hbm_gbs_step": round(step_gbs, 1), "step_frac_of_peak": round(step_gbs / peak, 4),
            "step_bytes": int(sb), "roofline": roof, "kernels": m["kernels"],
            "bytes_resident_per_token": {
                "unpadded": round(kvc.bytes_resident(cfg, w.entries, w.layers, False) / w.context, 2),
                "padded": round(kvc.bytes_resident(cfg, w.entries, w.layers, True) / w.context, 2)}}


def run_ours(args):
    import torch
    import torch.distributed as dist

    from fp4_compressed_kv_b200 import build, kvc, synth
    from fp4_compressed_kv_b200 import dist as kd

    rank, world, local = kd.world()
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    build.build()

    w0 = synth.WORKLOADS[args.config]
    w = kd.rank_workload(w0, rank)  # each rank decodes its own sequences
    B, L = w.batch, w.layers
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    peak, peak_kind = peaks()

    m = measure_decode(w, args.steps, args.warmup, dev, stream, args.hier, args.hier_block,
                       clocks_gpu=None if args.no_clocks else local)
    cfg, cache, status, ws = m["cfg"], m["cache"], m["status"], m["ws"]
    out, lse, topk, gate, n_before = m["out"], m["lse"], m["topk"], m["gate"], m["n_before"]
    modes = list(w.modes)
    line = workload_line(w, m, args.steps, world, peak, peak_kind)
    value, ms_max, launches, clk = line["value"], m["ms_max"], m["launches"], m["clocks"]
    heads_layers = sum(1 for x in modes if x != 2)

    # ---- pack throughput on fresh tokens (the batched workload's pack case)
    pack_info = None
    if w.pack_new:
        pk = synth.make_new_tokens(w, w.pack_new, dev, seed_offset=11)
        pcache = kvc.Cache(cfg, B, w.pack_new // 2, device=dev)
        for _ in range(3):
            pcache.n_entries.zero_()
            kvc.pack(cfg, pk["tokens"], gate, pk["idx_k"], pcache, status=status)
        torch.cuda.synchronize()
        reps = max(5, args.steps)
        kvc.trace_begin(4 * reps + 8)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            pcache.n_entries.zero_()
            kvc.pack(cfg, pk["tokens"], gate, pk["idx_k"], pcache, status=status)
        e1.record(stream)
        torch.cuda.synchronize()
        kvc.trace_end()
        pms = e0.elapsed_time(e1) / reps
        cnt, tot = kvc.trace_kernel("pack")
        kus = 1e3 * tot / cnt
        pbytes = pack_bytes(w, B * w.pack_new // 2)
        pack_info = {"new_tokens_per_seq": w.pack_new, "tokens_per_s": round(B * w.pack_new / (pms / 1e3)),
                     "ms_per_call": round(pms, 4), "kernel_us": round(kus, 2),
                     "kernel_gbs": round(pbytes / (kus * 1e-6) / 1e9, 1),
                     "kernel_frac": round(pbytes / (kus * 1e-6) / 1e9 / peak, 4),
                     "bytes_per_call": int(pbytes)}
        del pk, pcache

    # ---- end to end through the public API with host buffers.  Every step
    # uploads its own inputs (indexer queries, the completed token pair and
    # its indexer key, the query heads: a new set each step) from pinned host
    # memory and reads its result (the attention output and lse) back.
    # Within a step the queries (needed only by the attention) travel on a
    # copy stream while the pack, the scan and the selection run; the small
    # inputs go up in one copy and the result comes back in one.  Steps stay
    # serialised: a step starts after the previous one's result is read back.
    e2e = None
    if not args.no_e2e:
        def staged(parts, n_host=1):
            """n_host pinned host buffers and one device buffer, each holding
            tensors shaped like `parts` back to back (16-byte aligned); returns
            them and their views."""
            sizes = [(t.numel() * t.element_size() + 15) // 16 * 16 for t in parts]

            def views(buf):
                v, off = [], 0
                for t, n in zip(parts, sizes):
                    nb = t.numel() * t.element_size()
                    v.append(buf[off:off + nb].view(t.dtype).view(t.shape))
                    off += n
                return v
            hosts = [torch.empty(sum(sizes), dtype=torch.uint8).pin_memory()
                     for _ in range(n_host)]
            devb = torch.empty(sum(sizes), dtype=torch.uint8, device=dev)
            return hosts, devb, [views(h) for h in hosts], views(devb)

        reps = args.steps
        sets, newp = m["sets"], m["newp"]
        nsteps = args.warmup + args.steps
        step_ids = [args.warmup + (s % args.steps) for s in range(reps + 1)]
        hins, din, hviews, (diq, dtok, didx) = staged(
            [sets[0]["idx_q"], newp["tokens"][:, :2], newp["idx_k"][:, :1]], n_host=reps + 1)
        hqs = []
        for r, s in enumerate(step_ids):
            h_iq, h_tok, h_idx = hviews[r]
            h_iq.copy_(sets[s]["idx_q"])
            h_tok.copy_(newp["tokens"][:, 2 * s:2 * s + 2])
            h_idx.copy_(newp["idx_k"][:, s:s + 1])
            hqs.append(sets[s]["q"].cpu().pin_memory())
        dq = torch.empty_like(sets[0]["q"])
        (hres,), dres, ((h_out, h_lse),), (d_out, d_lse) = staged([out, lse])
        copy_stream = torch.cuda.Stream(device=dev)
        q_ready = torch.cuda.Event()
        split = modes == [synth.FULL] and args.hier == 0
        cache.n_entries.copy_(n_before)

        def e2e_step(r):
            windows = sets[step_ids[r]]["windows"]  # the windows stay on the device
            # the small inputs first: host-to-device copies run in order, and
            # the pack, scan and selection need only these
            din.copy_(hins[r], non_blocking=True)
            copy_stream.wait_stream(stream)  # the previous step no longer reads dq
            with torch.cuda.stream(copy_stream):
                dq.copy_(hqs[r], non_blocking=True)
                q_ready.record(copy_stream)
            kvc.pack(cfg, dtok, gate, didx, cache, status=status)
            if split:  # one Full layer: its scan and selection need no queries
                kvc.index_topk(cfg, diq[0], cache, topk[0], ws, status=status)
                stream.wait_event(q_ready)
                kvc.sparse_decode_attn(cfg, dq[0], cache, topk[0], windows[0], w.window, d_out[0],
                                       ws, lse=d_lse[0], status=status)
            else:
                stream.wait_event(q_ready)
                kvc.layer_group_step(cfg, modes, dq, diq, windows, w.window, cache, d_out, topk,
                                     ws, lse=d_lse, status=status, hier_blocks=args.hier,
                                     hier_block=args.hier_block)
            hres.copy_(dres, non_blocking=True)

        # warm-up: one pass over every step's pinned buffers (a first transfer
        # from a pinned buffer runs at a fraction of the link rate; a serving
        # loop reuses warm staging buffers), then the spare set
        for r in range(reps + 1):
            e2e_step(r)
            cache.n_entries.copy_(n_before)
        torch.cuda.synchronize()
        cache.n_entries.copy_(n_before)
        kd.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for r in range(reps):
            e2e_step(r)
        e1.record(stream)
        torch.cuda.synchronize()
        te_ms = kd.max_over_ranks(e0.elapsed_time(e1), device=dev)
        assert status.item() == 0, f"device status {status.item()}"
        h2d = (sum(t.numel() * t.element_size() for t in hviews[0])
               + hqs[0].numel() * hqs[0].element_size())
        d2h = sum(t.numel() * t.element_size() for t in (h_out, h_lse))
        e2e = {"value": round(kd.job_throughput(reps, B, world, te_ms), 1), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(te_ms / reps, 4),
               "inputs": "a new query set uploaded every step (each step's pinned buffer used once in the warm-up)",
               "api": ("kvc_pack, kvc_index_topk, kvc_sparse_decode_attn" if split else
                       "kvc_pack, kvc_layer_group_step"),
               "overlap": "small inputs first, then the query upload on a copy stream during pack, scan and selection"
                          if split else "none"}
        del hins, hqs

    # ---- the CSA2 group (8 x 256K, Full/Reindex/Reuse/Reuse) and the 1M-token
    # 20-layer stack measured like the headline (pack + layer group, a new
    # query set per step), and again with the hierarchical indexer (2048
    # blocks of 8)
    extra, workloads = None, None
    if not args.no_extra and world == 1 and args.hier == 0:
        del m
        torch.cuda.empty_cache()
        extra, workloads = {}, {}
        for name in ("csa2group", "stack1m"):
            wx = synth.WORKLOADS[name]
            mx = measure_decode(wx, 10, 3, dev, stream)
            lx = workload_line(wx, mx, 10, 1, peak, peak_kind)
            lx["steps"], lx["warmup"] = 10, 3
            lx["config"] = {"batch": wx.batch, "context_tokens": wx.context,
                            "entries": wx.entries, "group": wx.group,
                            "layers": [["Full", "Reindex", "Reuse"][x] for x in wx.modes]}
            del mx
            torch.cuda.empty_cache()
            mh = measure_decode(wx, 10, 3, dev, stream, 2048, 8)
            lx["hier_indexer_2048x8"] = {
                "value": round(kd.job_throughput(10, wx.batch, 1, mh["ms_max"]), 1),
                "ms_per_step": round(mh["ms_max"] / 10, 4)}
            del mh
            torch.cuda.empty_cache()
            workloads[name] = lx
            extra[name] = {}
        # every scoring layer's indexer query in one tensor-core pass, against
        # one scan per layer (a schedule where all queries are known up front)
        for name in ("csa2group", "stack1m"):
            wx = synth.WORKLOADS[name]
            one = time_scoring(wx, 10, 3, False, dev)
            bat = time_scoring(wx, 10, 3, True, dev)
            extra[name].update({"scoring_ms_per_layer_scans": round(one, 4),
                                "scoring_ms_batched_tensor_core": round(bat, 4)})
            torch.cuda.empty_cache()
        # the 18-layer encoder stack at 1M tokens: 3 groups (Full + 5 Reuse),
        # each with its own cache
        wx = synth.WORKLOADS["encoder1m"]
        enc = time_group(wx, 10, 3, 0, 8, dev)
        extra["encoder1m"] = {"ms_per_step": round(enc, 4),
                              "query_tokens_per_s": round(wx.batch / (enc * 1e-3), 1),
                              "layers": wx.groups * wx.layers,
                              "groups": "3 x (Full + 5 Reuse), own cache each"}
        torch.cuda.empty_cache()
        # the attention of this workload with the window in bf16 and in FP8
        extra["fp8_window"] = {
            "workload": w0.name,
            "attention_ms_bf16_window": round(time_attention_window(w0, 20, 3, False, dev), 4),
            "attention_ms_fp8_window": round(time_attention_window(w0, 20, 3, True, dev), 4)}
        torch.cuda.empty_cache()
        # the top-K call with FP4 indexer keys (72-byte rows) against int8 keys;
        # last, and recorded as an error string if it fails
        try:
            extra["fp4_indexer_keys"] = {"workload": w0.name,
                                         "index_topk_ms": time_index_fp4(w0, 20, 3, dev),
                                         "row_bytes": {"int8_keys": w0.idx_dim,
                                                       "fp4_keys": w0.idx_dim // 2 +
                                                       w0.idx_dim // 16}}
            torch.cuda.empty_cache()
        except Exception as e:  # a side measurement must not cost the headline line
            extra["fp4_indexer_keys"] = {"error": str(e)[:200]}

    # ---- CPU oracle baseline (rank 0, N=1 only): one process per host core
    # (up to 32), each decoding its own sequences concurrently, beside the
    # single-core figure
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        steps_c, secs, desc = oracle_decode_sample(w0, args.cpu_seconds / 2)
        single = round(steps_c / secs, 3)
        procs = max(1, min(32, host_cores()))
        try:
            rate, res = oracle_multicore(w0, args.cpu_seconds / 2, procs)
            cpu = {"value": round(rate, 3), "unit": UNIT, "cores": procs, "kind": "oracle",
                   "sample": (f"{sum(r[0] for r in res)} single-sequence decode steps of "
                              f"{w0.name} on {procs} processes (one per core, its own "
                              f"sequences; about {args.cpu_seconds / 2:.0f} s each), oracle C "
                              f"code"),
                   "host_cores": host_cores(),
                   "single_core": {"value": single, "sample": desc}}
        except Exception as e:  # the pool must not cost the headline line
            cpu = {"value": single, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc,
                   "multicore_error": str(e)[:200]}
        # the same two oracle legs for the CSA2 group and the 1M-token stack
        # (shorter samples: one 1M-token step takes about a second on one core)
        for name in (workloads or {}):
            wx = synth.WORKLOADS[name]
            secs_x = args.cpu_seconds / 4
            try:
                sx, tx, dx = oracle_decode_sample(wx, secs_x)
                rate_x, res_x = oracle_multicore(wx, secs_x, procs)
                workloads[name]["cpu_baseline"] = {
                    "value": round(rate_x, 3), "unit": UNIT, "cores": procs, "kind": "oracle",
                    "sample": (f"{sum(r[0] for r in res_x)} single-sequence decode steps of "
                               f"{wx.name} on {procs} processes (one per core, its own "
                               f"sequences; about {secs_x:.0f} s each), oracle C code"),
                    "single_core": {"value": round(sx / tx, 3), "sample": dx}}
            except Exception as e:  # a side measurement must not cost the headline line
                workloads[name]["cpu_baseline"] = {"error": str(e)[:200]}

    res = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 4),
        "ms_per_step_traced": line["ms_per_step_traced"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.act == "bf16" else "f32",
        "data": "synthetic (seeded; no weights or datasets)",
        "config": {"workload": w.name, "batch_per_gpu": B, "context_tokens": w.context,
                   "entries": w.entries, "layers": [["Full", "Reindex", "Reuse"][x] for x in modes],
                   "heads": w.heads, "latent": w.latent, "rope": w.rope, "group": w.group,
                   "scale": "ue4m3" if w.scale_fmt == 1 else "f32", "topk": w.topk,
                   "window": w.window, "idx_dim": w.idx_dim, "parallelism": f"dp{world}",
                   "hier_indexer": (f"{args.hier} blocks of {args.hier_block}" if args.hier
                                    else "off"),
                   "inputs": "a new set of queries, indexer queries and windows every step",
                   "l2": "inputs larger than L2 (indexer scan reads %.0f MB per step)"
                         % (B * scan_bytes(w, w.entries) * heads_layers / 1e6),
                   "timing": "K steps in one CUDA graph, CUDA events, max over ranks; "
                             "per-kernel times from a second replay with event nodes"},
        "hbm_gbs_step": line["hbm_gbs_step"],
        "step_frac_of_peak": line["step_frac_of_peak"],
        "step_bytes": line["step_bytes"],
        "roofline": line["roofline"],
        "kernels": line["kernels"],
        "pack": pack_info,
        "bytes_resident_per_token": line["bytes_resident_per_token"],
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clk,
        "workloads": workloads,
        "next_rows": extra,
    }
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        kd.barrier()
        dist.destroy_process_group()


def run_reference(args):
    from fp4_compressed_kv_b200 import synth
    from fp4_compressed_kv_b200 import dist as kd
    rank, world, _ = kd.world()
    if rank != 0:
        return
    w = synth.WORKLOADS[args.config]
    # warm-up samples, then K timed samples of one single-sequence step each
    oracle_decode_sample(w, 0.0)
    total_steps, total_s = 0, 0.0
    for k in range(args.steps):
        s, secs, desc = oracle_decode_sample(w, 0.0, seed_shift=k + 1)
        total_steps += s
        total_s += secs
    v = total_steps / total_s
    res = {"metric": METRIC, "value": round(v, 3), "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total_s / total_steps, 2),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded; no weights or datasets)", "impl": "reference",
           "config": {"workload": w.name, "batch_per_gpu": w.batch, "context_tokens": w.context,
                      "entries": w.entries, "sample": "one sequence per step"},
           "cpu_baseline": {"value": round(v, 3), "unit": UNIT, "cores": 1, "kind": "oracle",
                            "sample": desc},
           "e2e": {"value": round(v, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)
