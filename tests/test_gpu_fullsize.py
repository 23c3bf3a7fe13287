"""Parity at the workloads' full sizes, through kvc_layer_group_step as the
benchmark calls it.

The cache is built by the GPU pack of the whole context (device-generated raw
tokens).  The oracle never sees a value our kernels produced: it re-packs
sampled entries from the same raw tokens (copied to the host) and compares
records byte for byte; it recomputes every sequence's indexer scores and top-K
from the raw int8 keys and queries (bit-exact); and it recomputes attention for
sampled sequences and layers from its own packed records of the selected
entries, the raw window and the query (within 2e-3 x row norm).
"""
import numpy as np
import pytest
import torch

import oracle
from fp4_compressed_kv_b200 import synth
from helpers import assert_attn_close, f32, oracle_cfg

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _run_group(kvc, w):
    dev = torch.device("cuda")
    inp = synth.make_inputs(w, dev)
    cfg = kvc.config_for(w)
    cache = kvc.Cache(cfg, w.batch, w.entries, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    kvc.pack(cfg, inp["tokens"], inp["gate"], inp["idx_k"], cache, status=st)
    L, B, H = w.layers, w.batch, w.heads
    out = torch.empty(L, B, H, w.latent, device=dev)
    lse = torch.empty(L, B, H, device=dev)
    tk = torch.empty(L, B, w.topk, dtype=torch.int32, device=dev)
    ws = kvc.workspace(cfg, B, cache.capacity, device=dev)
    kvc.layer_group_step(cfg, list(w.modes), inp["q"], inp["idx_q"], inp["windows"], w.window,
                         cache, out, tk, ws, lse=lse, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return inp, cache, out, lse, tk


def _oracle_records(w, ocfg, tokens_b, gate, entries):
    """Oracle records of the given entry indices of one sequence, from raw tokens."""
    rb = oracle.record_bytes(ocfg)
    recs = {}
    g = f32(gate)
    for j in entries:
        pair = f32(tokens_b[2 * j:2 * j + 2])
        e = oracle.compress_pair(pair[0], pair[1], g)
        recs[int(j)] = oracle.quantize_entry(ocfg, e)[0]
    return recs, rb


def _check(kvc, name, seqs, layers):
    w = synth.WORKLOADS[name]
    inp, cache, out, lse, tk = _run_group(kvc, w)
    ocfg = oracle_cfg(w)
    N = w.entries
    rng = np.random.default_rng(0)
    tk = tk.cpu().numpy()
    heads = [l for l, m in enumerate(w.modes) if m != synth.REUSE]
    idx_k = inp["idx_k"].cpu().numpy()
    # ---- top-K of every sequence and every Full/Reindex layer, bit-exact
    n = np.full(w.batch, N, np.int32)
    for l in heads:
        otk = oracle.index_topk(ocfg, inp["idx_q"][l].cpu().numpy(), idx_k, n)
        assert np.array_equal(tk[l], otk), f"{name}: top-K differs at layer {l}"
    for l, m in enumerate(w.modes):
        if m == synth.REUSE:
            assert np.array_equal(tk[l], tk[max(h for h in heads if h < l)])
    # ---- records: sampled entries (plus every selected one of the checked
    # sequences) packed by the oracle from the raw tokens, byte for byte
    recs_gpu = cache.records
    for b in seqs:
        sel = np.unique(np.concatenate([tk[l, b] for l in heads]))
        sample = np.unique(np.concatenate([rng.choice(N, 64, replace=False), sel[sel >= 0],
                                           [0, N - 1]]))
        recs, rb = _oracle_records(w, ocfg, inp["tokens"][b], inp["gate"], sample)
        got = recs_gpu[b, torch.from_numpy(sample).cuda()].cpu().numpy()
        want = np.stack([recs[int(j)] for j in sample])
        assert np.array_equal(got, want), f"{name}: packed records differ in sequence {b}"
        # ---- attention of the sampled layers, from the oracle's own records
        rec_full = np.zeros((1, N, rb), np.uint8)
        for j, r in recs.items():
            rec_full[0, j] = r
        for l in layers:
            o_ref, lse_ref, st = oracle.sparse_decode(
                ocfg, f32(inp["q"][l, b:b + 1]), rec_full, np.array([N], np.int32),
                tk[l, b:b + 1], f32(inp["windows"][l, b:b + 1]), w.window)
            assert st == 0
            assert_attn_close(out[l, b:b + 1].cpu().numpy(), o_ref, f"{name} b={b} layer={l}")
            assert np.max(np.abs(lse[l, b].cpu().numpy() - lse_ref[0])) < \
                2e-3 * np.abs(lse_ref).max()


def test_batch32x128k_full(kvc):
    _check(kvc, "batch32x128k", seqs=[0, 17, 31], layers=[0])


def test_csa2group_full(kvc):
    _check(kvc, "csa2group", seqs=[0, 7], layers=[0, 1, 2, 3])


def test_stack1m_full(kvc):
    _check(kvc, "stack1m", seqs=[0], layers=[0, 1, 4, 5, 19])
