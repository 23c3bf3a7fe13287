"""Failure detection on the GPU without a GPU fault, and the operand range of
the tensor-core attention.

Every in-kernel wait is bounded.  kvc_debug_set_wait_limit_ns(0) turns each
wait into a single non-blocking poll, so the indexer scan's bulk-copy waits
and the attention's tensor-core and TMA waits give up at once: the kernels
must set KVC_DEV_TIMEOUT, let what they issued land (with the normal bound),
free their tensor memory and return, leaving the context usable.  After
zeroing the workspace the next call must again match the oracle exactly.

The attention runs record chunks with f16 operands (each query row scaled by
a power of two into the f16 range) and window chunks with bf16 operands, so
no finite bf16 query or window value may turn into inf or NaN.
"""
import numpy as np
import pytest
import torch

import oracle
from fp4_compressed_kv_b200 import synth
from helpers import assert_attn_close, f32, oracle_cfg, oracle_pack

pytestmark = pytest.mark.gpu

KVC_DEV_TIMEOUT = 0x8


def _setup(kvc, w):
    inp = synth.make_inputs(w)
    rec, ic, n, _ = oracle_pack(w, inp["tokens"], inp["gate"], inp["idx_k"])
    cfg = kvc.config_for(w)
    cache = kvc.Cache(cfg, w.batch, rec.shape[1])
    cache.records.copy_(torch.from_numpy(rec))
    cache.idx_k.copy_(torch.from_numpy(ic))
    cache.n_entries.copy_(torch.from_numpy(n))
    return inp, rec, ic, n, cfg, cache


def test_zero_wait_limit_times_out_then_recovers(kvc):
    w = synth.WORKLOADS["mla32k"].scaled(batch=2, context=2 * 20000, modes=(0, 2))
    inp, rec, ic, n, cfg, cache = _setup(kvc, w)
    L, B, H = w.layers, w.batch, w.heads
    ws = kvc.workspace(cfg, B, cache.capacity)
    out = torch.empty(L, B, H, w.latent, device="cuda")
    lse = torch.empty(L, B, H, device="cuda")
    tk = torch.empty(L, B, w.topk, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    args = (cfg, list(w.modes), inp["q"].cuda(), inp["idx_q"].cuda(), inp["windows"].cuda(),
            w.window, cache, out, tk, ws)
    kvc.debug_set_wait_limit_ns(0)
    try:
        kvc.layer_group_step(*args, lse=lse, status=st)  # returns normally
        torch.cuda.synchronize()  # and the kernels end: no hang
    finally:
        kvc.debug_set_wait_limit_ns(2_000_000_000)
    assert int(st.item()) & KVC_DEV_TIMEOUT, int(st.item())

    # the context is still usable: zero the workspace, run again, compare
    ws.zero_()
    st.zero_()
    kvc.layer_group_step(*args, lse=lse, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ocfg = oracle_cfg(w)
    ref, ref_lse, otk, ost = oracle.group_step(ocfg, list(w.modes), f32(inp["q"]),
                                               inp["idx_q"].numpy(), f32(inp["windows"]),
                                               w.window, rec, ic, n)
    assert ost == 0
    assert np.array_equal(tk.cpu().numpy(), otk)
    assert_attn_close(out.cpu().numpy(), ref, "after recovery")


@pytest.mark.parametrize("where", ["query_large", "query_small", "window_large"])
def test_attention_operand_range(kvc, where):
    """Query rows near the bf16 extremes (1e5 and 1e-6 in magnitude) and
    window rows of magnitude 1e5: the result matches the fp64 oracle and the
    status stays clean."""
    w = synth.WORKLOADS["mla32k"].scaled(context=2 * 3000)
    inp, rec, ic, n, cfg, cache = _setup(kvc, w)
    ocfg = oracle_cfg(w)
    tk = oracle.index_topk(ocfg, inp["idx_q"][0].numpy(), ic, n)
    q = inp["q"][0].float().clone()
    win = inp["windows"][0].float().clone()
    if where == "query_large":
        q[:, :8] *= 1e5   # 8 heads with rows far above the f16 range
    elif where == "query_small":
        q[:, 8:16] *= 1e-6  # 8 heads with rows far below the f16 normal range
    else:
        win[:, :5] *= 1e5  # 5 window rows far above the f16 range
    qb = q.to(torch.bfloat16)
    wb = win.to(torch.bfloat16)
    B, H = qb.shape[0], qb.shape[1]
    out = torch.empty(B, H, w.latent, device="cuda")
    lse = torch.empty(B, H, device="cuda")
    ws = kvc.workspace(cfg, B, cache.capacity)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvc.sparse_decode_attn(cfg, qb.cuda().contiguous(), cache, torch.from_numpy(tk).cuda(),
                           wb.cuda().contiguous(), w.window, out, ws, lse=lse, status=st)
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    assert int(st.item()) == 0
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse.cpu().numpy()))
    ref, ref_lse, ost = oracle.sparse_decode(ocfg, f32(qb), rec, n, tk, f32(wb), w.window)
    assert ost == 0
    assert_attn_close(o, ref, where)
    rl = np.asarray(ref_lse)
    assert np.max(np.abs(lse.cpu().numpy() - rl) / np.maximum(1.0, np.abs(rl))) < 2e-3


def test_pack_ring_zero_wait_limit_times_out_then_recovers(kvc):
    """A long bf16 append runs the pack ring (a producer thread, consumer warps
    and stage barriers).  Under a zero wait limit its consumers and producer
    give up at their first incomplete barrier: the call returns with
    KVC_DEV_TIMEOUT, the copies already issued land before the CTAs exit, and
    the next append (normal limit, fresh cache) equals the oracle byte for byte."""
    # 8 x 375 units of 8 entries: more units per CTA than stages, so the
    # producer waits on stages too
    w = synth.WORKLOADS["batch32x128k"].scaled(batch=8, context=2 * 3000)
    inp = synth.make_inputs(w)
    cfg = kvc.config_for(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tok, gate, idx = inp["tokens"].cuda(), inp["gate"].cuda(), inp["idx_k"].cuda()
    spoiled = kvc.Cache(cfg, w.batch, w.entries)
    kvc.debug_set_wait_limit_ns(0)
    try:
        kvc.pack(cfg, tok, gate, idx, spoiled, status=st)  # returns normally
        torch.cuda.synchronize()  # and the kernel ends: no hang
    finally:
        kvc.debug_set_wait_limit_ns(2_000_000_000)
    assert int(st.item()) & KVC_DEV_TIMEOUT, int(st.item())

    st.zero_()
    cache = kvc.Cache(cfg, w.batch, w.entries)
    kvc.pack(cfg, tok, gate, idx, cache, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rec, ic, n, _ = oracle_pack(w, inp["tokens"], inp["gate"], inp["idx_k"])
    assert np.array_equal(cache.records.cpu().numpy(), rec)
    assert np.array_equal(cache.idx_k.cpu().numpy(), ic)
    assert cache.n_entries.cpu().tolist() == n.tolist()
