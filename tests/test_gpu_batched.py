"""Batched indexer scoring on the tensor cores (several indexer queries per
sequence in one pass) vs the oracle: every query's int32 scores and top-K
bit-exact, including ragged lengths, forced ties, slices spanning sequences
and the 1M stack's five scoring layers at full size."""
import numpy as np
import pytest
import torch

import oracle
from fp4_compressed_kv_b200 import synth
from helpers import oracle_cfg, topk_set_equal

pytestmark = pytest.mark.gpu


def _run(kvc, w, idx_k, idx_q, n, cap):
    cfg = kvc.config_for(w)
    B = idx_k.shape[0]
    cache = kvc.Cache(cfg, B, cap)
    cache.idx_k[:, : idx_k.shape[1]] = idx_k.cuda()
    cache.n_entries.copy_(torch.as_tensor(n, dtype=torch.int32))
    nq = idx_q.shape[0]
    tk = torch.full((nq, B, w.topk), -7, dtype=torch.int32, device="cuda")
    ws = kvc.workspace_batched(cfg, nq, B, cap)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvc.index_topk_batched(cfg, idx_q.cuda().contiguous(), cache, tk, ws, status=st)
    torch.cuda.synchronize()
    return tk.cpu().numpy(), int(st.item()), cache, cfg


def _oracle(w, idx_k, idx_q, n, cap):
    ocfg = oracle_cfg(w)
    ic = np.zeros((idx_k.shape[0], cap, w.idx_dim), np.int8)
    ic[:, : idx_k.shape[1]] = idx_k.numpy()
    return np.stack([oracle.index_topk(ocfg, idx_q[q].numpy(), ic, np.asarray(n, np.int32))
                     for q in range(idx_q.shape[0])])


@pytest.mark.parametrize("nq", [1, 2, 5, 8])
def test_batched_matches_oracle(kvc, nq):
    w = synth.WORKLOADS["csa2group"].scaled(batch=5, context=2 * 9000)
    g = torch.Generator().manual_seed(40 + nq)
    idx_k = torch.randint(-127, 128, (5, 9000, 128), generator=g, dtype=torch.int8)
    idx_q = torch.randint(-127, 128, (nq, 5, 128), generator=g, dtype=torch.int8)
    n = [9000, 5000, 513, 512, 37]
    tk, st, cache, cfg = _run(kvc, w, idx_k, idx_q, n, 9008)
    assert st == 0
    want = _oracle(w, idx_k, idx_q, n, 9008)
    for q in range(nq):
        topk_set_equal(tk[q], want[q])
    # the same as nq single-query calls of the scan path
    ws = kvc.workspace(cfg, 5, 9008)
    for q in range(nq):
        one = torch.empty(5, w.topk, dtype=torch.int32, device="cuda")
        kvc.index_topk(cfg, idx_q[q].cuda().contiguous(), cache, one, ws)
        torch.cuda.synchronize()
        assert np.array_equal(one.cpu().numpy(), tk[q])


def test_batched_forced_ties_and_short_sequences(kvc):
    w = synth.WORKLOADS["mla32k"].scaled(batch=300, context=2 * 700)
    g = torch.Generator().manual_seed(9)
    idx_k = torch.randint(-3, 4, (300, 700, 128), generator=g, dtype=torch.int8)
    idx_k[:10] = 1  # constant rows: every score ties
    idx_q = torch.randint(-127, 128, (3, 300, 128), generator=g, dtype=torch.int8)
    n = np.random.default_rng(2).integers(400, 701, 300).astype(np.int32)
    tk, st, _, _ = _run(kvc, w, idx_k, idx_q, n, 700)
    assert st == 0
    want = _oracle(w, idx_k, idx_q, n, 700)
    for q in range(3):
        topk_set_equal(tk[q], want[q])


@pytest.mark.slow
def test_batched_stack1m_scoring_layers(kvc):
    """The 1M stack's Full and four Reindex indexer queries in one pass."""
    w = synth.WORKLOADS["stack1m"]
    inp = synth.make_inputs(w, with_tokens=False)
    heads = [i for i, m in enumerate(w.modes) if m != synth.REUSE]
    idx_q = inp["idx_q"][heads]
    tk, st, _, _ = _run(kvc, w, inp["idx_k"], idx_q, [w.entries], w.entries)
    assert st == 0
    want = _oracle(w, inp["idx_k"], idx_q, [w.entries], w.entries)
    for q in range(len(heads)):
        topk_set_equal(tk[q], want[q])


def test_batched_zero_wait_limit_times_out_then_recovers(kvc):
    """Under a zero wait limit the pipeline's waits (tile landed, products
    done, stage and accumulators released) give up at once: KVC_DEV_TIMEOUT,
    a normal return with every warp out of the pipeline and the loads in
    flight landed; after zeroing the workspace the next call is exact."""
    w = synth.WORKLOADS["csa2group"].scaled(batch=3, context=2 * 20000)
    g = torch.Generator().manual_seed(77)
    idx_k = torch.randint(-127, 128, (3, 20000, 128), generator=g, dtype=torch.int8)
    idx_q = torch.randint(-127, 128, (2, 3, 128), generator=g, dtype=torch.int8)
    n = [20000, 11111, 600]
    cfg = kvc.config_for(w)
    cache = kvc.Cache(cfg, 3, 20000)
    cache.idx_k.copy_(idx_k.cuda())
    cache.n_entries.copy_(torch.as_tensor(n, dtype=torch.int32))
    tk = torch.empty(2, 3, w.topk, dtype=torch.int32, device="cuda")
    ws = kvc.workspace_batched(cfg, 2, 3, 20000)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvc.debug_set_wait_limit_ns(0)
    try:
        kvc.index_topk_batched(cfg, idx_q.cuda().contiguous(), cache, tk, ws, status=st)
        torch.cuda.synchronize()
    finally:
        kvc.debug_set_wait_limit_ns(2_000_000_000)
    assert int(st.item()) & 0x8, int(st.item())  # KVC_DEV_TIMEOUT
    ws.zero_()
    st.zero_()
    kvc.index_topk_batched(cfg, idx_q.cuda().contiguous(), cache, tk, ws, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    want = _oracle(w, idx_k, idx_q, n, 20000)
    for q in range(2):
        topk_set_equal(tk.cpu().numpy()[q], want[q])
