"""kvc_index_topk_noalloc: the indexer top-K for callers that cannot allocate
device memory (a plugin whose host framework owns all device allocations, or a
path where cudaMalloc's implicit synchronisation is not allowed).  Its scratch
is a fixed array inside the library; its results must equal the
workspace-taking kvc_index_topk's exactly, call after call, since each call
reuses the array left over by the previous one.  This file is collected last so
that a stop-at-first-failure run has already run every other test."""
import numpy as np
import pytest
import torch

from fp4_compressed_kv_b200 import synth

pytestmark = pytest.mark.gpu


def _cache(kvc, w, n_entries, seed):
    cfg = kvc.config_for(w)
    B = len(n_entries)
    cap = max(n_entries)
    cache = kvc.Cache(cfg, B, cap)
    g = torch.Generator(device="cuda").manual_seed(seed)
    cache.idx_k.copy_(torch.randint(-127, 128, cache.idx_k.shape, generator=g, device="cuda",
                                    dtype=torch.int8))
    cache.n_entries.copy_(torch.tensor(n_entries, dtype=torch.int32))
    return cfg, cache, g


def test_noalloc_matches_workspace_entry_point_twice(kvc):
    w = synth.WORKLOADS["mla32k"]
    n_entries = [40000, 23000, 512, 9000]
    cfg, cache, g = _cache(kvc, w, n_entries, seed=5)
    B, cap = cache.batch, cache.capacity
    ws = kvc.workspace(cfg, B, cap)
    for call in range(2):  # two calls in a row, different queries
        q = torch.randint(-127, 128, (B, w.idx_dim), generator=g, device="cuda",
                          dtype=torch.int8)
        tk_ref = torch.empty(B, w.topk, dtype=torch.int32, device="cuda")
        sc_ref = torch.zeros(B, cap, dtype=torch.int32, device="cuda")
        kvc.index_topk(cfg, q, cache, tk_ref, ws, scores=sc_ref)
        tk = torch.full((B, w.topk), -7, dtype=torch.int32, device="cuda")
        sc = torch.zeros(B, cap, dtype=torch.int32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        kvc.index_topk_noalloc(cfg, q, cache, tk, scores=sc, status=st)
        tk2 = torch.full((B, w.topk), -7, dtype=torch.int32, device="cuda")
        kvc.index_topk_noalloc(cfg, q, cache, tk2, status=st)  # scores left in the array
        torch.cuda.synchronize()
        assert st.item() == 0
        assert torch.equal(tk, tk_ref), f"call {call}: top-K differs"
        assert torch.equal(tk2, tk_ref), f"call {call}: top-K (internal scores) differs"
        for b, n in enumerate(n_entries):
            assert torch.equal(sc[b, :n], sc_ref[b, :n])


def test_noalloc_heavy_ties_and_limits(kvc):
    w = synth.WORKLOADS["mla32k"]
    cfg, cache, _ = _cache(kvc, w, [20000], seed=6)
    cache.idx_k.fill_(3)  # every score equal: the candidate list overflows
    q = torch.full((1, w.idx_dim), 2, dtype=torch.int8, device="cuda")
    ws = kvc.workspace(cfg, 1, cache.capacity)
    ref = torch.empty(1, w.topk, dtype=torch.int32, device="cuda")
    kvc.index_topk(cfg, q, cache, ref, ws)
    for _ in range(2):
        tk = torch.empty(1, w.topk, dtype=torch.int32, device="cuda")
        kvc.index_topk_noalloc(cfg, q, cache, tk)
        torch.cuda.synchronize()
        assert torch.equal(tk, ref)
        assert torch.equal(tk[0], torch.arange(w.topk, dtype=torch.int32, device="cuda"))
    # beyond the fixed scratch: rejected before any work, with KVC_ERR_CAPACITY
    big_cfg, big, _ = _cache(kvc, w.scaled(batch=1), [(1 << 19) + 16], seed=7)
    with pytest.raises(kvc.KvcError) as e:
        kvc.index_topk_noalloc(big_cfg, q, big, torch.empty(1, w.topk, dtype=torch.int32,
                                                             device="cuda"))
    assert e.value.status == 2
    many_cfg, many, _ = _cache(kvc, w.scaled(batch=65), [100] * 65, seed=8)
    with pytest.raises(kvc.KvcError) as e:
        kvc.index_topk_noalloc(many_cfg, torch.zeros(65, w.idx_dim, dtype=torch.int8,
                                                     device="cuda"), many,
                               torch.empty(65, w.topk, dtype=torch.int32, device="cuda"))
    assert e.value.status == 2


@pytest.mark.parametrize("n_entries", [
    [1 << 19],                                        # one sequence at the row limit
    [8192 - 97 * (i % 7) for i in range(63)] + [8192],  # 64 ragged sequences, 2^19 rows
])
def test_noalloc_at_the_largest_accepted_shapes(kvc, n_entries):
    """The fixed scratch is sized for batch x capacity <= 2^19 rows and at most
    64 sequences; the shapes that fill it exactly must still equal
    kvc_index_topk, on two calls in a row."""
    w = synth.WORKLOADS["mla32k"]
    cfg, cache, g = _cache(kvc, w.scaled(batch=len(n_entries)), n_entries, seed=9)
    B, cap = cache.batch, cache.capacity
    assert B * cap == 1 << 19
    ws = kvc.workspace(cfg, B, cap)
    for call in range(2):
        q = torch.randint(-127, 128, (B, w.idx_dim), generator=g, device="cuda",
                          dtype=torch.int8)
        ref = torch.empty(B, w.topk, dtype=torch.int32, device="cuda")
        kvc.index_topk(cfg, q, cache, ref, ws)
        tk = torch.full((B, w.topk), -7, dtype=torch.int32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        kvc.index_topk_noalloc(cfg, q, cache, tk, status=st)
        torch.cuda.synchronize()
        assert st.item() == 0
        assert torch.equal(tk, ref), f"call {call}: top-K differs"
