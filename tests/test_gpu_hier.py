"""GPU hierarchical sparse indexer vs the oracle ("DeepSeek V1 到 V4.1-Flash
..." part 4, "层级稀疏索引器"): the Full layer's block pool and every Reindex
layer's top-K over the pool, bit-exact; attention of every layer within the
stated tolerance.  Ragged lengths (short last block, fewer blocks than kept,
n <= K), then the pages' sizes (2048 blocks of 8) on the CSA2 group and the
1M-token stack."""
import numpy as np
import pytest
import torch

import oracle
from fp4_compressed_kv_b200 import synth
from helpers import assert_attn_close, f32, oracle_cfg, oracle_pack

pytestmark = pytest.mark.gpu


def _gpu_group(kvc, w, cfg, cache, inp, keep, block):
    L, B, H = w.layers, cache.batch, w.heads
    out = torch.empty(L, B, H, w.latent, device="cuda")
    lse = torch.empty(L, B, H, device="cuda")
    tk = torch.empty(L, B, w.topk, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = kvc.workspace(cfg, B, cache.capacity, hier_blocks=keep, hier_block=block)
    kvc.layer_group_step(cfg, list(w.modes), inp["q"].cuda(), inp["idx_q"].cuda(),
                         inp["windows"].cuda(), w.window, cache, out, tk, ws, lse=lse, status=st,
                         hier_blocks=keep, hier_block=block)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy(), tk.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("keep,block", [(64, 8), (24, 16), (500, 8)])
def test_hier_group_ragged(kvc, keep, block):
    w = synth.WORKLOADS["csa2group"].scaled(batch=5, context=2 * 3001, modes=(0, 1, 2, 1))
    inp = synth.make_inputs(w)
    rec, ic, n, _ = oracle_pack(w, inp["tokens"], inp["gate"], inp["idx_k"])
    n = np.array([3001, 2999, 700, 512, 100], np.int32)  # short last blocks, n <= K
    cfg = kvc.config_for(w)
    cache = kvc.Cache(cfg, w.batch, rec.shape[1])
    cache.records.copy_(torch.from_numpy(rec))
    cache.idx_k.copy_(torch.from_numpy(ic))
    cache.n_entries.copy_(torch.from_numpy(n))
    out, lse, tk, st = _gpu_group(kvc, w, cfg, cache, inp, keep, block)
    ocfg = oracle_cfg(w)
    oout, olse, otk, ost = oracle.group_step(ocfg, list(w.modes), f32(inp["q"]),
                                             inp["idx_q"].numpy(), f32(inp["windows"]),
                                             w.window, rec, ic, n, hier_keep=keep,
                                             hier_block=block)
    assert st == 0 and ost == 0
    for layer in range(w.layers):
        assert np.array_equal(tk[layer], otk[layer]), f"layer {layer} top-K differs"
        assert_attn_close(out[layer], oout[layer], f"layer {layer}")
        assert np.max(np.abs(lse[layer] - olse[layer])) < 2e-3 * np.abs(olse[layer]).max()
    # the pool really restricts the Reindex layers when fewer blocks are kept
    plain = oracle.group_step(ocfg, list(w.modes), f32(inp["q"]), inp["idx_q"].numpy(),
                              f32(inp["windows"]), w.window, rec, ic, n)[2]
    if keep * block < 3001:
        assert not np.array_equal(plain[1], otk[1])


def _oracle_hier_topk(w, ocfg, idx_q, idx_k, n, keep, block):
    """Oracle top-K of every layer from the raw indexer keys and queries."""
    L = w.layers
    tks = [None] * L
    pools = None
    head = None
    for layer, m in enumerate(w.modes):
        if m == synth.FULL or (m == synth.REINDEX and pools is None):
            t, sc = oracle.index_topk(ocfg, idx_q[layer], idx_k, n, want_scores=True)
            tks[layer] = t
            if m == synth.FULL:
                pools = [oracle.block_pool(sc[b, :n[b]], block, keep)[1] for b in range(len(n))]
            head = layer
        elif m == synth.REINDEX:
            tks[layer] = np.stack([oracle.pool_topk(idx_q[layer][b], idx_k[b], pools[b], w.topk)
                                   for b in range(len(n))])
            head = layer
        else:
            tks[layer] = tks[head]
    return np.stack(tks)


@pytest.mark.slow
@pytest.mark.parametrize("name,seqs", [("csa2group", [0, 5]), ("stack1m", [0])])
def test_hier_fullsize(kvc, name, seqs):
    """The pages' parameters (2048 blocks of 8 -> 16,384-entry pool) at full
    size; the cache is packed on the GPU, the oracle works from the raw
    indexer keys and queries and re-packs the records it attends over."""
    w = synth.WORKLOADS[name]
    dev = torch.device("cuda")
    inp = synth.make_inputs(w, dev)
    cfg = kvc.config_for(w)
    cache = kvc.Cache(cfg, w.batch, w.entries, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    kvc.pack(cfg, inp["tokens"], inp["gate"], inp["idx_k"], cache, status=st)
    out, lse, tk, st2 = _gpu_group(kvc, w, cfg, cache, inp, 2048, 8)
    assert st.item() == 0 and st2 == 0
    ocfg = oracle_cfg(w)
    n = np.full(w.batch, w.entries, np.int32)
    idx_q, idx_k = inp["idx_q"].cpu().numpy(), inp["idx_k"].cpu().numpy()
    otk = _oracle_hier_topk(w, ocfg, idx_q, idx_k, n, 2048, 8)
    assert np.array_equal(tk, otk)
    # attention of the first Reindex layer (pool-selected) on sampled sequences
    layer = list(w.modes).index(synth.REINDEX)
    g = f32(inp["gate"])
    rb = oracle.record_bytes(ocfg)
    for b in seqs:
        rec = np.zeros((1, w.entries, rb), np.uint8)
        toks = inp["tokens"][b]
        for j in tk[layer, b]:
            pair = f32(toks[2 * j:2 * j + 2])
            rec[0, j] = oracle.quantize_entry(ocfg, oracle.compress_pair(pair[0], pair[1], g))[0]
        o_ref, l_ref, ost = oracle.sparse_decode(ocfg, f32(inp["q"][layer, b:b + 1]), rec,
                                                 np.array([w.entries], np.int32),
                                                 tk[layer, b:b + 1],
                                                 f32(inp["windows"][layer, b:b + 1]), w.window)
        assert ost == 0
        assert_attn_close(out[layer, b:b + 1], o_ref, f"{name} b={b}")
