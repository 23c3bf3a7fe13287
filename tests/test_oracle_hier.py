"""Pins of the oracle's hierarchical sparse indexer ("DeepSeek V1 到
V4.1-Flash ..." part 4, "层级稀疏索引器"): blocks of 8 entries scored by
their best entry, the best 2048 blocks form the pool, later Reindex layers
score only the pool.

- Block pool vs a brute force written here: block maxima from numpy slices,
  blocks ranked by (maximum descending, block index ascending), short last
  block, fewer blocks than kept, constant scores (ties to the lower block).
- Pool top-K vs a brute force over the pool's int64 scores.
- Reductions: keeping every block makes the hierarchical group step identical
  to the plain one; a Reindex layer given the Full layer's indexer query
  picks the Full layer's set (every entry of the top-K lies in a block whose
  maximum is at least the K-th score, so its block is kept when no more than
  `keep` blocks reach that score, e.g. keep >= K without ties).
"""
import numpy as np
import pytest

from fp4_compressed_kv_b200 import synth


def _brute_pool(scores, block, keep):
    n = scores.size
    nb = -(-n // block)
    bm = np.array([scores[i * block:min(n, (i + 1) * block)].max() for i in range(nb)], np.int64)
    order = sorted(range(nb), key=lambda i: (-bm[i], i))[:keep]
    blocks = sorted(order)
    pool = [j for i in blocks for j in range(i * block, min(n, (i + 1) * block))]
    return np.array(blocks + [-1] * (keep - len(blocks)), np.int32), np.array(pool, np.int32)


@pytest.mark.parametrize("n,block,keep,span", [(37, 8, 2, 200), (1000, 8, 16, 50),
                                               (5, 8, 4, 10), (64, 8, 8, 5), (4099, 8, 64, 3),
                                               (700, 4, 1, 1000)])
def test_block_pool_brute_force(orc, n, block, keep, span):
    rng = np.random.default_rng(n + keep)
    scores = rng.integers(-span, span + 1, n).astype(np.int32)
    blocks, pool = orc.block_pool(scores, block, keep)
    want_b, want_p = _brute_pool(scores, block, keep)
    assert np.array_equal(blocks, want_b)
    assert np.array_equal(pool, want_p)


def test_block_pool_constant_scores_take_lowest_blocks(orc):
    blocks, pool = orc.block_pool(np.zeros(100, np.int32), 8, 3)
    assert blocks.tolist() == [0, 1, 2]
    assert pool.tolist() == list(range(24))
    # the short last block (entries 96..99) holds the only maximum
    s = np.zeros(100, np.int32)
    s[98] = 5
    blocks, pool = orc.block_pool(s, 8, 2)
    assert blocks.tolist() == [0, 12] and pool.tolist() == list(range(8)) + [96, 97, 98, 99]


def test_pool_topk_brute_force(orc):
    rng = np.random.default_rng(5)
    keys = rng.integers(-127, 128, (3000, 32)).astype(np.int8)
    q = rng.integers(-127, 128, 32).astype(np.int8)
    pool = np.sort(rng.choice(3000, 700, replace=False)).astype(np.int32)
    s = keys[pool].astype(np.int64) @ q.astype(np.int64)
    for k in (64, 700, 1000):
        order = np.lexsort((pool, -s))[:k]
        want = np.sort(pool[order])
        want = np.concatenate([want, -np.ones(k - want.size, np.int64)]).astype(np.int32)
        assert np.array_equal(orc.pool_topk(q, keys, pool, k), want)


def _tiny_setup(orc, w):
    inp = synth.make_inputs(w)
    cfg = orc.make_cfg(w.latent, w.rope, w.group, w.scale_fmt, w.idx_dim, w.topk, w.window,
                       w.heads, w.sm_scale)
    B, T = inp["tokens"].shape[:2]
    rec = np.zeros((B, T // 2, orc.record_bytes(cfg)), np.uint8)
    ic = np.zeros((B, T // 2, w.idx_dim), np.int8)
    n = np.zeros(B, np.int32)
    assert orc.pack(cfg, inp["tokens"].float().numpy(), inp["gate"].numpy(),
                    inp["idx_k"].numpy(), rec, ic, n) == 0
    return cfg, inp, rec, ic, n


def test_hier_keep_all_blocks_is_the_plain_step(orc):
    w = synth.WORKLOADS["tiny"].scaled(modes=(0, 1, 2, 1), context=2 * 600)
    cfg, inp, rec, ic, n = _tiny_setup(orc, w)
    args = (cfg, list(w.modes), inp["q"].float().numpy(), inp["idx_q"].numpy(),
            inp["windows"].float().numpy(), w.window, rec, ic, n)
    plain = orc.group_step(*args)
    hier = orc.group_step(*args, hier_keep=600 // 8 + 1, hier_block=8)
    for a, b in zip(plain, hier):
        assert np.array_equal(np.asarray(a), np.asarray(b))


def test_hier_reindex_with_full_query_picks_full_set(orc):
    w = synth.WORKLOADS["tiny"].scaled(modes=(0, 1, 2), context=2 * 3000)
    cfg, inp, rec, ic, n = _tiny_setup(orc, w)
    iq = inp["idx_q"].numpy().copy()
    iq[1] = iq[0]
    # keep >= K blocks: every block holding a top-K entry is kept
    out, lse, tk, st = orc.group_step(cfg, list(w.modes), inp["q"].float().numpy(), iq,
                                      inp["windows"].float().numpy(), w.window, rec, ic, n,
                                      hier_keep=w.topk, hier_block=8)
    assert st == 0
    assert np.array_equal(tk[1], tk[0]) and np.array_equal(tk[2], tk[1])
    # and with another query the Reindex set lies inside the pool of the Full layer
    iq[1] = -iq[0]
    _, _, tk2, _ = orc.group_step(cfg, list(w.modes), inp["q"].float().numpy(), iq,
                                  inp["windows"].float().numpy(), w.window, rec, ic, n,
                                  hier_keep=16, hier_block=8)
    _, sc = orc.index_topk(cfg, iq[0], ic, n, want_scores=True)
    _, pool = orc.block_pool(sc[0, :n[0]], 8, 16)
    assert tk2[1][0].size == w.topk and set(tk2[1][0][tk2[1][0] >= 0]) <= set(pool.tolist())
    assert np.array_equal(tk2[1][0], orc.pool_topk(iq[1][0], ic[0], pool, w.topk))
