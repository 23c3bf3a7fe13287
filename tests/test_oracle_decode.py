"""Pins of the oracle's indexer, top-K, attention and CSA2 group step.

- Scores vs numpy's int64 matmul; top-K vs a brute-force lexicographic sort
  (score descending, index ascending), with forced ties and K >= N.
- Attention: with every entry selected and the window covering the rest it
  must equal dense softmax attention (torch, fp64); softmax rows sum to 1.
- Group step: a Reuse layer given its head's q and window reproduces the
  head; a Reindex layer given the Full layer's indexer q picks the same set.
"""
import numpy as np
import pytest
import torch

from fp4_compressed_kv_b200 import synth


def _brute_topk(scores, k):
    idx = np.arange(scores.size)
    order = np.lexsort((idx, -scores.astype(np.int64)))
    keep = np.sort(order[:k])
    return np.concatenate([keep, -np.ones(k - keep.size, np.int64)]).astype(np.int32)


def test_index_scores_match_matmul(orc):
    rng = np.random.default_rng(0)
    keys = rng.integers(-127, 128, (3000, 128)).astype(np.int8)
    q = rng.integers(-127, 128, 128).astype(np.int8)
    want = keys.astype(np.int64) @ q.astype(np.int64)
    assert np.array_equal(orc.index_scores(q, keys), want.astype(np.int32))
    extreme = np.full((1, 128), -128, np.int8)
    assert orc.index_scores(np.full(128, -128, np.int8), extreme)[0] == 128 * 128 * 128


@pytest.mark.parametrize("n,k,span", [(5000, 512, 10 ** 6), (5000, 512, 7), (700, 512, 3),
                                      (300, 512, 100), (512, 512, 2), (1, 64, 5), (0, 64, 1),
                                      (2000, 64, 1)])
def test_topk_brute_force(orc, n, k, span):
    rng = np.random.default_rng(n + k + span)
    scores = rng.integers(-span, span + 1, n).astype(np.int32)
    got = orc.topk(scores, k)
    assert np.array_equal(got, _brute_topk(scores, k))
    kept = got[got >= 0]
    assert np.all(np.diff(kept) > 0)
    assert kept.size == min(n, k)


def test_topk_ties_go_to_lower_index(orc):
    scores = np.zeros(1000, np.int32)
    assert np.array_equal(orc.topk(scores, 64), np.arange(64, dtype=np.int32))
    scores[900:] = 5
    got = orc.topk(scores, 150)
    assert np.array_equal(got, np.concatenate([np.arange(50), np.arange(900, 1000)]))


def test_index_topk_batch_respects_lengths(orc):
    rng = np.random.default_rng(3)
    cfg = orc.make_cfg(64, 16, 32, orc.SCALE_F32, 32, 64, 32, 8, 1.0)
    B, cap = 3, 400
    cache = rng.integers(-127, 128, (B, cap, 32)).astype(np.int8)
    q = rng.integers(-127, 128, (B, 32)).astype(np.int8)
    n = np.array([400, 37, 0], np.int32)
    tk, sc = orc.index_topk(cfg, q, cache, n, want_scores=True)
    for b in range(B):
        s = cache[b, : n[b]].astype(np.int64) @ q[b].astype(np.int64)
        assert np.array_equal(sc[b, : n[b]], s)
        assert np.array_equal(tk[b], _brute_topk(s.astype(np.int32), 64))


# ------------------------------------------------------------------ attention
def _dense(q, keys, scale, dv):
    qt = torch.from_numpy(q.astype(np.float64))
    kt = torch.from_numpy(keys.astype(np.float64))
    s = scale * qt @ kt.T
    return (torch.softmax(s, -1) @ kt[:, :dv]).numpy(), torch.logsumexp(s, -1).numpy()


def test_attention_is_dense_softmax_attention(orc):
    rng = np.random.default_rng(4)
    for H, D, dv, nk in ((8, 80, 64, 96), (64, 576, 512, 640), (4, 80, 64, 1)):
        q = rng.standard_normal((H, D)).astype(np.float32)
        keys = rng.standard_normal((nk, D)).astype(np.float32)
        out, lse = orc.attention(q, keys, D ** -0.5, dv)
        ref, ref_lse = _dense(q, keys, D ** -0.5, dv)
        assert np.max(np.abs(out - ref)) < 1e-12 and np.max(np.abs(lse - ref_lse)) < 1e-12


def test_attention_rows_sum_to_one(orc):
    rng = np.random.default_rng(5)
    q = (rng.standard_normal((16, 80)) * 3).astype(np.float32)
    keys = rng.standard_normal((200, 80)).astype(np.float32)
    keys[:, :64] = 1.0
    out, _ = orc.attention(q, keys, 1.0, 64)
    assert np.max(np.abs(out - 1.0)) < 1e-12


def test_attention_empty_key_set(orc):
    out, lse = orc.attention(np.ones((2, 80), np.float32), np.zeros((0, 80), np.float32), 1.0, 64)
    assert not out.any() and np.all(lse == -np.inf)


def _tiny_cache(orc, w):
    inp = synth.make_inputs(w)
    cfg = orc.make_cfg(w.latent, w.rope, w.group, w.scale_fmt, w.idx_dim, w.topk, w.window,
                       w.heads, w.sm_scale)
    cap = w.entries
    rec = np.zeros((w.batch, cap, orc.record_bytes(cfg)), np.uint8)
    ic = np.zeros((w.batch, cap, w.idx_dim), np.int8)
    n = np.zeros(w.batch, np.int32)
    orc.pack(cfg, inp["tokens"].float().numpy(), inp["gate"].numpy(), inp["idx_k"].numpy(),
             rec, ic, n)
    return cfg, inp, rec, ic, n


def test_sparse_decode_all_selected_reduces_to_dense(orc):
    w = synth.WORKLOADS["tiny"].scaled(context=96, topk=64)  # 48 entries <= K
    cfg, inp, rec, ic, n = _tiny_cache(orc, w)
    tk = orc.index_topk(cfg, inp["idx_q"][0].numpy(), ic, n)
    assert np.array_equal(tk[0, :48], np.arange(48)) and np.all(tk[0, 48:] == -1)
    win = inp["windows"][0].float().numpy()
    out, lse, st = orc.sparse_decode(cfg, inp["q"][0].float().numpy(), rec, n, tk, win, w.window)
    assert st == 0
    keys = np.concatenate([np.stack([orc.dequantize_entry(cfg, rec[0, j]) for j in range(48)]),
                           win[0]])
    ref, ref_lse = _dense(inp["q"][0, 0].float().numpy(), keys, w.sm_scale, w.latent)
    assert np.max(np.abs(out[0] - ref)) < 1e-12 and np.max(np.abs(lse[0] - ref_lse)) < 1e-12


def test_sparse_decode_skips_padding_and_flags_bad_indices(orc):
    w = synth.WORKLOADS["tiny"]
    cfg, inp, rec, ic, n = _tiny_cache(orc, w)
    q = inp["q"][0].float().numpy()
    win = inp["windows"][0].float().numpy()
    tk = np.full((1, w.topk), -1, np.int32)
    tk[0, :3] = [5, 9, 400]
    out, lse, st = orc.sparse_decode(cfg, q, rec, n, tk, win, 0)
    keys = np.stack([orc.dequantize_entry(cfg, rec[0, j]) for j in (5, 9, 400)])
    ref, _ = _dense(q[0], keys, w.sm_scale, w.latent)
    assert st == 0 and np.max(np.abs(out[0] - ref)) < 1e-12
    tk[0, 3] = 512  # == n_entries: not visible
    tk[0, 4] = -7
    out2, _, st2 = orc.sparse_decode(cfg, q, rec, n, tk, win, 0)
    assert st2 == orc.ST_BAD_INDEX and np.array_equal(out, out2)


def test_tiny_pipeline_brute_force(orc):
    """Whole decode step on the tiny workload against an independent brute force."""
    w = synth.WORKLOADS["tiny"]
    cfg, inp, rec, ic, n = _tiny_cache(orc, w)
    iq = inp["idx_q"][0].numpy()
    s = inp["idx_k"][0].numpy().astype(np.int64) @ iq[0].astype(np.int64)
    tk = orc.index_topk(cfg, iq, ic, n)
    assert np.array_equal(tk[0], _brute_topk(s.astype(np.int32), w.topk))
    q = inp["q"][0].float().numpy()
    win = inp["windows"][0].float().numpy()
    out, lse, _ = orc.sparse_decode(cfg, q, rec, n, tk, win, w.window)
    keys = np.concatenate([np.stack([orc.dequantize_entry(cfg, rec[0, j]) for j in tk[0]]),
                           inp["tokens"][0, -w.window:].float().numpy()])
    ref, ref_lse = _dense(q[0], keys, w.sm_scale, w.latent)
    assert np.max(np.abs(out[0] - ref)) < 1e-12 and np.max(np.abs(lse[0] - ref_lse)) < 1e-12


# ------------------------------------------------------------------ group step
def test_group_step_modes(orc):
    w = synth.WORKLOADS["tiny"].scaled(modes=(0, 2, 1, 2))
    cfg, inp, rec, ic, n = _tiny_cache(orc, w)
    q = inp["q"].float().numpy()
    iq = inp["idx_q"].numpy()
    win = inp["windows"].float().numpy()
    # layer 1 (Reuse) gets the head's q and window; layer 2 (Reindex) the head's indexer q
    q[1], win[1], iq[2] = q[0], win[0], iq[0]
    out, lse, tk, st = orc.group_step(cfg, [0, 2, 1, 2], q, iq, win, w.window, rec, ic, n)
    assert st == 0
    assert np.array_equal(out[1], out[0]) and np.array_equal(lse[1], lse[0])
    assert np.array_equal(tk[1], tk[0]) and np.array_equal(tk[2], tk[0])
    assert np.array_equal(tk[3], tk[2])
    # each layer equals the standalone calls
    for layer in range(4):
        head = {0: 0, 1: 0, 2: 2, 3: 2}[layer]
        t = orc.index_topk(cfg, iq[head], ic, n)
        assert np.array_equal(t, tk[layer])
        o, l_, _ = orc.sparse_decode(cfg, q[layer], rec, n, t, win[layer], w.window)
        assert np.array_equal(o, out[layer]) and np.array_equal(l_, lse[layer])
    with pytest.raises(ValueError):
        orc.group_step(cfg, [2, 0, 2, 2], q, iq, win, w.window, rec, ic, n)
