"""Pins of the oracle's 4:1 compression (four consecutive tokens per entry,
weights = softmax of their four gate logits; the 2x / 4x CSA2 compression
ratios of "DeepSeek V4.1 Flash KV Cache压缩实战" 4.3, the 2:1 rule of
"DeepSeek V1 到 V4.1-Flash ..." breakthrough 4 extended to four tokens).

- A zero gate gives equal weights: the entry is the plain mean of the four
  tokens (fp64 mean within fp32 rounding).
- A token whose logit exceeds the others by far more than 87 takes weight 1
  exactly: the entry is that token, bit for bit, and so is its record.
- Two tokens far below the other two: the entry is the pair's 2:1
  compression (the softmax of two logits) within fp32 rounding.
- Random tokens and gate: logits and entries against an fp64 evaluation.
- Pack bookkeeping: n_new / 4 entries per sequence, indexer rows, lengths,
  and n_new not a multiple of 4 rejected.
"""
import numpy as np
import pytest

import oracle as orc


def _tokens(rng, D, n=4, scale=1.0):
    return (rng.standard_normal((n, D)) * scale).astype(np.float32)


def test_zero_gate_is_the_mean():
    rng = np.random.default_rng(1)
    ks = _tokens(rng, 576)
    e = orc.compress_group4(ks, np.zeros(576, np.float32))
    mean = ks.astype(np.float64).mean(0)
    assert np.max(np.abs(e - mean)) <= 2.0 ** -22 * np.max(np.abs(ks))


@pytest.mark.parametrize("win", [0, 1, 2, 3])
def test_dominant_token_is_copied_exactly(win):
    rng = np.random.default_rng(2 + win)
    D = 576
    ks = _tokens(rng, D)
    g = np.zeros(D, np.float32)
    g[0] = 1.0
    ks[:, 0] = -60.0
    ks[win, 0] = 60.0  # logit 60 against -60: the others' weights underflow to 0
    e = orc.compress_group4(ks, g)
    assert np.array_equal(e.view(np.uint32), ks[win].view(np.uint32))
    cfg = orc.make_cfg(512, 64, 64, orc.SCALE_UE4M3, 128, 512, 128, 64, 1.0, ratio=4)
    rec_e, _ = orc.quantize_entry(cfg, e)
    rec_k, _ = orc.quantize_entry(cfg, ks[win])
    assert np.array_equal(rec_e, rec_k)


def test_two_far_tokens_reduce_to_the_pair():
    rng = np.random.default_rng(7)
    D = 96
    ks = _tokens(rng, D)
    g = (rng.standard_normal(D) / np.sqrt(D)).astype(np.float32)
    g[0] = 1.0
    ks[2:, 0] = -500.0  # logits of tokens 2, 3 hundreds below tokens 0, 1
    e4 = orc.compress_group4(ks, g)
    e2 = orc.compress_pair(ks[0], ks[1], g)
    assert np.max(np.abs(e4 - e2)) <= 2.0 ** -20 * np.max(np.abs(ks[:2]))


def test_random_groups_against_fp64():
    rng = np.random.default_rng(11)
    for D in (80, 576):
        for _ in range(20):
            ks = _tokens(rng, D, scale=rng.uniform(0.1, 4))
            g = (rng.standard_normal(D) * rng.uniform(0.01, 0.3)).astype(np.float32)
            lg = ks.astype(np.float64) @ g.astype(np.float64)
            for t in range(4):
                got = orc.gate_logit(ks[t], g)
                bound = 1e-5 * (np.abs(ks[t].astype(np.float64)) @ np.abs(g.astype(np.float64)) + 1e-30)
                assert abs(got - lg[t]) <= bound
            w = np.exp(lg - lg.max())
            w /= w.sum()
            ref = w @ ks.astype(np.float64)
            e = orc.compress_group4(ks, g)
            assert np.max(np.abs(e - ref)) <= 1e-5 * np.max(np.abs(ks))


def test_pack_ratio4_bookkeeping():
    rng = np.random.default_rng(3)
    cfg = orc.make_cfg(64, 16, 32, orc.SCALE_F32, 32, 64, 32, 8, 1.0, ratio=4)
    D, B, n_new, cap = 80, 2, 12, 10
    toks = _tokens(rng, D, n=B * n_new).reshape(B, n_new, D)
    g = (rng.standard_normal(D) / 8).astype(np.float32)
    idx = rng.integers(-127, 128, (B, n_new // 4, 32)).astype(np.int8)
    rb = orc.record_bytes(cfg, True)
    rec = np.zeros((B, cap, rb), np.uint8)
    ic = np.zeros((B, cap, 32), np.int8)
    n = np.array([0, 5], np.int32)
    assert orc.pack(cfg, toks, g, idx, rec, ic, n) == 0
    assert n.tolist() == [3, 8]
    for b, base in ((0, 0), (1, 5)):
        for i in range(3):
            want, _ = orc.quantize_entry(cfg, orc.compress_group4(toks[b, 4 * i:4 * i + 4], g))
            assert np.array_equal(rec[b, base + i], want)
            assert np.array_equal(ic[b, base + i], idx[b, i])
    with pytest.raises(ValueError):
        orc.pack(cfg, toks[:, :10], g, idx[:, :2], rec, ic, n)  # 10 tokens: not groups of 4
    with pytest.raises(ValueError):
        orc.pack(cfg, toks, g, idx, rec, ic, np.array([0, 8], np.int32))  # 8 + 3 > 10


def test_large_common_logit_offset():
    """Logits near 300 that differ by a few units: the weights come from the
    differences (exp of a logit itself would overflow fp32)."""
    rng = np.random.default_rng(21)
    D = 128
    ks = _tokens(rng, D)
    g = np.zeros(D, np.float32)
    g[0] = 1.0
    ks[:, 0] = np.array([300.0, 301.5, 299.0, 302.25], np.float32)
    e = orc.compress_group4(ks, g)
    lg = ks[:, 0].astype(np.float64)
    w = np.exp(lg - lg.max())
    w /= w.sum()
    ref = w @ ks.astype(np.float64)
    assert np.all(np.isfinite(e))
    assert np.max(np.abs(e - ref)) <= 1e-5 * np.max(np.abs(ks))
