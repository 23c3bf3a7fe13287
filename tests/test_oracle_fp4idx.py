"""Pins of the oracle's FP4 indexer keys (R18): a key of 128 channels as
E2M1 codes with one UE4M3 scale per 16 channels is the 72 bytes the pages
count ("DeepSeek V1 到 V4.1-Flash ...", "890 字节是怎么算出来的"), and its
score against the int8 query is exact.

- Row size: 64 code bytes + 8 scale bytes = 72 B for 128 channels.
- Exactness: the int64 score equals 2^10 times the fp64 dot product of the
  query with the row decoded here independently (E2M1 from its bit layout,
  the scale from torch's float8_e4m3fn), on random and extreme rows.
- Special cases: zero rows and zero queries score 0; rows already on the
  grid score exactly 2^10 q . k.
- Top-K over the scores against a brute-force sort, with forced ties.
"""
import numpy as np
import pytest
import torch

import oracle as orc

DI = 128


def _cfg(topk=64):
    return orc.make_cfg(512, 64, 32, orc.SCALE_UE4M3, DI, topk, 128, 64, 1.0)


def _e2m1_from_bits(code):
    e, m, s = (code >> 1) & 3, code & 1, -1.0 if code & 8 else 1.0
    mag = m / 2 if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
    return s * mag


def _decode(row):
    """Independent decode of one FP4 indexer row to fp64."""
    codes = np.empty(DI, np.int64)
    codes[0::2] = row[: DI // 2] & 15
    codes[1::2] = row[: DI // 2] >> 4
    scales = torch.from_numpy(row[DI // 2:DI // 2 + DI // 16].copy()).view(torch.float8_e4m3fn)
    scales = scales.to(torch.float64).numpy()
    vals = np.array([_e2m1_from_bits(int(c)) for c in codes])
    return vals * np.repeat(scales, 16)


def test_row_is_72_bytes():
    qc = orc.idx_fp4_cfg(_cfg())
    assert orc.record_bytes(qc, False) == DI // 2 + DI // 16 == 72


@pytest.mark.parametrize("scale", [0.01, 1.0, 30.0, 300.0])
def test_scores_are_exact(scale):
    rng = np.random.default_rng(int(scale * 100))
    keys = (rng.standard_normal((40, DI)) * scale).astype(np.float32)
    rows = orc.idx_fp4_quantize(_cfg(), keys)
    for _ in range(5):
        q = rng.integers(-128, 128, DI).astype(np.int8)
        for j in range(40):
            want = q.astype(np.float64) @ _decode(rows[j])
            got = orc.idx_fp4_score(q, rows[j], DI)
            assert got == want * 1024.0, (j, got, want)


def test_extreme_rows_stay_below_2_to_36():
    q = np.full(DI, -128, np.int8)
    keys = np.full((2, DI), 6.0 * 448.0, np.float32)
    keys[1] *= -1
    rows = orc.idx_fp4_quantize(_cfg(), keys)
    s = [orc.idx_fp4_score(q, r, DI) for r in rows]
    assert s[0] == -s[1] and abs(s[0]) == 128 * 6 * 448 * DI * 1024 and abs(s[0]) < 2 ** 36


def test_zero_and_grid_rows():
    rng = np.random.default_rng(4)
    q = rng.integers(-128, 128, DI).astype(np.int8)
    zero = orc.idx_fp4_quantize(_cfg(), np.zeros((1, DI), np.float32))[0]
    assert not zero.any() and orc.idx_fp4_score(q, zero, DI) == 0
    # a row whose groups have absmax 6 x 2^e holds grid values exactly
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    k = rng.choice(grid, DI) * rng.choice([-1, 1], DI).astype(np.float32)
    k[::16] = 6.0
    k = k * np.repeat(2.0 ** rng.integers(-3, 4, DI // 16), 16).astype(np.float32)
    row = orc.idx_fp4_quantize(_cfg(), k[None])[0]
    assert orc.idx_fp4_score(q, row, DI) == int(q.astype(np.int64) @ (k.astype(np.float64) * 1024))
    assert orc.idx_fp4_score(np.zeros(DI, np.int8), row, DI) == 0


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(9)
    B, cap, K = 2, 700, 64
    keys = rng.standard_normal((B, cap, DI)).astype(np.float32)
    keys[0, 100:160] = keys[0, 5]   # 61 equal rows
    keys[1, :] = keys[1, 0]         # every row equal: ties to the lower index
    rows = np.stack([orc.idx_fp4_quantize(_cfg(K), keys[b]) for b in range(B)])
    q = rng.integers(-128, 128, (B, DI)).astype(np.int8)
    n = np.array([700, 650], np.int32)
    tk, sc = orc.index_topk_fp4(_cfg(K), q, rows, n, want_scores=True)
    for b in range(B):
        s = [orc.idx_fp4_score(q[b], rows[b, j], DI) for j in range(n[b])]
        assert np.array_equal(sc[b, :n[b]], s)
        order = sorted(range(n[b]), key=lambda j: (-s[j], j))[:K]
        assert tk[b].tolist() == sorted(order)
    assert tk[1].tolist() == list(range(K))


@pytest.mark.parametrize("n,k", [(0, 8), (5, 8), (1000, 64), (3000, 512)])
def test_topk64_brute_force(n, k):
    """The 64-bit selection: scores beyond 32 bits, many ties, K >= N."""
    rng = np.random.default_rng(n + k)
    s = rng.integers(-(1 << 36), 1 << 36, n)
    if n > 10:
        s[rng.choice(n, n // 3, replace=False)] = s[0]  # a third of them tie
    got = orc.topk64(s.astype(np.int64), k)
    order = sorted(range(n), key=lambda j: (-int(s[j]), j))[:k]
    assert got.tolist() == sorted(order) + [-1] * (k - min(k, n))
