"""Pins of the oracle's scalar pieces against what the pages and the formats fix.

- KV-size formula vs the worked examples printed on the pages (golden).
- Entry-size accounting vs the printed 288 / 72 / 900 / 1/437 numbers (golden).
- E2M1: the grid derived from the bit layout the pages state, the printed
  magnitude list, the tie table, saturation, and a brute-force sweep.
- E4M3 scales: decode of all 256 bytes and RNE encode vs torch's float8_e4m3fn.
- exp (fp32, gate only): against the C library's exp within 3 fp32 ulp.
"""
import math
import os
import random

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


UNITS = {"KB": 1000, "GiB": 2 ** 30, "B": 1, "num": 1}


def test_kv_size_worked_examples(orc):
    rows = list(_rows("kv_size.txt"))
    assert len(rows) == 6
    for src, L, H, D, b, tokens, printed, unit, tol in rows:
        total = orc.kv_bytes_per_token(int(L), int(H), int(D), int(b)) * int(tokens)
        value = total / UNITS[unit]
        assert abs(value - float(printed)) <= float(tol) * float(printed) + 1e-9, (src, value)
    # the exact figures quoted beside the approximations
    assert orc.kv_bytes_per_token(95, 8, 128, 2) == 389_120
    assert orc.kv_bytes_per_token(60, 64, 128, 2) * 65536 == 128_849_018_880
    assert orc.kv_bytes_per_token(60, 64, 128, 2) * 65536 // 4 == 30 * 2 ** 30


def test_entry_accounting(orc):
    g = {k: int(v) for k, v in _rows("accounting.txt")}
    assert g["mla_latent"] + g["mla_rope"] == g["mla_entry_numbers"]
    # MLA entry vs MHA's 2 x 8 heads x 128 (golden kv_size row c)
    assert orc.kv_bytes_per_token(1, 8, 128, 1) == 2048
    # FP4 latent entry: 16 channels per 1-byte FP8 scale (part 4 "P4 main KV")
    main = orc.make_cfg(512, 0, 16, orc.SCALE_UE4M3, 128, 512, 128, 64, 1.0)
    assert orc.record_bytes(main, padded=False) == g["fp4_main_entry_bytes"]
    idxk = orc.make_cfg(128, 0, 16, orc.SCALE_UE4M3, 128, 512, 128, 64, 1.0)
    assert orc.record_bytes(idxk, padded=False) == g["fp4_indexer_key_bytes"]
    per = g["fp4_main_entry_bytes"] + g["fp4_indexer_key_bytes"]
    assert per == g["main_plus_indexer"]
    assert 3 * per // 2 == g["encoder_bytes"] and per == g["decoder_bytes"]
    assert g["encoder_bytes"] + g["decoder_bytes"] == g["total_estimate"]
    assert round(g["v1_bytes"] / g["report_total"]) == g["reduction"]


def test_group_counts_and_record_sizes(orc):
    c2 = orc.make_cfg(512, 64, 32, orc.SCALE_UE4M3, 128, 512, 128, 64, 1.0)
    c3 = orc.make_cfg(512, 64, 64, orc.SCALE_UE4M3, 128, 512, 128, 64, 1.0)
    c1 = orc.make_cfg(64, 16, 32, orc.SCALE_F32, 32, 64, 32, 8, 1.0)
    assert orc.n_groups(512, 64, 32) == 18 and orc.n_groups(512, 64, 64) == 9
    assert orc.n_groups(64, 16, 32) == 3
    assert [orc.record_bytes(c, False) for c in (c2, c3, c1)] == [306, 297, 52]
    assert [orc.record_bytes(c, True) for c in (c2, c3, c1)] == [320, 304, 64]


def test_pages_entry_bytes_and_encoder_accounting(orc):
    """The pages' estimate of the bytes a token occupies ("DeepSeek V1 到
    V4.1-Flash ...", "890 字节是怎么算出来的"): an FP4 main-KV entry of 512
    latent channels with one FP8 scale per 16 channels is 512 x 0.5 + 32 =
    288 B, which is this format's record with no RoPE channels.  With the
    RoPE channels the record holds 576 codes and 36 scales; the encoder's 3
    caches (one per group, 2 tokens per entry) and the decoder's one cache
    then hold (3 x 6-layer + 20-layer) bytes as below."""
    page = orc.make_cfg(512, 0, 16, orc.SCALE_UE4M3, 128, 512, 128, 64, 1.0)
    assert orc.record_bytes(page, False) == 512 // 2 + 512 // 16 == 288
    enc = orc.make_cfg(512, 64, 16, orc.SCALE_UE4M3, 128, 512, 128, 64, 1.0)
    assert orc.record_bytes(enc, False) == 576 // 2 + 576 // 16 == 324
    dec = orc.make_cfg(512, 64, 32, orc.SCALE_UE4M3, 128, 512, 128, 64, 1.0)
    entries = 500_000  # 1M tokens, 2 per entry
    window = 128 * 576 * 2  # one bf16 window per layer
    enc_b = orc.bytes_resident(enc, entries, 6, 2, padded=False)
    dec_b = orc.bytes_resident(dec, entries, 20, 2, padded=False)
    assert enc_b == entries * (324 + 128) + 6 * window
    assert dec_b == entries * (306 + 128) + 20 * window
    per_token = (3 * enc_b + dec_b) / 1_000_000
    assert 900 < per_token < 901  # int8 indexer keys, RoPE channels included


def test_bytes_resident_stack1m(orc):
    c = orc.make_cfg(512, 64, 32, orc.SCALE_UE4M3, 128, 512, 128, 64, 1.0)
    # 500,000 x 306 + 500,000 x 128 + 20 layers x 128 x 576 x 2
    assert orc.bytes_resident(c, 500_000, 20, 2, padded=False) == 219_949_120
    assert orc.bytes_resident(c, 500_000, 20, 2, padded=True) == 500_000 * 448 + 2_949_120


# ------------------------------------------------------------------ E2M1
def _e2m1_grid_from_bits():
    """E2M1 magnitudes from the bit layout: 2 exponent bits (bias 1), 1 mantissa bit."""
    mags = []
    for e in range(4):
        for m in range(2):
            mags.append(m / 2 if e == 0 else 2.0 ** (e - 1) * (1 + m / 2))
    return mags


def test_e2m1_grid(orc):
    printed = [float(x) for x in next(r for r in _rows("e2m1.txt") if r[0] == "magnitudes")[1:]]
    assert _e2m1_grid_from_bits() == printed
    assert [orc.e2m1_value(c) for c in range(8)] == printed
    assert [orc.e2m1_value(c | 8) for c in range(8)] == [-x for x in printed]
    # every code round-trips, with any positive scale that keeps v exact
    for c in range(16):
        v = orc.e2m1_value(c)
        expect = 0 if (c & 7) == 0 else c
        assert orc.e2m1_encode(v) == expect


def test_e2m1_ties_and_saturation(orc):
    for kind, x, y in ((r[0], r[1], r[2]) for r in _rows("e2m1.txt") if r[0] in ("tie", "sat")):
        for sign in (1, -1):
            v = sign * float(x)
            got = orc.e2m1_value(orc.e2m1_encode(v))
            want = sign * float(y)
            assert got == want or (want == 0 and got == 0), (kind, v, got)
    assert orc.e2m1_encode(-0.0) == 0 and orc.e2m1_encode(-0.2) == 0


def test_e2m1_brute_force_sweep(orc):
    grid = np.array(_e2m1_grid_from_bits())
    rng = np.random.default_rng(5)
    xs = np.concatenate([np.arange(-7.5, 7.5, 1 / 64), rng.uniform(-8, 8, 2000)]).astype(np.float32)
    for x in xs:
        m = abs(float(x))
        d = np.abs(grid - m)
        best = np.flatnonzero(d == d.min())
        code = int(best[0]) if len(best) == 1 else int(best[best % 2 == 0][0])
        want = grid[code] * (1 if x >= 0 else -1)
        assert orc.e2m1_value(orc.e2m1_encode(float(x))) == want, x


# ------------------------------------------------------------------ E4M3
def test_e4m3_decode_all_bytes(orc):
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float()
    for b in range(256):
        got, want = orc.e4m3_value(b), float(ref[b])
        if math.isnan(want):
            assert math.isnan(got)
        else:
            assert got == want, b
    assert orc.e4m3_value(0x7E) == 448.0 and orc.e4m3_value(1) == 2.0 ** -9
    for b in range(0x7F):  # every finite non-negative byte round-trips
        assert orc.e4m3_encode(orc.e4m3_value(b)) == b


def test_e4m3_encode_matches_torch_rne(orc):
    rng = np.random.default_rng(6)
    xs = np.concatenate([
        np.exp(rng.uniform(math.log(2 ** -12), math.log(447.0), 4000)),
        # exact midpoints between neighbouring representable values
        [(orc.e4m3_value(b) + orc.e4m3_value(b + 1)) / 2 for b in range(0x7D)],
    ]).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for x, r in zip(xs, ref):
        assert orc.e4m3_encode(float(x)) == int(r), float(x)
    assert orc.e4m3_encode(1000.0) == 0x7E and orc.e4m3_encode(0.0) == 0


# ------------------------------------------------------------------ exp
def _f32_ulp(x):
    x = np.float32(abs(x))
    return float(np.spacing(x))


def test_expf_within_three_ulp(orc):
    rnd = random.Random(7)
    xs = [rnd.uniform(-87, 88) for _ in range(20000)] + [rnd.uniform(-2, 2) for _ in range(20000)]
    xs += [0.0, 1.0, -1.0, 0.5 * math.log(2), -0.5 * math.log(2), 87.9, -86.9]
    for x in xs:
        x = float(np.float32(x))
        got, want = orc.expf(x), math.exp(x)
        assert abs(got - want) <= 3 * _f32_ulp(want), x
    assert orc.expf(0.0) == 1.0
    assert orc.expf(89.0) == math.inf and orc.expf(-88.0) == 0.0
