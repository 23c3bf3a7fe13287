"""Pins of the oracle's 2:1 compression, FP4 group quantisation and pack.

Compression (a reading: one gate vector, softmax over the pair's two logits)
is pinned by invariants the reading fixes and by an independent numpy
evaluation of the softmax-weighted sum.  Quantisation is pinned by exact
round-trips of representable entries, the error bound of round-to-nearest
onto the E2M1 grid, and the record layout.
"""
import numpy as np
import pytest

from fp4_compressed_kv_b200 import synth


def _cfgs(orc):
    return {
        "f32": orc.make_cfg(64, 16, 32, orc.SCALE_F32, 32, 64, 32, 8, 80 ** -0.5),
        "ue4m3_g32": orc.make_cfg(512, 64, 32, orc.SCALE_UE4M3, 128, 512, 128, 64, 576 ** -0.5),
        "ue4m3_g64": orc.make_cfg(512, 64, 64, orc.SCALE_UE4M3, 128, 512, 128, 64, 576 ** -0.5),
    }


# ------------------------------------------------------------------ compression
def test_compress_equal_pair_is_identity(orc):
    rng = np.random.default_rng(1)
    k = rng.standard_normal(576).astype(np.float32)
    g = rng.standard_normal(576).astype(np.float32)
    assert np.array_equal(orc.compress_pair(k, k, g), k)


def test_compress_zero_gate_is_mean(orc):
    rng = np.random.default_rng(2)
    k0, k1 = rng.standard_normal((2, 576)).astype(np.float32)
    e = orc.compress_pair(k0, k1, np.zeros(576, np.float32))
    mean = ((k0.astype(np.float64) + k1.astype(np.float64)) / 2).astype(np.float32)
    assert np.array_equal(e, mean)


def test_compress_matches_softmax_of_two_logits(orc):
    rng = np.random.default_rng(3)
    for D, scale in ((80, 80 ** -0.5), (576, 576 ** -0.5), (576, 0.2)):
        for _ in range(50):
            k0, k1 = rng.standard_normal((2, D)).astype(np.float32)
            g = (rng.standard_normal(D) * scale).astype(np.float32)
            l0 = float(np.dot(g.astype(np.float64), k0.astype(np.float64)))
            l1 = float(np.dot(g.astype(np.float64), k1.astype(np.float64)))
            m = max(l0, l1)
            w0 = np.exp(l0 - m) / (np.exp(l0 - m) + np.exp(l1 - m))
            ref = w0 * k0.astype(np.float64) + (1 - w0) * k1.astype(np.float64)
            e = orc.compress_pair(k0, k1, g)
            assert np.max(np.abs(e - ref)) <= 1e-6 * (np.abs(k0).max() + np.abs(k1).max())
            terms = np.abs(g.astype(np.float64) * (k0.astype(np.float64) - k1.astype(np.float64)))
            assert abs(orc.gate_delta(k0, k1, g) - (l0 - l1)) <= 1e-6 * (terms.sum() + 1e-30)
            # a convex combination, up to the fp32 rounding of the two products
            lo, hi = np.minimum(k0, k1), np.maximum(k0, k1)
            slack = 4 * np.spacing(np.maximum(np.abs(lo), np.abs(hi)))
            assert np.all(e >= lo - slack) and np.all(e <= hi + slack)


def test_compress_dominant_token_wins(orc):
    D = 80
    k0 = np.ones(D, np.float32)
    k1 = -np.ones(D, np.float32)
    g = np.full(D, 10.0, np.float32)  # logit_0 - logit_1 = 1600
    assert np.array_equal(orc.compress_pair(k0, k1, g), k0)
    assert np.array_equal(orc.compress_pair(k1, k0, g), k0)


# ------------------------------------------------------------------ quantisation
def _groups(cfg):
    out = []
    for s in range(0, cfg.latent_dim, cfg.group):
        out.append((s, min(cfg.group, cfg.latent_dim - s)))
    for s in range(0, cfg.rope_dim, cfg.group):
        out.append((cfg.latent_dim + s, min(cfg.group, cfg.rope_dim - s)))
    return out


@pytest.mark.parametrize("name", ["f32", "ue4m3_g32", "ue4m3_g64"])
def test_quantize_exact_roundtrip(orc, name):
    cfg = _cfgs(orc)[name]
    D = cfg.latent_dim + cfg.rope_dim
    rng = np.random.default_rng(4)
    grid = np.array([orc.e2m1_value(c) for c in range(16)], np.float32)
    for trial in range(20):
        codes = rng.integers(0, 16, D)
        codes[(codes & 7) == 0] = 0
        scales = []
        x = np.empty(D, np.float32)
        for gi, (s0, n) in enumerate(_groups(cfg)):
            codes[s0] = 7 | (codes[s0] & 8)  # each group reaches +-6
            if cfg.scale_fmt == orc.SCALE_UE4M3:
                sb = int(rng.integers(0x08, 0x70))
                s = orc.e4m3_value(sb)
            else:
                s = float(np.float32(rng.integers(1, 2 ** 18) * 2.0 ** rng.integers(-30, -10)))
                sb = None
            scales.append((sb, s))
            x[s0:s0 + n] = grid[codes[s0:s0 + n]] * np.float32(s)
        rec, nf = orc.quantize_entry(cfg, x)
        assert nf == 0
        got_codes = np.empty(D, np.int64)
        got_codes[0::2] = rec[: D // 2] & 15
        got_codes[1::2] = rec[: D // 2] >> 4
        assert np.array_equal(got_codes, codes)
        if cfg.scale_fmt == orc.SCALE_UE4M3:
            assert list(rec[D // 2: D // 2 + len(scales)]) == [sb for sb, _ in scales]
        else:
            got = np.frombuffer(rec[D // 2: D // 2 + 4 * len(scales)].tobytes(), np.float32)
            assert np.array_equal(got, np.array([s for _, s in scales], np.float32))
        assert np.array_equal(orc.dequantize_entry(cfg, rec), x)
        assert not rec[orc.record_bytes(cfg, False):].any()


@pytest.mark.parametrize("name", ["f32", "ue4m3_g32", "ue4m3_g64"])
def test_quantize_error_bound(orc, name):
    cfg = _cfgs(orc)[name]
    D = cfg.latent_dim + cfg.rope_dim
    rng = np.random.default_rng(5)
    for _ in range(50):
        x = (rng.standard_normal(D) * np.where(rng.random(D) < 0.02, 10, 1)).astype(np.float32)
        rec, _ = orc.quantize_entry(cfg, x)
        y = orc.dequantize_entry(cfg, rec)
        for gi, (s0, n) in enumerate(_groups(cfg)):
            a = np.abs(x[s0:s0 + n]).max()
            if cfg.scale_fmt == orc.SCALE_UE4M3:
                s = orc.e4m3_value(rec[D // 2 + gi])
                assert abs(s - a / 6) <= a / 6 / 16 + 2.0 ** -10  # E4M3 has 3 mantissa bits
            else:
                s = float(np.frombuffer(rec[D // 2 + 4 * gi: D // 2 + 4 * gi + 4].tobytes(),
                                        np.float32)[0])
                assert s == np.float32(a) / np.float32(6)
            v = np.abs(x[s0:s0 + n]) / s
            half_step = np.where(v < 2, 0.25, np.where(v < 4, 0.5, 1.0))
            bound = (half_step + np.maximum(v - 6, 0)) * s * (1 + 1e-6)
            assert np.all(np.abs(y[s0:s0 + n] - x[s0:s0 + n]) <= bound)


def test_quantize_layout_and_special_groups(orc):
    cfg = _cfgs(orc)["ue4m3_g32"]
    D = 576
    x = np.zeros(D, np.float32)
    x[0], x[1] = 0.5, 1.0      # group 0: absmax 1 -> scale 1/6 rounds in E4M3
    x[32:64] = 1e-5            # group 1: absmax/6 below half the smallest subnormal -> 0
    x[512] = np.nan            # RoPE group 0: non-finite is counted and coded 0
    x[513] = 3.0
    rec, nf = orc.quantize_entry(cfg, x)
    assert nf == 1
    s0 = orc.e4m3_value(rec[288])
    assert rec[288] == orc.e4m3_encode(np.float32(1.0) / np.float32(6.0))
    assert rec[0] == orc.e2m1_encode(np.float32(0.5) / np.float32(s0)) | \
        (orc.e2m1_encode(np.float32(1.0) / np.float32(s0)) << 4)
    assert rec[289] == 0 and not rec[16:32].any()
    assert rec[256] & 15 == 0 and rec[288 + 16] == orc.e4m3_encode(np.float32(0.5))
    assert rec.size == 320 and not rec[306:].any()


# ------------------------------------------------------------------ pack
def test_pack_appends_and_advances(orc):
    w = synth.WORKLOADS["tiny"]
    inp = synth.make_inputs(w)
    cfg = orc.make_cfg(w.latent, w.rope, w.group, w.scale_fmt, w.idx_dim, w.topk, w.window,
                       w.heads, w.sm_scale)
    cap = w.entries + 8
    rb = orc.record_bytes(cfg)
    tok = inp["tokens"].float().numpy()
    idxk = inp["idx_k"].numpy()
    rec = np.zeros((w.batch, cap, rb), np.uint8)
    ic = np.zeros((w.batch, cap, w.idx_dim), np.int8)
    n = np.zeros(w.batch, np.int32)
    # two appends (first 600 tokens, then the rest) equal one append of all
    assert orc.pack(cfg, tok[:, :600], inp["gate"].numpy(), idxk[:, :300], rec, ic, n) == 0
    assert list(n) == [300]
    orc.pack(cfg, tok[:, 600:], inp["gate"].numpy(), idxk[:, 300:], rec, ic, n)
    assert list(n) == [512]
    rec2 = np.zeros_like(rec)
    ic2 = np.zeros_like(ic)
    n2 = np.zeros(w.batch, np.int32)
    orc.pack(cfg, tok, inp["gate"].numpy(), idxk, rec2, ic2, n2)
    assert np.array_equal(rec, rec2) and np.array_equal(ic, ic2)
    assert np.array_equal(ic[0, :512], idxk[0])
    # entry 7 is the quantised compression of tokens 14 and 15
    e = orc.compress_pair(tok[0, 14], tok[0, 15], inp["gate"].numpy())
    assert np.array_equal(rec[0, 7], orc.quantize_entry(cfg, e)[0])
    assert not rec[0, 512:].any()
    with pytest.raises(ValueError):
        orc.pack(cfg, tok[:, :20], inp["gate"].numpy(), idxk[:, :10], rec, ic, n)  # capacity
    with pytest.raises(ValueError):
        orc.pack(cfg, tok[:, :3], inp["gate"].numpy(), idxk[:, :1], rec, ic, n)  # odd n_new
