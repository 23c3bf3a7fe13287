"""The oracle's packed records against an fp64 evaluation of the compression.

The pages ("DeepSeek V1 到 V4.1-Flash ..." part 3 breakthrough 4: two tokens
become one cache entry; part 4 "P4 main KV": E2M1 codes with 8-bit scales;
"DeepSeek V4.1 Flash KV Cache压缩实战" 3.1, 3.2, 4.3) fix what an entry is -- the
softmax-weighted sum of its tokens -- but not the precision or the order in
which the gate logits are summed.  The oracle takes one fp32 order (a
reading).  This test does not use that order at all: it evaluates the gate
from exact products (each fp32 x bf16 or fp32 x fp32 product is exact in
fp64) summed with math.fsum (correctly rounded), the softmax weights and the
weighted sum in fp64, and rounds the entry to fp32 once.  It then quantises
that entry with its own code -- the group maximum, absmax/6 as an IEEE fp32
division, torch's round-to-nearest-even cast to float8_e4m3fn for UE4M3
scales, and round-to-nearest-even onto the E2M1 grid -- and compares the
records byte for byte with the oracle's orc_pack.

A code or scale byte may differ only where the two entries straddle a rounding
decision: each differing nibble must have its fp64 quotient within the
oracle's proven entry error (divided by the scale) of an E2M1 midpoint, and
each differing scale byte must have an E4M3 rounding midpoint between the two
sides' absmax/6.  The entry error bound is derived below; the test also checks
every oracle entry against it before quantisation.  The share of differing
nibbles is reported and bounded.
"""
import math

import numpy as np
import pytest
import torch

from fp4_compressed_kv_b200 import synth

U32 = 2.0 ** -24  # unit roundoff of fp32
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
MID = (E2M1[1:] + E2M1[:-1]) / 2  # 0.25 0.75 1.25 1.75 2.5 3.5 5


def _groups(latent, rope, group):
    out = []
    for base, n in ((0, latent), (latent, rope)):
        for s in range(0, n, group):
            out.append((base + s, min(group, n - s)))
    return out


def _fsum_dot(g, k):
    """Correctly rounded g . k for each row of k (every product exact in fp64)."""
    prods = (k.astype(np.float64) * g.astype(np.float64)).tolist()
    return np.array([math.fsum(r) for r in prods])


def exact_entries(toks, g):
    """toks [n][r][D] (fp32 holding the inputs) -> fp64 entries [n][D], the
    fp64 weights [n][r] and the absolute gate sums sum_d |g_d k_d| [n][r]."""
    n, r, D = toks.shape
    logits = np.stack([_fsum_dot(g, toks[:, t]) for t in range(r)], 1)
    m = logits.max(1, keepdims=True)
    e = np.exp(logits - m)
    w = e / e.sum(1, keepdims=True)
    ent = np.einsum("nt,ntd->nd", w, toks.astype(np.float64))
    absg = np.stack([np.abs(toks[:, t].astype(np.float64) * g.astype(np.float64)).sum(1)
                     for t in range(r)], 1)
    return ent, w, absg


def entry_error_bound(toks, w, absg):
    """Bound on |oracle fp32 entry - exact entry| per channel.

    Each fp32 logit (or the pair's logit difference) is a sum of D products
    taken as 8 partial sums of at most ceil(D/64)*8 fused terms plus a 3-level
    tree, so its error is below (D/8 + 4) u times the sum of the absolute
    terms.  The weights are smooth in the logits with |dw_t/dl_s| <= 1/4 (two
    tokens) or <= w_t (four tokens; a shift of one logit by x moves every
    weight by at most w_t |x|); the own fp32 exp (within 3 ulps), the sum
    and the division add below 8 u relative.  The weighted sum takes one
    rounding per fused step (r - 1 of them, plus the product).  Each part is
    doubled for slack."""
    n, r, D = toks.shape
    k = toks.astype(np.float64)
    n_terms = D / 8 + 4
    if r == 2:
        dl = n_terms * U32 * (absg[:, 0] + absg[:, 1])  # error of logit_0 - logit_1
        dw = 0.25 * dl + 8 * U32  # absolute error of w0 (and of w1 = 1 - w0)
        spread = np.abs(k[:, 0] - k[:, 1])  # e = k1 + w0 (k0 - k1)
        err = dw[:, None] * spread + 3 * U32 * (np.abs(w[:, 0, None] * k[:, 0]) +
                                                np.abs(w[:, 1, None] * k[:, 1]))
    else:
        dl = n_terms * U32 * absg.max(1)  # every logit's error, and the max's
        dw = (2 * dl[:, None] + 8 * U32) * w  # absolute error of each weight
        err = np.einsum("nt,ntd->nd", dw, np.abs(k))
        err += (r + 1) * U32 * np.einsum("nt,ntd->nd", w, np.abs(k))
    return 2 * err + 1e-45


def quantise(cfg, ent32, f32_scale):
    """Records of fp32 entries [n][D] by this test's own codec: (codes
    [n][D] int, scale bytes [n][G] uint8 (UE4M3) or fp32 scales, decoded
    scales [n][G])."""
    n, D = ent32.shape
    groups = _groups(cfg["latent"], cfg["rope"], cfg["group"])
    codes = np.zeros((n, D), np.int64)
    sb = np.zeros((n, len(groups)), np.float32 if f32_scale else np.uint8)
    sdec = np.zeros((n, len(groups)), np.float64)
    for gi, (s0, ln) in enumerate(groups):
        x = ent32[:, s0:s0 + ln]
        a = np.abs(x).max(1)
        s = (a / np.float32(6.0)).astype(np.float32)  # IEEE fp32 division
        if f32_scale:
            sb[:, gi] = s
            sd = s
        else:
            f8 = torch.from_numpy(s).to(torch.float8_e4m3fn)
            sb[:, gi] = f8.view(torch.uint8).numpy()
            sd = f8.float().numpy()
        sdec[:, gi] = sd
        with np.errstate(divide="ignore", invalid="ignore"):
            v = (x / sd[:, None].astype(np.float32)).astype(np.float32)  # fp32 division
        mag = np.abs(v).astype(np.float64)
        idx = np.searchsorted(MID, mag, side="left")  # midpoints strictly below
        tie = (idx < 7) & (mag == MID[np.minimum(idx, 6)])
        idx = np.where(tie & (idx % 2 == 1), idx + 1, idx)  # a tie goes to the even code
        idx = np.where(sd[:, None] > 0, idx, 0)
        c = np.where((x < 0) & (idx > 0), idx | 8, idx)
        codes[:, s0:s0 + ln] = c
    return codes, sb, sdec


def oracle_records(orc, cfg_o, toks, g):
    """orc_pack over toks [n][r][D]: records [n][rb] and its entries."""
    n, r, D = toks.shape
    rb = orc.record_bytes(cfg_o)
    rec = np.zeros((1, n, rb), np.uint8)
    ic = np.zeros((1, n, 8), np.int8)
    cnt = np.zeros(1, np.int32)
    cfg_o.idx_dim = 8
    st = orc.pack(cfg_o, toks.reshape(1, n * r, D), g, np.zeros((1, n, 8), np.int8), rec, ic,
                  cnt)
    assert st == 0 and cnt[0] == n
    return rec[0]


def unpack(cfg, rec, f32_scale):
    D = cfg["latent"] + cfg["rope"]
    codes = np.zeros((rec.shape[0], D), np.int64)
    codes[:, 0::2] = rec[:, :D // 2] & 15
    codes[:, 1::2] = rec[:, :D // 2] >> 4
    ng = len(_groups(cfg["latent"], cfg["rope"], cfg["group"]))
    if f32_scale:
        sb = rec[:, D // 2:D // 2 + 4 * ng].copy().view(np.float32)
    else:
        sb = rec[:, D // 2:D // 2 + ng]
    return codes, sb


CASES = {
    # workload, ratio, entries
    "tiny_g32_f32": ("tiny", 2, 100_000),
    "mla32k_g32": ("mla32k", 2, 100_000),
    "batch32x128k_g64": ("batch32x128k", 2, 100_000),
    "mla32k_g32_ratio4": ("mla32k", 4, 100_000),
}


@pytest.mark.parametrize("case", list(CASES))
def test_oracle_records_match_fp64_compression(orc, case):
    wname, ratio, n_total = CASES[case]
    w = synth.WORKLOADS[wname].scaled(ratio=ratio)
    cfg = {"latent": w.latent, "rope": w.rope, "group": w.group}
    f32_scale = w.scale_fmt == synth.SCALE_F32
    cfg_o = orc.make_cfg(w.latent, w.rope, w.group, w.scale_fmt, w.idx_dim, w.topk, w.window,
                         w.heads, w.sm_scale, ratio=ratio)
    D = w.dim
    gen = synth.generator("cpu", 4242 + w.seed + ratio)
    g = (torch.randn(D, generator=gen) / math.sqrt(D)).float().numpy()
    groups = _groups(w.latent, w.rope, w.group)

    n_nib = n_diff = n_sdiff = 0
    worst_entry = 0.0
    chunk = 10_000
    for c0 in range(0, n_total, chunk):
        toks = synth._keys(w, (chunk * ratio,), gen, "cpu").float().numpy()
        toks = toks.reshape(chunk, ratio, D)
        ent, wts, absg = exact_entries(toks, g)
        bound = entry_error_bound(toks, wts, absg)

        # the oracle's fp32 entries against the exact ones, before quantisation
        sample = range(0, chunk, 97)
        for i in sample:
            if ratio == 2:
                e_o = orc.compress_pair(toks[i, 0], toks[i, 1], g)
            else:
                e_o = orc.compress_group4(toks[i], g)
            dev = np.abs(e_o.astype(np.float64) - ent[i])
            assert np.all(dev <= bound[i]), (case, i, float((dev / bound[i]).max()))
            worst_entry = max(worst_entry, float((dev / bound[i]).max()))

        ent32 = ent.astype(np.float32)  # one rounding of the exact entry
        codes_i, sb_i, sd_i = quantise(cfg, ent32, f32_scale)
        rec_o = oracle_records(orc, cfg_o, toks, g)
        codes_o, sb_o = unpack(cfg, rec_o, f32_scale)
        # padding bytes are zero
        used = D // 2 + len(groups) * (4 if f32_scale else 1)
        assert not rec_o[:, used:].any()

        for gi, (s0, ln) in enumerate(groups):
            a_ex = np.abs(ent[:, s0:s0 + ln]).max(1)
            a_b = bound[:, s0:s0 + ln].max(1)  # the exact absmax moves by at most this
            sdiff = sb_i[:, gi] != sb_o[:, gi]
            if f32_scale:
                # fp32 scales: the oracle's absmax/6 lies within the entry error
                # of the exact one (plus the division's rounding)
                s_o = sb_o[:, gi].astype(np.float64)
                assert np.all(np.abs(s_o - a_ex / 6) <= a_b / 6 + 2 * U32 * s_o), (case, gi)
                sd_o = s_o
                rescale = np.abs(sd_o - sd_i[:, gi]) / np.maximum(sd_i[:, gi], 1e-300)
                same = np.ones(chunk, bool)  # codes compared in every group
            else:
                if sdiff.any():
                    # a UE4M3 scale byte may differ only across a rounding decision
                    # of absmax/6: an E4M3 midpoint lies within the entry error
                    lo = ((a_ex[sdiff] - a_b[sdiff]) / 6).astype(np.float32)
                    hi = ((a_ex[sdiff] + a_b[sdiff]) / 6).astype(np.float32)
                    f_lo = torch.from_numpy(lo).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
                    f_hi = torch.from_numpy(hi).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
                    so = sb_o[sdiff, gi]
                    assert np.all((f_lo != f_hi) & (so >= f_lo) & (so <= f_hi)), (case, gi)
                    n_sdiff += int(sdiff.sum())
                rescale = np.zeros(chunk)
                same = ~sdiff  # a group whose scale byte moved: every code may move
            ci, co = codes_i[same, s0:s0 + ln], codes_o[same, s0:s0 + ln]
            n_nib += ci.size
            d = ci != co
            if d.any():
                rows, cols = np.nonzero(d)
                sd = sd_i[same, gi][rows]
                q = np.abs(ent[same, s0:s0 + ln][rows, cols]) / sd
                qb = bound[same, s0:s0 + ln][rows, cols] / sd + q * rescale[same][rows]
                dist = np.abs(q[:, None] - MID[None, :]).min(1)
                # the two quotients straddle a midpoint: within the entry's
                # error of it (plus the quotient's own fp32 rounding)
                assert np.all(dist <= qb + 4 * U32 * (q + 1)), (case, gi, float(dist.max()))
                n_diff += int(d.sum())
    frac = n_diff / max(1, n_nib)
    print(f"{case}: {n_diff} of {n_nib} nibbles differ ({frac:.2e}), {n_sdiff} scale bytes, "
          f"worst entry deviation {worst_entry:.2f} of its bound")
    assert frac <= 1e-4
    assert n_sdiff <= 1e-3 * n_total * len(groups)  # UE4M3 scale bytes that moved
