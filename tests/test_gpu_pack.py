"""GPU pack (2:1 compression + FP4 group quantisation + indexer append) vs the
oracle: bit-exact records (codes, scales, zero padding) and indexer rows."""
import numpy as np
import pytest
import torch

import oracle
from fp4_compressed_kv_b200 import synth
from helpers import Guarded, f32, oracle_cfg, oracle_pack

pytestmark = pytest.mark.gpu


def _gpu_pack(kvc, w, tokens, gate, idx_k, capacity=None, chunks=None):
    """Pack into a cache whose record and indexer arrays sit between canary
    regions (checked after the appends)."""
    cfg = kvc.config_for(w)
    B, T = tokens.shape[:2]
    cache = kvc.Cache(cfg, B, capacity or T // 2)
    grec = Guarded(cache.records.shape, cache.records.dtype, fill=0)
    gidx = Guarded(cache.idx_k.shape, cache.idx_k.dtype, fill=0)
    cache.records, cache.idx_k = grec.t, gidx.t
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    step = chunks or T
    for t0 in range(0, T, step):
        kvc.pack(cfg, tokens[:, t0:t0 + step].contiguous(), gate,
                 idx_k[:, t0 // 2:(t0 + step) // 2].contiguous(), cache, status=st)
    grec.check()
    gidx.check()
    return cache, int(st.item())


@pytest.mark.parametrize("name", ["tiny", "mla32k"])
def test_pack_bit_exact_full(kvc, name):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w)  # CPU generator
    rec, ic, n, ost = oracle_pack(w, inp["tokens"], inp["gate"], inp["idx_k"])
    cache, st = _gpu_pack(kvc, w, inp["tokens"].cuda(), inp["gate"].cuda(), inp["idx_k"].cuda())
    assert st == ost == 0
    assert cache.n_entries.cpu().tolist() == n.tolist()
    g = cache.records.cpu().numpy()
    diff = np.argwhere(g != rec)
    assert diff.size == 0, f"{len(diff)} bytes differ, first {diff[:5].tolist()}"
    assert np.array_equal(cache.idx_k.cpu().numpy(), ic)


def test_pack_group64_batch_ragged_appends(kvc):
    """Group 64 (the batched workload's format), 3 sequences, appends in odd-sized pieces."""
    w = synth.WORKLOADS["batch32x128k"].scaled(batch=3, context=3000)
    inp = synth.make_inputs(w)
    rec, ic, n, _ = oracle_pack(w, inp["tokens"], inp["gate"], inp["idx_k"], capacity=1600)
    cache, st = _gpu_pack(kvc, w, inp["tokens"].cuda(), inp["gate"].cuda(), inp["idx_k"].cuda(),
                          capacity=1600, chunks=998)
    assert st == 0
    assert cache.n_entries.cpu().tolist() == [1500] * 3
    assert np.array_equal(cache.records.cpu().numpy(), rec)
    assert np.array_equal(cache.idx_k.cpu().numpy(), ic)


def test_pack_capacity_and_nonfinite_flags(kvc):
    w = synth.WORKLOADS["mla32k"].scaled(context=64)
    inp = synth.make_inputs(w)
    tok = inp["tokens"].clone()
    tok[0, 5, 17] = float("nan")
    tok[0, 9, 600 - 64] = float("inf")
    rec, ic, n, ost = oracle_pack(w, tok, inp["gate"], inp["idx_k"])
    cache, st = _gpu_pack(kvc, w, tok.cuda(), inp["gate"].cuda(), inp["idx_k"].cuda())
    assert ost == oracle.ST_NONFINITE and st == kvc.DEV_NONFINITE
    assert np.array_equal(cache.records.cpu().numpy(), rec)
    # one more pair does not fit: sequence unchanged, capacity bit set
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    before = cache.records.clone()
    kvc.pack(kvc.config_for(w), tok[:, :2].cuda().contiguous(), inp["gate"].cuda(),
             inp["idx_k"][:, :1].cuda().contiguous(), cache, status=st2)
    torch.cuda.synchronize()
    assert st2.item() == kvc.DEV_CAPACITY
    assert cache.n_entries.item() == 32 and torch.equal(cache.records, before)


@pytest.mark.parametrize("name", ["batch32x128k", "mla32k"])
def test_pack_stream_nonfinite(kvc, name):
    """Appends of more than 4096 entries take the streaming kernel, whose
    group maxima propagate NaN and whose warps redo a chunk value by value
    when they meet a non-finite value: a NaN (the whole entry's gate goes
    NaN), +inf and -inf in different sequences and groups, against the oracle
    byte for byte."""
    w = synth.WORKLOADS[name].scaled(batch=3, context=2 * 3000)
    inp = synth.make_inputs(w)
    tok = inp["tokens"].clone()
    tok[1, 100, 5] = float("nan")
    tok[2, 2001, w.dim - 6] = float("inf")
    tok[0, 4000, 300] = float("-inf")
    rec, ic, n, ost = oracle_pack(w, tok, inp["gate"], inp["idx_k"])
    cache, st = _gpu_pack(kvc, w, tok.cuda(), inp["gate"].cuda(), inp["idx_k"].cuda())
    assert ost == oracle.ST_NONFINITE and st == kvc.DEV_NONFINITE
    g = cache.records.cpu().numpy()
    diff = np.argwhere(g != rec)
    assert diff.size == 0, f"{len(diff)} bytes differ, first {diff[:5].tolist()}"
    assert np.array_equal(cache.idx_k.cpu().numpy(), ic)


def test_pack_rejects_tokens_not_16_byte_aligned(kvc):
    """Token rows arrive by 16-byte loads and bulk copies: a start 2 bytes
    past a 16-byte boundary is refused before any work (KVC_ERR_INVALID),
    and the cache is untouched."""
    w = synth.WORKLOADS["batch32x128k"].scaled(batch=2, context=2 * 2600)
    inp = synth.make_inputs(w)
    tok = inp["tokens"]
    flat = torch.empty(tok.numel() + 8, dtype=tok.dtype, device="cuda")
    shifted = flat[1:1 + tok.numel()].view(tok.shape)
    shifted.copy_(tok.cuda())
    assert shifted.data_ptr() % 16 == 2 and shifted.is_contiguous()
    cfg = kvc.config_for(w)
    cache = kvc.Cache(cfg, 2, 2600)
    with pytest.raises(kvc.KvcError) as e:
        kvc.pack(cfg, shifted, inp["gate"].cuda(), inp["idx_k"].cuda(), cache)
    assert e.value.status == 1  # KVC_ERR_INVALID
    torch.cuda.synchronize()
    assert cache.n_entries.cpu().tolist() == [0, 0]


def test_pack_host_validation(kvc):
    w = synth.WORKLOADS["tiny"]
    cfg = kvc.config_for(w)
    cache = kvc.Cache(cfg, 1, 16)
    tok = torch.zeros(1, 3, 80, device="cuda")
    with pytest.raises(kvc.KvcError):
        kvc.pack(cfg, tok, torch.zeros(80, device="cuda"), torch.zeros(1, 1, 32, dtype=torch.int8,
                                                                        device="cuda"), cache)
    bad = kvc.config_for(w)
    bad.group = 48
    with pytest.raises(kvc.KvcError):
        kvc.pack(bad, tok[:, :2].contiguous(), torch.zeros(80, device="cuda"),
                 torch.zeros(1, 1, 32, dtype=torch.int8, device="cuda"), cache)


def test_codecs_match_oracle(kvc):
    """Hardware E2M1 / E4M3 conversions against the oracle's nearest-even search."""
    rng = np.random.default_rng(0)
    grid = np.array([oracle.e2m1_value(c) for c in range(8)])
    mids = (grid[1:] + grid[:-1]) / 2
    xs = np.concatenate([grid, -grid, mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 9),
                         rng.uniform(-7, 7, 20000), [7.0, -100.0, 1e30, -0.0]]).astype(np.float32)
    codes = torch.empty(xs.size, dtype=torch.uint8, device="cuda")
    kvc.e2m1_encode(torch.from_numpy(xs).cuda(), codes)
    want = np.array([oracle.e2m1_encode(float(x)) for x in xs])
    got = codes.cpu().numpy()
    assert np.array_equal(got, want), xs[got != want][:10]
    vals = np.array([oracle.e4m3_value(b) for b in range(0x7F)])
    ys = np.concatenate([vals, (vals[1:] + vals[:-1]) / 2, np.exp(rng.uniform(-14, 6.2, 20000)),
                         [500.0, 1e9, 0.0]]).astype(np.float32)
    out = torch.empty(ys.size, dtype=torch.uint8, device="cuda")
    kvc.e4m3_encode(torch.from_numpy(ys).cuda(), out)
    want = np.array([oracle.e4m3_encode(float(y)) for y in ys])
    assert np.array_equal(out.cpu().numpy(), want)


@pytest.mark.parametrize("name,batch,context", [("batch32x128k", 2, 2 * 4200),
                                                 ("mla32k", 1, 2 * 300)])
def test_pack_team_and_warp_variants(kvc, name, batch, context):
    """Large appends take the 8-lanes-per-entry kernel, small ones the
    warp-per-entry kernel; both must give the oracle's bytes."""
    w = synth.WORKLOADS[name].scaled(batch=batch, context=context)
    inp = synth.make_inputs(w)
    rec, ic, n, _ = oracle_pack(w, inp["tokens"], inp["gate"], inp["idx_k"])
    cache, st = _gpu_pack(kvc, w, inp["tokens"].cuda(), inp["gate"].cuda(), inp["idx_k"].cuda())
    assert st == 0 and cache.n_entries.cpu().tolist() == n.tolist()
    assert np.array_equal(cache.records.cpu().numpy(), rec)
    # one pair at a time (the decode append) gives the same bytes as one append
    cache2, _ = _gpu_pack(kvc, w, inp["tokens"][:, :64].cuda().contiguous(), inp["gate"].cuda(),
                          inp["idx_k"][:, :32].cuda().contiguous(), capacity=w.entries, chunks=2)
    assert np.array_equal(cache2.records.cpu().numpy()[:, :32], rec[:, :32])


def _midpoint_tokens(w, batch, pairs, seed):
    """Token pairs (k, k) whose entries land on and next to the E2M1 rounding
    midpoints: each group holds 6*s (so the group scale is s exactly), then
    s times midpoints {0.25, ..., 5}, grid points, and their nearest neighbours
    in the token dtype.  With a zero gate both weights are 1/2 and the entry is
    k exactly, so x / s falls on a midpoint or a unit in the last place away."""
    rng = np.random.default_rng(seed)
    dt = w.torch_dtype
    D = w.dim
    # midpoints and grid points below the group maximum 6 (which sets s)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0])
    scales = np.array([1.0, 0.75, 0.125, 3.0, 0.009765625])  # exact in E4M3, fp32 and bf16
    ent = np.empty((batch, pairs, D), np.float32)
    for b in range(batch):
        s = scales[rng.integers(0, len(scales), pairs)][:, None]
        v = torch.from_numpy((rng.choice(mids, (pairs, D)) * s).astype(np.float32)).to(dt)
        step = rng.integers(-1, 2, (pairs, D))  # -1, 0, +1 units in the last place
        up = torch.nextafter(v, torch.full_like(v, np.inf))
        dn = torch.nextafter(v, torch.full_like(v, -np.inf))
        v = torch.where(torch.from_numpy(step == 1), up, torch.where(torch.from_numpy(step == -1),
                                                                     dn, v))
        v = v.float().numpy() * rng.choice([-1.0, 1.0], (pairs, D))
        for g0 in list(range(0, w.latent, w.group)) + list(range(w.latent, D, w.group)):
            v[:, g0] = 6.0 * s[:, 0]
        ent[b] = v
    tok = torch.from_numpy(np.repeat(ent, 2, axis=1)).to(dt)
    return tok


@pytest.mark.parametrize("name,pairs", [("tiny", 300), ("tiny", 4100), ("mla32k", 200),
                                        ("mla32k", 2100)])
def test_pack_rounding_midpoints(kvc, name, pairs):
    """Both append kernels (warp per entry, 8 lanes per entry) against the
    oracle's exact division on quotients at and beside the rounding midpoints."""
    w = synth.WORKLOADS[name]
    batch = 2
    tok = _midpoint_tokens(w, batch, pairs, seed=7)
    assert torch.equal(tok[:, 0::2], tok[:, 1::2])
    gate = torch.zeros(w.dim, dtype=torch.float32)
    idx = torch.zeros(batch, pairs, w.idx_dim, dtype=torch.int8)
    rec, ic, n, ost = oracle_pack(w, tok, gate, idx)
    assert ost == 0
    cache, st = _gpu_pack(kvc, w, tok.cuda(), gate.cuda(), idx.cuda())
    assert st == 0
    got = cache.records.cpu().numpy()
    diff = np.argwhere(got != rec)
    assert diff.size == 0, f"{len(diff)} bytes differ, first {diff[:5].tolist()}"


@pytest.mark.parametrize("group", [8, 16, 32, 64])
def test_pack_ring_groups_ragged(kvc, group):
    """Appends of more than 4096 bf16 entries run the ring kernel (units of 16
    entries streamed through shared memory, one CTA per SM): every group width
    it takes, four sequences whose appends are not a multiple of the unit, the
    second append continuing a partly filled cache; byte for byte against the
    oracle."""
    w = synth.WORKLOADS["batch32x128k"].scaled(batch=4, context=2 * 2731, group=group)
    inp = synth.make_inputs(w)
    rec, ic, n, ost = oracle_pack(w, inp["tokens"], inp["gate"], inp["idx_k"])
    assert ost == 0
    cache, st = _gpu_pack(kvc, w, inp["tokens"].cuda(), inp["gate"].cuda(), inp["idx_k"].cuda(),
                          chunks=2 * 1366)
    assert st == 0
    assert cache.n_entries.cpu().tolist() == n.tolist() == [2731] * 4
    g = cache.records.cpu().numpy()
    diff = np.argwhere(g != rec)
    assert diff.size == 0, f"{len(diff)} bytes differ, first {diff[:5].tolist()}"
    assert np.array_equal(cache.idx_k.cpu().numpy(), ic)


def test_pack_ring_capacity(kvc):
    """A long append that one sequence has no room for: that sequence is left
    untouched and KVC_DEV_CAPACITY is set; the others are packed at their own
    offsets exactly as the oracle packs them."""
    w = synth.WORKLOADS["batch32x128k"].scaled(batch=3, context=2 * 2000)
    inp = synth.make_inputs(w)
    rec, ic, n, _ = oracle_pack(w, inp["tokens"], inp["gate"], inp["idx_k"])
    cfg = kvc.config_for(w)
    cache = kvc.Cache(cfg, 3, 2100)
    grec = Guarded(cache.records.shape, cache.records.dtype, fill=0)
    cache.records = grec.t
    cache.n_entries.copy_(torch.tensor([0, 200, 50], dtype=torch.int32))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvc.pack(cfg, inp["tokens"].cuda(), inp["gate"].cuda(), inp["idx_k"].cuda(), cache, status=st)
    torch.cuda.synchronize()
    grec.check()
    assert st.item() == kvc.DEV_CAPACITY
    assert cache.n_entries.cpu().tolist() == [2000, 200, 2050]
    g = cache.records.cpu().numpy()
    assert not g[1].any()
    assert np.array_equal(g[0, :2000], rec[0]) and not g[0, 2000:].any()
    assert np.array_equal(g[2, 50:2050], rec[2]) and not g[2, :50].any()
    gi = cache.idx_k.cpu().numpy()
    assert np.array_equal(gi[0, :2000], ic[0]) and np.array_equal(gi[2, 50:2050], ic[2])
    assert not gi[1].any()
