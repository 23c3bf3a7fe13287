"""GPU indexer scores and top-K vs the oracle: bit-exact int32 scores and
index sets (ties to the lower index), ragged lengths, K >= N, forced ties
(including the heavy-tie path that overflows the candidate list)."""
import numpy as np
import pytest
import torch

import oracle
from fp4_compressed_kv_b200 import synth
from helpers import Guarded, oracle_cfg, topk_set_equal

pytestmark = pytest.mark.gpu


def _run(kvc, w, idx_k, idx_q, n_entries, capacity):
    cfg = kvc.config_for(w)
    B = idx_k.shape[0]
    cache = kvc.Cache(cfg, B, capacity)
    cache.idx_k[:, : idx_k.shape[1]] = idx_k.cuda()
    cache.n_entries.copy_(torch.as_tensor(n_entries, dtype=torch.int32))
    tk = Guarded((B, w.topk), torch.int32)  # canary-guarded outputs, checked after the call
    sc = Guarded((B, capacity), torch.int32, fill=0)
    ws = kvc.workspace(cfg, B, capacity)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvc.index_topk(cfg, idx_q.cuda().contiguous(), cache, tk.t, ws, scores=sc.t, status=st)
    tk.check()
    sc.check()
    return tk.t.cpu().numpy(), sc.t.cpu().numpy(), int(st.item())


def _oracle(w, idx_k, idx_q, n_entries, capacity):
    cfg = oracle_cfg(w)
    ic = np.zeros((idx_k.shape[0], capacity, w.idx_dim), np.int8)
    ic[:, : idx_k.shape[1]] = idx_k.numpy()
    return oracle.index_topk(cfg, idx_q.numpy(), ic, np.asarray(n_entries, np.int32),
                             want_scores=True)


@pytest.mark.parametrize("name", ["tiny", "mla32k"])
def test_topk_bit_exact(kvc, name):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, with_tokens=False)
    n = [w.entries] * w.batch
    tk, sc, st = _run(kvc, w, inp["idx_k"], inp["idx_q"][0], n, w.entries)
    otk, osc = _oracle(w, inp["idx_k"], inp["idx_q"][0], n, w.entries)
    assert st == 0
    assert np.array_equal(sc, osc)
    topk_set_equal(tk, otk)


def test_topk_ragged_batch(kvc):
    w = synth.WORKLOADS["csa2group"].scaled(batch=6, context=2 * 9000)
    inp = synth.make_inputs(w, with_tokens=False)
    n = [9000, 5000, 513, 512, 100, 0]
    cap = 9008
    tk, sc, st = _run(kvc, w, inp["idx_k"], inp["idx_q"][0], n, cap)
    otk, osc = _oracle(w, inp["idx_k"], inp["idx_q"][0], n, cap)
    assert st == 0
    for b in range(6):
        assert np.array_equal(sc[b, : n[b]], osc[b, : n[b]])
    topk_set_equal(tk, otk)
    assert np.all(tk[4, 100:] == -1) and np.all(tk[5] == -1)


@pytest.mark.parametrize("pattern", ["constant", "few_values", "duplicated_rows", "top_tie"])
def test_topk_forced_ties(kvc, pattern):
    w = synth.WORKLOADS["mla32k"].scaled(context=2 * 20000)
    g = torch.Generator().manual_seed(11)
    N = w.entries
    idx_q = torch.randint(-127, 128, (1, 128), generator=g, dtype=torch.int8)
    if pattern == "constant":        # every score equal: heavy-tie path
        idx_k = torch.full((1, N, 128), 3, dtype=torch.int8)
    elif pattern == "few_values":    # 4 distinct rows, thousands of ties each
        rows = torch.randint(-127, 128, (4, 128), generator=g, dtype=torch.int8)
        idx_k = rows[torch.randint(0, 4, (N,), generator=g)].unsqueeze(0)
    elif pattern == "duplicated_rows":
        rows = torch.randint(-127, 128, (N // 8, 128), generator=g, dtype=torch.int8)
        idx_k = rows.repeat_interleave(8, 0).unsqueeze(0)
    else:                            # the threshold falls inside a block of equal scores
        idx_k = torch.randint(-20, 21, (1, N, 128), generator=g, dtype=torch.int8)
        idx_k[0, 1000:1800] = idx_k[0, 7]
    tk, sc, st = _run(kvc, w, idx_k, idx_q, [N], N)
    otk, osc = _oracle(w, idx_k, idx_q, [N], N)
    assert st == 0 and np.array_equal(sc, osc)
    topk_set_equal(tk, otk)


def test_topk_extreme_scores(kvc):
    """Rows at the ends of the int8 x int8 range land in the first and last bins."""
    w = synth.WORKLOADS["tiny"].scaled(context=2 * 300)
    N = w.entries
    idx_q = torch.full((1, 32), -128, dtype=torch.int8)
    idx_k = torch.randint(-127, 128, (1, N, 32), generator=torch.Generator().manual_seed(3),
                          dtype=torch.int8)
    idx_k[0, 10] = -128   # max score 32*16384
    idx_k[0, 20] = 127    # min score
    tk, sc, st = _run(kvc, w, idx_k, idx_q, [N], N)
    otk, osc = _oracle(w, idx_k, idx_q, [N], N)
    assert sc[0, 10] == 32 * 128 * 128 and np.array_equal(sc, osc)
    topk_set_equal(tk, otk)


def test_topk_workspace_validation(kvc):
    w = synth.WORKLOADS["tiny"]
    cfg = kvc.config_for(w)
    cache = kvc.Cache(cfg, 1, 64)
    tk = torch.empty(1, w.topk, dtype=torch.int32, device="cuda")
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(kvc.KvcError) as e:
        kvc.index_topk(cfg, torch.zeros(1, 32, dtype=torch.int8, device="cuda"), cache, tk, small)
    assert e.value.status == 7


def test_topk_scan_slices_span_sequences(kvc):
    """400 short sequences: each scan CTA's row slice covers parts of two or
    more sequences, so candidate segments start mid-slice and mid-sequence;
    lengths are ragged on both sides of K."""
    w = synth.WORKLOADS["mla32k"].scaled(batch=400, context=2 * 600)
    inp = synth.make_inputs(w, with_tokens=False)
    rng = np.random.default_rng(3)
    n = rng.integers(300, 601, 400).astype(np.int32)
    n[:3] = [600, 512, 513]
    tk, sc, st = _run(kvc, w, inp["idx_k"], inp["idx_q"][0], n, 600)
    otk, osc = _oracle(w, inp["idx_k"], inp["idx_q"][0], n, 600)
    assert st == 0
    for b in range(400):
        assert np.array_equal(sc[b, : n[b]], osc[b, : n[b]]), b
    topk_set_equal(tk, otk)


def test_workspace_reused_across_calls(kvc):
    """The workspace is zero-filled once; every call leaves its counters at zero,
    so calls of different lengths and queries on one workspace stay exact."""
    w = synth.WORKLOADS["csa2group"].scaled(batch=4, context=2 * 20000)
    cfg = kvc.config_for(w)
    g = torch.Generator().manual_seed(21)
    idx_k = torch.randint(-127, 128, (4, 20000, 128), generator=g, dtype=torch.int8)
    cache = kvc.Cache(cfg, 4, 20000)
    cache.idx_k.copy_(idx_k.cuda())
    ws = kvc.workspace(cfg, 4, 20000)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for rnd, n in enumerate([[20000, 9000, 300, 513], [511, 20000, 20000, 8192],
                             [20000, 20000, 20000, 20000], [1, 0, 600, 19999]]):
        q = torch.randint(-127, 128, (4, 128), generator=g, dtype=torch.int8)
        cache.n_entries.copy_(torch.as_tensor(n, dtype=torch.int32))
        tk = torch.empty(4, w.topk, dtype=torch.int32, device="cuda")
        kvc.index_topk(cfg, q.cuda(), cache, tk, ws, status=st)
        torch.cuda.synchronize()
        want = _oracle(w, idx_k, q, n, 20000)[0]
        assert st.item() == 0, rnd
        topk_set_equal(tk.cpu().numpy(), want)


def _rows_with_sums(sums, di=128):
    """int8 rows whose elements add up to the given sums (|sum| <= 127 * di)."""
    sums = np.asarray(sums, np.int64)
    base = np.floor_divide(sums, di)
    rem = sums - base * di
    rows = np.repeat(base[:, None], di, 1)
    rows += (np.arange(di)[None, :] < rem[:, None])
    assert np.all(rows.sum(1) == sums) and np.abs(rows).max() <= 127
    return torch.from_numpy(rows.astype(np.int8))


@pytest.mark.parametrize("ties", [100, 128, 129, 1000, 4096, 4097, 6000])
@pytest.mark.parametrize("cap", [20000, 9 * 8192, 9 * 16384])
def test_topk_tie_counts(kvc, ties, cap):
    """A chosen number of entries in the threshold bin, spread over every
    tile, on both sides of each path's limit: up to 128 (every CTA ranks
    them), up to 4096 (a block sorts them), more (the second-histogram
    pass).  A capacity of at most 8 tiles of 8,192 or of 16,384 scores
    selects inside one cluster per sequence, a larger one through the
    sequence's last tile CTA."""
    w = synth.WORKLOADS["mla32k"].scaled(context=2 * 20000)
    N, K = 20000, w.topk
    rng = np.random.default_rng(ties)
    pos = rng.permutation(N)
    sums = np.full(N, -5000, np.int64)
    sums[pos[:400]] = 8000 + np.arange(400)              # above the threshold bin
    sums[pos[400:400 + ties]] = 5000 + rng.integers(0, 4, ties)  # the threshold bin
    idx_k = _rows_with_sums(sums).unsqueeze(0)
    idx_q = torch.full((1, 128), 127, dtype=torch.int8)
    tk, sc, st = _run(kvc, w, idx_k, idx_q, [N], cap)
    otk, osc = _oracle(w, idx_k, idx_q, [N], cap)
    assert st == 0 and np.array_equal(sc[:, :N], osc[:, :N])
    topk_set_equal(tk, otk)
    assert np.array_equal(tk, otk)  # ascending, exactly K (no -1)
    assert np.all(tk >= 0) and tk.shape[1] == K


@pytest.mark.parametrize("cap", [8192 * 8, 8192 * 8 + 1, 16384 * 8, 16384 * 8 + 1])
def test_topk_cluster_tile_boundaries(kvc, cap):
    """Capacities at the edges of the selection layouts (8 tiles of 8,192,
    8 tiles of 16,384, beyond).  The winners crowd into the last 4,200
    entries (the most recent score highest): 200 distinct high scores and
    4,000 equal ones in the threshold bin, so one tile holds more candidate
    keys than its shared-memory buffer (they spill to global memory) and a
    block sorts the ties."""
    w = synth.WORKLOADS["mla32k"].scaled(batch=2, context=2 * 4096)
    g = torch.Generator().manual_seed(cap % 1000)
    n = [cap, cap - 1000]
    idx_q = torch.randint(-127, 128, (2, 128), generator=g, dtype=torch.int8)
    idx_k = torch.randint(-127, 128, (2, cap, 128), generator=g, dtype=torch.int8)
    for b in range(2):
        q16 = idx_q[b].to(torch.int16)
        lo = n[b] - 4200
        idx_k[b, lo:n[b]] = (q16 // 2).to(torch.int8)  # equal scores, about |q|^2 / 2
        hi = (q16 * 3 // 4).to(torch.int8).repeat(200, 1)
        hi[:, :8] = torch.randint(-127, 128, (200, 8), generator=g, dtype=torch.int8)
        idx_k[b, lo:n[b]:21] = hi                        # 200 rows above them
    tk, sc, st = _run(kvc, w, idx_k, idx_q, n, cap)
    otk, osc = _oracle(w, idx_k, idx_q, n, cap)
    assert st == 0
    for b in range(2):
        assert np.array_equal(sc[b, : n[b]], osc[b, : n[b]])
    topk_set_equal(tk, otk)
