"""GPU FP4 indexer keys (idx_fmt = 1; the pages' 72-byte indexer K, "DeepSeek
V1 到 V4.1-Flash ...", "890 字节是怎么算出来的") vs the oracle: the pack writes
the key rows bit for bit as the oracle quantises them; the exact 64-bit
scores give bit-exact top-K sets (ragged lengths, K >= N, forced ties); a
layer-group step over FP4 keys matches the oracle's selection and attention."""
import numpy as np
import pytest
import torch

import oracle
from fp4_compressed_kv_b200 import synth
from helpers import assert_attn_close, f32, oracle_cfg, oracle_pack

pytestmark = pytest.mark.gpu


def _keys(B, N, di, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(B, N, di, generator=g) * scale).to(torch.bfloat16)


def _packed(kvc, w, keys, chunks):
    """GPU cache of workload w's tokens with FP4 indexer rows from `keys`."""
    inp = synth.make_inputs(w)
    cfg = kvc.config_for(w)
    B, T = inp["tokens"].shape[:2]
    N = T // 2
    cache = kvc.Cache(cfg, B, N)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tok, gate, kd = inp["tokens"].cuda(), inp["gate"].cuda(), keys.cuda()
    for t0 in range(0, T, chunks):
        kvc.pack(cfg, tok[:, t0:t0 + chunks].contiguous(), gate,
                 kd[:, t0 // 2:(t0 + chunks) // 2].contiguous(), cache, status=st)
    torch.cuda.synchronize()
    return inp, cfg, cache, int(st.item())


def _oracle_rows(w, keys):
    ocfg = oracle_cfg(w)
    return np.stack([oracle.idx_fp4_quantize(ocfg, f32(keys[b])) for b in range(keys.shape[0])])


@pytest.mark.parametrize("chunks", [2, 3000])
def test_pack_writes_fp4_key_rows(kvc, chunks):
    w = synth.WORKLOADS["mla32k"].scaled(batch=2, context=2 * 1500, idx_fmt=1)
    keys = _keys(2, 1500, 128, 3, scale=5.0)
    inp, cfg, cache, st = _packed(kvc, w, keys, chunks)
    assert st == 0 and kvc.idx_row_bytes(cfg) == 72
    assert cache.n_entries.cpu().tolist() == [1500, 1500]
    assert np.array_equal(cache.idx_k.cpu().numpy(), _oracle_rows(w, keys))
    rec, _, _, _ = oracle_pack(w, inp["tokens"], inp["gate"], torch.zeros(2, 1500, 128,
                                                                          dtype=torch.int8))
    assert np.array_equal(cache.records.cpu().numpy(), rec)


def test_topk_over_fp4_keys(kvc):
    w = synth.WORKLOADS["mla32k"].scaled(batch=4, context=2 * 3000, idx_fmt=1)
    keys = _keys(4, 3000, 128, 5)
    keys[1, 1000:1400] = keys[1, 17]   # 401 equal rows: ties to the lower index
    keys[2] = keys[2, 0]               # every row equal
    inp, cfg, cache, st = _packed(kvc, w, keys, 6000)
    assert st == 0
    n = [3000, 2999, 2500, 400]        # ragged; the last below K
    cache.n_entries.copy_(torch.tensor(n, dtype=torch.int32))
    q = torch.randint(-128, 128, (4, 128), generator=torch.Generator().manual_seed(8),
                      dtype=torch.int8)
    tk = torch.empty(4, w.topk, dtype=torch.int32, device="cuda")
    ws = kvc.workspace(cfg, 4, cache.capacity)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvc.index_topk(cfg, q.cuda(), cache, tk, ws, status=st2)
    torch.cuda.synchronize()
    rows = _oracle_rows(w, keys)       # the oracle's own rows, equal to the GPU's
    assert np.array_equal(cache.idx_k.cpu().numpy(), rows)
    otk = oracle.index_topk_fp4(oracle_cfg(w), q.numpy(), rows, np.array(n, np.int32))
    assert int(st2.item()) == 0
    assert np.array_equal(tk.cpu().numpy(), otk)
    assert tk[2].cpu().tolist() == list(range(w.topk))
    assert tk[3].cpu().tolist()[:400] == list(range(400)) and (tk[3, 400:] == -1).all()


def test_group_step_over_fp4_keys(kvc):
    w = synth.WORKLOADS["csa2group"].scaled(batch=2, context=2 * 2500, idx_fmt=1)
    keys = _keys(2, 2500, 128, 11, scale=3.0)
    inp, cfg, cache, st = _packed(kvc, w, keys, 5000)
    assert st == 0
    L, B, H = w.layers, w.batch, w.heads
    out = torch.empty(L, B, H, w.latent, device="cuda")
    lse = torch.empty(L, B, H, device="cuda")
    tk = torch.empty(L, B, w.topk, dtype=torch.int32, device="cuda")
    ws = kvc.workspace(cfg, B, cache.capacity)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvc.layer_group_step(cfg, list(w.modes), inp["q"].cuda(), inp["idx_q"].cuda(),
                         inp["windows"].cuda(), w.window, cache, out, tk, ws, lse=lse, status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    ocfg = oracle_cfg(w)
    # the oracle's own cache (records from its pack, rows from its quantiser)
    recs, _, n, _ = oracle_pack(w, inp["tokens"], inp["gate"],
                                torch.zeros(2, 2500, 128, dtype=torch.int8))
    rows = _oracle_rows(w, keys)
    assert np.array_equal(cache.records.cpu().numpy(), recs)
    assert np.array_equal(cache.idx_k.cpu().numpy(), rows)
    head = None
    for l, m in enumerate(w.modes):
        if m != synth.REUSE:
            head = oracle.index_topk_fp4(ocfg, inp["idx_q"][l].numpy(), rows, n)
        assert np.array_equal(tk[l].cpu().numpy(), head), l
        ref, _, ost = oracle.sparse_decode(ocfg, f32(inp["q"][l]), recs, n, head,
                                           f32(inp["windows"][l]), w.window)
        assert ost == 0
        assert_attn_close(out[l].cpu().numpy(), ref, f"fp4 keys layer {l}")


def _random_rows(B, N, di, seed, scale_lo=0x20, scale_hi=0x48):
    """FP4 indexer rows with uniform random codes (every code, -0 included)
    and UE4M3 scales drawn from [scale_lo, scale_hi)."""
    g = np.random.default_rng(seed)
    rows = np.empty((B, N, di // 2 + di // 16), np.uint8)
    rows[:, :, :di // 2] = g.integers(0, 256, (B, N, di // 2))
    rows[:, :, di // 2:] = g.integers(scale_lo, scale_hi, (B, N, di // 16))
    return rows


@pytest.mark.parametrize("di,N,case", [
    (128, 20000, "all_equal"),   # bin t overflows the candidate slots: exact radix path
    (128, 65536, "random"),      # full-size sequences: 16 scan tiles, 8 select tiles
    (256, 9000, "tie_block"),    # 2000 copies of the best row: the cut sorts ~2000 ties
    (128, 9000, "wide_scales"),  # scales over the whole UE4M3 range (subnormal to 448)
    (128, 9001, "odd_rows"),     # 72-byte rows at odd positions; the buffer's last row read
    (64, 5000, "random"),        # 64-channel rows: the direct kernels
])
def test_fp4_scan_and_select_paths(kvc, di, N, case):
    """The FP4 key scan (tiled, log-scale threshold bins) and selection (tile
    candidates, last-CTA finish, exact radix fallback) against the oracle's
    exact top-K, bit for bit, on ragged lengths."""
    B = 3
    w = synth.WORKLOADS["mla32k"].scaled(batch=B, context=2 * N, idx_fmt=1, idx_dim=di)
    cfg = kvc.config_for(w)
    rows = (_random_rows(B, N, di, 21, 0x00, 0x7F) if case == "wide_scales"
            else _random_rows(B, N, di, 21))
    if case == "all_equal":
        rows[0] = rows[0, 5]
    n = np.array([N, N - 77, N // 2 + 3], np.int32)
    if case == "odd_rows":  # sequence 1 starts at an odd row; sequence 2 fills its capacity
        n = np.array([N - 77, N // 2 + 3, N], np.int32)
    q = torch.randint(-128, 128, (B, di), generator=torch.Generator().manual_seed(9),
                      dtype=torch.int8)
    if case == "tie_block":  # the threshold bin then holds all 2000 copies
        _, sc = oracle.index_topk_fp4(oracle_cfg(w), q.numpy(), rows, n, want_scores=True)
        rows[1, 2000:4000] = rows[1, int(np.argmax(sc[1, :n[1]]))]
    cache = kvc.Cache(cfg, B, N)
    cache.idx_k.copy_(torch.from_numpy(rows))
    cache.n_entries.copy_(torch.from_numpy(n))
    ws = kvc.workspace(cfg, B, N)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):  # twice: the counters must be left at zero
        tk = torch.full((B, w.topk), -7, dtype=torch.int32, device="cuda")
        kvc.index_topk(cfg, q.cuda(), cache, tk, ws, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        otk = oracle.index_topk_fp4(oracle_cfg(w), q.numpy(), rows, n)
        assert np.array_equal(tk.cpu().numpy(), otk), f"call {call}"
