"""GPU sparse decode attention vs the oracle (fp64) within
max|o_gpu - o_ref| <= 2e-3 x ||o_ref row||_2, plus the log-sum-exp, on the
fp32 SIMT path (tiny) and the bf16 tensor-core path (MLA shape); edge cases:
no window, every slot empty, padding, out-of-range indices, K >= N."""
import numpy as np
import pytest
import torch

import oracle
from fp4_compressed_kv_b200 import synth
from helpers import Guarded, assert_attn_close, f32, oracle_cfg, oracle_pack

pytestmark = pytest.mark.gpu


def _setup(kvc, w):
    """Pack the workload on the oracle side, upload the same records."""
    inp = synth.make_inputs(w)
    rec, ic, n, _ = oracle_pack(w, inp["tokens"], inp["gate"], inp["idx_k"])
    cfg = kvc.config_for(w)
    cache = kvc.Cache(cfg, w.batch, rec.shape[1])
    cache.records.copy_(torch.from_numpy(rec))
    cache.idx_k.copy_(torch.from_numpy(ic))
    cache.n_entries.copy_(torch.from_numpy(n))
    return inp, rec, ic, n, cfg, cache


def _attn(kvc, cfg, cache, q, tk, win, wl):
    """One attention call into canary-guarded outputs (checked after it)."""
    B, H = q.shape[0], q.shape[1]
    out = Guarded((B, H, cfg.latent_dim), torch.float32, fill=float("nan"))
    lse = Guarded((B, H), torch.float32, fill=float("nan"))
    ws = kvc.workspace(cfg, B, cache.capacity)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvc.sparse_decode_attn(cfg, q.cuda().contiguous(), cache, tk.cuda().contiguous(),
                           win.cuda().contiguous(), wl, out.t, ws, lse=lse.t, status=st)
    out.check()
    lse.check()
    return out.t.cpu().numpy(), lse.t.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("name", ["tiny", "mla32k"])
def test_attention_matches_oracle(kvc, name):
    w = synth.WORKLOADS[name]
    inp, rec, ic, n, cfg, cache = _setup(kvc, w)
    ocfg = oracle_cfg(w)
    tk = oracle.index_topk(ocfg, inp["idx_q"][0].numpy(), ic, n)
    q, win = inp["q"][0], inp["windows"][0]
    out, lse, st = _attn(kvc, cfg, cache, q, torch.from_numpy(tk), win, w.window)
    ref, ref_lse, ost = oracle.sparse_decode(ocfg, f32(q), rec, n, tk, f32(win), w.window)
    assert st == ost == 0
    ratio = assert_attn_close(out, ref, name)
    assert np.max(np.abs(lse - ref_lse)) < 2e-3 * max(1.0, np.abs(ref_lse).max())
    print(f"{name}: worst err/norm {ratio:.2e}")


@pytest.mark.parametrize("name", ["tiny", "mla32k"])
def test_attention_edge_cases(kvc, name):
    w = synth.WORKLOADS[name].scaled(context=2 * 1200)
    inp, rec, ic, n, cfg, cache = _setup(kvc, w)
    ocfg = oracle_cfg(w)
    q, win = inp["q"][0], inp["windows"][0]
    rng = np.random.default_rng(1)
    cases = {}
    # padding in the middle and at the end, plus a window shorter than W
    tk = np.sort(rng.choice(n[0], w.topk, replace=False)).astype(np.int32)[None]
    tk[0, 5:9] = -1
    tk[0, -3:] = -1
    cases["padded_short_window"] = (tk, w.window // 2, 0)
    cases["no_window"] = (tk, 0, 0)
    cases["only_window"] = (np.full((1, w.topk), -1, np.int32), w.window, 0)
    cases["nothing"] = (np.full((1, w.topk), -1, np.int32), 0, 0)
    bad = tk.copy()
    bad[0, 0] = n[0]
    bad[0, 1] = -5
    cases["bad_indices"] = (bad, w.window, oracle.ST_BAD_INDEX)
    for label, (t, wl, want_st) in cases.items():
        out, lse, st = _attn(kvc, cfg, cache, q, torch.from_numpy(t), win, wl)
        ref, ref_lse, ost = oracle.sparse_decode(ocfg, f32(q), rec, n, t, f32(win), wl)
        assert st == ost == want_st, label
        assert_attn_close(out, ref, label)
        if label == "nothing":
            assert np.all(lse == -np.inf) and not out.any()
        else:
            assert np.max(np.abs(lse - ref_lse)) < 2e-3 * max(1.0, np.abs(ref_lse).max()), label


def test_attention_all_selected_window_all_is_dense(kvc):
    """K >= N and the window holding the rest: the GPU result is dense attention."""
    w = synth.WORKLOADS["mla32k"].scaled(context=2 * 300)
    inp, rec, ic, n, cfg, cache = _setup(kvc, w)
    tk = np.concatenate([np.arange(300), -np.ones(212)]).astype(np.int32)[None]
    q, win = inp["q"][0], inp["windows"][0]
    out, _, _ = _attn(kvc, cfg, cache, q, torch.from_numpy(tk), win, w.window)
    ocfg = oracle_cfg(w)
    keys = np.concatenate([np.stack([oracle.dequantize_entry(ocfg, rec[0, j]) for j in range(300)]),
                           f32(win)[0]])
    qt = torch.from_numpy(f32(q)[0]).double()
    kt = torch.from_numpy(keys).double()
    dense = (torch.softmax(w.sm_scale * qt @ kt.T, -1) @ kt[:, : w.latent]).numpy()
    assert_attn_close(out[0], dense, "dense")


def test_attention_batch_splits(kvc):
    """Batch of sequences at different lengths through the split-K merge."""
    w = synth.WORKLOADS["csa2group"].scaled(batch=5, context=2 * 3000, modes=(0,))
    inp, rec, ic, n, cfg, cache = _setup(kvc, w)
    ocfg = oracle_cfg(w)
    n2 = np.array([3000, 2000, 700, 512, 60], np.int32)
    cache.n_entries.copy_(torch.from_numpy(n2))
    tk = oracle.index_topk(ocfg, inp["idx_q"][0].numpy(), ic, n2)
    q, win = inp["q"][0], inp["windows"][0]
    out, lse, st = _attn(kvc, cfg, cache, q, torch.from_numpy(tk), win, w.window)
    ref, ref_lse, _ = oracle.sparse_decode(ocfg, f32(q), rec, n2, tk, f32(win), w.window)
    assert st == 0
    assert_attn_close(out, ref, "batch")
    assert np.max(np.abs(lse - ref_lse)) < 2e-3 * np.abs(ref_lse).max()


def test_attention_online_rescale(kvc):
    """Window keys along head 0's query: their logits exceed the earlier chunks'
    maximum by far more than the lazy-rescale slack, so the running output in
    tensor memory must be rescaled; other heads see ordinary logits."""
    w = synth.WORKLOADS["mla32k"].scaled(context=2 * 1200)
    inp, rec, ic, n, cfg, cache = _setup(kvc, w)
    ocfg = oracle_cfg(w)
    tk = oracle.index_topk(ocfg, inp["idx_q"][0].numpy(), ic, n)
    q = inp["q"][0]
    win = inp["windows"][0].clone()
    win[0, : w.window // 2] = (q[0, 0].float() * 3).to(torch.bfloat16)
    out, lse, st = _attn(kvc, cfg, cache, q, torch.from_numpy(tk), win, w.window)
    ref, ref_lse, _ = oracle.sparse_decode(ocfg, f32(q), rec, n, tk, f32(win), w.window)
    assert st == 0
    assert ref_lse[0, 0] / np.log(2) > 60  # head 0's maximum jumped by > 8 (log2)
    assert_attn_close(out, ref, "rescale")
    assert np.max(np.abs(lse - ref_lse)) < 2e-3 * np.abs(ref_lse).max()


@pytest.mark.parametrize("topk", [192, 1024, 2048])
def test_attention_split_counts(kvc, topk):
    """Key counts that give 2 record chunks and a window chunk per sequence,
    and more record chunks than a cluster holds one per CTA (2 and 3 chunks
    per CTA, merged inside the cluster)."""
    w = synth.WORKLOADS["mla32k"].scaled(context=2 * 5000, topk=topk, batch=3)
    inp, rec, ic, n, cfg, cache = _setup(kvc, w)
    ocfg = oracle_cfg(w)
    tk = oracle.index_topk(ocfg, inp["idx_q"][0].numpy(), ic, n)
    q, win = inp["q"][0], inp["windows"][0]
    out, lse, st = _attn(kvc, cfg, cache, q, torch.from_numpy(tk), win, w.window)
    ref, ref_lse, _ = oracle.sparse_decode(ocfg, f32(q), rec, n, tk, f32(win), w.window)
    assert st == 0
    assert_attn_close(out, ref, f"topk={topk}")
    assert np.max(np.abs(lse - ref_lse)) < 2e-3 * np.abs(ref_lse).max()


@pytest.mark.parametrize("window_len", [128, 100])
def test_attention_wide_batch_folds_window(kvc, window_len):
    """32 sequences: one CTA per record chunk plus a window CTA would not all
    be resident as clusters, so each record CTA also takes the window for a
    quarter of the heads (bf16, folded into its running softmax); ragged
    lengths, padding, and a window shorter than its chunk."""
    w = synth.WORKLOADS["mla32k"].scaled(batch=32, context=2 * 700)
    inp, rec, ic, n, cfg, cache = _setup(kvc, w)
    ocfg = oracle_cfg(w)
    n2 = np.array([700 - 13 * (i % 9) for i in range(32)], np.int32)
    cache.n_entries.copy_(torch.from_numpy(n2))
    tk = oracle.index_topk(ocfg, inp["idx_q"][0].numpy(), ic, n2)
    tk[3, 7:30] = -1
    q, win = inp["q"][0], inp["windows"][0]
    out, lse, st = _attn(kvc, cfg, cache, q, torch.from_numpy(tk), win, window_len)
    ref, ref_lse, _ = oracle.sparse_decode(ocfg, f32(q), rec, n2, tk, f32(win), window_len)
    assert st == 0
    assert_attn_close(out, ref, f"wide batch, window {window_len}")
    assert np.max(np.abs(lse - ref_lse)) < 2e-3 * np.abs(ref_lse).max()
