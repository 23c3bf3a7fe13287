"""GPU 4:1 pack (four tokens per entry, softmax of four gate logits; the 4x
CSA2 ratio of "DeepSeek V4.1 Flash KV Cache压缩实战" 4.3) vs the oracle:
bit-exact records and indexer rows for decode appends (one entry per
sequence), bulk appends in pieces, fp32 and bf16 tokens, fp32 and UE4M3
scales, groups of 16 to 128; lengths, capacity and non-finite flags; and a
layer-group step over a 4:1 cache against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from fp4_compressed_kv_b200 import synth
from helpers import assert_attn_close, f32, oracle_cfg, oracle_pack

pytestmark = pytest.mark.gpu


def _gpu_pack(kvc, w, tokens, gate, idx_k, capacity, chunks):
    cfg = kvc.config_for(w)
    B, T = tokens.shape[:2]
    cache = kvc.Cache(cfg, B, capacity)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t0 in range(0, T, chunks):
        kvc.pack(cfg, tokens[:, t0:t0 + chunks].contiguous(), gate,
                 idx_k[:, t0 // 4:(t0 + chunks) // 4].contiguous(), cache, status=st)
    torch.cuda.synchronize()
    return cache, int(st.item())


@pytest.mark.parametrize("name,group,chunks", [("tiny", 32, 4), ("tiny", 16, 60),
                                               ("mla32k", 64, 4), ("mla32k", 16, 400),
                                               ("mla32k", 128, 1200)])
def test_pack4_bit_exact(kvc, name, group, chunks):
    w = synth.WORKLOADS[name].scaled(ratio=4, group=group, batch=3, context=1200)
    inp = synth.make_inputs(w)
    assert inp["idx_k"].shape[1] == 300
    rec, ic, n, ost = oracle_pack(w, inp["tokens"], inp["gate"], inp["idx_k"], capacity=310)
    cache, st = _gpu_pack(kvc, w, inp["tokens"].cuda(), inp["gate"].cuda(), inp["idx_k"].cuda(),
                          310, chunks)
    assert st == ost == 0
    assert n.tolist() == [300] * 3 and cache.n_entries.cpu().tolist() == [300] * 3
    g = cache.records.cpu().numpy()
    diff = np.argwhere(g != rec)
    assert diff.size == 0, f"{len(diff)} bytes differ, first {diff[:5].tolist()}"
    assert np.array_equal(cache.idx_k.cpu().numpy(), ic)


def test_pack4_capacity_and_nonfinite(kvc):
    w = synth.WORKLOADS["mla32k"].scaled(ratio=4, context=64)
    inp = synth.make_inputs(w)
    tok = inp["tokens"].clone()
    tok[0, 6, 30] = float("nan")
    rec, ic, n, ost = oracle_pack(w, tok, inp["gate"], inp["idx_k"])
    cache, st = _gpu_pack(kvc, w, tok.cuda(), inp["gate"].cuda(), inp["idx_k"].cuda(), 16, 64)
    assert st == ost == 1  # KVC_DEV_NONFINITE
    assert np.array_equal(cache.records.cpu().numpy(), rec)
    # a full cache: the append is refused on the device, the length unchanged
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    cfg = kvc.config_for(w)
    kvc.pack(cfg, tok[:, :4].cuda().contiguous(), inp["gate"].cuda(),
             inp["idx_k"][:, :1].cuda().contiguous(), cache, status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) & 4 and cache.n_entries.cpu().tolist() == [16]
    with pytest.raises(kvc.KvcError):  # 6 tokens are not groups of 4
        kvc.pack(cfg, tok[:, :6].cuda().contiguous(), inp["gate"].cuda(),
                 inp["idx_k"][:, :1].cuda().contiguous(), cache, status=st2)


def test_group_step_over_a_ratio4_cache(kvc):
    w = synth.WORKLOADS["csa2group"].scaled(ratio=4, batch=2, context=4 * 3000)
    inp = synth.make_inputs(w)
    cfg = kvc.config_for(w)
    cache, st = _gpu_pack(kvc, w, inp["tokens"].cuda(), inp["gate"].cuda(), inp["idx_k"].cuda(),
                          3000, 4 * 3000)
    rec, ic, n, _ = oracle_pack(w, inp["tokens"], inp["gate"], inp["idx_k"])
    assert st == 0 and np.array_equal(cache.records.cpu().numpy(), rec)
    L, B, H = w.layers, w.batch, w.heads
    out = torch.empty(L, B, H, w.latent, device="cuda")
    tk = torch.empty(L, B, w.topk, dtype=torch.int32, device="cuda")
    ws = kvc.workspace(cfg, B, cache.capacity)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvc.layer_group_step(cfg, list(w.modes), inp["q"].cuda(), inp["idx_q"].cuda(),
                         inp["windows"].cuda(), w.window, cache, out, tk, ws, status=st2)
    torch.cuda.synchronize()
    ref, _, otk, ost = oracle.group_step(oracle_cfg(w), list(w.modes), f32(inp["q"]),
                                         inp["idx_q"].numpy(), f32(inp["windows"]), w.window,
                                         rec, ic, n)
    assert int(st2.item()) == ost == 0
    assert np.array_equal(tk.cpu().numpy(), otk)
    assert_attn_close(out.cpu().numpy(), ref, "ratio4 group")
