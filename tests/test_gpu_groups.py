"""Other FP4 group sizes on the MLA shape: G = 16 (the pages' 16-channel
scales: 256 B of latent codes + 32 scale bytes = 288 B) and G = 8 and 128.
Pack bit-exact, attention (tensor-core path) within tolerance."""
import numpy as np
import pytest
import torch

import oracle
from fp4_compressed_kv_b200 import synth
from helpers import assert_attn_close, f32, oracle_cfg, oracle_pack

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("group", [8, 16, 128])
def test_group_size_pack_and_attention(kvc, group):
    w = synth.WORKLOADS["mla32k"].scaled(context=2 * 3000, group=group)
    inp = synth.make_inputs(w)
    rec, ic, n, ost = oracle_pack(w, inp["tokens"], inp["gate"], inp["idx_k"])
    assert ost == 0
    ocfg = oracle_cfg(w)
    assert rec.shape[2] == oracle.record_bytes(ocfg)
    cfg = kvc.config_for(w)
    cache = kvc.Cache(cfg, w.batch, w.entries)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvc.pack(cfg, inp["tokens"].cuda(), inp["gate"].cuda(), inp["idx_k"].cuda(), cache, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert np.array_equal(cache.records.cpu().numpy(), rec)
    tk = oracle.index_topk(ocfg, inp["idx_q"][0].numpy(), ic, n)
    q, win = inp["q"][0], inp["windows"][0]
    out = torch.empty(w.batch, w.heads, w.latent, device="cuda")
    lse = torch.empty(w.batch, w.heads, device="cuda")
    ws = kvc.workspace(cfg, w.batch, cache.capacity)
    kvc.sparse_decode_attn(cfg, q.cuda(), cache, torch.from_numpy(tk).cuda(), win.cuda(),
                           w.window, out, ws, lse=lse, status=st)
    torch.cuda.synchronize()
    ref, ref_lse, ost = oracle.sparse_decode(ocfg, f32(q), rec, n, tk, f32(win), w.window)
    assert st.item() == 0 and ost == 0
    assert_attn_close(out.cpu().numpy(), ref, f"G={group}")
    assert np.max(np.abs(lse.cpu().numpy() - ref_lse)) < 2e-3 * np.abs(ref_lse).max()
