"""GPU CSA2 layer-group step vs the oracle on the group layouts of the
workloads (Full, Reindex, Reuse, Reuse; and the 20-layer decoder stack) at
reduced context, with every layer's own q and window."""
import numpy as np
import pytest
import torch

import oracle
from fp4_compressed_kv_b200 import synth
from helpers import Guarded, assert_attn_close, f32, oracle_cfg, oracle_pack

pytestmark = pytest.mark.gpu


def _group(kvc, w, context, batch=None):
    w = w.scaled(context=context, batch=batch or w.batch)
    inp = synth.make_inputs(w)
    rec, ic, n, _ = oracle_pack(w, inp["tokens"], inp["gate"], inp["idx_k"])
    cfg = kvc.config_for(w)
    cache = kvc.Cache(cfg, w.batch, rec.shape[1])
    cache.records.copy_(torch.from_numpy(rec))
    cache.idx_k.copy_(torch.from_numpy(ic))
    cache.n_entries.copy_(torch.from_numpy(n))
    L, B, H = w.layers, w.batch, w.heads
    gout = Guarded((L, B, H, w.latent), torch.float32, fill=float("nan"))  # canaries around
    glse = Guarded((L, B, H), torch.float32)                                # every output
    gtk = Guarded((L, B, w.topk), torch.int32)
    out, lse, tk = gout.t, glse.t, gtk.t
    ws = kvc.workspace(cfg, B, cache.capacity)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvc.layer_group_step(cfg, list(w.modes), inp["q"].cuda(), inp["idx_q"].cuda(),
                         inp["windows"].cuda(), w.window, cache, out, tk, ws, lse=lse, status=st)
    for g in (gout, glse, gtk):
        g.check()
    ref, ref_lse, otk, ost = oracle.group_step(oracle_cfg(w), list(w.modes), f32(inp["q"]),
                                               inp["idx_q"].numpy(), f32(inp["windows"]), w.window,
                                               rec, ic, n)
    assert int(st.item()) == ost == 0
    assert np.array_equal(tk.cpu().numpy(), otk)
    assert_attn_close(out.cpu().numpy(), ref, w.name)
    assert np.max(np.abs(lse.cpu().numpy() - ref_lse)) < 2e-3 * np.abs(ref_lse).max()
    return w, tk.cpu().numpy()


def test_csa2_group_reduced(kvc):
    w, tk = _group(kvc, synth.WORKLOADS["csa2group"], context=2 * 6000, batch=3)
    assert np.array_equal(tk[2], tk[1]) and np.array_equal(tk[3], tk[1])
    assert not np.array_equal(tk[1], tk[0])  # Reindex picks its own set


def test_stack20_reduced(kvc):
    w, tk = _group(kvc, synth.WORKLOADS["stack1m"], context=2 * 5000)
    heads = [l for l, m in enumerate(w.modes) if m != synth.REUSE]
    assert heads == [0, 4, 8, 12, 16]
    for l, m in enumerate(w.modes):
        if m == synth.REUSE:
            assert np.array_equal(tk[l], tk[max(h for h in heads if h < l)])


def test_tiny_group_fp32(kvc):
    _group(kvc, synth.WORKLOADS["tiny"].scaled(modes=(0, 2, 1, 2)), context=1024)


def test_group_rejects_reuse_first(kvc):
    w = synth.WORKLOADS["tiny"]
    cfg = kvc.config_for(w)
    cache = kvc.Cache(cfg, 1, 16)
    z = torch.zeros(2, 1, 8, 80, device="cuda")
    with pytest.raises(kvc.KvcError):
        kvc.layer_group_step(cfg, [2, 0], z, torch.zeros(2, 1, 32, dtype=torch.int8, device="cuda"),
                             torch.zeros(2, 1, 32, 80, device="cuda"), 32, cache,
                             torch.zeros(2, 1, 8, 64, device="cuda"),
                             torch.zeros(2, 1, 64, dtype=torch.int32, device="cuda"),
                             kvc.workspace(cfg, 1, 16))


def test_encoder_groups_reduced(kvc):
    """The encoder stack's layout ("DeepSeek V1 到 V4.1-Flash ..." part 4, CSA2):
    3 groups of one Full and five Reuse layers, each group with its own cache
    and inputs, groups of 16 channels per scale; every Reuse layer attends over
    its group's Full selection."""
    base = synth.WORKLOADS["encoder1m"]
    assert base.groups == 3 and base.modes == (0, 2, 2, 2, 2, 2) and base.group == 16
    for gi in range(base.groups):
        w, tk = _group(kvc, base.scaled(seed=base.seed + 100 * gi), context=2 * 4000)
        assert all(np.array_equal(tk[l], tk[0]) for l in range(1, w.layers))
