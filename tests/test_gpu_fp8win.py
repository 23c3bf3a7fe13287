"""FP8 window (one fp32 scale per row, signed E4M3 codes): the GPU codes and
scales bit-exact against the oracle, and attention over top-K + an FP8 window
within the stated tolerance of the oracle's attention over the decoded
window, on the tensor-core path (MLA shape) and the CUDA-core path (tiny)."""
import numpy as np
import pytest
import torch

import oracle
from fp4_compressed_kv_b200 import synth
from helpers import assert_attn_close, f32, oracle_cfg, oracle_pack

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "mla32k"])
def test_window_fp8_codes_bit_exact(kvc, name):
    w = synth.WORKLOADS[name]
    g = torch.Generator().manual_seed(5)
    rows = (torch.randn(3, 40, w.dim, generator=g) *
            torch.tensor([0.02, 1.0, 40.0]).view(3, 1, 1)).to(w.torch_dtype)
    rows[1, 3, 7] = float("nan")
    rows[2, 0, :] = 0
    cfg = kvc.config_for(w)
    codes = torch.empty(rows.shape, dtype=torch.uint8, device="cuda")
    scales = torch.empty(rows.shape[:-1], dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvc.pack_window_fp8(cfg, rows.cuda().contiguous(), codes, scales, status=st)
    torch.cuda.synchronize()
    oc, osc, bad = oracle.window_fp8(f32(rows))
    assert bad == 1 and st.item() == kvc.DEV_NONFINITE
    assert np.array_equal(scales.cpu().numpy(), osc)
    assert np.array_equal(codes.cpu().numpy(), oc)


@pytest.mark.parametrize("name,batch", [("tiny", 2), ("mla32k", 2), ("mla32k", 32)])
def test_attention_with_fp8_window(kvc, name, batch):
    """batch 32 with the MLA shape takes the wide-batch launch (more record
    chunks per CTA, since FP8 window rows are never folded into them)."""
    w = synth.WORKLOADS[name].scaled(batch=batch, context=2 * (1500 if batch < 8 else 600))
    inp = synth.make_inputs(w)
    rec, ic, n, _ = oracle_pack(w, inp["tokens"], inp["gate"], inp["idx_k"])
    cfg = kvc.config_for(w)
    cache = kvc.Cache(cfg, w.batch, rec.shape[1])
    cache.records.copy_(torch.from_numpy(rec))
    cache.idx_k.copy_(torch.from_numpy(ic))
    cache.n_entries.copy_(torch.from_numpy(n))
    ocfg = oracle_cfg(w)
    tk = oracle.index_topk(ocfg, inp["idx_q"][0].numpy(), ic, n)
    q, win = inp["q"][0], inp["windows"][0]
    codes, scales, _ = oracle.window_fp8(f32(win))
    for wl in (w.window, w.window // 2 + 3, 0):
        out = torch.full((w.batch, w.heads, w.latent), float("nan"), device="cuda")
        lse = torch.empty(w.batch, w.heads, device="cuda")
        ws = kvc.workspace(cfg, w.batch, cache.capacity)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        kvc.sparse_decode_attn_fp8win(cfg, q.cuda().contiguous(), cache,
                                      torch.from_numpy(tk).cuda(),
                                      torch.from_numpy(codes).cuda(),
                                      torch.from_numpy(scales).cuda(), wl, out, ws, lse=lse,
                                      status=st)
        torch.cuda.synchronize()
        deq = oracle.window_fp8_dequant(codes, scales)
        ref, ref_lse, ost = oracle.sparse_decode(ocfg, f32(q), rec, n, tk, deq, wl)
        assert st.item() == 0 and ost == 0
        assert_attn_close(out.cpu().numpy(), ref, f"{name} window {wl}")
        assert np.max(np.abs(lse.cpu().numpy() - ref_lse)) < 2e-3 * max(1.0, np.abs(ref_lse).max())
