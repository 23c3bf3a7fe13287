"""Run one hot-path call a few times on synthetic inputs, for profilers.

    python -m fp4_compressed_kv_b200.profile_case \
        --kernel scan|scan_fp4|attn|pack|step|hier|batched \
        [--config NAME] [--batch B] [--entries N] [--iters 3]

scan  kvc_index_topk over B sequences of N int8 indexer rows (the indexer
      scan and selection kernels), inputs from the workload's shapes.
scan_fp4  the same over FP4 indexer rows (72 bytes at 128 channels: random
      codes, UE4M3 scales between 2^-8 and 2^1).
attn  kvc_sparse_decode_attn: B sequences, each with a cache of N packed
      entries, a top-K drawn uniformly from them and a full window.
pack  kvc_pack of the workload's pack case (pack_new raw tokens per sequence,
      or 4096 when the workload has none).
step  one decode step of the workload (pack of one pair + layer group).
hier  the same step with the hierarchical indexer (2048 blocks of 8 kept):
      block maxima, pool-mode scan and selection.
batched  kvc_index_topk_batched: every Full/Reindex layer's query of the
      workload against one cache in one tensor-core pass.
Sizes default to the workload's; pass --batch/--entries to shrink a case so a
profiler capture stays small (keep the streamed bytes above the 126 MB L2).
"""
from __future__ import annotations

import argparse

import torch

from fp4_compressed_kv_b200 import build, kvc, synth


def main():
    p = argparse.ArgumentParser()
    p.add_argument("--kernel", required=True,
                   choices=["scan", "scan_fp4", "attn", "pack", "step", "hier", "batched"])
    p.add_argument("--config", default="batch32x128k")
    p.add_argument("--batch", type=int, default=0)
    p.add_argument("--entries", type=int, default=0)
    p.add_argument("--iters", type=int, default=3)
    a = p.parse_args()
    build.build()
    w = synth.WORKLOADS[a.config]
    if a.batch:
        w = w.scaled(batch=a.batch)
    if a.entries:
        w = w.scaled(context=2 * a.entries)
    cfg = kvc.config_for(w)
    dev = torch.device("cuda")
    g = synth.generator(dev, w.seed)
    B, N = w.batch, w.entries
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    if a.kernel == "scan_fp4":  # FP4 indexer keys: random codes, scales 2^-8 .. 2^1
        cfg = kvc.config_for(w.scaled(idx_fmt=1))
    hier_blocks = 2048 if a.kernel == "hier" else 0
    if a.kernel in ("scan", "scan_fp4", "step", "attn", "hier", "batched"):
        cache = kvc.Cache(cfg, B, N + a.iters + 8, device=dev)
        ws = kvc.workspace(cfg, B, cache.capacity, device=dev, hier_blocks=hier_blocks)
    if a.kernel in ("scan", "step", "hier", "batched"):
        cache.idx_k[:, :N] = torch.randint(-127, 128, (B, N, w.idx_dim), generator=g, device=dev,
                                           dtype=torch.int8)
        cache.n_entries.fill_(N)
    if a.kernel == "scan_fp4":
        half = w.idx_dim // 2
        cache.idx_k[:, :N, :half] = torch.randint(0, 256, (B, N, half), generator=g, device=dev,
                                                  dtype=torch.uint8)
        cache.idx_k[:, :N, half:] = torch.randint(0x20, 0x40, (B, N, w.idx_dim // 16),
                                                  generator=g, device=dev, dtype=torch.uint8)
        cache.n_entries.fill_(N)
    if a.kernel in ("scan", "scan_fp4"):
        q = torch.randint(-127, 128, (B, w.idx_dim), generator=g, device=dev, dtype=torch.int8)
        tk = torch.empty(B, w.topk, dtype=torch.int32, device=dev)
        for _ in range(a.iters):
            kvc.index_topk(cfg, q, cache, tk, ws, status=st)
    elif a.kernel == "attn":
        # pack N entries per sequence from fresh raw tokens, in slices
        gate = (torch.randn(w.dim, generator=g, device=dev) / w.dim ** 0.5).float()
        step_tok = 8192
        for t0 in range(0, 2 * N, step_tok):
            n = min(step_tok, 2 * N - t0)
            nt = synth.make_new_tokens(w, n, dev, seed_offset=t0)
            kvc.pack(cfg, nt["tokens"], gate, nt["idx_k"], cache, status=st)
        tk = torch.sort(torch.stack([torch.randperm(N, generator=g, device=dev)[: w.topk]
                                     for _ in range(B)]), dim=1).values.int().contiguous()
        q = torch.randn(B, w.heads, w.dim, generator=g, device=dev).to(w.torch_dtype)
        win = torch.randn(B, w.window, w.dim, generator=g, device=dev).to(w.torch_dtype)
        out = torch.empty(B, w.heads, w.latent, device=dev)
        for _ in range(a.iters):
            kvc.sparse_decode_attn(cfg, q, cache, tk, win, w.window, out, ws, status=st)
    elif a.kernel == "pack":
        n_new = w.pack_new or 4096
        nt = synth.make_new_tokens(w, n_new, dev)
        gate = (torch.randn(w.dim, generator=g, device=dev) / w.dim ** 0.5).float()
        pc = kvc.Cache(cfg, B, n_new // 2, device=dev)
        for _ in range(a.iters):
            pc.n_entries.zero_()
            kvc.pack(cfg, nt["tokens"], gate, nt["idx_k"], pc, status=st)
    elif a.kernel == "batched":
        heads = [i for i, m in enumerate(w.modes) if m != synth.REUSE]
        q = torch.randint(-127, 128, (len(heads), B, w.idx_dim), generator=g, device=dev,
                          dtype=torch.int8)
        tk = torch.empty(len(heads), B, w.topk, dtype=torch.int32, device=dev)
        wsb = kvc.workspace_batched(cfg, len(heads), B, cache.capacity, device=dev)
        for _ in range(a.iters):
            kvc.index_topk_batched(cfg, q, cache, tk, wsb, status=st)
    else:  # step, hier
        inp = synth.make_inputs(w, dev, with_tokens=False)
        L = w.layers
        nt = synth.make_new_tokens(w, 2, dev)
        out = torch.empty(L, B, w.heads, w.latent, device=dev)
        tk = torch.empty(L, B, w.topk, dtype=torch.int32, device=dev)
        cache.records.random_(0, 120, generator=g)  # arbitrary codes, scale bytes below NaN
        for _ in range(a.iters):
            kvc.pack(cfg, nt["tokens"], inp["gate"], nt["idx_k"], cache, status=st)
            kvc.layer_group_step(cfg, list(w.modes), inp["q"], inp["idx_q"], inp["windows"],
                                 w.window, cache, out, tk, ws, status=st,
                                 hier_blocks=hier_blocks)
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    print(f"profile_case {a.kernel} {w.name} B={B} N={N} iters={a.iters} ok")


if __name__ == "__main__":
    main()
