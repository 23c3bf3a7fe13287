"""Seeded synthetic workloads for compressed-KV sparse decode.

This module only draws random inputs and describes their shapes; it holds
none of the method's arithmetic, so the CUDA path and the CPU oracle can
both consume what it produces.  The shapes follow the pages' MLA entry
(512 latent + 64 RoPE channels shared by all query heads), the 128-token
window, the top-512 indexer and the CSA2 decoder layout (group 1 = Full +
3 Reuse, groups 2-5 = Reindex + 3 Reuse) from "DeepSeek V1 到 V4.1-Flash，单
token 的 global KV 如何从 389,000 B 压缩到 890 B的？" (acejoy.com), parts 3
and 4.  There are no trained weights: keys, queries, gate and indexer
vectors are Gaussian or uniform draws.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

FULL, REINDEX, REUSE = 0, 1, 2
SCALE_F32, SCALE_UE4M3 = 0, 1


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int            # sequences
    context: int          # raw tokens already in each sequence
    latent: int           # latent channels (also the value width)
    rope: int             # RoPE channels appended to each key
    group: int            # FP4 group size
    scale_fmt: int        # SCALE_F32 or SCALE_UE4M3
    idx_dim: int          # indexer width
    topk: int
    window: int
    heads: int
    act: str              # "f32" or "bf16": dtype of tokens, queries, windows
    modes: tuple          # CSA2 layer modes, in layer order
    tail_channels: int    # channels scaled up for long tails
    tail_factor: float
    seed: int
    pack_new: int = 0     # new raw tokens per sequence for the pack benchmark
    groups: int = 1       # independent layer groups, each with its own cache and `modes`
    ratio: int = 2        # raw tokens per entry (2 or 4)
    idx_fmt: int = 0      # indexer keys: 0 int8, 1 FP4 rows

    @property
    def dim(self) -> int:
        return self.latent + self.rope

    @property
    def entries(self) -> int:
        return self.context // self.ratio

    @property
    def layers(self) -> int:
        """Layers of one group (every group has the same modes)."""
        return len(self.modes)

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.dim)

    @property
    def torch_dtype(self):
        return torch.float32 if self.act == "f32" else torch.bfloat16

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


_STACK20 = (FULL, REUSE, REUSE, REUSE) + (REINDEX, REUSE, REUSE, REUSE) * 4
_ENC6 = (FULL,) + (REUSE,) * 5

WORKLOADS = {
    # tiny single layer, fp32 everything, fp32 scales
    "tiny": Workload("tiny", 1, 1024, 64, 16, 32, SCALE_F32, 32, 64, 32, 8, "f32",
                     (FULL,), 2, 8.0, 0),
    # MLA-shaped single Full layer at 32K context
    "mla32k": Workload("mla32k", 1, 32768, 512, 64, 32, SCALE_UE4M3, 128, 512, 128, 64,
                       "bf16", (FULL,), 6, 10.0, 1),
    # 32 sequences x 128K context, one Full layer; pack of 4096 new tokens
    "batch32x128k": Workload("batch32x128k", 32, 131072, 512, 64, 64, SCALE_UE4M3, 128,
                             512, 128, 64, "bf16", (FULL,), 6, 10.0, 2, pack_new=4096),
    # one CSA2 decoder group: Full, Reindex, Reuse, Reuse
    "csa2group": Workload("csa2group", 8, 262144, 512, 64, 32, SCALE_UE4M3, 128, 512, 128,
                          64, "bf16", (FULL, REINDEX, REUSE, REUSE), 6, 10.0, 3),
    # 1M-token sequence through the 20-layer decoder stack
    "stack1m": Workload("stack1m", 1, 1_000_000, 512, 64, 32, SCALE_UE4M3, 128, 512, 128,
                        64, "bf16", _STACK20, 6, 10.0, 4),
    # 1M-token sequence through the 18-layer encoder stack: 3 groups of one
    # Full and five Reuse layers, each group with its own cache, groups of 16
    # channels per scale
    "encoder1m": Workload("encoder1m", 1, 1_000_000, 512, 64, 16, SCALE_UE4M3, 128, 512,
                          128, 64, "bf16", _ENC6, 6, 10.0, 5, groups=3),
}


def generator(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def tail_channels(w: Workload) -> torch.Tensor:
    """Indices of the heavy-tail channels (CPU generator, seed-stable)."""
    g = generator("cpu", 1000 + w.seed)
    return torch.randperm(w.dim, generator=g)[: w.tail_channels]


def _keys(w: Workload, shape, gen, device) -> torch.Tensor:
    x = torch.randn(*shape, w.dim, generator=gen, device=device, dtype=torch.float32)
    x[..., tail_channels(w).to(device)] *= w.tail_factor
    return x.to(w.torch_dtype)


def make_inputs(w: Workload, device="cpu", *, with_tokens: bool = True) -> dict:
    """All inputs of one decode step plus the raw token prefix.

    tokens   [B][T][D]     raw keys of the context (compressed 2:1 into the cache)
    gate     [D]  fp32     compression gate, N(0, 1/D)
    idx_k    [B][N][Di]    int8 indexer keys of the N = T/ratio entries, U[-127, 127]
    idx_q    [L][B][Di]    int8 indexer queries, one per layer
    q        [L][B][H][D]  query heads (already absorbed into the latent space)
    windows  [L][B][W][D]  per-layer sliding-window keys; layer 0 holds the last
                           W raw tokens of the context, the others their own draws
    """
    gen = generator(device, w.seed)
    L, B, T, N, D = w.layers, w.batch, w.context, w.entries, w.dim
    out = {}
    tokens = _keys(w, (B, T), gen, device) if with_tokens else None
    out["tokens"] = tokens
    out["gate"] = (torch.randn(D, generator=gen, device=device) / math.sqrt(D)).float()
    out["idx_k"] = torch.randint(-127, 128, (B, N, w.idx_dim), generator=gen, device=device,
                                 dtype=torch.int8)
    out["idx_q"] = torch.randint(-127, 128, (L, B, w.idx_dim), generator=gen, device=device,
                                 dtype=torch.int8)
    out["q"] = torch.randn(L, B, w.heads, D, generator=gen, device=device,
                           dtype=torch.float32).to(w.torch_dtype)
    win = _keys(w, (L, B, w.window), gen, device)
    if tokens is not None and T >= w.window:
        win[0] = tokens[:, T - w.window:]
    out["windows"] = win.contiguous()
    return out


def make_new_tokens(w: Workload, n_new: int, device="cpu", seed_offset: int = 7) -> dict:
    """Fresh raw tokens (and their indexer keys) to append with pack."""
    gen = generator(device, w.seed * 1000 + seed_offset)
    tokens = _keys(w, (w.batch, n_new), gen, device)
    idx_k = torch.randint(-127, 128, (w.batch, n_new // w.ratio, w.idx_dim), generator=gen,
                          device=device, dtype=torch.int8)
    return {"tokens": tokens, "idx_k": idx_k}


def make_step_inputs(w: Workload, n_steps: int, device="cpu", seed_offset: int = 13) -> list:
    """Distinct per-step decode inputs: for each of n_steps steps a fresh
    indexer query, query heads and window per layer (same shapes and
    distributions as make_inputs).  A real decode step brings new queries and
    so a new top-K selection every step; drawing them anew keeps a timed loop
    from re-reading one step's gathered rows out of L2."""
    gen = generator(device, w.seed * 1000 + seed_offset)
    L, B, D = w.layers, w.batch, w.dim
    sets = []
    for _ in range(n_steps):
        sets.append({
            "idx_q": torch.randint(-127, 128, (L, B, w.idx_dim), generator=gen, device=device,
                                   dtype=torch.int8),
            "q": torch.randn(L, B, w.heads, D, generator=gen, device=device,
                             dtype=torch.float32).to(w.torch_dtype),
            "windows": _keys(w, (L, B, w.window), gen, device).contiguous(),
        })
    return sets
