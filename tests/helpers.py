"""Shared helpers for the parity tests: build the same cache on both sides,
compare attention within the stated tolerance, and skip GPU tests cleanly."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from fp4_compressed_kv_b200 import synth

# Attention tolerance: max |o_gpu - o_ref| over a row <= 2e-3 x ||o_ref row||_2.
ATTN_RTOL = 2e-3


def oracle_cfg(w: synth.Workload) -> oracle.Cfg:
    return oracle.make_cfg(w.latent, w.rope, w.group, w.scale_fmt, w.idx_dim, w.topk, w.window,
                           w.heads, w.sm_scale, w.ratio)


def f32(t: torch.Tensor) -> np.ndarray:
    """Exact widening of bf16/fp32 tensors to numpy fp32 (on the host)."""
    return t.detach().to("cpu", torch.float32).numpy()


def oracle_pack(w: synth.Workload, tokens, gate, idx_k, capacity=None):
    """Oracle cache of the raw tokens: (records, idx_cache, n_entries, status)."""
    cfg = oracle_cfg(w)
    B, T = tokens.shape[0], tokens.shape[1]
    cap = capacity or T // w.ratio
    rec = np.zeros((B, cap, oracle.record_bytes(cfg)), np.uint8)
    ic = np.zeros((B, cap, w.idx_dim), np.int8)
    n = np.zeros(B, np.int32)
    st = oracle.pack(cfg, f32(tokens), f32(gate), idx_k.cpu().numpy(), rec, ic, n)
    return rec, ic, n, st


def assert_attn_close(out_gpu: np.ndarray, out_ref: np.ndarray, what=""):
    out_gpu = np.asarray(out_gpu, np.float64)
    err = np.abs(out_gpu - out_ref).max(axis=-1)
    norm = np.linalg.norm(out_ref, axis=-1)
    bad = err > ATTN_RTOL * norm
    empty = norm == 0
    assert not np.any(bad & ~empty), (
        f"{what}: {bad.sum()} rows over tolerance; worst ratio "
        f"{np.max(err[~empty] / norm[~empty]):.3e}")
    assert np.all(out_gpu[empty] == 0)
    return float(np.max(err[~empty] / norm[~empty])) if np.any(~empty) else 0.0


def topk_set_equal(a: np.ndarray, b: np.ndarray):
    assert np.array_equal(a, b), f"top-K differs at {np.argwhere(a != b)[:5].tolist()}"


class Guarded:
    """A device output buffer with canary regions on both sides: `t` is the
    contiguous view handed to the library, the 4 KiB before and after it hold
    a byte pattern that no kernel may touch.  `check()` raises if one changed,
    naming the side and the first changed offset."""

    GUARD = 4096
    PATTERN = 0xA5

    def __init__(self, shape, dtype, fill=None, device="cuda"):
        shape = tuple(shape)
        n = int(np.prod(shape)) if shape else 1
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        self._raw = torch.full((self.GUARD + nbytes + self.GUARD,), self.PATTERN,
                               dtype=torch.uint8, device=device)
        self.t = self._raw[self.GUARD:self.GUARD + nbytes].view(dtype).view(shape)
        if fill is not None:
            self.t.fill_(fill)

    def check(self):
        if self._raw.is_cuda:
            torch.cuda.synchronize()
        for side, g in (("before", self._raw[:self.GUARD]), ("after", self._raw[-self.GUARD:])):
            bad = torch.nonzero(g != self.PATTERN)
            if bad.numel():
                raise AssertionError(f"canary {side} the output changed at byte {int(bad[0])}")
