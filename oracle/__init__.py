"""CPU oracle for compressed-KV sparse decode (test infrastructure only).

The arithmetic lives in ``oracle.c`` (plain C, compiled with
``-ffp-contract=off``): fp64 where the pages fix no precision and no quantised
value depends on it (attention), fp32 for the compression gate whose result
decides the FP4 codes (the kernel's precision).  This module compiles it
into ``liboracle.so`` next to the source and wraps every entry point for
numpy arrays.  Only the tests, the smoke check and the benchmark's CPU
baseline leg may import it; the product library never does.

Parity status of each function is stated in ``oracle.c``'s header and in the
tests that pin it (``tests/test_oracle_*.py``).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

SCALE_F32 = 0
SCALE_UE4M3 = 1
MODE_FULL, MODE_REINDEX, MODE_REUSE = 0, 1, 2
ST_NONFINITE = 1
ST_BAD_INDEX = 2


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, no contraction of a*b+c)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".tmp"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
             "-fPIC", "-shared", SRC, "-o", tmp, "-lm"])
        os.replace(tmp, LIB)
    return LIB


class Cfg(C.Structure):
    _fields_ = [("latent_dim", C.c_int), ("rope_dim", C.c_int), ("group", C.c_int),
                ("scale_fmt", C.c_int), ("idx_dim", C.c_int), ("topk", C.c_int),
                ("window", C.c_int), ("n_heads", C.c_int), ("sm_scale", C.c_double),
                ("ratio", C.c_int)]


def make_cfg(latent_dim, rope_dim, group, scale_fmt, idx_dim, topk, window, n_heads,
             sm_scale, ratio=2) -> Cfg:
    """ratio: raw tokens per entry, 2 or 4."""
    if group <= 0 or latent_dim <= 0 or rope_dim < 0 or ratio not in (2, 4):
        raise ValueError("bad dims")
    return Cfg(latent_dim, rope_dim, group, scale_fmt, idx_dim, topk, window, n_heads,
               float(sm_scale), ratio)


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        P = C.c_void_p
        sig = {
            "orc_kv_bytes_per_token": (C.c_uint64, [C.c_int64] * 4),
            "orc_expf": (C.c_float, [C.c_float]),
            "orc_e2m1_value": (C.c_float, [C.c_int]),
            "orc_e2m1_encode": (C.c_int, [C.c_float]),
            "orc_e4m3_value": (C.c_float, [C.c_int]),
            "orc_e4m3_encode": (C.c_int, [C.c_float]),
            "orc_n_groups": (C.c_int, [C.c_int] * 3),
            "orc_record_bytes": (C.c_int, [P, C.c_int]),
            "orc_gate_delta": (C.c_float, [P, P, P, C.c_int]),
            "orc_compress_pair": (None, [P, P, P, C.c_int, P]),
            "orc_gate_logit": (C.c_float, [P, P, C.c_int]),
            "orc_idx_fp4_score": (C.c_int64, [P, P, C.c_int]),
            "orc_topk64": (C.c_int, [P, C.c_int, C.c_int, P]),
            "orc_index_topk_fp4": (C.c_int, [P, C.c_int, P, P, C.c_int, P, P, P]),
            "orc_compress_group4": (None, [P, P, P, P, P, C.c_int, P]),
            "orc_quantize_entry": (C.c_int, [P, P, P]),
            "orc_dequantize_entry": (None, [P, P, P]),
            "orc_pack": (C.c_int, [P, C.c_int, C.c_int, P, P, P, C.c_int, P, P, P, P]),
            "orc_index_scores": (None, [P, P, C.c_int, C.c_int, P]),
            "orc_topk": (C.c_int, [P, C.c_int, C.c_int, P]),
            "orc_index_topk": (C.c_int, [P, C.c_int, P, P, C.c_int, P, P, P]),
            "orc_attention": (None, [P, C.c_int, C.c_int, C.c_int, P, C.c_int, C.c_double,
                                     P, P]),
            "orc_sparse_decode": (C.c_int, [P, C.c_int, P, P, C.c_int, P, P, P, C.c_int, P,
                                            P, P]),
            "orc_bytes_resident": (C.c_uint64, [P, C.c_int64, C.c_int, C.c_int, C.c_int]),
            "orc_group_step": (C.c_int, [P, C.c_int, P, C.c_int, P, P, P, C.c_int, P, P,
                                         C.c_int, P, P, P, P, P]),
            "orc_group_step_hier": (C.c_int, [P, C.c_int, P, C.c_int, P, P, P, C.c_int, P, P,
                                              C.c_int, P, C.c_int, C.c_int, P, P, P, P]),
            "orc_block_pool": (C.c_int, [P, C.c_int, C.c_int, C.c_int, P, P]),
            "orc_window_fp8": (C.c_int, [P, C.c_int, P, P]),
            "orc_window_fp8_dequant": (None, [P, C.c_float, C.c_int, P]),
            "orc_pool_topk": (C.c_int, [P, P, C.c_int, P, C.c_int, C.c_int, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(_lib, name)
            fn.restype = res
            fn.argtypes = args
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- scalars
def kv_bytes_per_token(layers, heads, dim, bytes_per_elem) -> int:
    return int(lib().orc_kv_bytes_per_token(layers, heads, dim, bytes_per_elem))


def expf(x: float) -> float:
    """The fp32 exp of the gate (its result as a Python float)."""
    return lib().orc_expf(float(x))


def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(int(code))


def e2m1_encode(v: float) -> int:
    return lib().orc_e2m1_encode(float(v))


def e4m3_value(b: int) -> float:
    return lib().orc_e4m3_value(int(b))


def e4m3_encode(v: float) -> int:
    return lib().orc_e4m3_encode(float(v))


def n_groups(latent, rope, group) -> int:
    return lib().orc_n_groups(latent, rope, group)


def record_bytes(cfg: Cfg, padded: bool = True) -> int:
    return lib().orc_record_bytes(C.byref(cfg), int(padded))


def bytes_resident(cfg: Cfg, entries, n_layers, window_elem_bytes, padded) -> int:
    return int(lib().orc_bytes_resident(C.byref(cfg), int(entries), int(n_layers),
                                        int(window_elem_bytes), int(padded)))


# ---------------------------------------------------------------- entries
def gate_delta(k0, k1, g) -> float:
    k0, k1, g = _c(k0, np.float32), _c(k1, np.float32), _c(g, np.float32)
    return lib().orc_gate_delta(_p(k0), _p(k1), _p(g), k0.size)


def compress_pair(k0, k1, g) -> np.ndarray:
    k0, k1, g = _c(k0, np.float32), _c(k1, np.float32), _c(g, np.float32)
    e = np.empty_like(k0)
    lib().orc_compress_pair(_p(k0), _p(k1), _p(g), k0.size, _p(e))
    return e


def gate_logit(k, g) -> float:
    k, g = _c(k, np.float32), _c(g, np.float32)
    return lib().orc_gate_logit(_p(k), _p(g), k.size)


def compress_group4(ks, g) -> np.ndarray:
    """One entry from four tokens ks [4][D] (the 4:1 ratio)."""
    ks = [_c(k, np.float32) for k in ks]
    g = _c(g, np.float32)
    e = np.empty_like(ks[0])
    lib().orc_compress_group4(*[_p(k) for k in ks], _p(g), ks[0].size, _p(e))
    return e


def quantize_entry(cfg: Cfg, e) -> tuple[np.ndarray, int]:
    e = _c(e, np.float32)
    rec = np.zeros(record_bytes(cfg), np.uint8)
    nf = lib().orc_quantize_entry(C.byref(cfg), _p(e), _p(rec))
    return rec, nf


def dequantize_entry(cfg: Cfg, rec) -> np.ndarray:
    rec = _c(rec, np.uint8)
    x = np.empty(cfg.latent_dim + cfg.rope_dim, np.float32)
    lib().orc_dequantize_entry(C.byref(cfg), _p(rec), _p(x))
    return x


def pack(cfg: Cfg, tokens, g, idxk_new, records, idx_cache, n_entries) -> int:
    """In-place append; returns the status bits.  tokens [B][n_new][D]."""
    tokens = _c(tokens, np.float32)
    g = _c(g, np.float32)
    idxk_new = _c(idxk_new, np.int8)
    B, n_new, D = tokens.shape
    assert records.flags.c_contiguous and idx_cache.flags.c_contiguous
    assert n_entries.dtype == np.int32 and n_entries.flags.c_contiguous
    cap = records.shape[1]
    st = np.zeros(1, np.uint32)
    rc = lib().orc_pack(C.byref(cfg), B, n_new, _p(tokens), _p(g), _p(idxk_new), cap,
                        _p(records), _p(idx_cache), _p(n_entries), _p(st))
    if rc:
        raise ValueError(f"orc_pack failed: {rc}")
    return int(st[0])


# ---------------------------------------------------------------- indexer
def index_scores(q, keys) -> np.ndarray:
    q, keys = _c(q, np.int8), _c(keys, np.int8)
    n, di = keys.shape
    out = np.empty(n, np.int32)
    lib().orc_index_scores(_p(q), _p(keys), n, di, _p(out))
    return out


def topk(scores, k) -> np.ndarray:
    scores = _c(scores, np.int32)
    out = np.empty(k, np.int32)
    lib().orc_topk(_p(scores), scores.size, k, _p(out))
    return out


def index_topk(cfg: Cfg, idx_q, idx_cache, n_entries, want_scores=False):
    idx_q, idx_cache = _c(idx_q, np.int8), _c(idx_cache, np.int8)
    n_entries = _c(n_entries, np.int32)
    B, cap, _ = idx_cache.shape
    tk = np.empty((B, cfg.topk), np.int32)
    sc = np.zeros((B, cap), np.int32) if want_scores else None
    rc = lib().orc_index_topk(C.byref(cfg), B, _p(idx_q), _p(idx_cache), cap, _p(n_entries),
                              _p(tk), _p(sc) if sc is not None else None)
    if rc:
        raise ValueError(f"orc_index_topk failed: {rc}")
    return (tk, sc) if want_scores else tk


def idx_fp4_cfg(cfg: Cfg) -> Cfg:
    """The quantisation configuration of FP4 indexer keys (R18): Di channels,
    no RoPE, groups of 16, UE4M3 scales."""
    return make_cfg(cfg.idx_dim, 0, 16, SCALE_UE4M3, cfg.idx_dim, cfg.topk, cfg.window,
                    cfg.n_heads, cfg.sm_scale)


def idx_fp4_quantize(cfg: Cfg, keys) -> np.ndarray:
    """FP4 indexer rows [n][Di/2 + Di/16] of float keys [n][Di]."""
    keys = _c(keys, np.float32)
    qc = idx_fp4_cfg(cfg)
    rb = record_bytes(qc, False)
    out = np.empty((keys.shape[0], rb), np.uint8)
    for j in range(keys.shape[0]):
        out[j] = quantize_entry(qc, keys[j])[0][:rb]
    return out


def idx_fp4_score(q, row, di) -> int:
    """Exact score times 2^10 of int8 query q against one FP4 indexer row."""
    q, row = _c(q, np.int8), _c(row, np.uint8)
    return int(lib().orc_idx_fp4_score(_p(q), _p(row), int(di)))


def topk64(scores, k) -> np.ndarray:
    scores = _c(scores, np.int64)
    out = np.empty(k, np.int32)
    lib().orc_topk64(_p(scores), scores.size, k, _p(out))
    return out


def index_topk_fp4(cfg: Cfg, idx_q, keys, n_entries, want_scores=False):
    """Top-K over FP4 indexer rows keys [B][cap][Di/2 + Di/16]."""
    idx_q, keys = _c(idx_q, np.int8), _c(keys, np.uint8)
    n_entries = _c(n_entries, np.int32)
    B, cap, _ = keys.shape
    tk = np.empty((B, cfg.topk), np.int32)
    sc = np.zeros((B, cap), np.int64) if want_scores else None
    rc = lib().orc_index_topk_fp4(C.byref(cfg), B, _p(idx_q), _p(keys), cap, _p(n_entries),
                                  _p(tk), _p(sc) if sc is not None else None)
    if rc:
        raise ValueError(f"orc_index_topk_fp4 failed: {rc}")
    return (tk, sc) if want_scores else tk


# ---------------------------------------------------------------- attention
def attention(q, keys, sm_scale, dv):
    """Dense fp64 softmax attention of q [H][D] over keys [nk][D]."""
    q, keys = _c(q, np.float32), _c(keys, np.float32)
    H, D = q.shape
    nk = keys.shape[0]
    out = np.empty((H, dv), np.float64)
    lse = np.empty(H, np.float64)
    lib().orc_attention(_p(q), H, D, dv, _p(keys), nk, float(sm_scale), _p(out), _p(lse))
    return out, lse


def sparse_decode(cfg: Cfg, q, records, n_entries, topk_idx, window, window_len):
    q = _c(q, np.float32)
    records = _c(records, np.uint8)
    n_entries = _c(n_entries, np.int32)
    topk_idx = _c(topk_idx, np.int32)
    window = _c(window, np.float32)
    B = q.shape[0]
    cap = records.shape[1]
    out = np.empty((B, cfg.n_heads, cfg.latent_dim), np.float64)
    lse = np.empty((B, cfg.n_heads), np.float64)
    st = np.zeros(1, np.uint32)
    rc = lib().orc_sparse_decode(C.byref(cfg), B, _p(q), _p(records), cap, _p(n_entries),
                                 _p(topk_idx), _p(window), int(window_len), _p(out), _p(lse),
                                 _p(st))
    if rc:
        raise ValueError(f"orc_sparse_decode failed: {rc}")
    return out, lse, int(st[0])


def window_fp8(rows):
    """FP8 window rows [..][D] fp32 -> (codes uint8 [..][D], scales fp32 [..], bad rows)."""
    rows = _c(rows, np.float32)
    D = rows.shape[-1]
    flat = rows.reshape(-1, D)
    codes = np.zeros(flat.shape, np.uint8)
    scales = np.zeros(flat.shape[0], np.float32)
    bad = 0
    for i in range(flat.shape[0]):
        sc = C.c_float(0.0)
        bad |= lib().orc_window_fp8(_p(flat[i]), D, _p(codes[i]), C.byref(sc))
        scales[i] = sc.value
    return codes.reshape(rows.shape), scales.reshape(rows.shape[:-1]), bad


def window_fp8_dequant(codes, scales):
    """Decoded FP8 window rows, fp32."""
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.float32)
    D = codes.shape[-1]
    flat = codes.reshape(-1, D)
    sf = scales.reshape(-1)
    out = np.empty(flat.shape, np.float32)
    for i in range(flat.shape[0]):
        lib().orc_window_fp8_dequant(_p(flat[i]), float(sf[i]), D, _p(out[i]))
    return out.reshape(codes.shape)


def block_pool(scores, block, keep):
    """Hierarchical indexer pool of one sequence's scores: (blocks, pool)."""
    scores = _c(scores, np.int32)
    blocks = np.empty(keep, np.int32)
    pool = np.empty(keep * block, np.int32)
    n = lib().orc_block_pool(_p(scores), scores.size, block, keep, _p(blocks), _p(pool))
    return blocks, pool[:n].copy()


def pool_topk(q, keys, pool, k):
    """Top-K of one sequence over the pool's entries only."""
    q, keys, pool = _c(q, np.int8), _c(keys, np.int8), _c(pool, np.int32)
    out = np.empty(k, np.int32)
    lib().orc_pool_topk(_p(q), _p(keys), keys.shape[1], _p(pool), pool.size, k, _p(out))
    return out


def group_step(cfg: Cfg, modes, q, idx_q, windows, window_len, records, idx_cache,
               n_entries, hier_keep=0, hier_block=8):
    modes = np.ascontiguousarray(modes, dtype=np.int32)
    q, windows = _c(q, np.float32), _c(windows, np.float32)
    idx_q = _c(idx_q, np.int8)
    records, idx_cache = _c(records, np.uint8), _c(idx_cache, np.int8)
    n_entries = _c(n_entries, np.int32)
    L, B = q.shape[0], q.shape[1]
    cap = records.shape[1]
    out = np.empty((L, B, cfg.n_heads, cfg.latent_dim), np.float64)
    lse = np.empty((L, B, cfg.n_heads), np.float64)
    tk = np.empty((L, B, cfg.topk), np.int32)
    st = np.zeros(1, np.uint32)
    rc = lib().orc_group_step_hier(C.byref(cfg), L, _p(modes), B, _p(q), _p(idx_q),
                                   _p(windows), int(window_len), _p(records), _p(idx_cache),
                                   cap, _p(n_entries), int(hier_keep), int(hier_block),
                                   _p(out), _p(lse), _p(tk), _p(st))
    if rc:
        raise ValueError(f"orc_group_step failed: {rc}")
    return out, lse, tk, int(st[0])
