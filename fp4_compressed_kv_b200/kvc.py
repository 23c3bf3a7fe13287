"""Thin Python binding of libkvc.so (include/kvc.h): argument marshalling only.

Every call hands raw device pointers of torch tensors and the current CUDA
stream to the C ABI; all work runs in the library's sm_100a kernels.  There
is no fallback: if ``libkvc.so`` is missing or no sm_100 device is current,
the calls raise.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvc.so")

OK = 0
STATUS_NAMES = {0: "ok", 1: "invalid", 2: "capacity", 3: "cuda", 4: "unsupported", 5: "timeout",
                6: "device", 7: "workspace"}
SCALE_F32, SCALE_UE4M3 = 0, 1
FULL, REINDEX, REUSE = 0, 1, 2
F32, BF16 = 0, 1
DEV_NONFINITE, DEV_BAD_INDEX, DEV_CAPACITY, DEV_TIMEOUT, DEV_BAD_LENGTH = 1, 2, 4, 8, 16


class KvcError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)} ({_lib().kvc_status_string(status).decode()})")


class Config(C.Structure):
    _fields_ = [("latent_dim", C.c_int32), ("rope_dim", C.c_int32), ("group", C.c_int32),
                ("scale_fmt", C.c_int32), ("idx_dim", C.c_int32), ("topk", C.c_int32),
                ("window", C.c_int32), ("n_heads", C.c_int32), ("sm_scale", C.c_float),
                ("act_dtype", C.c_int32), ("ratio", C.c_int32), ("idx_fmt", C.c_int32)]


class CacheStruct(C.Structure):
    _fields_ = [("records", C.c_void_p), ("idx_k", C.c_void_p), ("n_entries", C.c_void_p),
                ("batch", C.c_int32), ("capacity", C.c_int32)]


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libkvc.so not built ({LIB_PATH}); run "
                               "`python -m fp4_compressed_kv_b200.build`")
        lib = C.CDLL(LIB_PATH)
        P, I, Z = C.c_void_p, C.c_int, C.c_size_t
        S = C.c_int  # kvc_status
        sig = {
            "kvc_record_bytes": (Z, [P]),
            "kvc_idx_row_bytes": (Z, [P]),
            "kvc_bytes_resident": (Z, [P, C.c_int64, I, I]),
            "kvc_workspace_bytes": (Z, [P, I, I]),
            "kvc_pack": (S, [P, P, I, P, P, P, P, P]),
            "kvc_index_topk": (S, [P, P, P, P, P, P, Z, P, P]),
            "kvc_index_topk_noalloc": (S, [P, P, P, P, P, P, P]),
            "kvc_sparse_decode_attn": (S, [P, P, P, P, P, I, P, P, P, Z, P, P]),
            "kvc_layer_group_step": (S, [P, I, P, P, P, P, I, P, P, P, P, P, Z, P, P]),
            "kvc_workspace_bytes_hier": (Z, [P, I, I, I, I]),
            "kvc_workspace_bytes_batched": (Z, [P, I, I, I]),
            "kvc_pack_window_fp8": (S, [P, P, C.c_int64, P, P, P, P]),
            "kvc_sparse_decode_attn_fp8win": (S, [P, P, P, P, P, P, I, P, P, P, Z, P, P]),
            "kvc_index_topk_batched": (S, [P, I, P, P, P, P, Z, P, P]),
            "kvc_layer_group_step_hier": (S, [P, I, I, I, P, P, P, P, I, P, P, P, P, P, Z, P,
                                              P]),
            "kvc_e2m1_encode": (S, [P, C.c_int64, P, P]),
            "kvc_e4m3_encode": (S, [P, C.c_int64, P, P]),
            "kvc_trace_begin": (S, [I]),
            "kvc_trace_end": (S, []),
            "kvc_trace_kernel": (S, [C.c_char_p, C.POINTER(C.c_int), C.POINTER(C.c_double)]),
            "kvc_launch_count": (C.c_uint64, []),
            "kvc_debug_set_wait_limit_ns": (S, [C.c_uint64]),
            "kvc_status_string": (C.c_char_p, [I]),
            "kvc_version": (C.c_char_p, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def lib():
    """The loaded C library (ctypes.CDLL); raises if it is not built."""
    return _lib()


def _check(fn, rc):
    if rc != OK:
        raise KvcError(fn, rc)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def make_config(latent_dim, rope_dim, group, scale_fmt, idx_dim, topk, window, n_heads, sm_scale,
                act_dtype, ratio=2, idx_fmt=0) -> Config:
    """ratio: raw tokens per entry, 2 or 4; idx_fmt: indexer keys as int8 (0)
    or FP4 rows (1)."""
    return Config(latent_dim, rope_dim, group, scale_fmt, idx_dim, topk, window, n_heads,
                  float(sm_scale), act_dtype, ratio, idx_fmt)


def config_for(w) -> Config:
    """kvc_config of a synth.Workload."""
    return make_config(w.latent, w.rope, w.group, w.scale_fmt, w.idx_dim, w.topk, w.window,
                       w.heads, w.sm_scale, F32 if w.act == "f32" else BF16, w.ratio,
                       w.idx_fmt)


def record_bytes(cfg: Config) -> int:
    return int(_lib().kvc_record_bytes(C.byref(cfg)))


def idx_row_bytes(cfg: Config) -> int:
    return int(_lib().kvc_idx_row_bytes(C.byref(cfg)))


def bytes_resident(cfg: Config, entries: int, n_layers: int, padded: bool) -> int:
    return int(_lib().kvc_bytes_resident(C.byref(cfg), entries, n_layers, int(padded)))


def workspace_bytes(cfg: Config, batch: int, capacity: int) -> int:
    return int(_lib().kvc_workspace_bytes(C.byref(cfg), batch, capacity))


class Cache:
    """Device buffers of one stored cache (records, indexer keys, lengths)."""

    def __init__(self, cfg: Config, batch: int, capacity: int, device="cuda"):
        rb = record_bytes(cfg)
        if rb == 0:
            raise ValueError("invalid kvc config")
        self.cfg, self.batch, self.capacity = cfg, batch, capacity
        self.records = torch.zeros(batch, capacity, rb, dtype=torch.uint8, device=device)
        if cfg.idx_fmt == 1:  # FP4 rows of idx_dim/2 + idx_dim/16 bytes
            self.idx_k = torch.zeros(batch, capacity, idx_row_bytes(cfg), dtype=torch.uint8,
                                     device=device)
        else:
            self.idx_k = torch.zeros(batch, capacity, cfg.idx_dim, dtype=torch.int8,
                                     device=device)
        self.n_entries = torch.zeros(batch, dtype=torch.int32, device=device)

    def struct(self) -> CacheStruct:
        return CacheStruct(self.records.data_ptr(), self.idx_k.data_ptr(),
                           self.n_entries.data_ptr(), self.batch, self.capacity)


def workspace(cfg: Config, batch: int, capacity: int, device="cuda", hier_blocks: int = 0,
              hier_block: int = 8) -> torch.Tensor:
    """Workspace for the calls on `batch` x `capacity` (and, with hier_blocks
    > 0, for the hierarchical group step)."""
    if hier_blocks:
        n = int(_lib().kvc_workspace_bytes_hier(C.byref(cfg), batch, capacity, hier_blocks,
                                                 hier_block))
    else:
        n = workspace_bytes(cfg, batch, capacity)
    if n == 0:
        raise KvcError("invalid workspace request")
    return torch.zeros(n + 256, dtype=torch.uint8, device=device)  # zero-filled before first use


def _ws(ws):
    # 256-byte aligned view into a workspace tensor
    base = ws.data_ptr()
    off = (-base) % 256
    return C.c_void_p(base + off), ws.numel() - off


def pack_window_fp8(cfg, rows, codes, scales, status=None, stream=None):
    """rows [..][D] -> codes [..][D] uint8 (signed E4M3), scales [..] fp32."""
    n = rows.numel() // rows.shape[-1]
    _check("kvc_pack_window_fp8", _lib().kvc_pack_window_fp8(
        C.byref(cfg), _ptr(rows), n, _ptr(codes), _ptr(scales), _ptr(status), _stream(stream)))


def sparse_decode_attn_fp8win(cfg, q, cache: Cache, topk_idx, win_codes, win_scales, window_len,
                              out, ws, lse=None, status=None, stream=None):
    p, n = _ws(ws)
    cs = cache.struct()
    _check("kvc_sparse_decode_attn_fp8win", _lib().kvc_sparse_decode_attn_fp8win(
        C.byref(cfg), _ptr(q), C.byref(cs), _ptr(topk_idx), _ptr(win_codes), _ptr(win_scales),
        int(window_len), _ptr(out), _ptr(lse), p, n, _ptr(status), _stream(stream)))


def workspace_batched(cfg: Config, nq: int, batch: int, capacity: int,
                      device="cuda") -> torch.Tensor:
    """Workspace for index_topk_batched with nq queries per sequence."""
    n = int(_lib().kvc_workspace_bytes_batched(C.byref(cfg), nq, batch, capacity))
    if n == 0:
        raise KvcError("invalid batched workspace request")
    return torch.zeros(n + 256, dtype=torch.uint8, device=device)  # zero-filled before first use


def index_topk_batched(cfg, idx_q, cache: Cache, topk_out, ws, status=None, stream=None):
    """idx_q [nq][B][Di] int8 -> topk_out [nq][B][K]: every query against the
    cache in one tensor-core pass."""
    p, n = _ws(ws)
    cs = cache.struct()
    _check("kvc_index_topk_batched", _lib().kvc_index_topk_batched(
        C.byref(cfg), idx_q.shape[0], _ptr(idx_q), C.byref(cs), _ptr(topk_out), p, n,
        _ptr(status), _stream(stream)))


def pack(cfg, tokens, gate, idx_k_new, cache: Cache, status=None, stream=None):
    n_new = tokens.shape[1]
    cs = cache.struct()
    _check("kvc_pack", _lib().kvc_pack(C.byref(cfg), _ptr(tokens), n_new, _ptr(gate),
                                       _ptr(idx_k_new), C.byref(cs), _ptr(status), _stream(stream)))


def index_topk(cfg, idx_q, cache: Cache, topk_out, ws, scores=None, status=None, stream=None):
    p, n = _ws(ws)
    cs = cache.struct()
    _check("kvc_index_topk", _lib().kvc_index_topk(C.byref(cfg), _ptr(idx_q), C.byref(cs),
                                                   _ptr(topk_out), _ptr(scores), p, n,
                                                   _ptr(status), _stream(stream)))


def index_topk_noalloc(cfg, idx_q, cache: Cache, topk_out, scores=None, status=None,
                       stream=None):
    """kvc_index_topk with the library's fixed scratch (no workspace argument)."""
    cs = cache.struct()
    _check("kvc_index_topk_noalloc", _lib().kvc_index_topk_noalloc(
        C.byref(cfg), _ptr(idx_q), C.byref(cs), _ptr(topk_out), _ptr(scores), _ptr(status),
        _stream(stream)))


def sparse_decode_attn(cfg, q, cache: Cache, topk, window, window_len, out, ws, lse=None,
                       status=None, stream=None):
    p, n = _ws(ws)
    cs = cache.struct()
    _check("kvc_sparse_decode_attn", _lib().kvc_sparse_decode_attn(
        C.byref(cfg), _ptr(q), C.byref(cs), _ptr(topk), _ptr(window), int(window_len), _ptr(out),
        _ptr(lse), p, n, _ptr(status), _stream(stream)))


def layer_group_step(cfg, modes, q, idx_q, windows, window_len, cache: Cache, out, topk, ws,
                     lse=None, status=None, stream=None, hier_blocks=0, hier_block=8):
    """One decode step through a CSA2 layer group; hier_blocks > 0 turns on
    the hierarchical indexer (the workspace must have been sized for it)."""
    modes_arr = (C.c_int32 * len(modes))(*modes)
    p, n = _ws(ws)
    cs = cache.struct()
    if hier_blocks:
        _check("kvc_layer_group_step_hier", _lib().kvc_layer_group_step_hier(
            C.byref(cfg), int(hier_blocks), int(hier_block), len(modes), modes_arr, _ptr(q),
            _ptr(idx_q), _ptr(windows), int(window_len), C.byref(cs), _ptr(out), _ptr(lse),
            _ptr(topk), p, n, _ptr(status), _stream(stream)))
        return
    _check("kvc_layer_group_step", _lib().kvc_layer_group_step(
        C.byref(cfg), len(modes), modes_arr, _ptr(q), _ptr(idx_q), _ptr(windows), int(window_len),
        C.byref(cs), _ptr(out), _ptr(lse), _ptr(topk), p, n, _ptr(status), _stream(stream)))


def e2m1_encode(x, codes, stream=None):
    _check("kvc_e2m1_encode", _lib().kvc_e2m1_encode(_ptr(x), x.numel(), _ptr(codes),
                                                     _stream(stream)))


def e4m3_encode(x, out, stream=None):
    _check("kvc_e4m3_encode", _lib().kvc_e4m3_encode(_ptr(x), x.numel(), _ptr(out),
                                                     _stream(stream)))


def trace_begin(max_launches: int = 4096):
    _check("kvc_trace_begin", _lib().kvc_trace_begin(max_launches))


def trace_end():
    _check("kvc_trace_end", _lib().kvc_trace_end())


def trace_kernel(name: str):
    n = C.c_int(0)
    ms = C.c_double(0.0)
    _check("kvc_trace_kernel", _lib().kvc_trace_kernel(name.encode(), C.byref(n), C.byref(ms)))
    return n.value, ms.value


def launch_count() -> int:
    return int(_lib().kvc_launch_count())


def debug_set_wait_limit_ns(ns: int):
    """Test hook: bound of every in-kernel wait of later launches (0 = one
    non-blocking poll; the library's default is 2_000_000_000)."""
    _check("kvc_debug_set_wait_limit_ns", _lib().kvc_debug_set_wait_limit_ns(int(ns)))


def version() -> str:
    return _lib().kvc_version().decode()
