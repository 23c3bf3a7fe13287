"""CPU checks of the C ABI: libkvc.so builds, loads and exports every function
include/kvc.h declares; host-side size arithmetic matches the oracle; host
validation rejects bad arguments before any device work, and with no sm_100
device current the calls fail loudly instead of falling back."""
import ctypes as C
import os
import re
import subprocess

import pytest

from fp4_compressed_kv_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from fp4_compressed_kv_b200 import build, kvc
    build.build()
    return kvc


def _declared():
    src = open(os.path.join(ROOT, "include", "kvc.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvc_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 15
    so = lib.lib()
    for n in names:
        assert hasattr(so, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r" T (kvc_\w+)", out))
    assert set(names) <= exported
    assert lib.version().startswith("kvc")


def test_sizes_match_oracle(lib, orc):
    for name, w in synth.WORKLOADS.items():
        cfg = lib.config_for(w)
        ocfg = orc.make_cfg(w.latent, w.rope, w.group, w.scale_fmt, w.idx_dim, w.topk, w.window,
                            w.heads, w.sm_scale, w.ratio)
        assert lib.record_bytes(cfg) == orc.record_bytes(ocfg, True), name
        for padded in (False, True):
            assert lib.bytes_resident(cfg, w.entries, w.layers, padded) == \
                orc.bytes_resident(ocfg, w.entries, w.layers, 2 if w.act == "bf16" else 4, padded)
        assert lib.workspace_bytes(cfg, w.batch, w.entries) > 0
    w = synth.WORKLOADS["stack1m"]
    assert lib.bytes_resident(lib.config_for(w), 500_000, 20, False) == 219_949_120


def test_invalid_configs_rejected(lib):
    base = synth.WORKLOADS["mla32k"]
    for field, value in [("group", 48), ("group", 1024), ("latent_dim", 500), ("idx_dim", 100),
                         ("topk", 0), ("topk", 5000), ("scale_fmt", 3), ("act_dtype", 7),
                         ("sm_scale", 0.0), ("n_heads", 0), ("ratio", 3), ("ratio", 8),
                         ("idx_fmt", 2), ("idx_fmt", -1)]:
        cfg = lib.config_for(base)
        setattr(cfg, field, value)
        assert lib.record_bytes(cfg) == 0, field
        assert lib.workspace_bytes(cfg, 1, 10) == 0, field


def test_host_validation_before_device(lib):
    so = lib.lib()
    cfg = lib.config_for(synth.WORKLOADS["tiny"])
    cache = lib.CacheStruct(16, 16, 16, 1, 8)  # fake aligned addresses: never dereferenced
    # odd n_new is invalid whatever the device
    assert so.kvc_pack(C.byref(cfg), C.c_void_p(16), 3, C.c_void_p(16), C.c_void_p(16),
                       C.byref(cache), None, None) == 1
    # at the 4:1 ratio n_new must be a multiple of 4
    cfg4 = lib.config_for(synth.WORKLOADS["tiny"].scaled(ratio=4))
    assert lib.record_bytes(cfg4) == lib.record_bytes(cfg)
    assert so.kvc_pack(C.byref(cfg4), C.c_void_p(16), 6, C.c_void_p(16), C.c_void_p(16),
                       C.byref(cache), None, None) == 1
    # misaligned tokens
    assert so.kvc_pack(C.byref(cfg), C.c_void_p(17), 2, C.c_void_p(16), C.c_void_p(16),
                       C.byref(cache), None, None) == 1
    # too-small workspace
    assert so.kvc_index_topk(C.byref(cfg), C.c_void_p(16), C.byref(cache), C.c_void_p(16), None,
                             C.c_void_p(256), 16, None, None) == 7
    # Reuse as the first layer
    modes = (C.c_int32 * 2)(2, 0)
    assert so.kvc_layer_group_step(C.byref(cfg), 2, modes, C.c_void_p(16), C.c_void_p(16),
                                   C.c_void_p(16), 32, C.byref(cache), C.c_void_p(16), None,
                                   C.c_void_p(16), C.c_void_p(256), 1 << 30, None, None) == 1


def test_no_device_fails_loudly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    so = lib.lib()
    cfg = lib.config_for(synth.WORKLOADS["tiny"])
    cache = lib.CacheStruct(16, 16, 16, 1, 8)
    rc = so.kvc_pack(C.byref(cfg), C.c_void_p(16), 2, C.c_void_p(16), C.c_void_p(16),
                     C.byref(cache), None, None)
    assert rc == 6  # KVC_ERR_DEVICE: nothing was enqueued


def test_hier_workspace_and_validation(lib):
    so = lib.lib()
    w = synth.WORKLOADS["stack1m"]
    cfg = lib.config_for(w)
    plain = so.kvc_workspace_bytes(C.byref(cfg), 1, w.entries)
    hier = so.kvc_workspace_bytes_hier(C.byref(cfg), 1, w.entries, 2048, 8)
    # block scores (4 B per 8 entries) + pool blocks + lengths, each 256-aligned
    assert plain + (w.entries // 8) * 4 <= hier <= plain + (w.entries // 8) * 4 + 2048 * 4 + 1024
    assert so.kvc_workspace_bytes_hier(C.byref(cfg), 1, w.entries, 0, 0) == plain
    assert so.kvc_workspace_bytes_hier(C.byref(cfg), 1, w.entries, 2048, 0) == 0
    assert so.kvc_workspace_bytes_hier(C.byref(cfg), 1, w.entries, -1, 8) == 0
    cache = lib.CacheStruct(16, 16, 16, 1, 8)
    modes = (C.c_int32 * 2)(0, 1)
    for blocks, block in ((2048, 0), (70000, 8), (16, 300)):
        assert so.kvc_layer_group_step_hier(
            C.byref(cfg), blocks, block, 2, modes, C.c_void_p(16), C.c_void_p(16),
            C.c_void_p(16), 32, C.byref(cache), C.c_void_p(16), None, C.c_void_p(16),
            C.c_void_p(256), 1 << 30, None, None) == 1


def test_batched_workspace_and_validation(lib):
    so = lib.lib()
    w = synth.WORKLOADS["stack1m"]
    cfg = lib.config_for(w)
    one = so.kvc_workspace_bytes_batched(C.byref(cfg), 1, 1, w.entries)
    assert one > 0 and so.kvc_workspace_bytes_batched(C.byref(cfg), 5, 1, w.entries) == 5 * one
    assert so.kvc_workspace_bytes_batched(C.byref(cfg), 0, 1, w.entries) == 0
    assert so.kvc_workspace_bytes_batched(C.byref(cfg), 9, 1, w.entries) == 0
    cache = lib.CacheStruct(16, 16, 16, 1, 8)
    tiny = lib.config_for(synth.WORKLOADS["tiny"])  # idx_dim 32: not supported
    assert so.kvc_index_topk_batched(C.byref(tiny), 2, C.c_void_p(16), C.byref(cache),
                                     C.c_void_p(16), C.c_void_p(256), 1 << 30, None, None) == 4
    assert so.kvc_index_topk_batched(C.byref(cfg), 9, C.c_void_p(16), C.byref(cache),
                                     C.c_void_p(16), C.c_void_p(256), 1 << 30, None, None) == 1


def test_fp4_indexer_rows_and_rejections(lib):
    """FP4 indexer keys: 72-byte rows at 128 channels (idx_dim/2 + idx_dim/16),
    counted in the bytes resident; the hierarchical, batched and fixed-scratch
    variants refuse them before touching the device."""
    so = lib.lib()
    w = synth.WORKLOADS["mla32k"]
    c8, c4 = lib.config_for(w), lib.config_for(w.scaled(idx_fmt=1))
    assert lib.idx_row_bytes(c8) == 128 and lib.idx_row_bytes(c4) == 72
    assert lib.record_bytes(c4) == lib.record_bytes(c8)
    assert lib.bytes_resident(c8, 1000, 0, False) - lib.bytes_resident(c4, 1000, 0, False) == \
        1000 * (128 - 72)
    for di, rb in ((16, 9), (32, 18), (64, 36), (256, 144)):
        assert lib.idx_row_bytes(lib.config_for(w.scaled(idx_fmt=1, idx_dim=di))) == rb
    cache = lib.CacheStruct(16, 16, 16, 1, 8)
    assert so.kvc_index_topk_noalloc(C.byref(c4), C.c_void_p(16), C.byref(cache),
                                     C.c_void_p(16), None, None, None) == 4
    assert so.kvc_index_topk_batched(C.byref(c4), 2, C.c_void_p(16), C.byref(cache),
                                     C.c_void_p(16), C.c_void_p(256), 1 << 30, None, None) == 4
    modes = (C.c_int32 * 1)(0)
    assert so.kvc_layer_group_step_hier(C.byref(c4), 2048, 8, 1, modes, C.c_void_p(16),
                                        C.c_void_p(16), C.c_void_p(16), 32, C.byref(cache),
                                        C.c_void_p(16), None, C.c_void_p(16), C.c_void_p(256),
                                        1 << 30, None, None) == 4
    # the exact scores are 64-bit: no int32 score output for FP4 keys
    assert so.kvc_index_topk(C.byref(c4), C.c_void_p(16), C.byref(cache), C.c_void_p(16),
                             C.c_void_p(16), C.c_void_p(256), 1 << 30, None, None) == 4


def test_workspace_holds_fp4_keys(lib):
    """FP4 indexer keys keep one 64-bit key (exact score and index) per entry
    in the workspace's candidate region and their selection candidates (half
    a tile of keys per tile of 8192 entries) in its score region: the
    workspace is at least the int8 one and at least B (8 cap + 8 x 4096 x
    ceil(cap / 8192)) bytes, at any capacity."""
    w = synth.WORKLOADS["mla32k"]
    c8, c4 = lib.config_for(w), lib.config_for(w.scaled(idx_fmt=1))
    for B, cap in ((1, 1), (3, 1000), (32, 65600), (2, 131073), (1, 500_000)):
        n8, n4 = lib.workspace_bytes(c8, B, cap), lib.workspace_bytes(c4, B, cap)
        tiles = -(-cap // 8192)
        assert n4 >= n8 > 0
        assert n4 >= B * (8 * cap + 8 * 4096 * tiles)


def test_capacity_limit_on_the_host(lib):
    """The top-K and the group step refuse capacities past 8,388,608 entries
    before looking for a device."""
    so = lib.lib()
    cfg = lib.config_for(synth.WORKLOADS["tiny"])
    big = lib.CacheStruct(16, 16, 16, 1, 8_388_609)
    assert so.kvc_index_topk(C.byref(cfg), C.c_void_p(16), C.byref(big), C.c_void_p(16), None,
                             C.c_void_p(256), 1 << 62, None, None) == 2
    modes = (C.c_int32 * 1)(0)
    assert so.kvc_layer_group_step(C.byref(cfg), 1, modes, C.c_void_p(16), C.c_void_p(16),
                                   C.c_void_p(16), 32, C.byref(big), C.c_void_p(16), None,
                                   C.c_void_p(16), C.c_void_p(256), 1 << 62, None, None) == 2
