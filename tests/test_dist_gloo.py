"""World-size-2 gloo tests (CPU) of the multi-rank host logic: each rank decodes
its own sequences (distinct seeds, same shapes), the timed value is the MAX
over ranks, and the job throughput counts every rank's sequences."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle
    from fp4_compressed_kv_b200 import dist as kd, synth
    r, ws, lr = kd.world()
    assert (r, ws, lr) == (rank, world, rank)
    w = kd.rank_workload(synth.WORKLOADS["tiny"], rank)
    inp = synth.make_inputs(w)
    # each rank runs its own (oracle) decode problem; report a per-rank "time"
    cfg = oracle.make_cfg(w.latent, w.rope, w.group, w.scale_fmt, w.idx_dim, w.topk, w.window,
                          w.heads, w.sm_scale)
    tk = oracle.index_topk(cfg, inp["idx_q"][0].numpy(), inp["idx_k"].numpy(),
                           np.array([w.entries], np.int32))
    fake_ms = 10.0 + 5.0 * rank
    kd.barrier()
    ms_max = kd.max_over_ranks(fake_ms)
    thr = kd.job_throughput(steps=4, batch_per_rank=w.batch, world_size=ws, ms_max=ms_max)
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), tk=tk, q=inp["q"].float().numpy(),
             ms_max=ms_max, thr=thr)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_replicas(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    r0 = np.load(tmp_path / "rank0.npz")
    r1 = np.load(tmp_path / "rank1.npz")
    # same shapes, different sequences
    assert r0["q"].shape == r1["q"].shape and not np.array_equal(r0["q"], r1["q"])
    assert not np.array_equal(r0["tk"], r1["tk"])
    # the slowest rank's time, on every rank
    assert float(r0["ms_max"]) == float(r1["ms_max"]) == 15.0
    # 4 steps x 1 sequence x 2 ranks in 15 ms
    assert float(r0["thr"]) == pytest.approx(4 * 1 * 2 / 0.015)


def test_single_process_fallbacks():
    from fp4_compressed_kv_b200 import dist as kd
    assert kd.max_over_ranks(3.5) == 3.5
    assert kd.job_throughput(10, 32, 1, 100.0) == pytest.approx(3200.0)
