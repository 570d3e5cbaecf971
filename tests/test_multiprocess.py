"""The multi-process (data-parallel) host logic on CPU: two gloo ranks.

Each rank draws its batch shard, runs the fp64 oracle on it, and the gathered
result must equal the oracle on the global batch (no cross-unit terms, shards
disjoint and complete); the timing reduction is a max over ranks.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from test_sequence_modeling_b200 import inputs as I
from test_sequence_modeling_b200 import sharding

CFG = I.CONFIGS["linear_ln_B16H32T8192"].replace(B=2, H=2, T=32)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_shard(cfg, data, rank_offset):
    import oracle
    f = {k: v.astype(np.float64) for k, v in data.items() if isinstance(v, np.ndarray)}
    return oracle.ttt_linear_ln(f["Q"], f["K"], f["V"], f["eta"], f["W0"], cfg.b, f["gamma"],
                                f["beta"], cfg.ln_eps, nthreads=1)


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg, off = sharding.shard(CFG, world, rank)
        data = I.make_inputs(cfg, bf16_as_bits=False, batch_offset=off)
        Z, W = _run_shard(cfg, data, off)
        zs = [torch.empty(Z.shape, dtype=torch.float64) for _ in range(world)]
        ws = [torch.empty(W.shape, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(zs, torch.from_numpy(Z))
        dist.all_gather(ws, torch.from_numpy(W))
        mx = sharding.max_over_ranks([float(rank + 1)], dist)
        if rank == 0:
            np.save(os.path.join(out_dir, "Z.npy"), torch.cat(zs).numpy())
            np.save(os.path.join(out_dir, "W.npy"), torch.cat(ws).numpy())
            np.save(os.path.join(out_dir, "max.npy"), np.array(mx))
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_equal_the_global_batch(tmp_path):
    import oracle
    oracle.build()
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn")
    Zg = np.load(tmp_path / "Z.npy")
    Wg = np.load(tmp_path / "W.npy")
    gcfg = sharding.global_config(CFG, world)
    Zr, Wr = _run_shard(gcfg, I.make_inputs(gcfg, bf16_as_bits=False), 0)
    assert np.array_equal(Zg, Zr) and np.array_equal(Wg, Wr)
    assert float(np.load(tmp_path / "max.npy")[0]) == world


def test_shard_offsets():
    offs = [sharding.shard(CFG, 4, r)[1] for r in range(4)]
    assert offs == [0, 2, 4, 6]
    with pytest.raises(ValueError):
        sharding.shard(CFG, 2, 2)
