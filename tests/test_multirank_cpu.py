"""The multi-GPU benchmark path's host logic on CPU: two gloo ranks.

Each rank scans its own sequences (its own seed); the only collective is the max over ranks
of the per-rank times, and the whole-job throughput is all ranks' tokens over that time.
"""
import json
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from quantized_mamba_ssd_b200 import dist_util
from quantized_mamba_ssd_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [3.0, 7.5][rank]
        ms_max = dist_util.max_over_ranks(ms, "cpu")
        case = W.make_prefill(1, 64, 2, 64, 16, 1, 64, seed=dist_util.rank_seed(1003, rank))
        digest = int(np.abs(case.x.astype(np.int64)).sum())
        res = {"rank": rank, "ms_max": ms_max, "digest": digest,
               "tps": dist_util.aggregate_tokens_per_s(100, world, ms_max)}
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_shard_the_batch(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    assert all(r["ms_max"] == 7.5 for r in res)              # max over ranks
    assert res[0]["digest"] != res[1]["digest"]               # each rank its own batch
    assert abs(res[0]["tps"] - 100 * 2 / 7.5e-3) < 1e-6       # all tokens / slowest rank


def test_single_process_max_is_identity():
    assert dist_util.max_over_ranks(4.25, "cpu") == 4.25
    assert dist_util.rank_seed(1003, 0) == 1003
