"""The multi-GPU path on CPU: world-size-2 `gloo` process groups.

SGMV has no cross-GPU exchange, so N GPUs run N independent replicas and the only
multi-rank logic is the host side of bench.py: every rank groups its own batch, times its
replica, and the job's time is the slowest rank's; the job's
throughput is all ranks' tokens over that time; the reference arm runs on rank 0 only.
These tests run that logic in two real processes over gloo (127.0.0.1), without a GPU.
"""
from __future__ import annotations

import json
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, outdir: str):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    from datetime import timedelta

    import bench
    import oracle
    from adapter_matmul_b200 import inputs, sgmv

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        # each replica's own token batch: the Zipf 70B decode draw with a rank-specific seed
        w = inputs.llama70b_decode(8192, seed=rank)
        seg, idx, perm = sgmv.lora_sgmv_group_segments(w.ids, w.num_adapters)
        oseg, oidx, operm = oracle.group_segments(w.ids, w.num_adapters)
        grouping_ok = bool(np.array_equal(seg, oseg) and np.array_equal(idx, oidx) and np.array_equal(perm, operm))
        # a rank-specific "elapsed" time; the job's time is the slowest rank's
        local_s = 0.010 + 0.005 * rank
        t_max = bench.max_over_ranks(local_s, world)
        value = bench.job_tokens_per_s(w.T * 100, world, t_max)
        # the reference arm: ranks other than 0 do no work and print nothing
        ref = None
        if rank != 0:
            ref = bench.run_reference(None, bench.make_spec("tiny"), rank)
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump({"grouping_ok": grouping_ok, "t_max": t_max, "value": value, "T": w.T,
                       "ids": [int(v) for v in w.ids[:32]], "ref_is_none": ref is None}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_over_gloo(tmp_path):
    import torch.multiprocessing as mp

    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["grouping_ok"]
        assert r["t_max"] == pytest.approx(0.015)  # the slower rank's time on every rank
        assert r["value"] == pytest.approx(r["T"] * 100 * world / 0.015)
    assert res[1]["ref_is_none"]
    # the two replicas drew different batches (their own seeds), grouped on their own
    assert res[0]["ids"] != res[1]["ids"]


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(0.25, 1) == 0.25
    assert bench.job_tokens_per_s(1000, 1, 0.5) == pytest.approx(2000.0)
    assert bench.job_tokens_per_s(1000, 4, 0.5) == pytest.approx(8000.0)
