"""Tensor-parallel SGMV host logic on CPU: two `gloo` ranks, each with its slices of H1 and H2.

adapter_matmul_b200.tp.tp_apply runs the library's shrink on the rank's H1 slice, sums the
partial V over the group and runs the expand on the rank's H2 slice. Without a GPU the two
kernel calls are replaced, in the rank processes of this test only, by the binary64 oracle
on the same shard arrays; what is checked is the host logic: the shard ranges, the order of
the steps and the all-reduce, against the unsharded binary64 oracle.
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


def test_shard_range_covers_and_aligns():
    sys.path.insert(0, ROOT)
    from adapter_matmul_b200.tp import shard_range

    for n in (0, 1, 8, 64, 72, 4096, 28672, 4100):
        for world in (1, 2, 3, 4, 8):
            parts = [shard_range(n, world, p) for p in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            for (lo, hi), (lo2, _) in zip(parts, parts[1:]):
                assert hi == lo2 and lo <= hi
            assert all(lo % 8 == 0 for lo, hi in parts if hi > lo)  # non-empty slices start aligned
    with pytest.raises(ValueError):
        shard_range(64, 2, 2)


def _rank_main(rank: int, world: int, port: int, outdir: str):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from datetime import timedelta

    import torch
    import torch.distributed as dist

    import oracle
    from adapter_matmul_b200 import inputs, sgmv, tp

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w = inputs.small_random(24, 3, 64, 48, 8, "f16", seed=3)
        seg, idx, _ = oracle.group_segments(w.ids, w.num_adapters)
        X, Y = w.x(), w.y_random()
        A = [w.adapter_a(i) for i in range(3)]
        B = [w.adapter_b(i) for i in range(3)]
        k0, k1 = tp.shard_range(w.H1, world, rank)
        n0, n1 = tp.shard_range(w.H2, world, rank)
        Xp = np.ascontiguousarray(X[:, k0:k1])
        Ap = [np.ascontiguousarray(a[k0:k1]) for a in A]
        Bp = [np.ascontiguousarray(b[:, n0:n1]) for b in B]
        y = oracle.decode(Y, w.dtype)

        # stand-ins for the two kernel calls, on this rank's shard arrays (binary64 oracle)
        def shrink(V, X_shard, A_ptrs, seg_starts, lora_idx, n, na, T, H1, r, dtype, status=None, stream=None):
            assert H1 == k1 - k0 and X_shard is Xp and r == w.r
            v, sk = oracle.shrink_f64(Xp, Ap, seg, idx, r, w.dtype)
            V.copy_(torch.from_numpy(v))

        def expand(Y_shard, V, B_ptrs, seg_starts, lora_idx, n, na, T, r, H2, scale, dtype, status=None, stream=None):
            assert H2 == n1 - n0
            out, sk = oracle.expand_f64(Y_shard.numpy(), V.numpy(), Bp, seg, idx, scale, w.dtype)
            Y_shard.copy_(torch.from_numpy(out))

        sgmv.lora_sgmv_shrink, sgmv.lora_sgmv_expand = shrink, expand
        V = torch.zeros((w.T, w.r), dtype=torch.float64)
        Y_shard = torch.from_numpy(np.ascontiguousarray(y[:, n0:n1]))
        tp.tp_apply(Y_shard, Xp, None, None, seg, idx, len(idx), w.num_adapters, w.T, k1 - k0, w.r, n1 - n0,
                    w.scale, sgmv.F16, V)
        full, _ = oracle.apply_f64(y, X, A, B, seg, idx, w.scale, w.dtype)
        ok = bool(np.allclose(Y_shard.numpy(), full[:, n0:n1], rtol=1e-12, atol=1e-12))
        v_full, _ = oracle.shrink_f64(X, A, seg, idx, w.r, w.dtype)
        v_ok = bool(np.allclose(V.numpy(), v_full, rtol=1e-12, atol=1e-12))
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump({"ok": ok, "v_ok": v_ok, "k": [k0, k1], "n": [n0, n1]}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_tensor_parallel_two_ranks_over_gloo(tmp_path):
    import torch.multiprocessing as mp

    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert [r["k"] for r in res] == [[0, 32], [32, 64]]
    assert [r["n"] for r in res] == [[0, 24], [24, 48]]
    for r in res:
        assert r["v_ok"], "the summed partial V differs from the unsharded shrink"
        assert r["ok"], "a Y shard differs from the unsharded oracle"
