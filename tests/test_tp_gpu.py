"""Tensor-parallel SGMV on one GPU: the library's kernels on sharded operands.

A layer split over N ranks gives rank p the columns K_p of X and the rows K_p of every A_i
(its share of H1), and the columns N_p of every B_i and of Y (its share of H2). Each rank
runs the shrink kernel on its K slice into a partial V (fp32), the partial V are summed,
and each rank runs the expand kernel on its N slice. Here the N ranks' steps run one after
another on the one device (the sum of the partial V stands in for the all-reduce); every
element of the stitched Y is compared with the unsharded oracle. A world-size-1 NCCL group
then runs adapter_matmul_b200.tp.tp_apply itself (shrink, NCCL all-reduce, expand).
"""
import os
import socket

import numpy as np
import pytest
import torch

from adapter_matmul_b200 import inputs, sgmv, tp
from gpu_helpers import DeviceProblem, assert_close, dt_code, from_dev, to_dev

pytestmark = pytest.mark.gpu


def _shard_tables(p: DeviceProblem, k_lo, k_hi, n_lo, n_hi):
    """Pointer tables of rank p's shards: A_i[K_p, :] is a run of whole rows of A_i (a pointer
    into it); B_i[:, N_p] is strided in B_i, so the rank holds its own dense copy."""
    w = p.w
    r = w.r
    a_ptrs, b_ptrs, keep = [], [], []
    for i in range(w.num_adapters):
        if i in p.dA:
            a_ptrs.append(p.dA[i].data_ptr() + k_lo * r * 2)
            b = p.dB[i][:, n_lo:n_hi].contiguous()
            keep.append(b)
            b_ptrs.append(b.data_ptr())
        else:
            a_ptrs.append(0)
            b_ptrs.append(0)
    return (torch.tensor(a_ptrs, dtype=torch.int64, device="cuda"),
            torch.tensor(b_ptrs, dtype=torch.int64, device="cuda"), keep)


@pytest.mark.parametrize("name", ["llama70b_decode_h28672", "llama70b_decode_h8192"])
@pytest.mark.parametrize("world", [2, 4])
def test_sharded_kernels_match_unsharded_oracle(name, world):
    w = inputs.make(name)
    p = DeviceProblem(w, y_random=True)
    dt = dt_code(w.dtype)
    V_parts, Y_out = [], torch.empty_like(p.Y)
    keep = []
    for rank in range(world):
        k_lo, k_hi = tp.shard_range(w.H1, world, rank)
        n_lo, n_hi = tp.shard_range(w.H2, world, rank)
        A_ptrs, B_ptrs, kb = _shard_tables(p, k_lo, k_hi, n_lo, n_hi)
        keep.append((A_ptrs, B_ptrs, kb))
        V = torch.full((w.T, w.r), float("nan"), dtype=torch.float32, device="cuda")
        if k_hi > k_lo:
            X_p = p.X[:, k_lo:k_hi].contiguous()
            sgmv.lora_sgmv_shrink(V, X_p, A_ptrs, p.d_seg, p.d_idx, p.n, w.num_adapters, w.T, k_hi - k_lo, w.r,
                                  dt, p.status)
        else:
            V.zero_()
        V_parts.append(V)
    V_sum = torch.stack(V_parts).sum(0)  # stands in for the all-reduce over the ranks
    for rank in range(world):
        n_lo, n_hi = tp.shard_range(w.H2, world, rank)
        if n_hi == n_lo:
            continue
        _, B_ptrs, _ = keep[rank]
        Y_p = p.Y[:, n_lo:n_hi].contiguous()
        sgmv.lora_sgmv_expand(Y_p, V_sum, B_ptrs, p.d_seg, p.d_idx, p.n, w.num_adapters, w.T, w.r, n_hi - n_lo,
                              w.scale, dt, p.status)
        Y_out[:, n_lo:n_hi] = Y_p
    torch.cuda.synchronize()
    assert int(p.status.item()) == 0
    assert_close(from_dev(Y_out), p.oracle_apply(), w.dtype, f"{name} over {world} shards")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_tp_apply_world_one_nccl():
    import torch.distributed as dist
    from datetime import timedelta

    w = inputs.make("llama70b_decode_h8192")
    p = DeviceProblem(w, y_random=True)
    own_group = not dist.is_initialized()
    if own_group:
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                                timeout=timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        V = torch.empty((w.T, w.r), dtype=torch.float32, device="cuda")
        tp.tp_apply(p.Y, p.X, p.A_ptrs, p.B_ptrs, p.d_seg, p.d_idx, p.n, w.num_adapters, w.T, w.H1, w.r, w.H2,
                    w.scale, dt_code(w.dtype), V, dev_status=p.status)
        torch.cuda.synchronize()
    finally:
        if own_group:
            dist.destroy_process_group()
    assert int(p.status.item()) == 0
    assert_close(from_dev(p.Y), p.oracle_apply(), w.dtype, "tp_apply, one NCCL rank")
