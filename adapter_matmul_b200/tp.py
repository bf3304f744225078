"""SGMV across the ranks of a tensor-parallel group (one process per GPU).

Sharding. A layer whose base weight is split over N ranks splits the SGMV operands the same
way: rank p holds X[:, K_p] (its slice of H1), the rows A_i[K_p, :] of every adapter, the
columns B_i[:, N_p] of every adapter and Y[:, N_p] (its slice of H2). Its share of the delta
(the batched LoRA term of the README page "Punica：多 LoRA 模型统一服务框架", LoRA and
multi-LoRA paragraphs) is

    Y[t, N_p] += scale * (sum_q X[t, K_q] @ A_i[K_q, :]) @ B_i[:, N_p],

so every rank runs the shrink on its K slice (a partial V in fp32), the partial V are summed
over the group (one all-reduce of T x r fp32 values, 64 KB for 256 tokens at r = 64), and
every rank runs the expand on its N slice. The shrink and the expand are this library's
kernels (lora_sgmv_shrink, lora_sgmv_expand); the sum is torch.distributed's all-reduce
(NCCL on GPUs), issued on the current stream between them.
"""
from __future__ import annotations

from typing import Tuple

from . import sgmv


def shard_range(n: int, world: int, rank: int, align: int = 8) -> Tuple[int, int]:
    """[lo, hi) of rank's contiguous slice of n columns: slices of equal size rounded up to a
    multiple of `align` (the kernels need 16-byte rows), the last one taking the remainder;
    trailing ranks may get an empty slice when n is small."""
    if world < 1 or not 0 <= rank < world or n < 0 or align < 1:
        raise ValueError(f"bad shard request n={n} world={world} rank={rank} align={align}")
    per = -(-n // world)
    per = -(-per // align) * align
    lo = min(n, rank * per)
    return lo, min(n, lo + per)


def tp_apply(Y_shard, X_shard, A_ptrs, B_ptrs, seg_starts, lora_idx, n_segments: int, num_adapters: int, T: int,
             H1_shard: int, r: int, H2_shard: int, scale: float, dtype: int, V, group=None,
             dev_status=None) -> None:
    """This rank's share of a tensor-parallel SGMV call.

    Y_shard   device [T, H2_shard], in/out: this rank's columns of Y.
    X_shard   device [T, H1_shard]: this rank's columns of X.
    A_ptrs    device table of num_adapters pointers to A_i[K_p, :] ([H1_shard, r] each).
    B_ptrs    device table of num_adapters pointers to B_i[:, N_p] ([r, H2_shard] each).
    V         device fp32 [T, r] scratch, summed in place over the group (rows of segments the
              kernels reject are left as they were and are not used).
    group     torch.distributed process group (None: the default group).
    Runs on the current CUDA stream, which the all-reduce also follows.
    """
    import torch.distributed as dist

    if H1_shard > 0:
        sgmv.lora_sgmv_shrink(V, X_shard, A_ptrs, seg_starts, lora_idx, n_segments, num_adapters, T, H1_shard, r,
                              dtype, dev_status)
    else:  # a rank without H1 columns contributes zeros
        V.zero_()
    dist.all_reduce(V, op=dist.ReduceOp.SUM, group=group)
    if H2_shard > 0:
        sgmv.lora_sgmv_expand(Y_shard, V, B_ptrs, seg_starts, lora_idx, n_segments, num_adapters, T, r, H2_shard,
                              scale, dtype, dev_status)
