"""Property tests (hypothesis) of the library's host logic, each against its plain definition.

- lora_sgmv_group_segments (host C++): the permutation is numpy's stable argsort of the ids,
  segments are the runs of equal ids in ascending order with their counts, none is empty;
- lora_sgmv_auto_variant: the rule its header comment states, written out here;
- bench.rows_share and tp.shard_range: brute force.
"""
from __future__ import annotations

import os
import sys

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from adapter_matmul_b200 import sgmv  # noqa: E402


@settings(max_examples=300, deadline=None)
@given(st.lists(st.integers(0, 40), min_size=1, max_size=400), st.integers(0, 5))
def test_group_segments_is_a_stable_sort_into_runs(ids, extra):
    ids = np.array(ids, np.int32)
    A = int(ids.max()) + 1 + extra
    seg, idx, perm = sgmv.lora_sgmv_group_segments(ids, A)
    assert np.array_equal(perm, np.argsort(ids, kind="stable"))
    counts = np.bincount(ids, minlength=A)
    assert np.array_equal(idx, np.nonzero(counts)[0])                  # ascending, no empty segment
    assert np.array_equal(np.diff(seg), counts[counts > 0])
    assert seg[0] == 0 and seg[-1] == len(ids)
    for s in range(len(idx)):
        assert np.all(ids[perm[seg[s]:seg[s + 1]]] == idx[s])


def _documented_rule(T, n, H1, r, H2, max_seg_len, sms):
    """The rule of lora_sgmv_auto_variant, as its header comment states it."""
    L = min(max_seg_len, T) if max_seg_len > 0 else -(-T // n)
    if L >= 128 and r in (16, 32, 64) and H1 >= 64 and H2 >= 64:
        return sgmv.VARIANT_GROUPED_TC
    if n > 8192:
        return sgmv.VARIANT_SPLIT
    if L > 2 and r in (32, 64) and H1 % 64 == 0 and H2 % 64 == 0:
        jobs = n if L <= 16 else min(n + -(-T // 16), T)
        if jobs < sms and r * H2 * 2 >= 1e6:
            return sgmv.VARIANT_SPLIT_TC
        return sgmv.VARIANT_FUSED_TC
    return sgmv.VARIANT_FUSED


@settings(max_examples=500, deadline=None)
@given(st.integers(1, 20000), st.integers(1, 9000), st.sampled_from([64, 256, 264, 4096, 8192]),
       st.sampled_from([8, 16, 32, 64, 128]), st.sampled_from([64, 136, 4096, 8192, 16384, 28672]),
       st.integers(-1, 3000), st.sampled_from([100, 132, 148]), st.sampled_from([sgmv.F16, sgmv.BF16]))
def test_auto_variant_follows_its_documented_rule(T, n, H1, r, H2, max_seg_len, sms, dt):
    n = min(n, T)
    got = sgmv.lora_sgmv_auto_variant(T, n, H1, r, H2, dt, max_seg_len, sms)
    assert got == _documented_rule(T, n, H1, r, H2, max_seg_len, sms)


@settings(max_examples=300, deadline=None)
@given(st.lists(st.integers(0, 6), min_size=1, max_size=30), st.data())
def test_rows_share_is_the_clipped_segments(lens, data):
    import bench

    seg = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(seg[-1])
    idx = np.arange(len(lens), dtype=np.int32) * 3 + 1
    a = data.draw(st.integers(0, T))
    b = data.draw(st.integers(a, T))
    s, i = bench.rows_share(seg, idx, a, b)
    # brute force: the owner of every row in [a, b), in order, as runs
    owner = [k for k in range(len(lens)) for _ in range(lens[k])][a:b]
    runs = [(k, sum(1 for _ in g)) for k, g in __import__("itertools").groupby(owner)]
    assert i.tolist() == [int(idx[k]) for k, _ in runs]
    assert np.diff(s).tolist() == [c for _, c in runs] and s[0] == 0


@settings(max_examples=300, deadline=None)
@given(st.integers(0, 40000), st.integers(1, 16), st.sampled_from([1, 8, 64]))
def test_shard_range_partitions(n, world, align):
    from adapter_matmul_b200.tp import shard_range

    covered = []
    for p in range(world):
        lo, hi = shard_range(n, world, p, align)
        assert 0 <= lo <= hi <= n
        if hi > lo:
            assert lo % align == 0
        covered.extend(range(lo, hi))
    assert covered == list(range(n))
