"""The whole layer on the GPU, Y = X@W + scale * (X@A_i)@B_i (lora_sgmv_gemm_apply), against
the oracle's base_plus_delta_f32 (README page "Punica：多 LoRA 模型统一服务框架", LoRA and
multi-LoRA paragraphs), element by element.

Small cases cover both forms of the layer kernel (single SMs with 128 x 256 tiles below 256
rows, SM pairs with 256 x 256 tiles from 256 rows, on either side of that boundary), ragged
tiles (T, H1 and H2 not multiples of the tile or of the 64-wide K step, down to a pair whose
second SM holds no column of H2), tiles that span several segments, empty and rejected
segments, rows in no segment, both storage types, every rank the kernel takes, and both
shrink kernels that make V (segments shorter and longer than 128 rows). The prefill-sized layer (T = 9771, H1 = H2 =
4096, r = 64, bf16) is checked on whole rows: the first and last row of every segment and a
random sample, every column. Tolerance: |gpu - oracle| <= 2e-2 + 1e-2 |oracle|.
"""
import numpy as np
import pytest
import torch

import oracle
from adapter_matmul_b200 import inputs, sgmv
from gpu_helpers import assert_close, dt_code, from_dev, to_dev

pytestmark = pytest.mark.gpu


class Layer:
    def __init__(self, w, seg, idx, proj=0):
        self.w = w
        self.seg = np.asarray(seg, np.int32)
        self.idx = np.asarray(idx, np.int32)
        self.x_bits = w.x(proj)
        self.w_bits = w.base_weight(proj)
        self.A = [w.adapter_a(i, proj) for i in range(w.num_adapters)]
        self.B = [w.adapter_b(i, proj) for i in range(w.num_adapters)]
        self.dA = [to_dev(a, w.dtype) for a in self.A]
        self.dB = [to_dev(b, w.dtype) for b in self.B]
        self.A_ptrs = sgmv.pointer_table(self.dA)
        self.B_ptrs = sgmv.pointer_table(self.dB)
        self.X = to_dev(self.x_bits, w.dtype)
        self.W = to_dev(self.w_bits, w.dtype)
        self.Y = torch.full((w.T, w.H2), float("nan"), dtype=self.X.dtype, device="cuda")
        self.d_seg = torch.from_numpy(self.seg).cuda()
        self.d_idx = torch.from_numpy(self.idx).cuda() if len(self.idx) else torch.zeros(1, dtype=torch.int32,
                                                                                           device="cuda")
        self.ws_bytes = sgmv.lora_sgmv_workspace_bytes(w.T, w.r)
        self.ws = torch.empty(self.ws_bytes // 4 + 64, dtype=torch.float32, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run(self, scale, max_seg_len=0):
        w = self.w
        sgmv.lora_sgmv_gemm_apply(self.Y, self.X, self.W, self.A_ptrs, self.B_ptrs, self.d_seg, self.d_idx,
                                  len(self.idx), w.num_adapters, w.T, w.H1, w.r, w.H2, scale, dt_code(w.dtype),
                                  max_seg_len, self.ws, self.ws_bytes, self.status)
        torch.cuda.synchronize()
        return from_dev(self.Y)

    def oracle_rows(self, rows, scale):
        """The oracle on the given rows only (rows are independent): each row becomes its own
        segment with its owner's adapter, or no segment."""
        owner = np.full(self.w.T, -1)
        for s in range(len(self.idx)):
            b, e, i = int(self.seg[s]), int(self.seg[s + 1]), int(self.idx[s])
            if 0 <= b <= e <= self.w.T and 0 <= i < self.w.num_adapters:
                owner[b:e] = i
        sub_seg, sub_idx = [0], []
        # covered rows first (each its own segment), then the rest with no segment
        cov = [t for t in rows if owner[t] >= 0]
        unc = [t for t in rows if owner[t] < 0]
        perm = cov + unc
        for n, t in enumerate(cov):
            sub_seg.append(n + 1)
            sub_idx.append(int(owner[t]))
        Xp = self.x_bits[np.asarray(perm)]
        out, _ = oracle.base_plus_delta_f32(Xp, self.w_bits, self.A, self.B, sub_seg, sub_idx, scale, self.w.dtype)
        pos = {t: n for n, t in enumerate(perm)}
        return np.stack([out[pos[t]] for t in rows])


@pytest.mark.parametrize("r", [16, 32, 64])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_layer_ragged_short_segments(r, dtype):
    # segments of 0..40 rows (the split-K shrink makes V), unsorted adapters, a gap, one
    # rejected segment; T, H1, H2 ragged against the tile
    lens = [7, 0, 40, 1, 33, 3, 12]
    seg = np.concatenate([[2], 2 + np.cumsum(lens)]).astype(np.int32)
    idx = np.array([3, 1, 0, 2, 9, 1, 4], np.int32)  # adapter 9 does not exist
    T = int(seg[-1]) + 5
    w = inputs.small_random(T, 5, 200, 264, r, dtype, seed=100 + r)
    L = Layer(w, seg, idx)
    got = L.run(0.75)
    assert int(L.status.item()) & sgmv.DEV_BAD_ADAPTER
    ref, _ = oracle.base_plus_delta_f32(L.x_bits, L.w_bits, L.A, L.B, seg, idx, 0.75, dtype)
    assert_close(got, ref, dtype, f"layer r={r} {dtype}")


@pytest.mark.parametrize("r", [16, 64])
def test_layer_long_segments_grouped_shrink(r):
    # segments longer than 128 rows (the grouped kernel's shrink makes V); tiles span two and
    # three segments; H1 a multiple of 64, H2 not a multiple of 256
    lens = [5, 300, 129, 128, 60, 250]
    seg = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    idx = np.array([2, 0, 1, 3, 0, 2], np.int32)
    w = inputs.small_random(int(seg[-1]), 4, 512, 520, r, "bf16", seed=7)
    L = Layer(w, seg, idx)
    got = L.run(-1.25, max_seg_len=300)
    assert int(L.status.item()) == 0
    ref, _ = oracle.base_plus_delta_f32(L.x_bits, L.w_bits, L.A, L.B, seg, idx, -1.25, "bf16")
    assert_close(got, ref, "bf16", f"layer long segments r={r}")


@pytest.mark.parametrize("T", [255, 256, 257, 700])
@pytest.mark.parametrize("r", [16, 64])
def test_layer_short_segments_around_the_pair_boundary(T, r):
    # segments of 0..57 rows over the whole batch (split-K shrink), adapters reused out of
    # order; H2 = 264 leaves the second SM of the last column pair without a valid column
    rng = np.random.default_rng(T * 7 + r)
    lens, left = [], T - 3
    while left > 0:
        lens.append(int(min(left, rng.integers(0, 58))))
        left -= lens[-1]
    seg = np.concatenate([[3], 3 + np.cumsum(lens)]).astype(np.int32)
    idx = rng.integers(0, 5, len(lens)).astype(np.int32)
    w = inputs.small_random(T, 5, 136, 264, r, "f16", seed=T + r)
    L = Layer(w, seg, idx)
    got = L.run(0.5)
    assert int(L.status.item()) == 0
    ref, _ = oracle.base_plus_delta_f32(L.x_bits, L.w_bits, L.A, L.B, seg, idx, 0.5, "f16")
    assert_close(got, ref, "f16", f"layer T={T} r={r}")


def test_layer_without_segments_is_the_base_product():
    w = inputs.small_random(77, 2, 136, 264, 16, "f16", seed=3)
    L = Layer(w, [0], [])
    got = L.run(1.0)
    ref, _ = oracle.base_plus_delta_f32(L.x_bits, L.w_bits, L.A[:1], L.B[:1], [0], [], 1.0, "f16")
    assert_close(got, ref, "f16", "base only")


def test_layer_prefill_shape_whole_rows():
    w = inputs.make("prefill")
    seg, idx, _ = oracle.group_segments(w.ids, w.num_adapters)
    L = Layer(w, seg, idx)
    got = L.run(w.scale, max_seg_len=int(np.max(np.diff(seg))))
    assert int(L.status.item()) == 0
    rng = np.random.default_rng(0)
    rows = sorted(set(int(v) for v in np.concatenate([seg[:-1], seg[1:] - 1, rng.integers(0, w.T, 24)])))
    ref = L.oracle_rows(rows, w.scale)
    assert_close(got[rows], ref, "bf16", "prefill layer rows")
    assert np.all(np.isfinite(L.Y.float().cpu().numpy()))
