"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, element by element.

Tolerance (written here, from the method's stated bar for fp16/bf16 outputs):
|gpu - oracle| <= 2e-2 + 1e-2 * |oracle| per element. The oracle accumulates in
fp32 in ascending order; the kernels accumulate in fp32 in another order, so
results differ by rounding only. Bookkeeping and untouched rows are bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
from adapter_matmul_b200 import inputs, sgmv
from gpu_helpers import DeviceProblem, assert_close, decode, dt_code, from_dev, to_dev

pytestmark = pytest.mark.gpu

SMALL_CONFIGS = ["tiny", "distinct", "uniform_h4096", "uniform_h11008", "skewed_h4096", "skewed_h11008",
                 "identical_h4096", "identical_h11008"]


@pytest.mark.parametrize("name", SMALL_CONFIGS)
@pytest.mark.parametrize("y_random", [False, True])
@pytest.mark.parametrize("variant", [sgmv.VARIANT_AUTO, sgmv.VARIANT_SPLIT, sgmv.VARIANT_FUSED])
def test_config_full_oracle(name, y_random, variant):
    w = inputs.make(name)
    p = DeviceProblem(w, y_random=y_random)
    got = p.apply(variant=variant)
    ref = p.oracle_apply()
    assert_close(got, ref, w.dtype, name)
    assert int(p.status.item()) == 0


@pytest.mark.parametrize("name", ["distinct", "skewed_h11008"])
def test_config_bf16_variant(name):
    w = inputs.make(name)
    w.dtype = "bf16"
    p = DeviceProblem(w, y_random=True)
    assert_close(p.apply(), p.oracle_apply(), "bf16", name + "/bf16")


@pytest.mark.parametrize("r", [8, 16, 32, 64, 128])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("T", [1, 37, 130])
@pytest.mark.parametrize("variant", [sgmv.VARIANT_SPLIT, sgmv.VARIANT_FUSED, sgmv.VARIANT_FUSED_TC,
                                     sgmv.VARIANT_SPLIT_TC])
def test_ragged_random_shapes(r, dtype, T, variant):
    # H1, H2 not multiples of the tile sizes; segments of every length (several token chunks)
    if not sgmv.lora_sgmv_rank_supported(r, variant):
        pytest.skip("rank not built for this variant")
    # the tensor-core decode kernel takes multiples of 64, still ragged against its stage sizes
    tc = variant in (sgmv.VARIANT_FUSED_TC, sgmv.VARIANT_SPLIT_TC)
    H1, H2 = (320, 192) if tc else (264, 136)
    w = inputs.small_random(T, 7, H1, H2, r, dtype, seed=T * 1000 + r)
    p = DeviceProblem(w, y_random=True)
    assert_close(p.apply(variant=variant), p.oracle_apply(), dtype, w.name)


@pytest.mark.parametrize("r", [16, 64])
@pytest.mark.parametrize("variant", [sgmv.VARIANT_FUSED, sgmv.VARIANT_FUSED_TC, sgmv.VARIANT_SPLIT_TC])
def test_fused_long_rows_many_tiles(r, variant):
    # H1 and H2 span many stages per CTA (several A and B tiles) with ragged ends
    H1, H2 = (8200, 11000) if variant == sgmv.VARIANT_FUSED else (8256, 11008)
    w = inputs.small_random(40, 5, H1, H2, r, "bf16", seed=r)
    p = DeviceProblem(w, y_random=True)
    assert_close(p.apply(variant=variant), p.oracle_apply(), "bf16", "long rows")


@pytest.mark.parametrize("H1,H2", [(512, 768), (640, 1280), (896, 1792)])
def test_decode_tc_odd_cluster_sizes(H1, H2):
    # few jobs and K/N extents of 3, 5 and 7 stages: the cost model picks clusters of 3, 5 or 7
    # CTAs (non-power-of-two), each with its own K- and N-slice and a V exchange among them
    seg = np.array([0, 5, 8, 8, 11], np.int32)
    idx = np.array([1, 0, 2, 1], np.int32)
    w = inputs.small_random(11, 3, H1, H2, 64, "bf16", seed=H1)
    p = DeviceProblem(w, y_random=True, adapters=[0, 1, 2], seg_starts=seg, lora_idx=idx)
    got = p.apply(variant=sgmv.VARIANT_FUSED_TC)
    assert int(p.status.item()) == 0
    assert_close(got, p.oracle_apply(), "bf16", f"decode tc {H1}x{H2}")


def test_decode_tc_many_segments():
    # ~8000 segments: the job prefix takes most of the shared memory the cluster's V tiles
    # would use, so the host must fall back to smaller clusters
    rng = np.random.default_rng(7)
    lens = np.concatenate([np.ones(7990, np.int64), rng.integers(3, 20, size=10)])
    seg = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    idx = (np.arange(len(lens)) % 64).astype(np.int32)
    w = inputs.small_random(int(seg[-1]), 64, 128, 192, 64, "bf16", seed=11)
    p = DeviceProblem(w, y_random=True, adapters=list(range(64)), seg_starts=seg, lora_idx=idx)
    got = p.apply(variant=sgmv.VARIANT_FUSED_TC)
    assert int(p.status.item()) == 0
    assert_close(got, p.oracle_apply(), "bf16", "decode tc, 8000 segments")


def test_batched_projections_with_different_shapes():
    # q/k/v/o-like problems sharing one token grouping, in one launch
    ids = inputs.skewed(4096).ids
    shapes = [(4096, 4096), (4096, 1024), (4096, 1024), (2048, 4096)]
    probs, refs = [], []
    for k, (H1, H2) in enumerate(shapes):
        w = inputs.Workload(f"proj{k}", H1, H2, 16, "f16", ids, 64, 0.5 + 0.25 * k, seed=k)
        p = DeviceProblem(w, y_random=True)
        probs.append(p)
        refs.append(p.oracle_apply())
    p0 = probs[0]
    sgmv.lora_sgmv_apply_batched(
        [dict(Y=p.Y, X=p.X, A_ptrs=p.A_ptrs, B_ptrs=p.B_ptrs, num_adapters=p.w.num_adapters, H1=p.w.H1,
              H2=p.w.H2, scale=p.w.scale) for p in probs],
        p0.d_seg, p0.d_idx, p0.n, p0.w.T, 16, sgmv.F16, p0.max_len(), p0.status)
    torch.cuda.synchronize()
    for p, ref in zip(probs, refs):
        assert_close(from_dev(p.Y), ref, "f16", p.w.name)
    assert int(p0.status.item()) == 0


@pytest.mark.parametrize("r,dtype", [(64, "bf16"), (32, "f16")])
def test_batched_projections_tensor_core_decode(r, dtype):
    # four problems with different shapes through the tensor-core decode kernel (segments of
    # several tokens, r >= 32): one launch, per-problem tensor maps and device-built adapter maps
    ids = inputs.llama70b_decode(8192).ids[:96]
    shapes = [(1024, 1024), (1024, 256), (512, 2048), (2048, 640)]
    probs, refs = [], []
    for k, (H1, H2) in enumerate(shapes):
        w = inputs.Workload(f"tcproj{k}", H1, H2, r, dtype, ids, 1024, 1.0 - 0.25 * k, seed=10 + k)
        p = DeviceProblem(w, y_random=True)
        probs.append(p)
        refs.append(p.oracle_apply())
    p0 = probs[0]
    assert p0.max_len() > 2
    sgmv.lora_sgmv_apply_batched(
        [dict(Y=p.Y, X=p.X, A_ptrs=p.A_ptrs, B_ptrs=p.B_ptrs, num_adapters=p.w.num_adapters, H1=p.w.H1,
              H2=p.w.H2, scale=p.w.scale) for p in probs],
        p0.d_seg, p0.d_idx, p0.n, p0.w.T, r, dt_code(dtype), p0.max_len(), p0.status)
    torch.cuda.synchronize()
    for p, ref in zip(probs, refs):
        assert_close(from_dev(p.Y), ref, dtype, p.w.name)
    assert int(p0.status.item()) == 0


# ---- shrink and expand entry points on their own ----------------------------------------------

@pytest.mark.parametrize("name", ["skewed_h4096", "tiny"])
def test_shrink_and_expand_entry_points(name):
    w = inputs.make(name)
    p = DeviceProblem(w, y_random=True)
    A = [p.A.get(i, np.zeros((w.H1, w.r), np.uint16)) for i in range(w.num_adapters)]
    B = [p.B.get(i, np.zeros((w.r, w.H2), np.uint16)) for i in range(w.num_adapters)]
    V = torch.full((w.T, w.r), float("nan"), dtype=torch.float32, device="cuda")
    sgmv.lora_sgmv_shrink(V, p.X, p.A_ptrs, p.d_seg, p.d_idx, p.n, w.num_adapters, w.T, w.H1, w.r,
                          dt_code(w.dtype), p.status)
    torch.cuda.synchronize()
    Vo, _ = oracle.shrink_f32(p.x_bits, A, p.seg, p.idx, w.r, w.dtype)
    np.testing.assert_allclose(V.cpu().numpy(), Vo, rtol=1e-4, atol=1e-4)
    # expand from the oracle's V (uploaded): isolates the expand kernel
    Vd = torch.from_numpy(Vo).cuda()
    sgmv.lora_sgmv_expand(p.Y, Vd, p.B_ptrs, p.d_seg, p.d_idx, p.n, w.num_adapters, w.T, w.r, w.H2, 0.5,
                          dt_code(w.dtype), p.status)
    torch.cuda.synchronize()
    ref, _ = oracle.expand_f32(p.y_bits, Vo, B, p.seg, p.idx, 0.5, w.dtype)
    assert_close(from_dev(p.Y), ref, w.dtype, name + " expand")
    assert int(p.status.item()) == 0


# ---- segment semantics and edge cases --------------------------------------------------------

def _custom(seg, idx, T=24, H1=512, H2=264, r=16, dtype="f16", na=5, seed=3):
    w = inputs.small_random(T, na, H1, H2, r, dtype, seed=seed)
    return DeviceProblem(w, y_random=True, adapters=list(range(na)), seg_starts=seg, lora_idx=idx)


def test_no_segments_is_noop():
    p = _custom([0], [])
    before = from_dev(p.Y)
    got = p.apply()
    assert np.array_equal(got, before)


def test_empty_repeated_unsorted_segments_and_uncovered_rows():
    # rows 0..1 and 22..23 uncovered; empty segments; adapter 3 twice; unsorted ids
    seg = [2, 2, 7, 7, 15, 16, 22]
    idx = [4, 3, 0, 3, 1, 2]
    p = _custom(seg, idx)
    before = from_dev(p.Y)
    got = p.apply()
    ref = p.oracle_apply()
    assert_close(got, ref, "f16", "custom segments")
    for t in (0, 1, 22, 23):
        assert np.array_equal(got[t], before[t])
    assert int(p.status.item()) == 0


@pytest.mark.parametrize("variant", [sgmv.VARIANT_SPLIT, sgmv.VARIANT_FUSED, sgmv.VARIANT_FUSED_TC,
                                     sgmv.VARIANT_SPLIT_TC])
@pytest.mark.parametrize("hint", [4, 40])
def test_bad_segments_are_skipped_and_reported(variant, hint):
    # [4,2) reversed; adapter 9 out of range; adapter 2 has a null table entry; [20,30) past T.
    # The length hint 4 makes the fused kernels take one entry per segment, 40 the chunk list.
    seg = np.array([0, 4, 2, 8, 12, 16, 20, 30], np.int32)
    idx = np.array([0, 1, 9, 3, 2, 4, 1], np.int32)
    tc = variant in (sgmv.VARIANT_FUSED_TC, sgmv.VARIANT_SPLIT_TC)
    p = _custom(seg, idx, H2=256 if tc else 264)
    p.A_ptrs[2] = 0
    before = from_dev(p.Y)
    got = p.apply(variant=variant, max_seg_len=hint)
    st = int(p.status.item())
    assert st & sgmv.DEV_BAD_SEGMENT and st & sgmv.DEV_BAD_ADAPTER and st & sgmv.DEV_BAD_POINTER
    # valid segments: [0,4) adapter 0, [8,12) adapter 3, [16,20) adapter 4
    ref = DeviceProblem(p.w, y_random=True, adapters=list(range(5)), seg_starts=[0, 4, 8, 12, 16, 20],
                        lora_idx=[0, 0, 3, 3, 4]).oracle_apply()
    for t in list(range(0, 4)) + list(range(8, 12)) + list(range(16, 20)):
        assert_close(got[t:t + 1], ref[t:t + 1], "f16", f"row {t}")
    for t in list(range(4, 8)) + list(range(12, 16)) + list(range(20, 24)):
        assert np.array_equal(got[t], before[t]), t


@pytest.mark.parametrize("scale", [0.0, -0.75, 2.0])
def test_scale(scale):
    p = _custom([0, 10, 24], [1, 3])
    before = from_dev(p.Y)
    got = p.apply(scale=scale)
    assert_close(got, p.oracle_apply(scale=scale), "f16", f"scale {scale}")
    if scale == 0.0:
        assert np.array_equal(got, before)


def test_deterministic_bits():
    w = inputs.make("skewed_h11008")
    p1 = DeviceProblem(w, y_random=True)
    p2 = DeviceProblem(w, y_random=True)
    assert np.array_equal(p1.apply(), p2.apply())


def test_wrong_length_hint_still_correct():
    w = inputs.make("skewed_h4096")
    for hint in (1, 1000, 0):
        p = DeviceProblem(w, y_random=True)
        assert_close(p.apply(max_seg_len=hint), p.oracle_apply(), w.dtype, f"hint {hint}")


def test_large_h1_and_many_segments():
    # H1 = 16384 (largest shrink slice), 300 segments of mixed length
    rng = np.random.default_rng(4)
    lens = rng.integers(0, 5, 300)
    seg = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(seg[-1])
    idx = rng.integers(0, 6, 300).astype(np.int32)
    w = inputs.small_random(T, 6, 16384, 520, 32, "bf16", seed=8)
    p = DeviceProblem(w, y_random=True, adapters=list(range(6)), seg_starts=seg, lora_idx=idx)
    assert_close(p.apply(), p.oracle_apply(), "bf16", "H1=16384")


# ---- grouped tensor-core kernel (prefill) ---------------------------------------------------

@pytest.mark.parametrize("r", [16, 32, 64])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("H1,H2", [(328, 392), (320, 448)])
def test_grouped_tc_ragged_tiles(r, dtype, H1, H2):
    # segments shorter than, equal to and longer than the 128-row tile; an empty segment; Y
    # non-zero. (328, 392): H1 not a multiple of the 64-wide K step, H2 not a multiple of the
    # 128-wide N tile (row-major 2-D copies). (320, 448): odd numbers of 64-column blocks, so the
    # last stage's 3-D copies of two blocks reach one block past H1 and past H2
    lens = [5, 128, 300, 0, 1, 129]
    seg = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    idx = np.array([2, 0, 1, 3, 2, 4], np.int32)
    w = inputs.small_random(int(seg[-1]), 5, H1, H2, r, dtype, seed=r)
    p = DeviceProblem(w, y_random=True, adapters=list(range(5)), seg_starts=seg, lora_idx=idx)
    got = p.apply(variant=sgmv.VARIANT_GROUPED_TC)
    assert int(p.status.item()) == 0
    assert_close(got, p.oracle_apply(), dtype, f"grouped r={r}")


def test_grouped_tc_bad_segments_skipped():
    seg = np.array([0, 200, 150, 400, 450], np.int32)  # [200,150) reversed
    idx = np.array([0, 1, 7, 2], np.int32)             # adapter 7 out of range
    w = inputs.small_random(450, 4, 256, 256, 64, "bf16", seed=5)
    p = DeviceProblem(w, y_random=True, adapters=list(range(4)), seg_starts=seg, lora_idx=idx)
    before = from_dev(p.Y)
    got = p.apply(variant=sgmv.VARIANT_GROUPED_TC)
    st = int(p.status.item())
    assert st & sgmv.DEV_BAD_SEGMENT and st & sgmv.DEV_BAD_ADAPTER
    ref = DeviceProblem(w, y_random=True, adapters=list(range(4)), seg_starts=[0, 200, 400, 450],
                        lora_idx=[0, 0, 2]).oracle_apply()
    # valid: [0,200) on adapter 0 and [400,450) on adapter 2; rows 200..399 only in rejected segments
    assert_close(got[:200], ref[:200], "bf16", "valid segment 0")
    assert_close(got[400:], ref[400:], "bf16", "valid segment 3")
    assert np.array_equal(got[200:400], before[200:400])


@pytest.mark.parametrize("variant", [sgmv.VARIANT_AUTO, sgmv.VARIANT_SPLIT])
def test_more_segments_than_the_flat_chunk_list(variant):
    # 9000 segments of 0..3 tokens: more than the shrink's flat chunk list holds (8192 segments),
    # so its clusters walk segment and chunk slots instead; AUTO takes the split kernels here
    rng = np.random.default_rng(12)
    lens = rng.integers(0, 4, 9000)
    seg = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    idx = rng.integers(0, 5, 9000).astype(np.int32)
    w = inputs.small_random(int(seg[-1]), 5, 256, 136, 16, "f16", seed=12)
    p = DeviceProblem(w, y_random=True, adapters=list(range(5)), seg_starts=seg, lora_idx=idx)
    got = p.apply(variant=variant)
    assert int(p.status.item()) == 0
    assert_close(got, p.oracle_apply(), "f16", f"9000 segments, variant {variant}")
