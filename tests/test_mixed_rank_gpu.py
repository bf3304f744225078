"""Mixed ranks on the GPU: adapters of different ranks padded with zeros to one rank by
lora_sgmv_pad_rank, then one SGMV call over all of them (the authors' answer on different
ranks, page "Punica: Serving multiple LoRA finetuned LLM as one", the Hacker News thread).

The padding kernel must match numpy's zero padding bit for bit; the SGMV result must match
the oracle on the numpy-padded adapters within the parity tolerance, and so (by the oracle
pins on padding) each adapter's own product at its own rank.
"""
import numpy as np
import pytest

import oracle
from adapter_matmul_b200 import inputs, sgmv

pytestmark = pytest.mark.gpu


def _dev(bits):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).cuda()


def _host(t):
    return t.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("dt", [sgmv.F16, sgmv.BF16])
@pytest.mark.parametrize("H1,H2,rs,r", [(64, 48, 8, 16), (264, 136, 5, 64), (4096, 4096, 16, 64), (8, 1, 1, 1),
                                        (72, 40, 32, 32)])
def test_pad_rank_matches_numpy_zero_padding(dt, H1, H2, rs, r):
    import torch

    rng = np.random.default_rng(H1 * 7 + rs)
    A = rng.integers(0, 1 << 16, size=(H1, rs), dtype=np.uint16)
    B = rng.integers(0, 1 << 16, size=(rs, H2), dtype=np.uint16)
    dA, dB = _dev(A), _dev(B)
    # destinations start as garbage: every element must be written
    dAp = torch.full((H1, r), 0x5A5A, dtype=torch.int16, device="cuda")
    dBp = torch.full((r, H2), 0x5A5A, dtype=torch.int16, device="cuda")
    sgmv.lora_sgmv_pad_rank(dAp, dA, dBp, dB, H1, H2, rs, r, dt)
    torch.cuda.synchronize()
    assert np.array_equal(_host(dAp), np.pad(A, ((0, 0), (0, r - rs))))
    assert np.array_equal(_host(dBp), np.pad(B, ((0, r - rs), (0, 0))))
    # one pair only: B untouched
    dBq = torch.full((r, H2), 0x5A5A, dtype=torch.int16, device="cuda")
    dAq = torch.full((H1, r), 0x5A5A, dtype=torch.int16, device="cuda")
    sgmv.lora_sgmv_pad_rank(dAq, dA, None, None, H1, 0, rs, r, dt)
    torch.cuda.synchronize()
    assert np.array_equal(_host(dAq), np.pad(A, ((0, 0), (0, r - rs))))
    assert bool((dBq == 0x5A5A).all())


@pytest.mark.parametrize("dtn", ["f16", "bf16"])
@pytest.mark.parametrize("variant", [sgmv.VARIANT_AUTO, sgmv.VARIANT_SPLIT, sgmv.VARIANT_FUSED,
                                     sgmv.VARIANT_FUSED_TC, sgmv.VARIANT_SPLIT_TC, sgmv.VARIANT_GROUPED_TC])
def test_mixed_rank_sgmv_matches_oracle(dtn, variant):
    import torch

    dt = sgmv.F16 if dtn == "f16" else sgmv.BF16
    rng = np.random.default_rng(41)
    T, H1, H2, r = 200, 512, 384, 64
    ranks = [8, 16, 64, 32]
    X = inputs.cast_f32_bits(rng.standard_normal((T, H1)).astype(np.float32), dtn)
    Y = inputs.cast_f32_bits(rng.standard_normal((T, H2)).astype(np.float32), dtn)
    A = [inputs.cast_f32_bits(rng.standard_normal((H1, k)).astype(np.float32) * 0.05, dtn) for k in ranks]
    B = [inputs.cast_f32_bits(rng.standard_normal((k, H2)).astype(np.float32) * 0.05, dtn) for k in ranks]
    seg = np.array([0, 37, 90, 91, 160, 200], np.int32)
    idx = np.array([3, 0, 2, 1, 0], np.int32)

    dA = [torch.empty((H1, r), dtype=torch.int16, device="cuda") for _ in ranks]
    dB = [torch.empty((r, H2), dtype=torch.int16, device="cuda") for _ in ranks]
    src = [(_dev(a), _dev(b)) for a, b in zip(A, B)]
    for i, k in enumerate(ranks):
        sgmv.lora_sgmv_pad_rank(dA[i], src[i][0], dB[i], src[i][1], H1, H2, k, r, dt)
    A_ptrs, B_ptrs = sgmv.pointer_table(dA), sgmv.pointer_table(dB)
    dX, dY = _dev(X), _dev(Y)
    d_seg, d_idx = torch.from_numpy(seg).cuda(), torch.from_numpy(idx).cuda()
    ws_bytes = sgmv.lora_sgmv_workspace_bytes(T, r)
    ws = torch.empty(ws_bytes // 4, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sgmv.lora_sgmv_apply_ex(dY, dX, A_ptrs, B_ptrs, d_seg, d_idx, len(idx), len(ranks), T, H1, r, H2, 0.5, dt,
                            69, ws, ws_bytes, status, variant)
    torch.cuda.synchronize()
    assert int(status.item()) == 0

    Ap = [np.pad(a, ((0, 0), (0, r - a.shape[1]))) for a in A]
    Bp = [np.pad(b, ((0, r - b.shape[0]), (0, 0))) for b in B]
    ref, sk = oracle.apply_f32(Y, X, Ap, Bp, seg, idx, 0.5, dtn)
    assert sk == 0

    def f64(bits):
        if dtn == "f16":
            return np.ascontiguousarray(bits).view(np.float16).astype(np.float64)
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).view(torch.bfloat16).double().numpy()

    g, o = f64(_host(dY)), f64(ref)
    err = np.abs(g - o)
    assert np.all(err <= 2e-2 + 1e-2 * np.abs(o)), f"max abs err {err.max()}"


# ---- adapters of different ranks without padding: lora_sgmv_apply_ranks ---------------------

def _own_rank_reference(X, Y, A, B, seg, idx, scale, dt, ranks_ok):
    """The oracle segment by segment, each at its adapter's own rank (unpadded matrices)."""
    out = np.array(Y, copy=True)
    for s in range(len(idx)):
        b, e, i = int(seg[s]), int(seg[s + 1]), int(idx[s])
        if e <= b or not ranks_ok(i):
            continue
        res, _ = oracle.apply_f32(Y[b:e], X[b:e], [A[i]], [B[i]], [0, e - b], [0], scale, dt)
        out[b:e] = res
    return out


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("r_max,ranks", [(64, [8, 16, 24, 40, 64, 12, 72]), (32, [8, 16, 24, 32]), (16, [8, 16])])
def test_apply_ranks_unpadded_matches_each_adapters_own_product(dt, r_max, ranks):
    import torch

    H1, H2 = 320, 392
    lens = [130, 3, 200, 0, 64, 129, 1, 90]
    seg = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    nA = len(ranks)
    idx = np.array([k % nA for k in range(len(lens))], np.int32)[::-1].copy()
    T = int(seg[-1])
    base = inputs.small_random(T, nA, H1, H2, 8, dt, seed=r_max)
    X, Y = base.x(), base.y_random()
    A = [inputs.small_random(T, nA, H1, H2, rk, dt, seed=100 + k).adapter_a(k) for k, rk in enumerate(ranks)]
    B = [inputs.small_random(T, nA, H1, H2, rk, dt, seed=100 + k).adapter_b(k) for k, rk in enumerate(ranks)]
    dA = [_dev(a) for a in A]
    dB = [_dev(b) for b in B]
    A_ptrs = torch.tensor([t.data_ptr() for t in dA], dtype=torch.int64, device="cuda")
    B_ptrs = torch.tensor([t.data_ptr() for t in dB], dtype=torch.int64, device="cuda")
    d_ranks = torch.tensor(ranks, dtype=torch.int32, device="cuda")
    dX, dY = _dev(X), _dev(Y)
    d_seg = torch.from_numpy(seg).cuda()
    d_idx = torch.from_numpy(idx).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    code = sgmv.F16 if dt == "f16" else sgmv.BF16
    sgmv.lora_sgmv_apply_ranks(dY, dX, A_ptrs, B_ptrs, d_ranks, d_seg, d_idx, len(idx), nA, T, H1, r_max, H2, 0.8,
                               code, status)
    torch.cuda.synchronize()

    def ok(i):
        return 8 <= ranks[i] <= r_max and ranks[i] % 8 == 0

    ref = _own_rank_reference(X, Y, A, B, seg, idx, 0.8, dt, ok)
    got = _host(dY)
    st = int(status.item())
    used_bad = any(not ok(int(idx[s])) and seg[s + 1] > seg[s] for s in range(len(idx)))
    assert bool(st & sgmv.DEV_BAD_RANK) == used_bad and not (st & ~sgmv.DEV_BAD_RANK)
    from gpu_helpers import assert_close

    assert_close(got, ref, dt, f"ranks {ranks} at r_max {r_max}")
    for s in range(len(idx)):  # rows of skipped segments are untouched, bit for bit
        if not ok(int(idx[s])):
            assert np.array_equal(got[seg[s]:seg[s + 1]], Y[seg[s]:seg[s + 1]])
