"""Pins for the CPU oracle: each test checks it against something other than itself.

What the pages fix (page “Punica：多 LoRA 模型统一服务框架”, the Punica README: LoRA paragraph and multi-LoRA paragraph):
the shapes A [H1, r], B [r, H2]; the identity x@(W + A@B) = x@W + x@A@B; the
batched definition in which each row uses its own adapter. The pins below are:
library conversions (numpy float16, torch bfloat16), a hand-worked example,
exact rational arithmetic, one-hot closed forms, a dense numpy GEMM for the
Identical distribution, and invariants of the segment semantics. Each is chosen
so that a plausible slip in the oracle (a transposed operand, a wrong index, a
dropped term, a sign) fails at least one of them.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from adapter_matmul_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f16_bits(vals):
    return np.asarray(vals, dtype=np.float64).astype(np.float16).view(np.uint16)


def dec(bits, dt):
    """Independent decode through numpy / torch (not the oracle)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dt == "f16":
        return bits.view(np.float16).astype(np.float64)
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()


# ---------------------------------------------------------------------------------------------
# storage conversions
# ---------------------------------------------------------------------------------------------

def test_f16_decode_all_patterns_match_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode(bits, "f16")
    ref = bits.view(np.float16).astype(np.float64)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    m = ~np.isnan(ref)
    assert np.array_equal(got[m], ref[m])
    assert np.array_equal(np.signbit(got[m]), np.signbit(ref[m]))


def test_bf16_decode_all_patterns_match_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode(bits, "bf16")
    ref = dec(bits, "bf16")
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    m = ~np.isnan(ref)
    assert np.array_equal(got[m], ref[m])
    assert np.array_equal(np.signbit(got[m]), np.signbit(ref[m]))


def _wide_doubles(n, seed):
    rng = np.random.default_rng(seed)
    mant = rng.random(n) * 2 - 1
    expo = rng.integers(-30, 20, n)
    v = np.ldexp(mant, expo)
    extra = [0.0, -0.0, 65504.0, 65519.99, 65520.0, -65520.0, 1e9, 2.0 ** -24, 2.0 ** -25,
             3 * 2.0 ** -26, 2.0 ** -14, 2.0 ** -14 * (1 - 2 ** -11), np.inf, -np.inf]
    return np.concatenate([v, np.array(extra)])


def test_f16_encode_matches_numpy_rne():
    v = _wide_doubles(200000, 1)
    got = oracle.encode(v, "f16")
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)  # numpy rounds binary64 -> binary16 to nearest even
    assert np.array_equal(got, ref)


def test_f16_encode_exact_ties_go_to_even():
    # 1 + k*2^-10 + 2^-11 is exactly halfway between two fp16 neighbours
    k = np.arange(0, 1024)
    v = 1.0 + k * 2.0 ** -10 + 2.0 ** -11
    got = oracle.decode(oracle.encode(v, "f16"), "f16")
    even = np.where(k % 2 == 0, 1.0 + k * 2.0 ** -10, 1.0 + (k + 1) * 2.0 ** -10)
    assert np.array_equal(got, even)


def test_bf16_encode_matches_torch_rne_on_fp32_values():
    v32 = _wide_doubles(200000, 2).astype(np.float32)
    v32 = np.concatenate([v32, np.array([3.3895314e38, -3.3895314e38, 1e-40, -1e-41], dtype=np.float32)])
    got = oracle.encode(v32.astype(np.float64), "bf16")
    ref = torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_encode_exact_ties_go_to_even():
    k = np.arange(0, 128)
    v = 1.0 + k * 2.0 ** -7 + 2.0 ** -8
    got = oracle.decode(oracle.encode(v, "bf16"), "bf16")
    even = np.where(k % 2 == 0, 1.0 + k * 2.0 ** -7, 1.0 + (k + 1) * 2.0 ** -7)
    assert np.array_equal(got, even)


# ---------------------------------------------------------------------------------------------
# the maths of the README
# ---------------------------------------------------------------------------------------------

def test_hand_worked_example_golden():
    g = json.load(open(os.path.join(GOLDEN, "lora_worked_example.json")))
    X = f16_bits(g["X"])
    A = [f16_bits(a) for a in g["A"]]
    B = [f16_bits(b) for b in g["B"]]
    W = np.array(g["W"])
    xw = dec(X, "f16") @ W
    # fp32 twin: V exactly as derived by hand, Y = x@W + delta
    V, sk = oracle.shrink_f32(X, A, g["seg_starts"], g["lora_idx"], g["r"], "f16")
    assert sk == 0
    assert np.array_equal(V, np.array(g["V"], dtype=np.float32))
    Y, _ = oracle.expand_f32(f16_bits(xw), V, B, g["seg_starts"], g["lora_idx"], 1.0, "f16")
    assert np.array_equal(dec(Y, "f16"), np.array(g["Y"]))
    Yd, _ = oracle.apply_f32(np.zeros((3, 2), np.uint16), X, A, B, g["seg_starts"], g["lora_idx"], 1.0, "f16")
    assert np.array_equal(dec(Yd, "f16"), np.array(g["delta"]))
    # binary64 twin
    Y64, _ = oracle.apply_f64(xw, X, A, B, g["seg_starts"], g["lora_idx"], 1.0, "f16")
    assert np.array_equal(Y64, np.array(g["Y"]))


def bf16_bits(vals):
    """Exact bfloat16 bits of values that bfloat16 holds (torch's conversion, not the oracle's)."""
    t = torch.tensor(np.asarray(vals, dtype=np.float64)).to(torch.bfloat16)
    assert torch.equal(t.to(torch.float64), torch.tensor(np.asarray(vals, dtype=np.float64)))
    return t.view(torch.int16).numpy().view(np.uint16)


def test_hand_worked_bf16_example_with_scale_and_ties_golden():
    g = json.load(open(os.path.join(GOLDEN, "lora_worked_example_bf16_ties.json")))
    X, Y0 = bf16_bits(g["X"]), bf16_bits(g["Y_base"])
    A = [bf16_bits(a) for a in g["A"]]
    B = [bf16_bits(b) for b in g["B"]]
    seg, idx, scale = g["seg_starts"], g["lora_idx"], g["scale"]
    V, sk = oracle.shrink_f32(X, A, seg, idx, g["r"], "bf16")
    assert sk == 0
    assert np.array_equal(V, np.array(g["V"], dtype=np.float32))
    Y, _ = oracle.apply_f32(Y0, X, A, B, seg, idx, scale, "bf16")
    assert np.array_equal(dec(Y, "bf16"), np.array(g["Y"]))  # the two ties went to the even neighbour
    Y64, _ = oracle.apply_f64(dec(Y0, "bf16"), X, A, B, seg, idx, scale, "bf16")
    assert np.array_equal(Y64, np.array(g["Y_unrounded"]))


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_identity_against_materialised_weight(dt):
    """x@(W + A@B) == x@W + (x@A)@B, with W + A@B materialised in fp64 by numpy."""
    rng = np.random.default_rng(7)
    T, H1, H2, r = 8, 24, 16, 4
    X = inputs.cast_f32_bits(rng.standard_normal((T, H1)).astype(np.float32), dt)
    A = [inputs.cast_f32_bits(rng.standard_normal((H1, r)).astype(np.float32) * 0.3, dt) for _ in range(3)]
    B = [inputs.cast_f32_bits(rng.standard_normal((r, H2)).astype(np.float32) * 0.5, dt) for _ in range(3)]
    W = rng.standard_normal((H1, H2))
    seg, idx = [0, 3, 5, 8], [2, 0, 1]
    x = dec(X, dt)
    ref = np.zeros((T, H2))
    for s in range(3):
        Wp = W + dec(A[idx[s]], dt) @ dec(B[idx[s]], dt)
        ref[seg[s]:seg[s + 1]] = x[seg[s]:seg[s + 1]] @ Wp
    got, sk = oracle.apply_f64(x @ W, X, A, B, seg, idx, 1.0, dt)
    assert sk == 0
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_one_hot_rows_pick_adapter_rows_and_columns(dt):
    """X[t] = e_k selects row k of A_i; V = e_j selects row j of B_i. Exact."""
    rng = np.random.default_rng(11)
    T, H1, H2, r, nA = 6, 20, 12, 5, 3
    A = [inputs.cast_f32_bits(rng.standard_normal((H1, r)).astype(np.float32), dt) for _ in range(nA)]
    B = [inputs.cast_f32_bits(rng.standard_normal((r, H2)).astype(np.float32), dt) for _ in range(nA)]
    seg, idx = [0, 2, 3, 6], [1, 2, 0]
    ks = [3, 17, 0, 19, 8, 11]
    js = [4, 0, 2, 1, 3, 4]
    one = inputs.cast_f32_bits(np.ones(1, np.float32), dt)[0]
    X = np.zeros((T, H1), np.uint16)
    for t, k in enumerate(ks):
        X[t, k] = one
    V, _ = oracle.shrink_f32(X, A, seg, idx, r, dt)
    V64, _ = oracle.shrink_f64(X, A, seg, idx, r, dt)
    Vs = np.zeros((T, r), np.float32)
    Y0 = np.zeros((T, H2), np.uint16)
    for s in range(3):
        for t in range(seg[s], seg[s + 1]):
            assert np.array_equal(V[t], dec(A[idx[s]][ks[t]], dt).astype(np.float32))
            assert np.array_equal(V64[t], dec(A[idx[s]][ks[t]], dt))
            Vs[t, js[t]] = 1.0
    Y, _ = oracle.expand_f32(Y0, Vs, B, seg, idx, 1.0, dt)
    for s in range(3):
        for t in range(seg[s], seg[s + 1]):
            assert np.array_equal(Y[t], B[idx[s]][js[t]])


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_identical_distribution_equals_dense_gemm(dt):
    """All tokens on one adapter: SGMV == dense (X@A)@B by numpy in fp64."""
    rng = np.random.default_rng(3)
    T, H1, H2, r = 16, 64, 48, 8
    X = inputs.cast_f32_bits(rng.standard_normal((T, H1)).astype(np.float32), dt)
    A = [inputs.cast_f32_bits((rng.standard_normal((H1, r)) / 8).astype(np.float32), dt)]
    B = [inputs.cast_f32_bits((rng.standard_normal((r, H2)) / 3).astype(np.float32), dt)]
    dense = (dec(X, dt) @ dec(A[0], dt)) @ dec(B[0], dt)
    got64, _ = oracle.apply_f64(np.zeros((T, H2)), X, A, B, [0, T], [0], 1.0, dt)
    np.testing.assert_allclose(got64, dense, rtol=1e-12, atol=1e-12)
    # fp32 twin: within one storage ulp plus the fp32 accumulation bound
    got32, _ = oracle.apply_f32(np.zeros((T, H2), np.uint16), X, A, B, [0, T], [0], 1.0, dt)
    ulp = 2.0 ** -10 if dt == "f16" else 2.0 ** -7
    err = np.abs(dec(got32, dt) - dense)
    assert np.all(err <= ulp * np.abs(dense) + 1e-5)
    # Distinct with every adapter equal gives the same fp32 result, row for row
    Ad = A * T
    Bd = B * T
    gotd, _ = oracle.apply_f32(np.zeros((T, H2), np.uint16), X, Ad, Bd, list(range(T + 1)), list(range(T)), 1.0, dt)
    assert np.array_equal(gotd, got32)


def test_brute_force_exact_rationals():
    """Tiny problem in exact rational arithmetic (Fraction) vs both twins."""
    rng = np.random.default_rng(5)
    T, H1, H2, r = 3, 5, 4, 2
    dt = "f16"
    X = f16_bits(rng.standard_normal((T, H1)))
    A = [f16_bits(rng.standard_normal((H1, r))), f16_bits(rng.standard_normal((H1, r)))]
    B = [f16_bits(rng.standard_normal((r, H2))), f16_bits(rng.standard_normal((r, H2)))]
    Y0 = f16_bits(rng.standard_normal((T, H2)))
    seg, idx = [0, 1, 3], [1, 0]
    F = lambda bits: [[Fraction(float(v)) for v in row] for row in dec(np.atleast_2d(bits), dt)]
    x, y0 = F(X), F(Y0)
    exact = [[None] * H2 for _ in range(T)]
    for s in range(2):
        a, b = F(A[idx[s]]), F(B[idx[s]])
        for t in range(seg[s], seg[s + 1]):
            v = [sum(x[t][k] * a[k][j] for k in range(H1)) for j in range(r)]
            for c in range(H2):
                exact[t][c] = y0[t][c] + sum(v[j] * b[j][c] for j in range(r))
    ex = np.array([[float(v) for v in row] for row in exact])
    got64, _ = oracle.apply_f64(dec(Y0, dt), X, A, B, seg, idx, 1.0, dt)
    np.testing.assert_allclose(got64, ex, rtol=1e-14, atol=1e-14)
    got32, _ = oracle.apply_f32(Y0, X, A, B, seg, idx, 1.0, dt)
    # fp32 accumulation then one fp16 rounding: within one fp16 ulp of the exact value
    assert np.all(np.abs(dec(got32, dt) - ex) <= 2.0 ** -10 * np.maximum(np.abs(ex), 2.0 ** -14) * 1.01)


# ---------------------------------------------------------------------------------------------
# segment semantics
# ---------------------------------------------------------------------------------------------

def _case(dt="f16", T=12, H1=32, H2=24, r=4, nA=4, seed=9):
    rng = np.random.default_rng(seed)
    X = inputs.cast_f32_bits(rng.standard_normal((T, H1)).astype(np.float32), dt)
    A = [inputs.cast_f32_bits((rng.standard_normal((H1, r)) / 5).astype(np.float32), dt) for _ in range(nA)]
    B = [inputs.cast_f32_bits((rng.standard_normal((r, H2)) / 2).astype(np.float32), dt) for _ in range(nA)]
    Y = inputs.cast_f32_bits(rng.standard_normal((T, H2)).astype(np.float32) + 0.01, dt)
    return X, A, B, Y


def test_zero_length_segments_are_noops():
    X, A, B, Y = _case()
    base, _ = oracle.apply_f32(Y, X, A, B, [0, 5, 12], [1, 3], 1.0, "f16")
    with_empty, sk = oracle.apply_f32(Y, X, A, B, [0, 0, 5, 5, 5, 12, 12], [2, 1, 0, 3, 3, 1], 1.0, "f16")
    assert sk == 0
    assert np.array_equal(base, with_empty)


def test_splitting_a_segment_is_bit_identical():
    X, A, B, Y = _case()
    one, _ = oracle.apply_f32(Y, X, A, B, [0, 12], [2], 1.0, "f16")
    split, _ = oracle.apply_f32(Y, X, A, B, [0, 4, 9, 12], [2, 2, 2], 1.0, "f16")
    assert np.array_equal(one, split)


def test_permuting_segments_permutes_rows():
    X, A, B, Y = _case()
    seg, idx = [0, 3, 7, 12], [0, 3, 1]
    out, _ = oracle.apply_f32(Y, X, A, B, seg, idx, 1.0, "f16")
    order = [2, 0, 1]
    rows = np.concatenate([np.arange(seg[s], seg[s + 1]) for s in order])
    lens = [seg[s + 1] - seg[s] for s in order]
    seg2 = np.concatenate([[0], np.cumsum(lens)])
    out2, _ = oracle.apply_f32(Y[rows], X[rows], A, B, seg2, [idx[s] for s in order], 1.0, "f16")
    assert np.array_equal(out2, out[rows])


def test_rows_outside_segments_and_bad_segments_untouched():
    X, A, B, Y = _case()
    # rows 0..1 and 10..11 in no segment; one segment with a bad adapter id; one reversed
    seg = [2, 5, 7, 6, 10]
    idx = [1, 9, 0, 2]
    out, sk = oracle.apply_f32(Y, X, A, B, seg, idx, 1.0, "f16")
    assert sk == 2
    # valid: [2,5) on adapter 1 and [6,10) on adapter 2
    for t in [0, 1, 5, 10, 11]:
        assert np.array_equal(out[t], Y[t])
    ref, _ = oracle.apply_f32(Y, X, A, B, [2, 5, 6, 10], [1, 0, 2], 1.0, "f16")
    for t in [2, 3, 4, 6, 7, 8, 9]:
        assert np.array_equal(out[t], ref[t])


def test_scale_linearity_powers_of_two_and_zero():
    X, A, B, Y = _case()
    Z = np.zeros_like(Y)
    seg, idx = [0, 6, 12], [3, 1]
    d1, _ = oracle.apply_f32(Z, X, A, B, seg, idx, 1.0, "f16")
    for k in (-2, 1, 3):
        dk, _ = oracle.apply_f32(Z, X, A, B, seg, idx, 2.0 ** k, "f16")
        a1, ak = dec(d1, "f16"), dec(dk, "f16")
        normal = np.abs(a1) * 2.0 ** k >= 2.0 ** -14
        assert np.array_equal(ak[normal], a1[normal] * 2.0 ** k)
    same, _ = oracle.apply_f32(Y, X, A, B, seg, idx, 0.0, "f16")
    assert np.array_equal(same, Y)


# ---------------------------------------------------------------------------------------------
# bookkeeping
# ---------------------------------------------------------------------------------------------

def test_group_segments_tiny_config_printed_segments():
    w = inputs.tiny()
    seg, idx, perm = oracle.group_segments(w.ids, w.num_adapters)
    assert seg.tolist() == [0, 1, 4, 6, 8]
    assert idx.tolist() == [0, 1, 2, 3]
    assert perm.tolist() == list(range(8))


@pytest.mark.parametrize("maker", [lambda: inputs.uniform(), lambda: inputs.skewed(),
                                   lambda: inputs.identical(), lambda: inputs.llama70b_decode()])
def test_group_segments_invariants_and_stable_argsort(maker):
    w = maker()
    seg, idx, perm = oracle.group_segments(w.ids, w.num_adapters)
    T = w.T
    assert seg[0] == 0 and seg[-1] == T
    assert np.all(np.diff(seg) > 0)
    assert np.all(np.diff(idx) > 0)
    assert np.array_equal(np.sort(perm), np.arange(T))
    for s in range(len(idx)):
        part = perm[seg[s]:seg[s + 1]]
        assert np.all(w.ids[part] == idx[s])
        assert np.all(np.diff(part) > 0)
    # independent library routine: a stable argsort by adapter id
    assert np.array_equal(perm, np.argsort(w.ids, kind="stable"))
    assert idx.tolist() == sorted(set(w.ids.tolist()))


def test_group_segments_rejects_out_of_range_ids():
    with pytest.raises(ValueError):
        oracle.group_segments([0, 5, 1], 4)


# ---------------------------------------------------------------------------------------------
# mixed ranks by zero padding (the authors' answer on different ranks, page "Punica: Serving
# multiple LoRA finetuned LLM as one", the Hacker News thread)
# ---------------------------------------------------------------------------------------------

def _mixed_rank_case(dt, seed):
    rng = np.random.default_rng(seed)
    T, H1, H2, r = 14, 24, 16, 8
    ranks = [2, 8, 5, 3]  # adapter i has rank ranks[i]; all are padded to r
    X = inputs.cast_f32_bits(rng.standard_normal((T, H1)).astype(np.float32), dt)
    Y = inputs.cast_f32_bits(rng.standard_normal((T, H2)).astype(np.float32), dt)
    A = [inputs.cast_f32_bits(rng.standard_normal((H1, k)).astype(np.float32) * 0.3, dt) for k in ranks]
    B = [inputs.cast_f32_bits(rng.standard_normal((k, H2)).astype(np.float32) * 0.5, dt) for k in ranks]
    Ap = [np.pad(a, ((0, 0), (0, r - a.shape[1]))) for a in A]  # zero columns
    Bp = [np.pad(b, ((0, r - b.shape[0]), (0, 0))) for b in B]  # zero rows
    seg, idx = [0, 3, 4, 9, 14], [2, 0, 3, 1]
    return X, Y, A, B, Ap, Bp, seg, idx


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_mixed_ranks_padded_equal_each_adapters_own_product(dt):
    """Padded to one rank, every segment still gets x@A_i@B_i at adapter i's own rank
    (numpy, fp64, with the unpadded matrices)."""
    X, Y, A, B, Ap, Bp, seg, idx = _mixed_rank_case(dt, 23)
    x, y = dec(X, dt), dec(Y, dt)
    ref = y.copy()
    for s in range(len(idx)):
        i = idx[s]
        ref[seg[s]:seg[s + 1]] += 0.75 * (x[seg[s]:seg[s + 1]] @ dec(A[i], dt)) @ dec(B[i], dt)
    got, sk = oracle.apply_f64(y, X, Ap, Bp, seg, idx, 0.75, dt)
    assert sk == 0
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_zero_padding_leaves_fp32_results_bit_identical(dt):
    """The fp32 oracle on padded adapters equals, bit for bit, one call per segment on the
    adapter at its own rank: the extra terms are exact zeros."""
    X, Y, A, B, Ap, Bp, seg, idx = _mixed_rank_case(dt, 29)
    got, sk = oracle.apply_f32(Y, X, Ap, Bp, seg, idx, 1.25, dt)
    assert sk == 0
    for s in range(len(idx)):
        b, e, i = seg[s], seg[s + 1], idx[s]
        own, sk1 = oracle.apply_f32(Y[b:e], X[b:e], [A[i]], [B[i]], [0, e - b], [0], 1.25, dt)
        assert sk1 == 0
        assert np.array_equal(got[b:e], own), s


# ---------------------------------------------------------------------------------------------
# algebraic invariants of the definition on random shapes (binary64 twin; small integer-valued
# operands are exact in fp16, so sums of them are exact too)
# ---------------------------------------------------------------------------------------------

from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


def _int_case(rng, T, H1, r, H2, nA, lo=-3, hi=4):
    X = f16_bits(rng.integers(lo, hi, (T, H1)))
    A = [f16_bits(rng.integers(lo, hi, (H1, r))) for _ in range(nA)]
    B = [f16_bits(rng.integers(lo, hi, (r, H2))) for _ in range(nA)]
    return X, A, B


@settings(max_examples=40, deadline=None)
@given(st.integers(1, 12), st.integers(1, 9), st.integers(1, 5), st.integers(1, 9), st.integers(0, 10 ** 6))
def test_delta_is_linear_in_scale_and_additive_in_B(T, H1, r, H2, seed):
    rng = np.random.default_rng(seed)
    X, A, B = _int_case(rng, T, H1, r, H2, 2)
    B2 = [f16_bits(rng.integers(-3, 4, (r, H2))) for _ in range(2)]
    Bsum = [f16_bits(dec(b, "f16") + dec(c, "f16")) for b, c in zip(B, B2)]  # |values| <= 6: exact
    cut = int(rng.integers(0, T + 1))
    seg, idx = [0, cut, T], [1, 0]
    zero = np.zeros((T, H2))
    d1, _ = oracle.apply_f64(zero, X, A, B, seg, idx, 1.0, "f16")
    d2, _ = oracle.apply_f64(zero, X, A, B2, seg, idx, 1.0, "f16")
    ds, _ = oracle.apply_f64(zero, X, A, Bsum, seg, idx, 1.0, "f16")
    assert np.array_equal(ds, d1 + d2)                       # additive in B_i (exact: integers)
    d3, _ = oracle.apply_f64(zero, X, A, B, seg, idx, -2.5, "f16")
    assert np.array_equal(d3, -2.5 * d1)                     # linear in scale (exact: dyadic)
    # against numpy's products, row by row with each row's own adapter
    x = dec(X, "f16")
    for t in range(T):
        i = idx[0] if t < cut else idx[1]
        assert np.array_equal(d1[t], (x[t] @ dec(A[i], "f16")) @ dec(B[i], "f16"))


@settings(max_examples=30, deadline=None)
@given(st.integers(2, 12), st.integers(1, 9), st.integers(1, 5), st.integers(1, 9), st.integers(0, 10 ** 6))
def test_zero_rows_of_x_leave_y_unchanged(T, H1, r, H2, seed):
    rng = np.random.default_rng(seed)
    X, A, B = _int_case(rng, T, H1, r, H2, 3)
    zero_rows = rng.random(T) < 0.5
    X[zero_rows] = 0
    Y = f16_bits(rng.integers(-8, 9, (T, H2)))
    got, _ = oracle.apply_f32(Y, X, A, B, [0, T], [int(rng.integers(0, 3))], 0.75, "f16")
    assert np.array_equal(got[zero_rows], Y[zero_rows])


# ---------------------------------------------------------------------------------------------
# the one-element function used for sampled checks at full size
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("r", [8, 16, 64, 128])
def test_element_function_equals_whole_batch_bit_for_bit(dt, r):
    # every element of ragged random problems (non-zero base output, scale not a power of two,
    # several adapters, empty segment): oracle_apply_f32_element must give the bits that
    # oracle_apply_f32 (pinned by everything above) writes there. A slip such as B_i indexed
    # as [c, j], a dropped base term or scale applied per term fails it.
    rng = np.random.default_rng(1000 + r)
    T, H1, H2, nA = 11, 72, 40, 3
    X = inputs.cast_f32_bits(rng.standard_normal((T, H1)).astype(np.float32), dt)
    A = [inputs.cast_f32_bits((rng.standard_normal((H1, r)) / np.sqrt(H1)).astype(np.float32), dt)
         for _ in range(nA)]
    B = [inputs.cast_f32_bits((rng.standard_normal((r, H2)) / np.sqrt(r)).astype(np.float32), dt)
         for _ in range(nA)]
    Y = inputs.cast_f32_bits(rng.standard_normal((T, H2)).astype(np.float32), dt)
    seg, idx = [0, 4, 4, 9, 11], [2, 0, 1, 2]
    for scale in (0.6180339887, -1.75):
        full, _ = oracle.apply_f32(Y, X, A, B, seg, idx, scale, dt)
        for s in range(len(idx)):
            for t in range(seg[s], seg[s + 1]):
                for c in range(H2):
                    got = oracle.apply_f32_element(X[t], A[idx[s]], B[idx[s]], int(Y[t, c]), c, scale, dt)
                    assert got == int(full[t, c]), (dt, r, scale, t, c)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_element_function_exact_on_integer_operands(dt):
    # small integers: every product and sum is exact in fp32, so the element equals numpy's
    # y + scale * (x @ A) @ B exactly (scale 0.5 keeps it dyadic), independently of the oracle
    rng = np.random.default_rng(77)
    H1, r, H2 = 24, 8, 16
    enc = f16_bits if dt == "f16" else bf16_bits
    x = enc(rng.integers(-3, 4, H1))
    Ai = enc(rng.integers(-2, 3, (H1, r)))
    Bi = enc(rng.integers(-2, 3, (r, H2)))
    y = enc(rng.integers(-20, 21, H2))
    exact = dec(y, dt) + 0.5 * ((dec(x, dt) @ dec(Ai, dt)) @ dec(Bi, dt))
    # one rounding of the exact value to the storage type, by numpy / torch
    if dt == "f16":
        ref = exact.astype(np.float16).astype(np.float64)
    else:
        ref = torch.tensor(exact).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    for c in range(H2):
        got = oracle.apply_f32_element(x, Ai, Bi, int(y[c]), c, 0.5, dt)
        assert dec(np.array([got], np.uint16), dt)[0] == ref[c], c


# ---------------------------------------------------------------------------------------------
# the whole layer, Y = X@W + the delta (README multi-LoRA paragraph): base_plus_delta_f32
# ---------------------------------------------------------------------------------------------

def _layer_int_case(rng, dt, T=13, H1=24, H2=20, r=4, nA=3):
    enc = f16_bits if dt == "f16" else bf16_bits
    X = enc(rng.integers(-3, 4, (T, H1)))
    W = enc(rng.integers(-3, 4, (H1, H2)))
    A = [enc(rng.integers(-2, 3, (H1, r))) for _ in range(nA)]
    B = [enc(rng.integers(-2, 3, (r, H2))) for _ in range(nA)]
    return X, W, A, B


def _round_to(values, dt):
    """One round-to-nearest-even of exact values to the storage type (numpy / torch)."""
    if dt == "f16":
        return values.astype(np.float16).astype(np.float64)
    return torch.tensor(values).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_layer_identity_with_materialised_weight(dt):
    # integer operands: every product and partial sum is exact in fp32, so the layer must equal,
    # bit for bit, x @ (W + scale * A_i @ B_i) with the merged weight built in fp64 by numpy --
    # the README identity x@(W + A@B) = x@W + x@A@B, row by row with each row's own adapter;
    # rows in no segment (0, 1 and 12) and the rejected segment's rows get x@W alone
    rng = np.random.default_rng(31)
    X, W, A, B = _layer_int_case(rng, dt)
    seg = [2, 5, 5, 9, 11, 12]
    idx = [2, 0, 1, 7, 0]  # [5,5) empty; adapter 7 does not exist: [9,11) rejected
    got, skipped = oracle.base_plus_delta_f32(X, W, A, B, seg, idx, 0.5, dt)
    assert skipped == 1
    x, w = dec(X, dt), dec(W, dt)
    owner = {t: i for s, i in enumerate(idx) if i < 3 for t in range(seg[s], seg[s + 1])}
    for t in range(X.shape[0]):
        merged = w if t not in owner else w + 0.5 * (dec(A[owner[t]], dt) @ dec(B[owner[t]], dt))
        assert np.array_equal(dec(got[t], dt), _round_to(x[t] @ merged, dt)), t


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_layer_with_zero_weight_is_the_delta_alone(dt):
    # W = 0: base is +0 everywhere, so each row equals what the SGMV oracle (pinned above) adds
    # onto a zero base, bit for bit
    rng = np.random.default_rng(5)
    T, H1, H2, r = 10, 40, 24, 8
    X = inputs.cast_f32_bits(rng.standard_normal((T, H1)).astype(np.float32), dt)
    A = [inputs.cast_f32_bits((rng.standard_normal((H1, r)) / 6).astype(np.float32), dt) for _ in range(2)]
    B = [inputs.cast_f32_bits((rng.standard_normal((r, H2)) / 3).astype(np.float32), dt) for _ in range(2)]
    W = np.zeros((H1, H2), np.uint16)
    seg, idx = [0, 4, 10], [1, 0]
    got, _ = oracle.base_plus_delta_f32(X, W, A, B, seg, idx, 0.7, dt)
    ref, _ = oracle.apply_f32(np.zeros((T, H2), np.uint16), X, A, B, seg, idx, 0.7, dt)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_layer_without_segments_is_the_base_product(dt):
    # no segments: Y = round(X@W); against numpy's fp64 product within the fp32 summation bound
    # plus one rounding of the storage type
    rng = np.random.default_rng(6)
    T, H1, H2 = 9, 96, 33
    X = inputs.cast_f32_bits(rng.standard_normal((T, H1)).astype(np.float32), dt)
    W = inputs.cast_f32_bits((rng.standard_normal((H1, H2)) / np.sqrt(H1)).astype(np.float32), dt)
    A = [np.zeros((H1, 4), np.uint16)]
    B = [np.zeros((4, H2), np.uint16)]
    got, _ = oracle.base_plus_delta_f32(X, W, A, B, [0], [], 1.0, dt)
    x, w = dec(X, dt), dec(W, dt)
    exact = x @ w
    bound = H1 * 2.0 ** -24 * (np.abs(x) @ np.abs(w))
    ulp = 2.0 ** (-10 if dt == "f16" else -7) * np.maximum(np.abs(exact), 2.0 ** -14)
    assert np.all(np.abs(dec(got, dt) - exact) <= ulp + bound)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_layer_random_operands_against_fp64_merged_weight(dt):
    # random normal operands, several adapters and a non-dyadic scale: within the fp32 bound of
    # the merged-weight product in fp64, plus one storage rounding
    rng = np.random.default_rng(8)
    T, H1, H2, r = 16, 64, 40, 8
    X = inputs.cast_f32_bits(rng.standard_normal((T, H1)).astype(np.float32), dt)
    W = inputs.cast_f32_bits((rng.standard_normal((H1, H2)) / np.sqrt(H1)).astype(np.float32), dt)
    A = [inputs.cast_f32_bits((rng.standard_normal((H1, r)) / np.sqrt(H1)).astype(np.float32), dt)
         for _ in range(3)]
    B = [inputs.cast_f32_bits((rng.standard_normal((r, H2)) / np.sqrt(r)).astype(np.float32), dt)
         for _ in range(3)]
    seg, idx = [0, 5, 11, 16], [2, 0, 1]
    scale = 0.37
    got, _ = oracle.base_plus_delta_f32(X, W, A, B, seg, idx, scale, dt)
    x, w = dec(X, dt), dec(W, dt)
    for s in range(3):
        a, b = dec(A[idx[s]], dt), dec(B[idx[s]], dt)
        rows = slice(seg[s], seg[s + 1])
        exact = x[rows] @ (w + scale * (a @ b))
        terms = np.abs(x[rows]) @ np.abs(w) + abs(scale) * ((np.abs(x[rows]) @ np.abs(a)) @ np.abs(b))
        bound = (H1 + r + 2) * 2.0 ** -24 * terms
        ulp = 2.0 ** (-10 if dt == "f16" else -7) * np.maximum(np.abs(exact), 2.0 ** -14)
        assert np.all(np.abs(dec(got[rows], dt) - exact) <= ulp + bound), s
