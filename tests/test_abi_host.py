"""Host-side checks of the C-ABI library; no GPU needed and no kernel is launched.

- the library loads and exports every function include/lora_sgmv.h declares;
- segment bookkeeping (host C++) is bit-exact against the oracle's grouping;
- every host-side validation error returns its code before any CUDA call.
"""
import os
import re

import numpy as np
import pytest

import oracle
from adapter_matmul_b200 import inputs, sgmv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lora_sgmv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lora_sgmv_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(sgmv.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = sgmv.load()
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_version_and_ranks():
    assert sgmv.lora_sgmv_version() >= 200  # 0.2.0 or later
    for r in (8, 16, 32, 64, 128):
        assert sgmv.lora_sgmv_rank_supported(r, sgmv.VARIANT_SPLIT)
        assert sgmv.lora_sgmv_rank_supported(r, sgmv.VARIANT_FUSED)
        assert sgmv.lora_sgmv_rank_supported(r, sgmv.VARIANT_FUSED_TC) == (r in (16, 32, 64))
        assert sgmv.lora_sgmv_rank_supported(r, sgmv.VARIANT_SPLIT_TC) == (r in (16, 32, 64))
        assert sgmv.lora_sgmv_rank_supported(r, sgmv.VARIANT_GROUPED_TC) == (r in (16, 32, 64))
    for r in (0, 4, 24, 256):
        assert not sgmv.lora_sgmv_rank_supported(r, sgmv.VARIANT_SPLIT)
    assert sgmv.lora_sgmv_workspace_bytes(32, 16) == 2048
    assert sgmv.lora_sgmv_workspace_bytes(3, 8) == 256
    assert sgmv.lora_sgmv_workspace_bytes(0, 8) == 0
    for st in range(9):
        assert sgmv.status_string(st)


# ---- bookkeeping: bit-exact against the oracle ---------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "distinct", "uniform_h4096", "skewed_h4096", "identical_h4096",
                                  "prefill", "llama70b_decode_h28672"])
def test_group_segments_bit_exact_on_configs(name):
    w = inputs.make(name)
    got = sgmv.lora_sgmv_group_segments(w.ids, w.num_adapters)
    ref = oracle.group_segments(w.ids, w.num_adapters)
    for g, o in zip(got, ref):
        assert g.dtype == np.int32 and np.array_equal(g, o)


def test_group_segments_bit_exact_random_and_edges():
    rng = np.random.default_rng(0)
    cases = [np.zeros(0, np.int32), np.array([5], np.int32), np.full(100, 3, np.int32),
             np.arange(50, dtype=np.int32)[::-1].copy()]
    for _ in range(200):
        T = int(rng.integers(1, 300))
        A = int(rng.integers(1, 70))
        cases.append(rng.integers(0, A, T).astype(np.int32))
    for ids in cases:
        A = int(ids.max()) + 1 if ids.size else 1
        A += int(rng.integers(0, 3))
        got = sgmv.lora_sgmv_group_segments(ids, A)
        ref = oracle.group_segments(ids, A)
        for g, o in zip(got, ref):
            assert np.array_equal(g, o)


def test_group_segments_errors():
    with pytest.raises(sgmv.SGMVError) as e:
        sgmv.lora_sgmv_group_segments(np.array([0, 4], np.int32), 4)
    assert e.value.status == 8
    with pytest.raises(sgmv.SGMVError) as e:
        sgmv.lora_sgmv_group_segments(np.array([0, -1], np.int32), 4)
    assert e.value.status == 8
    with pytest.raises(sgmv.SGMVError) as e:
        sgmv.lora_sgmv_group_segments(np.array([0], np.int32), 0)
    assert e.value.status == 2
    lib = sgmv.load()
    assert lib.lora_sgmv_group_segments(None, 3, 4, None, None, None, None) == 1


# ---- host validation: every error path returns before touching the GPU ------------------------

FAKE = 1 << 20  # a 16-byte-aligned non-null value; never dereferenced on these paths
MIS = FAKE + 2  # misaligned


def apply(**kw):
    a = dict(Y=FAKE, X=FAKE, A=FAKE, B=FAKE, seg=FAKE, idx=FAKE, n=2, na=4, T=8, H1=256, r=16, H2=256,
             scale=1.0, dt=0, mx=0, ws=FAKE, wsb=1 << 20, st=None, var=0)
    a.update(kw)
    return sgmv.load().lora_sgmv_apply_ex(a["Y"], a["X"], a["A"], a["B"], a["seg"], a["idx"], a["n"], a["na"],
                                          a["T"], a["H1"], a["r"], a["H2"], a["scale"], a["dt"], a["mx"], a["ws"],
                                          a["wsb"], a["st"], a["var"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(dt=7), 4), (dict(n=-1), 2), (dict(T=-1), 2), (dict(H1=0), 2), (dict(H2=-8), 2), (dict(r=0), 2),
    (dict(r=24), 5), (dict(r=256), 5), (dict(var=9), 5),
    (dict(Y=None), 1), (dict(X=None), 1), (dict(A=None), 1), (dict(B=None), 1), (dict(seg=None), 1),
    (dict(idx=None), 1), (dict(na=0), 2),
    (dict(Y=MIS), 3), (dict(X=MIS), 3), (dict(H1=260), 3), (dict(H2=100), 3),
    (dict(ws=None), 7), (dict(wsb=100), 7), (dict(ws=MIS), 3),
    # the tensor-core decode kernel takes H1 and H2 in multiples of 64 only
    (dict(var=4, H1=264), 5), (dict(var=4, H2=136), 5), (dict(var=4, r=8), 5),
    (dict(var=5, H1=264), 5), (dict(var=5, H2=136), 5), (dict(var=5, r=128), 5), (dict(var=6), 5),
])
def test_apply_validation_codes(kw, code):
    assert apply(**kw) == code


def test_empty_problems_are_noops_without_gpu():
    # n_segments == 0 or T == 0 returns OK before any CUDA call, even with NULL pointers
    assert apply(n=0, Y=None, X=None) == 0
    assert apply(T=0, Y=None) == 0
    lib = sgmv.load()
    assert lib.lora_sgmv_shrink(None, None, None, None, None, 0, 1, 5, 64, 16, 0, None, None) == 0
    assert lib.lora_sgmv_expand(None, None, None, None, None, 3, 1, 0, 16, 64, 1.0, 0, None, None) == 0


def test_shrink_expand_validation_codes():
    lib = sgmv.load()
    sh = lambda **k: lib.lora_sgmv_shrink(k.get("V", FAKE), k.get("X", FAKE), FAKE, FAKE, FAKE, 2, 4, 8,
                                          k.get("H1", 256), k.get("r", 16), k.get("dt", 0), None, None)
    ex = lambda **k: lib.lora_sgmv_expand(k.get("Y", FAKE), k.get("V", FAKE), FAKE, FAKE, FAKE, 2, 4, 8,
                                          k.get("r", 16), k.get("H2", 256), 1.0, k.get("dt", 0), None, None)
    assert sh(V=None) == 1 and sh(X=MIS) == 3 and sh(H1=12) == 3 and sh(r=12) == 5 and sh(dt=3) == 4
    assert ex(Y=None) == 1 and ex(V=MIS) == 3 and ex(H2=12) == 3 and ex(r=7) == 5 and ex(dt=-1) == 4


def test_pad_rank_validation_codes():
    lib = sgmv.load()

    def pad(Ad=FAKE, As=FAKE + 4096, Bd=FAKE + 8192, Bs=FAKE + 12288, H1=64, H2=48, rs=8, r=16, dt=0):
        return lib.lora_sgmv_pad_rank(Ad, As, Bd, Bs, H1, H2, rs, r, dt, None)

    assert pad(dt=2) == 4 and pad(dt=-1) == 4
    assert pad(Ad=None, As=None, Bd=None, Bs=None) == 1
    assert pad(Ad=None) == 1 and pad(Bs=None) == 1
    assert pad(rs=0) == 2 and pad(rs=17) == 2 and pad(r=4) == 2
    assert pad(H1=0) == 2 and pad(H2=-1) == 2
    # a pair left out makes its size unused
    assert pad(Ad=None, As=None, H1=0, rs=17) == 2


def test_batched_validation_codes():
    lib = sgmv.load()

    def call(n_problems=2, T=8, r=16, dt=0, n=2, **pk):
        arr = (sgmv.Problem * 8)()
        for i in range(8):
            q = dict(Y=FAKE, X=FAKE, A=FAKE, B=FAKE, na=4, H1=256, H2=512, scale=1.0)
            q.update(pk)
            arr[i] = sgmv.Problem(q["Y"], q["X"], q["A"], q["B"], q["na"], q["H1"], q["H2"], q["scale"])
        return lib.lora_sgmv_apply_batched(ctypes.addressof(arr), n_problems, FAKE, FAKE, n, T, r, dt, 0, None, None)

    import ctypes
    assert call(dt=5) == 4
    assert call(n_problems=0) == 2 and call(n_problems=9) == 2
    assert call(r=12) == 5
    assert call(Y=None) == 1 and call(A=None) == 1
    assert call(X=MIS) == 3 and call(H2=100) == 3
    assert call(na=0) == 2 and call(H1=0) == 2
    assert call(n=0, Y=None) == 0  # empty: OK before any CUDA call
    assert lib.lora_sgmv_apply_batched(None, 1, FAKE, FAKE, 1, 1, 16, 0, 0, None, None) == 1


@pytest.mark.parametrize("name,want", [
    ("tiny", "FUSED"), ("distinct", "FUSED"), ("uniform_h4096", "FUSED"), ("uniform_h11008", "FUSED"),
    ("skewed_h4096", "FUSED"), ("skewed_h11008", "FUSED"), ("identical_h4096", "FUSED"),
    ("identical_h11008", "FUSED"), ("prefill", "GROUPED_TC"), ("llama70b_decode_h28672", "SPLIT_TC"),
    ("llama70b_decode_h8192", "SPLIT_TC")])
def test_auto_variant_on_the_configurations(name, want):
    # the dispatcher's choice for each benchmark configuration on a 148-SM B200 (host only)
    w = inputs.make(name)
    seg, idx, _ = sgmv.lora_sgmv_group_segments(w.ids, w.num_adapters)
    dt = sgmv.F16 if w.dtype == "f16" else sgmv.BF16
    got = sgmv.lora_sgmv_auto_variant(w.T, len(idx), w.H1, w.r, w.H2, dt, int(np.max(np.diff(seg))), 148)
    assert got == getattr(sgmv, "VARIANT_" + want)


def test_auto_variant_rule_edges():
    V, F16, BF16 = sgmv, sgmv.F16, sgmv.BF16
    auto = sgmv.lora_sgmv_auto_variant
    # the grouped kernel from one M-tile of rows, for the ranks it has
    assert auto(4096, 8, 4096, 64, 4096, BF16, 128) == V.VARIANT_GROUPED_TC
    assert auto(4096, 8, 4096, 64, 4096, BF16, 127) != V.VARIANT_GROUPED_TC
    assert auto(4096, 8, 4096, 128, 4096, BF16, 512) == V.VARIANT_FUSED  # no tensor-core kernel at r = 128
    # unknown length: ceil(T / n)
    assert auto(1024, 8, 4096, 64, 4096, BF16, 0) == V.VARIANT_GROUPED_TC
    # more segments than the fused kernels hold
    assert auto(9000, 8193, 4096, 16, 4096, F16, 1) == V.VARIANT_SPLIT
    # tensor-core decode needs segments of 3+ tokens, r >= 32, H multiples of 64
    assert auto(256, 95, 8192, 64, 28672, BF16, 2) == V.VARIANT_FUSED
    assert auto(256, 95, 8192, 16, 28672, BF16, 56) == V.VARIANT_FUSED
    assert auto(256, 95, 8192, 64, 28680, BF16, 56) == V.VARIANT_FUSED
    # the split form: fewer jobs than SMs and B_i of 1,000,000 bytes or more
    assert auto(256, 95, 8192, 64, 28672, BF16, 56, 148) == V.VARIANT_SPLIT_TC
    assert auto(256, 95, 8192, 64, 28672, BF16, 56, 100) == V.VARIANT_FUSED_TC   # 111 jobs, 100 SMs
    assert auto(256, 95, 8192, 64, 8192, BF16, 56, 148) == V.VARIANT_SPLIT_TC    # 1,048,576 bytes
    assert auto(256, 95, 8192, 64, 7808, BF16, 56, 148) == V.VARIANT_FUSED_TC    # 999,424 bytes
    assert auto(256, 95, 8192, 32, 8192, BF16, 56, 148) == V.VARIANT_FUSED_TC    # 524,288 bytes
    # invalid sizes
    assert auto(0, 1, 64, 16, 64, F16, 1) == V.VARIANT_AUTO
    assert auto(8, 1, 64, 16, 64, 7, 1) == V.VARIANT_AUTO
    assert auto(8, 1, 64, 16, 64, F16, 1, 0) == V.VARIANT_AUTO


def gemm(**kw):
    a = dict(Y=FAKE, X=FAKE, W=FAKE, A=FAKE, B=FAKE, seg=FAKE, idx=FAKE, n=2, na=4, T=300, H1=256, r=64, H2=264,
             scale=1.0, dt=1, mx=0, ws=FAKE, wsb=1 << 20, st=None)
    a.update(kw)
    return sgmv.load().lora_sgmv_gemm_apply(a["Y"], a["X"], a["W"], a["A"], a["B"], a["seg"], a["idx"], a["n"],
                                            a["na"], a["T"], a["H1"], a["r"], a["H2"], a["scale"], a["dt"], a["mx"],
                                            a["ws"], a["wsb"], a["st"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(dt=7), 4), (dict(n=-1), 2), (dict(T=-1), 2), (dict(na=-1), 2), (dict(H1=0), 2), (dict(H2=-8), 2),
    (dict(r=0), 2), (dict(r=8), 5), (dict(r=128), 5), (dict(H1=260), 3), (dict(H2=100), 3),
    (dict(Y=None), 1), (dict(X=None), 1), (dict(W=None), 1), (dict(A=None), 1), (dict(seg=None), 1),
    (dict(na=0), 2), (dict(Y=MIS), 3), (dict(W=MIS), 3),
    (dict(ws=None), 7), (dict(wsb=300 * 64 * 4 - 4), 7), (dict(ws=MIS), 3),
])
def test_gemm_apply_validation_codes(kw, code):
    # the whole-layer entry point rejects bad arguments on the host, before any CUDA call
    assert gemm(**kw) == code


def test_gemm_apply_empty_batch_is_a_noop_without_gpu():
    assert gemm(T=0, Y=None, X=None, W=None) == 0


def ranks(**kw):
    a = dict(Y=FAKE, X=FAKE, A=FAKE, B=FAKE, rk=FAKE, seg=FAKE, idx=FAKE, n=2, na=4, T=300, H1=256, rmax=64,
             H2=264, scale=1.0, dt=1, st=None)
    a.update(kw)
    return sgmv.load().lora_sgmv_apply_ranks(a["Y"], a["X"], a["A"], a["B"], a["rk"], a["seg"], a["idx"], a["n"],
                                             a["na"], a["T"], a["H1"], a["rmax"], a["H2"], a["scale"], a["dt"],
                                             a["st"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(dt=7), 4), (dict(n=-1), 2), (dict(H1=0), 2), (dict(rmax=0), 2), (dict(rmax=8), 5), (dict(rmax=128), 5),
    (dict(H1=32), 5), (dict(H2=56), 5), (dict(rk=None), 1), (dict(Y=None), 1), (dict(idx=None), 1),
    (dict(na=0), 2), (dict(X=MIS), 3), (dict(H1=260), 3),
])
def test_apply_ranks_validation_codes(kw, code):
    assert ranks(**kw) == code


def test_apply_ranks_empty_batch_is_a_noop_without_gpu():
    assert ranks(n=0, Y=None, rk=None) == 0


def test_flags_other_than_early_reads_are_refused():
    lib = sgmv.load()
    for flags in (0x2, 0x80000000, 0x3):
        assert lib.lora_sgmv_apply_flags(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 4, 8, 256, 16, 256, 1.0, 0, 0, FAKE,
                                         1 << 20, None, 0, flags, None) == 5
        assert lib.lora_sgmv_apply_batched_flags(None, 1, FAKE, FAKE, 2, 8, 16, 0, 0, flags, None, None) == 5
    # the one defined flag passes validation (an empty batch then returns OK with no CUDA call)
    assert lib.lora_sgmv_apply_flags(None, None, None, None, None, None, 0, 4, 8, 256, 16, 256, 1.0, 0, 0, None, 0,
                                     None, 0, sgmv.FLAG_EARLY_READS, None) == 0


def test_step_host_validation_codes_before_any_copy():
    # every check of lora_sgmv_step_host returns before a copy or launch is enqueued
    import ctypes
    lib = sgmv.load()
    ids = np.array([0, 2, 1, 2], np.int32)
    meta = np.zeros(2 * 4 + 1, np.int32)
    probs = (sgmv.Problem * 1)(sgmv.Problem(FAKE, FAKE, FAKE, FAKE, 4, 256, 512, 1.0))
    cps = (sgmv.Copy * 1)(sgmv.Copy(FAKE, FAKE, 64))

    def call(ids_p=ids.ctypes.data, T=4, na=4, mh=meta.ctypes.data, md=FAKE, h2d=ctypes.addressof(cps), nh=1,
             pr=ctypes.addressof(probs), npr=1, d2h=ctypes.addressof(cps), nd=1):
        return lib.lora_sgmv_step_host(ids_p, T, na, mh, md, None, h2d, nh, pr, npr, 16, 0, 0, d2h, nd, None, None,
                                       None)

    assert call(mh=None) == 1 and call(md=None) == 1 and call(pr=None) == 1 and call(ids_p=None) == 1
    assert call(T=-1) == 2 and call(na=0) == 2 and call(npr=0) == 2 and call(npr=9) == 2
    assert call(h2d=None) == 1 and call(d2h=None) == 1 and call(nh=-1) == 1
    bad = (sgmv.Copy * 1)(sgmv.Copy(None, FAKE, 64))
    assert call(h2d=ctypes.addressof(bad)) == 1
    ids[1] = 4  # out of [0, num_adapters)
    assert call() == 8
    ids[1] = -1
    assert call() == 8
    assert not meta.any()  # nothing was written before the id check failed
