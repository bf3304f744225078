"""Overlap with the previous kernel (programmatic dependent launch), on the GPU.

The fused kernels start while the kernel before them on the stream finishes. By default
they read nothing the caller passed until that kernel has completed, so a kernel that
writes the segment arrays or the adapters right before an SGMV call must be seen by it.
These tests put such a writer immediately before the call on the same stream: a torch
kernel that writes seg_starts (whose previous contents describe no work at all), and the
library's own padding kernel writing the adapters (whose previous contents are NaN). Each
result is compared with the oracle. A third test passes LORA_SGMV_FLAG_EARLY_READS where the
statement holds (segments and adapters written by copies) and checks the result too.
"""
import numpy as np
import pytest
import torch

from adapter_matmul_b200 import inputs, sgmv
from gpu_helpers import DeviceProblem, assert_close, dt_code, from_dev, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,variant", [("skewed_h4096", sgmv.VARIANT_FUSED),
                                          ("llama70b_decode_h8192", sgmv.VARIANT_FUSED_TC),
                                          ("skewed_h4096", sgmv.VARIANT_AUTO)])
def test_kernel_writing_segments_right_before_the_call(name, variant):
    w = inputs.make(name)
    p = DeviceProblem(w, y_random=True)
    true_seg = p.d_seg.clone()
    p.d_seg.zero_()  # describes n empty segments: an early read would leave Y unchanged
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    torch.add(true_seg, 0, out=p.d_seg)  # a kernel, launched immediately before the call
    sgmv.lora_sgmv_apply_ex(p.Y, p.X, p.A_ptrs, p.B_ptrs, p.d_seg, p.d_idx, p.n, w.num_adapters, w.T, w.H1, w.r,
                            w.H2, w.scale, dt_code(w.dtype), p.max_len(), p.ws, p.ws_bytes, p.status, variant,
                            stream.cuda_stream)
    torch.cuda.synchronize()
    assert int(p.status.item()) == 0
    assert_close(from_dev(p.Y), p.oracle_apply(), w.dtype, f"{name}, segments written by the previous kernel")


def test_batched_call_after_a_kernel_writing_segments():
    w = inputs.distinct()
    probs = [DeviceProblem(inputs.distinct(), proj=k, y_random=True) for k in range(4)]
    p0 = probs[0]
    true_seg = p0.d_seg.clone()
    p0.d_seg.zero_()
    torch.cuda.synchronize()
    torch.add(true_seg, 0, out=p0.d_seg)
    sgmv.lora_sgmv_apply_batched(
        [dict(Y=p.Y, X=p.X, A_ptrs=p.A_ptrs, B_ptrs=p.B_ptrs, num_adapters=w.num_adapters, H1=w.H1, H2=w.H2,
              scale=w.scale) for p in probs],
        p0.d_seg, p0.d_idx, p0.n, w.T, w.r, dt_code(w.dtype), p0.max_len(), p0.status)
    torch.cuda.synchronize()
    assert int(p0.status.item()) == 0
    for k, p in enumerate(probs):
        assert_close(from_dev(p.Y), p.oracle_apply(), w.dtype, f"projection {k}")


@pytest.mark.parametrize("r_src,r,variant", [(8, 16, sgmv.VARIANT_FUSED), (48, 64, sgmv.VARIANT_FUSED_TC)])
def test_padding_kernel_right_before_the_call(r_src, r, variant):
    # the padded adapters start as NaN; lora_sgmv_pad_rank writes them and the SGMV call
    # follows at once on the same stream
    T, nA, H1, H2 = 48, 3, 512, 384
    w_src = inputs.small_random(T, nA, H1, H2, r_src, "bf16", seed=r)
    w = inputs.small_random(T, nA, H1, H2, r, "bf16", seed=r)  # same ids, X and Y (the draws do not use r)
    p = DeviceProblem(w, y_random=True)
    src_A = [w_src.adapter_a(i) for i in range(nA)]
    src_B = [w_src.adapter_b(i) for i in range(nA)]
    for i in range(nA):
        p.dA[i].fill_(float("nan"))
        p.dB[i].fill_(float("nan"))
    dsa = [to_dev(a, "bf16") for a in src_A]
    dsb = [to_dev(b, "bf16") for b in src_B]
    torch.cuda.synchronize()
    for i in range(nA):
        sgmv.lora_sgmv_pad_rank(p.dA[i], dsa[i], p.dB[i], dsb[i], H1, H2, r_src, r, sgmv.BF16)
    got = p.apply(variant=variant)
    assert int(p.status.item()) == 0
    # expected: the oracle on numpy's zero padding of the source adapters
    for i in range(nA):
        a = np.zeros((H1, r), np.uint16)
        a[:, :r_src] = src_A[i]
        b = np.zeros((r, H2), np.uint16)
        b[:r_src] = src_B[i]
        p.A[i], p.B[i] = a, b
    assert_close(got, p.oracle_apply(), "bf16", f"pad {r_src}->{r} then variant {variant}")


@pytest.mark.parametrize("variant", [sgmv.VARIANT_FUSED, sgmv.VARIANT_AUTO])
def test_early_reads_flag_when_inputs_come_from_copies(variant):
    w = inputs.make("skewed_h11008")
    p = DeviceProblem(w, y_random=True)
    host_seg = p.d_seg.cpu().pin_memory()
    p.d_seg.zero_()
    torch.cuda.synchronize()
    p.d_seg.copy_(host_seg, non_blocking=True)  # a copy (not a kernel) right before the call
    sgmv.lora_sgmv_apply_flags(p.Y, p.X, p.A_ptrs, p.B_ptrs, p.d_seg, p.d_idx, p.n, w.num_adapters, w.T, w.H1, w.r,
                               w.H2, w.scale, dt_code(w.dtype), p.max_len(), p.ws, p.ws_bytes, p.status, variant,
                               sgmv.FLAG_EARLY_READS)
    torch.cuda.synchronize()
    assert int(p.status.item()) == 0
    assert_close(from_dev(p.Y), p.oracle_apply(), w.dtype, "early reads after a copy")
