"""Full-size parity: every output element of the largest configurations against the oracle.

The prefill (T = 9771, H1 = H2 = 4096, r = 64, bf16) and the 70B-shaped decode (T = 256,
H1 = 8192, H2 = 28672 and 8192, r = 64, 1024 resident adapters, bf16) run in the launch
configuration the benchmark times (the dispatcher's choice) and in the other kernels that
take them; the Distinct decode runs as the benchmark's one batched launch of four
projections. The oracle (single-threaded C, run on row shares in threads) computes every
element; the bar is the parity tolerance |gpu - oracle| <= 2e-2 + 1e-2 |oracle|.
"""
import numpy as np
import pytest
import torch

from adapter_matmul_b200 import inputs, sgmv
from gpu_helpers import DeviceProblem, assert_close, dt_code, from_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,variant", [
    ("prefill", sgmv.VARIANT_AUTO),
    ("prefill", sgmv.VARIANT_SPLIT),
    ("llama70b_decode_h28672", sgmv.VARIANT_AUTO),
    ("llama70b_decode_h28672", sgmv.VARIANT_FUSED_TC),
    ("llama70b_decode_h8192", sgmv.VARIANT_AUTO),
    ("llama70b_decode_h8192", sgmv.VARIANT_FUSED_TC),
    ("llama70b_decode_h8192", sgmv.VARIANT_FUSED),
])
def test_full_size_every_element(name, variant):
    w = inputs.make(name)
    p = DeviceProblem(w, y_random=True)
    got = p.apply(variant=variant)
    assert int(p.status.item()) == 0
    assert_close(got, p.oracle_apply(), w.dtype, f"{name} variant {variant}")


def test_distinct_batched_launch_every_element():
    # the benchmark's step: four projections (own adapters, X and Y each) in one launch
    w = inputs.distinct()
    probs = []
    for proj in range(4):
        wp = inputs.distinct()
        probs.append(DeviceProblem(wp, proj=proj, y_random=True))
    p0 = probs[0]
    sgmv.lora_sgmv_apply_batched(
        [dict(Y=p.Y, X=p.X, A_ptrs=p.A_ptrs, B_ptrs=p.B_ptrs, num_adapters=w.num_adapters, H1=w.H1, H2=w.H2,
              scale=w.scale) for p in probs],
        p0.d_seg, p0.d_idx, p0.n, w.T, w.r, dt_code(w.dtype), p0.max_len(), p0.status)
    torch.cuda.synchronize()
    assert int(p0.status.item()) == 0
    for proj, p in enumerate(probs):
        assert_close(from_dev(p.Y), p.oracle_apply(), w.dtype, f"distinct projection {proj}")
