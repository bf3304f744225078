"""lora_sgmv_apply_noalloc against lora_sgmv_apply, through the C ABI.

lora_sgmv_apply_noalloc is for callers that may not allocate device memory
where they run SGMV -- a serving loop whose memory is fixed at start-up, or a
plugin whose host framework owns the device memory -- and so cannot pass the
workspace that lora_sgmv_apply takes. It keeps the fp32 scratch of the split
kernels in a fixed array inside the library. These tests check that two calls
in a row give what lora_sgmv_apply gives on the same inputs, within the
parity tolerance of the other GPU tests, that they match the CPU oracle
within the same tolerance, that a repeated call on the same inputs gives the
same bits and changes the device's free memory by nothing, and that oversize
problems are refused. This file sorts last so that a run stopping at its
first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from adapter_matmul_b200 import inputs, sgmv
from gpu_helpers import DeviceProblem, assert_close, dt_code, from_dev, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(p: DeviceProblem) -> np.ndarray:
    w = p.w
    sgmv.lora_sgmv_apply_noalloc(p.Y, p.X, p.A_ptrs, p.B_ptrs, p.d_seg, p.d_idx, p.n, w.num_adapters, w.T, w.H1,
                                 w.r, w.H2, w.scale, dt_code(w.dtype), p.max_len(), p.status)
    torch.cuda.synchronize()
    return from_dev(p.Y)


def test_noalloc_matches_apply_on_two_calls_in_a_row():
    # the second call runs on whatever the first left in the shared scratch array
    for name in ("skewed_h11008", "uniform_h4096"):
        w = inputs.make(name)
        ref = DeviceProblem(w, y_random=True).apply()  # existing entry point, caller workspace
        p = DeviceProblem(w, y_random=True)
        got = _noalloc(p)
        assert_close(got, ref, w.dtype, f"noalloc vs apply on {name}")
        assert_close(got, p.oracle_apply(), w.dtype, f"noalloc vs the oracle on {name}")
        assert int(p.status.item()) == 0


def test_noalloc_repeated_call_same_bits_and_no_device_memory_taken():
    w = inputs.make("skewed_h4096")
    p = DeviceProblem(w, y_random=True)
    first = _noalloc(p)  # warm-up: the scratch address is looked up here
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    p.Y.copy_(to_dev(p.y_bits, w.dtype))  # same base output again
    torch.cuda.synchronize()
    free_mid, _ = torch.cuda.mem_get_info()
    second = _noalloc(p)
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_mid, (free_before, free_mid, free_after)
    assert np.array_equal(first, second)
    assert_close(second, p.oracle_apply(), w.dtype, "noalloc, second call on the same inputs")


def test_noalloc_refuses_problems_above_its_scratch():
    lib = sgmv.load()
    fake = 1 << 20  # never dereferenced: the size check comes first
    st = lib.lora_sgmv_apply_noalloc(fake, fake, fake, fake, fake, fake, 1, 1, 1 << 15, 4096, 64, 4096, 1.0,
                                     sgmv.F16, 1, None, None)
    assert st == 7  # LORA_SGMV_ERR_WORKSPACE
