"""Device-side plumbing for the GPU tests: seeded workloads -> torch device buffers.

Only memory movement lives here; every computation under test runs in the
library's kernels through adapter_matmul_b200.sgmv, and every expected value
comes from the oracle on the same host bits.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from adapter_matmul_b200 import inputs, sgmv

TOL_ABS = 2e-2
TOL_REL = 1e-2


def to_dev(bits: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy())
    t = t.view(torch.float16 if dtype == "f16" else torch.bfloat16)
    return t.cuda()


def from_dev(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def decode(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Independent decode (numpy / torch), used to compare outputs."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dtype == "f16":
        return bits.view(np.float16).astype(np.float64)
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()


def dt_code(dtype: str) -> int:
    return sgmv.F16 if dtype == "f16" else sgmv.BF16


class DeviceProblem:
    """One workload on the device: X, Y, the touched adapters, pointer tables, segments."""

    def __init__(self, w: inputs.Workload, proj: int = 0, y_random: bool = False, adapters=None,
                 seg_starts=None, lora_idx=None):
        self.w = w
        if seg_starts is None:
            seg, idx, _ = sgmv.lora_sgmv_group_segments(w.ids, w.num_adapters)
            oseg, oidx, _ = oracle.group_segments(w.ids, w.num_adapters)
            assert np.array_equal(seg, oseg) and np.array_equal(idx, oidx)
        else:
            seg, idx = np.asarray(seg_starts, np.int32), np.asarray(lora_idx, np.int32)
        self.seg, self.idx = seg, idx
        self.x_bits = w.x(proj)
        self.y_bits = w.y_random(proj) if y_random else w.y0(proj)
        touched = sorted(set(int(i) for i in idx if 0 <= i < w.num_adapters)) if adapters is None else adapters
        self.A = {i: w.adapter_a(i, proj) for i in touched}
        self.B = {i: w.adapter_b(i, proj) for i in touched}
        self.dA = {i: to_dev(a, w.dtype) for i, a in self.A.items()}
        self.dB = {i: to_dev(b, w.dtype) for i, b in self.B.items()}
        ptr_a = [self.dA[i].data_ptr() if i in self.dA else 0 for i in range(w.num_adapters)]
        ptr_b = [self.dB[i].data_ptr() if i in self.dB else 0 for i in range(w.num_adapters)]
        self.A_ptrs = torch.tensor(ptr_a, dtype=torch.int64, device="cuda")
        self.B_ptrs = torch.tensor(ptr_b, dtype=torch.int64, device="cuda")
        self.X = to_dev(self.x_bits, w.dtype)
        self.Y = to_dev(self.y_bits, w.dtype)
        self.d_seg = torch.from_numpy(seg.astype(np.int32)).cuda()
        self.d_idx = torch.from_numpy(idx.astype(np.int32)).cuda() if len(idx) else torch.zeros(1, dtype=torch.int32,
                                                                                                 device="cuda")
        self.ws_bytes = sgmv.lora_sgmv_workspace_bytes(w.T, w.r)
        self.ws = torch.empty(max(self.ws_bytes, 256) // 4, dtype=torch.float32, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")

    @property
    def n(self) -> int:
        return int(len(self.idx))

    def max_len(self) -> int:
        return int(np.max(np.diff(self.seg))) if len(self.seg) > 1 else 0

    def apply(self, variant=sgmv.VARIANT_AUTO, scale=None, max_seg_len=None):
        w = self.w
        sgmv.lora_sgmv_apply_ex(self.Y, self.X, self.A_ptrs, self.B_ptrs, self.d_seg, self.d_idx, self.n,
                                w.num_adapters, w.T, w.H1, w.r, w.H2, w.scale if scale is None else scale,
                                dt_code(w.dtype), self.max_len() if max_seg_len is None else max_seg_len, self.ws,
                                self.ws_bytes, self.status, variant)
        torch.cuda.synchronize()
        return from_dev(self.Y)

    def oracle_apply(self, scale=None):
        w = self.w
        zA, zB = np.zeros((w.H1, w.r), np.uint16), np.zeros((w.r, w.H2), np.uint16)
        A = [self.A.get(i, zA) for i in range(w.num_adapters)]
        B = [self.B.get(i, zB) for i in range(w.num_adapters)]
        return oracle_apply_rows(self.y_bits, self.x_bits, A, B, self.seg, self.idx,
                                 w.scale if scale is None else scale, w.dtype)


def assert_close(got_bits, ref_bits, dtype, what=""):
    g, o = decode(got_bits, dtype), decode(ref_bits, dtype)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - o)
    bad = err > TOL_ABS + TOL_REL * np.abs(o)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance; first at {tuple(i)}: "
                             f"gpu={g[tuple(i)]} oracle={o[tuple(i)]}; max abs err {err.max():.3e}")
    return float(err.max())


def oracle_apply_rows(y_bits, x_bits, A, B, seg, idx, scale, dtype, threads=None):
    """The whole-batch oracle over all rows, run on row shares in threads (the C oracle
    releases the GIL): each thread takes rows [a, b) with the segments cut to that range.
    Rows are independent in the definition, so the stitched result is the oracle's own."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    from bench import rows_share

    T = y_bits.shape[0]
    seg = np.asarray(seg, np.int64)
    if len(seg) < 2 or seg[0] != 0 or seg[-1] != T or np.any(np.diff(seg) < 0):
        out, _ = oracle.apply_f32(y_bits, x_bits, A, B, seg, idx, scale, dtype)  # not a plain grouping
        return out
    n = max(1, min(threads or os.cpu_count() or 1, 64, T))
    bounds = [round(k * T / n) for k in range(n + 1)]
    out = np.array(y_bits, copy=True)

    def one(k):
        a, b = bounds[k], bounds[k + 1]
        if a == b:
            return
        sub_seg, sub_idx = rows_share(seg, idx, a, b)
        res, _ = oracle.apply_f32(y_bits[a:b], x_bits[a:b], A, B, sub_seg, sub_idx, scale, dtype)
        out[a:b] = res

    with ThreadPoolExecutor(n) as ex:
        list(ex.map(one, range(n)))
    return out
