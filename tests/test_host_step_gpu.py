"""lora_sgmv_step_host: one serving step from pinned host memory (grouping on the host, the
copies in, the batched launch, the copies out) against the oracle, against the same launch
from device buffers, and step after step on alternating streams."""
import numpy as np
import pytest
import torch

import oracle
from adapter_matmul_b200 import inputs, sgmv
from gpu_helpers import DeviceProblem, assert_close, dt_code, from_dev

pytestmark = pytest.mark.gpu


def _pinned(nbytes: int) -> torch.Tensor:
    return torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)


class HostBatch:
    """Pinned host buffer [meta | X_0 | Y_0 | X_1 | Y_1 ...], its device mirror, and the step."""

    def __init__(self, ids, shapes, r, dtype, num_adapters, seed=0):
        self.T = len(ids)
        self.ids = np.ascontiguousarray(ids, np.int32)
        self.probs, self.refs = [], []
        for k, (H1, H2) in enumerate(shapes):
            w = inputs.Workload(f"hs{k}", H1, H2, r, dtype, self.ids, num_adapters, 0.75 - 0.25 * k, seed=seed + k)
            p = DeviceProblem(w, y_random=True)
            self.probs.append(p)
            self.refs.append(p.oracle_apply())
        meta_bytes = ((2 * num_adapters + 1) * 4 + 255) // 256 * 256
        offs, off = [], meta_bytes
        for p in self.probs:
            xb, yb = p.x_bits.nbytes, p.y_bits.nbytes
            offs.append((off, off + xb, yb))
            off += xb + yb
        self.h = _pinned(off)
        self.d = torch.empty(off, dtype=torch.uint8, device="cuda")
        hn = self.h.numpy()
        for p, (xo, yo, yb) in zip(self.probs, offs):
            hn[xo:xo + p.x_bits.nbytes] = np.ascontiguousarray(p.x_bits).view(np.uint8).reshape(-1)
            hn[yo:yo + yb] = np.ascontiguousarray(p.y_bits).view(np.uint8).reshape(-1)
        self.outs = [_pinned(yb) for (_, _, yb) in offs]
        hb, db = self.h.data_ptr(), self.d.data_ptr()
        problems = [sgmv.Problem(db + yo, db + xo, p.A_ptrs.data_ptr(), p.B_ptrs.data_ptr(), num_adapters,
                                 p.w.H1, p.w.H2, p.w.scale) for p, (xo, yo, _) in zip(self.probs, offs)]
        self.meta = hn[:meta_bytes].view(np.int32)
        self.perm = np.empty(max(self.T, 1), np.int32)
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.step = sgmv.HostStep(self.ids, self.T, num_adapters, hb, db, [(hb, db, off)], problems, r, dt_code(dtype),
                                  [(db + yo, o.data_ptr(), yb) for (_, yo, yb), o in zip(offs, self.outs)],
                                  perm=self.perm, dev_status=self.status)

    def out(self, k: int) -> np.ndarray:
        p = self.probs[k]
        return self.outs[k].numpy().view(np.uint16).reshape(p.y_bits.shape).copy()


@pytest.mark.parametrize("r,dtype,name", [(16, "f16", "distinct"), (64, "bf16", "llama70b")])
def test_host_step_matches_the_oracle(r, dtype, name):
    ids = inputs.distinct().ids if name == "distinct" else inputs.llama70b_decode(8192).ids[:96]
    na = 64 if name == "distinct" else 1024
    hb = HostBatch(ids, [(1024, 1024), (1024, 512), (512, 768)], r, dtype, na, seed=3)
    s = torch.cuda.Stream()
    n = hb.step.run(s)
    s.synchronize()
    p0 = hb.probs[0]
    # the grouping written to the pinned metadata and perm is lora_sgmv_group_segments' (and the oracle's)
    seg, idx, perm = oracle.group_segments(hb.ids, na)
    assert n == p0.n == len(idx)
    assert np.array_equal(hb.meta[:n + 1], seg) and np.array_equal(hb.meta[n + 1:2 * n + 1], idx)
    assert np.array_equal(hb.perm[:hb.T], perm)
    for k, ref in enumerate(hb.refs):
        assert_close(hb.out(k), ref, dtype, f"step_host problem {k}")
    assert int(hb.status.item()) == 0


def test_host_step_equals_the_device_launch_and_repeats():
    # the same launch from device buffers gives the same bits; steps on alternating streams
    # (each re-copying the host X and Y) give the same bits every time
    ids = inputs.skewed(4096).ids[:48]
    hb = HostBatch(ids, [(1024, 2048), (2048, 1024)], 16, "f16", 64, seed=11)
    p0 = hb.probs[0]
    sgmv.lora_sgmv_apply_batched(
        [dict(Y=p.Y, X=p.X, A_ptrs=p.A_ptrs, B_ptrs=p.B_ptrs, num_adapters=p.w.num_adapters, H1=p.w.H1,
              H2=p.w.H2, scale=p.w.scale) for p in hb.probs],
        p0.d_seg, p0.d_idx, p0.n, p0.w.T, 16, sgmv.F16, p0.max_len(), p0.status)
    torch.cuda.synchronize()
    dev = [from_dev(p.Y) for p in hb.probs]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for i in range(4):
        s = streams[i % 2]
        hb.step.run(s)
        s.synchronize()
        got = [hb.out(k) for k in range(len(hb.probs))]
        for k in range(len(got)):
            assert np.array_equal(got[k], dev[k]), f"step {i} problem {k} differs from the device launch"
    assert int(hb.status.item()) == 0 and int(p0.status.item()) == 0


def test_host_step_rejects_an_out_of_range_id_before_anything_runs():
    ids = inputs.distinct().ids.copy()
    hb = HostBatch(ids, [(512, 512)], 16, "f16", 64, seed=5)
    hb.ids[3] = 64  # == num_adapters
    before = hb.outs[0].numpy().copy()
    with pytest.raises(sgmv.SGMVError, match="ERR_RANGE"):
        hb.step.run(torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert np.array_equal(hb.outs[0].numpy(), before)


def test_host_step_with_an_empty_batch_only_copies():
    # T = 0: no segment and no launch; the copies still run in order
    import ctypes
    lib = sgmv.load()
    meta = torch.empty(64, dtype=torch.int32, pin_memory=True)
    dmeta = torch.zeros(64, dtype=torch.int32, device="cuda")
    src = torch.arange(256, dtype=torch.uint8).pin_memory()
    dst = torch.zeros(256, dtype=torch.uint8, device="cuda")
    back = torch.zeros(256, dtype=torch.uint8, pin_memory=True)
    h2d = (sgmv.Copy * 1)(sgmv.Copy(src.data_ptr(), dst.data_ptr(), 256))
    d2h = (sgmv.Copy * 1)(sgmv.Copy(dst.data_ptr(), back.data_ptr(), 256))
    probs = (sgmv.Problem * 1)(sgmv.Problem(dst.data_ptr(), dst.data_ptr(), dmeta.data_ptr(), dmeta.data_ptr(), 4,
                                            64, 64, 1.0))
    n = ctypes.c_int32(-1)
    s = torch.cuda.Stream()
    st = lib.lora_sgmv_step_host(None, 0, 4, meta.data_ptr(), dmeta.data_ptr(), None, ctypes.addressof(h2d), 1,
                                 ctypes.addressof(probs), 1, 16, sgmv.F16, 0, ctypes.addressof(d2h), 1, None,
                                 ctypes.addressof(n), s.cuda_stream)
    s.synchronize()
    assert st == 0 and n.value == 0
    assert int(meta[0]) == 0
    assert torch.equal(back, src)
