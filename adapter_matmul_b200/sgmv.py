"""Thin Python binding of the SGMV C ABI (include/lora_sgmv.h).

Argument marshalling only: every function here converts its arguments to
plain pointers and integers and calls the entry point of the same name in
libsgmv_b200.so. Every step of the computation runs in that library's CUDA
kernels (or, for lora_sgmv_group_segments, its host C++). There is no Python
or CPU fallback: if the library cannot be loaded, every call raises.

Pointers may be given as integers or as torch tensors (their data_ptr() is
taken). Streams may be given as a torch.cuda.Stream, an integer handle, or
None for torch's current stream on the current device.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsgmv_b200.so")

F16 = 0
BF16 = 1
VARIANT_AUTO = 0
VARIANT_SPLIT = 1
VARIANT_GROUPED_TC = 2
VARIANT_FUSED = 3
VARIANT_FUSED_TC = 4
VARIANT_SPLIT_TC = 5
MAX_PROBLEMS = 8

DEV_BAD_SEGMENT = 0x1
DEV_BAD_ADAPTER = 0x2
DEV_BAD_POINTER = 0x4
DEV_TIMEOUT = 0x8
DEV_BAD_RANK = 0x10

FLAG_EARLY_READS = 0x1

STATUS_NAMES = {0: "OK", 1: "ERR_NULL", 2: "ERR_DIM", 3: "ERR_ALIGN", 4: "ERR_DTYPE", 5: "ERR_UNSUPPORTED",
                6: "ERR_CUDA", 7: "ERR_WORKSPACE", 8: "ERR_RANGE"}

EXPORTS = [
    "lora_sgmv_rank_supported", "lora_sgmv_status_string", "lora_sgmv_version", "lora_sgmv_launch_count",
    "lora_sgmv_last_error",
    "lora_sgmv_group_segments", "lora_sgmv_shrink", "lora_sgmv_expand", "lora_sgmv_workspace_bytes",
    "lora_sgmv_apply", "lora_sgmv_apply_ex", "lora_sgmv_apply_batched", "lora_sgmv_apply_noalloc",
    "lora_sgmv_pad_rank", "lora_sgmv_auto_variant", "lora_sgmv_apply_flags", "lora_sgmv_apply_batched_flags",
    "lora_sgmv_gemm_apply", "lora_sgmv_apply_ranks", "lora_sgmv_step_host",
]


class Problem(ctypes.Structure):
    """Mirror of lora_sgmv_problem."""
    _fields_ = [("Y", ctypes.c_void_p), ("X", ctypes.c_void_p), ("A_ptrs", ctypes.c_void_p),
                ("B_ptrs", ctypes.c_void_p), ("num_adapters", ctypes.c_int32), ("H1", ctypes.c_int32),
                ("H2", ctypes.c_int32), ("scale", ctypes.c_float)]


class Copy(ctypes.Structure):
    """Mirror of lora_sgmv_copy."""
    _fields_ = [("src", ctypes.c_void_p), ("dst", ctypes.c_void_p), ("bytes", ctypes.c_size_t)]


_lock = threading.Lock()
_lib = None


class SGMVError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = status_string(status)
        if status == 6:
            detail += ": " + load().lora_sgmv_last_error().decode()
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({detail})")


def load(path: Optional[str] = None):
    """Load the library (building it in-tree first if it is missing and nvcc exists)."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            from . import build as _build

            if not os.path.exists(_build.NVCC):
                raise RuntimeError(f"SGMV CUDA library not found at {p} and nvcc is unavailable")
            _build.build()
        lib = ctypes.CDLL(p)
        P, i32, u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        lib.lora_sgmv_rank_supported.restype = i32
        lib.lora_sgmv_rank_supported.argtypes = [i32, ctypes.c_int]
        lib.lora_sgmv_status_string.restype = ctypes.c_char_p
        lib.lora_sgmv_status_string.argtypes = [ctypes.c_int]
        lib.lora_sgmv_version.restype = i32
        lib.lora_sgmv_version.argtypes = []
        lib.lora_sgmv_last_error.restype = ctypes.c_char_p
        lib.lora_sgmv_last_error.argtypes = []
        lib.lora_sgmv_launch_count.restype = ctypes.c_uint64
        lib.lora_sgmv_launch_count.argtypes = []
        lib.lora_sgmv_group_segments.restype = ctypes.c_int
        lib.lora_sgmv_group_segments.argtypes = [P, i32, i32, P, P, P, P]
        lib.lora_sgmv_shrink.restype = ctypes.c_int
        lib.lora_sgmv_shrink.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, ctypes.c_int, P, P]
        lib.lora_sgmv_expand.restype = ctypes.c_int
        lib.lora_sgmv_expand.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, ctypes.c_float, ctypes.c_int, P, P]
        lib.lora_sgmv_workspace_bytes.restype = u64
        lib.lora_sgmv_workspace_bytes.argtypes = [i32, i32]
        lib.lora_sgmv_apply.restype = ctypes.c_int
        lib.lora_sgmv_apply.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, ctypes.c_float,
                                        ctypes.c_int, i32, P, u64, P, P]
        lib.lora_sgmv_apply_ex.restype = ctypes.c_int
        lib.lora_sgmv_apply_ex.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, ctypes.c_float,
                                           ctypes.c_int, i32, P, u64, P, ctypes.c_int, P]
        lib.lora_sgmv_apply_flags.restype = ctypes.c_int
        lib.lora_sgmv_apply_flags.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, ctypes.c_float,
                                              ctypes.c_int, i32, P, u64, P, ctypes.c_int, ctypes.c_uint32, P]
        lib.lora_sgmv_apply_batched_flags.restype = ctypes.c_int
        lib.lora_sgmv_apply_batched_flags.argtypes = [P, i32, P, P, i32, i32, i32, ctypes.c_int, i32,
                                                      ctypes.c_uint32, P, P]
        lib.lora_sgmv_apply_ranks.restype = ctypes.c_int
        lib.lora_sgmv_apply_ranks.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, ctypes.c_float,
                                              ctypes.c_int, P, P]
        lib.lora_sgmv_gemm_apply.restype = ctypes.c_int
        lib.lora_sgmv_gemm_apply.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, ctypes.c_float,
                                             ctypes.c_int, i32, P, u64, P, P]
        lib.lora_sgmv_apply_batched.restype = ctypes.c_int
        lib.lora_sgmv_apply_batched.argtypes = [P, i32, P, P, i32, i32, i32, ctypes.c_int, i32, P, P]
        lib.lora_sgmv_apply_noalloc.restype = ctypes.c_int
        lib.lora_sgmv_apply_noalloc.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, ctypes.c_float,
                                                ctypes.c_int, i32, P, P]
        lib.lora_sgmv_auto_variant.restype = ctypes.c_int
        lib.lora_sgmv_auto_variant.argtypes = [i32, i32, i32, i32, i32, ctypes.c_int, i32, i32]
        lib.lora_sgmv_pad_rank.restype = ctypes.c_int
        lib.lora_sgmv_pad_rank.argtypes = [P, P, P, P, i32, i32, i32, i32, ctypes.c_int, P]
        lib.lora_sgmv_step_host.restype = ctypes.c_int
        lib.lora_sgmv_step_host.argtypes = [P, i32, i32, P, P, P, P, i32, P, i32, i32, ctypes.c_int,
                                            ctypes.c_uint32, P, i32, P, P, P]
        if path is None:
            _lib = lib
        return lib


def _p(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):  # numpy host array
        return x.ctypes.data
    raise TypeError(f"cannot take a pointer from {type(x)}")


def _stream(s) -> Optional[int]:
    if s is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(st: int, where: str) -> None:
    if st != 0:
        raise SGMVError(st, where)


def status_string(st: int) -> str:
    return load().lora_sgmv_status_string(st).decode()


def lora_sgmv_version() -> int:
    return load().lora_sgmv_version()


def lora_sgmv_launch_count() -> int:
    return int(load().lora_sgmv_launch_count())


def lora_sgmv_rank_supported(r: int, variant: int = VARIANT_AUTO) -> bool:
    return bool(load().lora_sgmv_rank_supported(r, variant))


def lora_sgmv_workspace_bytes(T: int, r: int) -> int:
    return int(load().lora_sgmv_workspace_bytes(T, r))


def lora_sgmv_group_segments(ids, num_adapters: int):
    """Host bookkeeping. ids: int32 numpy array. Returns (seg_starts, lora_idx, perm) numpy arrays."""
    import numpy as np

    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T = ids.shape[0]
    seg = np.zeros(num_adapters + 1, np.int32)
    idx = np.zeros(max(num_adapters, 1), np.int32)
    perm = np.zeros(max(T, 1), np.int32)
    n = np.zeros(1, np.int32)
    _check(load().lora_sgmv_group_segments(_p(ids), T, num_adapters, _p(seg), _p(idx), _p(perm), _p(n)),
           "lora_sgmv_group_segments")
    k = int(n[0])
    return seg[: k + 1].copy(), idx[:k].copy(), perm[:T].copy()


def lora_sgmv_shrink(V, X, A_ptrs, seg_starts, lora_idx, n_segments: int, num_adapters: int, T: int, H1: int,
                     r: int, dtype: int, dev_status=None, stream=None) -> None:
    _check(load().lora_sgmv_shrink(_p(V), _p(X), _p(A_ptrs), _p(seg_starts), _p(lora_idx), n_segments,
                                   num_adapters, T, H1, r, dtype, _p(dev_status), _stream(stream)),
           "lora_sgmv_shrink")


def lora_sgmv_expand(Y, V, B_ptrs, seg_starts, lora_idx, n_segments: int, num_adapters: int, T: int, r: int,
                     H2: int, scale: float, dtype: int, dev_status=None, stream=None) -> None:
    _check(load().lora_sgmv_expand(_p(Y), _p(V), _p(B_ptrs), _p(seg_starts), _p(lora_idx), n_segments,
                                   num_adapters, T, r, H2, float(scale), dtype, _p(dev_status), _stream(stream)),
           "lora_sgmv_expand")


def lora_sgmv_apply(Y, X, A_ptrs, B_ptrs, seg_starts, lora_idx, n_segments: int, num_adapters: int, T: int,
                    H1: int, r: int, H2: int, scale: float, dtype: int, max_seg_len: int, workspace,
                    workspace_bytes: int, dev_status=None, stream=None) -> None:
    _check(load().lora_sgmv_apply(_p(Y), _p(X), _p(A_ptrs), _p(B_ptrs), _p(seg_starts), _p(lora_idx),
                                  n_segments, num_adapters, T, H1, r, H2, float(scale), dtype, max_seg_len,
                                  _p(workspace), workspace_bytes, _p(dev_status), _stream(stream)),
           "lora_sgmv_apply")


def lora_sgmv_apply_ex(Y, X, A_ptrs, B_ptrs, seg_starts, lora_idx, n_segments: int, num_adapters: int, T: int,
                       H1: int, r: int, H2: int, scale: float, dtype: int, max_seg_len: int, workspace,
                       workspace_bytes: int, dev_status=None, variant: int = VARIANT_AUTO, stream=None) -> None:
    _check(load().lora_sgmv_apply_ex(_p(Y), _p(X), _p(A_ptrs), _p(B_ptrs), _p(seg_starts), _p(lora_idx),
                                     n_segments, num_adapters, T, H1, r, H2, float(scale), dtype, max_seg_len,
                                     _p(workspace), workspace_bytes, _p(dev_status), variant, _stream(stream)),
           "lora_sgmv_apply_ex")


def lora_sgmv_apply_flags(Y, X, A_ptrs, B_ptrs, seg_starts, lora_idx, n_segments: int, num_adapters: int, T: int,
                          H1: int, r: int, H2: int, scale: float, dtype: int, max_seg_len: int, workspace,
                          workspace_bytes: int, dev_status=None, variant: int = VARIANT_AUTO, flags: int = 0,
                          stream=None) -> None:
    _check(load().lora_sgmv_apply_flags(_p(Y), _p(X), _p(A_ptrs), _p(B_ptrs), _p(seg_starts), _p(lora_idx),
                                        n_segments, num_adapters, T, H1, r, H2, float(scale), dtype, max_seg_len,
                                        _p(workspace), workspace_bytes, _p(dev_status), variant, flags,
                                        _stream(stream)),
           "lora_sgmv_apply_flags")


def _problem_array(problems):
    arr = (Problem * max(1, len(problems)))()
    for i, q in enumerate(problems):
        if isinstance(q, Problem):
            arr[i] = q
        else:
            arr[i] = Problem(_p(q["Y"]), _p(q["X"]), _p(q["A_ptrs"]), _p(q["B_ptrs"]), int(q["num_adapters"]),
                             int(q["H1"]), int(q["H2"]), float(q.get("scale", 1.0)))
    return arr


def lora_sgmv_apply_batched(problems, seg_starts, lora_idx, n_segments: int, T: int, r: int, dtype: int,
                            max_seg_len: int, dev_status=None, stream=None) -> None:
    """problems: sequence of dicts (Y, X, A_ptrs, B_ptrs, num_adapters, H1, H2, scale) or Problem structs."""
    arr = _problem_array(problems)
    _check(load().lora_sgmv_apply_batched(ctypes.addressof(arr), len(problems), _p(seg_starts), _p(lora_idx),
                                          n_segments, T, r, dtype, max_seg_len, _p(dev_status), _stream(stream)),
           "lora_sgmv_apply_batched")


def lora_sgmv_apply_batched_flags(problems, seg_starts, lora_idx, n_segments: int, T: int, r: int, dtype: int,
                                  max_seg_len: int, flags: int = 0, dev_status=None, stream=None) -> None:
    arr = _problem_array(problems)
    _check(load().lora_sgmv_apply_batched_flags(ctypes.addressof(arr), len(problems), _p(seg_starts),
                                                _p(lora_idx), n_segments, T, r, dtype, max_seg_len, flags,
                                                _p(dev_status), _stream(stream)),
           "lora_sgmv_apply_batched_flags")


def lora_sgmv_apply_noalloc(Y, X, A_ptrs, B_ptrs, seg_starts, lora_idx, n_segments: int, num_adapters: int,
                            T: int, H1: int, r: int, H2: int, scale: float, dtype: int, max_seg_len: int,
                            dev_status=None, stream=None) -> None:
    """lora_sgmv_apply without a workspace: for callers that cannot allocate device memory."""
    _check(load().lora_sgmv_apply_noalloc(_p(Y), _p(X), _p(A_ptrs), _p(B_ptrs), _p(seg_starts), _p(lora_idx),
                                          n_segments, num_adapters, T, H1, r, H2, float(scale), dtype, max_seg_len,
                                          _p(dev_status), _stream(stream)),
           "lora_sgmv_apply_noalloc")


def lora_sgmv_apply_ranks(Y, X, A_ptrs, B_ptrs, ranks, seg_starts, lora_idx, n_segments: int, num_adapters: int,
                          T: int, H1: int, r_max: int, H2: int, scale: float, dtype: int, dev_status=None,
                          stream=None) -> None:
    """SGMV over adapters of their own ranks (ranks: device int32 per adapter), unpadded."""
    _check(load().lora_sgmv_apply_ranks(_p(Y), _p(X), _p(A_ptrs), _p(B_ptrs), _p(ranks), _p(seg_starts),
                                        _p(lora_idx), n_segments, num_adapters, T, H1, r_max, H2, float(scale), dtype,
                                        _p(dev_status), _stream(stream)),
           "lora_sgmv_apply_ranks")


def lora_sgmv_gemm_apply(Y, X, W, A_ptrs, B_ptrs, seg_starts, lora_idx, n_segments: int, num_adapters: int, T: int,
                         H1: int, r: int, H2: int, scale: float, dtype: int, max_seg_len: int, workspace,
                         workspace_bytes: int, dev_status=None, stream=None) -> None:
    """The whole layer Y = X@W + scale * (X@A_i)@B_i (Y written, not read)."""
    _check(load().lora_sgmv_gemm_apply(_p(Y), _p(X), _p(W), _p(A_ptrs), _p(B_ptrs), _p(seg_starts), _p(lora_idx),
                                       n_segments, num_adapters, T, H1, r, H2, float(scale), dtype, max_seg_len,
                                       _p(workspace), workspace_bytes, _p(dev_status), _stream(stream)),
           "lora_sgmv_gemm_apply")


def lora_sgmv_auto_variant(T: int, n_segments: int, H1: int, r: int, H2: int, dtype: int, max_seg_len: int = 0,
                           sm_count: int = 148) -> int:
    """The variant lora_sgmv_apply (AUTO) runs for a call of these sizes (host only)."""
    return int(load().lora_sgmv_auto_variant(T, n_segments, H1, r, H2, dtype, max_seg_len, sm_count))


def lora_sgmv_pad_rank(A_dst, A_src, B_dst, B_src, H1: int, H2: int, r_src: int, r: int, dtype: int,
                       stream=None) -> None:
    """Pad one adapter of rank r_src with zeros to rank r (either pair may be None)."""
    _check(load().lora_sgmv_pad_rank(_p(A_dst), _p(A_src), _p(B_dst), _p(B_src), H1, H2, r_src, r, dtype,
                                     _stream(stream)),
           "lora_sgmv_pad_rank")


def pointer_table(tensors: Sequence, device=None):
    """Device int64 tensor holding the data pointers of `tensors` (plumbing for A_ptrs / B_ptrs)."""
    import torch

    ptrs = [t.data_ptr() for t in tensors]
    dev = device if device is not None else (tensors[0].device if tensors else "cuda")
    return torch.tensor(ptrs, dtype=torch.int64, device=dev)


class HostStep:
    """lora_sgmv_step_host with its arguments marshalled once: a serving loop calls run(stream)
    per step. ids_host, meta_host (pinned) and perm are host arrays (numpy, or pointers);
    meta_dev is device memory; h2d and d2h are sequences of (src, dst, bytes); problems as for
    lora_sgmv_apply_batched. The contents of ids_host are read at each run."""

    def __init__(self, ids_host, T: int, num_adapters: int, meta_host, meta_dev, h2d, problems, r: int,
                 dtype: int, d2h, flags: int = 0, perm=None, dev_status=None):
        self._lib = load()
        self._probs = _problem_array(problems)
        self._h2d = (Copy * max(1, len(h2d)))(*[Copy(_p(a), _p(b), int(n)) for a, b, n in h2d])
        self._d2h = (Copy * max(1, len(d2h)))(*[Copy(_p(a), _p(b), int(n)) for a, b, n in d2h])
        self._n = ctypes.c_int32(0)
        self._args = [_p(ids_host), int(T), int(num_adapters), _p(meta_host), _p(meta_dev), _p(perm),
                      ctypes.addressof(self._h2d), len(h2d), ctypes.addressof(self._probs), len(problems), int(r),
                      int(dtype), int(flags), ctypes.addressof(self._d2h), len(d2h), _p(dev_status),
                      ctypes.addressof(self._n)]
        self._fn = self._lib.lora_sgmv_step_host

    def run(self, stream) -> int:
        """Enqueue one step on `stream` (a cudaStream_t as int, or a torch stream); returns n."""
        st = self._fn(*self._args, _stream(stream))
        if st != 0:
            raise SGMVError(st, "lora_sgmv_step_host")
        return self._n.value
