"""CPU oracle for SGMV -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA library never loads it, and
this package never loads the CUDA library: the two share nothing but the
seeded input generator.

The arithmetic lives in ``sgmv_oracle.c`` (plain C, no CUDA, no BLAS), built
with gcc into ``liboracle.so`` beside it. This wrapper only marshals numpy
arrays. See that file's header for what is computed and from which passage
of the Punica README page “Punica：多 LoRA 模型统一服务框架”.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import List, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sgmv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F16 = 0
BF16 = 1
_DT = {"f16": F16, "bf16": BF16}


def build(force: bool = False) -> str:
    """Compile sgmv_oracle.c with gcc (no fast-math, no FMA contraction)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-o", tmp, _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i32 = ctypes.c_int32
            lib.oracle_f16_to_double.restype = ctypes.c_double
            lib.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_bf16_to_double.restype = ctypes.c_double
            lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_double_to_f16.restype = ctypes.c_uint16
            lib.oracle_double_to_f16.argtypes = [ctypes.c_double]
            lib.oracle_double_to_bf16.restype = ctypes.c_uint16
            lib.oracle_double_to_bf16.argtypes = [ctypes.c_double]
            lib.oracle_decode_array.argtypes = [P, P, ctypes.c_int64, ctypes.c_int]
            lib.oracle_encode_array.argtypes = [P, P, ctypes.c_int64, ctypes.c_int]
            lib.oracle_group_segments.restype = ctypes.c_int
            lib.oracle_group_segments.argtypes = [P, i32, i32, P, P, P, P]
            lib.oracle_shrink_f32.restype = ctypes.c_int
            lib.oracle_shrink_f32.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, ctypes.c_int]
            lib.oracle_expand_f32.restype = ctypes.c_int
            lib.oracle_expand_f32.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, ctypes.c_float, ctypes.c_int]
            lib.oracle_apply_f32.restype = ctypes.c_int
            lib.oracle_apply_f32.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, ctypes.c_float, ctypes.c_int]
            lib.oracle_shrink_f64.restype = ctypes.c_int
            lib.oracle_shrink_f64.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, ctypes.c_int]
            lib.oracle_expand_f64.restype = ctypes.c_int
            lib.oracle_expand_f64.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, ctypes.c_double, ctypes.c_int]
            lib.oracle_apply_f64.restype = ctypes.c_int
            lib.oracle_apply_f64.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, ctypes.c_double, ctypes.c_int]
            lib.oracle_base_plus_delta_f32.restype = ctypes.c_int
            lib.oracle_base_plus_delta_f32.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32,
                                                       ctypes.c_float, ctypes.c_int]
            lib.oracle_apply_f32_element.restype = ctypes.c_uint16
            lib.oracle_apply_f32_element.argtypes = [P, P, P, ctypes.c_uint16, i32, i32, i32, i32, ctypes.c_float, ctypes.c_int]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


class _Table:
    """Host pointer table over a list of uint16 adapter matrices (keeps them alive)."""

    def __init__(self, mats: Sequence[np.ndarray]):
        self.mats = [_u16(m) for m in mats]
        self.ptrs = np.array([_ptr(m) for m in self.mats] or [0], dtype=np.uint64)

    @property
    def ptr(self) -> int:
        return _ptr(self.ptrs)


# -- conversions ---------------------------------------------------------------

def decode(bits: np.ndarray, dtype: str) -> np.ndarray:
    bits = _u16(bits)
    out = np.empty(bits.shape, dtype=np.float64)
    _load().oracle_decode_array(_ptr(bits), _ptr(out), bits.size, _DT[dtype])
    return out


def encode(values: np.ndarray, dtype: str) -> np.ndarray:
    values = np.ascontiguousarray(values, dtype=np.float64)
    out = np.empty(values.shape, dtype=np.uint16)
    _load().oracle_encode_array(_ptr(values), _ptr(out), values.size, _DT[dtype])
    return out


# -- bookkeeping -------------------------------------------------------------------

def group_segments(ids, num_adapters: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Returns (seg_starts[n+1], lora_idx[n], perm[T]) as int32 arrays."""
    ids = _i32(ids)
    T = ids.shape[0]
    seg = np.zeros(num_adapters + 1, dtype=np.int32)
    idx = np.zeros(max(num_adapters, 1), dtype=np.int32)
    perm = np.zeros(max(T, 1), dtype=np.int32)
    n = np.zeros(1, dtype=np.int32)
    rc = _load().oracle_group_segments(_ptr(ids), T, num_adapters, _ptr(seg), _ptr(idx), _ptr(perm), _ptr(n))
    if rc != 0:
        raise ValueError("adapter id out of range")
    k = int(n[0])
    return seg[: k + 1].copy(), idx[:k].copy(), perm[:T].copy()


# -- fp32-accumulate twin ---------------------------------------------------------

def shrink_f32(X, A: Sequence[np.ndarray], seg_starts, lora_idx, r: int, dtype: str,
               V_init: np.ndarray = None) -> Tuple[np.ndarray, int]:
    X = _u16(X)
    T, H1 = X.shape
    seg, idx = _i32(seg_starts), _i32(lora_idx)
    V = np.zeros((T, r), dtype=np.float32) if V_init is None else np.array(V_init, dtype=np.float32, copy=True)
    tab = _Table(A)
    sk = _load().oracle_shrink_f32(_ptr(V), _ptr(X), tab.ptr, _ptr(seg), _ptr(idx), idx.shape[0], len(A),
                                   T, H1, r, _DT[dtype])
    return V, sk


def expand_f32(Y, V, B: Sequence[np.ndarray], seg_starts, lora_idx, scale: float, dtype: str) -> Tuple[np.ndarray, int]:
    Y = np.array(_u16(Y), copy=True)
    V = np.ascontiguousarray(V, dtype=np.float32)
    T, H2 = Y.shape
    r = V.shape[1]
    seg, idx = _i32(seg_starts), _i32(lora_idx)
    tab = _Table(B)
    sk = _load().oracle_expand_f32(_ptr(Y), _ptr(V), tab.ptr, _ptr(seg), _ptr(idx), idx.shape[0], len(B),
                                   T, r, H2, float(scale), _DT[dtype])
    return Y, sk


def apply_f32(Y, X, A: Sequence[np.ndarray], B: Sequence[np.ndarray], seg_starts, lora_idx,
              scale: float, dtype: str) -> Tuple[np.ndarray, int]:
    Y = np.array(_u16(Y), copy=True)
    X = _u16(X)
    T, H1 = X.shape
    H2 = Y.shape[1]
    r = A[0].shape[1] if len(A) else 0
    seg, idx = _i32(seg_starts), _i32(lora_idx)
    ta, tb = _Table(A), _Table(B)
    sk = _load().oracle_apply_f32(_ptr(Y), _ptr(X), ta.ptr, tb.ptr, _ptr(seg), _ptr(idx), idx.shape[0],
                                  len(A), T, H1, r, H2, float(scale), _DT[dtype])
    return Y, sk


def apply_f32_element(x_row, Ai, Bi, y_in_bits: int, c: int, scale: float, dtype: str) -> int:
    x_row, Ai, Bi = _u16(x_row), _u16(Ai), _u16(Bi)
    H1, r = Ai.shape
    H2 = Bi.shape[1]
    return int(_load().oracle_apply_f32_element(_ptr(x_row), _ptr(Ai), _ptr(Bi), int(y_in_bits), H1, r, H2,
                                                int(c), float(scale), _DT[dtype]))


def base_plus_delta_f32(X, W, A: Sequence[np.ndarray], B: Sequence[np.ndarray], seg_starts, lora_idx,
                        scale: float, dtype: str) -> Tuple[np.ndarray, int]:
    """Y = round(X@W + scale * (X@A_i)@B_i) per row (round(X@W) for rows in no valid segment)."""
    X, W = _u16(X), _u16(W)
    T, H1 = X.shape
    H2 = W.shape[1]
    assert W.shape[0] == H1
    r = A[0].shape[1] if len(A) else 0
    Y = np.zeros((T, H2), dtype=np.uint16)
    seg, idx = _i32(seg_starts), _i32(lora_idx)
    ta, tb = _Table(A), _Table(B)
    sk = _load().oracle_base_plus_delta_f32(_ptr(Y), _ptr(X), _ptr(W), ta.ptr, tb.ptr, _ptr(seg), _ptr(idx),
                                            idx.shape[0], len(A), T, H1, r, H2, float(scale), _DT[dtype])
    return Y, sk


# -- binary64 twin ------------------------------------------------------------------

def shrink_f64(X, A: Sequence[np.ndarray], seg_starts, lora_idx, r: int, dtype: str) -> Tuple[np.ndarray, int]:
    X = _u16(X)
    T, H1 = X.shape
    seg, idx = _i32(seg_starts), _i32(lora_idx)
    V = np.zeros((T, r), dtype=np.float64)
    tab = _Table(A)
    sk = _load().oracle_shrink_f64(_ptr(V), _ptr(X), tab.ptr, _ptr(seg), _ptr(idx), idx.shape[0], len(A),
                                   T, H1, r, _DT[dtype])
    return V, sk


def expand_f64(Y, V, B: Sequence[np.ndarray], seg_starts, lora_idx, scale: float, dtype: str) -> Tuple[np.ndarray, int]:
    Y = np.array(Y, dtype=np.float64, copy=True)
    V = np.ascontiguousarray(V, dtype=np.float64)
    T, H2 = Y.shape
    r = V.shape[1]
    seg, idx = _i32(seg_starts), _i32(lora_idx)
    tab = _Table(B)
    sk = _load().oracle_expand_f64(_ptr(Y), _ptr(V), tab.ptr, _ptr(seg), _ptr(idx), idx.shape[0], len(B),
                                   T, r, H2, float(scale), _DT[dtype])
    return Y, sk


def apply_f64(Y, X, A: Sequence[np.ndarray], B: Sequence[np.ndarray], seg_starts, lora_idx,
              scale: float, dtype: str) -> Tuple[np.ndarray, int]:
    """Y is a binary64 array (in/out copy); returns the unrounded result."""
    Y = np.array(Y, dtype=np.float64, copy=True)
    X = _u16(X)
    T, H1 = X.shape
    H2 = Y.shape[1]
    r = A[0].shape[1] if len(A) else 0
    seg, idx = _i32(seg_starts), _i32(lora_idx)
    ta, tb = _Table(A), _Table(B)
    sk = _load().oracle_apply_f64(_ptr(Y), _ptr(X), ta.ptr, tb.ptr, _ptr(seg), _ptr(idx), idx.shape[0],
                                  len(A), T, H1, r, H2, float(scale), _DT[dtype])
    return Y, sk
