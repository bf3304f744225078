"""Seeded synthetic SGMV workloads.

This module only draws random inputs. It holds none of the method's
arithmetic: no segment grouping, no products, no rounding other than the
storage cast of freshly drawn normals. Both the CUDA path (through the tests
and ``bench.py``) and the CPU oracle take their inputs from here.

Workloads follow the adapter-popularity distributions named in the Punica
README page ("Punica：多 LoRA 模型统一服务框架", text-generation benchmark
paragraph): Distinct (every request its own adapter), Identical (all
requests on one adapter), Uniform and Skewed (in between). The shapes are the
LoRA shapes of the README's LoRA paragraph: ``A`` is ``[H1, r]``, ``B`` is
``[r, H2]``, rows are tokens.

Random streams. Every array is drawn from its own PCG64 stream keyed by
``(seed, tag[, adapter id])``. A pool of 1024 adapters can therefore be
materialised lazily (only the adapters a batch touches), and any subset of
arrays is reproducible without drawing the rest. Normals are drawn in fp32
and cast once, round-to-nearest-even, to the storage type.

Storage values are returned as ``numpy.uint16`` bit patterns (fp16 or bf16),
so that the two consumers see identical bits and neither depends on the
other's conversion code.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

F16 = "f16"
BF16 = "bf16"

_TAGS = {"ids": 1, "x": 2, "a": 3, "b": 4, "y": 5, "len": 6, "w": 7}


def _stream(seed: int, tag: str, index: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _TAGS[tag], index])))


def cast_f32_bits(values: np.ndarray, dtype: str) -> np.ndarray:
    """Cast fp32 draws to fp16/bf16 storage (RNE) and return the uint16 bits."""
    values = np.ascontiguousarray(values, dtype=np.float32)
    if dtype == F16:
        return values.astype(np.float16).view(np.uint16)
    if dtype == BF16:
        import torch  # CPU cast only; torch rounds fp32 -> bf16 to nearest even

        t = torch.from_numpy(values).to(torch.bfloat16)
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    raise ValueError(f"unknown dtype {dtype!r}")


def _normal_bits(rng: np.random.Generator, shape, std: float, dtype: str) -> np.ndarray:
    v = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        v *= np.float32(std)
    return cast_f32_bits(v, dtype)


def zipf_ids(rng: np.random.Generator, n: int, num_adapters: int, s: float) -> np.ndarray:
    """Truncated Zipf over ranks 1..num_adapters, p_k proportional to k^-s.

    Rank k maps to adapter id k-1. Drawn by inverse CDF from uniform draws.
    """
    k = np.arange(1, num_adapters + 1, dtype=np.float64)
    p = k ** (-s)
    cdf = np.cumsum(p)
    cdf /= cdf[-1]
    u = rng.random(n)
    ids = np.searchsorted(cdf, u, side="right")
    return np.minimum(ids, num_adapters - 1).astype(np.int32)


@dataclasses.dataclass
class Workload:
    """One SGMV problem: a batch of tokens, per-token adapter ids, an adapter pool.

    ``ids`` is in arrival order. The batch that the kernels and the oracle see
    is the batch after grouping (tokens of one adapter contiguous); the
    generator draws the rows of ``X`` and ``Y`` for that grouped batch directly,
    since every row is an independent draw.
    """

    name: str
    H1: int
    H2: int
    r: int
    dtype: str
    ids: np.ndarray  # int32 [T], arrival order
    num_adapters: int
    scale: float = 1.0
    seed: int = 0
    y_zero: bool = True
    projections: int = 1
    given_segments: Optional[List[int]] = None  # segment lengths when the config prints them
    given_lora_idx: Optional[List[int]] = None

    @property
    def T(self) -> int:
        return int(self.ids.shape[0])

    @property
    def elem_bytes(self) -> int:
        return 2

    def x(self, proj: int = 0) -> np.ndarray:
        return _normal_bits(_stream(self.seed, "x", proj), (self.T, self.H1), 1.0, self.dtype)

    def y0(self, proj: int = 0) -> np.ndarray:
        if self.y_zero:
            return np.zeros((self.T, self.H2), dtype=np.uint16)
        return _normal_bits(_stream(self.seed, "y", proj), (self.T, self.H2), 1.0, self.dtype)

    def y_random(self, proj: int = 0) -> np.ndarray:
        """A non-zero base output, N(0,1), used to exercise the in-place add."""
        return _normal_bits(_stream(self.seed, "y", proj), (self.T, self.H2), 1.0, self.dtype)

    def base_weight(self, proj: int = 0) -> np.ndarray:
        """The frozen base weight W of shape [H1, H2], entries N(0, 1/H1) (so X@W ~ N(0, 1))."""
        return _normal_bits(_stream(self.seed, "w", proj), (self.H1, self.H2), 1.0 / math.sqrt(self.H1), self.dtype)

    def adapter_a(self, i: int, proj: int = 0) -> np.ndarray:
        """A_i of shape [H1, r], entries N(0, 1/H1)."""
        rng = _stream(self.seed, "a", proj * 1_000_003 + i)
        return _normal_bits(rng, (self.H1, self.r), 1.0 / math.sqrt(self.H1), self.dtype)

    def adapter_b(self, i: int, proj: int = 0) -> np.ndarray:
        """B_i of shape [r, H2], entries N(0, 1/r)."""
        rng = _stream(self.seed, "b", proj * 1_000_003 + i)
        return _normal_bits(rng, (self.r, self.H2), 1.0 / math.sqrt(self.r), self.dtype)

    def touched_adapters(self) -> List[int]:
        return sorted(set(int(v) for v in self.ids))

    def sorted_ids(self) -> np.ndarray:
        """Adapter id of each row of the grouped batch (ascending, stable)."""
        return np.sort(self.ids, kind="stable")

    def algorithmic_bytes(self) -> int:
        """Unique adapter bytes + X read + Y read and write, per projection."""
        U = len(self.touched_adapters())
        e = self.elem_bytes
        return U * (self.H1 * self.r + self.r * self.H2) * e + self.T * self.H1 * e + 2 * self.T * self.H2 * e

    def flops(self) -> int:
        return 2 * self.T * self.r * (self.H1 + self.H2)


def tiny(seed: int = 0) -> Workload:
    """H1=H2=256, r=8, 4 adapters, 8 tokens in segments [1,3,2,2] on adapters [0,1,2,3], fp16, Y=0."""
    lens = [1, 3, 2, 2]
    ids = np.repeat(np.arange(4, dtype=np.int32), lens)
    return Workload("tiny", 256, 256, 8, F16, ids, 4, 1.0, seed, True, 1, lens, [0, 1, 2, 3])


def distinct(seed: int = 0, projections: int = 4) -> Workload:
    """Llama-7B decode, Distinct: 32 tokens, each its own adapter, H1=H2=4096, r=16, fp16."""
    ids = np.arange(32, dtype=np.int32)
    return Workload("distinct", 4096, 4096, 16, F16, ids, 32, 1.0, seed, True, projections)


def uniform(H2: int = 4096, seed: int = 0) -> Workload:
    """64 single-token requests, ids uniform over 16 adapters, H1=4096, r=16, fp16."""
    ids = _stream(seed, "ids").integers(0, 16, size=64).astype(np.int32)
    return Workload(f"uniform_h{H2}", 4096, H2, 16, F16, ids, 16, 1.0, seed)


def skewed(H2: int = 4096, seed: int = 0) -> Workload:
    """64 single-token requests, ids Zipf(s=1.5) over 64 adapters, H1=4096, r=16, fp16."""
    ids = zipf_ids(_stream(seed, "ids"), 64, 64, 1.5)
    return Workload(f"skewed_h{H2}", 4096, H2, 16, F16, ids, 64, 1.0, seed)


def identical(H2: int = 4096, seed: int = 0) -> Workload:
    """64 single-token requests all on adapter 0, H1=4096, r=16, fp16."""
    ids = np.zeros(64, dtype=np.int32)
    return Workload(f"identical_h{H2}", 4096, H2, 16, F16, ids, 1, 1.0, seed)


def prefill(seed: int = 0) -> Workload:
    """8 prompt segments, lengths uniform in 128..2048, adapter s for segment s, H1=H2=4096, r=64, bf16."""
    lens = _stream(seed, "len").integers(128, 2049, size=8)
    ids = np.repeat(np.arange(8, dtype=np.int32), lens)
    return Workload("prefill", 4096, 4096, 64, BF16, ids, 8, 1.0, seed, True, 1,
                    [int(v) for v in lens], list(range(8)))


def llama70b_decode(H2: int = 28672, seed: int = 0) -> Workload:
    """256 single-token requests, ids Zipf(s=1.2) over a resident pool of 1024, H1=8192, r=64, bf16."""
    ids = zipf_ids(_stream(seed, "ids"), 256, 1024, 1.2)
    return Workload(f"llama70b_decode_h{H2}", 8192, H2, 64, BF16, ids, 1024, 1.0, seed)


def small_random(T: int, n_adapters: int, H1: int, H2: int, r: int, dtype: str, seed: int,
                 y_zero: bool = False) -> Workload:
    """Small ragged case for parity sweeps: uniform ids, arbitrary shapes."""
    ids = _stream(seed, "ids").integers(0, n_adapters, size=T).astype(np.int32)
    return Workload(f"random_t{T}_a{n_adapters}_{H1}x{r}x{H2}_{dtype}", H1, H2, r, dtype, ids,
                    n_adapters, 1.0, seed, y_zero)


CONFIGS: Dict[str, callable] = {
    "tiny": tiny,
    "distinct": distinct,
    "uniform_h4096": lambda seed=0: uniform(4096, seed),
    "uniform_h11008": lambda seed=0: uniform(11008, seed),
    "skewed_h4096": lambda seed=0: skewed(4096, seed),
    "skewed_h11008": lambda seed=0: skewed(11008, seed),
    "identical_h4096": lambda seed=0: identical(4096, seed),
    "identical_h11008": lambda seed=0: identical(11008, seed),
    "prefill": prefill,
    "llama70b_decode_h28672": lambda seed=0: llama70b_decode(28672, seed),
    "llama70b_decode_h8192": lambda seed=0: llama70b_decode(8192, seed),
}


def make(name: str, seed: int = 0) -> Workload:
    return CONFIGS[name](seed=seed)
