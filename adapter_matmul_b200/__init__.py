"""SGMV (Punica multi-LoRA delta) for NVIDIA B200: C-ABI library, binding and workloads.

The compute lives in libsgmv_b200.so (CUDA for sm_100a); ``adapter_matmul_b200.sgmv``
binds it. ``adapter_matmul_b200.inputs`` draws seeded synthetic workloads.
Importing this package loads nothing; the library is loaded on first use.
"""
__all__ = ["inputs", "sgmv", "build"]
__version__ = "0.1.0"
