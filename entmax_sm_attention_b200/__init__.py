"""Fused alpha-entmax attention for NVIDIA B200 (sm_100a).

The compute lives in ``libentmax_attn.so`` (CUDA kernels behind a C ABI declared
in ``include/entmax_attn.h``). ``entmax_sm_attention_b200.binding`` is a thin
ctypes layer over it. The library loads on first use and raises if the shared
object is missing: there is no fallback.
"""
from .workloads import WORKLOADS, Workload, make_inputs, make_kv_len  # noqa: F401

__all__ = ["WORKLOADS", "Workload", "make_inputs", "make_kv_len"]
