"""B200 (sm_100a) dense attention forward: O = softmax(scale Q K^T [causal]) V.

Thin Python binding over the C ABI in ``include/attn_b200.h``: it marshals
torch tensors into pointers and sizes and raises on a non-zero status.  Every
step of the computation runs in the CUDA kernels of ``libattn_b200.so``;
there is no CPU or PyTorch fallback: without the library or an sm_100 device
the calls raise.
"""
from __future__ import annotations

from ._abi import (ATTN_OK, AttnError, AttnOpts, attn_combine, attn_fwd, attn_fwd_chunk,
                   attn_fwd_fp4, attn_fwd_fp8, attn_fwd_pair, attn_fwd_pair_into,
                   attn_fwd_chunk_into, attn_fwd_host, attn_fwd_into, attn_fwd_noalloc_into,
                   attn_fwd_splitkv, attn_fwd_varlen, check_args, kmeans_assign,
                   last_device_error, library, library_path, quantize_e4m3, quantize_nvfp4,
                   selftest_wait_timeout, splitkv_slices, strerror)

__all__ = ["ATTN_OK", "AttnError", "AttnOpts", "attn_combine", "attn_fwd", "attn_fwd_chunk",
           "attn_fwd_fp4", "attn_fwd_fp8", "attn_fwd_pair", "attn_fwd_pair_into",
           "attn_fwd_chunk_into", "attn_fwd_host", "attn_fwd_into", "attn_fwd_noalloc_into",
           "attn_fwd_splitkv", "attn_fwd_varlen", "check_args", "kmeans_assign",
           "last_device_error", "library", "quantize_e4m3", "quantize_nvfp4",
           "library_path", "selftest_wait_timeout", "splitkv_slices", "strerror"]
