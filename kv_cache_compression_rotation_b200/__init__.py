"""TurboQuant KV-cache compression hot path for NVIDIA B200 (sm_100a).

The compute lives in ``libtq.so`` (CUDA C++, C ABI in ``include/tq.h``); this package is
its thin Python binding.  See :mod:`kv_cache_compression_rotation_b200.tq`.
"""
from . import tq
from .tq import (KIND_MSE, KIND_PROD, KIND_SPECTRAL, Packed, Pages, Quantizer, Split, TqError, codebook_build,
                 decode_attn, decode_attn_paged, decode_attn_split, decode_workspace_bytes, dequantize, get_status,
                 prefill_attn, quantize, quantize_split, quantize_ws, tq_quantize_workspace_bytes, score, score_split, set_wait_limit, spectral_calibrate,
                 spectral_unit_codebooks, version, waterfill)

__all__ = [
    "tq", "Quantizer", "Packed", "TqError", "quantize", "dequantize", "score", "decode_attn",
    "decode_workspace_bytes", "codebook_build", "waterfill", "spectral_calibrate",
    "spectral_unit_codebooks", "get_status", "set_wait_limit", "version", "KIND_MSE", "KIND_PROD",
    "KIND_SPECTRAL", "Split", "quantize_split", "score_split", "decode_attn_split", "Pages",
    "decode_attn_paged", "prefill_attn", "quantize_ws",
]
