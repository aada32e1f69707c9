"""Batch-invariant decoder forward and LM-head logprob on B200 (sm_100a).

The compute path is libbi.so (hand-written CUDA, C ABI in include/bi.h); this
package only marshals arguments to it.  There is no CPU fallback: importing
the binding raises if the library is missing.
"""
from ._lib import (BiError, lib, MODE_BF16, MODE_LAYERCAST, MODE_FP32, VARIANT_INVARIANT, VARIANT_FAST, DTYPE_BF16,
                   DTYPE_F32, EPI_NONE, EPI_SWIGLU, EPI_ROPE_KV_APPEND, GU_INTERLEAVE, ATTN_CHUNK, VOCAB_CHUNK)

__all__ = ["BiError", "lib", "MODE_BF16", "MODE_LAYERCAST", "MODE_FP32", "VARIANT_INVARIANT", "VARIANT_FAST",
           "DTYPE_BF16", "DTYPE_F32", "EPI_NONE", "EPI_SWIGLU", "EPI_ROPE_KV_APPEND", "GU_INTERLEAVE", "ATTN_CHUNK",
           "VOCAB_CHUNK"]
