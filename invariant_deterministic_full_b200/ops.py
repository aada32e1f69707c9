"""Thin torch-tensor wrappers over the C ABI (argument marshalling only).

torch provides device memory and the current stream; every step of the
computation runs in libbi's kernels.
"""
import ctypes

import torch

from ._lib import (lib, check, EpiArgs, KvLayout, MODE_BF16, MODE_LAYERCAST, VARIANT_INVARIANT, DTYPE_BF16,
                   DTYPE_F32, EPI_NONE, EPI_SWIGLU, EPI_ROPE_KV_APPEND)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def act_dtype(mode):
    """Activation and KV-cache dtype: f32 in LayerCast and FP32 modes, bf16 in the bf16 mode."""
    return torch.bfloat16 if mode == MODE_BF16 else torch.float32


def gemm(x, w, epilogue=EPI_NONE, mode=MODE_BF16, variant=VARIANT_INVARIANT, out_dtype=None, out=None, n_full=0):
    """y = x . w^T (bi_gemm).  x: [M,K] bf16 (BF16 mode) or f32 (LayerCast); w: [N,K] bf16 (f32 in FP32 mode).
    n_full: rows of the whole matrix when w is a row shard of it (tensor parallelism), else 0."""
    M, K = x.shape
    N = w.shape[0]
    n_out = N // 2 if epilogue == EPI_SWIGLU else N
    if out is None:
        out = torch.empty(M, n_out, dtype=out_dtype or act_dtype(mode), device=x.device)
    ydt = DTYPE_F32 if out.dtype == torch.float32 else DTYPE_BF16
    wsb = lib.bi_gemm_workspace_size(M, N, K, mode, variant)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=x.device)
    check(lib.bi_gemm(_ptr(x), x.stride(0), _ptr(w), _ptr(out), out.stride(0), ydt, M, N, K, int(n_full), epilogue,
                      None, mode, variant, _ptr(ws), wsb, _stream()), "bi_gemm")
    return out


def gemm_rope_kv(x, w_qkv, rope, rope_max_pos, kv, layer, slot, pos, n_heads, q_out=None, n_full=0):
    """QKV projection with RoPE and the KV append in its epilogue (bi_gemm, BI_EPI_ROPE_KV_APPEND, bf16 mode).
    x: [M, H] bf16; w_qkv: one layer of the fused weight in the paired row order; kv: a KVCache.  Returns q."""
    M, K = x.shape
    N = w_qkv.shape[0]
    head_dim = kv.layout.head_dim
    if q_out is None:
        q_out = torch.empty(M, n_heads * head_dim, dtype=torch.bfloat16, device=x.device)
    ea = EpiArgs(_ptr(rope).value, int(rope_max_pos), _ptr(q_out).value, ctypes.pointer(kv.layout), int(layer),
                 _ptr(slot).value, _ptr(pos).value, int(n_heads))
    check(lib.bi_gemm(_ptr(x), x.stride(0), _ptr(w_qkv), None, 0, DTYPE_BF16, M, N, K, int(n_full),
                      EPI_ROPE_KV_APPEND, ctypes.byref(ea), MODE_BF16, VARIANT_INVARIANT, None, 0, _stream()),
          "bi_gemm")
    return q_out


def rmsnorm(x, gamma, eps, residual_in=None, residual_out=None, want_f32=False, mode=MODE_BF16):
    M, H = x.shape
    y = torch.empty_like(x)
    y32 = torch.empty(M, H, dtype=torch.float32, device=x.device) if want_f32 else None
    check(lib.bi_rmsnorm(_ptr(x), _ptr(residual_in), _ptr(residual_out), _ptr(gamma), _ptr(y), _ptr(y32), M, H,
                         float(eps), mode, _stream()), "bi_rmsnorm")
    return (y, y32) if want_f32 else y


def rope_table(max_pos, head_dim, theta, device="cuda"):
    t = torch.empty(max_pos * head_dim, dtype=torch.float32, device=device)
    check(lib.bi_rope_table_fill(_ptr(t), max_pos, head_dim, float(theta), _stream()), "bi_rope_table_fill")
    return t


class KVCache:
    """Caller-owned KV cache: [n_slots][n_layers][n_kv_heads][capacity][head_dim] for k and for v."""

    def __init__(self, n_slots, n_layers, n_kv_heads, capacity, head_dim, mode=MODE_BF16, device="cuda"):
        dt = act_dtype(mode)
        shape = (n_slots, n_layers, n_kv_heads, capacity, head_dim)
        self.k = torch.zeros(shape, dtype=dt, device=device)
        self.v = torch.zeros(shape, dtype=dt, device=device)
        self.mode = mode
        self.layout = KvLayout(self.k.data_ptr(), self.v.data_ptr(), n_slots, n_layers, n_kv_heads, capacity,
                               head_dim, DTYPE_BF16 if mode == MODE_BF16 else DTYPE_F32)


def rope_kv_append(qkv, rope, rope_max_pos, kv, layer, slot, pos, Hq, mode=MODE_BF16, qk_paired=False):
    T = qkv.shape[0]
    d = kv.layout.head_dim
    q = torch.empty(T, Hq * d, dtype=act_dtype(mode), device=qkv.device)
    check(lib.bi_rope_kv_append(_ptr(qkv), _ptr(rope), rope_max_pos, _ptr(q), ctypes.byref(kv.layout), layer,
                                _ptr(slot), _ptr(pos), T, Hq, 1 if qk_paired else 0, mode, _stream()),
          "bi_rope_kv_append")
    return q


def attention(q, kv, layer, slot, pos, slot_host, pos_host, Hq, scale, mode=MODE_BF16, variant=VARIANT_INVARIANT):
    T = q.shape[0]
    d = kv.layout.head_dim
    sh = torch.as_tensor(slot_host, dtype=torch.int32).contiguous()
    ph = torch.as_tensor(pos_host, dtype=torch.int32).contiguous()
    max_pos = int(ph.max()) if T else 0
    wsb = lib.bi_attention_workspace_size(max(T, 1), Hq, d, max_pos)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=q.device)
    out = torch.empty_like(q)
    check(lib.bi_attention(_ptr(q), ctypes.byref(kv.layout), layer, _ptr(slot), _ptr(pos), _ptr(sh), _ptr(ph),
                           _ptr(out), T, Hq, float(scale), mode, variant, _ptr(ws), wsb, _stream()), "bi_attention")
    return out


def lmhead_logprob(h, W, target=None, threshold=0.1, mode=MODE_BF16, want_logits=False):
    """bi_lmhead_logprob on f32 rows h [B,H] and bf16 W [V,H]; returns a dict of device tensors."""
    B, H = h.shape
    V = W.shape[0]
    dev = h.device
    out = dict(logprob=torch.empty(B, dtype=torch.float32, device=dev),
               lse=torch.empty(B, dtype=torch.float32, device=dev),
               argmax=torch.empty(B, dtype=torch.int32, device=dev),
               margin=torch.empty(B, dtype=torch.float32, device=dev),
               recomputed=torch.empty(B, dtype=torch.uint8, device=dev))
    logits = torch.empty(B, V, dtype=torch.float32, device=dev) if want_logits else None
    wsb = lib.bi_lmhead_workspace_size(max(B, 1), H, V, mode)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev)
    check(lib.bi_lmhead_logprob(_ptr(h), _ptr(W), _ptr(target), B, H, V, float(threshold), mode,
                                _ptr(out["logprob"]), _ptr(out["lse"]), _ptr(out["argmax"]), _ptr(out["margin"]),
                                _ptr(out["recomputed"]), _ptr(logits), _ptr(ws), wsb, _stream()),
          "bi_lmhead_logprob")
    if want_logits:
        out["logits"] = logits
    return out


def synth_fill_bf16(dst, rows, cols, key, std, interleave=0, phase=0):
    check(lib.bi_synth_fill_bf16(_ptr(dst), rows, cols, ctypes.c_uint64(key), float(std), interleave, phase,
                                 _stream()), "bi_synth_fill_bf16")


def embed(ids, E, mode=MODE_BF16):
    """bi_embed: rows of the bf16 table E [V, H] for device int32 ids [T], in the mode's activation dtype."""
    T = ids.shape[0]
    V, H = E.shape
    x = torch.empty(T, H, dtype=act_dtype(mode), device=E.device)
    check(lib.bi_embed(_ptr(ids), _ptr(E), T, H, V, mode, _ptr(x), _stream()), "bi_embed")
    return x


def lmhead_split(h, parts):
    """bi_lmhead_split: bf16 GEMM rows [parts*B, H] of f32 rows h [B, H] (bf16(h), then the exact residual parts)."""
    B, H = h.shape
    out = torch.empty(parts * B, H, dtype=torch.bfloat16, device=h.device)
    check(lib.bi_lmhead_split(_ptr(h), B, H, parts, _ptr(out), _stream()), "bi_lmhead_split")
    return out


def lmhead_from_logits(z, B, parts, target=None, threshold=0.1):
    """bi_lmhead_from_logits on f32 logits z [parts*B, V]; returns the dict of bi_lmhead_logprob's outputs."""
    V = z.shape[1]
    dev = z.device
    out = dict(logprob=torch.empty(B, dtype=torch.float32, device=dev),
               lse=torch.empty(B, dtype=torch.float32, device=dev),
               argmax=torch.empty(B, dtype=torch.int32, device=dev),
               margin=torch.empty(B, dtype=torch.float32, device=dev),
               recomputed=torch.empty(B, dtype=torch.uint8, device=dev))
    wsb = lib.bi_lmhead_logits_workspace_size(max(B, 1), V)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev)
    check(lib.bi_lmhead_from_logits(_ptr(z), B, V, parts, _ptr(target), float(threshold), _ptr(out["logprob"]),
                                    _ptr(out["lse"]), _ptr(out["argmax"]), _ptr(out["margin"]),
                                    _ptr(out["recomputed"]), _ptr(ws), wsb, _stream()), "bi_lmhead_from_logits")
    return out


def greedy_advance(argmax, ids, pos):
    check(lib.bi_greedy_advance(_ptr(argmax), _ptr(ids), _ptr(pos), ids.shape[0], _stream()), "bi_greedy_advance")


def selftest_wait_timeout():
    """Enqueue the bounded-wait failure check (bi_selftest_wait_timeout) on the current stream."""
    check(lib.bi_selftest_wait_timeout(_stream()), "bi_selftest_wait_timeout")


def device_error(reset=True):
    v = ctypes.c_uint(0)
    check(lib.bi_device_error(ctypes.byref(v), 1 if reset else 0), "bi_device_error")
    return v.value
