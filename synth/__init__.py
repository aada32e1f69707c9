"""Seeded synthetic inputs shared, as data only, by the oracle and the GPU harness.

This module holds none of the decoder's arithmetic: it draws SplitMix64
counters, turns them into approximately normal deviates (Irwin-Hall sum of
twelve 16-bit uniforms, unit variance), rounds weights to bf16, and draws
uniform token ids.  The exact definitions are in synth.c; the GPU package has
an independent device implementation of the same published definitions for
tensors too large to generate on the host, and a GPU test checks the two agree
bit for bit.

Workload recipe (weights N(0, 0.02) in bf16, norms = 1, uniform token ids)
follows the model shapes listed in configs.py.
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_synth.so")
_lib = None

WEIGHT_SEED = 20261202
WEIGHT_STD = 0.02


def build(force=False):
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC",
                               src, "-o", _SO])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        lib.synth_key.restype = ctypes.c_uint64
        lib.synth_key.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_draw.restype = ctypes.c_uint64
        lib.synth_draw.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_normal_f64.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p]
        lib.synth_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_double,
                                          ctypes.c_void_p]
        lib.synth_tokens.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                     ctypes.c_void_p]
        _lib = lib
    return _lib


def key(seed, stream):
    return int(_load().synth_key(seed, stream))


def draw(k, i):
    return int(_load().synth_draw(k, i))


def normal_f64(k, n, start=0):
    out = np.empty(n, dtype=np.float64)
    _load().synth_normal_f64(k, start, n, out.ctypes.data)
    return out


def normal_bf16(k, n, std=WEIGHT_STD, start=0):
    """bf16 bit patterns (uint16) of std * normal."""
    out = np.empty(n, dtype=np.uint16)
    _load().synth_normal_bf16(k, start, n, float(std), out.ctypes.data)
    return out


def tokens(k, n, vocab, start=0):
    out = np.empty(n, dtype=np.int32)
    _load().synth_tokens(k, start, n, vocab, out.ctypes.data)
    return out


def bf16_to_f32(bits):
    """Decode bf16 bit patterns to float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x):
    """Encode float32 values to bf16 bit patterns, round-to-nearest-even (input preparation)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


# --- stream ids of the logical weight tensors (data layout of the recipe) ---
S_EMBED, S_LMHEAD = 1, 2
S_WQ, S_WK, S_WV, S_WO, S_WG, S_WU, S_WD = range(7)


def layer_stream(layer, which):
    return 100 + 16 * layer + which


def hidden_states(seed, rows, hidden):
    """fp32 rows N(0,1), each scaled to unit RMS (the LM-head workload recipe)."""
    z = normal_f64(key(seed, 7), rows * hidden).reshape(rows, hidden)
    z = z / np.sqrt(np.mean(z * z, axis=1, keepdims=True))
    return z.astype(np.float32)


def model_weights(cfg, seed=WEIGHT_SEED, std=WEIGHT_STD):
    """Logical (unfused) bf16 weights of a model config, as uint16 arrays.

    Norm gains are 1.0; every matrix and the embedding are N(0, std).
    Returns dict: embed [V,H], lm_head [V,H], final_norm [H], and per-layer
    stacks attn_norm/ffn_norm [L,H], wq [L,Hq*d,H], wk/wv [L,Hkv*d,H],
    wo [L,H,Hq*d], wg/wu [L,F,H], wd [L,H,F].
    """
    L, H, Hq, Hkv, d, F, V = (cfg["n_layers"], cfg["hidden"], cfg["n_heads"], cfg["n_kv_heads"],
                              cfg["head_dim"], cfg["ffn"], cfg["vocab"])
    one = np.uint16(0x3F80)
    w = {
        "embed": normal_bf16(key(seed, S_EMBED), V * H, std).reshape(V, H),
        "lm_head": normal_bf16(key(seed, S_LMHEAD), V * H, std).reshape(V, H),
        "final_norm": np.full(H, one, dtype=np.uint16),
        "attn_norm": np.full((L, H), one, dtype=np.uint16),
        "ffn_norm": np.full((L, H), one, dtype=np.uint16),
    }
    shapes = {S_WQ: (Hq * d, H), S_WK: (Hkv * d, H), S_WV: (Hkv * d, H), S_WO: (H, Hq * d),
              S_WG: (F, H), S_WU: (F, H), S_WD: (H, F)}
    names = {S_WQ: "wq", S_WK: "wk", S_WV: "wv", S_WO: "wo", S_WG: "wg", S_WU: "wu", S_WD: "wd"}
    for s, shp in shapes.items():
        w[names[s]] = np.stack([normal_bf16(key(seed, layer_stream(l, s)), shp[0] * shp[1], std).reshape(shp)
                                for l in range(L)])
    return w


def prompt_tokens(request, length, vocab, seed=1000):
    """Token ids of a synthetic prompt: uniform in [0, vocab), seed 1000 + request index."""
    return tokens(key(seed + request, 3), length, vocab)
