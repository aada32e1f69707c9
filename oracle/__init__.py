"""fp64 CPU oracle of the batch-invariant decoder forward (TEST INFRASTRUCTURE).

Only tests/, the package smoke check and bench.py's CPU-baseline leg may import
this package.  It shares no code with the CUDA path and imports nothing from
it; inputs come from synth/ (data only).

The arithmetic lives in oracle.c (plain fp64 loops, one function per step of
the definition, each citing the passage it follows).  This wrapper only
marshals numpy arrays.

Pins (tests/test_oracle_pins.py) tie every function to something other than
itself: the pages' non-associativity example rounded in bf16, softmax and
log-softmax identities, closed forms of RMSNorm and RoPE, integer-exact
matrix products, brute-force special cases of attention, and reductions of the
whole forward to a plain matrix product when the blocks are switched off.
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_oracle.so")
_lib = None

OR_EXACT, OR_BF16 = 0, 1


class _Cfg(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("hidden", ctypes.c_int), ("n_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("ffn", ctypes.c_int),
                ("vocab", ctypes.c_int), ("eps", ctypes.c_double), ("rope_theta", ctypes.c_double)]


_WNAMES = ["embed", "attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "wg", "wu", "wd", "final_norm", "lm_head"]


class _W(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _WNAMES]


def build(force=False):
    src = os.path.join(_HERE, "oracle.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared",
                               "-fPIC", src, "-o", _SO, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        P, I, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        lib.or_round_bf16.restype = D
        lib.or_round_bf16.argtypes = [D]
        lib.or_gemm.argtypes = [P, P, P, I, I, I]
        lib.or_rmsnorm.argtypes = [P, P, P, I, I, D]
        lib.or_rope.argtypes = [P, I, I, I, D]
        lib.or_attention_query.argtypes = [P, P, P, I, I, D, P]
        lib.or_logit_stats.argtypes = [P, I, I, P]
        lib.or_lmhead.argtypes = [P, P, P, I, I, I, P, P]
        lib.or_forward.restype = I
        lib.or_forward.argtypes = [ctypes.POINTER(_Cfg), ctypes.POINTER(_W), I, P, I, P, P, P]
        lib.or_forward_ctx.restype = I
        lib.or_forward_ctx.argtypes = [ctypes.POINTER(_Cfg), ctypes.POINTER(_W), I, P, I, I, P, P, P, P, P, P, P]
        _lib = lib
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


def round_bf16(x):
    """Round fp64 values to the nearest bf16 value (ties to even)."""
    lib = _load()
    x = np.asarray(x, dtype=np.float64)
    return np.vectorize(lambda v: lib.or_round_bf16(float(v)), otypes=[np.float64])(x)


def gemm(x, w_bits):
    """y = x . w^T in fp64; x [M,K] float, w [N,K] bf16 bits."""
    x, w = _f64(x), _u16(w_bits)
    M, K = x.shape
    N = w.shape[0]
    assert w.shape[1] == K
    y = np.empty((M, N), dtype=np.float64)
    _load().or_gemm(x.ctypes.data, w.ctypes.data, y.ctypes.data, M, N, K)
    return y


def rmsnorm(x, gamma_bits, eps):
    x, g = _f64(x), _u16(gamma_bits)
    M, H = x.shape
    y = np.empty_like(x)
    _load().or_rmsnorm(x.ctypes.data, g.ctypes.data, y.ctypes.data, M, H, float(eps))
    return y


def rope(x, n_heads, head_dim, pos, theta):
    """Rotate-half RoPE of n_heads vectors of size head_dim at position pos (returns a copy)."""
    x = _f64(x).copy()
    _load().or_rope(x.ctypes.data, n_heads, head_dim, int(pos), float(theta))
    return x


def attention_query(q, K, V, scale):
    q, K, V = _f64(q), _f64(K), _f64(V)
    n, d = K.shape
    out = np.empty(d, dtype=np.float64)
    _load().or_attention_query(q.ctypes.data, K.ctypes.data, V.ctypes.data, n, d, float(scale), out.ctypes.data)
    return out


def logit_stats(z, target=-1):
    """(lse, logprob(target or argmax), argmax, margin, second index) of one logit row."""
    z = _f64(z)
    res = np.empty(5, dtype=np.float64)
    _load().or_logit_stats(z.ctypes.data, z.shape[0], int(target), res.ctypes.data)
    return res


def lmhead(h, w_bits, target=None, want_logits=False):
    """LM-head statistics of B rows; returns (res [B,5], logits or None)."""
    h, w = _f64(h), _u16(w_bits)
    B, H = h.shape
    V = w.shape[0]
    res = np.empty((B, 5), dtype=np.float64)
    tg = None if target is None else np.ascontiguousarray(target, dtype=np.int32)
    logits = np.empty((B, V), dtype=np.float64) if want_logits else None
    _load().or_lmhead(h.ctypes.data, w.ctypes.data, None if tg is None else tg.ctypes.data, B, H, V,
                      res.ctypes.data, None if logits is None else logits.ctypes.data)
    return res, logits


def forward(cfg, weights, tokens, targets=None, mode=OR_BF16, want_h=False):
    """Full forward of one sequence; returns res [n,5] (lse, logprob, argmax, margin, 2nd idx) and h [n,H]."""
    lib = _load()
    c = _Cfg(cfg["n_layers"], cfg["hidden"], cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"], cfg["ffn"],
             cfg["vocab"], float(cfg["eps"]), float(cfg["rope_theta"]))
    keep = {n: _u16(weights[n]) for n in _WNAMES}
    w = _W(*[keep[n].ctypes.data for n in _WNAMES])
    tok = np.ascontiguousarray(tokens, dtype=np.int32)
    n = tok.shape[0]
    tg = None if targets is None else np.ascontiguousarray(targets, dtype=np.int32)
    res = np.empty((n, 5), dtype=np.float64)
    h = np.empty((n, cfg["hidden"]), dtype=np.float64) if want_h else None
    rc = lib.or_forward(ctypes.byref(c), ctypes.byref(w), int(mode), tok.ctypes.data, n,
                        None if tg is None else tg.ctypes.data, res.ctypes.data,
                        None if h is None else h.ctypes.data)
    if rc != 0:
        raise MemoryError("oracle forward: allocation failed")
    return res, h


def forward_ctx(cfg, weights, tokens, k_ctx=None, v_ctx=None, targets=None, mode=OR_BF16, want_h=False,
                want_kv=False):
    """Forward of new tokens that follow earlier positions of the same sequence, given those positions' stored
    keys and values per layer (k_ctx, v_ctx: [L, n_ctx, Hkv*d]; None for none).  Returns res [n,5], h [n,H] or
    None, and (k, v) [L, n, Hkv*d] of the new tokens or None."""
    lib = _load()
    c = _Cfg(cfg["n_layers"], cfg["hidden"], cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"], cfg["ffn"],
             cfg["vocab"], float(cfg["eps"]), float(cfg["rope_theta"]))
    keep = {n: _u16(weights[n]) for n in _WNAMES}
    w = _W(*[keep[n].ctypes.data for n in _WNAMES])
    tok = np.ascontiguousarray(tokens, dtype=np.int32)
    n = tok.shape[0]
    L, KD = cfg["n_layers"], cfg["n_kv_heads"] * cfg["head_dim"]
    n_ctx = 0 if k_ctx is None else int(np.shape(k_ctx)[1])
    kc = None if k_ctx is None else _f64(k_ctx)
    vc = None if v_ctx is None else _f64(v_ctx)
    assert kc is None or (kc.shape == (L, n_ctx, KD) and vc is not None and vc.shape == kc.shape)
    tg = None if targets is None else np.ascontiguousarray(targets, dtype=np.int32)
    res = np.empty((n, 5), dtype=np.float64)
    h = np.empty((n, cfg["hidden"]), dtype=np.float64) if want_h else None
    ko = np.empty((L, n, KD), dtype=np.float64) if want_kv else None
    vo = np.empty((L, n, KD), dtype=np.float64) if want_kv else None
    ptr = lambda a: None if a is None else a.ctypes.data
    rc = lib.or_forward_ctx(ctypes.byref(c), ctypes.byref(w), int(mode), tok.ctypes.data, n, n_ctx, ptr(kc),
                            ptr(vc), ptr(tg), res.ctypes.data, ptr(h), ptr(ko), ptr(vo))
    if rc != 0:
        raise MemoryError("oracle forward: allocation failed")
    return res, h, ((ko, vo) if want_kv else None)
