"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test ties one oracle function to a value the pages print, a closed form,
an invariant, exact integer arithmetic, or a brute-force special case, chosen
so that a dropped term, a wrong sign/index or a transposed operand fails.
"""
import math
import os

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle
import synth
from synth import configs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split()
            vals[k] = float(v)
    return vals


# ---------------------------------------------------------------- bf16 rounding
def test_nonassociativity_example_bf16():
    """The pages' (0.1+0.2)+(-0.1) vs 0.1+(0.2+(-0.1)) example, rounded in bf16."""
    g = _golden("nonassoc_bf16.txt")
    rb = lambda x: float(oracle.round_bf16(x))
    a, b, c = rb(0.1), rb(0.2), rb(-0.1)
    assert (a, b, c) == (g["a_bf16"], g["b_bf16"], g["c_bf16"])
    ab = rb(a + b)
    assert ab == g["ab_bf16"]
    left = rb(ab + c)
    bc = rb(b + c)
    right = rb(a + bc)
    assert bc == g["bc_bf16"]
    assert left == g["left_bf16"] and right == g["right_bf16"]
    assert left != right  # the orders differ in low precision
    # in fp32 the two orders still differ, but both round to the same bf16 value
    f = np.float32
    l32 = (f(0.1) + f(0.2)) + f(-0.1)
    r32 = f(0.1) + (f(0.2) + f(-0.1))
    assert l32 != r32
    assert rb(float(l32)) == rb(float(r32)) == g["right_bf16"]


def test_round_bf16_ties_and_neighbours():
    """Brute force over random bf16 neighbours: midpoints go to the even pattern, others to the nearest."""
    rng = np.random.default_rng(1)
    bits = rng.integers(0x0080, 0x7F00, size=2000, dtype=np.uint16)  # positive normal bf16
    lo = synth.bf16_to_f32(bits).astype(np.float64)
    hi = synth.bf16_to_f32(bits + 1).astype(np.float64)
    mid = (lo + hi) / 2.0  # exact in fp64
    even = np.where(bits % 2 == 0, lo, hi)
    assert np.array_equal(oracle.round_bf16(mid), even)
    assert np.array_equal(oracle.round_bf16(-mid), -even)
    eps = (hi - lo) * 1e-6
    assert np.array_equal(oracle.round_bf16(mid - eps), lo)
    assert np.array_equal(oracle.round_bf16(mid + eps), hi)
    assert np.array_equal(oracle.round_bf16(lo), lo)


# ---------------------------------------------------------------- GEMM
def test_gemm_integer_exact_nonsquare():
    """Integer-valued operands: the fp64 result equals exact integer arithmetic (catches transposes)."""
    rng = np.random.default_rng(2)
    M, N, K = 3, 5, 7
    x = rng.integers(-8, 9, size=(M, K))
    w = rng.integers(-8, 9, size=(N, K))
    y = oracle.gemm(x.astype(np.float64), synth.f32_to_bf16_bits(w.astype(np.float32)))
    assert np.array_equal(y, (x @ w.T).astype(np.float64))


def test_gemm_identity():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 16))
    eye = synth.f32_to_bf16_bits(np.eye(16, dtype=np.float32))
    assert np.array_equal(oracle.gemm(x, eye), x)


# ---------------------------------------------------------------- RMSNorm
def test_rmsnorm_closed_forms():
    H = 64
    ones = np.full(H, 0x3F80, dtype=np.uint16)
    # constant row c: every output is c / sqrt(c^2 + eps)
    for c in (0.5, -3.0, 1e-3):
        y = oracle.rmsnorm(np.full((1, H), c), ones, 1e-5)
        assert np.allclose(y, c / math.sqrt(c * c + 1e-5), rtol=1e-14, atol=0)
    rng = np.random.default_rng(4)
    x = rng.standard_normal((5, H))
    y = oracle.rmsnorm(x, ones, 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=1)), 1.0, rtol=1e-13)
    # scale invariance (eps = 0) and per-channel gain
    assert np.allclose(oracle.rmsnorm(7.5 * x, ones, 0.0), y, rtol=1e-13)
    gain = synth.f32_to_bf16_bits(np.arange(1, H + 1, dtype=np.float32))
    assert np.allclose(oracle.rmsnorm(x, gain, 0.0), y * np.arange(1, H + 1), rtol=1e-13)


# ---------------------------------------------------------------- RoPE
def test_rope_explicit_values():
    """d = 4, theta = 1e4: pairs (0,2) at frequency 1 and (1,3) at 1e4^-0.5 = 0.01."""
    out = oracle.rope([1.0, 0.0, 0.0, 0.0], 1, 4, 1, 10000.0)
    assert np.allclose(out, [math.cos(1), 0, math.sin(1), 0], rtol=0, atol=1e-15)
    out = oracle.rope([0.0, 0.0, 0.0, 1.0], 1, 4, 3, 10000.0)
    assert np.allclose(out, [0, -math.sin(0.03), 0, math.cos(0.03)], rtol=0, atol=1e-15)


def test_rope_identity_norm_and_relative_position():
    rng = np.random.default_rng(5)
    d, nh = 64, 3
    q = rng.standard_normal(nh * d)
    k = rng.standard_normal(nh * d)
    assert np.array_equal(oracle.rope(q, nh, d, 0, 1e4), q)
    r = oracle.rope(q, nh, d, 17, 1e4).reshape(nh, 2, d // 2)
    q3 = q.reshape(nh, 2, d // 2)
    assert np.allclose((r ** 2).sum(1), (q3 ** 2).sum(1), rtol=1e-12)  # each rotated pair keeps its norm
    # q(p) . k(p') depends only on p - p'
    def dot(p, pp):
        return float(np.dot(oracle.rope(q, nh, d, p, 1e4), oracle.rope(k, nh, d, pp, 1e4)))
    assert math.isclose(dot(5, 2), dot(105, 102), rel_tol=1e-9)
    assert math.isclose(dot(3, 3), float(np.dot(q, k)), rel_tol=1e-9)
    assert not math.isclose(dot(5, 2), dot(5, 3), rel_tol=1e-6)


# ---------------------------------------------------------------- attention
def test_attention_special_cases():
    rng = np.random.default_rng(6)
    d = 32
    K = rng.standard_normal((6, d))
    V = rng.standard_normal((6, d))
    # one key: the output is that value row
    assert np.allclose(oracle.attention_query(rng.standard_normal(d), K[:1], V[:1], 0.3), V[0], rtol=1e-14)
    # q = 0: equal scores, the output is the mean of the value rows
    assert np.allclose(oracle.attention_query(np.zeros(d), K, V, 0.3), V.mean(0), rtol=1e-13)
    # a dominant key selects its value row
    q = 50.0 * K[2] / np.linalg.norm(K[2])
    Ko = np.eye(6, d) * 1.0
    Ko[2] = K[2] / np.linalg.norm(K[2])
    out = oracle.attention_query(q, Ko, V, 1.0)
    assert np.allclose(out, V[2], atol=1e-15 + 1e-12 * np.abs(V).max() * 10)
    # key/value row permutation does not change the result
    perm = rng.permutation(6)
    q = rng.standard_normal(d)
    assert np.allclose(oracle.attention_query(q, K, V, 0.2), oracle.attention_query(q, K[perm], V[perm], 0.2),
                       rtol=1e-13)
    # brute force on a tiny case with scipy's softmax
    s = 0.2 * (K @ q)
    assert np.allclose(oracle.attention_query(q, K, V, 0.2), softmax(s) @ V, rtol=1e-12)


# ---------------------------------------------------------------- logit statistics
def test_logit_stats_uniform_and_ties():
    V = 1000
    res = oracle.logit_stats(np.full(V, 2.5))
    assert math.isclose(res[0], 2.5 + math.log(V), rel_tol=1e-15)
    assert math.isclose(res[1], -math.log(V), rel_tol=1e-13)
    assert res[2] == 0 and res[3] == 0.0  # lowest id on ties; duplicated maximum gives margin 0
    res = oracle.logit_stats(np.array([1.0, 3.0, 2.0, 3.0]))
    assert res[2] == 1 and res[3] == 0.0 and res[4] == 3
    res = oracle.logit_stats(np.array([0.0, 5.0, 2.0]), target=2)
    assert res[2] == 1 and res[3] == 3.0 and res[4] == 2
    assert math.isclose(res[1], 2.0 - logsumexp([0.0, 5.0, 2.0]), rel_tol=1e-14)


def test_logprobs_normalise():
    rng = np.random.default_rng(7)
    z = 3.0 * rng.standard_normal(500)
    lp = np.array([oracle.logit_stats(z, t)[1] for t in range(500)])
    assert math.isclose(np.exp(lp).sum(), 1.0, rel_tol=1e-12)
    assert np.allclose(lp, z - logsumexp(z), rtol=1e-13)


def test_lmhead_one_hot_rows_select_weight_columns():
    rng = np.random.default_rng(8)
    H, V = 16, 40
    W = synth.f32_to_bf16_bits(rng.standard_normal((V, H)).astype(np.float32))
    h = np.zeros((2, H))
    h[0, 3] = 1.0
    h[1, 11] = 1.0
    res, logits = oracle.lmhead(h, W, target=[5, 7], want_logits=True)
    Wf = synth.bf16_to_f32(W).astype(np.float64)
    assert np.array_equal(logits[0], Wf[:, 3]) and np.array_equal(logits[1], Wf[:, 11])
    assert res[0, 2] == int(np.argmax(Wf[:, 3]))
    assert math.isclose(res[1, 1], Wf[7, 11] - logsumexp(Wf[:, 11]), rel_tol=1e-13)


# ---------------------------------------------------------------- whole forward
def _tiny_weights(cfg, seed=11):
    return synth.model_weights(cfg, seed=seed)


def _rms(x):
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + 1e-5)


def test_forward_blocks_off_reduces_to_embedding_lmhead():
    """W_o = W_d = 0: the residual stays the embedding, logits = rmsnorm(E[id]) W_lm^T."""
    cfg = configs.shrink(configs.TINY, n_layers=2, vocab=512)
    w = _tiny_weights(cfg)
    w["wo"][:] = 0
    w["wd"][:] = 0
    tok = synth.tokens(synth.key(3, 3), 9, cfg["vocab"])
    tgt = np.roll(tok, -1)
    res, h = oracle.forward(cfg, w, tok, tgt, mode=oracle.OR_EXACT, want_h=True)
    E = synth.bf16_to_f32(w["embed"]).astype(np.float64)
    Wl = synth.bf16_to_f32(w["lm_head"]).astype(np.float64)
    hh = _rms(E[tok])
    assert np.allclose(h, hh, rtol=1e-13)
    z = hh @ Wl.T
    assert np.array_equal(res[:, 2].astype(int), np.argmax(z, axis=1))
    assert np.allclose(res[:, 0], logsumexp(z, axis=1), rtol=1e-13)
    assert np.allclose(res[:, 1], z[np.arange(9), tgt] - logsumexp(z, axis=1), rtol=1e-12, atol=1e-12)
    top2 = np.sort(z, axis=1)[:, -2:]
    assert np.allclose(res[:, 3], top2[:, 1] - top2[:, 0], rtol=1e-10, atol=1e-13)


def test_forward_uniform_attention_prefix_mean_gqa():
    """W_q = 0 makes every score equal: attention = causal prefix mean of v of the right kv head.

    W_o = I (Hq*d = H), W_d = 0, so h = rmsnorm(E + o) exposes o directly.
    GQA with 4 q heads on 2 kv heads: q head j reads kv head j // 2.
    """
    cfg = configs.shrink(configs.TINY, n_layers=1, n_kv_heads=2, vocab=512)
    H, d, Hq, Hkv = cfg["hidden"], cfg["head_dim"], cfg["n_heads"], cfg["n_kv_heads"]
    w = _tiny_weights(cfg, seed=12)
    w["wq"][:] = 0
    w["wd"][:] = 0
    w["wo"][0] = synth.f32_to_bf16_bits(np.eye(H, dtype=np.float32))
    n = 7
    tok = synth.tokens(synth.key(4, 3), n, cfg["vocab"])
    res, h = oracle.forward(cfg, w, tok, None, mode=oracle.OR_EXACT, want_h=True)
    E = synth.bf16_to_f32(w["embed"]).astype(np.float64)[tok]
    Wv = synth.bf16_to_f32(w["wv"][0]).astype(np.float64)
    v = (_rms(E) @ Wv.T).reshape(n, Hkv, d)
    o = np.zeros((n, Hq, d))
    for t in range(n):
        for j in range(Hq):
            o[t, j] = v[: t + 1, j // (Hq // Hkv)].mean(0)
    assert np.allclose(h, _rms(E + o.reshape(n, H)), rtol=1e-11, atol=1e-12)


def test_forward_two_token_brute_force():
    """Tiny full layer, 2 tokens, brute force with numpy + scipy (RoPE from the pinned or_rope)."""
    cfg = configs.shrink(configs.TINY, n_layers=1, n_heads=2, n_kv_heads=1, head_dim=8, hidden=16, ffn=24,
                         vocab=64)
    H, d, Hq, Hkv, F = 16, 8, 2, 1, 24
    w = _tiny_weights(cfg, seed=13)
    f = lambda a: synth.bf16_to_f32(a).astype(np.float64)
    tok = np.array([5, 41], dtype=np.int32)
    res, h = oracle.forward(cfg, w, tok, [41, 3], mode=oracle.OR_EXACT, want_h=True)
    x = f(w["embed"])[tok]
    u = _rms(x)
    q = u @ f(w["wq"][0]).T
    k = u @ f(w["wk"][0]).T
    v = u @ f(w["wv"][0]).T
    q = np.stack([oracle.rope(q[t], Hq, d, t, cfg["rope_theta"]) for t in range(2)]).reshape(2, Hq, d)
    k = np.stack([oracle.rope(k[t], Hkv, d, t, cfg["rope_theta"]) for t in range(2)]).reshape(2, Hkv, d)
    v = v.reshape(2, Hkv, d)
    o = np.zeros((2, Hq, d))
    for t in range(2):
        for j in range(Hq):
            p = softmax(np.array([q[t, j] @ k[s, 0] for s in range(t + 1)]) / math.sqrt(d))
            o[t, j] = p @ v[: t + 1, 0]
    x = x + o.reshape(2, H) @ f(w["wo"][0]).T
    u = _rms(x)
    g = u @ f(w["wg"][0]).T
    up = u @ f(w["wu"][0]).T
    x = x + ((g / (1 + np.exp(-g))) * up) @ f(w["wd"][0]).T
    hh = _rms(x)
    assert np.allclose(h, hh, rtol=1e-12, atol=1e-13)
    z = hh @ f(w["lm_head"]).T
    assert np.allclose(res[:, 1], z[[0, 1], [41, 3]] - logsumexp(z, axis=1), rtol=1e-11)


def test_forward_causal_and_bf16_mode_close_to_exact():
    cfg = configs.shrink(configs.TINY, vocab=512)
    w = _tiny_weights(cfg, seed=14)
    tok = synth.tokens(synth.key(5, 3), 12, cfg["vocab"])
    full, _ = oracle.forward(cfg, w, tok, None, mode=oracle.OR_BF16)
    pre, _ = oracle.forward(cfg, w, tok[:6], None, mode=oracle.OR_BF16)
    assert np.array_equal(full[:6], pre)  # later tokens never affect earlier positions
    ex, _ = oracle.forward(cfg, w, tok, None, mode=oracle.OR_EXACT)
    d = np.abs(full[:, 0] - ex[:, 0])
    assert d.max() < 0.05 and d.max() > 0  # bf16 storage changes results, but only slightly


def test_forward_bf16_mode_rounds_stored_values():
    """With the blocks off, the bf16 mode's LM-head input is the bf16 rounding of the exact h."""
    cfg = configs.shrink(configs.TINY, n_layers=1, vocab=256)
    w = _tiny_weights(cfg, seed=15)
    w["wo"][:] = 0
    w["wd"][:] = 0
    tok = np.array([1, 2, 3], dtype=np.int32)
    rb, hb = oracle.forward(cfg, w, tok, None, mode=oracle.OR_BF16, want_h=True)
    re, he = oracle.forward(cfg, w, tok, None, mode=oracle.OR_EXACT, want_h=True)
    assert np.array_equal(hb, he)  # same unrounded h (the residual is the bf16 embedding)
    res2, _ = oracle.lmhead(oracle.round_bf16(he), w["lm_head"])
    assert np.array_equal(rb[:, :4], res2[:, :4])
