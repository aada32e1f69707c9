"""Pins of the oracle's bf16-storage emulation (OR_BF16) (CPU only).

The bf16 path stores every inter-kernel activation in bf16 and accumulates in
fp32 ("Give Me FP32 or Give Me Death?", floating-point formats section: BF16
keeps 8 exponent bits and 7 stored mantissa bits).  The reading fixes the
storage points: the norm outputs, q/k/v after RoPE, the attention output,
every linear output, the residual after every add, the SwiGLU output and the
LM-head input.  These tests tie each of those points to something other than
the oracle's own code:

  * closed forms on hand-built weights where one rounding decision (a tie to
    even, or a value a known fraction of an ulp off) decides a result that is
    worked out exactly;
  * a brute-force numpy forward of a 2-layer model that rounds at exactly the
    listed points (RoPE and rounding from the separately pinned or_rope and
    round_bf16), and, for every point, a check that leaving that one point
    out changes the result -- so a dropped or misplaced rounding in the oracle
    cannot pass.
"""
import math

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle
import synth
from synth import configs

B16 = synth.f32_to_bf16_bits


def _probe_cfg(**kw):
    """One layer, hidden 16 = one head of 16, eps 0 so that norms of hand-built rows are exact."""
    c = configs.shrink(configs.TINY, n_layers=1, hidden=16, n_heads=1, n_kv_heads=1, head_dim=16, ffn=16, vocab=32,
                       eps=0.0)
    c.update(kw)
    return c


def _zero_weights(cfg):
    w = synth.model_weights(cfg, seed=5)
    for k in ("embed", "wq", "wk", "wv", "wo", "wg", "wu", "wd", "lm_head"):
        w[k][:] = 0
    return w  # norms keep gamma = 1.0


def _set(a, idx, val):
    a[idx] = B16(np.array([val], dtype=np.float32))[0]
    assert synth.bf16_to_f32(a[idx]) == np.float32(val), f"{val} is not a bf16 value"


def test_attention_output_rounds_to_even():
    """Position 1 averages v0 = 1 and v1 = 1 + 2^-7 (equal scores): o = 1 + 2^-8, a tie, stored as 1.0.

    W_o amplifies o[0] - o[1] by 2^10 into dim 2 of the residual: 0 when o is rounded, 4 when it is not.
    The final norm then shows it: h_1 = 4 e_1 (bf16 storage) or (e_1 + 4 e_2) * 4 / sqrt(17) (exact).
    """
    cfg = _probe_cfg()
    w = _zero_weights(cfg)
    _set(w["embed"], (0, 0), 1.0)  # token 0 -> e_0, token 1 -> e_1; rmsnorm gives 4 e_t (H = 16, eps = 0)
    _set(w["embed"], (1, 1), 1.0)
    _set(w["wv"], (0, 0, 0), 0.25)
    _set(w["wv"], (0, 1, 0), 0.25)
    _set(w["wv"], (0, 0, 1), (1 + 2 ** -7) / 4)
    _set(w["wv"], (0, 1, 1), 0.25)
    _set(w["wo"], (0, 2, 0), 2.0 ** 10)
    _set(w["wo"], (0, 2, 1), -2.0 ** 10)
    tok = np.array([0, 1], dtype=np.int32)
    _, hb = oracle.forward(cfg, w, tok, mode=oracle.OR_BF16, want_h=True)
    _, he = oracle.forward(cfg, w, tok, mode=oracle.OR_EXACT, want_h=True)
    e = np.eye(16)
    assert np.array_equal(hb[0], 4 * e[0]) and np.array_equal(he[0], 4 * e[0])
    assert np.array_equal(hb[1], 4 * e[1])
    assert np.allclose(he[1], (e[1] + 4 * e[2]) * 4 / math.sqrt(17), rtol=1e-14, atol=0)


def test_norm_output_rounding_345():
    """Embedding row (3, 4, 0, ...): rmsnorm = (2.4, 3.2), stored as (2.40625, 3.203125) (154 and 205 units of
    2^-6).  v[0] = u0 - 0.75 u1 is then 2^-8 instead of 0; W_o scales it by 2^10 into dim 2 of the residual.
    bf16 storage: r = (3, 4, 4) and h = r * 4 / sqrt(41); exact: h = (2.4, 3.2, 0)."""
    cfg = _probe_cfg()
    w = _zero_weights(cfg)
    _set(w["embed"], (0, 0), 3.0)
    _set(w["embed"], (0, 1), 4.0)
    _set(w["wv"], (0, 0, 0), 1.0)
    _set(w["wv"], (0, 0, 1), -0.75)
    _set(w["wo"], (0, 2, 0), 2.0 ** 10)
    tok = np.array([0], dtype=np.int32)
    _, hb = oracle.forward(cfg, w, tok, mode=oracle.OR_BF16, want_h=True)
    _, he = oracle.forward(cfg, w, tok, mode=oracle.OR_EXACT, want_h=True)
    r = np.zeros(16)
    r[:3] = (3.0, 4.0, 4.0)
    assert np.allclose(hb[0], r * 4 / math.sqrt(41), rtol=1e-14, atol=0)
    assert np.allclose(he[0, :2], (2.4, 3.2), rtol=1e-14) and abs(he[0, 2]) < 1e-9
    assert np.all(he[0, 3:] == 0)


def test_swiglu_output_rounding():
    """Residual row of ones (attention block off): the ffn norm gives ones.  Channel 0 computes
    silu(1) * 1 = 0.7310585786..., stored as 0.73046875 (187 units of 2^-8); channel 1 computes exactly
    0.73046875 (silu(64) = 64 in fp64, times 187 * 2^-14).  The down projection takes 2^10 * (a0 - a1) into
    dim 2: 0 with the SwiGLU output stored in bf16, 2^10 (silu(1) - 0.73046875) without."""
    cfg = _probe_cfg()
    w = _zero_weights(cfg)
    w["embed"][0, :] = B16(np.ones(16, dtype=np.float32))
    _set(w["wg"], (0, 0, 0), 1.0)
    _set(w["wu"], (0, 0, 0), 1.0)
    _set(w["wg"], (0, 1, 0), 64.0)
    _set(w["wu"], (0, 1, 0), 187 * 2.0 ** -14)
    _set(w["wd"], (0, 2, 0), 2.0 ** 10)
    _set(w["wd"], (0, 2, 1), -2.0 ** 10)
    tok = np.array([0], dtype=np.int32)
    _, hb = oracle.forward(cfg, w, tok, mode=oracle.OR_BF16, want_h=True)
    _, he = oracle.forward(cfg, w, tok, mode=oracle.OR_EXACT, want_h=True)
    assert np.array_equal(hb[0], np.ones(16))
    y = 2.0 ** 10 * (1.0 / (1.0 + math.exp(-1.0)) - 0.73046875)
    r = np.ones(16)
    r[2] += y
    assert np.allclose(he[0], r / math.sqrt(np.mean(r * r)), rtol=1e-13, atol=0)


def test_linear_output_then_residual_double_rounding():
    """o = (1, 1, 0, ...) (one token, v from a row of ones); W_o[2] = (2^-8, 2^-20) gives y2 = 2^-8 + 2^-20.
    Stored linear output: bf16(y2) = 2^-8 (2^-20 is below half its ulp), then 1 + 2^-8 is a tie and the
    residual stays 1.0: h = ones.  Without the linear-output rounding 1 + 2^-8 + 2^-20 rounds up to 1 + 2^-7;
    without the residual rounding it stays 1 + 2^-8 (+ 2^-20)."""
    cfg = _probe_cfg()
    w = _zero_weights(cfg)
    w["embed"][0, :] = B16(np.ones(16, dtype=np.float32))
    _set(w["wv"], (0, 0, 0), 1.0)  # u = ones: v[i] = row sum of W_v
    _set(w["wv"], (0, 1, 0), 1.0)
    _set(w["wo"], (0, 2, 0), 2.0 ** -8)
    _set(w["wo"], (0, 2, 1), 2.0 ** -20)
    tok = np.array([0], dtype=np.int32)
    _, hb = oracle.forward(cfg, w, tok, mode=oracle.OR_BF16, want_h=True)
    _, he = oracle.forward(cfg, w, tok, mode=oracle.OR_EXACT, want_h=True)
    assert np.array_equal(hb[0], np.ones(16))
    r = np.ones(16)
    r[2] += 2.0 ** -8 + 2.0 ** -20
    assert np.allclose(he[0], r / math.sqrt(np.mean(r * r)), rtol=1e-14, atol=0)


# ------------------------------------------------------------- brute force with every storage point
POINTS = ("norm_attn", "q", "k", "v", "attn_out", "o_proj", "resid_attn", "norm_ffn", "swiglu", "down_proj",
          "resid_ffn", "lm_in")


def _rb(x):
    return oracle.round_bf16(x)


def _brute_bf16(cfg, w, tok, skip=None):
    """The bf16-storage forward written out in numpy, rounding at the points of the reading; `skip` leaves one
    point unrounded.  Returns (lse, logprob of the argmax, margin) per position and h (before the LM-head
    rounding)."""
    f = lambda a: synth.bf16_to_f32(a).astype(np.float64)
    R = lambda name, x: x if name == skip else _rb(x)
    H, Hq, Hkv, d = cfg["hidden"], cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    G, n, eps = Hq // Hkv, len(tok), cfg["eps"]

    def rms(x, g):
        return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * f(g)

    x = f(w["embed"])[tok]
    for l in range(cfg["n_layers"]):
        u = R("norm_attn", rms(x, w["attn_norm"][l]))
        q = u @ f(w["wq"][l]).T
        k = u @ f(w["wk"][l]).T
        v = u @ f(w["wv"][l]).T
        q = np.stack([oracle.rope(q[t], Hq, d, t, cfg["rope_theta"]) for t in range(n)])
        k = np.stack([oracle.rope(k[t], Hkv, d, t, cfg["rope_theta"]) for t in range(n)])
        q = R("q", q).reshape(n, Hq, d)
        k = R("k", k).reshape(n, Hkv, d)
        v = R("v", v).reshape(n, Hkv, d)
        o = np.zeros((n, Hq, d))
        for t in range(n):
            for j in range(Hq):
                p = softmax(k[: t + 1, j // G] @ q[t, j] / math.sqrt(d))
                o[t, j] = p @ v[: t + 1, j // G]
        o = R("attn_out", o.reshape(n, Hq * d))
        x = R("resid_attn", x + R("o_proj", o @ f(w["wo"][l]).T))
        u = R("norm_ffn", rms(x, w["ffn_norm"][l]))
        g = u @ f(w["wg"][l]).T
        up = u @ f(w["wu"][l]).T
        a = R("swiglu", g / (1 + np.exp(-g)) * up)
        x = R("resid_ffn", x + R("down_proj", a @ f(w["wd"][l]).T))
    h = rms(x, w["final_norm"])
    z = R("lm_in", h) @ f(w["lm_head"]).T
    lse = logsumexp(z, axis=1)
    zs = np.sort(z, axis=1)
    return np.stack([lse, zs[:, -1] - lse, zs[:, -1] - zs[:, -2]], axis=1), h


@pytest.fixture(scope="module")
def brute_case():
    cfg = configs.shrink(configs.TINY, n_layers=2, hidden=16, n_heads=2, n_kv_heads=1, head_dim=8, ffn=24,
                         vocab=64)
    w = synth.model_weights(cfg, seed=21, std=0.25)  # block outputs comparable to the residual stream
    tok = synth.tokens(synth.key(21, 1), 5, cfg["vocab"])
    res, h = oracle.forward(cfg, w, tok, mode=oracle.OR_BF16, want_h=True)
    got = np.stack([res[:, 0], res[:, 1], res[:, 3]], axis=1)
    return cfg, w, tok, got, h


def test_bf16_forward_matches_brute_force(brute_case):
    cfg, w, tok, got, h = brute_case
    ref, href = _brute_bf16(cfg, w, tok)
    assert np.allclose(h, href, rtol=1e-11, atol=1e-13)
    assert np.allclose(got, ref, rtol=1e-11, atol=1e-12)
    ex, _ = oracle.forward(cfg, w, tok, mode=oracle.OR_EXACT)
    assert np.abs(ex[:, 0] - got[:, 0]).max() > 1e-4  # the storage points do change the result


@pytest.mark.parametrize("point", POINTS)
def test_bf16_forward_each_storage_point_matters(brute_case, point):
    """Leaving out any one storage point moves the brute force away from the oracle by far more than the
    agreement tolerance above, so the agreement pins every point."""
    cfg, w, tok, got, h = brute_case
    ref, href = _brute_bf16(cfg, w, tok, skip=point)
    dev = max(np.abs(got - ref).max(), np.abs(h - href).max())
    assert dev > 1e-7, f"leaving out {point} is invisible on this case"


@pytest.mark.parametrize("mode", [oracle.OR_EXACT, oracle.OR_BF16])
def test_forward_with_context_equals_whole_sequence(mode):
    """Decoding new tokens after a context given as stored keys/values gives, bit for bit, what the whole-sequence
    forward gives at those positions (the forward with a context is the pinned forward, resumed)."""
    cfg = configs.shrink(configs.TINY, n_layers=2, hidden=64, n_heads=4, n_kv_heads=2, head_dim=16, ffn=96,
                         vocab=128)
    w = synth.model_weights(cfg, seed=23, std=0.1)
    tok = synth.tokens(synth.key(23, 1), 11, cfg["vocab"])
    full, hf = oracle.forward(cfg, w, tok, mode=mode, want_h=True)
    _, _, (k7, v7) = oracle.forward_ctx(cfg, w, tok[:7], mode=mode, want_kv=True)
    res, h, (k4, v4) = oracle.forward_ctx(cfg, w, tok[7:], k7, v7, mode=mode, want_h=True, want_kv=True)
    assert np.array_equal(res, full[7:]) and np.array_equal(h, hf[7:])
    # the keys/values handed on are the stored ones (bf16 values in OR_BF16)
    if mode == oracle.OR_BF16:
        assert np.array_equal(k4, oracle.round_bf16(k4)) and np.array_equal(v7, oracle.round_bf16(v7))
    # a different context changes the result (the context is really read); reordering the context keys does
    # not change the attention sums beyond fp64 rounding, scaling the values does
    res2, _, _ = oracle.forward_ctx(cfg, w, tok[7:], k7, 2 * v7, mode=mode)
    assert not np.array_equal(res2[:, 0], res[:, 0])
