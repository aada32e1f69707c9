"""Kernel-level GPU tests through the C ABI: oracle parity and bitwise batch invariance.

Tolerances (floating point), derived from the arithmetic:
  * fp32-accumulated dot products of length K vs the fp64 oracle:
    |err| <= K * 2^-24 * sum_k |x_k w_k| (worst-case recursive-summation bound);
    index or layout mistakes give errors ~ sum|xw| / sqrt(K), far above it.
  * bf16-rounded outputs add one half-ulp of the result: 2^-8 |y|.
Integer-valued inputs make every product and partial sum exact in fp32, so
there the GPU must match exactly (pins layout and indexing with no rounding).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bi():
    import invariant_deterministic_full_b200 as pkg
    from invariant_deterministic_full_b200 import ops
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ops.device_error(reset=True)
    return ops


def _bf16_dev(a):
    return torch.from_numpy(np.ascontiguousarray(synth.f32_to_bf16_bits(np.asarray(a, np.float32))).view(np.int16)) \
        .cuda().view(torch.bfloat16)


def _f(t):
    return t.float().cpu().numpy().astype(np.float64)


def _after(bi):
    torch.cuda.synchronize()
    assert bi.device_error(reset=True) == 0


# ------------------------------------------------------------------ synthetic generator
def test_device_generator_matches_host(bi):
    k = synth.key(synth.WEIGHT_SEED, 12345)
    rows, cols = 64, 96
    d = torch.empty(rows, cols, dtype=torch.bfloat16, device="cuda")
    bi.synth_fill_bf16(d, rows, cols, k, 0.02)
    host = synth.normal_bf16(k, rows * cols, 0.02).reshape(rows, cols)
    assert np.array_equal(d.view(torch.int16).cpu().numpy().view(np.uint16), host)
    # gate/up interleave: logical row r -> fused row (r//16)*32 + phase*16 + r%16
    gu = torch.zeros(2 * rows, cols, dtype=torch.bfloat16, device="cuda")
    kg, ku = synth.key(1, 2), synth.key(1, 3)
    bi.synth_fill_bf16(gu, rows, cols, kg, 0.02, interleave=16, phase=0)
    bi.synth_fill_bf16(gu, rows, cols, ku, 0.02, interleave=16, phase=1)
    from invariant_deterministic_full_b200.model import interleave_gu
    ref = interleave_gu(synth.normal_bf16(kg, rows * cols).reshape(rows, cols),
                        synth.normal_bf16(ku, rows * cols).reshape(rows, cols))
    assert np.array_equal(gu.view(torch.int16).cpu().numpy().view(np.uint16), ref)
    # paired q/k head order (RoPE partners in one 32-row block), head_dim 128 and 64
    from invariant_deterministic_full_b200.model import pair_heads
    for hd in (128, 64):
        pq = torch.empty(2 * hd, cols, dtype=torch.bfloat16, device="cuda")
        bi.synth_fill_bf16(pq, 2 * hd, cols, kg, 0.02, interleave=-hd)
        ref = pair_heads(synth.normal_bf16(kg, 2 * hd * cols).reshape(2 * hd, cols), hd)
        assert np.array_equal(pq.view(torch.int16).cpu().numpy().view(np.uint16), ref)
    _after(bi)


# ------------------------------------------------------------------ GEMM
GEMM_SHAPES = [(1, 64, 64), (5, 192, 128), (32, 256, 320), (33, 4096, 256), (77, 8256, 128), (40, 16384, 64)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_integer_exact(bi, M, N, K):
    rng = np.random.default_rng(M * 1000 + N + K)
    x = rng.integers(-4, 5, size=(M, K)).astype(np.float32)
    w = rng.integers(-4, 5, size=(N, K)).astype(np.float32)
    exact = (x.astype(np.int64) @ w.T.astype(np.int64)).astype(np.float64)
    xd, wd = _bf16_dev(x), _bf16_dev(w)
    y = bi.gemm(xd, wd, out_dtype=torch.float32)
    assert np.array_equal(_f(y), exact)
    yb = bi.gemm(xd, wd, out_dtype=torch.bfloat16)
    assert np.array_equal(yb.view(torch.int16).cpu().numpy().view(np.uint16),
                          synth.f32_to_bf16_bits(exact.astype(np.float32)))
    # LayerCast: f32 activations, bf16 weights upcast in registers
    y32 = bi.gemm(torch.from_numpy(x).cuda(), wd, mode=1, out_dtype=torch.float32)
    assert np.array_equal(_f(y32), exact)
    _after(bi)


@pytest.mark.parametrize("mode", [0, 1])
def test_gemm_swiglu_epilogue(bi, mode):
    rng = np.random.default_rng(7 + mode)
    M, F, K = 9, 256, 128
    x = rng.integers(-2, 3, size=(M, K)).astype(np.float32)
    wg = rng.integers(-2, 3, size=(F, K)).astype(np.float32) * 0.125
    wu = rng.integers(-2, 3, size=(F, K)).astype(np.float32) * 0.125
    from invariant_deterministic_full_b200.model import interleave_gu
    wgu = interleave_gu(wg, wu)
    g = x.astype(np.float64) @ wg.T
    u = x.astype(np.float64) @ wu.T
    ref = g / (1 + np.exp(-g)) * u
    xd = _bf16_dev(x) if mode == 0 else torch.from_numpy(x).cuda()
    y = bi.gemm(xd, _bf16_dev(wgu), epilogue=1, mode=mode, out_dtype=torch.float32)
    assert np.allclose(_f(y), ref, rtol=1e-6, atol=1e-6)
    _after(bi)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("M,N,K", [(3, 128, 4096), (45, 6144, 512), (8, 4096, 14336)])
def test_gemm_random_vs_oracle(bi, mode, M, N, K):
    rng = np.random.default_rng(11)
    xb = synth.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    wb = synth.f32_to_bf16_bits((0.02 * rng.standard_normal((N, K))).astype(np.float32))
    x = synth.bf16_to_f32(xb)
    ref = oracle.gemm(x.astype(np.float64), wb)
    bound = K * 2.0 ** -24 * (np.abs(x).astype(np.float64) @ np.abs(synth.bf16_to_f32(wb)).astype(np.float64).T)
    xd = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16) if mode == 0 else torch.from_numpy(x).cuda()
    y = _f(bi.gemm(xd, torch.from_numpy(wb.view(np.int16)).cuda().view(torch.bfloat16), mode=mode,
                   out_dtype=torch.float32))
    assert (np.abs(y - ref) <= bound + 1e-30).all()
    _after(bi)


@pytest.mark.parametrize("mode", [0, 1])
def test_gemm_batch_invariance(bi, mode):
    """Row r of x.W^T is bitwise the same whatever the number of rows and the row's position."""
    rng = np.random.default_rng(5)
    N, K = 4096, 1024
    xs = rng.standard_normal((300, K)).astype(np.float32)
    if mode == 0:
        xs = synth.bf16_to_f32(synth.f32_to_bf16_bits(xs))
    w = _bf16_dev(0.02 * rng.standard_normal((N, K)))
    dev = lambda a: (_bf16_dev(a) if mode == 0 else torch.from_numpy(np.ascontiguousarray(a)).cuda())
    full = bi.gemm(dev(xs), w, mode=mode, out_dtype=torch.float32).cpu()
    for M, off in [(1, 0), (1, 57), (4, 30), (31, 2), (32, 40), (33, 17), (64, 36), (129, 40), (257, 43)]:
        part = bi.gemm(dev(xs[off:off + M]), w, mode=mode, out_dtype=torch.float32).cpu()
        assert torch.equal(part, full[off:off + M]), (M, off)
    _after(bi)


@pytest.mark.parametrize("epilogue", [0, 1])
def test_gemm_m_blocking_invariance(bi, epilogue):
    """128-row weight tiles stream each weight stage to four token tiles once M > 32 (M-blocking): a row's
    bits must not depend on which launch shape (one tile or a 128-row group, which slot in it) computed it."""
    rng = np.random.default_rng(15 + epilogue)
    N, K = 8448, 320
    xs = synth.bf16_to_f32(synth.f32_to_bf16_bits(rng.standard_normal((300, K)).astype(np.float32)))
    w = _bf16_dev(0.02 * rng.standard_normal((N, K)))
    full = bi.gemm(_bf16_dev(xs), w, epilogue=epilogue, out_dtype=torch.float32).cpu()
    for M, off in [(1, 0), (1, 299), (31, 5), (32, 100), (33, 17), (96, 3), (128, 150), (129, 40)]:
        part = bi.gemm(_bf16_dev(xs[off:off + M]), w, epilogue=epilogue, out_dtype=torch.float32).cpu()
        assert torch.equal(part, full[off:off + M]), (M, off)
    _after(bi)


def test_gemm_layercast_row_blocks_and_empty(bi):
    """LayerCast runs the exact 3-part split in passes of at most 256 token rows: a row's bits must not depend on
    which pass (or which batch) computed it; M = 0 is a no-op."""
    rng = np.random.default_rng(17)
    N, K = 1024, 512
    xs = rng.standard_normal((600, K)).astype(np.float32)
    w = _bf16_dev(0.02 * rng.standard_normal((N, K)))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    full = bi.gemm(dev(xs), w, mode=1, out_dtype=torch.float32).cpu()
    for M, off in [(1, 599), (255, 0), (256, 100), (257, 3), (300, 290)]:
        part = bi.gemm(dev(xs[off:off + M]), w, mode=1, out_dtype=torch.float32).cpu()
        assert torch.equal(part, full[off:off + M]), (M, off)
    ref = oracle.gemm(xs[:8].astype(np.float64), synth.f32_to_bf16_bits(_f(w).astype(np.float32)))
    bound = K * 2.0 ** -24 * (np.abs(xs[:8]).astype(np.float64) @ np.abs(_f(w)).T)
    assert (np.abs(_f(full[:8]) - ref) <= bound + 1e-30).all()
    empty = bi.gemm(dev(xs[:0]), w, mode=1, out_dtype=torch.float32)
    assert empty.shape == (0, N)
    _after(bi)


def test_gemm_fast_variant_is_not_invariant_but_close(bi):
    rng = np.random.default_rng(6)
    N, K = 4096, 4096
    xs = synth.bf16_to_f32(synth.f32_to_bf16_bits(rng.standard_normal((32, K)).astype(np.float32)))
    w = _bf16_dev(0.02 * rng.standard_normal((N, K)))
    inv = bi.gemm(_bf16_dev(xs), w, out_dtype=torch.float32).cpu()
    f1 = bi.gemm(_bf16_dev(xs[:1]), w, variant=1, out_dtype=torch.float32).cpu()
    f32 = bi.gemm(_bf16_dev(xs), w, variant=1, out_dtype=torch.float32).cpu()
    assert torch.allclose(f1[0], inv[0], rtol=1e-4, atol=1e-4)
    assert not torch.equal(f1[0], f32[0])  # split-K chosen from M changes the bits
    _after(bi)


@pytest.mark.parametrize("d,Hq,Hkv", [(128, 4, 2), (64, 4, 4)])
def test_gemm_rope_kv_epilogue_vs_oracle(bi, d, Hq, Hkv):
    """bi_gemm with BI_EPI_ROPE_KV_APPEND through the C ABI: q (natural order) and the appended k, v rows against
    the oracle's fp64 projection and rotate-half RoPE (or_rope), at positions on both sides of a 256-key chunk;
    every cache row not written stays untouched; v equals the unfused projection bit for bit."""
    from invariant_deterministic_full_b200.model import pair_heads
    from invariant_deterministic_full_b200.ops import KVCache, rope_table
    rng = np.random.default_rng(d + Hq)
    K, theta, cap, L = 256, 10000.0, 600, 2
    QD, KD = Hq * d, Hkv * d
    slot = np.array([0, 2, 1, 2, 0], dtype=np.int32)
    pos = np.array([0, 255, 256, 511, 7], dtype=np.int32)
    M = len(slot)
    x = synth.bf16_to_f32(synth.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32)))
    wq, wk, wv = (synth.f32_to_bf16_bits((0.05 * rng.standard_normal((n, K))).astype(np.float32))
                  for n in (QD, KD, KD))
    wf = np.concatenate([pair_heads(wq, d), pair_heads(wk, d), wv])
    kv = KVCache(3, L, Hkv, cap, d)
    table = rope_table(cap, d, theta)
    sd, pd = torch.from_numpy(slot).cuda(), torch.from_numpy(pos).cuda()
    wd = torch.from_numpy(wf.view(np.int16)).cuda().view(torch.bfloat16)
    q = bi.gemm_rope_kv(_bf16_dev(x), wd, table, cap, kv, 1, sd, pd, Hq)
    torch.cuda.synchronize()
    # oracle: fp64 projection then rotate-half RoPE at each row's position
    x64 = x.astype(np.float64)
    qr = oracle.gemm(x64, wq)
    kr = oracle.gemm(x64, wk)
    vr = oracle.gemm(x64, wv)
    qr = np.stack([oracle.rope(qr[m], Hq, d, int(pos[m]), theta) for m in range(M)])
    kr = np.stack([oracle.rope(kr[m], Hkv, d, int(pos[m]), theta) for m in range(M)])
    ax = np.abs(x64)
    bq = K * 2.0 ** -24 * (ax @ np.abs(synth.bf16_to_f32(wq)).T)
    bk = K * 2.0 ** -24 * (ax @ np.abs(synth.bf16_to_f32(wk)).T)
    bv = K * 2.0 ** -24 * (ax @ np.abs(synth.bf16_to_f32(wv)).T)
    # a rotated element mixes two products: twice the projection bound of its pair, the f32 table (2^-24
    # relative) and the final bf16 rounding (half an ulp, 2^-8 relative)
    pair = lambda b, H: np.maximum(b, b.reshape(M, H, 2, d // 2)[:, :, ::-1].reshape(M, H * d))
    gq = _f(q)
    assert (np.abs(gq - qr) <= 2.0 ** -8 * np.abs(qr) + 2 * pair(bq, Hq) + 2.0 ** -22 * np.abs(qr) + 1e-7).all()
    kc, vc = _f(kv.k), _f(kv.v)
    for m in range(M):
        gk = kc[slot[m], 1, :, pos[m]].reshape(KD)
        gv = vc[slot[m], 1, :, pos[m]].reshape(KD)
        assert (np.abs(gk - kr[m]) <= 2.0 ** -8 * np.abs(kr[m]) + 2 * pair(bk, Hkv)[m] + 1e-7).all(), m
        assert (np.abs(gv - vr[m]) <= 2.0 ** -8 * np.abs(vr[m]) + bv[m] + 1e-7).all(), m
    written = np.zeros((3, L, cap), dtype=bool)
    written[slot, 1, pos] = True
    assert not np.any(kc.transpose(0, 1, 3, 2, 4)[~written]) and not np.any(vc.transpose(0, 1, 3, 2, 4)[~written])
    # the unfused route (f32 projection, then the RoPE/append kernel) rotates with the same rounding: same bits
    qkv32 = bi.gemm(_bf16_dev(x), wd, out_dtype=torch.float32)
    kv2 = KVCache(3, L, Hkv, cap, d)
    q2 = bi.rope_kv_append(qkv32, table, cap, kv2, 1, sd, pd, Hq, qk_paired=True)
    torch.cuda.synchronize()
    assert torch.equal(kv2.v, kv.v) and torch.equal(kv2.k, kv.k) and torch.equal(q2, q)
    # the same rows inside a launch of more than 32 rows (the tcgen05 kernel) give the same bits
    reps = 9  # 45 rows: the five tokens repeated, each copy at its own slot and position
    slot_r = np.concatenate([slot + 0 * i for i in range(reps)]).astype(np.int32)
    pos_r = np.concatenate([pos + 0 * i for i in range(reps)]).astype(np.int32)
    kv3 = KVCache(3, L, Hkv, cap, d)
    xr = np.concatenate([x] * reps)
    q3 = bi.gemm_rope_kv(_bf16_dev(xr), wd, table, cap, kv3, 1, torch.from_numpy(slot_r).cuda(),
                         torch.from_numpy(pos_r).cuda(), Hq)
    torch.cuda.synchronize()
    assert torch.equal(q3[:M], q) and torch.equal(q3[-M:], q)
    assert torch.equal(kv3.k, kv.k) and torch.equal(kv3.v, kv.v)
    _after(bi)


# ------------------------------------------------------------------ RMSNorm
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("H", [256, 3584, 4096])
def test_rmsnorm_vs_oracle_and_invariance(bi, mode, H):
    rng = np.random.default_rng(H + mode)
    M = 19
    x = rng.standard_normal((M, H)).astype(np.float32) * 3
    r = rng.standard_normal((M, H)).astype(np.float32)
    gamma = synth.f32_to_bf16_bits((1 + 0.1 * rng.standard_normal(H)).astype(np.float32))
    dt = torch.float32 if mode else torch.bfloat16
    xd = torch.from_numpy(x).cuda().to(dt)
    rd = torch.from_numpy(r).cuda().to(dt)
    gd = torch.from_numpy(gamma.view(np.int16)).cuda().view(torch.bfloat16)
    rout = torch.empty_like(rd)
    y, y32 = bi.rmsnorm(xd, gd, 1e-5, residual_in=rd, residual_out=rout, want_f32=True, mode=mode)
    rsum = _f(xd) + _f(rd)
    if mode == 0:
        rsum = oracle.round_bf16(rsum)
        assert np.array_equal(_f(rout), rsum)
    else:
        assert np.allclose(_f(rout), rsum, rtol=2 ** -23, atol=0)
    ref = oracle.rmsnorm(_f(rout), gamma, 1e-5)
    assert np.allclose(_f(y32), ref, rtol=3e-6, atol=1e-7)
    if mode == 0:
        assert np.allclose(_f(y), ref, rtol=2 ** -8 + 3e-6, atol=1e-7)
    # invariance: each row alone equals the batched row
    for i in (0, 7, 18):
        ro = torch.empty_like(rd[i:i + 1])
        yi, y32i = bi.rmsnorm(xd[i:i + 1].contiguous(), gd, 1e-5, residual_in=rd[i:i + 1].contiguous(),
                              residual_out=ro, want_f32=True, mode=mode)
        assert torch.equal(yi, y[i:i + 1]) and torch.equal(y32i, y32[i:i + 1]) and torch.equal(ro, rout[i:i + 1])
    _after(bi)


# ------------------------------------------------------------------ attention
def _make_cache(bi, mode, n_slots, Hkv, cap, d, fill_upto, seed):
    rng = np.random.default_rng(seed)
    kv = bi.KVCache(n_slots, 1, Hkv, cap, d, mode=mode)
    k = rng.standard_normal((n_slots, 1, Hkv, cap, d)).astype(np.float32)
    v = rng.standard_normal((n_slots, 1, Hkv, cap, d)).astype(np.float32)
    if mode == 0:
        k = synth.bf16_to_f32(synth.f32_to_bf16_bits(k))
        v = synth.bf16_to_f32(synth.f32_to_bf16_bits(v))
    kv.k.copy_(torch.from_numpy(k))
    kv.v.copy_(torch.from_numpy(v))
    return kv, k, v


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("Hq,Hkv,d", [(32, 8, 128), (4, 4, 64), (28, 4, 128)])
def test_attention_vs_oracle(bi, mode, Hq, Hkv, d):
    cap = 1200
    kv, k, v = _make_cache(bi, mode, 3, Hkv, cap, d, cap, seed=Hq + d + mode)
    rng = np.random.default_rng(3)
    # a mixed batch: decode tokens of slots 0 and 2, and a 5-token prefill block of slot 1
    slots = np.array([0, 1, 1, 1, 1, 1, 2], dtype=np.int32)
    pos = np.array([700, 250, 251, 252, 253, 254, 1100], dtype=np.int32)
    T = len(slots)
    q = rng.standard_normal((T, Hq * d)).astype(np.float32)
    dt = torch.float32 if mode else torch.bfloat16
    qd = torch.from_numpy(q).cuda().to(dt)
    scale = 1.0 / math.sqrt(d)
    out = _f(bi.attention(qd, kv, 0, torch.from_numpy(slots).cuda(), torch.from_numpy(pos).cuda(), slots, pos, Hq,
                          np.float32(scale), mode=mode))
    qf = _f(qd)
    G = Hq // Hkv
    for t in range(T):
        for h in (0, Hq // 2 + 1, Hq - 1):
            hk = h // G
            ref = oracle.attention_query(qf[t, h * d:(h + 1) * d], k[slots[t], 0, hk, :pos[t] + 1],
                                         v[slots[t], 0, hk, :pos[t] + 1], float(np.float32(scale)))
            got = out[t, h * d:(h + 1) * d]
            tol = 2e-5 * np.abs(v[slots[t], 0, hk]).max() + (2 ** -8 * np.abs(ref) if mode == 0 else 0)
            assert (np.abs(got - ref) <= tol).all(), (t, h, np.abs(got - ref).max())
    _after(bi)


@pytest.mark.parametrize("mode", [0, 1])
def test_attention_invariance_decode_vs_prefill(bi, mode):
    """A query's output is bitwise the same alone, inside a prefill block, and beside other slots."""
    Hq, Hkv, d, cap = 32, 8, 128, 800
    kv, _, _ = _make_cache(bi, mode, 4, Hkv, cap, d, cap, seed=9 + mode)
    rng = np.random.default_rng(4)
    n = 40
    base = 230  # block crosses the chunk boundary at 256
    q = rng.standard_normal((n, Hq * d)).astype(np.float32)
    dt = torch.float32 if mode else torch.bfloat16
    qd = torch.from_numpy(q).cuda().to(dt)
    run = lambda qq, s, p: bi.attention(qq, kv, 0, torch.from_numpy(s).cuda(), torch.from_numpy(p).cuda(), s, p, Hq,
                                        0.08838834764831845, mode=mode).cpu()
    slots = np.full(n, 2, dtype=np.int32)
    pos = np.arange(base, base + n, dtype=np.int32)
    block = run(qd, slots, pos)
    for i in (0, 5, 25, 26, 39):
        alone = run(qd[i:i + 1].contiguous(), slots[i:i + 1], pos[i:i + 1])
        assert torch.equal(alone[0], block[i]), i
    # beside decode tokens of other slots
    s2 = np.array([0, 2, 3], dtype=np.int32)
    p2 = np.array([17, base + 25, 790], dtype=np.int32)
    q2 = torch.stack([qd[0], qd[25], qd[1]])
    mixed = run(q2, s2, p2)
    assert torch.equal(mixed[1], block[25])
    _after(bi)


def test_attention_invariance_across_work_splits(bi):
    """The tensor-core kernel cuts each (query block, kv head)'s chunks into segments by how many units a launch
    has: one segment merged inside the CTA (large decode batches), one chunk per CTA (a token alone) and
    multi-chunk segments (a few tokens at long context).  All must give the same bits, also against the oracle."""
    Hq, Hkv, d, cap, n = 32, 8, 128, 3072, 24
    kv, k, v = _make_cache(bi, 0, n, Hkv, cap, d, cap, seed=21)
    rng = np.random.default_rng(22)
    q = torch.from_numpy(rng.standard_normal((n, Hq * d)).astype(np.float32)).cuda().to(torch.bfloat16)
    slots = np.arange(n, dtype=np.int32)
    pos = np.concatenate([[cap - 1, 0, 255, 256, 2047], rng.integers(0, cap, n - 5)]).astype(np.int32)
    scale = np.float32(1.0 / math.sqrt(d))
    run = lambda idx: bi.attention(q[idx].contiguous(), kv, 0, torch.from_numpy(slots[idx]).cuda(),
                                   torch.from_numpy(pos[idx]).cuda(), slots[idx], pos[idx], Hq, scale).cpu()
    full = run(np.arange(n))                  # 192 units: one segment per CTA, merged in the CTA
    four = run(np.arange(4))                  # 32 units: segments of several chunks
    for i in range(n):
        alone = run(np.array([i]))            # 8 units: one chunk per CTA
        assert torch.equal(alone[0], full[i]), i
        if i < 4:
            assert torch.equal(four[i], full[i]), i
    qf = _f(q)
    out = _f(full)
    for t in (0, 3, 4):
        for h in (0, 17):
            ref = oracle.attention_query(qf[t, h * d:(h + 1) * d], k[slots[t], 0, h // 4, :pos[t] + 1],
                                         v[slots[t], 0, h // 4, :pos[t] + 1], float(scale))
            tol = 2e-5 * np.abs(v[slots[t], 0, h // 4]).max() + 2 ** -8 * np.abs(ref)
            assert (np.abs(out[t, h * d:(h + 1) * d] - ref) <= tol).all(), (t, h)
    _after(bi)


# ------------------------------------------------------------------ LM head
def _h_rows(B, H, seed=7):
    return synth.hidden_states(seed, B, H)


@pytest.mark.parametrize("mode", [0, 1])
def test_lmhead_vs_oracle_small_vocab(bi, mode):
    H, V, B = 512, 4096, 24
    rng = np.random.default_rng(8)
    Wb = synth.f32_to_bf16_bits((0.02 * rng.standard_normal((V, H))).astype(np.float32))
    # scale logits up so both flagged and unflagged rows occur
    h = _h_rows(B, H) * 4
    hd = torch.from_numpy(h).cuda()
    Wd = torch.from_numpy(Wb.view(np.int16)).cuda().view(torch.bfloat16)
    tgt = rng.integers(0, V, size=B).astype(np.int32)
    tgt[::3] = -1
    o = bi.lmhead_logprob(hd, Wd, torch.from_numpy(tgt).cuda(), threshold=0.1, mode=mode, want_logits=True)
    o = {k: v.cpu().numpy() for k, v in o.items()}
    hb = synth.bf16_to_f32(synth.f32_to_bf16_bits(h)).astype(np.float64) if mode == 0 else h.astype(np.float64)
    res_main, z_main = oracle.lmhead(hb, Wb, target=tgt, want_logits=True)
    res_exact, _ = oracle.lmhead(h.astype(np.float64), Wb, target=tgt)
    bound = H * 2.0 ** -24 * (np.abs(hb) @ np.abs(synth.bf16_to_f32(Wb)).astype(np.float64).T)
    assert (np.abs(o["logits"] - z_main) <= bound + 1e-30).all()
    # margin and the flag come from the main pass
    assert np.allclose(o["margin"], res_main[:, 3], atol=2e-5)
    if mode == 0:
        assert np.array_equal(o["recomputed"], (o["margin"] < 0.1).astype(np.uint8))
        assert 0 < o["recomputed"].sum() < B
    else:
        assert (o["recomputed"] == 0).all()
    for b in range(B):
        ref = res_exact[b] if (mode == 1 or o["recomputed"][b]) else res_main[b]
        assert abs(o["logprob"][b] - ref[1]) <= 1e-5 * abs(ref[1]) + 1e-6, b
        assert abs(o["lse"][b] - ref[0]) <= 1e-5 * abs(ref[0]) + 1e-6, b
        if ref[3] > 1e-4:
            assert o["argmax"][b] == int(ref[2]), b
    _after(bi)


@pytest.mark.parametrize("B", [4, 24, 64])  # one-pass and second-pass recompute layouts
def test_lmhead_recompute_enabled_but_no_row_flagged(bi, B):
    """With the recompute on but no row under the threshold, the recompute stage has a device-side row count of 0:
    it must finish cleanly (no wait running out) and leave the main-pass results.  Every row's top logit is made
    to stand out: W row 7b + 1 is bf16(h_b / |h_b|), so z = |h_b| (about 90) there against about 2 elsewhere,
    and no margin can fall under the threshold 1.0."""
    H, V = 512, 4096
    rng = np.random.default_rng(31)
    h = _h_rows(B, H) * 4
    Wf = 0.02 * rng.standard_normal((V, H))
    for b in range(B):
        Wf[7 * b + 1] = h[b] / np.linalg.norm(h[b])
    W = _bf16_dev(Wf)
    hd = torch.from_numpy(h).cuda()
    off = bi.lmhead_logprob(hd, W, None, threshold=0.0)
    on = bi.lmhead_logprob(hd, W, None, threshold=1.0)
    torch.cuda.synchronize()
    assert int(on["recomputed"].sum()) == 0
    assert float(on["margin"].min()) > 50.0
    assert torch.equal(on["argmax"].cpu(), torch.arange(B, dtype=torch.int32) * 7 + 1)
    for k in ("logprob", "lse", "argmax", "margin"):
        assert torch.equal(on[k], off[k]), k
    _after(bi)


def test_lmhead_layercast_full_size_tensor_core_blocks(bi):
    """LayerCast LM head at hidden 4096, vocab 128256 on the tensor cores, in vocabulary blocks: the logits are
    bitwise those of one unblocked LayerCast bi_gemm over the whole vocabulary, every row is bitwise equal across
    batch 1..64, and sampled rows match the exact oracle within the fp32 summation bound."""
    H, V = 4096, 128256
    W = torch.empty(V, H, dtype=torch.bfloat16, device="cuda")
    kW = synth.key(synth.WEIGHT_SEED, synth.S_LMHEAD)
    bi.synth_fill_bf16(W, V, H, kW, 0.02)
    h = _h_rows(64, H)
    hd = torch.from_numpy(h).cuda()
    ref = bi.lmhead_logprob(hd, W, None, 0.1, mode=1, want_logits=True)
    z = bi.gemm(hd, W, mode=1, out_dtype=torch.float32)
    assert torch.equal(ref["logits"], z)
    assert int(ref["recomputed"].sum()) == 0
    ref = {k: v.cpu() for k, v in ref.items()}
    for B in (1, 3, 11, 32, 40):
        for off in (0, 64 - B):
            o = bi.lmhead_logprob(hd[off:off + B].contiguous(), W, None, 0.1, mode=1)
            for k in ("logprob", "lse", "argmax", "margin"):
                assert torch.equal(o[k].cpu(), ref[k][off:off + B]), (B, off, k)
    Wb = synth.normal_bf16(kW, V * H).reshape(V, H)
    rows = [0, 33, 63]
    res, zx = oracle.lmhead(h[rows].astype(np.float64), Wb, want_logits=True)
    Wa = np.abs(synth.bf16_to_f32(Wb)).astype(np.float64)
    for i, r in enumerate(rows):
        bound = (H + 2) * 2.0 ** -24 * (Wa @ np.abs(h[r]).astype(np.float64))
        assert (np.abs(ref["logits"][r].numpy() - zx[i]) <= bound).all(), r
        assert abs(ref["logprob"][r].item() - res[i][1]) <= 1e-5 * abs(res[i][1]) + 1e-6, r
        assert abs(ref["lse"][r].item() - res[i][0]) <= 1e-5 * abs(res[i][0]) + 1e-6, r
    _after(bi)


def test_lmhead_full_size_invariance_and_samples(bi):
    """LM head alone at hidden 4096, vocab 128256: each row bitwise equal across batch 1..256."""
    H, V = 4096, 128256
    W = torch.empty(V, H, dtype=torch.bfloat16, device="cuda")
    kW = synth.key(synth.WEIGHT_SEED, synth.S_LMHEAD)
    bi.synth_fill_bf16(W, V, H, kW, 0.02)
    h = _h_rows(256, H)
    hd = torch.from_numpy(h).cuda()
    ref = {k: v.cpu() for k, v in bi.lmhead_logprob(hd, W, None, 0.1).items()}
    for B in (1, 2, 4, 8, 10, 11, 16, 32, 42, 43, 64, 128):  # one-pass recompute up to 42 rows, two passes above
        for off in (0, 256 - B):
            o = bi.lmhead_logprob(hd[off:off + B].contiguous(), W, None, 0.1)
            for k in ("logprob", "lse", "argmax", "margin", "recomputed"):
                assert torch.equal(o[k].cpu(), ref[k][off:off + B]), (B, off, k)
    # sampled oracle parity on 3 rows (host weights regenerated from the same seed)
    Wb = synth.normal_bf16(kW, V * H).reshape(V, H)
    rows = [0, 100, 255]
    recomputed = ref["recomputed"].numpy()
    hb = synth.bf16_to_f32(synth.f32_to_bf16_bits(h[rows])).astype(np.float64)
    res_main, _ = oracle.lmhead(hb, Wb)
    res_exact, _ = oracle.lmhead(h[rows].astype(np.float64), Wb)
    for i, r in enumerate(rows):
        rr = res_exact[i] if recomputed[r] else res_main[i]
        assert abs(ref["logprob"][r].item() - rr[1]) <= 1e-5 * abs(rr[1]) + 1e-6
        assert abs(ref["margin"][r].item() - res_main[i][3]) <= 1e-4
    rate = recomputed.mean()
    assert 0.0 < rate < 1.0
    _after(bi)
