#!/usr/bin/env python
"""Batch-invariant greedy decode throughput on the Llama-3.1-8B-shaped random-init model.

One step = one bi_decode_step over a batch of B decode tokens (every row of the
hot path: embed, 32 x [RMSNorm, QKV GEMM + RoPE/KV append, chunked attention +
merge, O GEMM, RMSNorm, gate/up GEMM + SwiGLU, down GEMM], final RMSNorm, LM
head + logsumexp/top-2 merge + selective FP32 recompute) plus the greedy
feedback (next ids, positions) -- replayed as one CUDA graph, inputs resident
in HBM.  value = B * K / (device time of K steps), max over ranks, summed over
ranks (replicas: every rank decodes its own batch, no collective on the data
path).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--batch B] [--impl ours|reference]

--impl reference times the fp64 CPU oracle (the only other implementation of
this computation here) on the host cores, on a bounded sample of the same
workload scaled to tok/s.
"""
import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "batch-invariant decode tok/s (8B shape, bs 1-32); % of HBM roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=4)
    ap.add_argument("--batch", type=int, default=32)
    ap.add_argument("--prompt", type=int, default=512)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--mode", default="bf16", choices=["bf16", "layercast"])
    ap.add_argument("--sweep", default="1,4,8,16,32", help="extra batch sizes to report ('' = none)")
    ap.add_argument("--no-fast", action="store_true", help="skip the non-invariant FAST-variant comparison")
    ap.add_argument("--no-layercast", action="store_true", help="skip the LayerCast-mode line")
    ap.add_argument("--no-lmhead", action="store_true", help="skip the LM-head-alone timing")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill throughput line")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling case: the 8B shape with this many layers (0 = all 32; not the headline workload)")
    return ap.parse_args()


# ---------------------------------------------------------------- distributed plumbing
def dist_init(args, backend="nccl"):
    """One process per GPU (torchrun env).  Replicas only: the process group carries the barrier around the timed
    region and the max-over-ranks of the measured time, never data."""
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws):
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(units_per_rank, ms_max, ws):
    """Whole-job throughput of ws replicas: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * ws / (ms_max / 1e3)


# ---------------------------------------------------------------- clocks during the timed region
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index, self.rows, self.proc = index, [], None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        time.sleep(0.25)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([c.strip() for c in line.split(",")])

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in self.rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
                for n, v in zip(names, r[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                pass
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- roofline bookkeeping
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def step_bytes(cfg, B, ctx_lens, f32_kv=False):
    """Algorithmic bytes one decode step must move: every weight once, the embedding rows, the KV rows read
    (positions 0..ctx of every sequence, every layer) and written."""
    L, H, Hq, Hkv, d, F, V = (cfg["n_layers"], cfg["hidden"], cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"],
                              cfg["ffn"], cfg["vocab"])
    w = 2 * (L * ((Hq + 2 * Hkv) * d * H + H * Hq * d + 3 * F * H + 2 * H) + V * H + H)
    kv_row = L * Hkv * d * 2 * (4 if f32_kv else 2)  # k and v of one position, all layers
    kv = sum((c + 1) * kv_row for c in ctx_lens) + B * kv_row
    return w + B * H * 2 + kv


# DRAM bytes (read + write) of the four projection GEMM launches of one decoder layer at batch 32, from one ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum) of the same shapes on the 2-layer 8B-width case (the
# weights per launch do not depend on the layer count).  Valid only for the GEMM kernel source that was captured,
# recognised by gemm_source_digest; None until a capture of this source.
GEMM_TRAFFIC = {"gemm_source_sha256": "78b8680b7f0e5605458b68383829e3543da3c923c0f7aff97d799c6585c493f3",
                "batch": 32, "per_layer_bytes": 445704448}

CSRC = os.path.join(ROOT, "invariant_deterministic_full_b200", "csrc")


def gemm_source_digest(mma_text, plan_text):
    """sha256 of the code (comments and whitespace removed) that decides the dominant kernel's memory traffic: the
    whole mma.sync kernel file (the projections of a decode step at <= 32 token rows run on it), and the launch
    planning and dispatch of gemm.cuh (from the tile plan to the end of the bf16 dispatcher).  The tcgen05 kernel
    (prefill), the FAST split heuristic, workspace sizing and the LayerCast kernels are left out."""
    import hashlib
    import re
    a = plan_text.index("struct TcPlan {")
    b = plan_text.index("// LayerCast on tensor cores: rows of x per pass")
    c0 = plan_text.index("template <int BN, int MT, int KS, int EPI>\nstatic int launch_tc_t")
    c1 = plan_text.index("int gemm_f32(")
    code = re.sub(r"/\*.*?\*/", " ", mma_text + plan_text[a:b] + plan_text[c0:c1], flags=re.S)
    code = re.sub(r"//[^\n]*", " ", code)
    return hashlib.sha256(" ".join(code.split()).encode()).hexdigest()


def current_gemm_digest():
    txt = lambda n: open(os.path.join(CSRC, n)).read()
    return gemm_source_digest(txt("gemm_mma.cuh"), txt("gemm.cuh"))


def gemm_traffic_per_launch(cfg, B):
    """Measured DRAM bytes per launch of the timed GEMM set, or None when they no longer apply."""
    try:
        h = current_gemm_digest()
    except (OSError, ValueError):
        return None
    if (GEMM_TRAFFIC["gemm_source_sha256"] is None or h != GEMM_TRAFFIC["gemm_source_sha256"]
            or B != GEMM_TRAFFIC["batch"] or cfg["hidden"] != 4096):
        return None
    return GEMM_TRAFFIC["per_layer_bytes"] / 4


def gemm_bytes(cfg, B):
    """Algorithmic bytes of the projection GEMM launches of one bf16 decode step (weights + inputs + outputs):
    QKV, O, gate/up (SwiGLU output) and down of every layer."""
    L, H, Hq, Hkv, d, F, V = (cfg["n_layers"], cfg["hidden"], cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"],
                              cfg["ffn"], cfg["vocab"])
    QKV = (Hq + 2 * Hkv) * d
    per_layer = [(QKV, H, 2), (H, Hq * d, 2), (2 * F, H, 2), (H, F, 2)]  # (N, K, output bytes per element)
    tot, n = 0, 0
    for N, K, ob in per_layer:
        tot += L * (N * K * 2 + B * K * 2 + B * (N // 2 if N == 2 * F else N) * ob)
        n += L
    return tot, n


# ---------------------------------------------------------------- our arm
def run_decode(m, B, P, K, W, ws, rank, graph=True):
    """Prefill B prompts of P tokens (one batched call), then time K greedy decode steps (CUDA graph replay)."""
    import numpy as np
    import torch

    import synth
    from invariant_deterministic_full_b200 import ops

    V = m.cfg["vocab"]
    prompts = [synth.prompt_tokens(1000 * rank + r, P, V) for r in range(B)]
    ids = np.concatenate(prompts).astype(np.int32)
    slots = np.repeat(np.arange(B), P).astype(np.int32)
    pos = np.tile(np.arange(P), B).astype(np.int32)
    lm = np.full(B * P, -1, dtype=np.int32)
    lm[np.arange(B) * P + P - 1] = np.arange(B)
    o = m.step(ids, slots, pos, lm)
    dev = m.device
    ids_d = o["argmax"].clone()
    pos_d = torch.full((B,), P, dtype=torch.int32, device=dev)
    slot_d = torch.arange(B, dtype=torch.int32, device=dev)
    lm_d = torch.arange(B, dtype=torch.int32, device=dev)
    slots_h = torch.arange(B, dtype=torch.int32)
    total = W + K + 1
    pos_plan = torch.full((B,), P + total - 1, dtype=torch.int32)  # positions the replays will reach
    out = m.alloc_out(B)
    m.workspace(B, B, P + total)

    def one_step():
        m.step_dev(B, ids_d, slot_d, pos_d, slots_h, pos_plan, lm_d, B, None, out, max_pos=P + total)
        ops.greedy_advance(out["argmax"], ids_d, pos_d)

    # one eager step (library one-time set-up happens outside capture), then capture
    from invariant_deterministic_full_b200._lib import lib
    c0 = lib.bi_launch_count()
    one_step()
    launches = lib.bi_launch_count() - c0
    torch.cuda.synchronize()
    if graph:
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(g, stream=s):
            one_step()
        torch.cuda.current_stream().wait_stream(s)
        run = g.replay
    else:
        run = one_step
    for _ in range(W):
        run()
    torch.cuda.synchronize()
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record()
        for _ in range(K):
            run()
        e1.record()
        e1.synchronize()
    ms = e0.elapsed_time(e1)
    torch.cuda.synchronize()
    err = ops.device_error()
    if err:
        raise RuntimeError(f"device error flags 0x{err:x}")
    ctx_first = P + 1 + W  # position of the first timed step
    ctx_lens = [ctx_first + i for i in range(K)]
    rec = dict(ms=ms, launches=launches, clocks=clk.summary(), ctx_lens=ctx_lens,
               recompute_rate=float(out["recomputed"].float().mean().item()))
    if graph:
        del g
    return rec


def prefill_flops(cfg, B, P):
    """FLOPs of one batched prefill of B prompts of P tokens with the LM head on each prompt's last token:
    2 x projection weights x tokens, causal attention (q.k and p.v over positions 0..t of every q head), LM head."""
    L, H, Hq, Hkv, d, F, V = (cfg["n_layers"], cfg["hidden"], cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"],
                              cfg["ffn"], cfg["vocab"])
    proj = (Hq + 2 * Hkv) * d * H + H * Hq * d + 3 * F * H
    att = 2 * 2 * d * Hq * L * B * (P * (P + 1) // 2)
    return 2 * L * proj * B * P + att + 2 * V * H * B


def time_prefill(m, B, P, rank, reps=2):
    """Device time of the batched prefill of B prompts of P tokens (one bi_decode_step over B*P tokens), averaged
    over reps identical calls after an untimed one; every call writes the same KV rows.  Returns (ms, clocks sampled
    during the timed calls)."""
    import numpy as np
    import torch
    import synth
    V = m.cfg["vocab"]
    prompts = [synth.prompt_tokens(1000 * rank + r, P, V) for r in range(B)]
    ids = np.concatenate(prompts).astype(np.int32)
    slots = np.repeat(np.arange(B), P).astype(np.int32)
    pos = np.tile(np.arange(P), B).astype(np.int32)
    lm = np.full(B * P, -1, dtype=np.int32)
    lm[np.arange(B) * P + P - 1] = np.arange(B)
    m.step(ids, slots, pos, lm)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record()
        for _ in range(reps):
            m.step(ids, slots, pos, lm)
        e1.record()
        e1.synchronize()
    return e0.elapsed_time(e1) / reps, clk.summary()


def time_lmhead(m, batches=(1, 4, 32, 256), reps=20):
    """The LM-head logprob alone (hidden 4096, vocab 128256): per batch, the time of one bi_lmhead_logprob call with
    the selective recompute at threshold 0.1 and with it disabled, the recompute rate, and the weight GB/s."""
    import ctypes
    import torch
    import synth
    from invariant_deterministic_full_b200._lib import lib
    W = m.w["lm_head"]
    V, H = W.shape
    dev = m.device
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    res = {}
    for B in batches:
        h = torch.from_numpy(synth.hidden_states(7, B, H)).to(dev)
        out = [torch.empty(B, dtype=t, device=dev) for t in (torch.float32, torch.float32, torch.int32, torch.float32,
                                                               torch.uint8)]
        wsb = lib.bi_lmhead_workspace_size(B, H, V, 0)
        ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
        p = lambda t: ctypes.c_void_p(t.data_ptr())

        def call(th):
            rc = lib.bi_lmhead_logprob(p(h), p(W), None, B, H, V, th, 0, *[p(o) for o in out], None, p(ws), wsb, st)
            assert rc == 0, lib.bi_last_error()

        row = {}
        for name, th in (("recompute", 0.1), ("no_recompute", 0.0)):
            for _ in range(3):
                call(th)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                call(th)
            e1.record()
            e1.synchronize()
            us = e0.elapsed_time(e1) / reps * 1e3
            row[name + "_us"] = round(us, 1)
            if name == "recompute":
                row["recompute_rate"] = round(float(out[4].float().mean().item()), 4)
        row["weight_GBps"] = round(V * H * 2 / (row["no_recompute_us"] * 1e-6) / 1e9, 1)
        row["recompute_overhead"] = round(row["recompute_us"] / row["no_recompute_us"] - 1, 4)
        res[str(B)] = row
    return res


def time_gemms(m, B, reps=3):
    """Duration of the projection GEMM launches of one decode step, timed alone with CUDA events on the
    launching stream (all layers' QKV, O, gate/up and down, B token rows).  The launches are captured once in a
    CUDA graph and replayed, so the host never paces the GPU between them."""
    import torch
    from invariant_deterministic_full_b200 import ops
    cfg, w, dev = m.cfg, m.w, m.device
    L, H, F = cfg["n_layers"], cfg["hidden"], cfg["ffn"]
    QD = cfg["n_heads"] * cfg["head_dim"]
    x_h, x_q, x_f = (torch.randn(B, n, device=dev).to(torch.bfloat16) for n in (H, QD, F))
    o_qkv = torch.empty(B, w["w_qkv"].shape[1], dtype=torch.bfloat16, device=dev)
    o_h = torch.empty(B, H, dtype=torch.bfloat16, device=dev)
    o_f = torch.empty(B, F, dtype=torch.bfloat16, device=dev)

    def once():
        for l in range(L):
            ops.gemm(x_h, w["w_qkv"][l], out=o_qkv)
            ops.gemm(x_q, w["w_o"][l], out=o_h)
            ops.gemm(x_h, w["w_gu"][l], epilogue=1, out=o_f)
            ops.gemm(x_f, w["w_down"][l], out=o_h)

    once()  # one-time library set-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=st):
        once()
    torch.cuda.current_stream().wait_stream(st)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    e1.synchronize()
    del g
    return e0.elapsed_time(e1) / reps


def run_e2e(m, B, P, K, rank, graph=True):
    """Same metric through the public API with host buffers: per step an H2D copy of the step's inputs from
    pinned host memory, bi_decode_step, and a D2H read of the step's results; the host feeds the next ids.
    graph=True: the step is bi_decode_step captured once in a CUDA graph (after one eager step) and replayed,
    the way a serving loop issues it; graph=False: bi_decode_step is called eagerly every step."""
    import numpy as np
    import torch
    import synth
    V = m.cfg["vocab"]
    dev = m.device
    prompts = [synth.prompt_tokens(1000 * rank + 500 + r, P, V) for r in range(B)]
    ids = np.concatenate(prompts).astype(np.int32)
    slots = np.repeat(np.arange(B), P).astype(np.int32)
    pos = np.tile(np.arange(P), B).astype(np.int32)
    lm = np.full(B * P, -1, dtype=np.int32)
    lm[np.arange(B) * P + P - 1] = np.arange(B)
    o = m.step(ids, slots, pos, lm)
    nxt = o["argmax"].cpu().numpy()
    h_in = torch.empty(4, B, dtype=torch.int32).pin_memory()  # ids, slot, pos, lm_row
    h_out_ids = torch.empty(B, dtype=torch.int32).pin_memory()
    h_out_lp = torch.empty(B, dtype=torch.float32).pin_memory()
    d_in = torch.empty(4, B, dtype=torch.int32, device=dev)
    out = m.alloc_out(B)
    slots_h = torch.arange(B, dtype=torch.int32)
    max_pos = P + K + 1
    pos_plan = torch.full((B,), max_pos, dtype=torch.int32)  # the last position the steps reach, for planning
    m.workspace(B, B, max_pos)

    def one_step():
        m.step_dev(B, d_in[0], d_in[1], d_in[2], slots_h, pos_plan, d_in[3], B, None, out, max_pos=max_pos)

    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = P
    run, g = one_step, None
    for it in range(K + 1):
        if it == 1:
            if graph:  # capture after the eager first step (one-time library set-up stays outside the capture)
                g = torch.cuda.CUDAGraph()
                s = torch.cuda.Stream()
                s.wait_stream(st)
                with torch.cuda.graph(g, stream=s):
                    one_step()
                st.wait_stream(s)
                run = g.replay
            e0.record()
        h_in[0].copy_(torch.from_numpy(nxt))
        h_in[1].copy_(slots_h)
        h_in[2].fill_(cur)
        h_in[3].copy_(torch.arange(B, dtype=torch.int32))
        d_in.copy_(h_in, non_blocking=True)
        run()
        h_out_ids.copy_(out["argmax"], non_blocking=True)
        h_out_lp.copy_(out["logprob"], non_blocking=True)
        st.synchronize()
        nxt = h_out_ids.numpy().copy()
        cur += 1
    e1.record()
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    if g is not None:
        del g
    return dict(ms=ms, h2d=4 * B * 4, d2h=B * 4 + B * 4)


class CpuSample:
    """The fp64 oracle as it stands, on the host cores: NEW teacher-forced decode tokens at the positions of the
    timed steps (after a PROMPT-token prompt and the warm-up steps), through 8B-width models of 0 and 4 layers
    (both with the 128256-row LM head); every token attends to a context of that many cached positions per layer
    (seeded synthetic keys/values: the arithmetic per token is the workload's).  The per-layer time is scaled to
    32 layers -> tok/s."""

    LAYERS = 4
    NEW = 4

    def __init__(self, prompt=512, warmup=4):
        import numpy as np
        import oracle
        import synth
        from synth import configs
        self.oracle = oracle
        self.cfg32 = configs.LLAMA8B
        self.cfgL = configs.shrink(self.cfg32, n_layers=self.LAYERS)
        self.cfg0 = configs.shrink(self.cfg32, n_layers=0)
        self.wL = synth.model_weights(self.cfgL)
        self.w0 = {k: (v[:0] if (v.ndim == 3 or k in ("attn_norm", "ffn_norm")) else v) for k, v in self.wL.items()}
        self.pos0 = prompt + 1 + warmup  # position of the first timed decode step
        self.tok = synth.prompt_tokens(0, self.NEW, self.cfgL["vocab"])
        KD = self.cfgL["n_kv_heads"] * self.cfgL["head_dim"]
        kv = synth.normal_f64(synth.key(77, 1), 2 * self.LAYERS * self.pos0 * KD)
        kv = oracle.round_bf16(kv.reshape(2, self.LAYERS, self.pos0, KD))  # stored as bf16, as the path stores them
        self.k_ctx, self.v_ctx = kv[0], kv[1]
        self.k0 = np.zeros((0, self.pos0, KD))

    def once(self):
        t = time.perf_counter()
        self.oracle.forward_ctx(self.cfg0, self.w0, self.tok, self.k0, self.k0)
        t0 = time.perf_counter() - t
        t = time.perf_counter()
        self.oracle.forward_ctx(self.cfgL, self.wL, self.tok, self.k_ctx, self.v_ctx)
        tL = time.perf_counter() - t
        per_layer = max(tL - t0, 1e-9) / self.LAYERS
        return (t0 + per_layer * self.cfg32["n_layers"]) / self.NEW, t0, tL

    def describe(self, n, t0, tL):
        return (f"fp64 oracle, {self.NEW} teacher-forced decode tokens at positions {self.pos0}..{self.pos0 + self.NEW - 1}"
                f" (each attending to {self.pos0}+ cached positions per layer) through 0- and {self.LAYERS}-layer "
                f"8B-width models with the 128256-row LM head; per-layer time scaled to 32 layers; median of {n} "
                f"repeats ({t0:.3f} s, {tL:.3f} s per call)")


def cores():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def cpu_baseline(seconds, prompt=512, warmup=4):
    cs = CpuSample(prompt, warmup)
    t_end = time.time() + seconds
    runs = []
    while not runs or time.time() < t_end:
        runs.append(cs.once())
    med = sorted(runs)[len(runs) // 2]
    return {"value": round(1.0 / med[0], 4), "unit": "tok/s", "cores": cores(), "kind": "oracle",
            "sample": cs.describe(len(runs), med[1], med[2])}


def main_ours(args):
    import numpy as np
    import torch
    from synth import configs
    from invariant_deterministic_full_b200 import model as mdl
    ws, rank, local = dist_init(args)
    cfg = dict(configs.LLAMA8B)
    if args.layers:
        cfg["n_layers"] = args.layers
    B, P, K, W = args.batch, args.prompt, args.steps, args.warmup
    assert W >= 3, "at least 3 warm-up steps"
    mode = 1 if args.mode == "layercast" else 0
    sweep = [int(b) for b in args.sweep.split(",") if b.strip()] if args.sweep else []
    n_slots = max([B] + sweep)
    cap = P + W + K + 8
    m = mdl.Model(cfg, mode=mode, n_slots=n_slots, capacity=cap, init="device", device="cuda")
    r = run_decode(m, B, P, K, W, ws, rank)
    ms = max_over_ranks(r["ms"], ws)
    value = replica_throughput(B * K, ms, ws)
    hbm, tf_burst, tf_sus, src = peaks()
    sb = step_bytes(cfg, B, [0] * B, f32_kv=(mode == 1))  # weights + rows at one position, per step
    kv_row = cfg["n_layers"] * cfg["n_kv_heads"] * cfg["head_dim"] * 2 * (4 if mode else 2)
    tot_bytes = sum(step_bytes(cfg, B, [c] * B, f32_kv=(mode == 1)) for c in r["ctx_lens"])
    step_frac = tot_bytes / (ms / 1e3) / 1e9 / hbm
    line = {"metric": METRIC, "value": round(value, 2), "unit": "tok/s", "n_gpus": ws, "steps": K, "warmup": W,
            "ms_per_step": round(ms / K, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if mode == 0 else "f32 (bf16 weights)",
            "data": "synthetic: random-init bf16 weights N(0,0.02) (seed 20261202), uniform random prompt ids",
            "config": {"workload": f"llama3.1-8b-shape{' (%d layers)' % args.layers if args.layers else ''} "
                                   f"greedy decode, batch {B} per GPU, prompt {P}, "
                                   f"{K} timed steps (positions {P + 1 + W}..{P + W + K})",
                       "model": cfg["name"] + " (random init)", "global_batch": B * ws, "seq_len": P + W + K + 1,
                       "parallelism": "replicas" if ws > 1 else "single GPU",
                       "mode": args.mode, "variant": "invariant", "margin_threshold": 0.1,
                       "l2": "inputs larger than L2: every step streams 16 GB of weights"
                             if not args.layers else "profiling case (reduced layer count)"},
            "hbm_roofline_frac_step": round(step_frac, 4),
            "recompute_rate": r["recompute_rate"],
            "gpu_launches": int(r["launches"] * K),
            "clocks": r["clocks"],
            "gpu": torch.cuda.get_device_name(torch.cuda.current_device())}
    # dominant kernel: the weight-streaming projection GEMM (all layers' projections of one step), timed alone
    if mode == 0:
        gms = time_gemms(m, B)
        gb, gl = gemm_bytes(cfg, B)
        ach = gb / (gms / 1e3) / 1e9
        tr = gemm_traffic_per_launch(cfg, B)
        line["roofline"] = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                            "frac": round(ach / hbm, 4), "traffic": round(tr) if tr else None,
                            "traffic_note": "DRAM read+write bytes per launch (ncu, the same four GEMM shapes on "
                                            "the 2-layer case)" if tr else "no capture for this GEMM source/batch",
                            "kernel": "gemm_bf16_kernel (weight-streaming mma.sync GEMM, <= 32 token rows)" if B <= 32
                                      else "gemm_tc_kernel (weight-streaming tcgen05/TMEM GEMM)",
                            "per_launch": f"{gb / gl / 1e6:.1f} MB algorithmic over {gl} launches, "
                                          f"{gms / gl * 1e3:.1f} us average",
                            "peak_source": f"{src} hbm_gbs (copy), kernel timed alone"}
    else:
        line["roofline"] = {"bound": "alu", "achieved": None, "peak": None, "unit": "TFLOP/s", "frac": None,
                            "traffic": None}
    if rank == 0 and mode == 0 and not args.no_prefill:
        pms, pclk = time_prefill(m, B, P, rank)
        pf = prefill_flops(cfg, B, P)
        tfl = pf / (pms / 1e3) / 1e12
        line["prefill"] = {"tokens": B * P, "ms": round(pms, 3), "tok_s": round(B * P / (pms / 1e3), 1),
                           "tflops": round(tfl, 1), "peak_tflops": tf_sus, "frac": round(tfl / tf_sus, 4),
                           "peak_tflops_burst": tf_burst, "frac_of_burst": round(tfl / tf_burst, 4),
                           "clocks": pclk,
                           "note": f"one bi_decode_step over {B} prompts x {P} tokens, LM head on each last token; "
                                   f"FLOPs = 2 x projection weights x tokens + causal attention + LM head; peak = "
                                   f"{src} cuBLAS bf16 sustained (the timed region is {pms * 2:.0f} ms of back-to-back "
                                   f"tensor work under the power cap; the burst figure beside it); tcgen05 GEMMs"}
    if rank == 0 and not args.no_e2e:
        ke = min(K, 32)
        e = run_e2e(m, B, P, ke, rank, graph=True)
        ee = run_e2e(m, B, P, ke, rank, graph=False)
        line["e2e"] = {"value": round(B * ke / (e["ms"] / 1e3) * ws, 2), "unit": "tok/s",
                       "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"],
                       "call": "bi_decode_step captured once in a CUDA graph, replayed per step between the "
                               "pinned H2D copy of the step's inputs and the D2H read of its results",
                       "eager_value": round(B * ke / (ee["ms"] / 1e3) * ws, 2)}
    # batch sweep and the non-invariant comparison (same weights)
    extra, extra_frac = {}, {}
    for b in sweep:
        if b == B:
            extra[str(b)] = round(value / ws, 2)
            extra_frac[str(b)] = round(step_frac, 4)
            continue
        rb = run_decode(m, b, P, min(K, 32), W, 1, rank)
        extra[str(b)] = round(b * min(K, 32) / (rb["ms"] / 1e3), 2)
        bb = sum(step_bytes(cfg, b, [c] * b, f32_kv=(mode == 1)) for c in rb["ctx_lens"])
        extra_frac[str(b)] = round(bb / (rb["ms"] / 1e3) / 1e9 / hbm, 4)
    if extra:
        line["sweep_tok_s_per_gpu"] = extra
        line["sweep_hbm_roofline_frac"] = extra_frac
    if not args.no_fast:
        # the non-invariant variant at the headline batch and at the small batches where its split-K is active
        mf = mdl.Model(cfg, mode=mode, variant=1, n_slots=n_slots, capacity=cap, init="device")
        rf = run_decode(mf, B, P, K, W, 1, rank)
        per = {}
        for b in sorted({1, 4, 8} - {B}):
            rb = run_decode(mf, b, P, min(K, 32), W, 1, rank)
            per[str(b)] = round(b * min(K, 32) / (rb["ms"] / 1e3), 2)
        per[str(B)] = round(B * K / (rf["ms"] / 1e3), 2)
        inv = {k: v for k, v in extra.items() if k in per}
        line["fast_variant"] = {"value": per[str(B)], "unit": "tok/s", "per_batch": per,
                                "invariant_per_batch": inv,
                                "invariant_over_fast": {k: round(inv[k] / per[k], 4) for k in inv},
                                "note": "non-invariant variant on the same weights: split-K chosen from the batch "
                                        "(active at batch <= 16) and a KV split chosen from the batch"}
        mf.close()
        del mf
        torch.cuda.empty_cache()
    if mode == 0 and not args.no_lmhead and cfg["hidden"] == 4096:
        line["lmhead_alone"] = {"config": "hidden 4096, vocab 128256, bf16 W, fp32 rows N(0,1) RMS-normalised "
                                          "(seed 7), threshold 0.1 vs recompute off",
                                "per_batch": time_lmhead(m)}
    if mode == 0 and not args.no_layercast:
        ml = mdl.Model(cfg, mode=1, n_slots=max(B, 1), capacity=cap, init="device")
        rl = run_decode(ml, B, P, min(K, 16), W, 1, rank)
        line["layercast"] = {"value": round(B * min(K, 16) / (rl["ms"] / 1e3), 2), "unit": "tok/s",
                             "batch": B, "note": "bf16 weights, fp32 activations/KV; projections as exact fp32 "
                                                 "products on tensor cores (3-way bf16 split of the activations)"}
        ml.close()
        del ml
    if rank == 0 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds, P, W) if ws == 1 else None
    m.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main_reference(args):
    """Reference arm: the oracle, timed as it stands on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cs = CpuSample(args.prompt, args.warmup)
    for _ in range(args.warmup):
        cs.once()
    t0 = time.perf_counter()
    ts = [cs.once() for _ in range(args.steps)]
    wall = time.perf_counter() - t0
    med = sorted(ts)[len(ts) // 2]
    per_tok = med[0]
    v = 1.0 / per_tok
    cb = {"value": round(v, 4), "unit": "tok/s", "cores": cores(), "kind": "oracle",
          "sample": cs.describe(len(ts), med[1], med[2])}
    line = {"metric": METRIC, "value": round(v, 4), "unit": "tok/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(per_tok * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "impl": "reference",
            "data": "synthetic: same recipe as the GPU arm",
            "config": {"workload": f"llama3.1-8b-shape greedy decode, batch {args.batch} per GPU, prompt "
                                   f"{args.prompt}, {args.steps} timed steps (positions {args.prompt + 1 + args.warmup}"
                                   f"..{args.prompt + args.warmup + args.steps})",
                       "model": "llama3.1-8b-shape (random init)", "global_batch": args.batch * args.gpus,
                       "seq_len": args.prompt + args.warmup + args.steps + 1, "parallelism": "host cores (rank 0)",
                       "mode": args.mode, "variant": "invariant", "margin_threshold": 0.1,
                       "sample": "each step is a bounded sample of the workload: the oracle's time per decode token "
                                 "(tokens are independent on the host, so tok/s does not depend on the batch); "
                                 "see cpu_baseline.sample"},
            "cpu_baseline": cb,
            "e2e": {"value": round(v, 4), "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": round(wall, 1)}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        main_reference(a)
    else:
        main_ours(a)
