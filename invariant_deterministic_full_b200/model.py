"""Synthetic random-init decoder on the device, driven through bi_decode_step.

Weights are the seeded recipe of synth/ (bf16 N(0, 0.02), norm gains 1):
small models are generated on the host and copied; large ones are generated
on the device by bi_synth_fill_bf16 (the same definition, checked bit for bit
against the host generator by the GPU tests).  Layouts follow include/bi.h:
fused q/k/v rows, gate/up interleaved by 16 rows.
"""
import ctypes

import numpy as np
import torch

import synth
from . import ops
from ._lib import (lib, check, ModelDesc, Weights, Batch, StepOut, MODE_BF16, MODE_LAYERCAST, MODE_FP32,
                   VARIANT_INVARIANT, GU_INTERLEAVE)


def _to_dev_bf16(bits, device):
    a = np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)
    return torch.from_numpy(a).to(device).view(torch.bfloat16)


def paired_rows(d):
    """Fused row of each element of a head of size d in the paired q/k order (see bi_weights.w_qkv)."""
    i = np.arange(d)
    half = d // 2
    return np.where(i < half, 32 * (i // 16) + i % 16, 32 * ((i - half) // 16) + 16 + (i - half) % 16)


def pair_heads(w, d):
    """[rows, H] q or k weight with rows in natural head order -> paired order."""
    out = np.empty_like(w)
    rows = np.arange(w.shape[0])
    out[(rows // d) * d + paired_rows(d)[rows % d]] = w
    return out


def interleave_gu(wg, wu, g=GU_INTERLEAVE):
    """[F,H] gate and up -> [2F,H]: g gate rows, then the g up rows of the same outputs, ..."""
    F, H = wg.shape
    out = np.empty((2 * F, H), dtype=wg.dtype)
    blk = np.arange(F) // g
    r = np.arange(F) % g
    out[blk * 2 * g + r] = wg
    out[blk * 2 * g + g + r] = wu
    return out


class Model:
    """Device weights, RoPE table, KV cache and a bi_ctx for one synthetic config."""

    def __init__(self, cfg, mode=MODE_BF16, variant=VARIANT_INVARIANT, n_slots=8, capacity=1024,
                 margin_threshold=0.1, seed=synth.WEIGHT_SEED, device="cuda", init="auto", host_weights=None):
        self.cfg = dict(cfg)
        self.mode, self.variant, self.device = mode, variant, device
        L, H, Hq, Hkv, d, F, V = (cfg["n_layers"], cfg["hidden"], cfg["n_heads"], cfg["n_kv_heads"],
                                  cfg["head_dim"], cfg["ffn"], cfg["vocab"])
        QKV = (Hq + 2 * Hkv) * d
        if init == "auto":
            init = "host" if (host_weights is not None or L * (QKV + 3 * F) * H + 2 * V * H < 2e8) else "device"
        self.init = init
        if init == "host":
            w = host_weights if host_weights is not None else synth.model_weights(cfg, seed=seed)
            self.host_weights = w
            qkv = np.concatenate([np.stack([pair_heads(w["wq"][l], d) for l in range(L)]),
                                  np.stack([pair_heads(w["wk"][l], d) for l in range(L)]), w["wv"]], axis=1)
            gu = np.stack([interleave_gu(w["wg"][l], w["wu"][l]) for l in range(L)])
            t = {"embed": w["embed"], "lm_head": w["lm_head"], "final_norm": w["final_norm"],
                 "attn_norm": w["attn_norm"], "ffn_norm": w["ffn_norm"], "w_qkv": qkv, "w_o": w["wo"],
                 "w_gu": gu, "w_down": w["wd"]}
            self.w = {k: _to_dev_bf16(v, device) for k, v in t.items()}
        else:
            self.host_weights = None
            self.w = self._device_init(seed)
        if mode == MODE_FP32:
            # FP32 storage: the same weight values held as f32 (an exact upcast; the norm gains stay bf16)
            for k in ("embed", "lm_head", "w_qkv", "w_o", "w_gu", "w_down"):
                self.w[k] = self.w[k].float()
        self.rope_max_pos = capacity
        self.rope = ops.rope_table(capacity, d, cfg["rope_theta"], device)
        self.kv = ops.KVCache(n_slots, L, Hkv, capacity, d, mode, device)
        self.desc = ModelDesc(L, H, Hq, Hkv, d, F, V, float(cfg["eps"]), mode, variant, float(margin_threshold))
        w = self.w
        self.weights = Weights(w["embed"].data_ptr(), w["lm_head"].data_ptr(), w["final_norm"].data_ptr(),
                               w["attn_norm"].data_ptr(), w["ffn_norm"].data_ptr(), w["w_qkv"].data_ptr(),
                               w["w_o"].data_ptr(), w["w_gu"].data_ptr(), w["w_down"].data_ptr(),
                               self.rope.data_ptr(), capacity)
        ctx = ctypes.c_void_p()
        check(lib.bi_ctx_create(ctypes.byref(self.desc), ctypes.byref(self.weights), ctypes.byref(self.kv.layout),
                                ctypes.byref(ctx)), "bi_ctx_create")
        self.ctx = ctx
        self._ws = None

    def _device_init(self, seed):
        c, dev = self.cfg, self.device
        L, H, Hq, Hkv, d, F, V = (c["n_layers"], c["hidden"], c["n_heads"], c["n_kv_heads"], c["head_dim"], c["ffn"],
                                  c["vocab"])
        QD, KD = Hq * d, Hkv * d
        e = lambda *s: torch.empty(*s, dtype=torch.bfloat16, device=dev)
        w = {"embed": e(V, H), "lm_head": e(V, H), "final_norm": torch.ones(H, dtype=torch.bfloat16, device=dev),
             "attn_norm": torch.ones(L, H, dtype=torch.bfloat16, device=dev),
             "ffn_norm": torch.ones(L, H, dtype=torch.bfloat16, device=dev),
             "w_qkv": e(L, QD + 2 * KD, H), "w_o": e(L, H, QD), "w_gu": e(L, 2 * F, H), "w_down": e(L, H, F)}
        std = synth.WEIGHT_STD
        ops.synth_fill_bf16(w["embed"], V, H, synth.key(seed, synth.S_EMBED), std)
        ops.synth_fill_bf16(w["lm_head"], V, H, synth.key(seed, synth.S_LMHEAD), std)
        for l in range(L):
            ls = lambda s: synth.key(seed, synth.layer_stream(l, s))
            q = w["w_qkv"][l]
            ops.synth_fill_bf16(q[:QD], QD, H, ls(synth.S_WQ), std, interleave=-d)
            ops.synth_fill_bf16(q[QD:QD + KD], KD, H, ls(synth.S_WK), std, interleave=-d)
            ops.synth_fill_bf16(q[QD + KD:], KD, H, ls(synth.S_WV), std)
            ops.synth_fill_bf16(w["w_o"][l], H, QD, ls(synth.S_WO), std)
            ops.synth_fill_bf16(w["w_gu"][l], F, H, ls(synth.S_WG), std, interleave=GU_INTERLEAVE, phase=0)
            ops.synth_fill_bf16(w["w_gu"][l], F, H, ls(synth.S_WU), std, interleave=GU_INTERLEAVE, phase=1)
            ops.synth_fill_bf16(w["w_down"][l], H, F, ls(synth.S_WD), std)
        return w

    def close(self):
        if self.ctx:
            lib.bi_ctx_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace(self, T, n_lm, max_pos):
        need = lib.bi_decode_workspace_size(self.ctx, T, n_lm, max_pos)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self._ws

    def step(self, ids, slots, positions, lm_rows=None, targets=None, want_logits=False, want_h=False):
        """One bi_decode_step.  ids/slots/positions: per-token ints (host).  lm_rows: per-token output row or -1
        (default: every token, row = token index).  targets: per output row (None = greedy).
        Returns a dict of device tensors over the output rows."""
        dev = self.device
        T = len(ids)
        slots_h = torch.as_tensor(np.asarray(slots), dtype=torch.int32).contiguous()
        pos_h = torch.as_tensor(np.asarray(positions), dtype=torch.int32).contiguous()
        if lm_rows is None:
            lm_rows = np.arange(T)
        lm_h = torch.as_tensor(np.asarray(lm_rows), dtype=torch.int32).contiguous()
        n_lm = int((lm_h >= 0).sum())
        d_ids = torch.as_tensor(np.asarray(ids), dtype=torch.int32).to(dev)
        d_slot, d_pos, d_lm = slots_h.to(dev), pos_h.to(dev), lm_h.to(dev)
        d_tg = None if targets is None else torch.as_tensor(np.asarray(targets), dtype=torch.int32).to(dev)
        out = self.alloc_out(n_lm, want_logits, want_h)
        self.step_dev(T, d_ids, d_slot, d_pos, slots_h, pos_h, d_lm, n_lm, d_tg, out)
        return out

    def alloc_out(self, n_lm, want_logits=False, want_h=False):
        dev = self.device
        out = dict(logprob=torch.empty(n_lm, dtype=torch.float32, device=dev),
                   lse=torch.empty(n_lm, dtype=torch.float32, device=dev),
                   argmax=torch.empty(n_lm, dtype=torch.int32, device=dev),
                   margin=torch.empty(n_lm, dtype=torch.float32, device=dev),
                   recomputed=torch.empty(n_lm, dtype=torch.uint8, device=dev))
        if want_logits:
            out["logits"] = torch.empty(n_lm, self.cfg["vocab"], dtype=torch.float32, device=dev)
        if want_h:
            out["h"] = torch.empty(n_lm, self.cfg["hidden"], dtype=torch.float32, device=dev)
        return out

    def step_dev(self, T, d_ids, d_slot, d_pos, slots_h, pos_h, d_lm, n_lm, d_tg, out, max_pos=None):
        """bi_decode_step on device arrays (host slot/pos copies for planning).  max_pos (optional) sizes the
        workspace for later steps that reuse this call's structure (graph replay)."""
        mp = int(pos_h.max()) if max_pos is None else max_pos
        ws = self.workspace(T, n_lm, mp)
        p = lambda t: 0 if t is None else t.data_ptr()
        self._batch = Batch(T, p(d_ids), p(d_slot), p(d_pos), p(slots_h), p(pos_h), p(d_lm), n_lm, p(d_tg))
        self._out = StepOut(p(out["logprob"]), p(out["lse"]), p(out["argmax"]), p(out["margin"]),
                            p(out["recomputed"]), p(out.get("logits")), p(out.get("h")))
        check(lib.bi_decode_step(self.ctx, ctypes.byref(self._batch), ctypes.byref(self._out),
                                 ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)), "bi_decode_step")


def to_host(out):
    return {k: v.cpu().numpy() for k, v in out.items()}


def prefill(model, slot, tokens, start=0, chunk=None, lm_every=1, targets=None):
    """Run a prompt through bi_decode_step in chunks of `chunk` tokens (None = whole).
    Returns host arrays over the positions that produced logprobs (every lm_every-th and the last)."""
    n = len(tokens)
    chunk = chunk or n
    outs = []
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        idx = np.arange(c0, c1)
        want = (idx % lm_every == 0) | (idx == n - 1)
        lm_rows = np.where(want, np.cumsum(want) - 1, -1)
        tg = None if targets is None else np.asarray(targets)[idx[want]]
        o = model.step(tokens[c0:c1], [slot] * (c1 - c0), start + idx, lm_rows, tg)
        o = to_host(o)
        o["pos"] = start + idx[want]
        outs.append(o)
    return {k: np.concatenate([o[k] for o in outs]) for k in outs[0]}


def greedy_generate(model, prompts, n_steps, chunk=None, slots=None):
    """Prefill each prompt (its own slot), then n_steps batched greedy decode steps.
    Returns (tokens [B][len+n_steps], per-sequence dict of decode-step outputs)."""
    B = len(prompts)
    slots = list(range(B)) if slots is None else slots
    last = []
    for b, p in enumerate(prompts):
        o = prefill(model, slots[b], p, chunk=chunk, lm_every=len(p))
        last.append(int(o["argmax"][-1]))
    seqs = [list(map(int, p)) + [last[b]] for b, p in enumerate(prompts)]
    rec = {k: [] for k in ("logprob", "lse", "argmax", "margin", "recomputed")}
    for s in range(n_steps):
        ids = [seqs[b][-1] for b in range(B)]
        pos = [len(seqs[b]) - 1 for b in range(B)]
        o = to_host(model.step(ids, slots, pos))
        for k in rec:
            rec[k].append(o[k])
        for b in range(B):
            seqs[b].append(int(o["argmax"][b]))
    return seqs, {k: np.stack(v, axis=1) for k, v in rec.items()}
