"""Invariant tensor parallelism ("Meituan bitwise train/infer consistency", key-practices list, the TP item:
compute over the full K dimension instead of a segmented reduce-scatter, so that sharding never reorders a sum).

Every projection is split by OUTPUT rows across the tp ranks; a rank computes its rows over the full K with the
same tensor-core GEMM as an unsharded call, naming the unsharded row count (n_full) so that its accumulation
structure -- K ascending in 16-wide steps, the interleaved accumulator sets of the whole matrix and their fixed
combining tree -- is exactly the unsharded call's.  The activations are then all-gathered -- concatenated in
rank order, which moves bits and adds nothing.  There is no reduce-scatter and no all-reduce anywhere, so a token's logprob is bitwise the
same for tp = 1, 2, 4, 8:

  layer:  RMSNorm (replicated) -> QKV rows of the rank's heads (+ RoPE, KV append into the rank's cache)
          -> attention over the rank's heads -> all-gather -> O-proj rows -> all-gather
          -> residual + RMSNorm (replicated) -> gate/up rows (+ SwiGLU) -> all-gather -> down rows -> all-gather
  head:   final RMSNorm (replicated) -> the bf16 split rows of h -> LM-head rows of the rank's vocabulary chunks
          -> all-gather of the logits -> the fixed-order vocabulary reduction and selective recompute (replicated)

Heads are split so that rank r holds q heads [r Hq/tp, (r+1) Hq/tp) and the kv heads they read; the vocabulary is
split on the 256-id chunk grid of the reduction, so the gathered logits are exactly the unsharded ones.

Two communicators: LocalComm runs all ranks in one process, one after another, on one GPU (the all-gather is a
concatenation) -- this is how the single-GPU tests check the invariance; DistComm is one rank per process over
torch.distributed (NCCL between GPUs, gloo on CPU for the host-side tests).  Only argument marshalling and data
movement happen here: every arithmetic step is a libbi call.
"""
import numpy as np
import torch

from . import ops
from ._lib import VOCAB_CHUNK


class Sharding:
    """Which output rows of each weight rank r owns (all ranges contiguous, in rank order)."""

    def __init__(self, cfg, tp):
        H, Hq, Hkv, d, F, V = (cfg["hidden"], cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"], cfg["ffn"],
                               cfg["vocab"])
        if Hq % tp or Hkv % tp:
            raise ValueError(f"tp={tp} must divide the q heads ({Hq}) and the kv heads ({Hkv})")
        if H % (64 * tp) or F % (32 * tp):
            raise ValueError(f"tp={tp}: hidden {H} / ffn {F} shards are not multiples of the GEMM's 64 rows")
        self.tp, self.cfg = tp, cfg
        self.hq, self.hkv, self.d = Hq // tp, Hkv // tp, d
        # rows of the unsharded matrices: every shard's GEMM names them, so it accumulates exactly as they do
        self.n_full = {"w_qkv": (Hq + 2 * Hkv) * d, "w_o": H, "w_gu": 2 * F, "w_down": H, "lm_head": V}
        self.h_rows, self.f_rows = H // tp, F // tp
        nch = -(-V // VOCAB_CHUNK)
        cuts = [r * nch // tp for r in range(tp + 1)]
        self.vocab = [(cuts[r] * VOCAB_CHUNK, min(V, cuts[r + 1] * VOCAB_CHUNK)) for r in range(tp)]
        if any((b - a) % 64 for a, b in self.vocab):
            raise ValueError("vocabulary shards must be multiples of 64 ids")

    def qkv_rows(self, r):
        """Rows of the fused QKV weight (q heads, k heads, v heads; paired order kept inside each head)."""
        Hq, Hkv, d = self.cfg["n_heads"], self.cfg["n_kv_heads"], self.d
        q = np.arange(r * self.hq * d, (r + 1) * self.hq * d)
        k = Hq * d + np.arange(r * self.hkv * d, (r + 1) * self.hkv * d)
        v = (Hq + Hkv) * d + np.arange(r * self.hkv * d, (r + 1) * self.hkv * d)
        return np.concatenate([q, k, v])

    def o_rows(self, r):
        return np.arange(r * self.h_rows, (r + 1) * self.h_rows)

    down_rows = o_rows

    def gu_rows(self, r):
        """Rows of the gate/up weight (interleaved in 16-row granules, so whole 32-row gate/up blocks)."""
        return np.arange(2 * r * self.f_rows, 2 * (r + 1) * self.f_rows)

    def vocab_rows(self, r):
        a, b = self.vocab[r]
        return np.arange(a, b)


class LocalComm:
    """All ranks in this process (run one after another): all-gather = concatenation along the last dimension."""

    def __init__(self, tp):
        self.tp = tp
        self.ranks = list(range(tp))

    def all_gather(self, parts):
        return torch.cat(parts, dim=-1)


class DistComm:
    """One rank per process over an initialised torch.distributed group (NCCL on GPUs, gloo on CPU)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.tp = dist.get_world_size(group)
        self.ranks = [dist.get_rank(group)]

    def all_gather(self, parts):
        (x,) = parts
        x = x.contiguous()
        buf = [torch.empty_like(x) for _ in range(self.tp)]
        self.dist.all_gather(buf, x, group=self.group)
        return torch.cat(buf, dim=-1)


class TPModel:
    """The shards of a Model's bf16 weights for the ranks this process runs, each rank with its own KV cache for its
    kv heads, and a decode step that runs through libbi one rank-shard at a time."""

    def __init__(self, model, tp, comm=None, margin_threshold=0.1):
        if model.mode != 0 or model.variant != 0:
            raise ValueError("tensor parallelism is built for the bf16 invariant path")
        self.m, self.cfg, self.tp = model, model.cfg, tp
        self.sh = Sharding(model.cfg, tp)
        self.comm = comm or LocalComm(tp)
        self.thresh = margin_threshold
        w, dev = model.w, model.device
        take = lambda t, rows: t.index_select(-2, torch.as_tensor(rows, device=dev)).contiguous()
        self.w = {}
        cap = model.kv.layout.capacity
        for r in self.comm.ranks:
            self.w[r] = {"w_qkv": take(w["w_qkv"], self.sh.qkv_rows(r)), "w_o": take(w["w_o"], self.sh.o_rows(r)),
                         "w_gu": take(w["w_gu"], self.sh.gu_rows(r)),
                         "w_down": take(w["w_down"], self.sh.down_rows(r)),
                         "lm_head": take(w["lm_head"], self.sh.vocab_rows(r)),
                         "kv": ops.KVCache(model.kv.layout.n_slots, self.cfg["n_layers"], self.sh.hkv, cap,
                                           self.cfg["head_dim"], 0, dev)}

    def step(self, ids, slots, positions, targets=None):
        """One step over T tokens (every token gets a logprob row, as bi_decode_step with lm_row = t).  Host int
        arrays in; a dict of device tensors out (the keys of Model.step)."""
        m, c, sh, comm = self.m, self.cfg, self.sh, self.comm
        nf = sh.n_full
        dev = m.device
        L, H, d = c["n_layers"], c["hidden"], c["head_dim"]
        T = len(ids)
        slots_h = torch.as_tensor(np.asarray(slots), dtype=torch.int32).contiguous()
        pos_h = torch.as_tensor(np.asarray(positions), dtype=torch.int32).contiguous()
        d_ids = torch.as_tensor(np.asarray(ids), dtype=torch.int32).to(dev)
        d_slot, d_pos = slots_h.to(dev), pos_h.to(dev)
        d_tg = None if targets is None else torch.as_tensor(np.asarray(targets), dtype=torch.int32).to(dev)
        scale = float(np.float32(1.0) / np.sqrt(np.float32(d)))
        y = ops.embed(d_ids, m.w["embed"])
        res = torch.empty_like(y)
        for l in range(L):
            u = ops.rmsnorm(y, m.w["attn_norm"][l], c["eps"], residual_in=None if l == 0 else res, residual_out=res)
            o = []
            for r in comm.ranks:
                wr = self.w[r]
                q = ops.gemm_rope_kv(u, wr["w_qkv"][l], m.rope, m.rope_max_pos, wr["kv"], l, d_slot, d_pos, sh.hq,
                                     n_full=nf["w_qkv"])
                o.append(ops.attention(q, wr["kv"], l, d_slot, d_pos, slots_h, pos_h, sh.hq, scale))
            o = comm.all_gather(o)
            y = comm.all_gather([ops.gemm(o, self.w[r]["w_o"][l], n_full=nf["w_o"]) for r in comm.ranks])
            u = ops.rmsnorm(y, m.w["ffn_norm"][l], c["eps"], residual_in=res, residual_out=res)
            a = comm.all_gather([ops.gemm(u, self.w[r]["w_gu"][l], epilogue=1, n_full=nf["w_gu"]) for r in comm.ranks])
            y = comm.all_gather([ops.gemm(a, self.w[r]["w_down"][l], n_full=nf["w_down"]) for r in comm.ranks])
        _, h32 = ops.rmsnorm(y, m.w["final_norm"], c["eps"], residual_in=res, residual_out=res, want_f32=True)
        parts = 3 if self.thresh > 0 else 1
        rows = ops.lmhead_split(h32, parts)
        z = comm.all_gather([ops.gemm(rows, self.w[r]["lm_head"], out_dtype=torch.float32, n_full=nf["lm_head"])
                             for r in comm.ranks])
        return ops.lmhead_from_logits(z, T, parts, d_tg, self.thresh)
