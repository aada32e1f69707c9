"""Host-side logic of the invariant tensor-parallel path (no GPU): the shard bookkeeping, and the all-gather of
row shards over a gloo process group of world size 2, with exact integer products standing in for the GEMM."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from synth import configs


def _tp():
    from invariant_deterministic_full_b200 import tp
    return tp


@pytest.mark.parametrize("tp", [1, 2, 4, 8])
def test_shards_cover_every_row_once_in_rank_order(tp):
    cfg = configs.LLAMA8B
    sh = _tp().Sharding(cfg, tp)
    H, Hq, Hkv, d, F, V = (cfg["hidden"], cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"], cfg["ffn"],
                           cfg["vocab"])
    qkv = np.concatenate([sh.qkv_rows(r) for r in range(tp)])
    assert np.array_equal(np.sort(qkv), np.arange((Hq + 2 * Hkv) * d))
    for rows, n in ((sh.o_rows, H), (sh.gu_rows, 2 * F), (sh.down_rows, H), (sh.vocab_rows, V)):
        cat = np.concatenate([rows(r) for r in range(tp)])
        assert np.array_equal(cat, np.arange(n))  # rank-order concatenation is the natural order
    for r in range(tp):
        q_heads = sh.qkv_rows(r)[: sh.hq * d] // d
        k_heads = (sh.qkv_rows(r)[sh.hq * d: (sh.hq + sh.hkv) * d] - Hq * d) // d
        # the kv head each of the rank's q heads reads (GQA) is one of the rank's kv heads
        assert set(np.unique(q_heads) // (Hq // Hkv)) == set(np.unique(k_heads))
        a, b = sh.vocab[r]
        assert a % 256 == 0 and (b % 256 == 0 or b == V) and (b - a) % 64 == 0
        assert len(sh.gu_rows(r)) % 32 == 0  # whole gate/up granule pairs


def test_shards_reject_degrees_that_split_a_head_or_a_tile():
    tp = _tp()
    with pytest.raises(ValueError):
        tp.Sharding(configs.QWEN7B, 8)  # 4 kv heads
    with pytest.raises(ValueError):
        tp.Sharding(configs.shrink(configs.LLAMA8B, hidden=4160), 4)  # 1040-row shards


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(ws), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    tp = _tp()
    cfg = configs.shrink(configs.TINY, hidden=256, ffn=1024, vocab=4096)
    sh = tp.Sharding(cfg, ws)
    comm = tp.DistComm()
    assert comm.ranks == [rank] and comm.tp == ws
    rng = np.random.default_rng(3)  # the same full matrices on every rank
    x = torch.from_numpy(rng.integers(-3, 4, size=(5, 256)).astype(np.float64))
    res = {}
    for name, rows, n in (("o", sh.o_rows, 256), ("gu", sh.gu_rows, 2048), ("vocab", sh.vocab_rows, 4096)):
        W = torch.from_numpy(rng.integers(-3, 4, size=(n, 256)).astype(np.float64))
        mine = x @ W[torch.as_tensor(rows(rank))].T  # this rank's output rows over the full K (exact integers)
        full = comm.all_gather([mine])
        res[name] = bool(torch.equal(full, x @ W.T))
    out[rank] = res
    dist.destroy_process_group()


def test_all_gather_of_row_shards_rebuilds_the_unsharded_product():
    ws = 2
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_rank, args=(ws, _free_port(), out), nprocs=ws, join=True)
        res = dict(out)
    assert res == {r: {"o": True, "gu": True, "vocab": True} for r in range(ws)}


def test_local_comm_concatenates_in_rank_order():
    c = _tp().LocalComm(3)
    parts = [torch.full((2, r + 1), float(r)) for r in range(3)]
    assert torch.equal(c.all_gather(parts), torch.tensor([[0., 1., 1., 2., 2., 2.]] * 2))
