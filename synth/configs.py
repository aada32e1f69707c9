"""Model shapes of the synthetic workloads (data only).

Tiny decoder, a Llama-3.1-8B-shaped model and a Qwen2.5-7B-shaped model, all
random-init.  eps = 1e-5 for every shape; RoPE base 1e4 / 5e5 / 1e6.
"""

TINY = dict(name="tiny", n_layers=1, hidden=256, n_heads=4, n_kv_heads=4, head_dim=64, ffn=1024, vocab=4096,
            eps=1e-5, rope_theta=10000.0)
LLAMA8B = dict(name="llama3.1-8b-shape", n_layers=32, hidden=4096, n_heads=32, n_kv_heads=8, head_dim=128,
               ffn=14336, vocab=128256, eps=1e-5, rope_theta=500000.0)
QWEN7B = dict(name="qwen2.5-7b-shape", n_layers=28, hidden=3584, n_heads=28, n_kv_heads=4, head_dim=128,
              ffn=18944, vocab=152064, eps=1e-5, rope_theta=1000000.0)

CONFIGS = {c["name"]: c for c in (TINY, LLAMA8B, QWEN7B)}


def shrink(cfg, **kw):
    """A copy of a config with some fields replaced (small parity cases of the same structure)."""
    c = dict(cfg)
    c.update(kw)
    return c
