"""The seeded generator (data only): published SplitMix64 outputs and the recipe's statistics."""
import numpy as np

import synth
from synth import configs


def test_splitmix64_published_outputs():
    # First outputs of SplitMix64 seeded with 0 and with 1234567 (reference implementation by S. Vigna).
    assert [synth.draw(0, i) for i in range(3)] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    assert [synth.draw(1234567, i) for i in range(2)] == [6457827717110365317, 3203168211198807973]


def test_normal_statistics_and_determinism():
    k = synth.key(synth.WEIGHT_SEED, 1)
    z = synth.normal_f64(k, 400000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01
    assert np.array_equal(z[1000:1010], synth.normal_f64(k, 10, start=1000))
    b = synth.normal_bf16(k, 1000, std=0.02)
    assert np.array_equal(b, synth.f32_to_bf16_bits((z[:1000] * 0.02).astype(np.float32)))


def test_tokens_uniform_range():
    t = synth.tokens(synth.key(1000, 3), 100000, 4096)
    assert t.min() >= 0 and t.max() < 4096
    assert abs(t.mean() - 2047.5) < 30


def test_model_weights_shapes():
    w = synth.model_weights(configs.TINY)
    assert w["wq"].shape == (1, 256, 256) and w["wg"].shape == (1, 1024, 256) and w["wd"].shape == (1, 256, 1024)
    assert w["embed"].shape == (4096, 256) and (w["final_norm"] == 0x3F80).all()
