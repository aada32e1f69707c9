"""Host logic of the divergence study (no GPU): the divergence index, its summary, and the memory model of
LayerCast against bf16 and FP32 storage."""
import pytest

from invariant_deterministic_full_b200 import divergence as dv
from synth import configs


def test_divergence_index_first_differing_position():
    assert dv.divergence_index([5, 6, 7], [5, 6, 7]) is None
    assert dv.divergence_index([5, 6, 7], [9, 6, 7]) == 0
    assert dv.divergence_index([5, 6, 7], [5, 6, 8]) == 2
    assert dv.divergence_index([5, 6, 7, 1], [5, 6, 8, 1]) == 2  # later agreement does not undo a divergence
    assert dv.divergence_index([5, 6], [5, 6, 7]) == 2           # a shorter run differs where it ends
    assert dv.divergence_index([], []) is None


def test_compare_summary():
    ref = [[1, 2, 3], [1, 2, 3], [4, 4, 4], [7, 8, 9]]
    run = [[1, 2, 3], [1, 0, 3], [0, 4, 4], [7, 8, 0]]
    c = dv.compare(ref, run)
    assert c["indices"] == [None, 1, 0, 2]
    assert c["exact_agreement"] == 0.25 and c["diverged"] == 0.75
    assert c["median_index"] == 1 and c["mean_index"] == 1.0
    same = dv.compare(ref, ref)
    assert same["exact_agreement"] == 1.0 and same["median_index"] is None


def test_param_count_is_the_published_llama31_8b_count():
    assert dv.param_count(configs.LLAMA8B) == 8_030_261_248  # Llama 3.1 8B (untied embedding and LM head)


def test_memory_model():
    c = configs.LLAMA8B
    P = dv.param_count(c)
    assert dv.memory_bytes(c, 0, "bf16") == 2 * P
    assert dv.memory_bytes(c, 0, "fp32") == 4 * P
    assert dv.memory_bytes(c, 0, "layercast") == 2 * P          # weights stay bf16
    # one cached position: k and v, 32 layers x 8 heads x 128, at 2 or 4 bytes (128 KiB in bf16)
    assert dv.memory_bytes(c, 1, "bf16") - 2 * P == 128 * 1024
    assert dv.memory_bytes(c, 1, "layercast") - 2 * P == 256 * 1024
    assert dv.memory_bytes(c, 1, "fp32") - 4 * P == 256 * 1024
    # LayerCast saves half of FP32 storage with no KV cache, less as the fp32 cache grows
    lc = lambda n: 1 - dv.memory_bytes(c, n, "layercast") / dv.memory_bytes(c, n, "fp32")
    assert lc(0) == pytest.approx(0.5)
    assert 0 < lc(1 << 20) < lc(1 << 16) < 0.5
