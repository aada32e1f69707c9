"""Host-side bookkeeping of bench.py: the algorithmic byte counts behind the roofline fractions, the stored ncu
traffic and its source guard, and the clock-record parser (no GPU)."""
import pytest

import bench
from synth import configs

L8 = configs.LLAMA8B
# Llama 3.1 8B: 8,030,261,248 parameters (embedding and LM head untied); its model card rounds this to 8.03B.
LLAMA31_8B_PARAMS = 8_030_261_248


def test_step_weight_bytes_match_the_published_parameter_count():
    # A decode step streams every weight once except the embedding table, of which it gathers only B rows.
    embed = L8["vocab"] * L8["hidden"]
    assert bench.step_bytes(L8, 0, []) == 2 * (LLAMA31_8B_PARAMS - embed)


@pytest.mark.parametrize("ctx", [0, 1, 517, 4095])
def test_step_kv_bytes_are_128_kib_per_position(ctx):
    # GQA with 8 KV heads of 128: k and v, bf16, 32 layers -> 128 KiB per cached position of one sequence.
    w = bench.step_bytes(L8, 0, [])
    got = bench.step_bytes(L8, 1, [ctx]) - w - 2 * L8["hidden"]
    assert got == (ctx + 2) * 128 * 1024  # positions 0..ctx read, one position written
    assert bench.step_bytes(L8, 1, [ctx], f32_kv=True) - w - 2 * L8["hidden"] == 2 * got


def test_gemm_set_is_the_four_projections_of_every_layer():
    tot, n = bench.gemm_bytes(L8, 32)
    assert n == 4 * L8["n_layers"]
    H, V, L = L8["hidden"], L8["vocab"], L8["n_layers"]
    # every weight of the step except the norm gains and the LM head
    assert bench.gemm_bytes(L8, 0)[0] == bench.step_bytes(L8, 0, []) - 2 * L * 2 * H - 2 * H - 2 * V * H
    # per layer: QKV 6144x4096, O 4096x4096, gate/up 28672x4096 (SwiGLU halves the output), down 4096x14336;
    # bf16 weights, 32 bf16 input rows and 32 output rows each
    w = 2 * 4096 * (6144 + 4096 + 28672 + 14336)
    io = 32 * 2 * ((4096 + 6144) + (4096 + 4096) + (4096 + 14336) + (14336 + 4096))
    assert tot / n == (w + io) / 4


def test_stored_gemm_traffic_applies_to_this_source_and_equals_the_algorithmic_bytes():
    assert len(bench.current_gemm_digest()) == 64  # the digest's landmarks are all present
    t = bench.gemm_traffic_per_launch(L8, 32)
    if t is None:
        pytest.skip("GEMM kernel source changed since the stored ncu capture: traffic is reported as null")
    tot, n = bench.gemm_bytes(L8, 32)
    # no re-reads beyond the algorithmic bytes; the epilogues' 2-byte stores write whole 32-byte sectors, which
    # puts the measured DRAM writes a few MB per layer above the algorithmic outputs
    assert tot / n <= t <= 1.02 * tot / n
    assert bench.gemm_traffic_per_launch(L8, 16) is None  # captured at batch 32 only


def test_gemm_source_digest_ignores_comments_and_code_outside_the_kernel():
    rd = lambda n: open(bench.os.path.join(bench.CSRC, n)).read()
    mma, plan = rd("gemm_mma.cuh"), rd("gemm.cuh")
    h = bench.gemm_source_digest(mma, plan)
    assert bench.gemm_source_digest(mma, plan + "\n// trailing helper\n") == h
    i = mma.index("template <int BN, int EPI, int MT, int CPS>")
    assert bench.gemm_source_digest(mma[:i] + "// a comment\n  /* and another */ " + mma[i:], plan) == h
    assert bench.gemm_source_digest(mma[:i] + "constexpr int kExtra = 1;\n" + mma[i:], plan) != h
    j = plan.index("struct TcPlan {")
    assert bench.gemm_source_digest(mma, plan[:j] + "static int kMore = 4;\n" + plan[j:]) == h  # before the plan
    k = plan.index("static TcPlan tc_plan(")
    assert bench.gemm_source_digest(mma, plan[:k] + "static int kMore = 4;\n" + plan[k:]) != h
    w = plan.index("size_t gemm_ws_bytes(")  # workspace sizing does not decide the traffic
    assert bench.gemm_source_digest(mma, plan[:w] + "static int kWs = 3;\n" + plan[w:]) == h


def test_clock_summary_median_and_reasons():
    c = bench.ClockSampler(0)
    row = lambda mhz, pc: ["0", str(mhz), "1965", "700", "0x4", "Not Active", "Not Active", "Not Active", pc]
    c.rows = [row(1965, "Not Active"), row(1800, "Active"), row(1965, "Not Active"), ["garbage"]]
    s = c.summary()
    assert s == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_prefill_flops_from_the_parameter_count():
    c = L8
    L, H, V, d, Hq = c["n_layers"], c["hidden"], c["vocab"], c["head_dim"], c["n_heads"]
    matmul_params = LLAMA31_8B_PARAMS - 2 * V * H - H - 2 * L * H  # projections only: no embedding, LM head, norms
    B, P = 3, 5
    causal_pairs = B * P * (P + 1) // 2  # (query, key) pairs with key <= query, per head and layer
    want = 2 * matmul_params * B * P + 4 * d * Hq * L * causal_pairs + 2 * V * H * B
    assert bench.prefill_flops(c, B, P) == want
