"""Accounting helpers against the numbers the pages print (tests/golden)."""
import json
import os

from sparse_mixture_experts_histogram_b200 import accounting as acc
from sparse_mixture_experts_histogram_b200 import synth

G = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_numbers.json")))


def test_layer_param_count_is_50_3M_for_every_sweep_row():
    p = G["moe_param_count"]
    for row in G["granularity_sweep"]["rows"]:
        assert row["E"] * row["d_ff"] == p["E_times_d_ff"]
        n = acc.moe_expert_params(p["d"], row["E"], row["d_ff"])
        assert n == 50_331_648
        assert round(n / 1e6, 1) == p["params_millions_printed"]
    # the sweep the package runs is the page's list minus the dense row
    assert [(r["E"], r["d_ff"], r["k"]) for r in G["granularity_sweep"]["rows"][1:]] == \
        list(synth.SWEEP)


def test_expert_calls_equal_T_times_k():
    p = G["expert_calls"]
    assert p["T"] * p["k"] == p["calls"]
    assert synth.Workload("w", p["T"], 512, p["E"], 256, p["k"]).S == p["calls"]


def test_estimator_worked_example():
    p = G["estimator_example"]
    d, D, E, k = p["d"], p["d_hidden"], p["E"], p["k"]
    dense = acc.ffn_params(d, D)
    assert dense == 308_281_344
    assert round(dense / 1e8, 2) == p["dense_params_1e8"]
    assert round(dense * 2 / 1e9, 2) == p["dense_gb"]  # bf16/fp16 bytes
    h = acc.match_dense_hidden(d, D, E)
    assert h == p["moe_hidden_size"]
    active = acc.active_params_per_token(d, E, h, k)
    assert active == 77_127_680
    assert round(active / 1e8, 2) == p["active_params_1e8"]
    assert round(active * 2 / 1e9, 2) == p["active_gb"]
    moe_total = acc.moe_expert_params(d, E, h) + acc.router_params(d, E)
    assert abs(moe_total - dense) / dense < 1e-3
    assert abs(active / moe_total - p["activation_ratio"]) < 0.01
    assert acc.ffn_params(d, D, matrices=2) == 2 * d * D  # GELU: two matrices


def test_memory_model_numbers():
    p = G["memory_model"]
    dense_bytes = acc.ffn_params(p["d"], p["d_ff"]) * 2
    assert dense_bytes == 352_321_536
    assert round(dense_bytes / 1e6) == p["dense_ffn_fp16_mb"]
    gate = acc.router_params(p["d"], p["E"]) * 2
    assert gate == 65_536 and gate // 1024 == p["gate_fp16_kb"]


def test_flops_and_bytes_closed_forms():
    # small layer: 2*3*d*d_ff*k*T + 2*T*d*E
    assert acc.active_flops(512, 512, 8, 4096, 2) == 2 * 3 * 512 * 4096 * 2 * 512 + 2 * 512 * 512 * 8
    assert abs(acc.active_flops(512, 512, 8, 4096, 2) / 1e9 - 12.89) < 0.01
    # Mixtral prefill T=8192: 5.773 TFLOP
    assert abs(acc.active_flops(8192, 4096, 8, 14336, 2) / 1e12 - 5.773) < 0.001
    # the expert FFN kernels (routed + shared) carry all expert FLOPs
    for (T, d, f, k, fs) in [(512, 512, 4096, 2, 0), (8192, 7168, 2048, 8, 2048)]:
        assert acc.ffn_flops(T, d, f, k) + acc.ffn_flops(T, d, fs, 1) == \
            acc.active_flops(T, d, 1, f, k, fs) - 2 * T * d
    # the FFN kernel's bytes: all hit experts' weights once, rows in, fp32 rows out
    assert acc.ffn_bytes(512, 512, 4096, 2, 8) == 2 * 3 * 8 * 512 * 4096 + 6 * 512 * 512
    # decode T=1 streams the two hit experts: 0.70 GB
    b = acc.algorithmic_bytes(1, 4096, 8, 14336, 2, experts_hit=2)
    assert abs(b / 1e9 - 0.705) < 0.001


def test_fp8_bytes_count_one_byte_per_weight_and_the_row_scales():
    # e4m3 experts: one byte per weight plus an fp32 scale per W1, W3 and W2
    # row; everything else as in the bf16 layer.
    d, f, E, T, k = 4096, 14336, 8, 8, 2
    assert acc.fp8_scale_bytes(d, f) == 4 * (2 * f + d)
    b16 = acc.algorithmic_bytes(T, d, E, f, k, experts_hit=8)
    b8 = acc.algorithmic_bytes(T, d, E, f, k, experts_hit=8, fp8=True)
    assert b16 - b8 == 8 * (3 * d * f - acc.fp8_scale_bytes(d, f))
    assert acc.ffn_bytes(T, d, f, k, 8, fp8=True) == 8 * (3 * d * f + 4 * (2 * f + d)) + 6 * T * d
