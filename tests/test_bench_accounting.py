"""The benchmark's workload arithmetic on CPU: the decode schedule, the flush
steps and the algorithmic bytes per decode call, checked against closed forms
written out by hand for each workload (96 B per quantized (token, kv head) and
512 B per residual token at head_dim 128 and G = 32, plus q in bf16 and out in
fp32), and the byte accounting against the Llama-2-13B record's 128,000 B per
token."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from bit_asymmetric_kv_prefill_b200 import synth  # noqa: E402

W = synth.WORKLOADS


def test_schedule_and_flushes_of_the_llama2_7b_layer():
    w = W["llama2_7b_layer"]
    sched = bench.decode_schedule(w)
    assert len(sched) == 64
    # prefill of 4,096 tokens leaves 3,968 quantized + 128 residual; the first
    # append flushes, then the residual grows by one per step
    assert sched[0] == (4096, 1) and sched[63] == (4096, 64)
    assert bench.flush_steps(w) == [True] + [False] * 63


def test_schedule_of_the_gqa_stream_flushes_at_steps_1_and_129():
    w = W["mistral_gqa"]
    flushes = [j + 1 for j, f in enumerate(bench.flush_steps(w)) if f]
    assert flushes == [1, 129]
    sched = bench.decode_schedule(w)
    assert sched[127] == (32768, 128) and sched[128] == (32896, 1) and sched[255] == (32896, 128)


@pytest.mark.parametrize("s", [1, 2, 64])
def test_decode_bytes_llama2_7b_layer(s):
    w = W["llama2_7b_layer"]
    n_q, r = bench.decode_schedule(w)[s - 1]
    assert bench.decode_bytes(w, n_q, r) == 100_663_296 + 131_072 * s + 196_608


def test_decode_bytes_llama2_13b_layer_and_record_basis():
    w = W["llama2_13b_cache"]
    # one decode over the prefilled cache: 3,968 quantized tokens + 128 residual
    assert bench.decode_bytes(w, 3968, 128) == 286_228_480
    # codes + full residual per token at 4,096 tokens, 40 layers: the record's
    # 102,400 + 25,600 = 128,000 B/token
    per_layer_codes = w.B * w.H_kv * 4096 * w.D * 2 * 2 // 8
    per_layer_res = w.B * w.H_kv * w.R * w.D * 2 * 2
    per_token = 40 * (per_layer_codes + per_layer_res) // (w.B * 4096)
    assert per_token == 128_000


@pytest.mark.parametrize("n_q,r", [(32768, 1), (32768, 128), (32896, 64)])
def test_decode_bytes_mistral_gqa(n_q, r):
    w = W["mistral_gqa"]
    assert bench.decode_bytes(w, n_q, r) == 49_152 * n_q + 262_144 * r + 1_572_864


def test_decode_bytes_long_context():
    w = W["long_context"]
    n_q, r = bench.decode_schedule(w)[0]
    assert (n_q, r) == (131072, 1)
    assert bench.decode_bytes(w, n_q, r) == 100_663_296 + 4_096 * r + 24_576


def test_units_are_kv_tokens_times_heads():
    w = W["llama2_7b_layer"]
    assert bench.decode_units(w, 4096, 5) == 8 * 32 * 4101


def test_workloads_without_decode_steps_decode_once_over_the_prefill():
    w = W["llama2_13b_cache"]
    assert bench.decode_calls(w) == [(3968, 128, "none")]
    assert bench.flush_steps(w) == [False]


def test_decode_calls_mark_flushes_and_fused_appends():
    kinds = [k for _, _, k in bench.decode_calls(W["mistral_gqa"])]
    assert kinds.count("flush") == 2 and kinds[0] == kinds[128] == "flush"
    assert kinds.count("fused") == 254


def test_prefill_bytes_of_the_128k_pre_rope_context():
    # 8 kv heads x 131,072 tokens x 128 channels of K and V read (bf16), 4,092
    # packed groups of 3,072 B and 128 residual rows of K and V per sequence
    w = W["long_context"]
    assert bench.prefill_bytes(w) == 637_960_192
    assert bench.prefill_bytes(w) == 8 * (2 * 131072 * 128 * 2 + 4092 * 3072 + 2 * 128 * 128 * 2)


def test_cache_record_bytes_of_the_llama2_13b_cache():
    # record kv-efficiency/kivi-2bit-llama2-13b-mha-4k, "KV bytes basis": 40
    # layers at 4,096 tokens hold 128,000 B/token of codes and residual; fp16
    # scale/zero per 32 add 51,200 B/token
    assert bench.cache_record_bytes(W["llama2_13b_cache"], 40) == (128_000, 51_200)


def test_oracle_sample_units():
    w = W["mistral_gqa"]
    one, calls, units = bench.oracle_sample(w, 8)
    assert (one.B, one.H_kv, one.H_q) == (1, 1, 4) and len(calls) == 8
    assert units == sum(n + r for n, r, _ in bench.decode_calls(w)[:8])


def test_decode_flops_and_fma_peak():
    w = W["mistral_gqa"]
    # 4*D flops per (token, query head): 64 x 32 query heads x 32,769 tokens
    assert bench.decode_flops(w, 32768, 1) == 4 * 128 * 64 * 32 * 32769
    # 148 SMs x 4 schedulers x 32 lanes x 2 flops at 1,965 MHz
    assert abs(bench.fma_peak_tflops(148, 1965.0) - 74.4499) < 1e-3


def test_roofline_names_the_closer_bound():
    import types
    w = W["mistral_gqa"]
    n_q, r = 32768, 1
    wb = types.SimpleNamespace(bytes_step=bench.decode_bytes(w, n_q, r), n_dec=1,
                               flops_step=bench.decode_flops(w, n_q, r), sms=148)
    t = {"clocks": {"sm_mhz": 1965.0}}
    # at 930 us: ~1.69 TB/s (26% of 6,454 GB/s) but ~36.9 TFLOP/s (50% of 74.4)
    roof = bench.roofline(wb, 0.930, t, 6454.3, "measured", None)
    assert roof["bound"] == "alu" and roof["unit"] == "TFLOP/s"
    assert 0.49 < roof["frac"] < 0.51 and roof["other_bound"]["bound"] == "hbm"
    assert 0.25 < roof["other_bound"]["frac"] < 0.27
    # one query head per kv head at the MHA layer's 38 us: HBM is the closer bound
    w2 = W["llama2_7b_layer"]
    wb2 = types.SimpleNamespace(bytes_step=bench.decode_bytes(w2, 4096, 1), n_dec=1,
                                flops_step=bench.decode_flops(w2, 4096, 1), sms=148)
    roof2 = bench.roofline(wb2, 0.038, t, 6454.3, "measured", 1.0)
    assert roof2["bound"] == "hbm" and roof2["traffic"] == 1.0 and roof2["other_bound"]["bound"] == "alu"
