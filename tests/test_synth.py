"""Checks of the seeded input generator (CPU only).

The skew constants in ``synth`` were found with the oracle; these tests
re-measure the skew they produce with the oracle's exact histogram, so a
change to the generator that moves the workloads away from their stated
shape fails here.
"""
import numpy as np
import pytest

import oracle
import synth


def test_deterministic_and_thread_independent(monkeypatch):
    a = synth.normal_f32(3 * synth.CHUNK + 17, 0, 1, 2)
    monkeypatch.setattr(synth, "_threads", lambda: 1)
    b = synth.normal_f32(3 * synth.CHUNK + 17, 0, 1, 2)
    np.testing.assert_array_equal(a, b)
    h1 = synth.bf16_normal(100, 64, 0, 9)
    h2 = synth.bf16_normal(100, 64, 0, 9)
    np.testing.assert_array_equal(h1, h2)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -2.5, 0.0, -0.0,
                  1.0 + 2 ** -9], dtype=np.float32)
    h = synth.f32_to_bf16_bits(x)
    back = synth.bf16_bits_to_f32(h)
    # 1 + 2^-9 is a tie between 1 and 1 + 2^-7 -> even (1.0)
    np.testing.assert_array_equal(back, np.array([1.0, 1.0, 1.0 + 2 ** -7, -2.5, 0.0, -0.0, 1.0],
                                                 dtype=np.float32))


def test_small_workload_shapes():
    w = synth.WORKLOADS["small_r8_e64"]
    lg = synth.logits(w)
    assert lg.shape == (4096, 64) and lg.dtype == np.float32
    assert np.isfinite(lg).all()
    hd = synth.hidden(w)
    assert hd.shape == (4096, 256) and hd.dtype == np.uint16
    f = synth.bf16_bits_to_f32(hd)
    assert abs(float(f.mean())) < 0.01 and abs(float(f.std()) - 1.0) < 0.01


def masters_skew(w, load_e):
    return load_e.reshape(w.R, w.M).sum(axis=1).max() / (w.Q / w.R)


@pytest.mark.slow_cpu
def test_qwen3_layer_pre_balance_skew_is_2_5():
    w = synth.WORKLOADS["qwen3_layer_r64_e128"]
    idx, _ = oracle.gate_topk(synth.logits(w), w.K)
    _, load_e = oracle.count(idx, w.R, w.T, w.E)
    assert abs(masters_skew(w, load_e) - 2.5) <= 0.05


@pytest.mark.slow_cpu
def test_dsv3_layer_hotspots_draw_8_percent_each():
    w = synth.WORKLOADS["dsv3_layer_r64_e256"]
    lg, info = synth.logits(w, with_info=True)
    idx, _ = oracle.gate_topk(lg, w.K)
    _, load_e = oracle.count(idx, w.R, w.T, w.E)
    for h in info["hot"]:
        assert abs(load_e[h] / w.Q - 0.08) <= 0.001


@pytest.mark.slow_cpu
def test_sweep_single_expert_case_takes_30_percent_of_tokens():
    w = synth.WORKLOADS["sweep_48x8_r64_e128"]
    lg, info = synth.logits(w, layer=0, mb=1, with_info=True)
    assert info["kind"] == "single_expert_30pct"
    idx, _ = oracle.gate_topk(lg, w.K)
    _, load_e = oracle.count(idx, w.R, w.T, w.E)
    assert abs(load_e[info["hot"][0]] / w.N - 0.30) <= 0.005


@pytest.mark.slow_cpu
@pytest.mark.parametrize("i,target", [(0, 1.51), (1, 2.01), (2, 3.03)])
def test_pages_layer_initial_imbalances(i, target):
    # the pages' runtime test (EP64, 256 experts, 4 masters per rank) at its
    # three stated initial imbalances
    w = synth.WORKLOADS["pages_ep64_e256_t8k"]
    idx, _ = oracle.gate_topk(synth.logits(w, alpha=synth.ALPHA_PAGES[i]), w.K)
    _, load_e = oracle.count(idx, w.R, w.T, w.E)
    assert abs(masters_skew(w, load_e) - target) <= 0.01


def test_sweep_uniform_case_has_no_bias():
    w = synth.WORKLOADS["sweep_48x8_r64_e128"]
    bias, info = synth.logit_bias(w, 0, 0)
    assert info["kind"] == "uniform" and np.all(bias == 0.0)


def test_prefill_per_rank_exponents_differ():
    w = synth.WORKLOADS["prefill_ep40_e160"]
    bias, info = synth.logit_bias(w)
    assert bias.shape == (40, 160)
    assert info["s_r"].min() >= 0.8 and info["s_r"].max() <= 1.5
    assert len(np.unique(np.round(info["s_r"], 6))) == 40


@pytest.mark.slow_cpu
def test_stored_sweep_digests_are_the_oracles():
    """The stored digests of the sweep (written by tests/golden/sweep_digests.py
    from the oracle) match the oracle recomputed here on the uniform
    instance, the 30%-single-expert instance and one Zipf instance."""
    import json
    import os

    from tests.routing_digest import flatten_oracle, routing_digest
    path = os.path.join(os.path.dirname(__file__), "golden", "sweep_digests.json")
    with open(path) as f:
        doc = json.load(f)
    w = synth.WORKLOADS[doc["workload"]]
    for layer, mb in [(0, 0), (0, 1), (17, 3)]:
        o = oracle.run_path(synth.logits(w, layer, mb), w.R, w.T, w.S, w.K)
        assert routing_digest(flatten_oracle(o)) == \
            doc["digests"]["greedy"][layer * w.microbatches + mb], (layer, mb)
