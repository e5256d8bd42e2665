"""The algorithmic bytes behind every roofline fraction bench.py reports,
pinned to the per-step byte counts of the path (reads plus writes of each
step's operands) and to their totals on the five workloads.

Per step, with N tokens, E experts, K picks, d the hidden size, Q = N*K:
gate 4NE + 8Q (fp32 logits in; int32 ids and fp32 weights out); count 4Q;
plan ~0 (latency bound, reported in µs); reroute 4Q + 8Q; permute 2Nd + 2Qd
(bf16 rows read once, written K times); combine 2Qd + 8Q + 4Nd (K bf16 rows,
ids and weights in; an fp32 row out). The totals below are the sums for the
gate-to-permute steps, the count left out as if fused into the gate (its 4Q
bytes are checked on their own), and for the combine, in GB.
"""
import pytest

import bench
import synth


@pytest.mark.parametrize("name,gate_to_permute_gb,combine_gb", [
    ("qwen3_layer_r64_e128", 19.50, 21.49),
    ("dsv3_layer_r64_e256", 17.07, 18.80),
    ("prefill_ep40_e160", 30.46, 33.58),
    ("sweep_48x8_r64_e128", 19.50, 21.49),
])
def test_totals_per_workload(name, gate_to_permute_gb, combine_gb):
    w = synth.WORKLOADS[name]
    b = bench.algorithmic_bytes(w)
    g2p = sum(b[k] for k in ("gate_topk", "plan", "reroute", "permute"))
    assert abs(g2p / 1e9 - gate_to_permute_gb) < 0.005
    assert b["count"] == 4 * w.Q
    assert abs(b["combine"] / 1e9 - combine_gb) < 0.005


def test_per_step_counts_on_a_small_case():
    w = synth.WORKLOADS["small_r8_e64"]
    N, E, K, d = w.N, w.E, w.K, w.d
    Q = N * K
    b = bench.algorithmic_bytes(w)
    assert b == {
        "gate_topk": 4 * N * E + 4 * Q + 4 * Q,
        "count": 4 * Q,
        "plan": 0,
        "reroute": 4 * Q + 4 * Q + 4 * Q,
        "permute": 2 * N * d + K * 2 * N * d,
        "combine": K * 2 * N * d + 4 * Q + 4 * Q + 4 * N * d,
    }
