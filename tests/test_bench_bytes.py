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
    g2p = sum(b[k] for k in ("gate_count", "plan", "reroute", "permute"))
    assert abs(g2p / 1e9 - gate_to_permute_gb) < 0.005
    assert b["count"] == 4 * w.Q
    assert abs(b["combine"] / 1e9 - combine_gb) < 0.005


def test_per_step_counts_on_a_small_case():
    w = synth.WORKLOADS["small_r8_e64"]
    N, E, K, d = w.N, w.E, w.K, w.d
    Q = N * K
    b = bench.algorithmic_bytes(w)
    assert b == {
        "gate_count": 4 * N * E + 4 * Q + 4 * Q,
        "count": 4 * Q,
        "plan": 0,
        "reroute": 4 * Q + 4 * Q + 4 * Q,
        "permute": 2 * N * d + K * 2 * N * d,
        "combine": K * 2 * N * d + 4 * Q + 4 * Q + 4 * N * d,
    }


def test_row_bytes_on_the_qwen3_layer():
    """The rows beside the path on the Qwen3-shaped layer with Qwen3-235B-sized
    experts (18,874,368 elements: fc1 2*4096*1536 + fc2 4096*1536) and the
    layer's greedy plan: 128 used replica slots over 107 replicated experts."""
    w = synth.WORKLOADS["qwen3_layer_r64_e128"]
    numel = 2 * 4096 * 1536 + 4096 * 1536
    assert numel == bench.EXPERT_NUMEL
    b = bench.row_bytes(N=w.N, K=w.K, d=w.d, used=128, replicated=107,
                        bytes_per_expert=2 * numel, numel=numel)
    assert abs(b["combine_backward"] / 1e9 - 38.68) < 0.005
    assert abs(b["permute_backward"] / 1e9 - 21.48) < 0.005
    assert abs(b["weight_sync"] / 1e9 - 9.66) < 0.005
    assert abs(b["grad_reduce"] / 1e9 - 25.82) < 0.005
    # per-operand form on a small case
    N, K, d = 10, 4, 16
    Q = N * K
    b = bench.row_bytes(N=N, K=K, d=d, used=3, replicated=2, bytes_per_expert=32, numel=8)
    assert b["combine_backward"] == 4 * N * d + K * 2 * N * d + 4 * Q + 4 * Q + K * 2 * N * d + 4 * Q
    assert b["permute_backward"] == K * 2 * N * d + 4 * Q + 4 * N * d
    assert b["weight_sync"] == 3 * 32 * 2
    assert b["grad_reduce"] == 4 * 8 * (2 + 2 + 3)


def test_threaded_cpu_baseline_equals_the_oracle():
    """The threaded CPU baseline (the oracle's own C functions split over host
    threads by token range) gives exactly the single-threaded oracle's
    outputs on a small workload, for several thread counts."""
    import synth
    w = synth.WORKLOADS["small_r8_e64"]
    lg, hd = synth.logits(w), synth.hidden(w)
    for threads in (1, 3, 8):
        res = bench.threaded_oracle_slice(w, lg, hd, w.T, threads)
        bench.check_threaded_slice(w, lg, hd, w.T, res)
    pairs, secs, n = bench.threaded_oracle_slices(w, lg, hd, 128, 0.0, 2, 4)
    assert pairs == w.R * 128 * w.K and n == 1 and secs > 0


@pytest.mark.parametrize("name,launches", [
    ("prefill_ep40_e160", 5), ("qwen3_layer_r64_e128", 5), ("dsv3_layer_r64_e256", 5),
    ("sweep_48x8_r64_e128", 5), ("pages_ep64_e256_t8k", 5), ("small_r8_e64", 6),
])
def test_kernel_launches_per_step(name, launches):
    """The `gpu_launches` claim: five kernels a step where the gate takes the
    count in (K = 8, E a multiple of 32 from 64 to 256), gate, count, plan,
    reroute, permute and combine otherwise (the small layer has K = 4). The
    plan and the reroute stay two kernels when one call launches both."""
    assert bench.kernels_per_step(synth.WORKLOADS[name]) == launches
