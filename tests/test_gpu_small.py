"""GPU parity at sizes the oracle finishes in seconds: every output of every
step, element by element, through the C ABI, against the CPU oracle.

Cases: the R=8 x 512 tokens, E=64, K=4, S=2, d=256 workload, and edge shapes
(ragged tiles and row groups, E below and above a warp, K = 1, K = E, K not
dividing 32, S = 0 and S = 8, the widest rows), tie-heavy logits with signed
zeros, an exactly uniform routing (no replication), and an extreme skew that
uses every slot.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import token_rerouting_b200 as ue
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu


def run_case(R, T, E, K, S, d, logits, seed=0):
    """Run the whole path on the GPU and on the oracle; compare everything
    (the routing both through ue_gate_count and ue_plan_reroute, and through
    ue_gate_topk, ue_count, ue_plan and ue_reroute)."""
    N, Q = R * T, R * T * K
    hidden = synth.bf16_normal(N, d, seed, 7, R, T, E)
    y = synth.bf16_normal(Q, d, seed, 8, R, T, E)
    o = oracle.run_path(logits, R, T, S, K)
    disp_or = oracle.permute(hidden, K, o["dest_row"])
    out_or = oracle.combine(y, N, K, o["dest_row"], o["w"])

    L = gh.make_layer(R, T, E, K, S, d)
    try:
        gh.load_inputs(L, logits, hidden)
        y_dev = gh.bf16_to_device(y, L.device)
        L.run_routing()
        L.permute()
        L.combine(y=y_dev)
        assert L.error() == 0
        g = gh.routing_results(L)
        gh.assert_routing_equal(g, o)
        np.testing.assert_array_equal(gh.bf16_to_host_u16(L.dispatch), disp_or,
                                      err_msg="dispatch rows")
        rows = y[o["dest_row"].ravel()].reshape(N, K, d)
        gh.assert_combine_close(L.out.cpu().numpy(), out_or, gh.combine_scale(rows, o["w"]))
        # the separate gate, count, plan and reroute calls give the same
        # routing as the fused and overlapped ones
        L.run_routing(fused=False, overlap=False)
        assert L.error() == 0
        gh.assert_routing_equal(gh.routing_results(L), o)
        return g, o
    finally:
        L.close()


def test_small_workload_r8_e64():
    w = synth.WORKLOADS["small_r8_e64"]
    g, o = run_case(w.R, w.T, w.E, w.K, w.S, w.d, synth.logits(w))
    # the skewed workload does replicate
    assert o["plan"].stats[0] > 0


EDGE = [
    # R, T, E, K, S, d
    (3, 37, 6, 3, 2, 24),        # E < 32, K = 3 (10 rows per warp group), one partial tile
    (5, 411, 40, 5, 1, 40),      # E = 40 (partial second lane slot), K = 5, ragged tiles
    (1, 100, 4, 4, 3, 8),        # one rank, K = E, 8-element rows
    (4, 700, 256, 8, 8, 64),     # E = 256 (8 logits per lane), S = 8
    (16, 200, 32, 1, 0, 16),     # K = 1 (32 rows per warp group), no redundant slots
    (2, 2500, 16, 16, 2, 8),     # K = 16, 40 tiles
    (40, 64, 160, 8, 1, 5120),   # prefill-shaped rows
    (64, 16, 256, 8, 2, 7168),   # DeepSeek-V3-shaped rows (896 chunks of 16 B)
    (4, 64, 8, 2, 1, 16384),     # widest rows (3 warps x 2 ring buffers)
    (128, 9, 128, 6, 2, 16),     # R = 128, K = 6
]


@pytest.mark.parametrize("R,T,E,K,S,d", EDGE)
def test_edge_shapes(R, T, E, K, S, d):
    wl = synth.custom(R, T, E, K, S, d, cid=1000 + E + K + S, zipf_s=1.3)
    run_case(R, T, E, K, S, d, synth.logits(wl))


def test_ties_and_signed_zeros():
    rng = np.random.default_rng(5)
    R, T, E, K, S, d = 8, 300, 64, 4, 2, 32
    vals = np.array([-1.0, -0.0, 0.0, 0.5, 1.0], dtype=np.float32)
    logits = vals[rng.integers(0, len(vals), size=(R * T, E))]
    g, o = run_case(R, T, E, K, S, d, logits)


def test_all_equal_logits_pick_lowest_ids():
    R, T, E, K, S, d = 4, 64, 64, 8, 2, 16
    logits = np.zeros((R * T, E), dtype=np.float32)
    logits[::2] = -0.0
    g, o = run_case(R, T, E, K, S, d, logits)
    assert (g["idx"] == np.arange(K)).all()
    assert (g["w"] == np.float32(1.0 / K)).all()


def test_exactly_uniform_routing_makes_no_copies():
    R, T, E, K, S, d = 8, 64, 64, 4, 2, 32
    N = R * T
    n = np.arange(N)[:, None]
    e = np.arange(E)[None, :]
    # token n ranks experts (n*K + j) mod E first: every expert is hit Q/E times
    logits = (-((e - n * K) % E)).astype(np.float32)
    g, o = run_case(R, T, E, K, S, d, logits)
    assert (o["load_e"] == N * K // E).all()
    assert g["stats"][0] == 0 and (g["slot_expert"] == -1).all()


def test_extreme_skew_uses_every_slot():
    R, T, E, K, S, d = 8, 128, 64, 4, 2, 16
    row = np.linspace(1.0, -1.0, E).astype(np.float32)
    logits = np.tile(row, (R * T, 1))
    g, o = run_case(R, T, E, K, S, d, logits)
    assert g["stats"][0] == R * S


def test_reroute_is_deterministic_across_launches():
    w = synth.WORKLOADS["small_r8_e64"]
    L = gh.make_layer(w.R, w.T, w.E, w.K, w.S, w.d, with_rows=False)
    try:
        gh.load_inputs(L, synth.logits(w))
        L.run_routing()
        first = L.dest_row.clone()
        for _ in range(5):
            L.reroute()
            torch.cuda.synchronize()
            assert torch.equal(L.dest_row, first)
        assert L.error() == 0
    finally:
        L.close()


@pytest.mark.parametrize("R,T,E,K,S", [(8, 512, 64, 4, 2), (5, 411, 40, 5, 1), (64, 37, 128, 8, 2)])
def test_reroute_from_ids_not_16_byte_aligned(R, T, E, K, S):
    """The reroute copies a tile's ids into shared memory with 16-byte
    asynchronous copies when the id buffer is 16-byte aligned, and with 4-byte
    copies otherwise. Ids at offsets of one to three int32 take the second
    path and must give the oracle's slots and rows, as the aligned call does."""
    wl = synth.custom(R, T, E, K, S, 8, cid=2000 + E + K, zipf_s=1.3)
    logits = synth.logits(wl)
    o = oracle.run_path(logits, R, T, S, K)
    N, Q = R * T, R * T * K
    L = gh.make_layer(R, T, E, K, S, 8, with_rows=False)
    try:
        gh.load_inputs(L, logits)
        L.run_routing()
        assert L.error() == 0
        np.testing.assert_array_equal(L.dest_row.cpu().numpy(), o["dest_row"])
        buf = torch.empty(Q + 3, dtype=torch.int32, device=L.device)
        for off in (1, 2, 3):
            ids = buf[off:off + Q].view(N, K)
            ids.copy_(L.idx)
            phys = torch.full_like(L.phys_slot, -7)
            dest = torch.full_like(L.dest_row, -7)
            ue.ue_reroute(L.ctx, ids, L.plan, phys, dest)
            assert L.error() == 0
            np.testing.assert_array_equal(phys.cpu().numpy(), o["phys_slot"])
            np.testing.assert_array_equal(dest.cpu().numpy(), o["dest_row"])
    finally:
        L.close()


@pytest.mark.parametrize("R,T,E,K,S,seed", [(3, 1, 6, 1, 2, 0), (4, 1, 8, 1, 4, 3),
                                            (5, 1, 10, 1, 3, 0)])
def test_replicas_with_zero_quota(R, T, E, K, S, seed):
    """A layout the greedy cannot balance (the master of a hot expert shares
    its rank with another master that keeps the remainder) goes on placing
    copies until the slots run out: experts end with more copies than pairs,
    so some copies get a quota of 0 (floor(L/c) = 0). The reroute's record of
    each expert's first copy in the tile and its division path must skip
    those copies as the oracle does."""
    rng = np.random.default_rng(seed)
    logits = rng.normal(size=(R * T, E)).astype(np.float32)
    logits[:, 0] += 4.0
    logits[:, 1] += 2.0
    o = oracle.run_path(logits, R, T, S, K)
    L = o["load_e"]
    nc = np.asarray(o["plan"].n_copies)
    assert ((nc > L) & (L > 0)).any()
    run_case(R, T, E, K, S, 8, logits)
