"""GPU parity of the planner variants ("UltraEP" README, "Performance Tuning /
Replication planning"): the greedy with a minimal load per replica, the
capacity planner (bisection on max/mean with a quota oracle), the reroute of
its general quotas, the interleaved order, and the locality-aware split with
its reroute. Everything here is integer: bit-exact against the oracle
(plans, splits, physical slots, dispatch rows), through the C ABI.

Sizes: every hand-worked case, random skewed loads over the whole range of
the config limits (R = 1 .. 128, E up to 256, S up to 8, tiny and large
minimums, eps down to 1e-4, thresholds above 1, zero-load masters), edge
shapes whose reroute tiles straddle many source ranks, and the three full
layer workloads (Q = 1 M to 2.6 M pairs; the oracle's reroute is one pass).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
import token_rerouting_b200 as ue
from tests import gpu_helpers as gh
from tests.test_oracle_plan import zipf_loads

pytestmark = pytest.mark.gpu

PLAN_KEYS = ("slot_expert", "n_copies", "slot_quota", "slot_offset", "rank_load", "stats")


def golden(kind):
    with open(os.path.join(os.path.dirname(__file__), "golden", "variant_cases.json")) as f:
        return json.load(f)[kind]


def gpu_plan(L, load_e, opts):
    L.load_e.copy_(torch.from_numpy(np.ascontiguousarray(load_e, dtype=np.int32)))
    L.plan_ex(opts)
    assert L.error() == 0
    return L.plan_arrays()


def assert_plan_equal(g, pl, what=""):
    for key in PLAN_KEYS:
        np.testing.assert_array_equal(g[key], getattr(pl, key), err_msg=f"{what} {key}")


def bisect_opts(m=1024, D=100, thr=None, zero=False):
    return ue.plan_opts(ue.UE_SOLVER_BISECT, min_tokens=m, eps_inv=D, threshold=thr,
                        allow_zero_master=zero)


# ------------------------------------------------------------------ plans

def test_bisect_hand_cases():
    for c in golden("bisect"):
        L = gh.make_layer(c["R"], 1, c["E"], 1, c["S"], 8, with_rows=False)
        try:
            g = gpu_plan(L, c["load_e"], bisect_opts(c["min_tokens"], c["eps_inv"], c["threshold"],
                                                     bool(c["allow_zero"])))
            for key in PLAN_KEYS:
                assert g[key].tolist() == c[key], (c["name"], key)
        finally:
            L.close()


def test_greedy_min_tokens_hand_cases():
    for c in golden("greedy_min_tokens"):
        L = gh.make_layer(c["R"], 1, c["E"], 1, c["S"], 8, with_rows=False)
        try:
            g = gpu_plan(L, c["load_e"], ue.plan_opts(ue.UE_SOLVER_GREEDY,
                                                       min_tokens=c["min_tokens"]))
            for key in PLAN_KEYS:
                assert g[key].tolist() == c[key], (c["name"], key)
        finally:
            L.close()


PLAN_CONFIGS = [
    # R, E, S, zipf s, pairs per rank
    (8, 64, 2, 1.2, 2048),
    (64, 128, 2, 1.0, 32768),
    (64, 256, 2, 1.3, 16384),
    (40, 160, 1, 1.1, 65536),
    (128, 256, 2, 1.4, 4096),     # four ranks per lane, M = 2
    (128, 128, 2, 1.2, 4096),     # M = 1
    (2, 256, 8, 1.5, 100000),     # M = 128, eight experts per lane
    (16, 16, 8, 1.5, 1000),
    (3, 9, 1, 0.5, 300),
    (1, 8, 4, 2.0, 5000),         # one rank: never overloaded
]


@pytest.mark.parametrize("R,E,S,s,per_rank", PLAN_CONFIGS)
def test_bisect_random_loads(R, E, S, s, per_rank):
    rng = np.random.default_rng(R * 7 + E + S)
    L = gh.make_layer(R, 1, E, 1, S, 8, with_rows=False)
    try:
        options = [(1024, 100, None, False), (1, 100, None, False), (64, 1000, None, True),
                   (16, 10000, None, False), (256, 100, 105, False), (8, 7, 9, True)]
        for trial in range(6):
            load_e = zipf_loads(rng, E, 1, per_rank * R, s)
            if trial == 5:
                load_e[:] = 0
                load_e[rng.integers(E)] = per_rank * R      # one expert takes everything
            for m, D, thr, zero in options:
                pl = oracle.plan_bisect(load_e, R, S, eps_inv=D, threshold=thr, min_tokens=m,
                                        allow_zero_master=zero)
                g = gpu_plan(L, load_e, bisect_opts(m, D, thr, zero))
                assert_plan_equal(g, pl, f"trial {trial} m={m} D={D} thr={thr} zero={zero}")
        # uniform and empty loads
        for load_e in (np.full(E, per_rank * R // E, np.int32), np.zeros(E, np.int32)):
            g = gpu_plan(L, load_e, bisect_opts())
            assert_plan_equal(g, oracle.plan_bisect(load_e, R, S), "flat")
    finally:
        L.close()


@pytest.mark.parametrize("R,E,S,s,per_rank", PLAN_CONFIGS)
def test_greedy_min_tokens_random_loads(R, E, S, s, per_rank):
    rng = np.random.default_rng(R * 11 + E + S)
    L = gh.make_layer(R, 1, E, 1, S, 8, with_rows=False)
    try:
        for trial in range(4):
            load_e = zipf_loads(rng, E, 1, per_rank * R, s)
            for m in (0, 1, 1024, per_rank // 4):
                pl = oracle.plan(load_e, R, S, min_tokens=m)
                g = gpu_plan(L, load_e, ue.plan_opts(ue.UE_SOLVER_GREEDY, min_tokens=m))
                assert_plan_equal(g, pl, f"trial {trial} m={m}")
    finally:
        L.close()


def test_plan_ex_rejects_bad_options():
    L = gh.make_layer(8, 16, 64, 4, 2, 8, with_rows=False)
    try:
        lib = ue.load_library()
        bad = [ue.ue_plan_opts(2, 0, 100, 100, 0),          # unknown solver
               ue.ue_plan_opts(0, -1, 100, 100, 0),         # negative minimum
               ue.ue_plan_opts(1, 0, 100, 100, 0),          # bisection needs m >= 1
               ue.ue_plan_opts(1, 1, 0, 100, 0),            # eps_inv 0
               ue.ue_plan_opts(1, 1, 10001, 100, 0),        # eps_inv too large
               ue.ue_plan_opts(1, 1, 100, -1, 0),           # negative threshold
               ue.ue_plan_opts(1, 1, 100, 100, 2)]          # allow_zero not 0/1
        import ctypes
        for o in bad:
            rc = lib.ue_plan_ex(L.ctx, L.load_e.data_ptr(), ctypes.byref(o), ctypes.byref(L.plan),
                                None)
            assert rc == ue.UE_ERR_INVALID_ARG
    finally:
        L.close()


# ---------------------------------------------------- reroutes on real routing

SHAPES = [
    # R, T, E, K, S, d (d unused: routing only)
    (8, 512, 64, 4, 2, 8),
    (3, 37, 6, 3, 2, 8),        # tiles straddle many source ranks
    (5, 411, 40, 5, 1, 8),
    (16, 200, 32, 1, 0, 8),     # no redundant slot
    (2, 2500, 16, 16, 2, 8),
    (128, 9, 128, 6, 2, 8),     # R = 128, 54 pairs per rank
    (4, 700, 256, 8, 8, 8),
]


def routing(R, T, E, K, S, zipf_s=1.4):
    wl = synth.custom(R, T, E, K, S, 8, cid=2000 + E + K + S, zipf_s=zipf_s)
    return synth.logits(wl)


def planners(R, T, K):
    m_small = max(1, (T * K) // 64)
    return [("greedy", ue.plan_opts(ue.UE_SOLVER_GREEDY), lambda le, S: oracle.plan(le, R, S)),
            ("bisect", bisect_opts(m_small),
             lambda le, S: oracle.plan_bisect(le, R, S, min_tokens=m_small))]


def run_variant(R, T, E, K, S, logits, kind):
    """GPU: gate, count, a plan, then the reroute variant; oracle: the same.
    Returns (gpu dict, oracle dict)."""
    idx, _ = oracle.gate_topk(logits, K)
    load_re, load_e = oracle.count(idx, R, T, E)
    L = gh.make_layer(R, T, E, K, S, 8, with_rows=False)
    out = []
    try:
        gh.load_inputs(L, logits)
        for name, opts, oplan in planners(R, T, K):
            L.gate()
            L.count()
            L.plan_ex(opts)
            pl = oplan(load_e, S)
            if kind == "prefix":
                L.reroute()
                phys, dest = oracle.reroute(idx, R, E, S, pl)
            elif kind == "interleave":
                L.reroute_ex(ue.UE_ORDER_INTERLEAVE)
                phys, dest = oracle.reroute_interleave(idx, R, T, E, S, pl)
            else:
                L.locality_split()
                L.reroute_local()
                sq, so = oracle.locality_split(load_re, S, pl)
                phys, dest = oracle.reroute_local(idx, R, T, E, S, pl, sq, so)
            assert L.error() == 0
            torch.cuda.synchronize()
            np.testing.assert_array_equal(L.idx.cpu().numpy(), idx)
            assert_plan_equal(L.plan_arrays(), pl, name)
            if kind == "local":
                np.testing.assert_array_equal(L.src_quota.cpu().numpy(), sq, err_msg="src_quota")
                np.testing.assert_array_equal(L.src_offset.cpu().numpy(), so, err_msg="src_offset")
            np.testing.assert_array_equal(L.phys_slot.cpu().numpy(), phys, err_msg=f"{name} phys")
            np.testing.assert_array_equal(L.dest_row.cpu().numpy(), dest, err_msg=f"{name} dest")
            out.append((name, pl))
        return out
    finally:
        L.close()


@pytest.mark.parametrize("kind", ["prefix", "interleave", "local"])
@pytest.mark.parametrize("R,T,E,K,S,d", SHAPES)
def test_reroute_variants_small(R, T, E, K, S, d, kind):
    run_variant(R, T, E, K, S, routing(R, T, E, K, S), kind)


@pytest.mark.parametrize("kind", ["prefix", "interleave", "local"])
@pytest.mark.parametrize("name", ["qwen3_layer_r64_e128", "dsv3_layer_r64_e256",
                                  "prefill_ep40_e160"])
def test_reroute_variants_full_size(name, kind):
    w = synth.WORKLOADS[name]
    res = run_variant(w.R, w.T, w.E, w.K, w.S, synth.logits(w), kind)
    # the capacity planner does replicate on these skewed layers
    assert (res[1][1].slot_expert >= 0).any()


def test_locality_split_rejects_loads_of_other_ids():
    R, T, E, K, S = 8, 512, 64, 4, 2
    logits = routing(R, T, E, K, S)
    L = gh.make_layer(R, T, E, K, S, 8, with_rows=False)
    try:
        gh.load_inputs(L, logits)
        L.run_routing()
        assert L.error() == 0
        # per-rank loads that no longer sum to the quotas
        L.load_re[0, 0] += 1
        L.locality_split()
        assert L.error() == ue.UE_ERR_DEVICE_BOUNDS
        # a consistent split of other per-rank loads: each source rank's pairs
        # then no longer match its split, which the reroute reports
        L.load_re[0, 0] -= 1
        L.load_re[0, 1] -= 1
        L.load_re[1, 1] += 1
        L.locality_split()
        assert L.error() == 0
        L.reroute_local()
        assert L.error() == ue.UE_ERR_DEVICE_BOUNDS
    finally:
        L.close()
