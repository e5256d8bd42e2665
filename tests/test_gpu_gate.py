"""GPU parity of the gate's two selection paths for K = 8 and E a multiple of
32 from 64 to 256, and of the gate with the exact histogram fused in.

The fast path ranks packed keys (an order key whose low log2(E) bits carry
the expert id) and re-selects, with full keys and the lower-id tie rule, every
row whose first K+1 picks are not separated above the dropped bits. These
tests mix, inside the same warp groups of four rows, rows of distinct normal
logits (packed picks kept), rows of exact ties and signed zeros, and rows of
values a few fp32 ulps apart (both re-selected), with a ragged last group.
Each lane pops from a short list of its largest keys; rows whose leading
values sit in one lane (three or more of them, before or at the last round)
test the hand-over from a lane that ran out of its list.
Both paths must give the oracle's ids bit for bit and its weights within one
fp32 ulp; a logits buffer that is not 16-byte aligned takes the generic
kernel, which must agree as well.

ue_gate_count must give the same ids and weights and the oracle's counts
bit for bit, on shapes whose CTAs cover one to three source ranks (the
histogram inside the gate kernel) and on one where they cover more (the
gate kernel, then the count kernel), on calls in a row and on replays of a
captured CUDA graph (the fused kernel's scratch is left ready by each launch).

"UltraEP" README, "Interface / 2. Forward and backward" (probs, routing_map
from the router); "What Happened" (routing from the exact probabilities).
"""
import numpy as np
import pytest
import torch

import oracle
import token_rerouting_b200 as ue
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu


def mixed_logits(N, E, seed):
    rng = np.random.default_rng(seed)
    out = rng.standard_normal((N, E)).astype(np.float32)
    kind = rng.integers(0, 4, size=N)
    ties = np.array([-1.0, -0.0, 0.0, 0.5, 1.0], dtype=np.float32)
    t_rows = kind == 1
    out[t_rows] = ties[rng.integers(0, len(ties), size=(int(t_rows.sum()), E))]
    c_rows = kind == 2
    steps = rng.integers(0, 200, size=(int(c_rows.sum()), E)).astype(np.float64)
    out[c_rows] = (1.0 + steps * 2.0 ** -23).astype(np.float32)
    # kind 3: normal rows whose two leaders sit one ulp apart
    n_rows = np.flatnonzero(kind == 3)
    lead = np.argmax(out[n_rows], axis=1)
    other = (lead + 1 + rng.integers(0, E - 1, size=len(n_rows))) % E
    top = out[n_rows, lead]
    out[n_rows, other] = np.nextafter(top, np.float32(-np.inf))
    return out


def run_gate(E, N, logits, offset_floats=0):
    R = 2 if N % 2 == 0 else 1
    T = N // R
    K = 8
    dev = torch.device("cuda", 0)
    cfg = ue.make_config(R, T, E, K, 1, 8)
    ctx = ue.ue_init(cfg, 0)
    try:
        buf = torch.empty(N * E + offset_floats, dtype=torch.float32, device=dev)
        lg = buf[offset_floats:]
        lg.copy_(torch.from_numpy(np.ascontiguousarray(logits).ravel()))
        idx = torch.full((N, K), -7, dtype=torch.int32, device=dev)
        w = torch.full((N, K), -1.0, dtype=torch.float32, device=dev)
        ue.ue_gate_topk(ctx, lg, idx, w)
        assert ue.ue_get_error(ctx) == ue.UE_OK
        torch.cuda.synchronize()
        return idx.cpu().numpy(), w.cpu().numpy()
    finally:
        ue.ue_destroy(ctx)


@pytest.mark.parametrize("E", [64, 96, 128, 160, 192, 224, 256])
@pytest.mark.parametrize("N", [2002, 4099])
def test_packed_and_exact_rows_in_one_group(E, N):
    gh.ensure_built()
    logits = mixed_logits(N, E, seed=E + N)
    idx_or, w_or = oracle.gate_topk(logits, 8)
    idx, w = run_gate(E, N, logits)
    np.testing.assert_array_equal(idx, idx_or)
    gh.assert_weights_close(w, w_or)


@pytest.mark.parametrize("E", [128, 256])
def test_unaligned_logits_take_the_generic_kernel(E):
    gh.ensure_built()
    N = 1030
    logits = mixed_logits(N, E, seed=3 * E)
    idx_or, w_or = oracle.gate_topk(logits, 8)
    idx_a, w_a = run_gate(E, N, logits, offset_floats=0)
    idx_u, w_u = run_gate(E, N, logits, offset_floats=1)
    np.testing.assert_array_equal(idx_a, idx_or)
    np.testing.assert_array_equal(idx_u, idx_or)
    gh.assert_weights_close(w_a, w_or)
    gh.assert_weights_close(w_u, w_or)
    np.testing.assert_array_equal(w_a, w_u)


def lane_experts(E, lane):
    """Experts one lane of the fast kernel holds: 128 c + 4 lane + j for each
    16-byte chunk c, then 128 C + 32 t + lane for each 4-byte tail load t."""
    nch, nt = E // 128, (E % 128) // 32
    ids = [128 * c + 4 * lane + j for c in range(nch) for j in range(4)]
    return ids + [128 * nch + 32 * t + lane for t in range(nt)]


# positions among the leading K+1 values that one lane's experts take
CLUSTERS = [(0, 1, 2), (0, 1, 8), (0, 4, 7), (5, 6, 7, 8), (1, 2, 3, 4), (0, 1, 2, 3, 4, 5),
            (2, 7), (7, 8)]


def clustered_logits(N, E, seed):
    """Rows whose leading values sit in one lane of the fast kernel, at the
    positions CLUSTERS lists (a lane that gives up its whole list before the
    last round, or exactly at it), between rows of distinct normal logits."""
    rng = np.random.default_rng(seed)
    out = rng.standard_normal((N, E)).astype(np.float32)
    for n in range(0, N, 2):
        pos = CLUSTERS[(n // 2) % len(CLUSTERS)]
        mine = lane_experts(E, int(rng.integers(32)))
        pos = pos[:len(mine)]
        out[n] -= 10.0
        others = rng.permutation(np.setdiff1d(np.arange(E), mine))
        chosen = rng.permutation(mine)[:len(pos)]
        o = 0
        for p in range(9):
            if p in pos:
                e = chosen[pos.index(p)]
            else:
                e = others[o]
                o += 1
            out[n, e] = np.float32(10.0 - p)
    return out


@pytest.mark.parametrize("E", [64, 96, 128, 160, 192, 224, 256])
def test_one_lane_holding_many_leading_picks(E):
    gh.ensure_built()
    N = 2002
    logits = clustered_logits(N, E, seed=7 * E)
    idx_or, w_or = oracle.gate_topk(logits, 8)
    idx, w = run_gate(E, N, logits)
    np.testing.assert_array_equal(idx, idx_or)
    gh.assert_weights_close(w, w_or)
    (res,) = run_gate_count(2, N // 2, E, [logits])
    np.testing.assert_array_equal(res[0], idx_or)
    lre_or, le_or = oracle.count(idx_or, 2, N // 2, E)
    np.testing.assert_array_equal(res[2], lre_or)
    np.testing.assert_array_equal(res[3], le_or)


def test_all_rows_equal_pick_the_lowest_ids():
    gh.ensure_built()
    N, E = 37, 256
    logits = np.zeros((N, E), dtype=np.float32)
    logits[1::3] = -0.0
    idx, w = run_gate(E, N, logits)
    assert (idx == np.arange(8)).all()
    assert (w == np.float32(1.0 / 8)).all()


def run_gate_count(R, T, E, logits_list, graph=False):
    """ue_gate_count over each logits array in turn (eagerly, or as replays of
    one captured graph); returns the outputs of every call."""
    N, K = R * T, 8
    dev = torch.device("cuda", 0)
    cfg = ue.make_config(R, T, E, K, 1, 8)
    ctx = ue.ue_init(cfg, 0)
    try:
        lg = torch.empty((N, E), dtype=torch.float32, device=dev)
        idx = torch.full((N, K), -7, dtype=torch.int32, device=dev)
        w = torch.full((N, K), -1.0, dtype=torch.float32, device=dev)
        load_re = torch.full((R, E), 12345, dtype=torch.int32, device=dev)
        load_e = torch.full((E,), 12345, dtype=torch.int32, device=dev)
        s = torch.cuda.Stream(device=dev)
        g = None
        if graph:
            lg.copy_(torch.from_numpy(logits_list[0]))
            with torch.cuda.stream(s):
                ue.ue_gate_count(ctx, lg, idx, w, load_re, load_e, s)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                ue.ue_gate_count(ctx, lg, idx, w, load_re, load_e, s)
            torch.cuda.synchronize()
        res = []
        for logits in logits_list:
            lg.copy_(torch.from_numpy(logits))
            torch.cuda.synchronize()
            if g is not None:
                g.replay()
            else:
                ue.ue_gate_count(ctx, lg, idx, w, load_re, load_e)
            assert ue.ue_get_error(ctx, s if g is not None else None) == ue.UE_OK
            torch.cuda.synchronize()
            res.append((idx.cpu().numpy(), w.cpu().numpy(), load_re.cpu().numpy(),
                        load_e.cpu().numpy()))
        return res
    finally:
        ue.ue_destroy(ctx)


@pytest.mark.parametrize("R,T,E", [(2, 2049, 128), (128, 2, 128), (64, 3, 192), (40, 1001, 160),
                                   (32, 777, 224), (32, 33, 96), (64, 65, 64), (8, 4099, 256),
                                   (128, 1, 256)])
@pytest.mark.parametrize("graph", [False, True])
def test_gate_count_matches_the_oracle(R, T, E, graph):
    gh.ensure_built()
    lgs = [mixed_logits(R * T, E, seed=R * 1000 + T + s) for s in range(3)]
    for logits, (idx, w, load_re, load_e) in zip(lgs, run_gate_count(R, T, E, lgs, graph)):
        idx_or, w_or = oracle.gate_topk(logits, 8)
        np.testing.assert_array_equal(idx, idx_or)
        gh.assert_weights_close(w, w_or)
        lre_or, le_or = oracle.count(idx_or, R, T, E)
        np.testing.assert_array_equal(load_re, lre_or)
        np.testing.assert_array_equal(load_e, le_or)
