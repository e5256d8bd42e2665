"""The non-stationary sweep: 48 layers x 8 microbatches of the Qwen3-shaped
layer (R=64, 4096 tokens per rank, E=128, K=8, S=2, d=4096), Zipf exponent
and hot set redrawn per instance, with a uniform instance (0,0) and a
30%-single-expert instance (0,1). The whole path is captured once as a CUDA
graph over fixed buffers; each instance's logits are staged into the input
buffer and the graph is replayed.

Every instance is checked on the device by properties that hold at any size
(dest_row is a permutation of the pairs; each slot receives exactly its
quota; each pair lands on a copy of its own expert; rank loads sum to the
pairs). Eight instances, the two special ones included, are compared with
the oracle element by element on the routing and on sampled dispatch rows.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu


def slot_owner(L, dev):
    """Expert held by every physical slot (-1 for an empty redundant slot)."""
    M, S, R = L.M, L.S, L.R
    p = torch.arange(L.P, device=dev)
    r, l = p // (M + S), p % (M + S)
    owner = torch.where(l < M, r * M + l, torch.full_like(p, -1))
    if L.G > 0:
        g = r * S + (l - M)
        rep = L.slot_expert[: L.G].long()[g.clamp(0, L.G - 1)]
        owner = torch.where(l < M, owner, rep)
    return owner


def test_sweep_graph_captured():
    w = synth.WORKLOADS["sweep_48x8_r64_e128"]
    L = gh.make_layer(w.R, w.T, w.E, w.K, w.S, w.d)
    dev = L.device
    try:
        hidden = synth.hidden(w)
        L.hidden.copy_(gh.bf16_to_device(hidden, dev))
        L.logits.copy_(torch.from_numpy(synth.logits(w, 0, 0)))
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            L.run(stream=s)
        torch.cuda.current_stream(dev).wait_stream(s)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            L.run(stream=s)
        torch.cuda.synchronize(dev)

        rng = np.random.default_rng(5)
        others = [(int(x) // w.microbatches, int(x) % w.microbatches)
                  for x in rng.choice(np.arange(2, w.layers * w.microbatches), 6, replace=False)]
        exact = {(0, 0), (0, 1), *others}
        ar = torch.arange(w.Q, device=dev, dtype=torch.int32)
        iters, skew_before, skew_after = [], [], []
        for layer in range(w.layers):
            for mb in range(w.microbatches):
                logits = synth.logits(w, layer, mb)
                L.logits.copy_(torch.from_numpy(logits))
                graph.replay()
                torch.cuda.synchronize(dev)
                # properties, on the device
                dest = L.dest_row.flatten()
                assert torch.equal(torch.sort(dest).values, ar), (layer, mb)
                phys = L.phys_slot.flatten().long()
                counts = torch.bincount(phys, minlength=L.P)
                assert torch.equal(counts.int(), L.slot_quota), (layer, mb)
                owner = slot_owner(L, dev)
                assert torch.equal(owner[phys], L.idx.flatten().long()), (layer, mb)
                assert int(L.rank_load.long().sum()) == w.Q
                st = L.stats.cpu().numpy()
                iters.append(int(st[0]))
                skew_before.append(st[1] / (w.Q / w.R))
                skew_after.append(st[2] / (w.Q / w.R))
                if (layer, mb) in exact:
                    o = oracle.run_path(logits, w.R, w.T, w.S, w.K)
                    gh.assert_routing_equal(gh.routing_results(L), o)
                    rows = np.sort(rng.choice(w.Q, 2048, replace=False))
                    got = gh.bf16_to_host_u16(L.dispatch[torch.from_numpy(rows).to(dev)])
                    np.testing.assert_array_equal(
                        got, oracle.permute_rows(hidden, w.K, o["dest_row"], rows))
        assert L.error() == 0
        # the sweep spans balanced and heavily skewed instances
        assert min(skew_before) < 1.1 and max(skew_before) > 2.0
        assert len(iters) == w.layers * w.microbatches
    finally:
        L.close()
