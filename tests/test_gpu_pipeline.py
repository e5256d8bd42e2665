"""The benchmark's pipelined schedule, checked against the oracle: two layer
instances alternate; each step's routing (the gate with the count fused,
then ue_plan_reroute, whose reroute starts while the plan runs) goes on a
second, higher-priority stream while the other instance permutes and
combines on the main stream, with events ordering each instance's uses.
After several steps every routing output of both instances and every
dispatch row must equal the oracle's."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

R, T, E, K, S, d = 64, 256, 128, 8, 2, 512


def test_pipelined_steps_match_the_oracle():
    ws = [synth.custom(R, T, E, K, S, d, cid=3100 + i, zipf_s=1.0 + 0.3 * i) for i in range(2)]
    logits = [synth.logits(w) for w in ws]
    hidden = [synth.hidden(w) for w in ws]
    insts = [gh.make_layer(R, T, E, K, S, d) for _ in ws]
    try:
        for L, lg, hd in zip(insts, logits, hidden):
            gh.load_inputs(L, lg, hd)
        dev = insts[0].device
        main = torch.cuda.current_stream(dev)
        side = torch.cuda.Stream(dev, priority=-5)
        ev_routed = [torch.cuda.Event() for _ in insts]
        ev_done = [torch.cuda.Event() for _ in insts]
        for e in ev_done:
            e.record(main)
        for i in range(8):
            x = i % 2
            L = insts[x]
            side.wait_event(ev_done[x])
            L.gate_count(stream=side)
            L.plan_reroute(stream=side)
            ev_routed[x].record(side)
            main.wait_event(ev_routed[x])
            L.permute(stream=main)
            L.combine(stream=main)
            ev_done[x].record(main)
        torch.cuda.synchronize(dev)
        for L, lg, hd in zip(insts, logits, hidden):
            assert L.error() == 0
            o = oracle.run_path(lg, R, T, S, K)
            gh.assert_routing_equal(gh.routing_results(L), o)
            gh.assert_dispatch_all_rows(L, hd, K, o["dest_row"])
    finally:
        for L in insts:
            L.close()
