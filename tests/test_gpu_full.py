"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times (Qwen3-shaped layer, DeepSeek-V3-shaped layer, EP40
prefill), every output element against the oracle:

* the routing half (top-k ids and weights, counts, every plan array, the
  reroute): every element, bit-exact (weights within one ulp), through the
  fused gate and count; the separate gate and count calls must give the
  same bits;
* the permute: every dispatch row against the oracle's permute, byte for
  byte;
* the combine: every output element against the oracle's fp64 combine
  within the normwise 1e-6 tolerance, with expert outputs that are
  independent of the routing: dispatch row r holds hidden[sigma[r]] for a
  seeded random sigma, so a row read from the wrong place is caught;
* and, for the identity experts the benchmark uses (the combine reads the
  dispatch buffer the permute wrote), the property
  out[n] = hidden[n] * sum_k w[n,k] within fp32 rounding on a token sample.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

FULL = ["qwen3_layer_r64_e128", "dsv3_layer_r64_e256", "prefill_ep40_e160"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workload(name):
    w = synth.WORKLOADS[name]
    logits = synth.logits(w)
    hidden = synth.hidden(w)
    o = oracle.run_path(logits, w.R, w.T, w.S, w.K)
    L = gh.make_layer(w.R, w.T, w.E, w.K, w.S, w.d)
    try:
        gh.load_inputs(L, logits, hidden)
        L.run_routing()
        L.permute()
        L.combine()  # identity experts, as in the benchmark
        assert L.error() == 0
        g = gh.routing_results(L)
        gh.assert_routing_equal(g, o)
        # the separate gate and count calls give the same ids, weights and counts
        fused = [t.clone() for t in (L.idx, L.w, L.load_re, L.load_e)]
        L.gate()
        L.count()
        assert L.error() == 0
        assert all(torch.equal(a, b) for a, b in zip(fused, (L.idx, L.w, L.load_re, L.load_e)))

        # every dispatch row
        gh.assert_dispatch_all_rows(L, hidden, w.K, o["dest_row"])

        # identity experts: out[n] = hidden[n] * sum_k w[n, k] up to fp32 rounding
        rng = np.random.default_rng(w.cid)
        toks = np.sort(rng.choice(w.N, 4096, replace=False))
        toks_dev = torch.from_numpy(toks).to(L.device)
        out = L.out[toks_dev].cpu().numpy().astype(np.float64)
        h = synth.bf16_bits_to_f32(hidden[toks]).astype(np.float64)
        wsum = g["w"][toks].astype(np.float64)
        expect = h * wsum.sum(axis=1, keepdims=True)
        bound = (w.K + 1) * 2.0 ** -24 * np.abs(h) * np.abs(wsum).sum(axis=1, keepdims=True)
        assert (np.abs(out - expect) <= bound + 1e-30).all()

        # every combine element, with independent expert outputs in the whole
        # dispatch buffer
        sigma = synth.expert_output_rows(w)
        gh.expert_outputs_on_device(L, hidden, sigma)
        L.combine()
        assert L.error() == 0
        gh.assert_combine_all_tokens(L, hidden, sigma, w.K, o["dest_row"], o["w"])
    finally:
        L.close()
