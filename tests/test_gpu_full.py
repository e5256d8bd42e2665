"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times.

Routing half (top-k ids and weights, counts, plan, reroute): every element
against the oracle. Rows: a sample of dispatch rows (random ones plus the
first and last row of every non-empty slot) against the oracle's permute at
those rows; the combine on a sample of tokens whose K expert-output rows are
independent random rows written at the oracle's destination rows; and, for
the identity experts the benchmark uses, the property
out[n] = hidden[n] * sum_k w[n,k] within fp32 rounding.
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

        rng = np.random.default_rng(w.cid)
        pl = o["plan"]
        nz = np.nonzero(pl.slot_quota)[0]
        edges = np.concatenate([pl.slot_offset[nz], pl.slot_offset[nz + 1] - 1])
        rows = np.unique(np.concatenate([rng.choice(w.Q, 4096, replace=False), edges]))
        rows_dev = torch.from_numpy(rows).to(L.device)
        got = gh.bf16_to_host_u16(L.dispatch[rows_dev])
        np.testing.assert_array_equal(got, oracle.permute_rows(hidden, w.K, o["dest_row"], rows))

        # identity experts: out[n] = hidden[n] * sum_k w[n, k] up to fp32 rounding
        toks = np.sort(rng.choice(w.N, 512, replace=False))
        toks_dev = torch.from_numpy(toks).to(L.device)
        out = L.out[toks_dev].cpu().numpy().astype(np.float64)
        h = synth.bf16_bits_to_f32(hidden[toks]).astype(np.float64)
        wsum = g["w"][toks].astype(np.float64)
        expect = h * wsum.sum(axis=1, keepdims=True)
        bound = (w.K + 1) * 2.0 ** -24 * np.abs(h) * np.abs(wsum).sum(axis=1, keepdims=True)
        assert (np.abs(out - expect) <= bound + 1e-30).all()

        # independent expert outputs for the sampled tokens, at the oracle's rows
        yk = synth.bf16_normal(len(toks) * w.K, w.d, 0, 9, w.cid)
        dst = o["dest_row"][toks].ravel()
        L.dispatch[torch.from_numpy(dst).to(L.device)] = gh.bf16_to_device(yk, L.device)
        L.combine()
        assert L.error() == 0
        dest_c = np.zeros((w.N, w.K), dtype=np.int32)
        dest_c[toks] = np.arange(len(toks) * w.K, dtype=np.int32).reshape(-1, w.K)
        out_or = oracle.combine(yk, w.N, w.K, dest_c, o["w"], tokens=toks)
        scale = gh.combine_scale(yk.reshape(len(toks), w.K, w.d), o["w"][toks])
        gh.assert_combine_close(L.out[toks_dev].cpu().numpy(), out_or, scale)
    finally:
        L.close()
