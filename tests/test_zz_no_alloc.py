"""ue_reroute_noalloc against ue_reroute, through the C ABI.

ue_reroute_noalloc serves callers that cannot allocate device memory: it
takes no context and keeps its look-back scratch in a fixed array inside the
library. Its routing must be identical (bit-exact, as every integer output of
the path) to the context-based ue_reroute on the same ids and plan, on two
calls in a row, for two workload sizes one after the other (the shared
scratch keeps the previous call's contents, so each call must clear what it
uses). Sizes beyond the fixed array are refused before any launch.

This file is collected last so that a failure here cannot hide the result
of any other test; it passes on its own in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
import token_rerouting_b200 as ue
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["small_r8_e64", "dsv3_layer_r64_e256"])
def test_noalloc_reroute_matches_context_reroute(name):
    w = synth.WORKLOADS[name]
    L = gh.make_layer(w.R, w.T, w.E, w.K, w.S, w.d, with_rows=False)
    try:
        gh.load_inputs(L, synth.logits(w))
        L.run_routing()
        assert L.error() == ue.UE_OK
        phys = torch.empty_like(L.phys_slot)
        dest = torch.empty_like(L.dest_row)
        err = torch.zeros(2, dtype=torch.int32, device=L.device)
        for _ in range(2):
            phys.fill_(-7)
            dest.fill_(-7)
            ue.ue_reroute_noalloc(L.cfg, L.idx, L.plan, phys, dest, err)
            torch.cuda.synchronize()
            assert err.tolist() == [0, 0]
            assert torch.equal(phys, L.phys_slot)
            assert torch.equal(dest, L.dest_row)
    finally:
        L.close()


def test_noalloc_refuses_sizes_beyond_its_scratch():
    gh.ensure_built()
    lib = ue.load_library()
    # 64 x 32768 tokens x 16 = 33.5M pairs: 4096 tiles x 256 experts > 262144 words
    cfg = ue.make_config(64, 32768, 256, 16, 2, 64)
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    pl = ue.placement(dummy, dummy, dummy, dummy, dummy, dummy)
    rc = lib.ue_reroute_noalloc(ctypes.byref(cfg), dummy.data_ptr(), ctypes.byref(pl),
                                dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(),
                                torch.cuda.current_stream().cuda_stream)
    assert rc == ue.UE_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert int(dummy.abs().sum()) == 0
