"""ue_reroute_noalloc against the oracle and against ue_reroute, through the
C ABI.

ue_reroute_noalloc serves callers that cannot allocate device memory: it
takes no context and keeps its look-back scratch in a fixed array inside the
library. Its routing must equal the oracle's reroute (bit-exact, as every
integer output of the path) and the context-based ue_reroute on the same ids
and plan, on two calls in a row, for two workload sizes one after the other
(the shared scratch keeps the previous call's contents, so each call must
leave it ready for the next). A call that ends in a device-side error (an
expert id out of range) reports it through the caller's error word and
leaves the scratch ready: the next valid call matches again. Sizes beyond
the fixed array, a missing error word and host memory are refused before
any launch.

This file is collected last so that a failure here cannot hide the result
of any other test; it passes on its own in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import token_rerouting_b200 as ue
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu


def oracle_reroute(w, L):
    """The oracle's reroute of the GPU's own ids under the GPU's own plan
    (both already checked against the oracle by the other tests)."""
    torch.cuda.synchronize()
    pa = L.plan_arrays()
    pl = oracle.Plan(pa["slot_expert"], pa["n_copies"], pa["slot_quota"], pa["slot_offset"],
                     pa["rank_load"], pa["stats"], np.empty(0, np.int32), np.empty(0, np.int32))
    return oracle.reroute(L.idx.cpu().numpy(), w.R, w.E, w.S, pl)


@pytest.mark.parametrize("name", ["small_r8_e64", "dsv3_layer_r64_e256"])
def test_noalloc_reroute_matches_oracle_and_context_reroute(name):
    w = synth.WORKLOADS[name]
    L = gh.make_layer(w.R, w.T, w.E, w.K, w.S, w.d, with_rows=False)
    try:
        gh.load_inputs(L, synth.logits(w))
        L.run_routing()
        assert L.error() == ue.UE_OK
        phys_or, dest_or = oracle_reroute(w, L)
        phys = torch.empty_like(L.phys_slot)
        dest = torch.empty_like(L.dest_row)
        err = torch.zeros(2, dtype=torch.int32, device=L.device)
        for _ in range(2):
            phys.fill_(-7)
            dest.fill_(-7)
            ue.ue_reroute_noalloc(L.cfg, L.idx, L.plan, phys, dest, err)
            torch.cuda.synchronize()
            assert err.tolist() == [0, 0]
            np.testing.assert_array_equal(phys.cpu().numpy(), phys_or)
            np.testing.assert_array_equal(dest.cpu().numpy(), dest_or)
            assert torch.equal(phys, L.phys_slot)
            assert torch.equal(dest, L.dest_row)
    finally:
        L.close()


def test_noalloc_device_error_then_clean_call():
    w = synth.WORKLOADS["small_r8_e64"]
    L = gh.make_layer(w.R, w.T, w.E, w.K, w.S, w.d, with_rows=False)
    try:
        gh.load_inputs(L, synth.logits(w))
        L.run_routing()
        assert L.error() == ue.UE_OK
        phys_or, dest_or = oracle_reroute(w, L)
        phys = torch.empty_like(L.phys_slot)
        dest = torch.empty_like(L.dest_row)
        err = torch.zeros(2, dtype=torch.int32, device=L.device)
        bad = L.idx.clone()
        n, k = 1234, 2
        bad[n, k] = w.E + 3  # one expert id out of range: reported, not a fault
        ue.ue_reroute_noalloc(L.cfg, bad, L.plan, phys, dest, err)
        torch.cuda.synchronize()
        assert err.tolist() == [ue.UE_ERR_DEVICE_BOUNDS, n * w.K + k]
        assert int(phys[n, k]) == -1 and int(dest[n, k]) == -1
        # the shared scratch is ready for the next call
        err.zero_()
        phys.fill_(-7)
        dest.fill_(-7)
        ue.ue_reroute_noalloc(L.cfg, L.idx, L.plan, phys, dest, err)
        torch.cuda.synchronize()
        assert err.tolist() == [0, 0]
        np.testing.assert_array_equal(phys.cpu().numpy(), phys_or)
        np.testing.assert_array_equal(dest.cpu().numpy(), dest_or)
        assert torch.equal(phys, L.phys_slot) and torch.equal(dest, L.dest_row)
    finally:
        L.close()


def _raw_call(lib, cfg, idx, pl, phys, dest, err):
    return lib.ue_reroute_noalloc(ctypes.byref(cfg), idx, ctypes.byref(pl), phys, dest, err,
                                  torch.cuda.current_stream().cuda_stream)


def test_noalloc_refuses_before_launch():
    gh.ensure_built()
    lib = ue.load_library()
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = dummy.data_ptr()
    pl = ue.placement(dummy, dummy, dummy, dummy, dummy, dummy)
    # 64 x 32768 tokens x 16 = 33.5M pairs: 4096 tiles x 256 experts > 262144 words
    big = ue.make_config(64, 32768, 256, 16, 2, 64)
    assert _raw_call(lib, big, p, pl, p, p, p) == ue.UE_ERR_UNSUPPORTED
    small = ue.make_config(1, 4, 4, 1, 0, 8)
    # no error word
    assert _raw_call(lib, small, p, pl, p, p, None) == ue.UE_ERR_INVALID_ARG
    # host memory in place of device buffers
    host = np.zeros(16, dtype=np.int32)
    hp = host.ctypes.data
    assert _raw_call(lib, small, hp, pl, p, p, p) == ue.UE_ERR_INVALID_ARG
    assert _raw_call(lib, small, p, pl, hp, p, p) == ue.UE_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert int(dummy.abs().sum()) == 0 and int(np.abs(host).sum()) == 0
