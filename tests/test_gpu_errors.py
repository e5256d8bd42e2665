"""Device-side error paths, without faulting the GPU.

Bad ids and rows are caught by the kernels' own bounds checks (the access is
skipped and UE_ERR_DEVICE_BOUNDS recorded); a look-back wait is made to run
out by a test hook that keeps the first reroute tile from publishing (a flag
nothing sets) with a short poll limit, and must end with UE_ERR_TIMEOUT. After
each error the same context keeps working and matches the oracle again.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import token_rerouting_b200 as ue
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

R, T, E, K, S, d = 8, 512, 64, 4, 2, 64


@pytest.fixture()
def layer():
    L = gh.make_layer(R, T, E, K, S, d)
    yield L
    L.close()


def check_clean_run(L, logits):
    gh.load_inputs(L, logits)
    L.run_routing()
    assert L.error() == ue.UE_OK
    gh.assert_routing_equal(gh.routing_results(L), oracle.run_path(logits, R, T, S, K))


def test_bad_expert_id_in_count_and_reroute(layer):
    w = synth.custom(R, T, E, K, S, d, cid=501)
    logits = synth.logits(w)
    gh.load_inputs(layer, logits)
    layer.run_routing()
    assert layer.error() == ue.UE_OK
    layer.idx[3, 1] = E + 7
    layer.idx[100, 0] = -2
    layer.count()
    assert layer.error() == ue.UE_ERR_DEVICE_BOUNDS
    layer.reroute()
    assert layer.error() == ue.UE_ERR_DEVICE_BOUNDS
    # the bad pairs get no slot and no row
    assert int(layer.dest_row[3, 1]) == -1 and int(layer.phys_slot[100, 0]) == -1
    check_clean_run(layer, logits)


def test_rows_out_of_range_in_permute_and_combine(layer):
    w = synth.custom(R, T, E, K, S, d, cid=502)
    logits = synth.logits(w)
    gh.load_inputs(layer, logits, synth.hidden(w))
    layer.run_routing()
    layer.dispatch.zero_()
    layer.dest_row[0, 0] = -1
    layer.dest_row[7, 2] = R * T * K + 5
    layer.permute()
    assert layer.error() == ue.UE_ERR_DEVICE_BOUNDS
    layer.combine()
    assert layer.error() == ue.UE_ERR_DEVICE_BOUNDS
    check_clean_run(layer, logits)


def test_negative_load_in_plan(layer):
    load = torch.full((E,), 10, dtype=torch.int32, device=layer.device)
    load[5] = -3
    ue.ue_plan(layer.ctx, load, layer.plan)
    assert layer.error() == ue.UE_ERR_DEVICE_BOUNDS


def test_lookback_wait_runs_out_and_context_recovers(layer):
    w = synth.custom(R, T, E, K, S, d, cid=503)
    logits = synth.logits(w)
    gh.load_inputs(layer, logits)
    layer.run_routing()
    assert layer.error() == ue.UE_OK
    ue.ue_debug_set_lookback_limit(layer.ctx, 1000)
    ue.ue_debug_drop_first_publish(layer.ctx, True)
    layer.reroute()
    assert layer.error() == ue.UE_ERR_TIMEOUT
    ue.ue_debug_drop_first_publish(layer.ctx, False)
    ue.ue_debug_set_lookback_limit(layer.ctx, 1 << 22)
    check_clean_run(layer, logits)


def test_host_rejects_misaligned_and_overlapping_rows(layer):
    base = layer.hidden.view(torch.int16)
    with pytest.raises(ue.UEError):
        ue.ue_permute(layer.ctx, base.data_ptr() + 2, layer.dest_row, layer.dispatch)
    with pytest.raises(ue.UEError):
        ue.ue_permute(layer.ctx, layer.dispatch, layer.dest_row, layer.dispatch)
    with pytest.raises(ue.UEError):
        ue.ue_combine(layer.ctx, layer.dispatch, layer.dest_row, layer.w,
                      layer.out.data_ptr() + 4)
    assert layer.error() == ue.UE_OK


def test_variant_paths_report_bad_ids_and_loads(layer):
    """The planner variants' kernels check their inputs the same way: a
    negative load in the capacity planner, an out-of-range id in the
    interleaved and locality reroutes; the context then runs clean."""
    w = synth.custom(R, T, E, K, S, d, cid=504)
    logits = synth.logits(w)
    gh.load_inputs(layer, logits)
    layer.run_routing()
    assert layer.error() == ue.UE_OK
    bisect = ue.plan_opts(ue.UE_SOLVER_BISECT, min_tokens=4)
    good_load = layer.load_e.clone()
    layer.load_e[9] = -1
    layer.plan_ex(bisect)
    assert layer.error() == ue.UE_ERR_DEVICE_BOUNDS
    layer.load_e.copy_(good_load)
    layer.plan_ex(bisect)
    layer.locality_split()
    assert layer.error() == ue.UE_OK
    layer.idx[11, 2] = E
    layer.reroute_ex(ue.UE_ORDER_INTERLEAVE)
    assert layer.error() == ue.UE_ERR_DEVICE_BOUNDS
    assert int(layer.dest_row[11, 2]) == -1
    layer.reroute_local()
    assert layer.error() == ue.UE_ERR_DEVICE_BOUNDS
    assert int(layer.phys_slot[11, 2]) == -1
    check_clean_run(layer, logits)


def test_variant_calls_reject_bad_arguments(layer):
    with pytest.raises(ue.UEError):
        ue.ue_reroute_ex(layer.ctx, layer.idx, layer.plan, 7, layer.phys_slot, layer.dest_row)
    with pytest.raises(ue.UEError):
        ue.ue_locality_split(layer.ctx, layer.load_re, layer.plan,
                             layer.src_quota.data_ptr() + 2, layer.src_offset)
    with pytest.raises(ue.UEError):
        ue.ue_reroute_local(layer.ctx, layer.idx, layer.load_re, layer.plan, layer.src_quota,
                            layer.src_offset, layer.phys_slot, layer.dest_row.data_ptr() + 1)
    assert layer.error() == ue.UE_OK


def test_overlapped_plan_and_reroute_report_errors_and_recover(layer):
    """ue_plan_reroute (the reroute launched as the plan kernel's dependent):
    a look-back wait that runs out and an id out of range are reported as
    by the separate calls, and the context then runs clean."""
    w = synth.custom(R, T, E, K, S, d, cid=505)
    logits = synth.logits(w)
    gh.load_inputs(layer, logits)
    layer.run_routing()
    assert layer.error() == ue.UE_OK
    ue.ue_debug_set_lookback_limit(layer.ctx, 1000)
    ue.ue_debug_drop_first_publish(layer.ctx, True)
    layer.plan_reroute()
    assert layer.error() == ue.UE_ERR_TIMEOUT
    ue.ue_debug_drop_first_publish(layer.ctx, False)
    ue.ue_debug_set_lookback_limit(layer.ctx, 1 << 22)
    check_clean_run(layer, logits)
    layer.idx[5, 3] = E + 1
    layer.plan_reroute()
    assert layer.error() == ue.UE_ERR_DEVICE_BOUNDS
    assert int(layer.dest_row[5, 3]) == -1 and int(layer.phys_slot[5, 3]) == -1
    check_clean_run(layer, logits)
