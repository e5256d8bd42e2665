"""GPU parity of the weight sync and the gradient reduction.

* Weight sync: bytes, bit-exact: every used slot receives its expert's
  master bytes, empty slots keep their contents (against the oracle at small
  size; at the Qwen3-235B expert size, 2*h*f + h*f bf16 weights per expert
  with h = 4096 and f = 1536, every slot is checked on the device).
* Gradient reduction: against the fp64 oracle within c 2^-24 sum |terms|
  (c = the expert's replica count, one fp32 rounding per addition); the same
  bits on a second run; and at full expert size bit-exact against a plain
  fp32 PyTorch reference that adds the replicas in ascending slot order;
  hand placements (no replica at all, more replicas than experts, an id out
  of range) bit-exact against the same ordered fp32 sum.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import token_rerouting_b200 as ue
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

H, F = 4096, 1536
NUMEL = 2 * H * F + H * F  # fc1 (2*h*f) + fc2 (h*f)


def plan_for(w, seed=0):
    """An oracle plan for a workload's logits (the slot -> expert map)."""
    o = oracle.run_path(synth.logits(w, 0, seed), w.R, w.T, w.S, w.K)
    return o["plan"]


def placement_from(pl, G, E, dev):
    """A ue_placement over device copies of the plan's slot_expert. The
    struct holds raw pointers: the caller keeps the returned tensor alive."""
    se = torch.from_numpy(np.ascontiguousarray(pl.slot_expert if G else np.full(1, -1),
                                               dtype=np.int32)).to(dev)
    dummy = torch.zeros(max(E, 4), dtype=torch.int32, device=dev)
    return ue.placement(se if G else None, dummy, dummy, dummy, dummy, dummy), se


@pytest.mark.parametrize("name,bpe", [("small_r8_e64", 4096 + 48), ("small_r8_e64", 16)])
def test_weight_sync_small(name, bpe):
    w = synth.WORKLOADS[name]
    pl = plan_for(w)
    L = gh.make_layer(w.R, w.T, w.E, w.K, w.S, w.d, with_rows=False)
    dev = L.device
    try:
        rng = np.random.default_rng(3)
        master = rng.integers(0, 256, size=(w.E, bpe), dtype=np.uint8)
        before = rng.integers(0, 256, size=(w.G, bpe), dtype=np.uint8)
        plc, se_keep = placement_from(pl, w.G, w.E, dev)  # keep the buffer alive
        m_t = torch.from_numpy(master).to(dev)
        r_t = torch.from_numpy(before).to(dev)
        ue.ue_weight_sync(L.ctx, plc, m_t, r_t, bpe)
        assert L.error() == 0
        np.testing.assert_array_equal(r_t.cpu().numpy(), oracle.weight_sync(pl.slot_expert, master, before))
    finally:
        L.close()


def test_weight_sync_qwen3_expert_size():
    w = synth.WORKLOADS["qwen3_layer_r64_e128"]
    pl = plan_for(w)
    L = gh.make_layer(w.R, w.T, w.E, w.K, w.S, 8, with_rows=False)
    dev = L.device
    try:
        bpe = NUMEL * 2
        g = torch.Generator(device=dev).manual_seed(5)
        master = torch.randint(-30000, 30000, (w.E, NUMEL), dtype=torch.int16, device=dev, generator=g)
        reps = torch.full((w.G, NUMEL), 7, dtype=torch.int16, device=dev)
        plc, se_keep = placement_from(pl, w.G, w.E, dev)  # keep the buffer alive
        ue.ue_weight_sync(L.ctx, plc, master, reps, bpe)
        assert L.error() == 0
        for gg in range(w.G):
            e = int(pl.slot_expert[gg])
            if e >= 0:
                assert torch.equal(reps[gg], master[e]), gg
            else:
                assert bool((reps[gg] == 7).all()), gg
    finally:
        L.close()


@pytest.mark.parametrize("name,numel", [("small_r8_e64", 1028), ("small_r8_e64", 4)])
def test_grad_reduce_small(name, numel):
    w = synth.WORKLOADS[name]
    pl = plan_for(w)
    L = gh.make_layer(w.R, w.T, w.E, w.K, w.S, w.d, with_rows=False)
    dev = L.device
    try:
        master = synth.normal_f32(w.E * numel, 0, 51).reshape(w.E, numel)
        reps = synth.normal_f32(w.G * numel, 0, 52).reshape(w.G, numel)
        plc, se_keep = placement_from(pl, w.G, w.E, dev)  # keep the buffer alive
        outs = []
        for _ in range(2):
            m_t = torch.from_numpy(master).to(dev)
            ue.ue_grad_reduce(L.ctx, plc, torch.from_numpy(reps).to(dev), m_t, numel)
            assert L.error() == 0
            outs.append(m_t.cpu().numpy())
        np.testing.assert_array_equal(outs[0], outs[1])  # deterministic
        ref = oracle.grad_reduce(pl.slot_expert, reps, master)
        cnt = np.bincount(pl.slot_expert[pl.slot_expert >= 0], minlength=w.E)
        scale = np.abs(master).astype(np.float64)
        for gg, e in enumerate(pl.slot_expert):
            if e >= 0:
                scale[e] += np.abs(reps[gg])
        err = np.abs(outs[0].astype(np.float64) - ref)
        assert (err <= cnt[:, None] * 2.0 ** -24 * scale + 1e-30).all()
        # experts without replicas are untouched
        np.testing.assert_array_equal(outs[0][cnt == 0], master[cnt == 0])
    finally:
        L.close()


def test_grad_reduce_qwen3_expert_size_matches_ordered_fp32():
    w = synth.WORKLOADS["qwen3_layer_r64_e128"]
    pl = plan_for(w)
    L = gh.make_layer(w.R, w.T, w.E, w.K, w.S, 8, with_rows=False)
    dev = L.device
    try:
        g = torch.Generator(device=dev).manual_seed(9)
        master = torch.randn((w.E, NUMEL), dtype=torch.float32, device=dev, generator=g)
        reps = torch.randn((w.G, NUMEL), dtype=torch.float32, device=dev, generator=g)
        ref = master.clone()
        for gg in range(w.G):  # ascending slot order, plain fp32 additions
            e = int(pl.slot_expert[gg])
            if e >= 0:
                ref[e] = ref[e] + reps[gg]
        plc, se_keep = placement_from(pl, w.G, w.E, dev)  # keep the buffer alive
        ue.ue_grad_reduce(L.ctx, plc, reps, master, NUMEL)
        assert L.error() == 0
        assert torch.equal(master, ref)
    finally:
        L.close()


@pytest.mark.parametrize("se_list", [
    [-1] * 16,                                            # no replica anywhere
    [3, 3, 3, 3, 0, 1, -1, 3, 2, 2, 5, 3, -1, 7, 7, 3],   # G = 16 > E = 8, expert 3 seven times
    [6, -1, 6, 9, 1, -1, -1, -1, -1, -1, -1, -1, 1, -1, 6, -1],  # an id out of range (9 >= E)
])
def test_grad_reduce_hand_placements(se_list):
    """Hand placements: the reduction's list of replicated experts may be
    empty, longer than E replicas for one expert, or hold an id out of range
    (that slot is skipped and UE_ERR_DEVICE_BOUNDS set). The result is the
    master plus the replicas added in ascending g in fp32, bit for bit; 1100
    float4 per expert make a ragged last piece."""
    R, T, E, K, S, d = 8, 4, 8, 2, 2, 8
    G = R * S
    numel = 4 * 1100
    L = gh.make_layer(R, T, E, K, S, d, with_rows=False)
    dev = L.device
    try:
        se = torch.tensor(se_list, dtype=torch.int32, device=dev)
        dummy = torch.zeros(max(E, 4), dtype=torch.int32, device=dev)
        plc = ue.placement(se, dummy, dummy, dummy, dummy, dummy)
        master = torch.from_numpy(synth.normal_f32(E * numel, 1, 53).reshape(E, numel))
        reps = torch.from_numpy(synth.normal_f32(G * numel, 1, 54).reshape(G, numel))
        m_t = master.to(dev)
        ue.ue_grad_reduce(L.ctx, plc, reps.to(dev), m_t, numel)
        bad = any(e >= E for e in se_list)
        assert L.error() == (ue.UE_ERR_DEVICE_BOUNDS if bad else ue.UE_OK)
        ref = master.clone()
        for g, e in enumerate(se_list):
            if 0 <= e < E:
                ref[e] = ref[e] + reps[g]
        np.testing.assert_array_equal(m_t.cpu().numpy().view(np.uint32), ref.numpy().view(np.uint32))
    finally:
        L.close()
