"""One layer instance of the rebalancing hot path: device buffers (PyTorch
tensors) plus the C-ABI calls in order. Plumbing only: the work is done by
the kernels behind each ``ue_*`` call.

Step order ("UltraEP" README, "Interface / 2. Forward and backward"):
router top-k -> exact load -> update_placement (plan) -> reroute ->
dispatch (permute) -> experts (outside; identity here unless ``y`` is given)
-> combine.
"""
from __future__ import annotations

from . import (make_config, placement, ue_combine, ue_count, ue_destroy, ue_gate_count,
               ue_gate_topk,
               ue_get_error, ue_init, ue_locality_split, ue_permute, ue_plan, ue_plan_ex,
               ue_plan_reroute, ue_reroute, ue_reroute_ex, ue_reroute_local)


class Layer:
    """Buffers for sizes (R, T, E, K, S, d) on one CUDA device."""

    def __init__(self, R, T, E, K, S, d, device: int = 0, with_rows: bool = True):
        import torch

        self.R, self.T, self.E, self.K, self.S, self.d = R, T, E, K, S, d
        self.M = E // R
        self.N = R * T
        self.Q = self.N * K
        self.G = R * S
        self.P = R * (self.M + S)
        self.device = torch.device("cuda", device)
        self.cfg = make_config(R, T, E, K, S, d)
        self.ctx = ue_init(self.cfg, device)
        dev, i32 = self.device, torch.int32
        self.logits = torch.empty((self.N, E), dtype=torch.float32, device=dev)
        self.idx = torch.empty((self.N, K), dtype=i32, device=dev)
        self.w = torch.empty((self.N, K), dtype=torch.float32, device=dev)
        self.load_re = torch.empty((R, E), dtype=i32, device=dev)
        self.load_e = torch.empty(E, dtype=i32, device=dev)
        self.slot_expert = torch.empty(max(self.G, 1), dtype=i32, device=dev)
        self.n_copies = torch.empty(E, dtype=i32, device=dev)
        self.slot_quota = torch.empty(self.P, dtype=i32, device=dev)
        self.slot_offset = torch.empty(self.P + 1, dtype=i32, device=dev)
        self.rank_load = torch.empty(R, dtype=i32, device=dev)
        self.stats = torch.empty(4, dtype=i32, device=dev)
        self.plan = placement(self.slot_expert if self.G > 0 else None, self.n_copies,
                              self.slot_quota, self.slot_offset, self.rank_load, self.stats)
        self.phys_slot = torch.empty((self.N, K), dtype=i32, device=dev)
        self.dest_row = torch.empty((self.N, K), dtype=i32, device=dev)
        # locality-aware split of the quotas over the source ranks
        self.src_quota = torch.empty((R, self.P), dtype=i32, device=dev)
        self.src_offset = torch.empty((R, self.P), dtype=i32, device=dev)
        self.with_rows = with_rows
        if with_rows:
            self.hidden = torch.empty((self.N, d), dtype=torch.bfloat16, device=dev)
            self.dispatch = torch.empty((self.Q, d), dtype=torch.bfloat16, device=dev)
            self.out = torch.empty((self.N, d), dtype=torch.float32, device=dev)

    # -- the steps ---------------------------------------------------------
    def gate(self, stream=None):
        ue_gate_topk(self.ctx, self.logits, self.idx, self.w, stream)

    def count(self, stream=None):
        ue_count(self.ctx, self.idx, self.load_re, self.load_e, stream)

    def gate_count(self, stream=None):
        """Top-k, weights and the exact histogram in one call."""
        ue_gate_count(self.ctx, self.logits, self.idx, self.w, self.load_re, self.load_e, stream)

    def plan_step(self, stream=None):
        ue_plan(self.ctx, self.load_e, self.plan, stream)

    def reroute(self, stream=None):
        ue_reroute(self.ctx, self.idx, self.plan, self.phys_slot, self.dest_row, stream)

    def plan_reroute(self, stream=None):
        """Plan then reroute in one call, the reroute's plan-free part
        overlapping the plan kernel (ue_plan_reroute)."""
        ue_plan_reroute(self.ctx, self.load_e, self.idx, self.plan, self.phys_slot,
                        self.dest_row, stream)

    # -- planner variants ("Performance Tuning / Replication planning") -----
    def plan_ex(self, opts, stream=None):
        """ue_plan_ex with a ue_plan_opts (see token_rerouting_b200.plan_opts)."""
        ue_plan_ex(self.ctx, self.load_e, opts, self.plan, stream)

    def reroute_ex(self, order, stream=None):
        ue_reroute_ex(self.ctx, self.idx, self.plan, order, self.phys_slot, self.dest_row, stream)

    def locality_split(self, stream=None):
        ue_locality_split(self.ctx, self.load_re, self.plan, self.src_quota, self.src_offset,
                          stream)

    def reroute_local(self, stream=None):
        ue_reroute_local(self.ctx, self.idx, self.load_re, self.plan, self.src_quota,
                         self.src_offset, self.phys_slot, self.dest_row, stream)

    def permute(self, stream=None):
        ue_permute(self.ctx, self.hidden, self.dest_row, self.dispatch, stream)

    def combine(self, y=None, stream=None):
        ue_combine(self.ctx, self.dispatch if y is None else y, self.dest_row, self.w,
                   self.out, stream)

    def run_routing(self, stream=None, fused=True, overlap=True):
        """gate -> count -> plan -> reroute; with fused=True the gate and the
        count are one call (ue_gate_count), with overlap=True the plan and
        the reroute are one call (ue_plan_reroute)."""
        if fused:
            self.gate_count(stream)
        else:
            self.gate(stream)
            self.count(stream)
        if overlap:
            self.plan_reroute(stream)
        else:
            self.plan_step(stream)
            self.reroute(stream)

    def run(self, y=None, stream=None):
        """The whole path: gate -> count -> plan -> reroute -> permute ->
        combine (identity experts unless ``y`` is given)."""
        self.run_routing(stream)
        self.permute(stream)
        self.combine(y, stream)

    def error(self, stream=None) -> int:
        return ue_get_error(self.ctx, stream)

    def close(self):
        if self.ctx is not None:
            ue_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def plan_arrays(self):
        """Host copies of the plan (for checks and reports)."""
        return dict(slot_expert=self.slot_expert[: self.G].cpu().numpy(),
                    n_copies=self.n_copies.cpu().numpy(),
                    slot_quota=self.slot_quota.cpu().numpy(),
                    slot_offset=self.slot_offset.cpu().numpy(),
                    rank_load=self.rank_load.cpu().numpy(),
                    stats=self.stats.cpu().numpy())


__all__ = ["Layer"]
