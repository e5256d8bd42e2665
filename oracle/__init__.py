"""CPU oracle for the exact-load expert rebalancing hot path (UltraEP).

TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import this package. The product path (the
CUDA library and its binding) never imports, links or calls it, and the two
share no code: they meet only at the seeded input generator in ``synth``.

The arithmetic lives in ``oracle.c`` (plain C, single-threaded, fp64 for the
gate weights and the combine). This module only builds it with gcc and
marshals numpy arrays through ctypes. Every function cites the page section
it follows in ``oracle.c``.

Each function is pinned by tests that do not re-use it: brute force on tiny
inputs, closed forms, hand-worked plans (``tests/golden``), and invariants
that determine the result.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (no FMA contraction)."""
    if force or not os.path.exists(_LIB) or (
        os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fPIC", "-shared",
             "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _bind(lib):
    i32, i64 = ctypes.c_int32, ctypes.c_int64
    p = ctypes.c_void_p
    lib.or_gate_topk.argtypes = [p, i64, i32, i32, p, p]
    lib.or_count.argtypes = [p, i32, i32, i32, i32, p, p]
    lib.or_plan.argtypes = [i32, i32, i32, p, i32, p, p, p, p, p, p, p, p]
    lib.or_plan_bisect.argtypes = [i32, i32, i32, p, i32, i32, i32, i32, p, p, p, p, p, p]
    lib.or_reroute.argtypes = [p, i64, i32, i32, i32, p, p, p, p, p]
    lib.or_reroute_interleave.argtypes = [p, i32, i32, i32, i32, i32, p, p, p, p, p]
    lib.or_locality_split.argtypes = [i32, i32, i32, p, p, p, p, p, p]
    lib.or_reroute_local.argtypes = [p, i32, i32, i32, i32, i32, p, p, p, p, p]
    lib.or_permute.argtypes = [p, i64, i32, i32, p, p]
    lib.or_permute_rows.argtypes = [p, i64, i32, i32, p, p, i64, p]
    lib.or_combine.argtypes = [p, i64, i32, i32, p, p, p, i64, p]
    lib.or_combine_backward.argtypes = [p, p, i64, i32, i32, p, p, p, i64, p, p]
    lib.or_permute_backward.argtypes = [p, i64, i32, i32, p, p, i64, p]
    lib.or_weight_sync.argtypes = [i32, p, i32, p, p, i64]
    lib.or_grad_reduce.argtypes = [i32, p, i32, p, p, i64, p]
    for f in ("or_gate_topk", "or_count", "or_plan", "or_plan_bisect", "or_reroute",
              "or_reroute_interleave", "or_locality_split", "or_reroute_local",
              "or_permute", "or_permute_rows", "or_combine", "or_combine_backward",
              "or_permute_backward", "or_weight_sync", "or_grad_reduce"):
        getattr(lib, f).restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(_LIB))
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its input (code {rc})")


def gate_topk(logits: np.ndarray, K: int):
    """Top-K expert ids per row (descending logit, ties to the lower id) and
    the fp64 softmax over the selected logits. logits: float32 [N, E]."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    N, E = logits.shape
    idx = np.empty((N, K), dtype=np.int32)
    w = np.empty((N, K), dtype=np.float64)
    _check(_load().or_gate_topk(_ptr(logits), N, E, K, _ptr(idx), _ptr(w)),
           "gate_topk")
    return idx, w


def count(idx: np.ndarray, R: int, T: int, E: int):
    """Per-source-rank [R, E] and per-expert [E] pair counts."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    K = idx.shape[1]
    load_re = np.empty((R, E), dtype=np.int32)
    load_e = np.empty(E, dtype=np.int32)
    _check(_load().or_count(_ptr(idx), R, T, E, K, _ptr(load_re),
                            _ptr(load_e)), "count")
    return load_re, load_e


@dataclass
class Plan:
    slot_expert: np.ndarray  # [G] int32, -1 = empty
    n_copies: np.ndarray     # [E]
    slot_quota: np.ndarray   # [P]
    slot_offset: np.ndarray  # [P+1]
    rank_load: np.ndarray    # [R]
    stats: np.ndarray        # [4] iterations, max before, max after, co-located
    trace_e: np.ndarray      # [iterations] chosen expert per iteration
    trace_r: np.ndarray      # [iterations] chosen rank per iteration


def plan(load_e: np.ndarray, R: int, S: int, min_tokens: int = 0) -> Plan:
    """Greedy quota-driven replication plan from the exact per-expert load
    (min_tokens > 0: an expert takes another copy only if each of its copies
    keeps at least min_tokens pairs)."""
    load_e = np.ascontiguousarray(load_e, dtype=np.int32)
    E = load_e.shape[0]
    M = E // R
    G, P = R * S, R * (M + S)
    slot_expert = np.empty(max(G, 1), dtype=np.int32)
    n_copies = np.empty(E, dtype=np.int32)
    slot_quota = np.empty(P, dtype=np.int32)
    slot_offset = np.empty(P + 1, dtype=np.int32)
    rank_load = np.empty(R, dtype=np.int32)
    stats = np.empty(4, dtype=np.int32)
    te = np.full(max(G, 1), -1, dtype=np.int32)
    tr = np.full(max(G, 1), -1, dtype=np.int32)
    _check(_load().or_plan(R, E, S, _ptr(load_e), min_tokens, _ptr(slot_expert),
                           _ptr(n_copies), _ptr(slot_quota), _ptr(slot_offset),
                           _ptr(rank_load), _ptr(stats), _ptr(te), _ptr(tr)),
           "plan")
    it = int(stats[0])
    return Plan(slot_expert[:G].copy(), n_copies, slot_quota, slot_offset,
                rank_load, stats, te[:it].copy(), tr[:it].copy())


def plan_bisect(load_e: np.ndarray, R: int, S: int, eps_inv: int = 100,
                threshold: int | None = None, min_tokens: int = 1024,
                allow_zero_master: bool = False) -> Plan:
    """Capacity planner: bisection on max/mean over the grid k/eps_inv with a
    quota oracle per probe. threshold is the early-stop ratio in units of
    1/eps_inv (default eps_inv, i.e. 1.0). stats = {probes, max before, max
    after, final k}; trace_e / trace_r are empty."""
    load_e = np.ascontiguousarray(load_e, dtype=np.int32)
    E = load_e.shape[0]
    M = E // R
    G, P = R * S, R * (M + S)
    thr = eps_inv if threshold is None else threshold
    slot_expert = np.empty(max(G, 1), dtype=np.int32)
    n_copies = np.empty(E, dtype=np.int32)
    slot_quota = np.empty(P, dtype=np.int32)
    slot_offset = np.empty(P + 1, dtype=np.int32)
    rank_load = np.empty(R, dtype=np.int32)
    stats = np.empty(4, dtype=np.int32)
    _check(_load().or_plan_bisect(R, E, S, _ptr(load_e), eps_inv, thr, min_tokens,
                                  int(bool(allow_zero_master)), _ptr(slot_expert),
                                  _ptr(n_copies), _ptr(slot_quota), _ptr(slot_offset),
                                  _ptr(rank_load), _ptr(stats)), "plan_bisect")
    empty = np.empty(0, dtype=np.int32)
    return Plan(slot_expert[:G].copy(), n_copies, slot_quota, slot_offset, rank_load,
                stats, empty, empty)


def _slot_expert_arg(pl: Plan):
    se = np.ascontiguousarray(pl.slot_expert, dtype=np.int32)
    return se if se.size else np.full(1, -1, dtype=np.int32)


def reroute_interleave(idx: np.ndarray, R: int, T: int, E: int, S: int, pl: Plan):
    """Prefix-fill reroute with the pairs taken in (token, rank, k) order."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    K = idx.size // (R * T) if R * T else 1
    phys = np.empty(idx.shape, dtype=np.int32)
    dest = np.empty(idx.shape, dtype=np.int32)
    _check(_load().or_reroute_interleave(_ptr(idx), R, T, K, E, S, _ptr(_slot_expert_arg(pl)),
                                         _ptr(np.ascontiguousarray(pl.slot_quota)),
                                         _ptr(np.ascontiguousarray(pl.slot_offset)),
                                         _ptr(phys), _ptr(dest)), "reroute_interleave")
    return phys, dest


def locality_split(load_re: np.ndarray, S: int, pl: Plan):
    """Per-source-rank split of every copy's quota, own rank first:
    (src_quota [R][P], src_offset [R][P])."""
    load_re = np.ascontiguousarray(load_re, dtype=np.int32)
    R, E = load_re.shape
    P = pl.slot_quota.size
    src_quota = np.empty((R, P), dtype=np.int32)
    src_offset = np.empty((R, P), dtype=np.int32)
    _check(_load().or_locality_split(R, E, S, _ptr(load_re), _ptr(_slot_expert_arg(pl)),
                                     _ptr(np.ascontiguousarray(pl.slot_quota)),
                                     _ptr(np.ascontiguousarray(pl.slot_offset)),
                                     _ptr(src_quota), _ptr(src_offset)), "locality_split")
    return src_quota, src_offset


def reroute_local(idx: np.ndarray, R: int, T: int, E: int, S: int, pl: Plan,
                  src_quota: np.ndarray, src_offset: np.ndarray):
    """Reroute under the locality-aware split."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    K = idx.size // (R * T) if R * T else 1
    phys = np.empty(idx.shape, dtype=np.int32)
    dest = np.empty(idx.shape, dtype=np.int32)
    _check(_load().or_reroute_local(_ptr(idx), R, T, K, E, S, _ptr(_slot_expert_arg(pl)),
                                    _ptr(np.ascontiguousarray(src_quota, dtype=np.int32)),
                                    _ptr(np.ascontiguousarray(src_offset, dtype=np.int32)),
                                    _ptr(phys), _ptr(dest)), "reroute_local")
    return phys, dest


def reroute(idx: np.ndarray, R: int, E: int, S: int, pl: Plan):
    """Physical slot and dispatch row of every pair (global order)."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    Q = idx.size
    phys = np.empty(idx.shape, dtype=np.int32)
    dest = np.empty(idx.shape, dtype=np.int32)
    se = np.ascontiguousarray(pl.slot_expert, dtype=np.int32)
    if se.size == 0:
        se = np.full(1, -1, dtype=np.int32)
    _check(_load().or_reroute(_ptr(idx), Q, R, E, S, _ptr(se),
                              _ptr(np.ascontiguousarray(pl.slot_quota)),
                              _ptr(np.ascontiguousarray(pl.slot_offset)),
                              _ptr(phys), _ptr(dest)), "reroute")
    return phys, dest


def permute(hidden_u16: np.ndarray, K: int, dest_row: np.ndarray):
    """dispatch[dest_row[n, k]] = hidden[n]; rows are bf16 bit patterns."""
    hidden_u16 = np.ascontiguousarray(hidden_u16, dtype=np.uint16)
    N, d = hidden_u16.shape
    dest_row = np.ascontiguousarray(dest_row, dtype=np.int32)
    out = np.empty((N * K, d), dtype=np.uint16)
    _check(_load().or_permute(_ptr(hidden_u16), N, d, K, _ptr(dest_row),
                              _ptr(out)), "permute")
    return out


def permute_rows(hidden_u16: np.ndarray, K: int, dest_row: np.ndarray,
                 rows: np.ndarray, out: np.ndarray | None = None):
    """The permute's result at the given dispatch rows only (written into
    ``out`` if given: a C-contiguous uint16 [len(rows), d] array)."""
    hidden_u16 = np.ascontiguousarray(hidden_u16, dtype=np.uint16)
    N, d = hidden_u16.shape
    dest_row = np.ascontiguousarray(dest_row, dtype=np.int32)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    if out is None:
        out = np.empty((rows.size, d), dtype=np.uint16)
    assert out.dtype == np.uint16 and out.shape == (rows.size, d)
    _check(_load().or_permute_rows(_ptr(hidden_u16), N, d, K, _ptr(dest_row),
                                   _ptr(rows), rows.size, _ptr(out)),
           "permute_rows")
    return out


def combine(y_u16: np.ndarray, N: int, K: int, dest_row: np.ndarray,
            w: np.ndarray, tokens: np.ndarray | None = None,
            out: np.ndarray | None = None):
    """fp64 out[n] = sum_k w[n, k] * y[dest_row[n, k]] (all tokens, or the
    listed ones; written into ``out`` if given: a C-contiguous float64 array
    with one row per evaluated token)."""
    y_u16 = np.ascontiguousarray(y_u16, dtype=np.uint16)
    d = y_u16.shape[1]
    dest_row = np.ascontiguousarray(dest_row, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    if tokens is not None:
        tokens = np.ascontiguousarray(tokens, dtype=np.int64)
        nt = tokens.size
    else:
        nt = 0
    rows_out = tokens.size if tokens is not None else N
    if out is None:
        out = np.empty((rows_out, d), dtype=np.float64)
    assert out.dtype == np.float64 and out.shape == (rows_out, d) and out.flags["C_CONTIGUOUS"]
    _check(_load().or_combine(_ptr(y_u16), N, d, K, _ptr(dest_row), _ptr(w),
                              _ptr(tokens), nt, _ptr(out)), "combine")
    return out


def combine_backward(dout: np.ndarray, y_u16: np.ndarray, K: int, dest_row: np.ndarray,
                     w: np.ndarray, tokens: np.ndarray | None = None):
    """fp64 (dy rows per (token, k), dw [tokens][K]) of the combine's backward.
    dout fp32 [N][d], y bf16 [Q][d], w fp32 [N][K]."""
    dout = np.ascontiguousarray(dout, dtype=np.float32)
    N, d = dout.shape
    y_u16 = np.ascontiguousarray(y_u16, dtype=np.uint16)
    dest_row = np.ascontiguousarray(dest_row, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    if tokens is not None:
        tokens = np.ascontiguousarray(tokens, dtype=np.int64)
        cnt = tokens.size
    else:
        cnt = N
    dy = np.empty((cnt * K, d), dtype=np.float64)
    dw = np.empty((cnt, K), dtype=np.float64)
    _check(_load().or_combine_backward(_ptr(dout), _ptr(y_u16), N, d, K, _ptr(dest_row),
                                       _ptr(w), _ptr(tokens), cnt if tokens is not None else 0,
                                       _ptr(dy), _ptr(dw)), "combine_backward")
    return dy, dw


def permute_backward(ddispatch_u16: np.ndarray, N: int, K: int, dest_row: np.ndarray,
                     tokens: np.ndarray | None = None):
    """fp64 dhidden[n] = sum_k ddispatch[dest_row[n, k]] (all or listed tokens)."""
    ddispatch_u16 = np.ascontiguousarray(ddispatch_u16, dtype=np.uint16)
    d = ddispatch_u16.shape[1]
    dest_row = np.ascontiguousarray(dest_row, dtype=np.int32)
    if tokens is not None:
        tokens = np.ascontiguousarray(tokens, dtype=np.int64)
        cnt = tokens.size
    else:
        cnt = N
    out = np.empty((cnt, d), dtype=np.float64)
    _check(_load().or_permute_backward(_ptr(ddispatch_u16), N, d, K, _ptr(dest_row),
                                       _ptr(tokens), cnt if tokens is not None else 0,
                                       _ptr(out)), "permute_backward")
    return out


def weight_sync(slot_expert: np.ndarray, master: np.ndarray, replicas: np.ndarray):
    """replicas[g] = master[slot_expert[g]] for every used slot (in place on a
    copy of `replicas`); rows are raw bytes [E][B] and [G][B]."""
    master = np.ascontiguousarray(master, dtype=np.uint8)
    out = np.array(replicas, dtype=np.uint8, copy=True, order="C")
    se = np.ascontiguousarray(slot_expert, dtype=np.int32)
    G = se.size
    E, B = master.shape
    _check(_load().or_weight_sync(G, _ptr(se) if G else None, E, _ptr(master),
                                  _ptr(out) if G else None, B), "weight_sync")
    return out


def grad_reduce(slot_expert: np.ndarray, replicas: np.ndarray, master: np.ndarray):
    """fp64 master[e] + sum of e's replica gradients (ascending slot)."""
    master = np.ascontiguousarray(master, dtype=np.float32)
    E, W = master.shape
    se = np.ascontiguousarray(slot_expert, dtype=np.int32)
    G = se.size
    replicas = np.ascontiguousarray(replicas, dtype=np.float32)
    out = np.empty((E, W), dtype=np.float64)
    _check(_load().or_grad_reduce(G, _ptr(se) if G else None, E,
                                  _ptr(replicas) if G else None, _ptr(master), W, _ptr(out)),
           "grad_reduce")
    return out


def run_path(logits: np.ndarray, R: int, T: int, S: int, K: int):
    """Integer part of the path end to end: top-k, counts, plan, reroute."""
    E = logits.shape[1]
    idx, w = gate_topk(logits, K)
    load_re, load_e = count(idx, R, T, E)
    pl = plan(load_e, R, S)
    phys, dest = reroute(idx, R, E, S, pl)
    return dict(idx=idx, w=w, load_re=load_re, load_e=load_e, plan=pl,
                phys_slot=phys, dest_row=dest)
