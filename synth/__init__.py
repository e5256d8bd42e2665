"""Seeded synthetic inputs for the exact-load rebalancing hot path.

This module only draws random numbers: router logits (fp32 N(0,1) noise plus
a per-expert Zipf log-weight bias in a random expert permutation) and bf16
rows. It holds none of the method's arithmetic (no top-k, histogram, plan or
reroute), so both the CUDA path and the CPU oracle can take their inputs from
it without sharing any computation.

The pages measure on production routing traces and real models ("UltraEP"
README, "Tests": test_solving.py draws Zipf-distributed expert loads at
target rank-level imbalance ratios). None of those traces are available, so
these generators stand in for them, with the same shapes as the workloads
the pages describe (EP64 training layers, EP40 prefill).

Determinism: every tensor is drawn in fixed chunks of ``CHUNK`` elements,
chunk c from its own stream ``SeedSequence([seed, tensor tag..., c])``, so the
result does not depend on the number of threads used to draw it.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

CHUNK = 1 << 22

# Skew constants. They were found by bisection with the CPU oracle
# (tests/golden/tune_skew.py prints them) and are pinned by tests that
# re-measure the skew they produce.
#   ALPHA_QWEN3: scale of the s=1.0 Zipf bias that makes the masters-only
#                max/mean rank load of the Qwen3-shaped layer about 2.5.
#   HOT_BOOST_DSV3: additive logit boosts of the two hotspot experts of the
#                DeepSeek-V3-shaped layer, each drawing 8% of all pairs.
#   HOT_BOOST_30PCT: boost that sends 30% of tokens to one expert in the
#                sweep's single-expert case.
#   ALPHA_PAGES: scales of the s=1.0 Zipf bias that give the EP64, 256-expert
#                layer of the pages' runtime test ("UltraEP" README, "Tests":
#                4 master + 2 redundant experts per rank, top-8, 8k tokens per
#                rank) its three stated initial imbalances, 1.51, 2.01, 3.03.
ALPHA_QWEN3 = 0.1845703125
HOT_BOOST_DSV3 = (4.3984375, 4.91796875)
HOT_BOOST_30PCT = 1.0234375
ALPHA_PAGES = (0.107421875, 0.177734375, 0.2841796875)

_TAG_LOGITS, _TAG_HIDDEN, _TAG_Y, _TAG_PERM, _TAG_PARAMS = 1, 2, 3, 4, 5


@dataclass(frozen=True)
class Workload:
    """One layer instance's sizes and logit recipe."""
    name: str
    cid: int          # numeric id used in the seed
    R: int            # simulated EP ranks
    T: int            # tokens per rank
    E: int            # experts
    K: int            # top-k
    S: int            # redundant slots per rank
    d: int            # hidden size (bf16)
    recipe: str       # "zipf", "hotspots", "per_rank", "sweep"
    zipf_s: float = 1.0
    layers: int = 1
    microbatches: int = 1
    extra: dict = field(default_factory=dict)

    @property
    def N(self):
        return self.R * self.T

    @property
    def M(self):
        return self.E // self.R

    @property
    def Q(self):
        return self.N * self.K

    @property
    def G(self):
        return self.R * self.S

    @property
    def P(self):
        return self.R * (self.M + self.S)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("small_r8_e64", 1, R=8, T=512, E=64, K=4, S=2, d=256,
                 recipe="zipf", zipf_s=1.2),
        Workload("qwen3_layer_r64_e128", 2, R=64, T=4096, E=128, K=8, S=2,
                 d=4096, recipe="zipf", zipf_s=1.0),
        Workload("dsv3_layer_r64_e256", 3, R=64, T=2048, E=256, K=8, S=2,
                 d=7168, recipe="hotspots", zipf_s=1.3),
        Workload("prefill_ep40_e160", 4, R=40, T=8192, E=160, K=8, S=1,
                 d=5120, recipe="per_rank"),
        Workload("sweep_48x8_r64_e128", 5, R=64, T=4096, E=128, K=8, S=2,
                 d=4096, recipe="sweep", layers=48, microbatches=8),
        Workload("pages_ep64_e256_t8k", 6, R=64, T=8192, E=256, K=8, S=2,
                 d=7168, recipe="zipf", zipf_s=1.0),
    ]
}


def _threads():
    return max(1, min(32, os.cpu_count() or 1))


def _stream(seed, *tags):
    return np.random.default_rng([int(seed) & 0xFFFFFFFF] + [int(t) for t in tags])


def normal_f32(count: int, seed: int, *tags) -> np.ndarray:
    """``count`` standard normal fp32 values, drawn chunk by chunk."""
    out = np.empty(count, dtype=np.float32)
    nchunks = (count + CHUNK - 1) // CHUNK

    def job(c):
        lo = c * CHUNK
        hi = min(count, lo + CHUNK)
        out[lo:hi] = _stream(seed, *tags, c).standard_normal(hi - lo,
                                                             dtype=np.float32)

    if nchunks <= 1:
        for c in range(nchunks):
            job(c)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(job, range(nchunks)))
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); finite inputs only."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_normal(rows: int, cols: int, seed: int, *tags) -> np.ndarray:
    """[rows, cols] N(0,1) values rounded to bf16, as uint16 bit patterns."""
    count = rows * cols
    out = np.empty(count, dtype=np.uint16)
    nchunks = (count + CHUNK - 1) // CHUNK

    def job(c):
        lo = c * CHUNK
        hi = min(count, lo + CHUNK)
        x = _stream(seed, *tags, c).standard_normal(hi - lo, dtype=np.float32)
        out[lo:hi] = f32_to_bf16_bits(x)

    if nchunks <= 1:
        for c in range(nchunks):
            job(c)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(job, range(nchunks)))
    return out.reshape(rows, cols)


def zipf_log_weights(E: int, s: float, perm: np.ndarray) -> np.ndarray:
    """Natural log of Zipf weights i^-s, i = 1..E, placed by a permutation:
    expert e gets -s * ln(perm[e] + 1)."""
    return (-s * np.log(perm.astype(np.float64) + 1.0)).astype(np.float64)


def _perm(E, seed, *tags):
    return _stream(seed, _TAG_PERM, *tags).permutation(E)


def logit_bias(w: Workload, layer: int = 0, mb: int = 0, seed: int = 0,
               alpha: float | None = None, boosts=None):
    """Per-token-rank bias [R, E] (fp64) of one layer instance, plus a dict
    describing how it was drawn (permutation, hot experts, per-rank s)."""
    R, E = w.R, w.E
    info = {}
    if w.recipe == "zipf":
        perm = _perm(E, seed, w.cid, layer, mb)
        a = ({"qwen3": ALPHA_QWEN3, "pages": ALPHA_PAGES[1]}.get(w.name.split("_")[0], 1.0)
             if alpha is None else alpha)
        b = a * zipf_log_weights(E, w.zipf_s, perm)
        bias = np.tile(b, (R, 1))
        info.update(perm=perm, alpha=a, s=w.zipf_s)
    elif w.recipe == "hotspots":
        perm = _perm(E, seed, w.cid, layer, mb)
        b = zipf_log_weights(E, w.zipf_s, perm)
        hot = _stream(seed, _TAG_PARAMS, w.cid, layer, mb).choice(E, size=2, replace=False)
        bst = HOT_BOOST_DSV3 if boosts is None else boosts
        b = b.copy()
        b[hot[0]] += bst[0]
        b[hot[1]] += bst[1]
        bias = np.tile(b, (R, 1))
        info.update(perm=perm, hot=hot, boosts=tuple(bst), s=w.zipf_s)
    elif w.recipe == "per_rank":
        perm = _perm(E, seed, w.cid, layer, mb)
        s_r = _stream(seed, _TAG_PARAMS, w.cid, layer, mb).uniform(0.8, 1.5, size=R)
        bias = np.stack([zipf_log_weights(E, s, perm) for s in s_r])
        info.update(perm=perm, s_r=s_r)
    elif w.recipe == "sweep":
        perm = _perm(E, seed, w.cid, layer, mb)
        s = float(_stream(seed, _TAG_PARAMS, w.cid, layer, mb).uniform(0.0, 1.6))
        kind = "zipf"
        if (layer, mb) == (0, 0):
            s, kind = 0.0, "uniform"
        b = zipf_log_weights(E, s, perm)
        if (layer, mb) == (0, 1):
            s, kind = 0.0, "single_expert_30pct"
            b = zipf_log_weights(E, 0.0, perm)
            hot = int(_stream(seed, _TAG_PARAMS, w.cid, layer, mb, 1).integers(E))
            b = b.copy()
            b[hot] += HOT_BOOST_30PCT if boosts is None else boosts[0]
            info.update(hot=np.array([hot]))
        bias = np.tile(b, (R, 1))
        info.update(perm=perm, s=s, kind=kind)
    else:
        raise ValueError(w.recipe)
    return bias, info


def logits(w: Workload, layer: int = 0, mb: int = 0, seed: int = 0,
           alpha: float | None = None, boosts=None, with_info: bool = False):
    """Router logits fp32 [N, E] = N(0,1) noise + the instance's bias."""
    bias, info = logit_bias(w, layer, mb, seed, alpha, boosts)
    noise = normal_f32(w.N * w.E, seed, _TAG_LOGITS, w.cid, layer, mb).reshape(w.N, w.E)
    # add the bias rank by rank: tokens r*T .. (r+1)*T-1 come from rank r
    out = noise.reshape(w.R, w.T, w.E)
    out += bias.astype(np.float32)[:, None, :]
    res = out.reshape(w.N, w.E)
    return (res, info) if with_info else res


def hidden(w: Workload, seed: int = 0) -> np.ndarray:
    """Token hidden states bf16 [N, d] ~ N(0,1), uint16 bit patterns. One
    tensor per workload (shared by every layer instance of a sweep)."""
    return bf16_normal(w.N, w.d, seed, _TAG_HIDDEN, w.cid)


def expert_outputs(w: Workload, seed: int = 0) -> np.ndarray:
    """Independent bf16 [Q, d] ~ N(0,1) rows that stand in for expert outputs
    in dispatch order (so a mis-mapped row cannot cancel out)."""
    return bf16_normal(w.Q, w.d, seed, _TAG_Y, w.cid)


def expert_output_rows(w: Workload, seed: int = 0) -> np.ndarray:
    """Seeded source rows sigma [Q] int64 in [0, N) for a cheaper stand-in for
    expert outputs at full size: y[r] = hidden[sigma[r]]. Each dispatch row
    gets its own randomly chosen N(0,1) bf16 row, independent of the routing,
    so a row read from the wrong place differs from the right one unless two
    draws coincide (probability 1/N per pair of rows)."""
    return _stream(seed, _TAG_Y, w.cid, 1).integers(0, w.N, size=w.Q, dtype=np.int64)


def custom(R, T, E, K, S, d, name="custom", cid=99, recipe="zipf", zipf_s=1.2):
    """A workload of arbitrary sizes (tests: ragged and edge cases)."""
    return Workload(name, cid, R=R, T=T, E=E, K=K, S=S, d=d, recipe=recipe,
                    zipf_s=zipf_s)


def describe(w: Workload) -> str:
    return (f"{w.name}: R={w.R} T={w.T} N={w.N} E={w.E} M={w.M} K={w.K} "
            f"S={w.S} d={w.d} Q={w.Q} recipe={w.recipe}")


__all__ = ["Workload", "WORKLOADS", "logits", "hidden", "expert_outputs", "expert_output_rows",
           "bf16_normal", "normal_f32", "f32_to_bf16_bits", "bf16_bits_to_f32",
           "logit_bias", "custom", "describe"]
