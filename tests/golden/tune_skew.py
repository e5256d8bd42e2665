"""Find the skew constants of the synthetic workloads with the CPU oracle.

Prints ALPHA_QWEN3, HOT_BOOST_DSV3, HOT_BOOST_30PCT and ALPHA_PAGES for
``synth``. The
values are found by bisection on the oracle's exact histogram:

* Qwen3-shaped layer: scale of the s=1.0 Zipf bias so that the masters-only
  max/mean rank load is 2.5 (the workload's stated pre-balance skew).
* DeepSeek-V3-shaped layer: additive boosts of the two hotspot experts so
  that each draws 8% of all pairs.
* Sweep single-expert case: boost so that 30% of tokens route to one expert.
* The pages' runtime-test layer (EP64, 256 experts): scales of the s=1.0
  Zipf bias for masters-only max/mean 1.51, 2.01 and 3.03.

Only the oracle and the input generator are used. Run:
    python tests/golden/tune_skew.py
"""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.abspath(os.path.join(os.path.dirname(__file__), "..", "..")))

import oracle  # noqa: E402
import synth  # noqa: E402


def masters_max_over_mean(w, load_e):
    rank = load_e.reshape(w.R, w.M).sum(axis=1)
    return rank.max() / (w.Q / w.R)


def loads(w, **kw):
    lg = synth.logits(w, **kw)
    idx, _ = oracle.gate_topk(lg, w.K)
    _, load_e = oracle.count(idx, w.R, w.T, w.E)
    return load_e


def bisect(f, lo, hi, target, tol, iters=40):
    flo = f(lo)
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        fm = f(mid)
        if abs(fm - target) <= tol:
            return mid, fm
        if (fm < target) == (flo < target):
            lo, flo = mid, fm
        else:
            hi = mid
    return mid, fm


def tune_qwen3():
    w = synth.WORKLOADS["qwen3_layer_r64_e128"]
    f = lambda a: masters_max_over_mean(w, loads(w, alpha=a))
    a, v = bisect(f, 0.0, 4.0, 2.5, 0.005)
    print(f"ALPHA_QWEN3 = {a!r}  # masters-only max/mean {v:.4f}")
    return a


def tune_dsv3():
    w = synth.WORKLOADS["dsv3_layer_r64_e256"]
    _, info = synth.logit_bias(w, boosts=(0.0, 0.0))
    hot = info["hot"]
    b = [2.0, 2.0]
    for _ in range(6):
        for h in range(2):
            def share(x, h=h):
                bb = list(b)
                bb[h] = x
                le = loads(w, boosts=tuple(bb))
                return le[hot[h]] / w.Q
            b[h], v = bisect(share, -2.0, 12.0, 0.08, 0.0005)
        le = loads(w, boosts=tuple(b))
        s0, s1 = le[hot[0]] / w.Q, le[hot[1]] / w.Q
        if abs(s0 - 0.08) <= 0.001 and abs(s1 - 0.08) <= 0.001:
            break
    print(f"HOT_BOOST_DSV3 = ({b[0]!r}, {b[1]!r})  # shares {s0:.4f} {s1:.4f}")
    return b


def tune_30pct():
    w = synth.WORKLOADS["sweep_48x8_r64_e128"]
    _, info = synth.logit_bias(w, layer=0, mb=1, boosts=(0.0,))
    hot = int(info["hot"][0])

    def share(x):
        le = loads(w, layer=0, mb=1, boosts=(x,))
        return le[hot] / w.N
    x, v = bisect(share, 0.0, 8.0, 0.30, 0.001)
    print(f"HOT_BOOST_30PCT = {x!r}  # token share {v:.4f}")
    return x


def tune_pages():
    """The pages' runtime-test layer (EP64, E=256, M=4, S=2, K=8, T=8192):
    Zipf scales for masters-only max/mean 1.51, 2.01 and 3.03."""
    w = synth.WORKLOADS["pages_ep64_e256_t8k"]
    f = lambda a: masters_max_over_mean(w, loads(w, alpha=a))
    out = []
    for target in (1.51, 2.01, 3.03):
        a, v = bisect(f, 0.0, 4.0, target, 0.005, iters=24)
        out.append(a)
        print(f"  alpha {a!r} -> masters-only max/mean {v:.4f} (target {target})")
    print(f"ALPHA_PAGES = ({out[0]!r}, {out[1]!r}, {out[2]!r})")
    return out


if __name__ == "__main__":
    which = sys.argv[1:] or ["qwen3", "dsv3", "30pct", "pages"]
    if "qwen3" in which:
        tune_qwen3()
    if "dsv3" in which:
        tune_dsv3()
    if "30pct" in which:
        tune_30pct()
    if "pages" in which:
        tune_pages()
