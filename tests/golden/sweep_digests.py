"""Write the oracle's routing digests of every instance of the
non-stationary sweep (48 layers x 8 microbatches of the Qwen3-shaped layer)
to ``sweep_digests.json``.

For each instance the logits come from ``synth``; the oracle computes the
top-k ids, the counts, the plan (the path's greedy rule, and the capacity
planner at the pages' defaults: "UltraEP" README, "Performance Tuning /
Replication planning", eps 0.01, early stop 1.0, at least 1024 pairs per
replica) and the reroute under each plan. The stored value is
``tests.routing_digest.routing_digest`` of those arrays. Only the oracle and
the input generator are used. The GPU sweep test compares the digest of its
own outputs with these, instance by instance.

Run (about ten minutes on eight cores):
    python tests/golden/sweep_digests.py [--workers N]
"""
import argparse
import json
import multiprocessing as mp
import os
import sys

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), "..", ".."))
sys.path.insert(0, ROOT)

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "sweep_digests.json")
NAME = "sweep_48x8_r64_e128"


def instance_digests(lm):
    import numpy as np  # noqa: F401

    import oracle
    import synth
    from tests.routing_digest import flatten_oracle, routing_digest
    layer, mb = lm
    w = synth.WORKLOADS[NAME]
    logits = synth.logits(w, layer, mb)
    idx, wts = oracle.gate_topk(logits, w.K)
    load_re, load_e = oracle.count(idx, w.R, w.T, w.E)
    res = {}
    for planner in ("greedy", "bisect"):
        pl = oracle.plan(load_e, w.R, w.S) if planner == "greedy" else \
            oracle.plan_bisect(load_e, w.R, w.S)
        phys, dest = oracle.reroute(idx, w.R, w.E, w.S, pl)
        o = dict(idx=idx, w=wts, load_re=load_re, load_e=load_e, plan=pl, phys_slot=phys,
                 dest_row=dest)
        res[planner] = routing_digest(flatten_oracle(o))
    return layer, mb, res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workers", type=int, default=os.cpu_count() or 1)
    args = ap.parse_args()
    import numpy as np

    import synth
    w = synth.WORKLOADS[NAME]
    todo = [(l, m) for l in range(w.layers) for m in range(w.microbatches)]
    ctx = mp.get_context("spawn")
    out = {"greedy": [None] * len(todo), "bisect": [None] * len(todo)}
    with ctx.Pool(args.workers) as pool:
        for layer, mb, res in pool.imap_unordered(instance_digests, todo):
            i = layer * w.microbatches + mb
            for k, v in res.items():
                out[k][i] = v
            print(f"{layer:2d} {mb} {res['greedy'][:12]} {res['bisect'][:12]}", flush=True)
    doc = {"workload": NAME, "instances": "index = layer * 8 + microbatch",
           "numpy": np.__version__,
           "arrays": "tests.routing_digest.ARRAYS, int32 little-endian, name and size first",
           "digests": out}
    with open(OUT, "w") as f:
        json.dump(doc, f, indent=0)
        f.write("\n")
    print("wrote", OUT)


if __name__ == "__main__":
    main()
