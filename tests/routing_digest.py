"""One SHA-256 digest over every integer output of the routing half of the
path (top-k ids, counts, the plan arrays, the reroute), so that a stored
digest written from the oracle can be compared with the GPU's outputs of
the same layer instance byte for byte.

Each array is hashed as little-endian int32 after its name and element
count, in the fixed order of ``ARRAYS``. Equal digests mean equal arrays;
on a mismatch the caller recomputes the oracle to name the array that
differs.
"""
from __future__ import annotations

import hashlib

import numpy as np

ARRAYS = ("idx", "load_re", "load_e", "slot_expert", "n_copies", "slot_quota", "slot_offset",
          "rank_load", "stats", "phys_slot", "dest_row")


def flatten_oracle(o: dict) -> dict:
    """The oracle's result dict (``oracle.run_path`` form, with a Plan under
    "plan") as flat named arrays."""
    pl = o["plan"]
    return dict(idx=o["idx"], load_re=o["load_re"], load_e=o["load_e"],
                slot_expert=pl.slot_expert, n_copies=pl.n_copies, slot_quota=pl.slot_quota,
                slot_offset=pl.slot_offset, rank_load=pl.rank_load, stats=pl.stats,
                phys_slot=o["phys_slot"], dest_row=o["dest_row"])


def routing_digest(arrays: dict) -> str:
    h = hashlib.sha256()
    for name in ARRAYS:
        a = np.ascontiguousarray(arrays[name], dtype="<i4").ravel()
        h.update(name.encode())
        h.update(np.int64(a.size).astype("<i8").tobytes())
        h.update(a.tobytes())
    return h.hexdigest()
