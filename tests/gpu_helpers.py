"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
CUDA path through the C ABI, and compare with the oracle.

Tolerances (written here once, used by every GPU test):

* integer, index and byte outputs: bit-exact.
* gate weights w (fp32, computed in fp64 and rounded once): within one fp32
  ulp of the oracle's fp64 value, |w_gpu - w| <= 2^-23 |w| (+ 2^-149).
* combine (fp32, K fused multiply-adds): normwise per element,
  |out_gpu - out| <= 1e-6 * sum_k |w_k y_k| + 1e-30. The fp32 error is at most
  the rounding of each w_k (2^-24 relative) plus K roundings of the running
  sum (K * 2^-24 of sum_k |w_k y_k|), (K + 1) * 2^-24 < 1e-6 for K <= 15.
"""
from __future__ import annotations

import numpy as np
import torch

import token_rerouting_b200 as ue
from token_rerouting_b200 import build as ue_build

W_RTOL = 2.0 ** -23
W_ATOL = 2.0 ** -149
COMBINE_RTOL = 1e-6
COMBINE_ATOL = 1e-30


def ensure_built():
    ue_build.build()
    ue.load_library()


def bf16_to_device(h_u16: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(h_u16).view(np.int16)).to(dev).view(torch.bfloat16)


def bf16_to_host_u16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def make_layer(R, T, E, K, S, d, with_rows=True):
    ensure_built()
    return ue.Layer(R, T, E, K, S, d, device=0, with_rows=with_rows)


def load_inputs(layer, logits: np.ndarray, hidden_u16: np.ndarray | None = None):
    layer.logits.copy_(torch.from_numpy(np.ascontiguousarray(logits, dtype=np.float32)))
    if hidden_u16 is not None:
        layer.hidden.copy_(bf16_to_device(hidden_u16, layer.device))


def routing_results(layer):
    torch.cuda.synchronize()
    return dict(idx=layer.idx.cpu().numpy(), w=layer.w.cpu().numpy(),
                load_re=layer.load_re.cpu().numpy(), load_e=layer.load_e.cpu().numpy(),
                phys_slot=layer.phys_slot.cpu().numpy(), dest_row=layer.dest_row.cpu().numpy(),
                **layer.plan_arrays())


def assert_weights_close(w_gpu, w_or):
    w_gpu = np.asarray(w_gpu, dtype=np.float64)
    err = np.abs(w_gpu - w_or)
    bound = W_RTOL * np.abs(w_or) + W_ATOL
    bad = err > bound
    assert not bad.any(), (f"{bad.sum()} weights off by more than one ulp; "
                           f"worst {err.max():.3e} at {np.argwhere(bad)[:3].tolist()}")


def assert_routing_equal(g, o):
    """Every integer output of the routing half of the path, bit-exact, and
    the weights within one ulp."""
    np.testing.assert_array_equal(g["idx"], o["idx"], err_msg="top-k ids")
    assert_weights_close(g["w"], o["w"])
    np.testing.assert_array_equal(g["load_re"], o["load_re"], err_msg="load_re")
    np.testing.assert_array_equal(g["load_e"], o["load_e"], err_msg="load_e")
    pl = o["plan"]
    np.testing.assert_array_equal(g["slot_expert"], pl.slot_expert, err_msg="slot_expert")
    np.testing.assert_array_equal(g["n_copies"], pl.n_copies, err_msg="n_copies")
    np.testing.assert_array_equal(g["slot_quota"], pl.slot_quota, err_msg="slot_quota")
    np.testing.assert_array_equal(g["slot_offset"], pl.slot_offset, err_msg="slot_offset")
    np.testing.assert_array_equal(g["rank_load"], pl.rank_load, err_msg="rank_load")
    np.testing.assert_array_equal(g["stats"], pl.stats, err_msg="stats")
    np.testing.assert_array_equal(g["phys_slot"], o["phys_slot"], err_msg="phys_slot")
    np.testing.assert_array_equal(g["dest_row"], o["dest_row"], err_msg="dest_row")


def combine_scale(y_u16_rows_by_k: np.ndarray, w: np.ndarray) -> np.ndarray:
    """sum_k |w_k * y_k| per element: the scale of the combine tolerance.
    y_u16_rows_by_k: [n, K, d] bf16 bits; w: [n, K]."""
    y = (y_u16_rows_by_k.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.einsum("nk,nkd->nd", np.abs(w), np.abs(y))


def assert_combine_close(out_gpu, out_or, scale):
    err = np.abs(np.asarray(out_gpu, dtype=np.float64) - out_or)
    bound = COMBINE_RTOL * scale + COMBINE_ATOL
    bad = err > bound
    assert not bad.any(), (f"{bad.sum()} combine elements out of tolerance; worst ratio "
                           f"{(err / bound).max():.3e}")


def _workers():
    import os
    return max(1, min(16, os.cpu_count() or 1))


def assert_dispatch_all_rows(layer, hidden_u16, K, dest_row_or, chunk_rows=1 << 15):
    """Every dispatch row of the device against the oracle's permute (built
    from the oracle's own dest_row), chunk by chunk so that the rows are
    never all on the host at once. The oracle calls and the comparisons run
    in threads (both release the interpreter lock)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    Q = layer.Q

    def job(r0):
        r1 = min(Q, r0 + chunk_rows)
        got = bf16_to_host_u16(layer.dispatch[r0:r1])
        exp = oracle.permute_rows(hidden_u16, K, dest_row_or, np.arange(r0, r1, dtype=np.int64))
        if np.array_equal(got, exp):
            return None
        bad = np.nonzero((got != exp).any(axis=1))[0]
        return (r0 + bad[:4]).tolist(), int(bad.size)

    with ThreadPoolExecutor(_workers()) as ex:
        res = [r for r in ex.map(job, range(0, Q, chunk_rows)) if r is not None]
    assert not res, (f"{sum(n for _, n in res)} dispatch rows differ from the oracle's permute; "
                     f"first {res[0][0]}")


def expert_outputs_on_device(layer, hidden_u16, sigma):
    """Write the stand-in expert outputs y[r] = hidden[sigma[r]] into the
    layer's dispatch buffer (input construction for the combine check)."""
    import torch
    sig = torch.from_numpy(np.ascontiguousarray(sigma, dtype=np.int64)).to(layer.device)
    step = 1 << 18
    for r0 in range(0, layer.Q, step):
        r1 = min(layer.Q, r0 + step)
        torch.index_select(layer.hidden, 0, sig[r0:r1], out=layer.dispatch[r0:r1])
    torch.cuda.synchronize(layer.device)


def assert_combine_all_tokens(layer, hidden_u16, sigma, K, dest_row_or, w_or,
                              tokens=None, chunk_tokens=2048):
    """Every element of the device's combine output (or those of the listed
    tokens) against the oracle's fp64 combine of the same expert outputs
    y[r] = hidden[sigma[r]] at the oracle's dest_row with the oracle's
    weights, within the normwise tolerance. For each chunk of tokens the
    oracle is given the chunk's K rows per token, gathered on the host, with
    dest_row renumbered to them; the tolerance scale sum_k |w_k y_k| is the
    oracle's combine of |y| with |w|."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    N = layer.N
    toks = np.arange(N, dtype=np.int64) if tokens is None else np.asarray(tokens, np.int64)
    out_dev = layer.out

    def job(c0):
        t = toks[c0:c0 + chunk_tokens]
        n = t.size
        if tokens is None:
            got = out_dev[int(t[0]):int(t[-1]) + 1].cpu().numpy()
        else:
            import torch
            got = out_dev[torch.from_numpy(t).to(layer.device)].cpu().numpy()
        rows = dest_row_or[t].ravel()
        ych = np.ascontiguousarray(hidden_u16[sigma[rows]])
        dloc = np.arange(n * K, dtype=np.int32).reshape(n, K)
        wt = np.ascontiguousarray(w_or[t], dtype=np.float64)
        exp = oracle.combine(ych, n, K, dloc, wt)
        np.bitwise_and(ych, np.uint16(0x7FFF), out=ych)
        scale = oracle.combine(ych, n, K, dloc, np.abs(wt))
        err = np.abs(got.astype(np.float64) - exp)
        bound = COMBINE_RTOL * scale + COMBINE_ATOL
        bad = err > bound
        if not bad.any():
            return None
        return int(bad.sum()), float((err / bound).max()), int(t[np.argwhere(bad)[0][0]])

    with ThreadPoolExecutor(_workers()) as ex:
        res = [r for r in ex.map(job, range(0, toks.size, chunk_tokens)) if r is not None]
    assert not res, (f"{sum(r[0] for r in res)} combine elements out of tolerance; worst ratio "
                     f"{max(r[1] for r in res):.3e}; first token {res[0][2]}")
