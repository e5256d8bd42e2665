"""GPU parity of the backward of the combine and of the permute.

Tolerances, from the arithmetic:
* dy = w * dout is one fp32 product rounded to bf16 (8 bits of precision,
  unit roundoff 2^-8): within (2^-8 + 2^-23) |w dout| of the exact value
  (+ the bf16 subnormal step).
* dw is a dot product of d terms accumulated in fp32 by each thread of the
  token's group of cw threads (whole warps) over its chunks (T_p = 8
  ceil((d/8)/cw) terms), then by a fixed butterfly over each warp's 32 lanes
  (5 levels) and a sum over the group's cw/32 warps in order: normwise
  |dw_gpu - dw| <= (T_p + 5 + cw/32 - 1 + 2) 2^-24 sum_c |dout_c y_c|.
  cw follows the kernel's launch shape: the chunks rounded up to whole warps
  (one chunk per thread for K = 4 or 8 and d <= 8192; otherwise at most 512
  threads for K <= 8, 256 for K <= 16, 128 above).
* dhidden is K bf16 rows summed in fp32: normwise K 2^-24 sum_k |ddispatch|.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu


def dw_bound_factor(d, K):
    C = d // 8
    if K in (4, 8) and C <= 1024:
        cw = 32 * math.ceil(C / 32)          # one chunk per thread
    else:
        nt = 512 if K <= 8 else (256 if K <= 16 else 128)
        cw = min(32 * math.ceil(C / 32), nt)  # threads per token
    per_thread = 8 * math.ceil(C / cw)       # terms each thread accumulates
    return (per_thread + 5 + cw // 32 - 1 + 2) * 2.0 ** -24


def inputs(N, K, d, seed):
    rng = np.random.default_rng(seed)
    dest = rng.permutation(N * K).astype(np.int32).reshape(N, K)
    w = rng.random((N, K)).astype(np.float32)
    dout = synth.normal_f32(N * d, seed, 41).reshape(N, d)
    y = synth.bf16_normal(N * K, d, seed, 42)
    return dest, w, dout, y


def run_gpu(L, dest, w, dout, y):
    dev = L.device
    dest_t = torch.from_numpy(dest).to(dev)
    w_t = torch.from_numpy(w).to(dev)
    dout_t = torch.from_numpy(dout).to(dev)
    y_t = gh.bf16_to_device(y, dev)
    dy_t = torch.empty_like(y_t)
    dw_t = torch.empty_like(w_t)
    import token_rerouting_b200 as ue
    ue.ue_combine_backward(L.ctx, dout_t, y_t, dest_t, w_t, dy_t, dw_t)
    dh_t = torch.empty((dest.shape[0], y.shape[1]), dtype=torch.float32, device=dev)
    ue.ue_permute_backward(L.ctx, y_t, dest_t, dh_t)
    assert L.error() == 0
    return gh.bf16_to_host_u16(dy_t), dw_t.cpu().numpy(), dh_t.cpu().numpy()


def check(dest, w, dout, y, dy_g, dw_g, dh_g, tokens=None):
    N, K = dest.shape
    d = y.shape[1]
    toks = np.arange(N) if tokens is None else tokens
    dy_o, dw_o = oracle.combine_backward(dout, y, K, dest, w, tokens=tokens)
    # dy: rows of the sampled tokens, in (token, k) order
    rows = dest[toks].reshape(-1)
    got = synth.bf16_bits_to_f32(dy_g[rows]).astype(np.float64)
    err = np.abs(got - dy_o)
    bound = (2.0 ** -8 + 2.0 ** -23) * np.abs(dy_o) + 2.0 ** -133
    assert (err <= bound).all(), f"dy off by {np.max(err / bound):.3g} of the bound"
    # dw
    yf = synth.bf16_bits_to_f32(y[rows]).astype(np.float64).reshape(len(toks), K, d)
    scale = np.einsum("nd,nkd->nk", np.abs(dout[toks].astype(np.float64)), np.abs(yf))
    err = np.abs(dw_g[toks].astype(np.float64) - dw_o)
    bound = dw_bound_factor(d, K) * scale + 1e-30
    assert (err <= bound).all(), f"dw off by {np.max(err / bound):.3g} of the bound"
    # dhidden
    dh_o = oracle.permute_backward(y, N, K, dest, tokens=tokens)
    scale = np.abs(yf).sum(axis=1)
    err = np.abs(dh_g[toks].astype(np.float64) - dh_o)
    assert (err <= K * 2.0 ** -24 * scale + 1e-30).all()


@pytest.mark.parametrize("R,T,E,K,S,d", [(8, 512, 64, 4, 2, 256), (3, 37, 6, 3, 2, 24),
                                         (4, 100, 16, 8, 1, 4096), (2, 64, 8, 2, 1, 7168)])
def test_backward_small(R, T, E, K, S, d):
    L = gh.make_layer(R, T, E, K, S, d, with_rows=False)
    try:
        dest, w, dout, y = inputs(R * T, K, d, seed=R + T + K)
        dy_g, dw_g, dh_g = run_gpu(L, dest, w, dout, y)
        check(dest, w, dout, y, dy_g, dw_g, dh_g)
    finally:
        L.close()


def test_backward_full_size_sampled():
    """Qwen3-shaped layer (N = 262144, K = 8, d = 4096): the GPU runs on every
    token; 256 sampled tokens carry random gradients and expert rows, every
    other row is zero, and the sampled tokens are checked."""
    w_ = synth.WORKLOADS["qwen3_layer_r64_e128"]
    N, K, d = w_.N, w_.K, w_.d
    L = gh.make_layer(w_.R, w_.T, w_.E, K, w_.S, d, with_rows=False)
    dev = L.device
    try:
        rng = np.random.default_rng(77)
        dest = rng.permutation(N * K).astype(np.int32).reshape(N, K)
        w = rng.random((N, K)).astype(np.float32)
        toks = np.sort(rng.choice(N, 256, replace=False))
        dout_s = synth.normal_f32(len(toks) * d, 0, 43).reshape(len(toks), d)
        y_s = synth.bf16_normal(len(toks) * K, d, 0, 44)
        import token_rerouting_b200 as ue
        dest_t = torch.from_numpy(dest).to(dev)
        w_t = torch.from_numpy(w).to(dev)
        dout_t = torch.zeros((N, d), dtype=torch.float32, device=dev)
        dout_t[torch.from_numpy(toks).to(dev)] = torch.from_numpy(dout_s).to(dev)
        y_t = torch.zeros((N * K, d), dtype=torch.bfloat16, device=dev)
        rows = dest[toks].reshape(-1)
        y_t[torch.from_numpy(rows.astype(np.int64)).to(dev)] = gh.bf16_to_device(y_s, dev)
        dy_t = torch.empty_like(y_t)
        dw_t = torch.empty_like(w_t)
        ue.ue_combine_backward(L.ctx, dout_t, y_t, dest_t, w_t, dy_t, dw_t)
        dh_t = torch.empty((N, d), dtype=torch.float32, device=dev)
        ue.ue_permute_backward(L.ctx, y_t, dest_t, dh_t)
        assert L.error() == 0
        # compact oracle inputs for the sampled tokens
        dest_c = np.arange(len(toks) * K, dtype=np.int32).reshape(len(toks), K)
        dy_c = gh.bf16_to_host_u16(dy_t[torch.from_numpy(rows.astype(np.int64)).to(dev)])
        dw_c = dw_t[torch.from_numpy(toks).to(dev)].cpu().numpy()
        dh_c = dh_t[torch.from_numpy(toks).to(dev)].cpu().numpy()
        check(dest_c, w[toks], dout_s, y_s, dy_c, dw_c, dh_c)
    finally:
        L.close()
