"""GPU parity of the combine's one-token-per-CTA kernel (K = 4 or 8, d/8
chunks per row between 128 and 1024) and of the permute's backward, which is
the same kernel with unit weights.

Cases: both K, the narrowest and the widest rows the kernel takes (d = 1024
and d = 8192), rows out of range (they contribute nothing and set
UE_ERR_DEVICE_BOUNDS), and a dest_row buffer that is not 16-byte aligned,
which takes the persistent kernel and must give the same bits. The combine's
backward, which loads a token's indices and weights as vectors only when
both buffers are 16-byte aligned, must also give the same bits either way.

Tolerance (the combine's, from its arithmetic): K fused multiply-adds into
an fp32 sum starting from 0, k ascending, and the rounding of each w_k to
fp32: |out_gpu - out| <= 1e-6 sum_k |w_k y_k| + 1e-30 ((K + 1) 2^-24 < 1e-6).

"UltraEP" README, "Interface / 2. Forward and backward": combine(recv_tokens)
after the experts; the backward gathers gradients back to logical experts.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import token_rerouting_b200 as ue
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu


def inputs(N, K, d, seed):
    rng = np.random.default_rng(seed)
    dest = rng.permutation(N * K).astype(np.int32).reshape(N, K)
    w = rng.random((N, K)).astype(np.float32)
    y = synth.bf16_normal(N * K, d, seed, 43)
    return dest, w, y


def scale_of(y, dest, w):
    N, K = dest.shape
    yf = synth.bf16_bits_to_f32(y[dest.reshape(-1)]).astype(np.float64).reshape(N, K, -1)
    return np.einsum("nk,nkd->nd", np.abs(w.astype(np.float64)), np.abs(yf)), np.abs(yf).sum(axis=1)


def run(N, K, d, dest, w, y, dest_offset=0):
    """combine and permute backward through the C ABI; dest_row placed at an
    offset of dest_offset int32 words into its buffer."""
    R, T = 1, N
    L = gh.make_layer(R, T, K, K, 1, d, with_rows=False)
    try:
        dev = L.device
        buf = torch.zeros(N * K + dest_offset, dtype=torch.int32, device=dev)
        dest_t = buf[dest_offset:].view(N, K)
        dest_t.copy_(torch.from_numpy(dest))
        w_t = torch.from_numpy(w).to(dev)
        y_t = gh.bf16_to_device(y, dev)
        out = torch.full((N, d), float("nan"), dtype=torch.float32, device=dev)
        dh = torch.full((N, d), float("nan"), dtype=torch.float32, device=dev)
        ue.ue_combine(L.ctx, y_t, dest_t, w_t, out)
        ue.ue_permute_backward(L.ctx, y_t, dest_t, dh)
        rc = L.error()
        torch.cuda.synchronize()
        return out.cpu().numpy(), dh.cpu().numpy(), rc
    finally:
        L.close()


@pytest.mark.parametrize("K", [4, 8])
@pytest.mark.parametrize("d,N", [(1024, 300), (8192, 40)])
def test_token_kernel_matches_the_oracle(K, d, N):
    gh.ensure_built()
    dest, w, y = inputs(N, K, d, seed=K * 7 + d)
    out, dh, rc = run(N, K, d, dest, w, y)
    assert rc == ue.UE_OK
    sc, sc1 = scale_of(y, dest, w)
    out_or = oracle.combine(y, N, K, dest, w)
    assert (np.abs(out.astype(np.float64) - out_or) <= 1e-6 * sc + 1e-30).all()
    dh_or = oracle.permute_backward(y, N, K, dest)
    assert (np.abs(dh.astype(np.float64) - dh_or) <= K * 2.0 ** -24 * sc1 + 1e-30).all()


@pytest.mark.parametrize("K", [4, 8])
def test_rows_out_of_range_contribute_nothing(K):
    gh.ensure_built()
    N, d = 64, 1024
    dest, w, y = inputs(N, K, d, seed=90 + K)
    bad = dest.copy()
    bad[3, 0] = -1
    bad[10, K - 1] = N * K + 7
    bad[11, 1] = np.iinfo(np.int32).max
    out, dh, rc = run(N, K, d, bad, w, y)
    assert rc == ue.UE_ERR_DEVICE_BOUNDS
    # expected: the bad rows left out (weight 0, any in-range row)
    keep = (bad >= 0) & (bad < N * K)
    dest0 = np.where(keep, bad, 0).astype(np.int32)
    w0 = np.where(keep, w, 0.0).astype(np.float32)
    sc, _ = scale_of(y, dest0, w0)
    out_or = oracle.combine(y, N, K, dest0, w0)
    assert (np.abs(out.astype(np.float64) - out_or) <= 1e-6 * sc + 1e-30).all()
    ones = keep.astype(np.float32)
    sc1, _ = scale_of(y, dest0, ones)
    dh_or = oracle.combine(y, N, K, dest0, ones)
    assert (np.abs(dh.astype(np.float64) - dh_or) <= K * 2.0 ** -24 * sc1 + 1e-30).all()


@pytest.mark.parametrize("K", [4, 8])
def test_unaligned_rows_take_the_persistent_kernel(K):
    gh.ensure_built()
    N, d = 200, 2048
    dest, w, y = inputs(N, K, d, seed=300 + K)
    out_a, dh_a, rc_a = run(N, K, d, dest, w, y, dest_offset=0)
    out_u, dh_u, rc_u = run(N, K, d, dest, w, y, dest_offset=1)
    assert rc_a == ue.UE_OK and rc_u == ue.UE_OK
    np.testing.assert_array_equal(out_a.view(np.uint32), out_u.view(np.uint32))
    np.testing.assert_array_equal(dh_a.view(np.uint32), dh_u.view(np.uint32))


@pytest.mark.parametrize("K", [4, 8])
def test_combine_backward_unaligned_rows_give_the_same_bits(K):
    """The combine's backward loads a token's indices and weights as vectors
    when dest_row and w are 16-byte aligned, one by one otherwise."""
    gh.ensure_built()
    N, d = 150, 2048
    dest, w, y = inputs(N, K, d, seed=500 + K)
    dout = synth.normal_f32(N * d, 7, 44).reshape(N, d)
    L = gh.make_layer(1, N, K, K, 1, d, with_rows=False)
    try:
        dev = L.device
        y_t = gh.bf16_to_device(y, dev)
        dout_t = torch.from_numpy(dout).to(dev)
        res = []
        for off in (0, 1):
            dbuf = torch.zeros(N * K + off, dtype=torch.int32, device=dev)
            wbuf = torch.zeros(N * K + off, dtype=torch.float32, device=dev)
            dest_t = dbuf[off:].view(N, K)
            w_t = wbuf[off:].view(N, K)
            dest_t.copy_(torch.from_numpy(dest))
            w_t.copy_(torch.from_numpy(w))
            dy = torch.zeros_like(y_t)
            dw = torch.zeros((N, K), dtype=torch.float32, device=dev)
            ue.ue_combine_backward(L.ctx, dout_t, y_t, dest_t, w_t, dy, dw)
            assert L.error() == ue.UE_OK
            res.append((gh.bf16_to_host_u16(dy), dw.cpu().numpy()))
        np.testing.assert_array_equal(res[0][0], res[1][0])
        np.testing.assert_array_equal(res[0][1].view(np.uint32), res[1][1].view(np.uint32))
    finally:
        L.close()
