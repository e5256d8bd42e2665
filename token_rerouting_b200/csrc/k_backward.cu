// k_backward.cu -- backward of the gate-weighted combine.
//
// "UltraEP" README, "Interface / 2. Forward and backward": reroute expands
// logical routing to physical replicas in the forward and gathers gradients
// back to logical experts in the backward. With the compact [N][K] routing
// each pair maps to one physical row, so the gradient that reaches the
// router's gates and the one that reaches the expert outputs are those of
// the combine out[n] = sum_k w[n][k] * y[dest_row[n*K+k]]:
//     dy[dest_row[n*K+k]] = w[n][k] * dout[n]      (bf16, rounded once)
//     dw[n][k]            = <dout[n], y[dest_row[n*K+k]]>   (fp32)
// (The permute's backward, dhidden[n] = sum_k ddispatch[dest_row[n*K+k]], is
// the combine with unit weights and runs in k_combine.cu.)
//
// Design (B200): HBM-bound (per pair: 2d bytes of y read, 2d bytes of dy
// written; per token 4d bytes of dout read once). One warp owns a token; each
// lane owns every 32nd 16-byte chunk of the row (8 elements), reads the
// token's fp32 gradient chunk once, issues the K y-chunk loads before using
// any, accumulates the K dot products in fp32 (chunks in order) and writes
// w*dout as bf16. The lanes' partial dots are then summed by a fixed
// butterfly of warp shuffles, so dw is the same on every run, and no
// block-wide barrier is needed.
#include <cuda_bf16.h>

#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdWarps = kBwdThreads / 32;

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
    const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return a | (b << 16);
}

// K <= 8 fits in 80 registers without spilling, which leaves room for three
// CTAs (24 token warps) per SM; larger K keeps the default budget.
template <int KMAX>
__global__ void __launch_bounds__(kBwdThreads, KMAX <= 8 ? 3 : 1)
combine_bwd_kernel(const float* __restrict__ dout, const uint16_t* __restrict__ y,
                   const int32_t* __restrict__ dest_row, const float* __restrict__ w,
                   uint16_t* __restrict__ dy, float* __restrict__ dw, int64_t N, int K, int d,
                   int64_t Q, int* err)
{
    const int C = d >> 3;
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t n = gwarp; n < N; n += nwarps) {
        int rows[KMAX];
        float wk[KMAX], part[KMAX];
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            rows[k] = -1;
            wk[k] = 0.0f;
            part[k] = 0.0f;
            if (k < K) {
                const int r = __ldg(dest_row + n * K + k);
                if (r >= 0 && (int64_t)r < Q) {
                    rows[k] = r;
                    wk[k] = __ldg(w + n * K + k);
                } else if (lane == 0) {
                    raise_error(err, UE_ERR_DEVICE_BOUNDS, (int)min(n * K + k, (int64_t)INT_MAX));
                }
            }
        }
        const float4* g_row = reinterpret_cast<const float4*>(dout + n * d);
        for (int c = lane; c < C; c += 32) {
            const float4 g0 = __ldcs(g_row + 2 * c);
            const float4 g1 = __ldcs(g_row + 2 * c + 1);
            uint4 v[KMAX];
#pragma unroll
            for (int k = 0; k < KMAX; ++k)
                v[k] = rows[k] >= 0 ? __ldcs(reinterpret_cast<const uint4*>(y + (int64_t)rows[k] * d) + c)
                                    : make_uint4(0u, 0u, 0u, 0u);
            const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
            for (int k = 0; k < KMAX; ++k) {
                if (rows[k] < 0) continue;
                const uint32_t u[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    part[k] = fmaf(g[2 * q], __uint_as_float(u[q] << 16), part[k]);
                    part[k] = fmaf(g[2 * q + 1], __uint_as_float(u[q] & 0xffff0000u), part[k]);
                }
                uint4 o;
                o.x = pack_bf16x2(wk[k] * g[0], wk[k] * g[1]);
                o.y = pack_bf16x2(wk[k] * g[2], wk[k] * g[3]);
                o.z = pack_bf16x2(wk[k] * g[4], wk[k] * g[5]);
                o.w = pack_bf16x2(wk[k] * g[6], wk[k] * g[7]);
                __stcs(reinterpret_cast<uint4*>(dy + (int64_t)rows[k] * d) + c, o);
            }
        }
        // dw: fixed butterfly over the warp; lane k writes dw[n][k]
        float mine = 0.0f;
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            float p = part[k];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(kFull, p, off);
            if (lane == k) mine = p;
        }
        if (lane < K && lane < KMAX) {
            // every lane holds the rows of all K pairs; pick pair (n, lane)'s
            // without dynamic register indexing
            int r_l = -1;
#pragma unroll
            for (int k = 0; k < KMAX; ++k)
                if (k == lane) r_l = rows[k];
            if (r_l >= 0) dw[n * K + lane] = mine;
        }
    }
}

template <int KMAX>
cudaError_t shape_k(const Sizes& z, int num_sms, int* grid)
{
    int per_sm = 0;
    cudaError_t ce = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, combine_bwd_kernel<KMAX>,
                                                                   kBwdThreads, 0);
    if (ce != cudaSuccess) return ce;
    per_sm = std::max(per_sm, 1);
    const int64_t need = std::max<int64_t>(1, (z.N + kBwdWarps - 1) / kBwdWarps);
    *grid = (int)std::min<int64_t>(need, (int64_t)num_sms * per_sm);
    return cudaSuccess;
}

}  // namespace

cudaError_t plan_combine_backward_grid(const Sizes& z, int num_sms, int* grid)
{
    if (z.K <= 4) return shape_k<4>(z, num_sms, grid);
    if (z.K <= 8) return shape_k<8>(z, num_sms, grid);
    if (z.K <= 16) return shape_k<16>(z, num_sms, grid);
    return shape_k<32>(z, num_sms, grid);
}

cudaError_t launch_combine_backward(const Sizes& z, const float* dout, const uint16_t* y,
                                    const int32_t* dest_row, const float* w, uint16_t* dy,
                                    float* dw, int grid, int* err, cudaStream_t st)
{
    if (z.N == 0) return cudaSuccess;
#define UE_BWD(KM)                                                                              \
    combine_bwd_kernel<KM><<<grid, kBwdThreads, 0, st>>>(dout, y, dest_row, w, dy, dw, z.N, z.K, \
                                                         z.d, z.Q, err)
    if (z.K <= 4) UE_BWD(4);
    else if (z.K <= 8) UE_BWD(8);
    else if (z.K <= 16) UE_BWD(16);
    else UE_BWD(32);
#undef UE_BWD
    return cudaGetLastError();
}

}  // namespace ue
