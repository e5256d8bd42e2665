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
// written; per token 4d bytes of dout read once), the same scattered-write
// pattern as the permute, and built like it: short-lived CTAs, each token
// owned by a group of whole warps with one 16-byte chunk (8 elements) per
// thread. A thread reads the token's fp32 gradient chunk once, issues its K
// y-chunk loads before using any, accumulates the K dot products in fp32 and
// writes w*dout as bf16. dw is then summed by a fixed butterfly of warp
// shuffles and a fixed-order pass over the token's warps, so it is the same
// on every run. For the common shapes (K = 4 or 8, d <= 8192) a CTA holds
// one token and a thread exactly one chunk, with no loop and the row checks
// kept off the hot path (a row out of range is masked and reported after the
// work), which keeps it near 50 registers: two 512-thread CTAs per SM. Other
// shapes loop over their chunks. (A persistent warp-per-token form reached
// 0.90 of the copy bandwidth; the same CTA shape with a chunk loop, per-pair
// branches or several tokens per CTA spilled registers and reached 0.87-0.90.)
#include <cuda_bf16.h>

#include "ue_internal.cuh"

namespace ue {
namespace {

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
    const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return a | (b << 16);
}

// dy chunk = w * dout chunk, rounded to bf16
__device__ __forceinline__ uint4 scaled_bf16(float wk, const float (&g)[8])
{
    uint4 o;
    o.x = pack_bf16x2(wk * g[0], wk * g[1]);
    o.y = pack_bf16x2(wk * g[2], wk * g[3]);
    o.z = pack_bf16x2(wk * g[4], wk * g[5]);
    o.w = pack_bf16x2(wk * g[6], wk * g[7]);
    return o;
}

// part += <g, bf16 chunk v>, elements in order
__device__ __forceinline__ float dot_bf16(float part, const float (&g)[8], uint4 v)
{
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        part = fmaf(g[2 * q], __uint_as_float(u[q] << 16), part);
        part = fmaf(g[2 * q + 1], __uint_as_float(u[q] & 0xffff0000u), part);
    }
    return part;
}

// One chunk per thread, K known at compile time (4 or 8), d <= 8192: one
// token per CTA, blockDim = cw = the row's chunks rounded up to whole warps.
// A row out of range is only masked: its loads read row 0, which is in range,
// it stores nothing, and the error is recorded after the work. VEC: dest_row
// and w are 16-byte aligned, and the token's K indices and weights arrive as
// K/4 vector loads each.
template <int K, bool VEC>
__global__ void __launch_bounds__(1024)
combine_bwd_chunk_kernel(const float* __restrict__ dout, const uint16_t* __restrict__ y,
                         const int32_t* __restrict__ dest_row, const float* __restrict__ w,
                         uint16_t* __restrict__ dy, float* __restrict__ dw, int64_t N, int d,
                         int cw, int64_t Q, int* err)
{
    constexpr unsigned kAll = (1u << K) - 1u;
    __shared__ float s_part[32][K];
    const int C = d >> 3;
    const int c = threadIdx.x;             // this thread's chunk of the row
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t n = blockIdx.x;
    const bool live = n < N;
    int rows[K];
    float wk[K], part[K];
    unsigned valid = 0u;  // pairs with a row in range
    if (VEC) {
#pragma unroll
        for (int h = 0; h < K / 4; ++h) {
            int4 r4 = make_int4(0, 0, 0, 0);
            float4 w4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (live) {
                r4 = __ldg(reinterpret_cast<const int4*>(dest_row + n * K) + h);
                w4 = __ldg(reinterpret_cast<const float4*>(w + n * K) + h);
            }
            rows[4 * h] = r4.x;
            rows[4 * h + 1] = r4.y;
            rows[4 * h + 2] = r4.z;
            rows[4 * h + 3] = r4.w;
            wk[4 * h] = w4.x;
            wk[4 * h + 1] = w4.y;
            wk[4 * h + 2] = w4.z;
            wk[4 * h + 3] = w4.w;
        }
    } else {
#pragma unroll
        for (int k = 0; k < K; ++k) {
            rows[k] = live ? __ldg(dest_row + n * K + k) : 0;
            wk[k] = live ? __ldg(w + n * K + k) : 0.0f;
        }
    }
#pragma unroll
    for (int k = 0; k < K; ++k) {
        const int r = rows[k];
        const bool ok = (unsigned long long)(unsigned)r < (unsigned long long)Q;  // r >= 0 && r < Q
        rows[k] = ok ? r : 0;
        valid |= ok ? (1u << k) : 0u;
        part[k] = 0.0f;
    }
    if (live && c < C) {
        const float4* g_row = reinterpret_cast<const float4*>(dout + n * d);
        const float4 g0 = __ldcs(g_row + 2 * c);
        const float4 g1 = __ldcs(g_row + 2 * c + 1);
        const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        uint4 v[K];
#pragma unroll
        for (int k = 0; k < K; ++k)
            v[k] = __ldcs(reinterpret_cast<const uint4*>(y + (int64_t)rows[k] * d) + c);
#pragma unroll
        for (int k = 0; k < K; ++k) {
            part[k] = dot_bf16(part[k], g, v[k]);
            if ((valid >> k) & 1u)
                __stcs(reinterpret_cast<uint4*>(dy + (int64_t)rows[k] * d) + c, scaled_bf16(wk[k], g));
        }
    }
    // dw: butterfly inside each warp, then the token's warps in order
#pragma unroll
    for (int k = 0; k < K; ++k) {
        float p = part[k];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(kFull, p, off);
        if (lane == 0) s_part[warp][k] = p;
    }
    __syncthreads();
    if (live && c < K && ((valid >> c) & 1u)) {
        const int wpt = cw / 32;
        float acc = 0.0f;
        for (int ww = 0; ww < wpt; ++ww) acc += s_part[ww][c];
        dw[n * K + c] = acc;
    }
    if (live && c == 0 && valid != kAll) {
        const int k = __ffs(~valid & kAll) - 1;  // the first pair out of range
        raise_error(err, UE_ERR_DEVICE_BOUNDS, (int)min(n * K + k, (int64_t)INT_MAX));
    }
}

// threads per CTA of the looping kernel, by the largest K (registers: K rows,
// weights and partial dots, plus K 16-byte chunks in flight)
template <int KMAX>
__host__ __device__ constexpr int bwd_threads() { return KMAX <= 8 ? 512 : (KMAX <= 16 ? 256 : 128); }

// Any other shape: a thread loops over its chunks of the row; any K <= KMAX.
template <int KMAX>
__global__ void __launch_bounds__(bwd_threads<KMAX>())
combine_bwd_kernel(const float* __restrict__ dout, const uint16_t* __restrict__ y,
                   const int32_t* __restrict__ dest_row, const float* __restrict__ w,
                   uint16_t* __restrict__ dy, float* __restrict__ dw, int64_t N, int K, int d,
                   int cw, int64_t Q, int* err)
{
    constexpr int NT = bwd_threads<KMAX>();
    __shared__ float s_part[NT / 32][KMAX];
    const int C = d >> 3;
    const int tpc = NT / cw;               // tokens per CTA
    const int sub = threadIdx.x / cw;      // the token within the CTA
    const int lt = threadIdx.x - sub * cw; // the thread within the token's group
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t n = (int64_t)blockIdx.x * tpc + sub;
    const bool live = sub < tpc && n < N;
    int rows[KMAX];
    float wk[KMAX], part[KMAX];
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
        rows[k] = -1;
        wk[k] = 0.0f;
        part[k] = 0.0f;
        if (live && k < K) {
            const int r = __ldg(dest_row + n * K + k);
            if (r >= 0 && (int64_t)r < Q) {
                rows[k] = r;
                wk[k] = __ldg(w + n * K + k);
            } else if (lt == 0) {
                raise_error(err, UE_ERR_DEVICE_BOUNDS, (int)min(n * K + k, (int64_t)INT_MAX));
            }
        }
    }
    const float4* g_row = reinterpret_cast<const float4*>(dout + (live ? n : 0) * d);
    for (int c = lt; live && c < C; c += cw) {
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
            part[k] = dot_bf16(part[k], g, v[k]);
            __stcs(reinterpret_cast<uint4*>(dy + (int64_t)rows[k] * d) + c, scaled_bf16(wk[k], g));
        }
    }
    // dw: butterfly inside each warp, then the token's warps in order
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
        float p = part[k];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(kFull, p, off);
        if (lane == 0) s_part[warp][k] = p;
    }
    __syncthreads();
    if (live && lt < K) {
        const int wpt = cw / 32;
        const int w0 = (sub * cw) / 32;
        float acc = 0.0f;
        for (int ww = 0; ww < wpt; ++ww) acc += s_part[w0 + ww][lt];
        // every thread of the group holds the rows; pick pair (n, lt)'s
        int r_l = -1;
#pragma unroll
        for (int k = 0; k < KMAX; ++k)
            if (k == lt) r_l = rows[k];
        if (r_l >= 0) dw[n * K + lt] = acc;
    }
}

template <int KMAX>
void shape_loop(const Sizes& z, BwdShape* out)
{
    constexpr int NT = bwd_threads<KMAX>();
    const int C = z.d / 8;
    const int cw = std::min(((C + 31) / 32) * 32, NT);  // whole warps per token
    const int tpc = NT / cw;
    out->cw = cw;
    out->threads = NT;
    out->single = 0;
    out->grid = (int)std::max<int64_t>(1, (z.N + tpc - 1) / tpc);
}

}  // namespace

cudaError_t plan_combine_backward_shape(const Sizes& z, BwdShape* out)
{
    const int C = z.d / 8;
    if ((z.K == 4 || z.K == 8) && C <= 1024) {
        // one chunk per thread, one token per CTA
        const int cw = ((C + 31) / 32) * 32;
        out->cw = cw;
        out->threads = cw;
        out->single = 1;
        out->grid = (int)std::max<int64_t>(1, z.N);
        return cudaSuccess;
    }
    if (z.K <= 4) shape_loop<4>(z, out);
    else if (z.K <= 8) shape_loop<8>(z, out);
    else if (z.K <= 16) shape_loop<16>(z, out);
    else shape_loop<32>(z, out);
    return cudaSuccess;
}

cudaError_t launch_combine_backward(const Sizes& z, const BwdShape& sh, const float* dout,
                                    const uint16_t* y, const int32_t* dest_row, const float* w,
                                    uint16_t* dy, float* dw, int* err, cudaStream_t st)
{
    if (z.N == 0) return cudaSuccess;
    if (sh.single) {
        const bool vec = ((reinterpret_cast<uintptr_t>(dest_row) |
                           reinterpret_cast<uintptr_t>(w)) & 15u) == 0;
#define UE_BWD_CHUNK(KK, V)                                                                      \
    combine_bwd_chunk_kernel<KK, V><<<sh.grid, sh.cw, 0, st>>>(dout, y, dest_row, w, dy, dw, z.N, \
                                                              z.d, sh.cw, z.Q, err)
        if (z.K == 8 && vec) UE_BWD_CHUNK(8, true);
        else if (z.K == 8) UE_BWD_CHUNK(8, false);
        else if (vec) UE_BWD_CHUNK(4, true);
        else UE_BWD_CHUNK(4, false);
#undef UE_BWD_CHUNK
        return cudaGetLastError();
    }
#define UE_BWD(KM)                                                                               \
    combine_bwd_kernel<KM><<<sh.grid, bwd_threads<KM>(), 0, st>>>(dout, y, dest_row, w, dy, dw,  \
                                                                  z.N, z.K, z.d, sh.cw, z.Q, err)
    if (z.K <= 4) UE_BWD(4);
    else if (z.K <= 8) UE_BWD(8);
    else if (z.K <= 16) UE_BWD(16);
    else UE_BWD(32);
#undef UE_BWD
    return cudaGetLastError();
}

}  // namespace ue
