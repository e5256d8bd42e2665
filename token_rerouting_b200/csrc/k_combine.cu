// k_combine.cu -- gate-weighted combine / unpermute.
//
// "UltraEP" README, "Interface / 2. Forward and backward": combine(recv_tokens)
// after the experts. out[n] = sum_{k=0..K-1} w[n][k] * y[dest_row[n*K+k]],
// fp32, one fused multiply-add per term in k order starting from 0.
//
// Design (B200): HBM-bound gather (2*K*d bytes read, 4*d written per token).
// Each thread owns 16-byte chunks (8 bf16) of a token's row, issues all K
// chunk loads before the first FMA (K*16 bytes in flight per thread), widens
// bf16 to fp32 with shifts, and writes its 8 fp32 results as two 16-byte
// streaming stores. Rows are read with evict-first hints since each expert
// row is used by exactly one token.
// For K = 4 or 8 and 1024 <= d <= 8192, a CTA lives for one token with one
// chunk per thread and reads the token's K row indices and weights as 16-byte
// vectors (32 registers, so an SM holds 2048 threads' loads). On the
// Qwen3-shaped layer this moved 7.05 TB/s where the persistent form below
// (a grid of resident CTAs looping over tokens, several chunks per thread,
// scalar index loads) moved 6.77 TB/s; reads alone reach 7.5-7.6 TB/s. Other
// shapes take the persistent form.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kCombineThreads = 256;

// UNIT: every weight is 1 (the backward of the permute: the sum of a token's
// K dispatched rows); w is not read.
template <int KMAX, bool UNIT>
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const uint16_t* __restrict__ y, const int32_t* __restrict__ dest_row,
               const float* __restrict__ w, float* __restrict__ out, int64_t N, int K,
               int d, int tpt, int64_t Q, int* err)
{
    const int C = d >> 3;  // 16-byte chunks per row
    const int tpb = blockDim.x / tpt;
    const int sub = threadIdx.x / tpt;
    const int lt = threadIdx.x - sub * tpt;
    if (sub >= tpb) return;
    for (int64_t n = (int64_t)blockIdx.x * tpb + sub; n < N; n += (int64_t)gridDim.x * tpb) {
        int rows[KMAX];
        float wk[KMAX];
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            rows[k] = -1;
            wk[k] = 0.0f;
            if (k < K) {
                const int r = __ldg(dest_row + n * K + k);
                if (r >= 0 && (int64_t)r < Q) {
                    rows[k] = r;
                    wk[k] = UNIT ? 1.0f : __ldg(w + n * K + k);
                } else if (lt == 0) {
                    raise_error(err, UE_ERR_DEVICE_BOUNDS, (int)min(n * K + k, (int64_t)INT_MAX));
                }
            }
        }
        for (int c = lt; c < C; c += tpt) {
            uint4 v[KMAX];
#pragma unroll
            for (int k = 0; k < KMAX; ++k) {
                if (rows[k] >= 0)
                    v[k] = __ldcs(reinterpret_cast<const uint4*>(y + (int64_t)rows[k] * d) + c);
                else
                    v[k] = make_uint4(0u, 0u, 0u, 0u);
            }
            float acc[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
#pragma unroll
            for (int k = 0; k < KMAX; ++k) {
                if (rows[k] >= 0) {
                    const uint32_t u[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        acc[2 * q] = fmaf(wk[k], __uint_as_float(u[q] << 16), acc[2 * q]);
                        acc[2 * q + 1] = fmaf(wk[k], __uint_as_float(u[q] & 0xffff0000u), acc[2 * q + 1]);
                    }
                }
            }
            float4* dst = reinterpret_cast<float4*>(out + n * d) + 2 * c;
            __stcs(dst, make_float4(acc[0], acc[1], acc[2], acc[3]));
            __stcs(dst + 1, make_float4(acc[4], acc[5], acc[6], acc[7]));
        }
    }
}

// One token per CTA (blockIdx.x), one 16-byte chunk per thread (threadIdx.x
// < C = d/8); dest_row and w are 16-byte aligned, so the token's K indices and
// weights arrive as K/4 vector loads. A row out of range gets weight 0 and is
// read from the zero row zrow, so its term is fma(0, 0, acc) = acc exactly
// (acc starts at +0 and never becomes -0); it is reported before the loads.
// Nothing but the indices, weights and accumulators is live across the K
// loads, which keeps the kernel at 32 registers: 2048 threads per SM.
template <int K, bool UNIT>
__global__ void __launch_bounds__(1024, 2)
combine_token_kernel(const uint4* __restrict__ y, const int32_t* __restrict__ dest_row,
                     const float* __restrict__ w, float4* __restrict__ out,
                     const uint4* __restrict__ zrow, int C, unsigned Q, int* err)
{
    static_assert(K == 4 || K == 8, "one token per CTA: K = 4 or 8");
    const int64_t n = blockIdx.x;
    const int c = threadIdx.x;
    int rows[K];
    float wk[K];
#pragma unroll
    for (int h = 0; h < K / 4; ++h) {
        const int4 r4 = __ldg(reinterpret_cast<const int4*>(dest_row + n * K) + h);
        rows[4 * h] = r4.x;
        rows[4 * h + 1] = r4.y;
        rows[4 * h + 2] = r4.z;
        rows[4 * h + 3] = r4.w;
        if (UNIT) {
            wk[4 * h] = wk[4 * h + 1] = wk[4 * h + 2] = wk[4 * h + 3] = 1.0f;
        } else {
            const float4 w4 = __ldg(reinterpret_cast<const float4*>(w + n * K) + h);
            wk[4 * h] = w4.x;
            wk[4 * h + 1] = w4.y;
            wk[4 * h + 2] = w4.z;
            wk[4 * h + 3] = w4.w;
        }
    }
    bool all_ok = true;
#pragma unroll
    for (int k = 0; k < K; ++k) {
        const bool ok = (unsigned)rows[k] < Q;
        all_ok &= ok;
        wk[k] = ok ? wk[k] : 0.0f;
    }
    if (!all_ok && c == 0) {
#pragma unroll
        for (int k = 0; k < K; ++k) {
            if ((unsigned)rows[k] >= Q) {
                raise_error(err, UE_ERR_DEVICE_BOUNDS, (int)min(n * K + k, (int64_t)INT_MAX));
                break;
            }
        }
    }
    uint4 v[K];
#pragma unroll
    for (int k = 0; k < K; ++k)
        v[k] = __ldcs(((unsigned)rows[k] < Q ? y + (int64_t)rows[k] * C : zrow) + c);
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
#pragma unroll
    for (int k = 0; k < K; ++k) {
        const uint32_t u[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            acc[2 * q] = fmaf(wk[k], __uint_as_float(u[q] << 16), acc[2 * q]);
            acc[2 * q + 1] = fmaf(wk[k], __uint_as_float(u[q] & 0xffff0000u), acc[2 * q + 1]);
        }
    }
    float4* dst = out + (n * C + c) * 2;
    __stcs(dst, make_float4(acc[0], acc[1], acc[2], acc[3]));
    __stcs(dst + 1, make_float4(acc[4], acc[5], acc[6], acc[7]));
}

template <int KMAX>
cudaError_t shape_k(const Sizes& z, int num_sms, CombineShape* out)
{
    const int C = z.d / 8;
    int tpt = 32;
    while (tpt < C && tpt < kCombineThreads) tpt <<= 1;
    const int tpb = kCombineThreads / tpt;
    int per_sm = 0;
    cudaError_t ce = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, combine_kernel<KMAX, false>,
                                                                   kCombineThreads, 0);
    if (ce != cudaSuccess) return ce;
    per_sm = std::max(per_sm, 1);
    const int64_t need = std::max<int64_t>(1, (z.N + tpb - 1) / tpb);
    out->grid = (int)std::min<int64_t>(need, (int64_t)num_sms * per_sm);
    out->tpt = tpt;
    return cudaSuccess;
}

}  // namespace

cudaError_t plan_combine_shape(const Sizes& z, int num_sms, CombineShape* out)
{
    const int C = z.d / 8;
    out->token = (z.K == 4 || z.K == 8) && C >= 128 && C <= 1024 ? 1 : 0;
    if (z.K <= 4) return shape_k<4>(z, num_sms, out);
    if (z.K <= 8) return shape_k<8>(z, num_sms, out);
    if (z.K <= 16) return shape_k<16>(z, num_sms, out);
    return shape_k<32>(z, num_sms, out);
}

cudaError_t launch_combine(const Sizes& z, const CombineShape& sh, const uint16_t* y,
                           const int32_t* dest_row, const float* w, float* out,
                           const uint16_t* zrow, int* err, cudaStream_t st)
{
    if (z.N == 0) return cudaSuccess;
    const bool unit = (w == nullptr);
    const bool vec_ok = (reinterpret_cast<uintptr_t>(dest_row) & 15u) == 0 &&
                        (unit || (reinterpret_cast<uintptr_t>(w) & 15u) == 0);
    if (sh.token && vec_ok && zrow != nullptr) {
        const int C = z.d / 8;
        const uint4* yv = reinterpret_cast<const uint4*>(y);
        float4* ov = reinterpret_cast<float4*>(out);
        const uint4* zv = reinterpret_cast<const uint4*>(zrow);
        const unsigned grid = (unsigned)z.N;
        const unsigned q32 = (unsigned)z.Q;  // Q < 2^31 (ue_init bounds it)
#define UE_COMBINE_TOKEN(KK)                                                                   \
    do {                                                                                       \
        if (unit)                                                                              \
            combine_token_kernel<KK, true><<<grid, C, 0, st>>>(yv, dest_row, w, ov, zv, C, q32, err); \
        else                                                                                   \
            combine_token_kernel<KK, false><<<grid, C, 0, st>>>(yv, dest_row, w, ov, zv, C, q32, err); \
    } while (0)
        if (z.K == 4) UE_COMBINE_TOKEN(4);
        else UE_COMBINE_TOKEN(8);
#undef UE_COMBINE_TOKEN
        return cudaGetLastError();
    }
#define UE_COMBINE(KM)                                                                         \
    do {                                                                                       \
        if (unit)                                                                              \
            combine_kernel<KM, true><<<sh.grid, kCombineThreads, 0, st>>>(                     \
                y, dest_row, w, out, z.N, z.K, z.d, sh.tpt, z.Q, err);                         \
        else                                                                                   \
            combine_kernel<KM, false><<<sh.grid, kCombineThreads, 0, st>>>(                    \
                y, dest_row, w, out, z.N, z.K, z.d, sh.tpt, z.Q, err);                         \
    } while (0)
    if (z.K <= 4) UE_COMBINE(4);
    else if (z.K <= 8) UE_COMBINE(8);
    else if (z.K <= 16) UE_COMBINE(16);
    else UE_COMBINE(32);
#undef UE_COMBINE
    return cudaGetLastError();
}

}  // namespace ue
