// k_combine.cu -- gate-weighted combine / unpermute.
//
// "UltraEP" README, "Interface / 2. Forward and backward": combine(recv_tokens)
// after the experts. out[n] = sum_{k=0..K-1} w[n][k] * y[dest_row[n*K+k]],
// fp32, one fused multiply-add per term in k order starting from 0.
//
// Design (B200): HBM-bound gather (2*K*d bytes read, 4*d written per token).
// A group of threads owns a token; each thread owns 16-byte chunks (8 bf16)
// of the row, issues all K chunk loads before the first FMA (K*16 bytes in
// flight per thread), widens bf16 to fp32 with shifts, and writes its 8 fp32
// results as two 16-byte streaming stores. Rows are read with evict-first
// hints since each expert row is used by exactly one token.
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
    if (z.K <= 4) return shape_k<4>(z, num_sms, out);
    if (z.K <= 8) return shape_k<8>(z, num_sms, out);
    if (z.K <= 16) return shape_k<16>(z, num_sms, out);
    return shape_k<32>(z, num_sms, out);
}

cudaError_t launch_combine(const Sizes& z, const CombineShape& sh, const uint16_t* y,
                           const int32_t* dest_row, const float* w, float* out, int* err,
                           cudaStream_t st)
{
    if (z.N == 0) return cudaSuccess;
    const bool unit = (w == nullptr);
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
