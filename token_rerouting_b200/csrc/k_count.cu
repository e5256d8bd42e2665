// k_count.cu -- exact per-expert load: per-source-rank and total pair counts.
//
// "UltraEP" README intro: rebalancing uses the exact post-gating load;
// "Performance Tuning / NVSHMEM": each rank's load is gathered before
// planning. On one GPU the R simulated ranks' counts are produced directly
// as load_re[R][E]; load_e[E] is their sum.
//
// Design (B200): each CTA owns a chunk of one source rank's pairs and counts
// them in shared memory, one private histogram per warp so that a hot expert
// contends only within a warp; shared-memory atomics resolve the rest. Each
// CTA then adds its non-zero bins to global memory with one atomic per bin. The outputs are zeroed on the stream first. Integer atomics
// are exact, so the result does not depend on their order.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kCountThreads = 256;
constexpr int kCountWarps = kCountThreads / 32;
constexpr int kCountChunk = 2048;  // pairs per CTA

__global__ void __launch_bounds__(kCountThreads)
count_kernel(const int32_t* __restrict__ idx, int64_t TK, int E, int chunks_per_rank,
             int32_t* __restrict__ load_re, int32_t* __restrict__ load_e, int* err)
{
    __shared__ int hist[kCountWarps][kMaxE];  // one private histogram per warp
    const int r = blockIdx.x / chunks_per_rank;
    const int c = blockIdx.x - r * chunks_per_rank;
    const int64_t beg = (int64_t)r * TK + (int64_t)c * kCountChunk;
    const int64_t end = min((int64_t)(r + 1) * TK, beg + kCountChunk);
    const int warp = threadIdx.x >> 5;
    for (int x = threadIdx.x; x < kCountWarps * kMaxE; x += blockDim.x) (&hist[0][0])[x] = 0;
    __syncthreads();
    for (int64_t i = beg + threadIdx.x; i < end; i += blockDim.x) {
        const int e = __ldg(idx + i);
        if ((unsigned)e < (unsigned)E)
            atomicAdd(&hist[warp][e], 1);
        else
            raise_error(err, UE_ERR_DEVICE_BOUNDS, (int)min(i, (int64_t)INT_MAX));
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int h = 0;
#pragma unroll
        for (int w = 0; w < kCountWarps; ++w) h += hist[w][e];
        if (h) {
            atomicAdd(&load_re[(int64_t)r * E + e], h);
            atomicAdd(&load_e[e], h);
        }
    }
}

}  // namespace

cudaError_t launch_count(const Sizes& z, const int32_t* idx, int32_t* load_re,
                         int32_t* load_e, int* err, cudaStream_t st)
{
    cudaError_t ce = cudaMemsetAsync(load_re, 0, sizeof(int32_t) * (size_t)z.R * z.E, st);
    if (ce != cudaSuccess) return ce;
    ce = cudaMemsetAsync(load_e, 0, sizeof(int32_t) * (size_t)z.E, st);
    if (ce != cudaSuccess) return ce;
    const int64_t TK = (int64_t)z.T * z.K;
    if (TK == 0) return cudaSuccess;
    const int chunks = (int)((TK + kCountChunk - 1) / kCountChunk);
    count_kernel<<<z.R * chunks, kCountThreads, 0, st>>>(idx, TK, z.E, chunks, load_re, load_e,
                                                         err);
    return cudaGetLastError();
}

}  // namespace ue
