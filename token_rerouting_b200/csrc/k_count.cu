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
// CTA then adds its non-zero bins to the outputs with one global atomic per
// bin. Chunks of 4096 pairs give a few CTAs per SM (512 on the Qwen3-shaped
// layer), so the kernel's length is a few load and atomic latencies; each bin
// of load_e takes one atomic per CTA. Every thread issues all its loads
// before it counts. Integer sums are exact, so the result does not depend on
// the order of the additions.
//
// The outputs are zeroed inside the kernel, as in the gate with the count
// fused: the first CTA to take a ticket (which waits for nothing, so it
// always runs) zeroes them and then sets a flag carrying the launch epoch;
// every CTA waits for that flag (bounded) before its global atomics, and the
// last CTA to finish resets the ticket and advances the epoch. No memset
// precedes the launch.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kCountThreads = 512;
constexpr int kCountWarps = kCountThreads / 32;
constexpr int kCountChunk = 4096;  // pairs per CTA

constexpr long long kCountWaitLimit = 1LL << 22;

template <bool VEC>
__global__ void __launch_bounds__(kCountThreads)
count_kernel(const int32_t* __restrict__ idx, int64_t TK, int R, int E, int chunks_per_rank,
             int32_t* __restrict__ load_re, int32_t* __restrict__ load_e, uint32_t* sync,
             int* err)
{
    __shared__ int hist[kCountWarps][kMaxE];  // one private histogram per warp (16 KB)
    __shared__ uint32_t s_epoch, s_ticket, s_ok;
    if (threadIdx.x == 0) {
        s_epoch = *reinterpret_cast<volatile uint32_t*>(sync + 2);
        s_ticket = atomicAdd(sync, 1u);
    }
    const int r = blockIdx.x / chunks_per_rank;
    const int c = blockIdx.x - r * chunks_per_rank;
    const int64_t beg = (int64_t)r * TK + (int64_t)c * kCountChunk;
    const int n = (int)min((int64_t)kCountChunk, (int64_t)(r + 1) * TK - beg);
    const int warp = threadIdx.x >> 5;
    for (int x = threadIdx.x; x < kCountWarps * kMaxE; x += blockDim.x) (&hist[0][0])[x] = 0;
    __syncthreads();
    if (s_ticket == 0u) {
        // the first CTA zeroes the outputs, then sets the flag
        for (int x = threadIdx.x; x < R * E; x += blockDim.x) load_re[x] = 0;
        for (int x = threadIdx.x; x < E; x += blockDim.x) load_e[x] = 0;
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) st_release_gpu(sync + 3, s_epoch + 1u);
    }
    const int32_t* src = idx + beg;
    // issue all of this thread's loads before using any of them
    constexpr int kPer = kCountChunk / kCountThreads;
    int v[kPer];
    if (VEC) {
        // beg and n are multiples of 4 here: 16-byte loads
#pragma unroll
        for (int q = 0; q < kPer / 4; ++q) {
            const int x = 4 * (threadIdx.x + q * kCountThreads);
            int4 w4 = make_int4(-1, -1, -1, -1);
            if (x < n) w4 = __ldg(reinterpret_cast<const int4*>(src + x));
            v[4 * q] = w4.x;
            v[4 * q + 1] = w4.y;
            v[4 * q + 2] = w4.z;
            v[4 * q + 3] = w4.w;
        }
    } else {
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int x = threadIdx.x + q * kCountThreads;
            v[q] = x < n ? __ldg(src + x) : -1;
        }
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int x = VEC ? 4 * (threadIdx.x + (q / 4) * kCountThreads) + (q % 4)
                          : threadIdx.x + q * kCountThreads;
        if (x >= n) continue;
        const int e = v[q];
        if ((unsigned)e < (unsigned)E)
            atomicAdd(&hist[warp][e], 1);
        else
            raise_error(err, UE_ERR_DEVICE_BOUNDS, (int)min(beg + x, (int64_t)INT_MAX));
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t ok = 0u;
        for (long long spin = 0; spin < kCountWaitLimit; ++spin) {
            if (ld_acquire_gpu(sync + 3) == s_epoch + 1u) {
                ok = 1u;
                break;
            }
            __nanosleep(64);
        }
        if (!ok) raise_error(err, UE_ERR_TIMEOUT, (int)blockIdx.x);
        s_ok = ok;
    }
    __syncthreads();
    // add this CTA's bins to the outputs (zeroed by the first CTA)
    if (s_ok) {
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
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const uint32_t done = atomicAdd(sync + 1, 1u);
        if (done == gridDim.x - 1) {
            // last CTA: ready for the next launch
            sync[0] = 0u;
            sync[1] = 0u;
            __threadfence();
            sync[2] = s_epoch + 1u;
        }
    }
}

}  // namespace

cudaError_t launch_count(const Sizes& z, const int32_t* idx, int32_t* load_re,
                         int32_t* load_e, uint32_t* sync, int* err, cudaStream_t st)
{
    const int64_t TK = (int64_t)z.T * z.K;
    const int chunks = (int)std::max<int64_t>(1, (TK + kCountChunk - 1) / kCountChunk);
    const bool vec = (TK % 4 == 0) && ((uintptr_t)idx % 16 == 0);
    if (vec)
        count_kernel<true><<<z.R * chunks, kCountThreads, 0, st>>>(
            idx, TK, z.R, z.E, chunks, load_re, load_e, sync, err);
    else
        count_kernel<false><<<z.R * chunks, kCountThreads, 0, st>>>(
            idx, TK, z.R, z.E, chunks, load_re, load_e, sync, err);
    return cudaGetLastError();
}

}  // namespace ue
