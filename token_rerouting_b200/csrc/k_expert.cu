// k_expert.cu -- weight sync to replica slots and gradient reduction to master
// experts, on one GPU.
//
// "UltraEP" README, "Interface / 2. Forward and backward": weight_sync
// materializes the replication plan by distributing master-expert weights to
// the replica slots; grad_reduce reduces replica Wgrad into the master
// experts' gradients. "Performance Tuning / Expert communication": the
// reduction is deterministic and non-atomic. "Interface / 1.
// Initialization": replica buffers live in redundant slots reused across
// layers; weights are bf16 (or fp8 with scales), gradients fp32.
//
// On one GPU both are HBM copies driven by the plan's slot_expert:
//   weight sync:    replicas[g] = master[slot_expert[g]] for every used slot
//   grad reduce:    master[e] = master[e] + replicas[g1] + replicas[g2] + ...
//                   over e's replica slots in ascending g, fp32, in that order
// Design (B200): 16-byte streaming loads and stores, four chunks in flight
// per thread, and CTAs that each copy or reduce one piece of 4096 16-byte
// chunks and exit. On Qwen3-235B-sized experts (128 slots over 107 experts)
// this moved 6.94 TB/s for the weight sync and 7.08 TB/s for the reduction,
// where grids of resident CTAs striding over the same pieces moved 6.1-6.4.
// The weight sync runs a 2-D grid (piece, slot); empty slots exit at once.
// The reduction first builds, in one small CTA, the list of experts that
// have replicas and each one's replica slots in ascending g (context
// scratch); then a 2-D grid (piece, list entry) reduces, and entries past
// the list's end exit at once. Each element is the master value plus the
// replicas added one by one in ascending g, so the result is the same on
// every run and for every launch shape.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kExpThreads = 256;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kExpThreads)
weight_sync_kernel(const int32_t* __restrict__ slot_expert, int E, const uint4* __restrict__ master,
                   uint4* __restrict__ replicas, int64_t n16, int* err)
{
    const int g = blockIdx.y;
    const int e = __ldg(slot_expert + g);
    if (e < 0) return;
    if (e >= E) {
        if (threadIdx.x == 0 && blockIdx.x == 0) raise_error(err, UE_ERR_DEVICE_BOUNDS, g);
        return;
    }
    const uint4* src = master + (int64_t)e * n16;
    uint4* dst = replicas + (int64_t)g * n16;
    const int64_t step = (int64_t)gridDim.x * blockDim.x * kUnroll;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x * kUnroll + threadIdx.x; base < n16;
         base += step) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = base + (int64_t)u * blockDim.x;
            if (i < n16) v[u] = __ldcs(src + i);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = base + (int64_t)u * blockDim.x;
            if (i < n16) __stcs(dst + i, v[u]);
        }
    }
}

// Scratch layout of the reduction tables (int32): list of replicated experts,
// first entry and count of each expert's replica slots, the slots by expert
// in ascending g, and the list's length.
constexpr int kGrList = 0;
constexpr int kGrFirst = kGrList + kMaxE;
constexpr int kGrCnt = kGrFirst + kMaxE;
constexpr int kGrReps = kGrCnt + kMaxE;
constexpr int kGrN = kGrReps + kMaxG;
static_assert(kGrN + 1 == kGrTableWords, "reduction table layout");

__global__ void __launch_bounds__(kExpThreads)
grad_reduce_setup_kernel(const int32_t* __restrict__ slot_expert, int G, int E,
                         int32_t* __restrict__ tab, int* err)
{
    __shared__ int s_cnt[kMaxE];      // replicas per expert
    __shared__ int s_start[kMaxE];    // next free entry of the expert in the slot list
    __shared__ int s_wsum[kExpThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < E; e += blockDim.x) s_cnt[e] = 0;
    __syncthreads();
    for (int g = tid; g < G; g += blockDim.x) {
        const int se = __ldg(slot_expert + g);
        if (se >= E) raise_error(err, UE_ERR_DEVICE_BOUNDS, g);
        else if (se >= 0) atomicAdd(&s_cnt[se], 1);
    }
    __syncthreads();
    {
        // exclusive scans over experts: replica entries, and replicated experts
        const int c = tid < E ? s_cnt[tid] : 0;
        int incl = c;
        const int has = c > 0;
        const unsigned hb = __ballot_sync(kFull, has);
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(kFull, incl, off);
            if (lane >= off) incl += o;
        }
        if (lane == 31) s_wsum[warp] = incl;
        __syncthreads();
        int wofs = 0;
        for (int w = 0; w < warp; ++w) wofs += s_wsum[w];
        if (tid < E) {
            s_start[tid] = wofs + incl - c;
            tab[kGrFirst + tid] = wofs + incl - c;
            tab[kGrCnt + tid] = c;
        }
        __syncthreads();
        if (lane == 0) s_wsum[warp] = __popc(hb);
        __syncthreads();
        int lofs = 0, ltot = 0;
        for (int w = 0; w < kExpThreads / 32; ++w) {
            if (w < warp) lofs += s_wsum[w];
            ltot += s_wsum[w];
        }
        if (has && tid < E) tab[kGrList + lofs + __popc(hb & ((1u << lane) - 1u))] = tid;
        if (tid == 0) tab[kGrN] = ltot;
        __syncthreads();
    }
    if (warp == 0) {
        // replica slots in ascending g within each expert
        for (int g0 = 0; g0 < G; g0 += 32) {
            const int g = g0 + lane;
            int e = -1;
            if (g < G) {
                e = __ldg(slot_expert + g);
                if (e >= E) e = -1;
            }
            const unsigned peers = __match_any_sync(kFull, e);
            if (e >= 0) tab[kGrReps + s_start[e] + __popc(peers & ((1u << lane) - 1u))] = g;
            __syncwarp();
            if (e >= 0 && lane == __ffs(peers) - 1) s_start[e] += __popc(peers);
            __syncwarp();
        }
    }
}

// blockIdx.y: entry of the replicated-expert list; blockIdx.x: piece of
// kExpThreads * kUnroll float4 of the expert
__global__ void __launch_bounds__(kExpThreads)
grad_reduce_kernel(const int32_t* __restrict__ tab, const float4* __restrict__ replicas,
                   float4* __restrict__ master, int64_t n4)
{
    const int y = blockIdx.y;
    if (y >= __ldg(tab + kGrN)) return;
    const int e = __ldg(tab + kGrList + y);
    const int first = __ldg(tab + kGrFirst + e);
    const int cnt = __ldg(tab + kGrCnt + e);
    const int64_t base = (int64_t)blockIdx.x * kExpThreads * kUnroll + threadIdx.x;
    float4 acc[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + (int64_t)u * kExpThreads;
        if (i < n4) acc[u] = master[(int64_t)e * n4 + i];
    }
    for (int j = 0; j < cnt; ++j) {
        const int64_t row = (int64_t)__ldg(tab + kGrReps + first + j) * n4;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = base + (int64_t)u * kExpThreads;
            if (i < n4) {
                const float4 r = __ldcs(replicas + row + i);
                acc[u].x += r.x;
                acc[u].y += r.y;
                acc[u].z += r.z;
                acc[u].w += r.w;
            }
        }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + (int64_t)u * kExpThreads;
        if (i < n4) master[(int64_t)e * n4 + i] = acc[u];
    }
}

int64_t pieces(int64_t units)
{
    const int64_t per_cta = (int64_t)kExpThreads * kUnroll;
    return (units + per_cta - 1) / per_cta;
}

}  // namespace

cudaError_t launch_weight_sync(const Sizes& z, const int32_t* slot_expert, const void* master,
                               void* replicas, int64_t bytes_per_expert, int num_sms, int* err,
                               cudaStream_t st)
{
    if (z.G == 0 || bytes_per_expert == 0) return cudaSuccess;
    (void)num_sms;
    const int64_t n16 = bytes_per_expert / 16;
    const dim3 grid((unsigned)pieces(n16), z.G);
    weight_sync_kernel<<<grid, kExpThreads, 0, st>>>(slot_expert, z.E,
                                                     reinterpret_cast<const uint4*>(master),
                                                     reinterpret_cast<uint4*>(replicas), n16, err);
    return cudaGetLastError();
}

cudaError_t launch_grad_reduce(const Sizes& z, const int32_t* slot_expert, const float* replicas,
                               float* master, int64_t numel_per_expert, int32_t* tables, int* err,
                               cudaStream_t st)
{
    if (z.G == 0 || numel_per_expert == 0) return cudaSuccess;
    grad_reduce_setup_kernel<<<1, kExpThreads, 0, st>>>(slot_expert, z.G, z.E, tables, err);
    cudaError_t ce = cudaGetLastError();
    if (ce != cudaSuccess) return ce;
    const int64_t n4 = numel_per_expert / 4;
    const dim3 grid((unsigned)pieces(n4), (unsigned)std::min(z.E, z.G));
    grad_reduce_kernel<<<grid, kExpThreads, 0, st>>>(tables,
                                                     reinterpret_cast<const float4*>(replicas),
                                                     reinterpret_cast<float4*>(master), n4);
    return cudaGetLastError();
}

}  // namespace ue
