// k_gate.cu -- router gating: per-token top-K experts and their gate weights.
//
// "UltraEP" README, "Interface / 2. Forward and backward": the router returns
// probs and routing_map; "What Happened" (aikit-app piece): routing from the
// exact routing probabilities. Selection rule: larger logit first, equal
// logits (IEEE ==, -0.0 == +0.0) to the lower expert id. Weights: softmax over
// the K selected logits, w_k = exp(v_k - v_0) / sum_j exp(v_j - v_0), in fp64,
// rounded once to fp32.
//
// Design (B200): one warp per row, the row's E logits spread over the lanes
// (expert e = lane + 32 j), read once with coalesced streaming loads. Each
// logit becomes an order-preserving 32-bit key; each lane keeps its keys in a
// small sorted list so that a round of the K-round selection is two warp
// `redux` reductions (max key, then min expert id among lanes holding it) and
// a pop. A warp handles 32/K rows at a time so that the fp64 exponentials of
// the weights use every lane. The kernel is bound by HBM reads of the logits
// (4*E bytes per token) plus the selection arithmetic.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kGateThreads = 256;
constexpr int kGateBatch = 4;  // rows whose logits are loaded ahead

// Order-preserving map of a finite float to uint32 (larger float -> larger
// key). -0.0 is mapped like +0.0 so that the two tie. 0 is never produced for
// a finite input, so it marks "taken" or "absent".
__device__ __forceinline__ uint32_t order_key(float v)
{
    uint32_t u = __float_as_uint(v);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t k)
{
    const uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// Selection of one row's top-K from the lane's VPL logits (expert ids
// lane + 32 j); lane (base + k) records round k's winner.
template <int VPL, int KT>
__device__ __forceinline__ void select_row(const float (&v)[VPL], int E, int K, int base,
                                           int lane, uint32_t& cap_key, uint32_t& cap_e)
{
    uint32_t key[VPL];
    uint32_t ke[VPL];
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
        const int e = lane + 32 * j;
        key[j] = (e < E) ? order_key(v[j]) : 0u;
        ke[j] = (uint32_t)e;
    }
    // stable descending sort of the lane's keys; ids ascend with j, so equal
    // keys keep the lower id first
#pragma unroll
    for (int pass = 0; pass < VPL - 1; ++pass) {
#pragma unroll
        for (int j = 0; j < VPL - 1 - pass; ++j) {
            const bool sw = key[j + 1] > key[j];
            const uint32_t k0 = key[j], k1 = key[j + 1];
            const uint32_t e0 = ke[j], e1 = ke[j + 1];
            key[j] = sw ? k1 : k0;
            key[j + 1] = sw ? k0 : k1;
            ke[j] = sw ? e1 : e0;
            ke[j + 1] = sw ? e0 : e1;
        }
    }
    constexpr int KU = KT > 0 ? KT : kMaxK;
#pragma unroll
    for (int k = 0; k < KU; ++k) {
        if (KT == 0 && k >= K) break;
        const uint32_t m = __reduce_max_sync(kFull, key[0]);
        const uint32_t cand = (key[0] == m) ? ke[0] : 0xffffffffu;
        const uint32_t ew = __reduce_min_sync(kFull, cand);
        if (lane == base + k) {
            cap_key = m;
            cap_e = ew;
        }
        const bool pop = (ke[0] == ew);
#pragma unroll
        for (int j = 0; j < VPL - 1; ++j) {
            key[j] = pop ? key[j + 1] : key[j];
            ke[j] = pop ? ke[j + 1] : ke[j];
        }
        if (pop) {
            key[VPL - 1] = 0u;
            ke[VPL - 1] = 0xfffffffeu;
        }
    }
}

// KT > 0: K == KT at compile time; KT == 0: any K <= 32.
template <int VPL, int KT>
__global__ void __launch_bounds__(kGateThreads)
gate_topk_kernel(const float* __restrict__ logits, int64_t N, int E, int Krt,
                 int32_t* __restrict__ idx, float* __restrict__ w)
{
    const int K = KT > 0 ? KT : Krt;
    const int rpg = 32 / K;  // rows per warp group
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t ngroups = (N + rpg - 1) / rpg;

    for (int64_t grp = gwarp; grp < ngroups; grp += nwarps) {
        const int64_t row0 = grp * rpg;
        const int rows = (int)min((int64_t)rpg, N - row0);
        // lane L records round (L % K) of row (L / K) of the group
        uint32_t cap_key = 0u;
        uint32_t cap_e = 0u;

        for (int rb = 0; rb < rows; rb += kGateBatch) {
            float v[kGateBatch][VPL];
#pragma unroll
            for (int b = 0; b < kGateBatch; ++b) {
                const bool rowok = rb + b < rows;
                const float* src = logits + (row0 + rb + b) * (int64_t)E;
#pragma unroll
                for (int j = 0; j < VPL; ++j) {
                    const int e = lane + 32 * j;
                    v[b][j] = (rowok && e < E) ? __ldcs(src + e) : 0.0f;
                }
            }
            if (rb + kGateBatch <= rows) {
                // full batch: no row-count branches, consecutive rows interleave
#pragma unroll
                for (int b = 0; b < kGateBatch; ++b)
                    select_row<VPL, KT>(v[b], E, K, (rb + b) * K, lane, cap_key, cap_e);
            } else {
#pragma unroll
                for (int b = 0; b < kGateBatch; ++b)
                    if (rb + b < rows)
                        select_row<VPL, KT>(v[b], E, K, (rb + b) * K, lane, cap_key, cap_e);
            }
        }

        // gate weights of the whole group at once, fp64
        const int r = lane / K;
        const int k = lane - r * K;
        const bool act = r < rows;
        const int lead = act ? r * K : 0;
        const double v_own = (double)key_value(cap_key);
        const double v0 = __shfl_sync(kFull, v_own, lead);
        const double x = act ? exp(v_own - v0) : 0.0;
        double z = 0.0;
        constexpr int KU = KT > 0 ? KT : kMaxK;
#pragma unroll
        for (int kk = 0; kk < KU; ++kk) {
            if (KT == 0 && kk >= K) break;
            z += __shfl_sync(kFull, x, act ? lead + kk : 0);
        }
        if (act) {
            const int64_t pos = (row0 + r) * (int64_t)K + k;
            idx[pos] = (int32_t)cap_e;
            w[pos] = (float)(x / z);
        }
    }
}

template <int VPL>
cudaError_t launch_vpl(const Sizes& z, const float* logits, int32_t* idx,
                       float* w, int grid, cudaStream_t st)
{
    if (z.K == 8)
        gate_topk_kernel<VPL, 8><<<grid, kGateThreads, 0, st>>>(logits, z.N, z.E, z.K, idx, w);
    else if (z.K == 4)
        gate_topk_kernel<VPL, 4><<<grid, kGateThreads, 0, st>>>(logits, z.N, z.E, z.K, idx, w);
    else
        gate_topk_kernel<VPL, 0><<<grid, kGateThreads, 0, st>>>(logits, z.N, z.E, z.K, idx, w);
    return cudaGetLastError();
}

}  // namespace

int gate_topk_grid(const Sizes& z, int num_sms)
{
    const int rpg = 32 / z.K;
    const int64_t groups = (z.N + rpg - 1) / rpg;
    const int64_t blocks_needed = (groups + (kGateThreads / 32) - 1) / (kGateThreads / 32);
    const int64_t cap = (int64_t)num_sms * 4;
    return (int)std::max<int64_t>(1, std::min(blocks_needed, cap));
}

cudaError_t launch_gate_topk(const Sizes& z, const float* logits, int32_t* idx,
                             float* w, int grid, cudaStream_t st)
{
    if (z.N == 0) return cudaSuccess;
    switch ((z.E + 31) / 32) {
    case 1: return launch_vpl<1>(z, logits, idx, w, grid, st);
    case 2: return launch_vpl<2>(z, logits, idx, w, grid, st);
    case 3: return launch_vpl<3>(z, logits, idx, w, grid, st);
    case 4: return launch_vpl<4>(z, logits, idx, w, grid, st);
    case 5: return launch_vpl<5>(z, logits, idx, w, grid, st);
    case 6: return launch_vpl<6>(z, logits, idx, w, grid, st);
    case 7: return launch_vpl<7>(z, logits, idx, w, grid, st);
    case 8: return launch_vpl<8>(z, logits, idx, w, grid, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace ue
