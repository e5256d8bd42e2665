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

// ---------------------------------------------------------------------------
// Fast path for K = 8 and E = 32 * VPL, VPL in {4, 8} (E = 128 or 256).
//
// Each logit's order key keeps its high bits and carries (E-1-e) in its low
// log2(E) bits, so keys are unique within a row and a round of the selection
// is one `redux` max and a pop. The packed order is the exact order (larger
// value first, lower id first among equal values) wherever the values differ
// above the dropped bits. A (K+1)-th round checks exactly that: if the first
// K+1 packed picks of a row differ pairwise in their high parts (adjacent
// ones suffice: they are sorted), every unpicked key lies strictly below the
// K-th pick, and the picks are in exact order. Rows that fail the check (two
// of the leading values within 2^-16 relative of each other, or exact ties)
// are selected again with full keys and the id tie rule from the copy of the
// row staged in shared memory. The results are identical to the generic
// kernel's in every case.
//
// Lane l holds experts e = 128 c + 4 l + j (chunk c < VPL/4, j < 4): one
// 16-byte load per chunk, ids ascending along the lane's list.
constexpr int kFastK = 8;
constexpr int kFastRows = 32 / kFastK;  // rows per warp group
constexpr int kGateWarps = kGateThreads / 32;

// Order key of a finite float with -0.0 made +0.0 first (the sum -0 + +0 is
// +0 under round-to-nearest; finite inputs are otherwise unchanged).
__device__ __forceinline__ uint32_t order_key_finite(float v)
{
    const uint32_t u = __float_as_uint(__fadd_rn(v, 0.0f));
    return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
}

__device__ __forceinline__ void cas_desc(uint32_t& a, uint32_t& b)
{
    const uint32_t hi = max(a, b), lo = min(a, b);
    a = hi;
    b = lo;
}

// descending sort of distinct keys by a sorting network (5 or 19 comparators)
template <int VPL>
__device__ __forceinline__ void sort_desc(uint32_t (&k)[VPL])
{
    if constexpr (VPL == 4) {
        cas_desc(k[0], k[1]); cas_desc(k[2], k[3]);
        cas_desc(k[0], k[2]); cas_desc(k[1], k[3]);
        cas_desc(k[1], k[2]);
    } else {
        static_assert(VPL == 8, "fast gate path: VPL 4 or 8");
        cas_desc(k[0], k[1]); cas_desc(k[2], k[3]); cas_desc(k[4], k[5]); cas_desc(k[6], k[7]);
        cas_desc(k[0], k[2]); cas_desc(k[1], k[3]); cas_desc(k[4], k[6]); cas_desc(k[5], k[7]);
        cas_desc(k[1], k[2]); cas_desc(k[5], k[6]);
        cas_desc(k[0], k[4]); cas_desc(k[1], k[5]); cas_desc(k[2], k[6]); cas_desc(k[3], k[7]);
        cas_desc(k[2], k[4]); cas_desc(k[3], k[5]);
        cas_desc(k[1], k[2]); cas_desc(k[3], k[4]); cas_desc(k[5], k[6]);
    }
}

// The K+1 packed picks of one row into win[0..K]; lane 0 writes them.
template <int VPL>
__device__ __forceinline__ void select_packed(const float4 (&v)[VPL / 4], const uint32_t (&lo)[VPL],
                                              uint32_t* win, bool writer)
{
    constexpr int LOB = VPL == 4 ? 7 : 8;
    constexpr uint32_t kHi = ~((1u << LOB) - 1u);
    uint32_t key[VPL];
#pragma unroll
    for (int c = 0; c < VPL / 4; ++c) {
        key[4 * c + 0] = (order_key_finite(v[c].x) & kHi) | lo[4 * c + 0];
        key[4 * c + 1] = (order_key_finite(v[c].y) & kHi) | lo[4 * c + 1];
        key[4 * c + 2] = (order_key_finite(v[c].z) & kHi) | lo[4 * c + 2];
        key[4 * c + 3] = (order_key_finite(v[c].w) & kHi) | lo[4 * c + 3];
    }
    sort_desc<VPL>(key);
#pragma unroll
    for (int k = 0; k < kFastK; ++k) {
        const uint32_t m = __reduce_max_sync(kFull, key[0]);
        if (writer) win[k] = m;
        const bool pop = key[0] == m;
#pragma unroll
        for (int j = 0; j < VPL - 1; ++j) key[j] = pop ? key[j + 1] : key[j];
        key[VPL - 1] = pop ? 0u : key[VPL - 1];
    }
    const uint32_t m = __reduce_max_sync(kFull, key[0]);
    if (writer) win[kFastK] = m;
}

// Exact selection of one staged row: full keys, equal keys to the lower id.
// win[k] = E-1-e_k, which decodes like a packed pick.
template <int VPL>
__device__ __forceinline__ void select_exact_staged(const float4* row, int lane, uint32_t* win)
{
    constexpr int E = 32 * VPL;
    uint32_t key[VPL], ke[VPL];
#pragma unroll
    for (int c = 0; c < VPL / 4; ++c) {
        const float4 x = row[c * 32 + lane];
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            key[4 * c + j] = order_key_finite(xs[j]);
            ke[4 * c + j] = (uint32_t)(128 * c + 4 * lane + j);
        }
    }
    // stable descending bubble sort: equal keys keep the lower id first
#pragma unroll
    for (int pass = 0; pass < VPL - 1; ++pass) {
#pragma unroll
        for (int j = 0; j < VPL - 1 - pass; ++j) {
            const bool sw = key[j + 1] > key[j];
            const uint32_t k0 = key[j], k1 = key[j + 1], e0 = ke[j], e1 = ke[j + 1];
            key[j] = sw ? k1 : k0;
            key[j + 1] = sw ? k0 : k1;
            ke[j] = sw ? e1 : e0;
            ke[j + 1] = sw ? e0 : e1;
        }
    }
#pragma unroll
    for (int k = 0; k < kFastK; ++k) {
        const uint32_t m = __reduce_max_sync(kFull, key[0]);
        const uint32_t ew = __reduce_min_sync(kFull, key[0] == m ? ke[0] : 0xffffffffu);
        if (lane == 0) win[k] = (uint32_t)(E - 1) - ew;
        const bool pop = ke[0] == ew;
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

template <int VPL>
__global__ void __launch_bounds__(kGateThreads, 4)
gate_topk_fast_kernel(const float* __restrict__ logits, int64_t N, int32_t* __restrict__ idx,
                      float* __restrict__ w)
{
    constexpr int E = 32 * VPL;
    constexpr int NCH = VPL / 4;
    constexpr int LOB = VPL == 4 ? 7 : 8;
    constexpr uint32_t kLo = (1u << LOB) - 1u;
    __shared__ float4 s_row[kGateWarps][kFastRows][E / 4];
    __shared__ uint32_t s_win[kGateWarps][kFastRows][kFastK + 1];

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t gwarp = (int64_t)blockIdx.x * kGateWarps + warp;
    const int64_t nwarps = (int64_t)gridDim.x * kGateWarps;
    const int64_t ngroups = (N + kFastRows - 1) / kFastRows;
    uint32_t lo[VPL];
#pragma unroll
    for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int j = 0; j < 4; ++j) lo[4 * c + j] = (uint32_t)(E - 1 - (128 * c + 4 * lane + j));
    const int r = lane / kFastK;   // this lane's row of the group in the epilogue
    const int k = lane % kFastK;   // and its rank among the row's picks

    for (int64_t grp = gwarp; grp < ngroups; grp += nwarps) {
        const int64_t row0 = grp * kFastRows;
        const int rows = (int)min((int64_t)kFastRows, N - row0);
        float4 v[kFastRows][NCH];
#pragma unroll
        for (int b = 0; b < kFastRows; ++b) {
            const float4* src = reinterpret_cast<const float4*>(logits + (row0 + b) * (int64_t)E);
#pragma unroll
            for (int c = 0; c < NCH; ++c)
                v[b][c] = b < rows ? __ldcs(src + c * 32 + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int b = 0; b < kFastRows; ++b)
#pragma unroll
            for (int c = 0; c < NCH; ++c) s_row[warp][b][c * 32 + lane] = v[b][c];
        if (rows == kFastRows) {
#pragma unroll
            for (int b = 0; b < kFastRows; ++b)
                select_packed<VPL>(v[b], lo, s_win[warp][b], lane == 0);
        } else {
#pragma unroll
            for (int b = 0; b < kFastRows; ++b)
                if (b < rows) select_packed<VPL>(v[b], lo, s_win[warp][b], lane == 0);
        }
        __syncwarp();
        // rows whose leading picks agree above the dropped bits: exact again
        const bool act = r < rows;
        const uint32_t a = s_win[warp][r][k];
        const uint32_t nx = s_win[warp][r][k + 1];
        unsigned redo = __ballot_sync(kFull, act && (a >> LOB) == (nx >> LOB));
        while (redo) {
            const int rr = (__ffs(redo) - 1) / kFastK;
            select_exact_staged<VPL>(s_row[warp][rr], lane, s_win[warp][rr]);
            redo &= ~(0xffu << (rr * kFastK));
        }
        __syncwarp();
        // gate weights of the whole group at once, fp64
        const uint32_t e = (uint32_t)(E - 1) - (s_win[warp][r][k] & kLo);
        const float vf = reinterpret_cast<const float*>(s_row[warp][r])[e];
        const int lead = act ? r * kFastK : 0;
        const double v_own = (double)vf;
        const double v0 = __shfl_sync(kFull, v_own, lead);
        const double x = act ? exp(v_own - v0) : 0.0;
        double z = 0.0;
#pragma unroll
        for (int kk = 0; kk < kFastK; ++kk) z += __shfl_sync(kFull, x, act ? lead + kk : 0);
        if (act) {
            const int64_t pos = (row0 + r) * (int64_t)kFastK + k;
            idx[pos] = (int32_t)e;
            w[pos] = (float)(x / z);
        }
        __syncwarp();  // the staged rows and picks are rewritten by the next group
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
    if (z.K == kFastK && (reinterpret_cast<uintptr_t>(logits) & 15u) == 0) {
        if (z.E == 128) {
            gate_topk_fast_kernel<4><<<grid, kGateThreads, 0, st>>>(logits, z.N, idx, w);
            return cudaGetLastError();
        }
        if (z.E == 256) {
            gate_topk_fast_kernel<8><<<grid, kGateThreads, 0, st>>>(logits, z.N, idx, w);
            return cudaGetLastError();
        }
    }
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
