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
// Fast path for K = 8 and E = 128 * NCH4 + 32 * NT (a multiple of 32, 64 to
// 256), optionally with the exact histogram fused in.
//
// Each logit's order key keeps its high bits and carries (E-1-e) in its low
// LOB bits (7 for E <= 128, 8 above), so keys are unique within a row and a
// round of the selection is one `redux` max and a pop. The packed order is
// the exact order (larger value first, lower id first among equal values)
// wherever the values differ above the dropped bits. A (K+1)-th round checks
// exactly that: if the first K+1 packed picks of a row differ pairwise in
// their high parts (adjacent ones suffice: they are sorted), every unpicked
// key lies strictly below the K-th pick, and the picks are in exact order.
// Each lane pops from a list of its three largest keys only (select_packed);
// a lane that gives up its whole list shows up as two equal adjacent picks.
// Rows that fail the check (two of the leading values within 2^-16 relative
// of each other, exact ties, or a lane holding three or more of the first K
// picks) are selected again with full keys and the id tie rule, from the row
// read again (an L1 hit: the loads allocate in L1). The results are
// identical to the generic kernel's in every case.
//
// Lane l holds experts e = 128 c + 4 l + j (chunk c < NCH4, j < 4: one
// 16-byte load per chunk) and then 128 NCH4 + 32 t + l (t < NT: one 4-byte
// load each), ids ascending along the lane's list.
//
// Each CTA owns a contiguous block of rows, so with the count fused it
// touches only a few source ranks: each pick is added to a shared histogram
// per source rank, and the CTA adds its non-zero bins to load_re and load_e
// at the end. The outputs are zeroed by the first CTA to take a ticket
// (which waits for nothing, so it always runs), which then sets a flag;
// every CTA waits for that flag (bounded) before its global atomics. The
// flag carries the launch epoch, and the last CTA to finish resets the
// ticket and advances the epoch, so nothing is cleared between launches.
constexpr int kFastK = 8;
constexpr int kFastRows = 32 / kFastK;  // rows per warp group
constexpr int kGateWarps = kGateThreads / 32;
constexpr int kGateHist = 4;            // source ranks one CTA may touch (fused count)
constexpr long long kGateWaitLimit = 1LL << 22;

// packed key: order key of the finite float v (-0.0 made +0.0 first; the sum
// -0 + +0 is +0 under round-to-nearest) with its low bits replaced by lo:
// x = u ^ (s & 0x7fffffff) ^ 0x80000000 with s the sign mask (lop3 0x1e),
// then (x & khi) | lo (lop3 0xea)
__device__ __forceinline__ uint32_t packed_key(float v, uint32_t lo, uint32_t khi)
{
    const uint32_t u = __float_as_uint(__fadd_rn(v, 0.0f));
    const uint32_t sgn = (uint32_t)((int32_t)u >> 31);
    uint32_t x, k;
    asm("lop3.b32 %0, %1, %2, 0x80000000, 0x1e;" : "=r"(x) : "r"(u), "r"(sgn));
    asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(k) : "r"(x), "r"(khi), "r"(lo));
    return k;
}

// full order key of a finite float (-0.0 made +0.0 first)
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

// descending sort of distinct keys by a sorting network
template <int VPL>
__device__ __forceinline__ void sort_desc(uint32_t (&k)[VPL])
{
    if constexpr (VPL == 2) {
        cas_desc(k[0], k[1]);
    } else if constexpr (VPL == 3) {
        cas_desc(k[0], k[1]); cas_desc(k[1], k[2]); cas_desc(k[0], k[1]);
    } else if constexpr (VPL == 4) {
        cas_desc(k[0], k[1]); cas_desc(k[2], k[3]);
        cas_desc(k[0], k[2]); cas_desc(k[1], k[3]);
        cas_desc(k[1], k[2]);
    } else if constexpr (VPL == 5) {
        cas_desc(k[0], k[1]); cas_desc(k[3], k[4]); cas_desc(k[2], k[4]);
        cas_desc(k[2], k[3]); cas_desc(k[0], k[3]); cas_desc(k[0], k[2]);
        cas_desc(k[1], k[4]); cas_desc(k[1], k[3]); cas_desc(k[1], k[2]);
    } else if constexpr (VPL == 6) {
        cas_desc(k[1], k[2]); cas_desc(k[4], k[5]); cas_desc(k[0], k[2]);
        cas_desc(k[3], k[5]); cas_desc(k[0], k[1]); cas_desc(k[3], k[4]);
        cas_desc(k[2], k[5]); cas_desc(k[0], k[3]); cas_desc(k[1], k[4]);
        cas_desc(k[2], k[4]); cas_desc(k[1], k[3]); cas_desc(k[2], k[3]);
    } else if constexpr (VPL == 7) {
        cas_desc(k[1], k[2]); cas_desc(k[3], k[4]); cas_desc(k[5], k[6]);
        cas_desc(k[0], k[2]); cas_desc(k[3], k[5]); cas_desc(k[4], k[6]);
        cas_desc(k[0], k[1]); cas_desc(k[4], k[5]); cas_desc(k[2], k[6]);
        cas_desc(k[0], k[4]); cas_desc(k[1], k[5]); cas_desc(k[0], k[3]);
        cas_desc(k[2], k[5]); cas_desc(k[1], k[3]); cas_desc(k[2], k[4]);
        cas_desc(k[2], k[3]);
    } else {
        static_assert(VPL == 8, "fast gate path: 2 to 8 values per lane");
        cas_desc(k[0], k[1]); cas_desc(k[2], k[3]); cas_desc(k[4], k[5]); cas_desc(k[6], k[7]);
        cas_desc(k[0], k[2]); cas_desc(k[1], k[3]); cas_desc(k[4], k[6]); cas_desc(k[5], k[7]);
        cas_desc(k[1], k[2]); cas_desc(k[5], k[6]);
        cas_desc(k[0], k[4]); cas_desc(k[1], k[5]); cas_desc(k[2], k[6]); cas_desc(k[3], k[7]);
        cas_desc(k[2], k[4]); cas_desc(k[3], k[5]);
        cas_desc(k[1], k[2]); cas_desc(k[3], k[4]); cas_desc(k[5], k[6]);
    }
}

// descending sort of four distinct keys held anywhere
__device__ __forceinline__ void sort4_desc(uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d)
{
    cas_desc(a, b); cas_desc(c, d);
    cas_desc(a, c); cas_desc(b, d);
    cas_desc(b, c);
}

// The D largest of VPL distinct keys into k[0..D-1], descending (the rest of
// k is left unspecified). D >= VPL sorts the whole list; otherwise the first
// four are sorted and the others merged in: two sorted quadruples through
// the max of opposite ends (the top D of both, a bitonic sequence, then
// sorted), single keys by insertion at the bottom of the top D.
template <int VPL, int D>
__device__ __forceinline__ void top_desc(uint32_t (&k)[VPL])
{
    if constexpr (D >= VPL || VPL == 4) {
        sort_desc<VPL>(k);
    } else if constexpr (VPL == 8) {
        static_assert(D == 3 || D == 4, "fast gate path: list depth 3 or 4");
        sort4_desc(k[0], k[1], k[2], k[3]);
        sort4_desc(k[4], k[5], k[6], k[7]);
#pragma unroll
        for (int i = 0; i < D; ++i) k[i] = max(k[i], k[4 + D - 1 - i]);
        if constexpr (D == 4) {
            cas_desc(k[0], k[2]); cas_desc(k[1], k[3]);
            cas_desc(k[0], k[1]); cas_desc(k[2], k[3]);
        } else {
            cas_desc(k[0], k[1]); cas_desc(k[1], k[2]); cas_desc(k[0], k[1]);
        }
    } else {
        static_assert(VPL > 4 && VPL < 8 && (D == 3 || D == 4),
                      "fast gate path: list depth 3 or 4");
        sort4_desc(k[0], k[1], k[2], k[3]);
#pragma unroll
        for (int i = 4; i < VPL; ++i) {
            k[D - 1] = max(k[D - 1], k[i]);
#pragma unroll
            for (int j = D - 1; j > 0; --j) cas_desc(k[j - 1], k[j]);
        }
    }
}

template <int NCH4, int NT>
struct FastRow {
    float4 c4[NCH4 > 0 ? NCH4 : 1];
    float t1[NT > 0 ? NT : 1];

    __device__ __forceinline__ void load(const float* row, int lane, bool ok)
    {
#pragma unroll
        for (int c = 0; c < NCH4; ++c)
            c4[c] = ok ? __ldg(reinterpret_cast<const float4*>(row) + c * 32 + lane)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int t = 0; t < NT; ++t) t1[t] = ok ? __ldg(row + 128 * NCH4 + 32 * t + lane) : 0.f;
    }
    __device__ __forceinline__ float at(int i) const
    {
        if (i < 4 * NCH4) {
            const float4 x = c4[i >> 2];
            const int j = i & 3;
            return j == 0 ? x.x : j == 1 ? x.y : j == 2 ? x.z : x.w;
        }
        return t1[i - 4 * NCH4];
    }
};

// expert id held in position i of lane `lane`'s list
template <int NCH4>
__device__ __forceinline__ int fast_expert(int i, int lane)
{
    return i < 4 * NCH4 ? 128 * (i >> 2) + 4 * lane + (i & 3) : 128 * NCH4 + 32 * (i - 4 * NCH4) + lane;
}

// Depth of the per-lane lists of the packed selection: every key when a
// lane holds at most three, else the three largest.
__host__ __device__ constexpr int fast_depth(int vpl) { return vpl < 3 ? vpl : 3; }

// The K+1 packed picks of one row into win[0..K]; the lane holding a pick
// writes it (keys are distinct within a row, so exactly one lane does, and
// the pick stays in a vector register). Each lane keeps its D largest keys,
// sorted, and a pop shifts the list up.
// With at most three keys a lane (D = VPL) the pop fills the bottom with 0,
// which never wins, and every pick is exact. Otherwise the pop leaves the
// last entry in place: a lane that gives up all D keys before the last round
// then offers its last key again, which is the largest key left in the row
// and is picked again at once. Those two equal adjacent picks send the row to
// the exact selection (the caller checks adjacent picks); without them every
// pick is exact, since a lane's keys below its list lie below its last entry.
template <int NCH4, int NT>
__device__ __forceinline__ void select_packed(const FastRow<NCH4, NT>& v,
                                              const uint32_t (&lo)[4 * NCH4 + NT], uint32_t khi,
                                              uint32_t* win)
{
    constexpr int VPL = 4 * NCH4 + NT;
    constexpr int D = fast_depth(VPL);
    constexpr bool kFill = VPL < 4;
    uint32_t key[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) key[i] = packed_key(v.at(i), lo[i], khi);
    top_desc<VPL, D>(key);
#pragma unroll
    for (int k = 0; k < kFastK; ++k) {
        const uint32_t m = __reduce_max_sync(kFull, key[0]);
        const bool pop = key[0] == m;
        if (pop) win[k] = key[0];
#pragma unroll
        for (int j = 0; j < D - 1; ++j) key[j] = pop ? key[j + 1] : key[j];
        if constexpr (kFill) key[D - 1] = pop ? 0u : key[D - 1];
    }
    const uint32_t m = __reduce_max_sync(kFull, key[0]);
    if (key[0] == m) win[kFastK] = key[0];
}

// Exact selection of one row read again from global memory: full keys,
// equal keys to the lower id. win[k] = E-1-e_k, which decodes like a packed
// pick.
template <int NCH4, int NT>
__device__ __forceinline__ void select_exact_row(const float* row, int lane, uint32_t* win)
{
    constexpr int VPL = 4 * NCH4 + NT;
    constexpr int E = 128 * NCH4 + 32 * NT;
    FastRow<NCH4, NT> v;
    v.load(row, lane, true);
    uint32_t key[VPL], ke[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        key[i] = order_key_finite(v.at(i));
        ke[i] = (uint32_t)fast_expert<NCH4>(i, lane);
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

template <int NCH4, int NT, bool COUNT>
__global__ void __launch_bounds__(kGateThreads, 4)
gate_topk_fast_kernel(const float* __restrict__ logits, int64_t N, int64_t rows_per_cta,
                      int32_t* __restrict__ idx, float* __restrict__ w, GateCount cnt)
{
    constexpr int VPL = 4 * NCH4 + NT;
    constexpr int E = 128 * NCH4 + 32 * NT;
    constexpr int LOB = E <= 128 ? 7 : 8;
    constexpr uint32_t kLo = (1u << LOB) - 1u;
    constexpr uint32_t kHi = ~kLo;
    constexpr int HE = COUNT ? E : 1;
    __shared__ uint32_t s_win[kGateWarps][kFastRows][kFastK + 1];
    __shared__ int s_hist[COUNT ? kGateHist : 1][HE];
    __shared__ uint32_t s_epoch, s_ticket, s_ok;

    // row indices fit 32 bits here: K = 8 and Q < 2^30 give N < 2^27
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int row_beg = (int)blockIdx.x * (int)rows_per_cta;
    const int row_end = (int)min(N, (int64_t)row_beg + rows_per_cta);
    int rank0 = 0;
    int bnd[kGateHist - 1] = {};  // first rows of the source ranks after rank0
    if constexpr (COUNT) {
        for (int x = threadIdx.x; x < kGateHist * E; x += blockDim.x) (&s_hist[0][0])[x] = 0;
        if (threadIdx.x == 0) {
            s_epoch = *reinterpret_cast<volatile uint32_t*>(cnt.sync + 2);
            s_ticket = atomicAdd(cnt.sync, 1u);
        }
        __syncthreads();
        if (s_ticket == 0u) {
            // the first CTA zeroes the outputs, then sets the flag
            const int re = cnt.R * E;
            for (int x = threadIdx.x; x < re; x += blockDim.x) cnt.load_re[x] = 0;
            for (int x = threadIdx.x; x < E; x += blockDim.x) cnt.load_e[x] = 0;
            __threadfence();
            __syncthreads();
            if (threadIdx.x == 0) st_release_gpu(cnt.sync + 3, s_epoch + 1u);
        }
        rank0 = row_beg / cnt.T;
#pragma unroll
        for (int q = 1; q < kGateHist; ++q) bnd[q - 1] = (rank0 + q) * cnt.T;
    }

    uint32_t lo[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) lo[i] = (uint32_t)(E - 1 - fast_expert<NCH4>(i, lane));
    const int r = lane / kFastK;   // this lane's row of the group in the epilogue
    const int k = lane % kFastK;   // and its rank among the row's picks

    for (int row0 = row_beg + warp * kFastRows; row0 < row_end; row0 += kGateWarps * kFastRows) {
        const int rows = min(kFastRows, row_end - row0);
        const float* grp_rows = logits + (size_t)row0 * E;
        FastRow<NCH4, NT> v[kFastRows];
        if (rows == kFastRows) {
#pragma unroll
            for (int b = 0; b < kFastRows; ++b) v[b].load(grp_rows + b * E, lane, true);
#pragma unroll
            for (int b = 0; b < kFastRows; ++b)
                select_packed<NCH4, NT>(v[b], lo, kHi, s_win[warp][b]);
        } else {
            // the last group of the CTA: rows past its end read the last row
#pragma unroll
            for (int b = 0; b < kFastRows; ++b)
                v[b].load(grp_rows + min(b, rows - 1) * E, lane, true);
#pragma unroll
            for (int b = 0; b < kFastRows; ++b)
                if (b < rows) select_packed<NCH4, NT>(v[b], lo, kHi, s_win[warp][b]);
        }
        __syncwarp();
        // rows whose leading picks agree above the dropped bits: exact again
        const bool act = r < rows;
        const uint32_t a = s_win[warp][r][k];
        const uint32_t nx = s_win[warp][r][k + 1];
        unsigned redo = __ballot_sync(kFull, act && (a >> LOB) == (nx >> LOB));
        while (redo) {
            const int rr = (__ffs(redo) - 1) / kFastK;
            select_exact_row<NCH4, NT>(grp_rows + rr * E, lane, s_win[warp][rr]);
            redo &= ~(0xffu << (rr * kFastK));
        }
        __syncwarp();
        // gate weights of the whole group at once, fp64
        // (lanes of rows past the end hold stale picks: they read nothing)
        const int e = act ? (E - 1) - (int)(s_win[warp][r][k] & kLo) : 0;
        const int row = row0 + (act ? r : 0);
        const float vf = act ? __ldg(grp_rows + r * E + e) : 0.0f;
        const int lead = act ? r * kFastK : 0;
        const double v_own = (double)vf;
        const double v0 = __shfl_sync(kFull, v_own, lead);
        const double x = act ? exp(v_own - v0) : 0.0;
        // the row's sum over its eight lanes (an aligned group): every lane
        // of the group ends with the same value, the pairs being added in
        // the same (commutative) pairs
        double z = x;
        z += __shfl_xor_sync(kFull, z, 1);
        z += __shfl_xor_sync(kFull, z, 2);
        z += __shfl_xor_sync(kFull, z, 4);
        if (act) {
            const int pos = row * kFastK + k;
            idx[pos] = (int32_t)e;
            w[pos] = (float)(x * __drcp_rn(z));
            if constexpr (COUNT) {
                // source rank of the row, relative to the CTA's first rank
                int hs = 0;
#pragma unroll
                for (int q = 0; q < kGateHist - 1; ++q) hs += row >= bnd[q] ? 1 : 0;
                atomicAdd(&s_hist[hs][e], 1);
            }
        }
        __syncwarp();  // the picks are rewritten by the next group
    }

    if constexpr (COUNT) {
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t ok = 0u;
            for (long long spin = 0; spin < kGateWaitLimit; ++spin) {
                if (ld_acquire_gpu(cnt.sync + 3) == s_epoch + 1u) {
                    ok = 1u;
                    break;
                }
                __nanosleep(64);
            }
            if (!ok) raise_error(cnt.err, UE_ERR_TIMEOUT, (int)blockIdx.x);
            s_ok = ok;
        }
        __syncthreads();
        if (s_ok) {
            for (int x = threadIdx.x; x < kGateHist * E; x += blockDim.x) {
                const int h = (&s_hist[0][0])[x];
                if (h) {
                    const int hs = x / E, ex = x - hs * E;
                    atomicAdd(&cnt.load_re[(size_t)(rank0 + hs) * E + ex], h);
                    atomicAdd(&cnt.load_e[ex], h);
                }
            }
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            const uint32_t done = atomicAdd(cnt.sync + 1, 1u);
            if (done == gridDim.x - 1) {
                // last CTA: ready for the next launch
                cnt.sync[0] = 0u;
                cnt.sync[1] = 0u;
                __threadfence();
                cnt.sync[2] = s_epoch + 1u;
            }
        }
    }
}

template <int NCH4, int NT>
cudaError_t launch_fast(const Sizes& z, const GateShape& sh, const float* logits, int32_t* idx,
                        float* w, const GateCount* cnt, cudaStream_t st)
{
    if (cnt != nullptr)
        gate_topk_fast_kernel<NCH4, NT, true><<<sh.grid, kGateThreads, 0, st>>>(
            logits, z.N, sh.rows_per_cta, idx, w, *cnt);
    else
        gate_topk_fast_kernel<NCH4, NT, false><<<sh.grid, kGateThreads, 0, st>>>(
            logits, z.N, sh.rows_per_cta, idx, w, GateCount{});
    return cudaGetLastError();
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

bool gate_fast_shape(const Sizes& z)
{
    return z.K == kFastK && z.E % 32 == 0 && z.E >= 64 && z.E <= 256;
}

GateShape plan_gate_shape(const Sizes& z, int num_sms)
{
    GateShape sh;
    // generic kernel: grid-stride over warp groups, at most 4 CTAs per SM
    const int rpg = 32 / z.K;
    const int64_t groups = (z.N + rpg - 1) / rpg;
    const int64_t blocks_needed = (groups + (kGateThreads / 32) - 1) / (kGateThreads / 32);
    sh.grid = (int)std::max<int64_t>(1, std::min(blocks_needed, (int64_t)num_sms * 4));
    sh.rows_per_cta = 0;
    sh.fast = gate_fast_shape(z) ? 1 : 0;
    sh.fused = 0;
    if (sh.fast) {
        // contiguous blocks of whole warp groups, one wave of at most 4 CTAs per SM
        const int64_t target = std::max<int64_t>(1, (int64_t)num_sms * 4);
        int64_t rpc = (z.N + target - 1) / target;
        rpc = std::max<int64_t>(kFastRows, (rpc + kFastRows - 1) / kFastRows * kFastRows);
        sh.rows_per_cta = rpc;
        sh.grid = (int)std::max<int64_t>(1, (z.N + rpc - 1) / rpc);
        // the fused count needs every CTA's rows within kGateHist source ranks
        const int64_t spans = (rpc + z.T - 1) / z.T + 1;
        sh.fused = spans <= kGateHist ? 1 : 0;
    }
    return sh;
}

cudaError_t launch_gate_topk(const Sizes& z, const GateShape& sh, const float* logits,
                             int32_t* idx, float* w, const GateCount* cnt, cudaStream_t st)
{
    if (z.N == 0) {
        if (cnt == nullptr) return cudaSuccess;
        return launch_count(z, idx, cnt->load_re, cnt->load_e, cnt->sync, cnt->err, st);
    }
    if (sh.fast && (reinterpret_cast<uintptr_t>(logits) & 15u) == 0) {
        const GateCount* fc = (cnt != nullptr && sh.fused) ? cnt : nullptr;
        cudaError_t ce;
        switch (z.E) {
        case 64: ce = launch_fast<0, 2>(z, sh, logits, idx, w, fc, st); break;
        case 96: ce = launch_fast<0, 3>(z, sh, logits, idx, w, fc, st); break;
        case 128: ce = launch_fast<1, 0>(z, sh, logits, idx, w, fc, st); break;
        case 160: ce = launch_fast<1, 1>(z, sh, logits, idx, w, fc, st); break;
        case 192: ce = launch_fast<1, 2>(z, sh, logits, idx, w, fc, st); break;
        case 224: ce = launch_fast<1, 3>(z, sh, logits, idx, w, fc, st); break;
        default: ce = launch_fast<2, 0>(z, sh, logits, idx, w, fc, st); break;
        }
        if (ce != cudaSuccess || cnt == nullptr || fc != nullptr) return ce;
        return launch_count(z, idx, cnt->load_re, cnt->load_e, cnt->sync, cnt->err, st);
    }
    cudaError_t ce;
    switch ((z.E + 31) / 32) {
    case 1: ce = launch_vpl<1>(z, logits, idx, w, sh.grid, st); break;
    case 2: ce = launch_vpl<2>(z, logits, idx, w, sh.grid, st); break;
    case 3: ce = launch_vpl<3>(z, logits, idx, w, sh.grid, st); break;
    case 4: ce = launch_vpl<4>(z, logits, idx, w, sh.grid, st); break;
    case 5: ce = launch_vpl<5>(z, logits, idx, w, sh.grid, st); break;
    case 6: ce = launch_vpl<6>(z, logits, idx, w, sh.grid, st); break;
    case 7: ce = launch_vpl<7>(z, logits, idx, w, sh.grid, st); break;
    case 8: ce = launch_vpl<8>(z, logits, idx, w, sh.grid, st); break;
    default: return cudaErrorInvalidValue;
    }
    if (ce != cudaSuccess || cnt == nullptr) return ce;
    return launch_count(z, idx, cnt->load_re, cnt->load_e, cnt->sync, cnt->err, st);
}

}  // namespace ue
