// k_plan.cu -- quota-driven replication plan (the pages' update_placement).
//
// "Xiaohongshu's UltraEP Balances MoE Experts in 300 us", "How balancing in
// 300 microseconds works": a quota-driven scheduler reacts to the load right
// after gating, every microbatch and every layer. "UltraEP" README,
// "Interface / 2. Forward and backward": update_placement computes the
// per-microbatch replication plan from the exact load.
//
// Rule: start with the masters only (expert e on rank e/M). The quota of copy
// j of expert e (j = 0 the master, then replicas by ascending redundant slot
// g) is floor(L_e/c_e) plus one for the first L_e mod c_e copies; a rank's
// load is the sum of its copies' quotas. Repeat: stop if
// 50*R*max_r load_r <= 51*Q or no slot is free; else e* = argmax L_e/c_e
// (exact, ties to the lowest e), r* = argmin load_r over ranks with a free
// slot (ties to the lowest r); the copy goes into r*'s lowest free slot.
//
// Design (B200): the greedy is serial (at most G iterations), so its speed is
// the latency of one iteration, and one warp runs it entirely in registers.
// Lane l owns experts l, l+32, ... (load, copies, selection key) and ranks
// l, l+32, ... together with those ranks' redundant slots (expert held,
// quota). Every load change then lands in the lane that owns the rank, so an
// iteration needs no shared memory and no atomics:
//  - Expert side: L/c is compared through the integer key floor(L*2^24/c),
//    one 64-bit multiply-high with a table of ceil(2^64/c). For c <= 257 and
//    L < 2^30 this map is exact and order preserving (two different ratios
//    differ by more than 1/66049, i.e. by more than 250 after scaling, and
//    equal ratios give equal keys). The expert id is packed below the key, so
//    the argmax with ties to the lowest e is two warp `redux` max reductions.
//  - Rank side: the stop test (max load) and the least-loaded rank with a
//    free slot are `redux` reductions, issued together with the expert one.
//  - Update: the replicas of e* are found by ballots over the slot registers
//    in ascending slot order; each replica's new quota changes its owner
//    lane's rank load locally. The master's quota goes from ceil(L/(c-1)) to
//    ceil(L/c); every lane knows that change and the master's owner applies
//    it.
// The other warps write the outputs and scan the slot offsets at the end.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kPlanThreads = 256;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kKeyShift = 24;

__device__ __forceinline__ unsigned div_by(unsigned x, unsigned c, const unsigned long long* recip)
{
    // floor(x / c) for x < 2^40, c <= 257: exact with ceil(2^64 / c)
    return c == 1u ? x : (unsigned)__umul64hi((unsigned long long)x, recip[c]);
}

// floor(L * 2^24 / c) with the expert id below it: larger ratio first, then
// lower id
__device__ __forceinline__ unsigned long long packed_key(unsigned L, unsigned c, int e,
                                                         const unsigned long long* recip)
{
    const unsigned long long x = (unsigned long long)L << kKeyShift;
    const unsigned long long k = c == 1u ? x : __umul64hi(x, recip[c]);
    return (k << 9) | (unsigned long long)(511 - e);
}

template <int NJ, int SM>
__global__ void __launch_bounds__(kPlanThreads)
plan_kernel(const int32_t* __restrict__ load_e, int R, int E, int S, ue_placement out, int* err)
{
    __shared__ unsigned long long sRecip[kMaxG + 2];  // ceil(2^64 / c), c = 2 .. G+1
    __shared__ int sL[kMaxE];       // exact load per expert
    __shared__ int sC[kMaxE];       // copies per expert (final)
    __shared__ int sRank[kMaxR];    // rank loads (initial, then final)
    __shared__ int sSlotE[kMaxG];   // expert of redundant slot g, -1 empty (final)
    __shared__ int sSlotQ[kMaxG];   // quota of redundant slot g (final)
    __shared__ unsigned long long sQ;
    __shared__ int sStats[4];
    __shared__ int sWarpSum[kPlanWarps];

    const int M = E / R;
    const int G = R * S;
    const int P = R * (M + S);
    const int tid = threadIdx.x;

    if (tid == 0) sQ = 0ull;
    for (int r = tid; r < R; r += blockDim.x) sRank[r] = 0;
    for (int c = tid + 2; c <= G + 1; c += blockDim.x)
        sRecip[c] = (0xffffffffffffffffull / (unsigned long long)c) + 1ull;
    __syncthreads();
    unsigned long long part = 0ull;
    for (int e = tid; e < E; e += blockDim.x) {
        int L = __ldg(load_e + e);
        if (L < 0) {
            raise_error(err, UE_ERR_DEVICE_BOUNDS, e);
            L = 0;
        }
        sL[e] = L;
        atomicAdd(&sRank[e / M], L);
        part += (unsigned long long)L;
    }
    if (part) atomicAdd(&sQ, part);
    __syncthreads();

    if (tid < 32) {
        const int lane = tid;
        const long long Q = (long long)sQ;
        const long long stop_rhs = 51LL * Q;
        unsigned Lr[NJ], cr[NJ];
        unsigned long long key[NJ];
        unsigned load[NJ];
        int used[NJ];
        int slotE[NJ][SM], slotQ[NJ][SM];
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            const int e = lane + 32 * j;
            Lr[j] = e < E ? (unsigned)sL[e] : 0u;
            cr[j] = 1u;
            key[j] = e < E ? packed_key(Lr[j], 1u, e, sRecip) : 0ull;
            const int r = lane + 32 * j;
            load[j] = r < R ? (unsigned)sRank[r] : 0u;
            used[j] = r < R ? 0 : S;  // ranks beyond R never offer a slot
#pragma unroll
            for (int s = 0; s < SM; ++s) {
                slotE[j][s] = -1;
                slotQ[j][s] = 0;
            }
        }
        int iters = 0, colocated = 0;
        unsigned max_before = 0u;
        for (;;) {
            unsigned maxl = 0u, bestl = 0xffffffffu, bestr = 0xffffffffu;
            unsigned long long best = 0ull;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                maxl = max(maxl, load[j]);
                if (used[j] < S && load[j] < bestl) {
                    bestl = load[j];
                    bestr = (unsigned)(lane + 32 * j);
                }
                best = key[j] > best ? key[j] : best;
            }
            maxl = __reduce_max_sync(kFull, maxl);
            const unsigned ml = __reduce_min_sync(kFull, bestl);
            const unsigned hi = __reduce_max_sync(kFull, (unsigned)(best >> 32));
            if (iters == 0) max_before = maxl;
            if (50LL * R * (long long)maxl <= stop_rhs) break;
            if (ml == 0xffffffffu) break;  // no free slot anywhere
            const int rstar = (int)__reduce_min_sync(kFull, bestl == ml ? bestr : 0xffffffffu);
            const unsigned lo = __reduce_max_sync(kFull, (unsigned)(best >> 32) == hi ? (unsigned)best : 0u);
            const int estar = 511 - (int)(lo & 511u);
            const int rj = rstar >> 5;
            const bool rown = lane == (rstar & 31);
            const int ej = estar >> 5;
            const bool eown = lane == (estar & 31);

            // r*'s lowest free slot; does r* already hold a copy of e*?
            int s_new = 0;
            bool held = false;
#pragma unroll
            for (int j = 0; j < NJ; ++j)
                if (j == rj) {
                    s_new = used[j];
#pragma unroll
                    for (int s = 0; s < SM; ++s) held |= rown && s < S && slotE[j][s] == estar;
                }
            s_new = __shfl_sync(kFull, s_new, rstar & 31);
            if (estar / M == rstar || __any_sync(kFull, held)) colocated += 1;
            if (rown) {
#pragma unroll
                for (int j = 0; j < NJ; ++j)
                    if (j == rj) {
                        used[j] += 1;
#pragma unroll
                        for (int s = 0; s < SM; ++s)
                            if (s == s_new) slotE[j][s] = estar;
                    }
            }

            // e* gains a copy: new key and quotas
            unsigned Le = 0u, ce = 0u;
#pragma unroll
            for (int j = 0; j < NJ; ++j)
                if (j == ej) {
                    Le = Lr[j];
                    ce = cr[j];
                }
            Le = __shfl_sync(kFull, Le, estar & 31);
            ce = __shfl_sync(kFull, ce, estar & 31) + 1u;
            const unsigned long long nk = packed_key(Le, ce, estar, sRecip);
            if (eown) {
#pragma unroll
                for (int j = 0; j < NJ; ++j)
                    if (j == ej) {
                        cr[j] = ce;
                        key[j] = nk;
                    }
            }
            const unsigned qb = div_by(Le, ce, sRecip);
            const unsigned rem = Le - qb * ce;
            // master: ceil(L/(c-1)) -> ceil(L/c), applied by the master rank's owner
            const int rm = estar / M;
            const unsigned q0_new = qb + (rem > 0u ? 1u : 0u);
            const unsigned q0_old = div_by(Le + ce - 2u, ce - 1u, sRecip);
            if (lane == (rm & 31)) {
#pragma unroll
                for (int j = 0; j < NJ; ++j)
                    if (j == (rm >> 5)) load[j] = load[j] + q0_new - q0_old;
            }
            // replicas, ascending slot g = r*S + s (r = lane + 32 j)
            unsigned before = 0u;
            const unsigned lt = (1u << lane) - 1u;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                unsigned lower = 0u;   // e* replicas in lower lanes of group j
                unsigned total = 0u;   // e* replicas in group j
                unsigned msk[SM];
#pragma unroll
                for (int s = 0; s < SM; ++s) {
                    msk[s] = __ballot_sync(kFull, s < S && slotE[j][s] == estar);
                    lower += __popc(msk[s] & lt);
                    total += __popc(msk[s]);
                }
                unsigned mine = 0u;  // e* replicas in this lane's lower slots
#pragma unroll
                for (int s = 0; s < SM; ++s) {
                    if (s < S && slotE[j][s] == estar) {
                        const unsigned pos = 1u + before + lower + mine;
                        const int qn = (int)(qb + (pos < rem ? 1u : 0u));
                        load[j] = load[j] + (unsigned)(qn - slotQ[j][s]);
                        slotQ[j][s] = qn;
                        mine += 1u;
                    }
                }
                before += total;
            }
            iters += 1;
        }
        unsigned mx = 0u;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            const int idx = lane + 32 * j;
            if (idx < R) {
                mx = max(mx, load[j]);
                sRank[idx] = (int)load[j];
#pragma unroll
                for (int s = 0; s < SM; ++s)
                    if (s < S) {
                        sSlotE[idx * S + s] = slotE[j][s];
                        sSlotQ[idx * S + s] = slotQ[j][s];
                    }
            }
            if (idx < E) sC[idx] = (int)cr[j];
        }
        mx = __reduce_max_sync(kFull, mx);
        if (lane == 0) {
            sStats[0] = iters;
            sStats[1] = (int)max_before;
            sStats[2] = (int)mx;
            sStats[3] = colocated;
        }
    }
    __syncthreads();

    for (int e = tid; e < E; e += blockDim.x) out.n_copies[e] = sC[e];
    for (int g = tid; g < G; g += blockDim.x) out.slot_expert[g] = sSlotE[g];
    for (int r = tid; r < R; r += blockDim.x) out.rank_load[r] = sRank[r];
    if (tid < 4) out.stats[tid] = sStats[tid];

    // slot quotas in physical order and their exclusive running sum; each
    // thread owns slots 2*tid and 2*tid+1 (P <= 512). A master's quota is
    // ceil(L/c).
    int q2[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int p = 2 * tid + h;
        int q = 0;
        if (p < P) {
            const int r = p / (M + S);
            const int l = p - r * (M + S);
            if (l < M) {
                const int e = r * M + l;
                const unsigned c = (unsigned)sC[e];
                q = (int)div_by((unsigned)sL[e] + c - 1u, c, sRecip);
            } else {
                q = sSlotQ[r * S + (l - M)];
            }
            out.slot_quota[p] = q;
        }
        q2[h] = q;
    }
    const int lane = tid & 31, warp = tid >> 5;
    const int mine = q2[0] + q2[1];
    int incl = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) sWarpSum[warp] = incl;
    __syncthreads();
    int wofs = 0;
    for (int w = 0; w < warp; ++w) wofs += sWarpSum[w];
    const int excl = wofs + incl - mine;
    if (2 * tid < P) out.slot_offset[2 * tid] = excl;
    if (2 * tid + 1 < P) out.slot_offset[2 * tid + 1] = excl + q2[0];
    if (tid == 0) out.slot_offset[P] = (int)sQ;
}

template <int NJ>
cudaError_t launch_nj(const Sizes& z, const int32_t* load_e, const ue_placement& out, int* err,
                      cudaStream_t st)
{
    if (z.S <= 1)
        plan_kernel<NJ, 1><<<1, kPlanThreads, 0, st>>>(load_e, z.R, z.E, z.S, out, err);
    else if (z.S <= 2)
        plan_kernel<NJ, 2><<<1, kPlanThreads, 0, st>>>(load_e, z.R, z.E, z.S, out, err);
    else if (z.S <= 4)
        plan_kernel<NJ, 4><<<1, kPlanThreads, 0, st>>>(load_e, z.R, z.E, z.S, out, err);
    else
        plan_kernel<NJ, 8><<<1, kPlanThreads, 0, st>>>(load_e, z.R, z.E, z.S, out, err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_plan(const Sizes& z, const int32_t* load_e,
                        const ue_placement& out, int* err, cudaStream_t st)
{
    const int need = std::max(z.E, z.R);
    if (need <= 32) return launch_nj<1>(z, load_e, out, err, st);
    if (need <= 64) return launch_nj<2>(z, load_e, out, err, st);
    if (need <= 128) return launch_nj<4>(z, load_e, out, err, st);
    return launch_nj<8>(z, load_e, out, err, st);
}

}  // namespace ue
