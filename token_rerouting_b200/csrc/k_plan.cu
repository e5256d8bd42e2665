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
// With a minimum of m pairs per replica ("UltraEP" README, "Performance
// Tuning / Replication planning": minimal load allocated to a replica) only
// experts with L_e >= m*(c_e + 1) may take a copy, and the greedy also stops
// when none may; m = 0 lets every expert grow.
//
// Design (B200): the greedy is serial, so its speed is the latency of one
// iteration. The choice of e* depends only on the copy counts, never on the
// ranks: the sequence of experts the greedy picks is fixed by the loads
// alone (a highest-ratio apportionment). So two warps of one CTA run it as a
// pipeline:
//  - warp 1 (expert side) produces the picks in order: e*, its new copy
//    count and the quota parameters of that step, pushed into a shared-memory
//    queue with a ready flag per entry. L/c is compared through the integer
//    key floor(L*2^24/c), one 64-bit multiply-high with a table of
//    ceil(2^64/c); for c <= 257 and L < 2^30 the map is exact and order
//    preserving (two different ratios differ by more than 1/66049, i.e. by
//    more than 250 after scaling; equal ratios give equal keys). The expert id
//    sits below the key, so the argmax with ties to the lowest e is two warp
//    `redux` max reductions. An expert that may not grow has key 0; when
//    every key is 0 the expert side pushes an end marker (e = -1).
//  - warp 0 (rank side) keeps the rank loads and the redundant slots in
//    registers (lane l owns ranks l, l+32, ... and their slots, so every
//    load change lands in the lane that owns the rank). Per iteration: the
//    stop test and the least loaded rank with a free slot (two `redux`
//    reductions, max load and min of (load << 7 | r), when Q < 2^25; three
//    otherwise), with the pick's ready flag and the pick itself loaded before
//    them, the
//    placement in r*'s lowest free slot, and the new quotas of e*'s copies: the
//    master's goes from ceil(L/(c-1)) to ceil(L/c); a first replica takes
//    floor(L/2); later replicas are found by ballots in ascending slot order.
//    The count of co-located copies does not depend on the order of
//    placement and is taken from the final slots.
// Warp 1 needs far fewer instructions per step, so warp 0 rarely waits; its
// wait on a queue entry is bounded. The rest of the CTA writes the outputs
// and scans the slot offsets at the end.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kPlanThreads = 256;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kKeyShift = 24;
constexpr long long kPickWaitLimit = 1LL << 24;

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

// may an expert with load L and c copies take copy c+1 and keep at least m
// pairs on each?
__device__ __forceinline__ bool may_grow(unsigned L, unsigned c, unsigned m)
{
    return (unsigned long long)m * (c + 1u) <= (unsigned long long)L;
}

struct Pick {
    int e;         // expert receiving the copy (-1: no expert may grow)
    unsigned c;    // its copy count with the new copy
    unsigned qb;   // floor(L / c)
    unsigned rem;  // L mod c
    unsigned dq0;  // master quota change: ceil(L/c) - ceil(L/(c-1)) (two's complement)
    int rm;        // the master's rank, e / M
};

template <int NJE, int NJR, int SM>
__global__ void __launch_bounds__(kPlanThreads, 1)
plan_kernel(const int32_t* __restrict__ load_e, int R, int E, int S, unsigned min_tokens,
            ue_placement out, int* err)
{
    __shared__ unsigned long long sRecip[kMaxG + 2];  // ceil(2^64 / c), c = 2 .. G+1
    __shared__ int sL[kMaxE];       // exact load per expert
    __shared__ int sC[kMaxE];       // copies per expert (final)
    __shared__ int sRank[kMaxR];    // rank loads (initial, then final)
    __shared__ int sSlotE[kMaxG];   // expert of redundant slot g, -1 empty (final)
    __shared__ int sSlotQ[kMaxG];   // quota of redundant slot g (final)
    __shared__ Pick sPick[kMaxG];   // the expert side's picks, in order
    __shared__ volatile int sReady[kMaxG];
    __shared__ volatile int sDone;  // the rank side has stopped
    __shared__ int sUsedPicks;
    __shared__ unsigned long long sQ;
    __shared__ int sStats[4];
    __shared__ int sWarpSum[kPlanWarps];
    __shared__ int sColoc;

    const int M = E / R;
    const int G = R * S;
    const int P = R * (M + S);
    const int tid = threadIdx.x;

    if (tid == 0) {
        sQ = 0ull;
        sUsedPicks = 0;
        sDone = 0;
        sColoc = 0;
    }
    for (int r = tid; r < R; r += blockDim.x) sRank[r] = 0;
    for (int g = tid; g < G; g += blockDim.x) sReady[g] = 0;
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

    const int warp = tid >> 5;
    const int lane = tid & 31;
    if (warp == 1) {
        // ---- expert side: the greedy's picks, independent of the ranks ----
        unsigned Lr[NJE], cr[NJE];
        unsigned long long key[NJE];
#pragma unroll
        for (int j = 0; j < NJE; ++j) {
            const int e = lane + 32 * j;
            Lr[j] = e < E ? (unsigned)sL[e] : 0u;
            cr[j] = 1u;
            key[j] = (e < E && may_grow(Lr[j], 1u, min_tokens)) ? packed_key(Lr[j], 1u, e, sRecip)
                                                                 : 0ull;
        }
        for (int t = 0; t < G; ++t) {
            if (__any_sync(kFull, sDone != 0)) break;
            unsigned long long best = 0ull;
#pragma unroll
            for (int j = 0; j < NJE; ++j) best = key[j] > best ? key[j] : best;
            const unsigned hi = __reduce_max_sync(kFull, (unsigned)(best >> 32));
            const unsigned lo = __reduce_max_sync(kFull, (unsigned)(best >> 32) == hi ? (unsigned)best : 0u);
            if (hi == 0u && lo == 0u) {
                // no expert may take another copy: end marker
                if (lane == 0) {
                    sPick[t] = Pick{-1, 0u, 0u, 0u, 0u, 0};
                    __threadfence_block();
                    sReady[t] = 1;
                }
                break;
            }
            const int estar = 511 - (int)(lo & 511u);
            const int ej = estar >> 5;
            unsigned Le = 0u, ce = 0u;
#pragma unroll
            for (int j = 0; j < NJE; ++j)
                if (j == ej) {
                    Le = Lr[j];
                    ce = cr[j];
                }
            Le = __shfl_sync(kFull, Le, estar & 31);
            ce = __shfl_sync(kFull, ce, estar & 31) + 1u;
            const unsigned long long nk =
                may_grow(Le, ce, min_tokens) ? packed_key(Le, ce, estar, sRecip) : 0ull;
            if (lane == (estar & 31)) {
#pragma unroll
                for (int j = 0; j < NJE; ++j)
                    if (j == ej) {
                        cr[j] = ce;
                        key[j] = nk;
                    }
            }
            if (lane == 0) {
                const unsigned qb = div_by(Le, ce, sRecip);
                const unsigned rem = Le - qb * ce;
                const unsigned q0_new = qb + (rem > 0u ? 1u : 0u);
                const unsigned q0_old = div_by(Le + ce - 2u, ce - 1u, sRecip);
                sPick[t] = Pick{estar, ce, qb, rem, q0_new - q0_old, estar / M};
                __threadfence_block();
                sReady[t] = 1;
            }
        }
    } else if (warp == 0) {
        // ---- rank side: stop test, least loaded free rank, bookkeeping ----
        const long long Q = (long long)sQ;
        const long long stop_rhs = 51LL * Q;
        unsigned load[NJR];
        int used[NJR];
        int slotE[NJR][SM], slotQ[NJR][SM];
#pragma unroll
        for (int j = 0; j < NJR; ++j) {
            const int r = lane + 32 * j;
            load[j] = r < R ? (unsigned)sRank[r] : 0u;
            used[j] = r < R ? 0 : S;  // ranks beyond R never offer a slot
#pragma unroll
            for (int s = 0; s < SM; ++s) {
                slotE[j][s] = -1;
                slotQ[j][s] = 0;
            }
        }
        int iters = 0;
        unsigned max_before = 0u;
        // with every rank load below 2^25 (Q < 2^25), a rank's load and its
        // index (< 128) pack into one 32-bit key, and the least loaded rank
        // with a free slot (ties to the lowest r) is one reduction
        const bool packed = Q < (1LL << 25);
        for (;;) {
            // this iteration's pick: its flag is read first and the pick
            // right after it (acquire orders the read), so that both loads
            // overlap the reductions below; a pick read before its flag was
            // set is read again after the wait
            // (iters reaches G only when every slot is used and the loop is
            // about to stop; the index is clamped so that these early reads
            // stay inside the arrays)
            const int it0 = iters < kMaxG ? iters : kMaxG - 1;
            int ready = 0;
            asm volatile("ld.acquire.cta.shared.u32 %0, [%1];"
                         : "=r"(ready)
                         : "r"((unsigned)__cvta_generic_to_shared((const void*)&sReady[it0]))
                         : "memory");
            const int ready0 = ready;
            const Pick pk_early = sPick[it0];
            unsigned maxl = 0u, bestl = 0xffffffffu, bestr = 0xffffffffu;
            int rstar;
            if (packed) {
                unsigned key = 0xffffffffu;
#pragma unroll
                for (int j = 0; j < NJR; ++j) {
                    maxl = max(maxl, load[j]);
                    if (used[j] < S) key = min(key, (load[j] << 7) | (unsigned)(lane + 32 * j));
                }
                maxl = __reduce_max_sync(kFull, maxl);
                key = __reduce_min_sync(kFull, key);
                if (iters == 0) max_before = maxl;
                if (50LL * R * (long long)maxl <= stop_rhs) break;
                if (key == 0xffffffffu) break;  // no free slot anywhere
                rstar = (int)(key & 127u);
            } else {
#pragma unroll
                for (int j = 0; j < NJR; ++j) {
                    maxl = max(maxl, load[j]);
                    if (used[j] < S && load[j] < bestl) {
                        bestl = load[j];
                        bestr = (unsigned)(lane + 32 * j);
                    }
                }
                maxl = __reduce_max_sync(kFull, maxl);
                const unsigned ml = __reduce_min_sync(kFull, bestl);
                if (iters == 0) max_before = maxl;
                if (50LL * R * (long long)maxl <= stop_rhs) break;
                if (ml == 0xffffffffu) break;  // no free slot anywhere
                rstar = (int)__reduce_min_sync(kFull, bestl == ml ? bestr : 0xffffffffu);
            }

            // the pick is normally ready long before: the expert side needs
            // far fewer instructions per step. The wait is bounded.
            for (long long spin = 0; !ready && spin < kPickWaitLimit; ++spin)
                asm volatile("ld.acquire.cta.shared.u32 %0, [%1];"
                             : "=r"(ready)
                             : "r"((unsigned)__cvta_generic_to_shared((const void*)&sReady[iters]))
                             : "memory");
            ready = __all_sync(kFull, ready);
            if (!ready) {
                if (lane == 0) raise_error(err, UE_ERR_TIMEOUT, iters);
                break;
            }
            const Pick pk = ready0 ? pk_early : sPick[iters];
            if (pk.e < 0) break;  // no expert may take another copy
            const int estar = pk.e;
            const int rj = rstar >> 5;
            const bool rown = lane == (rstar & 31);

            // the new copy goes into r*'s lowest free slot (the slot index is
            // made warp-uniform so that the slot arrays stay in registers)
            int s_new = 0;
#pragma unroll
            for (int j = 0; j < NJR; ++j)
                if (j == rj) s_new = used[j];
            s_new = __shfl_sync(kFull, s_new, rstar & 31);
            if (rown) {
#pragma unroll
                for (int j = 0; j < NJR; ++j)
                    if (j == rj) {
                        used[j] += 1;
#pragma unroll
                        for (int s = 0; s < SM; ++s)
                            if (s == s_new) slotE[j][s] = estar;
                    }
            }
            // master quota change, on the master rank's owner
            const int rm = pk.rm;
            if (lane == (rm & 31)) {
#pragma unroll
                for (int j = 0; j < NJR; ++j)
                    if (j == (rm >> 5)) load[j] += pk.dq0;
            }
            if (pk.c == 2u) {
                // first replica: the only other copy is the master, and the
                // replica's quota is floor(L/2) (L mod 2 < 2 keeps the +1 on
                // the master)
                if (rown) {
#pragma unroll
                    for (int j = 0; j < NJR; ++j)
                        if (j == rj) {
#pragma unroll
                            for (int s = 0; s < SM; ++s)
                                if (s < S && slotE[j][s] == estar) slotQ[j][s] = (int)pk.qb;
                            load[j] += pk.qb;
                        }
                }
            } else {
                // replicas, ascending slot g = r*S + s (r = lane + 32 j)
                unsigned before = 0u;
                const unsigned lt = (1u << lane) - 1u;
#pragma unroll
                for (int j = 0; j < NJR; ++j) {
                    unsigned lower = 0u;   // e* replicas in lower lanes of group j
                    unsigned total = 0u;   // e* replicas in group j
#pragma unroll
                    for (int s = 0; s < SM; ++s) {
                        const unsigned msk = __ballot_sync(kFull, s < S && slotE[j][s] == estar);
                        lower += __popc(msk & lt);
                        total += __popc(msk);
                    }
                    unsigned mine = 0u;  // e* replicas in this lane's lower slots
#pragma unroll
                    for (int s = 0; s < SM; ++s) {
                        if (s < S && slotE[j][s] == estar) {
                            const unsigned pos = 1u + before + lower + mine;
                            const int qn = (int)(pk.qb + (pos < pk.rem ? 1u : 0u));
                            load[j] = load[j] + (unsigned)(qn - slotQ[j][s]);
                            slotQ[j][s] = qn;
                            mine += 1u;
                        }
                    }
                    before += total;
                }
            }
            iters += 1;
        }
        unsigned mx = 0u;
#pragma unroll
        for (int j = 0; j < NJR; ++j) {
            const int r = lane + 32 * j;
            if (r < R) {
                mx = max(mx, load[j]);
                sRank[r] = (int)load[j];
#pragma unroll
                for (int s = 0; s < SM; ++s)
                    if (s < S) {
                        sSlotE[r * S + s] = slotE[j][s];
                        sSlotQ[r * S + s] = slotQ[j][s];
                    }
            }
        }
        mx = __reduce_max_sync(kFull, mx);
        if (lane == 0) {
            sStats[0] = iters;
            sStats[1] = (int)max_before;
            sStats[2] = (int)mx;
            sUsedPicks = iters;
            sDone = 1;
        }
    }
    __syncthreads();

    // copies per expert: 1 + its picks among the first `iters` of the queue
    const int iters = sUsedPicks;
    for (int e = tid; e < E; e += blockDim.x) sC[e] = 1;
    __syncthreads();
    for (int t = tid; t < iters; t += blockDim.x) atomicAdd(&sC[sPick[t].e], 1);
    // copies placed on a rank that already held a copy of the same expert:
    // for each (expert, rank) every copy but the first one there, which is
    // the same count whatever the order of placement (a replica counts unless
    // it is the lowest slot of its expert on a rank without the master)
    for (int g = tid; g < G; g += blockDim.x) {
        const int e = sSlotE[g];
        if (e >= 0) {
            const int r = g / S, sl = g - r * S;
            bool first = r != e / M;
            for (int s2 = 0; s2 < sl; ++s2) first = first && sSlotE[r * S + s2] != e;
            if (!first) atomicAdd(&sColoc, 1);
        }
    }
    __syncthreads();

    for (int e = tid; e < E; e += blockDim.x) out.n_copies[e] = sC[e];
    for (int g = tid; g < G; g += blockDim.x) out.slot_expert[g] = sSlotE[g];
    for (int r = tid; r < R; r += blockDim.x) out.rank_load[r] = sRank[r];
    if (tid < 3) out.stats[tid] = sStats[tid];
    if (tid == 3) out.stats[3] = sColoc;

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

template <int NJE, int NJR>
cudaError_t launch_s(const Sizes& z, const int32_t* load_e, unsigned m, const ue_placement& out,
                     int* err, cudaStream_t st)
{
    if (z.S <= 2)
        plan_kernel<NJE, NJR, 2><<<1, kPlanThreads, 0, st>>>(load_e, z.R, z.E, z.S, m, out, err);
    else
        plan_kernel<NJE, NJR, 8><<<1, kPlanThreads, 0, st>>>(load_e, z.R, z.E, z.S, m, out, err);
    return cudaGetLastError();
}

template <int NJE>
cudaError_t launch_r(const Sizes& z, const int32_t* load_e, unsigned m, const ue_placement& out,
                     int* err, cudaStream_t st)
{
    if (z.R <= 32) return launch_s<NJE, 1>(z, load_e, m, out, err, st);
    if (z.R <= 64) return launch_s<NJE, 2>(z, load_e, m, out, err, st);
    return launch_s<NJE, 4>(z, load_e, m, out, err, st);
}

}  // namespace

cudaError_t launch_plan(const Sizes& z, const int32_t* load_e, int min_tokens,
                        const ue_placement& out, int* err, cudaStream_t st)
{
    const unsigned m = (unsigned)min_tokens;
    if (z.E <= 32) return launch_r<1>(z, load_e, m, out, err, st);
    if (z.E <= 64) return launch_r<2>(z, load_e, m, out, err, st);
    if (z.E <= 128) return launch_r<4>(z, load_e, m, out, err, st);
    return launch_r<8>(z, load_e, m, out, err, st);
}

}  // namespace ue
