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
// ranks: the experts the greedy picks, in order, are fixed by the loads
// alone. Each step takes the largest current ratio L_e/c_e (ties to the
// lowest e) and then moves e to L_e/(c_e+1), so the picks are the keys
// (L_e/c, e), c = 1, 2, ..., in descending order of ratio (equal ratios:
// lower e first), truncated where an expert may not grow. One CTA therefore
// computes the whole pick sequence in parallel before the serial part:
//  - candidates: with Q > 0 every key of ratio >= Q/(G+E) is kept, c <= min(G,
//    floor(L_e (G+E) / Q)) per expert. That is at least G + 1 keys when no
//    expert is capped (sum floor(x_e) > sum x_e - E = G) and at most G + E,
//    so the top G keys are among them. With a minimum per replica some
//    experts are capped (c <= floor(L_e/m) - 1); while the candidates are
//    fewer than G and some expert is cut by the threshold, the threshold is
//    halved (at most 2G + E candidates);
//  - each candidate is one 64-bit key: floor(L_e 2^17 / c) (exact and order
//    preserving for c <= 257: two different ratios differ by more than
//    2^-17), then 255 - e, then c - 1; each key's place in pick order is the
//    number of larger keys, counted by one thread per key against all the
//    others, and each pick's quota parameters follow in parallel (fewer
//    than G picks end with an end marker).
// Then one warp runs the rank side alone, with the picks already in shared
// memory: it keeps the rank loads and the redundant slots in registers (lane
// l owns ranks l, l+32, ... and their slots, so every load change lands in
// the lane that owns the rank). Per iteration: the stop test as a vote (is
// any load above floor(51 Q / (50 R))?) and the least loaded rank with a free
// slot as one `redux` min of (load << 7 | r) when Q < 2^25 (two reductions
// otherwise), the placement in r*'s lowest free slot, and the new quotas of
// e*'s copies: the master's goes from ceil(L/(c-1)) to ceil(L/c); a first
// replica takes floor(L/2); later replicas are found by ballots in ascending
// slot order. The count of co-located copies does not depend on the order of
// placement and is taken from the final slots. The rest of the CTA writes the
// outputs and scans the slot offsets at the end.
// The kernel lets a dependent launch start at once (programmatic dependent
// launch): a reroute launched that way does its plan-free part, counting its
// tiles and looking back, on the other SMs while this one CTA runs.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kPlanThreads = 512;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kRatioShift = 17;
constexpr int kCandMax = 1024;  // candidate keys: at most 2G + E <= 768

__device__ __forceinline__ unsigned div_by(unsigned x, unsigned c, const unsigned long long* recip)
{
    // floor(x / c) for x < 2^40, c <= 257: exact with ceil(2^64 / c)
    return c == 1u ? x : (unsigned)__umul64hi((unsigned long long)x, recip[c]);
}

struct Pick {
    int e;         // expert receiving the copy (-1: no expert may grow)
    unsigned c;    // its copy count with the new copy
    unsigned qb;   // floor(L / c)
    unsigned rem;  // L mod c
    unsigned dq0;  // master quota change: ceil(L/c) - ceil(L/(c-1)) (two's complement)
    int rm;        // the master's rank, e / M
};

// floor(x / d) for 0 < d < 2^31 and a quotient below 2^51 (here x < 2^50, or
// x < 2^63 with x / d < 2^33): the fp64 estimate x * (1/d) is within one unit
// of it, and the exact remainder moves the estimate to the right side
__device__ __forceinline__ unsigned long long floor_div_exact(unsigned long long x,
                                                              unsigned long long d, double inv)
{
    unsigned long long q = (unsigned long long)((double)x * inv);
    if (q * d > x) --q;
    else if ((q + 1ull) * d <= x) ++q;
    return q;
}

// block-wide sum of v over all threads (every thread gets the total)
__device__ __forceinline__ long long block_sum(long long v, long long* scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    __syncthreads();
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    long long t = 0;
    for (int w = 0; w < kPlanWarps; ++w) t += scratch[w];
    return t;
}

template <int NJR, int SM>
__global__ void __launch_bounds__(kPlanThreads, 1)
plan_kernel(const int32_t* __restrict__ load_e, int R, int E, int S, unsigned min_tokens,
            ue_placement out, int* err)
{
    __shared__ unsigned long long sRecip[kMaxG + 2];  // ceil(2^64 / c), c = 2 .. G+1
    __shared__ int sL[kMaxE];       // exact load per expert
    __shared__ int sCnt[kMaxE + 1]; // candidates per expert, then their exclusive scan
    __shared__ int sC[kMaxE];       // copies per expert (final)
    __shared__ int sRank[kMaxR];    // rank loads (initial, then final)
    __shared__ int sSlotE[kMaxG];   // expert of redundant slot g, -1 empty (final)
    __shared__ int sSlotQ[kMaxG];   // quota of redundant slot g (final)
    __shared__ __align__(16) unsigned long long sKey[kCandMax];
    __shared__ unsigned long long sOrd[kMaxG];  // the first G keys in pick order
    __shared__ Pick sPick[kMaxG + 1];  // the picks in order (then an end marker)
    __shared__ long long sRed[kPlanWarps];
    __shared__ int sUsedPicks;
    __shared__ unsigned long long sQ;
    __shared__ int sStats[4];
    __shared__ int sWarpSum[kPlanWarps];
    __shared__ int sColoc;

    const int M = E / R;
    const int G = R * S;
    const int P = R * (M + S);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // a reroute launched as this kernel's programmatic dependent may start
    // now: it counts its tiles and looks back while the plan runs
    pdl_trigger();
    if (tid == 0) {
        sQ = 0ull;
        sUsedPicks = 0;
        sColoc = 0;
    }
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
    const unsigned long long Qall = (unsigned long long)block_sum((long long)part, sRed);
    if (tid == 0) sQ = Qall;
    const double invQ = Qall > 0ull ? 1.0 / (double)Qall : 0.0;

    // ---- the pick sequence, in parallel ----
    // candidates per expert at threshold Q/(G+E)/2^lvl (one thread per expert)
    int total = 0;
    if (Qall > 0ull && G > 0) {
        for (int lvl = 0;; ++lvl) {
            int cnt = 0, cut = 0;
            if (tid < E) {
                const long long L = sL[tid];
                long long cap = G;
                if (min_tokens > 0u) cap = min(cap, L / (long long)min_tokens - 1);
                if (L > 0 && cap > 0) {
                    const unsigned long long num = (unsigned long long)L * (unsigned)(G + E);
                    long long th;
                    if (lvl >= 10 && num >= Qall) th = cap;  // num 2^lvl / Q >= 1024 > cap
                    else th = (long long)floor_div_exact(num << lvl, Qall, invQ);
                    cnt = (int)min(cap, th);
                    cut = th < cap;
                }
                sCnt[tid] = cnt;
            }
            const long long both = block_sum(((long long)cut << 32) | cnt, sRed);
            total = (int)(both & 0xffffffffll);
            if (total >= G || (both >> 32) == 0 || lvl >= 33) break;
        }
    } else if (tid < E) {
        sCnt[tid] = 0;
    }
    __syncthreads();
    // exclusive scan of the counts (E <= 256 <= blockDim)
    {
        const int c = tid < E ? sCnt[tid] : 0;
        int incl = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(kFull, incl, off);
            if (lane >= off) incl += o;
        }
        if (lane == 31) sWarpSum[warp] = incl;
        __syncthreads();
        int wofs = 0;
        for (int w = 0; w < warp; ++w) wofs += sWarpSum[w];
        __syncthreads();
        if (tid < E) sCnt[tid] = wofs + incl - c;
        if (tid == 0) sCnt[E] = total;
    }
    __syncthreads();
    // the keys: position p belongs to the expert whose range holds it
    for (int p = tid; p < total; p += blockDim.x) {
        int lo = 0, hi = E - 1;  // last e with sCnt[e] <= p
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (sCnt[mid] <= p) lo = mid;
            else hi = mid - 1;
        }
        const int e = lo;
        const unsigned c = (unsigned)(p - sCnt[e] + 1);
        const unsigned long long x = (unsigned long long)sL[e] << kRatioShift;
        const unsigned long long ratio = c == 1u ? x : __umul64hi(x, sRecip[c]);
        sKey[p] = (ratio << 16) | ((unsigned long long)(255 - e) << 8) | (c - 1u);
    }
    __syncthreads();
    // pick order: a key's place is the number of larger keys (keys are
    // distinct), counted against every candidate (broadcast reads); the first
    // G places are kept
    for (int p = tid; p < total; p += blockDim.x) {
        const unsigned long long key = sKey[p];
        int place = 0;
        int q = 0;
        const ulonglong2* key2 = reinterpret_cast<const ulonglong2*>(sKey);
        for (; q + 4 <= total; q += 4) {
            const ulonglong2 a = key2[q >> 1], b = key2[(q >> 1) + 1];
            place += (a.x > key) + (a.y > key) + (b.x > key) + (b.y > key);
        }
        for (; q < total; ++q) place += sKey[q] > key;
        if (place < G) sOrd[place] = key;
    }
    __syncthreads();
    const int npicks = min(G, total);
    for (int t = tid; t <= npicks && t < G + 1; t += blockDim.x) {
        if (t == npicks) {
            sPick[t] = Pick{-1, 0u, 0u, 0u, 0u, 0};
        } else {
            const unsigned long long key = sOrd[t];
            const int e = 255 - (int)((key >> 8) & 255ull);
            const unsigned c = (unsigned)(key & 255ull) + 1u;  // copies before the pick
            const unsigned ce = c + 1u;
            const unsigned Le = (unsigned)sL[e];
            const unsigned qb = div_by(Le, ce, sRecip);
            const unsigned rem = Le - qb * ce;
            const unsigned q0_new = qb + (rem > 0u ? 1u : 0u);
            const unsigned q0_old = div_by(Le + c - 1u, c, sRecip);
            sPick[t] = Pick{e, ce, qb, rem, q0_new - q0_old, e / M};
        }
    }
    __syncthreads();

    if (warp == 0) {
        // ---- rank side: stop test, least loaded free rank, bookkeeping ----
        const long long Q = (long long)sQ;
        // the stop test 50 R max_r load_r <= 51 Q, as max_r load_r <= floor(51 Q / (50 R))
        const unsigned stop_max = (unsigned)((51LL * Q) / (50LL * R));
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
#pragma unroll
        for (int j = 0; j < NJR; ++j) max_before = max(max_before, load[j]);
        max_before = __reduce_max_sync(kFull, max_before);
        // with every rank load below 2^25 (Q < 2^25), a rank's load and its
        // index (< 128) pack into one 32-bit key, and the least loaded rank
        // with a free slot (ties to the lowest r) is one reduction
        const bool packed = Q < (1LL << 25);
        Pick pk = sPick[0];
        for (;;) {
            // the next pick is read now, so that its load overlaps the
            // reductions (iters + 1 <= G always: the loop stops once every
            // slot is used)
            const Pick pk_next = sPick[min(iters + 1, kMaxG)];
            // the stop test as a vote: is any load above stop_max?
            bool over = false;
            unsigned bestl = 0xffffffffu, bestr = 0xffffffffu;
            int rstar;
            if (packed) {
                unsigned key = 0xffffffffu;
#pragma unroll
                for (int j = 0; j < NJR; ++j) {
                    over = over || load[j] > stop_max;
                    if (used[j] < S) key = min(key, (load[j] << 7) | (unsigned)(lane + 32 * j));
                }
                const bool any_over = __any_sync(kFull, over);
                key = __reduce_min_sync(kFull, key);
                if (!any_over) break;
                if (key == 0xffffffffu) break;  // no free slot anywhere
                rstar = (int)(key & 127u);
            } else {
#pragma unroll
                for (int j = 0; j < NJR; ++j) {
                    over = over || load[j] > stop_max;
                    if (used[j] < S && load[j] < bestl) {
                        bestl = load[j];
                        bestr = (unsigned)(lane + 32 * j);
                    }
                }
                const bool any_over = __any_sync(kFull, over);
                const unsigned ml = __reduce_min_sync(kFull, bestl);
                if (!any_over) break;
                if (ml == 0xffffffffu) break;  // no free slot anywhere
                rstar = (int)__reduce_min_sync(kFull, bestl == ml ? bestr : 0xffffffffu);
            }

            if (pk.e < 0) break;  // no expert may take another copy
            const int estar = pk.e;
            const int rj = rstar >> 5;  // warp-uniform, as are rm and first
            const bool rown = lane == (rstar & 31);
            const int rm = pk.rm;
            const bool mown = lane == (rm & 31);
            const bool first = pk.c == 2u;
            // without branches on the lane: the new copy goes into r*'s lowest
            // free slot; a first replica takes floor(L/2) (L mod 2 < 2 keeps
            // the +1 on the master, the only other copy); the master's quota
            // change lands on its rank's owner
#pragma unroll
            for (int j = 0; j < NJR; ++j) {
                const bool own = rown && j == rj;
                const int sn = used[j];
#pragma unroll
                for (int s = 0; s < SM; ++s) {
                    const bool here = own && s == sn;
                    slotE[j][s] = here ? estar : slotE[j][s];
                    slotQ[j][s] = (here && first) ? (int)pk.qb : slotQ[j][s];
                }
                used[j] += own ? 1 : 0;
                unsigned add = (own && first) ? pk.qb : 0u;
                add += (mown && j == (rm >> 5)) ? pk.dq0 : 0u;
                load[j] += add;
            }
            if (!first) {
                // replicas, ascending slot g = r*S + s (r = lane + 32 j)
                unsigned before = 0u;
                const unsigned lt = (1u << lane) - 1u;
#pragma unroll
                for (int j = 0; j < NJR; ++j) {
                    unsigned lower = 0u;   // e* replicas in lower lanes of group j
                    unsigned grp = 0u;     // e* replicas in group j
#pragma unroll
                    for (int s = 0; s < SM; ++s) {
                        const unsigned msk = __ballot_sync(kFull, s < S && slotE[j][s] == estar);
                        lower += __popc(msk & lt);
                        grp += __popc(msk);
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
                    before += grp;
                }
            }
            iters += 1;
            pk = pk_next;
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

template <int NJR>
cudaError_t launch_s(const Sizes& z, const int32_t* load_e, unsigned m, const ue_placement& out,
                     int* err, cudaStream_t st)
{
    if (z.S <= 2)
        plan_kernel<NJR, 2><<<1, kPlanThreads, 0, st>>>(load_e, z.R, z.E, z.S, m, out, err);
    else
        plan_kernel<NJR, 8><<<1, kPlanThreads, 0, st>>>(load_e, z.R, z.E, z.S, m, out, err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_plan(const Sizes& z, const int32_t* load_e, int min_tokens,
                        const ue_placement& out, int* err, cudaStream_t st)
{
    const unsigned m = (unsigned)min_tokens;
    if (z.R <= 32) return launch_s<1>(z, load_e, m, out, err, st);
    if (z.R <= 64) return launch_s<2>(z, load_e, m, out, err, st);
    return launch_s<4>(z, load_e, m, out, err, st);
}

}  // namespace ue
