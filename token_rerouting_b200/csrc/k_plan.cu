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
// (exact: L_a*c_b > L_b*c_a, ties to the lowest e), r* = argmin load_r over
// ranks with a free slot (ties to the lowest r); the copy goes into r*'s
// lowest free slot.
//
// Design (B200): the loop is serial (at most G iterations) and latency
// bound, so it runs on one warp of one CTA with the whole state in shared
// memory: rank loads, used-slot counts, L_e, c_e and every copy's current
// quota. An iteration is a handful of warp reductions (redux max/min for the
// rank side, a shuffle butterfly with exact cross-multiplied comparisons for
// the expert side) and an incremental update of the chosen expert's quotas:
// the position of each of its replicas in copy order comes from a ballot over
// the slot array, and each changed quota moves its rank's load by the
// difference. The rest of the CTA writes the outputs and scans the slot
// offsets at the end.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kPlanThreads = 256;
constexpr int kPlanWarps = kPlanThreads / 32;

__global__ void __launch_bounds__(kPlanThreads)
plan_kernel(const int32_t* __restrict__ load_e, int R, int E, int S,
            ue_placement out, int* err)
{
    __shared__ int sL[kMaxE];       // exact load per expert
    __shared__ int sC[kMaxE];       // copies per expert
    __shared__ int sMq[kMaxE];      // quota of each expert's master
    __shared__ int sRank[kMaxR];    // rank loads
    __shared__ int sUsed[kMaxR];    // used redundant slots per rank
    __shared__ int sSlotE[kMaxG];   // expert of redundant slot g, -1 empty
    __shared__ int sSlotQ[kMaxG];   // quota of redundant slot g
    __shared__ unsigned long long sQ;
    __shared__ int sStats[4];
    __shared__ int sWarpSum[kPlanWarps];

    const int M = E / R;
    const int G = R * S;
    const int P = R * (M + S);
    const int tid = threadIdx.x;

    if (tid == 0) sQ = 0ull;
    for (int r = tid; r < R; r += blockDim.x) {
        sRank[r] = 0;
        sUsed[r] = 0;
    }
    for (int g = tid; g < G; g += blockDim.x) {
        sSlotE[g] = -1;
        sSlotQ[g] = 0;
    }
    __syncthreads();
    unsigned long long part = 0ull;
    for (int e = tid; e < E; e += blockDim.x) {
        int L = __ldg(load_e + e);
        if (L < 0) {
            raise_error(err, UE_ERR_DEVICE_BOUNDS, e);
            L = 0;
        }
        sL[e] = L;
        sC[e] = 1;
        sMq[e] = L;
        atomicAdd(&sRank[e / M], L);
        part += (unsigned long long)L;
    }
    if (part) atomicAdd(&sQ, part);
    __syncthreads();

    if (tid < 32) {
        const int lane = tid;
        const long long Q = (long long)sQ;
        int iters = 0, colocated = 0;
        unsigned max_before = 0u;
        for (;;) {
            // rank side: max load (stop test) and least-loaded rank with a
            // free slot; lane covers ranks lane, lane+32, ...
            unsigned maxl = 0u, bestl = 0xffffffffu, bestr = 0xffffffffu;
#pragma unroll
            for (int j = 0; j < kMaxR / 32; ++j) {
                const int r = lane + 32 * j;
                if (r < R) {
                    const unsigned ld = (unsigned)sRank[r];
                    maxl = max(maxl, ld);
                    if (sUsed[r] < S && ld < bestl) {
                        bestl = ld;
                        bestr = (unsigned)r;
                    }
                }
            }
            maxl = __reduce_max_sync(kFull, maxl);
            if (iters == 0) max_before = maxl;
            if (50LL * R * (long long)maxl <= 51LL * Q) break;
            const unsigned ml = __reduce_min_sync(kFull, bestl);
            if (ml == 0xffffffffu) break;  // no free slot anywhere
            const int rstar = (int)__reduce_min_sync(kFull, bestl == ml ? bestr : 0xffffffffu);

            // expert side: argmax L_e / c_e, exact, ties to the lowest e
            int bL = -1, bc = 1, be = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < kMaxE / 32; ++j) {
                const int e = lane + 32 * j;
                if (e < E) {
                    const int Le = sL[e], ce = sC[e];
                    if (bL < 0 || (long long)Le * bc > (long long)bL * ce) {
                        bL = Le;
                        bc = ce;
                        be = e;
                    }
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const int oL = __shfl_xor_sync(kFull, bL, off);
                const int oc = __shfl_xor_sync(kFull, bc, off);
                const int oe = __shfl_xor_sync(kFull, be, off);
                const long long lhs = (long long)oL * bc, rhs = (long long)bL * oc;
                const bool take = oL >= 0 && (bL < 0 || lhs > rhs || (lhs == rhs && oe < be));
                if (take) {
                    bL = oL;
                    bc = oc;
                    be = oe;
                }
            }
            const int estar = be;

            // place the copy in r*'s lowest free slot
            const int s = sUsed[rstar];
            const int g = rstar * S + s;
            const bool held = lane < S && sSlotE[rstar * S + lane] == estar;
            if (estar / M == rstar || __any_sync(kFull, held)) colocated += 1;
            __syncwarp();
            if (lane == 0) {
                sSlotE[g] = estar;
                sUsed[rstar] = s + 1;
                sC[estar] += 1;
            }
            __syncwarp();

            // new quotas of e*'s copies; each change moves its rank's load
            const int c = sC[estar];
            const int L = sL[estar];
            const int qb = L / c;
            const int rem = L - qb * c;
            if (lane == 0) {
                const int q0 = qb + (rem > 0 ? 1 : 0);
                atomicAdd(&sRank[estar / M], q0 - sMq[estar]);
                sMq[estar] = q0;
            }
            int before = 0;  // replicas of e* at lower slot indices
#pragma unroll
            for (int j = 0; j < kMaxG / 32; ++j) {
                const int gg = 32 * j + lane;
                const bool has = gg < G && sSlotE[gg] == estar;
                const unsigned msk = __ballot_sync(kFull, has);
                if (has) {
                    const int pos = 1 + before + __popc(msk & ((1u << lane) - 1u));
                    const int qn = qb + (pos < rem ? 1 : 0);
                    atomicAdd(&sRank[gg / S], qn - sSlotQ[gg]);
                    sSlotQ[gg] = qn;
                }
                before += __popc(msk);
            }
            __syncwarp();
            iters += 1;
        }
        unsigned mx = 0u;
#pragma unroll
        for (int j = 0; j < kMaxR / 32; ++j) {
            const int r = lane + 32 * j;
            if (r < R) mx = max(mx, (unsigned)sRank[r]);
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
    // thread owns slots 2*tid and 2*tid+1 (P <= 512)
    int q2[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int p = 2 * tid + h;
        int q = 0;
        if (p < P) {
            const int r = p / (M + S);
            const int l = p - r * (M + S);
            q = (l < M) ? sMq[r * M + l] : sSlotQ[r * S + (l - M)];
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

}  // namespace

cudaError_t launch_plan(const Sizes& z, const int32_t* load_e,
                        const ue_placement& out, int* err, cudaStream_t st)
{
    plan_kernel<<<1, kPlanThreads, 0, st>>>(load_e, z.R, z.E, z.S, out, err);
    return cudaGetLastError();
}

}  // namespace ue
