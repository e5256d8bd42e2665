// k_split.cu -- locality-aware split of every copy's quota over the source
// ranks.
//
// "UltraEP" README, "Performance Tuning / Replication planning": a
// locality-aware per-rank quota decomposition cuts remote traffic. The pages
// name the knob only; the rule implemented here is this library's reading:
// for expert e with copies j in copy order (master first, then replicas by
// ascending redundant slot g) on host ranks h_j with quotas q_j, and
// per-source-rank loads s_r (load_re[r][e], which must sum to the quotas):
//   local pass:  every copy j, in copy order, first takes min(s_{h_j}, q_j)
//                pairs from its own host rank;
//   remote pass: every copy j, in copy order, fills the rest of its quota
//                from the source ranks in ascending r.
// Outputs, rank-major [R][P]:
//   src_quota[r][p]   pairs of source rank r assigned to slot p;
//   src_offset[r][p]  dispatch row of the first of them: a slot holds its
//                     pairs by source rank, then in the source's own order.
//
// Design: one CTA per expert, no serial walk. The remote pass is the
// north-west-corner fill of the copies' remaining quotas (copy order) from
// the sources' remaining pairs (ascending r), so the pairs source r gives
// copy j are the overlap of j's interval [A_j, A_j + q'_j) and r's interval
// [B_r, B_r + s'_r) on the line of cumulative remainders (A, B exclusive
// prefix sums). Steps: each copy's own-rank take (a thread per copy; copies
// that share a host are taken in copy order), the remainders, two warp
// scans, and one thread per copy sweeping the source ranks once to write both
// output columns (pairs and first row) with no global reads. Empty redundant
// slots are written by the CTA of their rank's first master.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kSplitThreads = 128;
constexpr int kMaxCopies = 1 + kMaxG;

// exclusive scan of v[0..n) into out[0..n), by one warp; returns the total
__device__ int warp_exclusive_scan(const int* v, int* out, int n, int lane)
{
    int base = 0;
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        const int x = i < n ? v[i] : 0;
        int incl = x;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(kFull, incl, off);
            if (lane >= off) incl += y;
        }
        if (i < n) out[i] = base + incl - x;
        base += __shfl_sync(kFull, incl, 31);
    }
    return base;
}

__global__ void __launch_bounds__(kSplitThreads)
locality_split_kernel(const int32_t* __restrict__ load_re, int R, int E, int S,
                      ue_placement plan, int32_t* __restrict__ src_quota,
                      int32_t* __restrict__ src_offset, int* err)
{
    __shared__ int s_cp[kMaxCopies];   // physical slot of copy j
    __shared__ int s_q[kMaxCopies];    // quota of copy j, then what is left after its own-rank take
    __shared__ int s_loc[kMaxCopies];  // pairs copy j takes from its own rank
    __shared__ int s_A[kMaxCopies];    // exclusive prefix of the copies' remainders
    __shared__ int s_s[kMaxR];         // pairs of source rank r, then what is left
    __shared__ int s_B[kMaxR];         // exclusive prefix of the sources' remainders
    __shared__ int s_n, s_tq, s_ts;
    const int e = blockIdx.x;
    const int M = E / R;
    const int G = R * S;
    const int P = R * (M + S);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int h0 = e / M;

    if (warp == 0) {
        // copies in copy order: the master, then replicas by ascending g
        int n = 1;
        if (lane == 0) s_cp[0] = h0 * (M + S) + e % M;
        for (int g0 = 0; g0 < G; g0 += 32) {
            const int g = g0 + lane;
            const bool mine = g < G && __ldg(plan.slot_expert + g) == e;
            const unsigned b = __ballot_sync(kFull, mine);
            if (mine) s_cp[n + __popc(b & ((1u << lane) - 1u))] = (g / S) * (M + S) + M + g % S;
            n += __popc(b);
        }
        if (lane == 0) s_n = n;
    }
    for (int r = tid; r < R; r += blockDim.x) s_s[r] = __ldg(load_re + (size_t)r * E + e);
    if (e % M == 0) {
        // empty redundant slots of this rank: no pairs, rows at the slot's start
        for (int x = tid; x < R * S; x += blockDim.x) {
            const int r = x / S, sl = x - r * S;
            const int g = h0 * S + sl;
            const int se = __ldg(plan.slot_expert + g);
            if (se < 0 || se >= E) {
                const int p = h0 * (M + S) + M + sl;
                src_quota[(size_t)r * P + p] = 0;
                src_offset[(size_t)r * P + p] = __ldg(plan.slot_offset + p);
                if (se >= E && r == 0) raise_error(err, UE_ERR_DEVICE_BOUNDS, g);
            }
        }
    }
    __syncthreads();
    const int n = s_n;
    for (int j = tid; j < n; j += blockDim.x) s_q[j] = __ldg(plan.slot_quota + s_cp[j]);
    __syncthreads();
    // local pass: copy j takes min(what its host has left, its quota); the
    // copies before it on the same host have taken first
    for (int j = tid; j < n; j += blockDim.x) {
        const int h = s_cp[j] / (M + S);
        int left = s_s[h], take = 0;
        for (int jj = 0; jj <= j; ++jj) {
            if (s_cp[jj] / (M + S) != h) continue;
            take = min(left, s_q[jj]);
            left -= take;
        }
        s_loc[j] = take;
    }
    __syncthreads();
    for (int j = tid; j < n; j += blockDim.x) {
        s_q[j] -= s_loc[j];
        atomicSub(&s_s[s_cp[j] / (M + S)], s_loc[j]);
    }
    __syncthreads();
    // prefix sums of the remainders (copies in copy order, sources by r)
    if (warp == 0) {
        const int t = warp_exclusive_scan(s_q, s_A, n, lane);
        if (lane == 0) s_tq = t;
    } else if (warp == 1) {
        const int t = warp_exclusive_scan(s_s, s_B, R, lane);
        if (lane == 0) s_ts = t;
    }
    __syncthreads();
    // the loads must sum to the quotas (equal local takes leave the
    // remainders' totals equal exactly when they do)
    const bool ok = s_tq == s_ts;
    if (!ok && tid == 0) raise_error(err, UE_ERR_DEVICE_BOUNDS, e);
    for (int j = tid; j < n; j += blockDim.x) {
        const int p = s_cp[j];
        const int h = p / (M + S);
        const int a0 = s_A[j], a1 = a0 + s_q[j];
        int run = __ldg(plan.slot_offset + p);
        for (int r = 0; r < R; ++r) {
            int x = 0;
            if (ok) {
                const int b0 = s_B[r], b1 = b0 + s_s[r];
                x = max(0, min(a1, b1) - max(a0, b0)) + (r == h ? s_loc[j] : 0);
            }
            src_quota[(size_t)r * P + p] = x;
            src_offset[(size_t)r * P + p] = run;
            run += x;
        }
    }
}

}  // namespace

cudaError_t launch_locality_split(const Sizes& z, const int32_t* load_re,
                                  const ue_placement& plan, int32_t* src_quota,
                                  int32_t* src_offset, int* err, cudaStream_t st)
{
    locality_split_kernel<<<z.E, kSplitThreads, 0, st>>>(load_re, z.R, z.E, z.S, plan,
                                                         src_quota, src_offset, err);
    return cudaGetLastError();
}

}  // namespace ue
