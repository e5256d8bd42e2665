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
// Design: one CTA per expert. The passes are short serial walks (at most
// 1 + G copies and R sources) done by one thread in shared memory; they
// produce at most 2*(1 + G) + R nonzero entries, each (r, j) at most once
// (after copy j's local step either its host has no pairs left or its quota
// is full), so the block zeroes the expert's [R] x [copies] block of the
// output and then stores the entries. The row offsets are a scan over r per
// copy. Empty redundant slots are written by the CTA of their rank's first
// master.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kSplitThreads = 128;
constexpr int kMaxEntries = 2 * (1 + kMaxG) + kMaxR;

__global__ void __launch_bounds__(kSplitThreads)
locality_split_kernel(const int32_t* __restrict__ load_re, int R, int E, int S,
                      ue_placement plan, int32_t* __restrict__ src_quota,
                      int32_t* __restrict__ src_offset, int* err)
{
    __shared__ int s_cp[1 + kMaxG];   // physical slot of copy j
    __shared__ int s_q[1 + kMaxG];    // quota left of copy j
    __shared__ int s_s[kMaxR];        // pairs left of source rank r
    __shared__ int s_er[kMaxEntries], s_ej[kMaxEntries], s_ea[kMaxEntries];
    __shared__ int s_n, s_ne, s_bad;
    const int e = blockIdx.x;
    const int M = E / R;
    const int G = R * S;
    const int P = R * (M + S);
    const int tid = threadIdx.x;
    const int h0 = e / M;

    if (tid < 32) {
        int n = 1;
        if (tid == 0) s_cp[0] = h0 * (M + S) + e % M;
        for (int g0 = 0; g0 < G; g0 += 32) {
            const int g = g0 + tid;
            const bool mine = g < G && __ldg(plan.slot_expert + g) == e;
            const unsigned b = __ballot_sync(kFull, mine);
            if (mine) s_cp[n + __popc(b & ((1u << tid) - 1u))] = (g / S) * (M + S) + M + g % S;
            n += __popc(b);
        }
        if (tid == 0) {
            s_n = n;
            s_ne = 0;
            s_bad = 0;
        }
    }
    for (int r = tid; r < R; r += blockDim.x) s_s[r] = __ldg(load_re + (size_t)r * E + e);
    __syncthreads();
    const int n = s_n;
    for (int j = tid; j < n; j += blockDim.x) s_q[j] = __ldg(plan.slot_quota + s_cp[j]);
    for (int x = tid; x < R * n; x += blockDim.x) {
        const int r = x / n, j = x - r * n;
        src_quota[(size_t)r * P + s_cp[j]] = 0;
    }
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
    if (tid == 0) {
        long long sum_s = 0, sum_q = 0;
        for (int r = 0; r < R; ++r) sum_s += s_s[r];
        for (int j = 0; j < n; ++j) sum_q += s_q[j];
        int ne = 0;
        if (sum_s != sum_q) {
            raise_error(err, UE_ERR_DEVICE_BOUNDS, e);
            s_bad = 1;
        } else {
            // local pass
            for (int j = 0; j < n; ++j) {
                const int h = s_cp[j] / (M + S);
                const int a = min(s_s[h], s_q[j]);
                if (a > 0) {
                    s_er[ne] = h;
                    s_ej[ne] = j;
                    s_ea[ne] = a;
                    ++ne;
                    s_s[h] -= a;
                    s_q[j] -= a;
                }
            }
            // remote pass: sources in ascending r (what earlier copies took
            // is gone, so one pointer over r serves every copy)
            int r = 0;
            for (int j = 0; j < n; ++j) {
                while (s_q[j] > 0 && r < R) {
                    const int a = min(s_s[r], s_q[j]);
                    if (a > 0) {
                        s_er[ne] = r;
                        s_ej[ne] = j;
                        s_ea[ne] = a;
                        ++ne;
                        s_s[r] -= a;
                        s_q[j] -= a;
                    }
                    if (s_s[r] == 0) ++r;
                }
            }
        }
        s_ne = ne;
    }
    __syncthreads();
    const int ne = s_ne;
    for (int x = tid; x < ne; x += blockDim.x)
        src_quota[(size_t)s_er[x] * P + s_cp[s_ej[x]]] = s_ea[x];
    __syncthreads();
    for (int j = tid; j < n; j += blockDim.x) {
        const int p = s_cp[j];
        int run = __ldg(plan.slot_offset + p);
        for (int r = 0; r < R; ++r) {
            src_offset[(size_t)r * P + p] = run;
            run += src_quota[(size_t)r * P + p];
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
