// k_reroute.cu -- logical -> physical routing (the pages' reroute).
//
// "UltraEP" README, "Interface / 2. Forward and backward": reroute expands
// logical routing to physical replicas. Pairs are taken in global order
// (rank, token, k) and fill each expert's copies by prefix sum: the o-th pair
// of expert e (o counted in that order) goes to the copy j whose quota range
// [start_j, start_j + q_j) holds o, copies ordered master first, then replicas
// by ascending redundant slot, at dispatch row slot_offset[p] + (o - start_j).
// With the plan's quotas q_j = b + [j < rem] (b = floor(L/c), rem = L mod c),
// j and the offset follow from o by one division.
//
// Design (B200): a single-pass stable counting sort with a decoupled
// look-back. Each CTA takes a tile of 4096 pairs by an atomic ticket (so every
// tile it waits on is already running), stages the ids in shared memory and
// counts them per warp sub-range, then publishes its per-expert tile counts
// at once so that successors never wait on its later work. While its
// predecessors finish, it rebuilds the plan's copy lists (at most 512
// entries). The look-back runs one thread per expert column and reads a
// window of 16 predecessors per step with independent loads, adding their
// counts until it meets an inclusive prefix; with every tile resident at
// once this cuts the serial chain of L2 round trips by the window width.
// Every wait is bounded: when it runs out the tile publishes an error flag,
// records UE_ERR_TIMEOUT and writes nothing. Finally each warp re-walks its
// 512 pairs in order, ranking equal ids within 32 lanes by popcount of the
// lanes that match, and writes the physical slot and dispatch row.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kTile = kRerouteTile;
constexpr int kThreads = kRerouteThreads;
constexpr int kWarps = kRerouteWarps;
constexpr int kPerWarp = kTile / kWarps;
constexpr int kRounds = kPerWarp / 32;
constexpr int kWindow = 16;  // predecessors read per look-back step

__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p)
{
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed(uint32_t* p, uint32_t v)
{
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__global__ void __launch_bounds__(kThreads)
reroute_kernel(const int32_t* __restrict__ idx, int64_t Q, int R, int E, int S,
               ue_placement plan, int32_t* __restrict__ phys_slot,
               int32_t* __restrict__ dest_row, uint32_t* status,
               uint32_t* tile_counter, int64_t spin_limit, int drop_first,
               int* err)
{
    __shared__ short s_idx[kTile];        // expert ids of the tile (-1: none)
    __shared__ int s_wh[kWarps][kMaxE];   // per-warp counts, then start offsets
    __shared__ int s_pre[kMaxE];          // tile prefix per expert
    __shared__ int s_cnt[kMaxE], s_lrep[kMaxE], s_run[kMaxE];
    __shared__ int s_L[kMaxE], s_b[kMaxE], s_rem[kMaxE];
    __shared__ int s_master[kMaxE], s_repstart[kMaxE];
    __shared__ int s_rep[kMaxG];          // replica slots, by expert then g
    __shared__ int s_off[kMaxE + kMaxG + 1];
    __shared__ int s_se[kMaxG];           // plan: slot_expert
    __shared__ int s_sq[kMaxE + kMaxG];   // plan: slot_quota
    __shared__ int s_wsum[kWarps];
    __shared__ int s_tile;
    __shared__ int s_fail;

    const int M = E / R;
    const int G = R * S;
    const int P = R * (M + S);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;

    if (tid == 0) {
        s_tile = (int)atomicAdd(tile_counter, 1u);
        s_fail = 0;
    }
    for (int x = tid; x < kWarps * kMaxE; x += kThreads) (&s_wh[0][0])[x] = 0;
    for (int e = tid; e < E; e += kThreads) {
        s_cnt[e] = 0;
        s_lrep[e] = 0;
        s_run[e] = 0;
    }
    __syncthreads();

    // ---- stage the tile and count it per warp sub-range ----
    const int tile = s_tile;
    const int64_t t0 = (int64_t)tile * kTile;
    const int cnt_tile = (int)min((int64_t)kTile, Q - t0);
    for (int x = tid; x < kTile; x += kThreads) {
        int e = -1;
        if (x < cnt_tile) {
            e = __ldg(idx + t0 + x);
            if ((unsigned)e >= (unsigned)E) {
                raise_error(err, UE_ERR_DEVICE_BOUNDS, (int)min(t0 + x, (int64_t)INT_MAX));
                e = -1;
            }
        }
        s_idx[x] = (short)e;
    }
    __syncthreads();
#pragma unroll 4
    for (int rd = 0; rd < kRounds; ++rd) {
        const int e = s_idx[warp * kPerWarp + rd * 32 + lane];
        if (e >= 0) atomicAdd(&s_wh[warp][e], 1);
    }
    __syncthreads();

    // ---- publish this tile's counts ----
    int acc = 0;
    uint32_t* mine = status + (size_t)tile * E + tid;
    if (tid < E) {
        for (int w = 0; w < kWarps; ++w) {
            const int t = s_wh[w][tid];
            s_wh[w][tid] = acc;
            acc += t;
        }
        if (tile == 0) {
            if (!drop_first) st_relaxed(mine, (kFlagPrefix << 30) | (uint32_t)acc);
        } else {
            st_relaxed(mine, (kFlagAggregate << 30) | (uint32_t)acc);
        }
    }

    // ---- copy lists of every expert, from the plan (overlaps the wait) ----
    for (int p = tid; p <= P; p += kThreads) s_off[p] = __ldg(plan.slot_offset + p);
    for (int p = tid; p < P; p += kThreads) s_sq[p] = __ldg(plan.slot_quota + p);
    for (int g = tid; g < G; g += kThreads) s_se[g] = __ldg(plan.slot_expert + g);
    __syncthreads();
    for (int g = tid; g < G; g += kThreads) {
        const int e = s_se[g];
        if (e >= 0 && e < E) {
            const int p = (g / S) * (M + S) + M + (g % S);
            atomicAdd(&s_cnt[e], 1);
            atomicAdd(&s_lrep[e], s_sq[p]);
        } else if (e >= E) {
            raise_error(err, UE_ERR_DEVICE_BOUNDS, g);
        }
    }
    __syncthreads();
    {
        // exclusive scan of replica counts over experts (E <= kThreads)
        const int c = tid < E ? s_cnt[tid] : 0;
        int incl = c;
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
            const int e = tid;
            const int mp = (e / M) * (M + S) + (e % M);
            const int copies = 1 + c;
            const int L = s_sq[mp] + s_lrep[e];
            const int b = L / copies;
            s_L[e] = L;
            s_b[e] = b;
            s_rem[e] = L - b * copies;
            s_master[e] = mp;
            s_repstart[e] = wofs + incl - c;
        }
        __syncthreads();
    }
    if (warp == 0) {
        // replica slots in ascending g within each expert
        for (int g0 = 0; g0 < G; g0 += 32) {
            const int g = g0 + lane;
            int e = -1;
            if (g < G) {
                e = s_se[g];
                if (e >= E) e = -1;
            }
            const unsigned peers = __match_any_sync(kFull, e);
            if (e >= 0) {
                const int pos = s_run[e] + __popc(peers & ((1u << lane) - 1u));
                s_rep[s_repstart[e] + pos] = (g / S) * (M + S) + M + (g % S);
            }
            __syncwarp();
            if (e >= 0 && lane == __ffs(peers) - 1) s_run[e] += __popc(peers);
            __syncwarp();
        }
    }

    // ---- look back over predecessor tiles, publish the inclusive prefix ----
    if (tid < E) {
        if (tile == 0) {
            s_pre[tid] = 0;
        } else {
            uint32_t excl = 0;
            int base = tile - 1;  // nearest predecessor not yet added
            int64_t polls = 0;
            bool fail = false, done = false;
            while (!done && !fail) {
                uint32_t v[kWindow];
#pragma unroll
                for (int i = 0; i < kWindow; ++i)
                    v[i] = (base - i >= 0) ? ld_relaxed(status + (size_t)(base - i) * E + tid)
                                           : (kFlagPrefix << 30);
#pragma unroll
                for (int i = 0; i < kWindow; ++i) {
                    if (!done && !fail) {
                        uint32_t sw = v[i];
                        while ((sw >> 30) == kFlagInvalid && !fail) {
                            if (++polls > spin_limit) {
                                raise_error(err, UE_ERR_TIMEOUT, tile);
                                fail = true;
                            } else {
                                __nanosleep(64);
                                sw = ld_relaxed(status + (size_t)(base - i) * E + tid);
                            }
                        }
                        if ((sw >> 30) == kFlagError) fail = true;
                        if (!fail) {
                            if (base - i >= 0) excl += sw & kValueMask;
                            if ((sw >> 30) == kFlagPrefix) done = true;
                        }
                    }
                }
                base -= kWindow;
            }
            if (fail) {
                st_relaxed(mine, kFlagError << 30);
                atomicOr(&s_fail, 1);
            } else {
                st_relaxed(mine, (kFlagPrefix << 30) | ((excl + (uint32_t)acc) & kValueMask));
                s_pre[tid] = (int)excl;
            }
        }
    }
    __syncthreads();
    if (s_fail) return;
    if (tid < E) {
        const int pre = s_pre[tid];
        for (int w = 0; w < kWarps; ++w) s_wh[w][tid] += pre;
    }
    __syncthreads();

    // ---- in-order ranks, copy, dispatch row ----
#pragma unroll 1
    for (int rd = 0; rd < kRounds; ++rd) {
        const int x = warp * kPerWarp + rd * 32 + lane;
        const int e = s_idx[x];
        const unsigned peers = __match_any_sync(kFull, e);
        int o = 0;
        if (e >= 0) o = s_wh[warp][e] + __popc(peers & ((1u << lane) - 1u));
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) s_wh[warp][e] += __popc(peers);
        __syncwarp();
        if (x < cnt_tile) {
            int p = -1, row = -1;
            if (e >= 0) {
                if (o < s_L[e]) {
                    const int b = s_b[e], rem = s_rem[e];
                    const int thr = rem * (b + 1);
                    int j, off;
                    if (o < thr) {
                        j = o / (b + 1);
                        off = o - j * (b + 1);
                    } else {
                        const int o2 = o - thr;
                        j = rem + o2 / b;
                        off = o2 - (j - rem) * b;
                    }
                    p = (j == 0) ? s_master[e] : s_rep[s_repstart[e] + j - 1];
                    row = s_off[p] + off;
                } else {
                    // the plan does not cover this pair (plan from other ids)
                    raise_error(err, UE_ERR_DEVICE_BOUNDS, (int)min(t0 + x, (int64_t)INT_MAX));
                }
            }
            phys_slot[t0 + x] = p;
            dest_row[t0 + x] = row;
        }
    }
}

}  // namespace

cudaError_t launch_reroute(const Sizes& z, const int32_t* idx,
                           const ue_placement& plan, int32_t* phys_slot,
                           int32_t* dest_row, uint32_t* status,
                           uint32_t* tile_counter, int64_t spin_limit,
                           int drop_first, int* err, cudaStream_t st)
{
    if (z.Q == 0) return cudaSuccess;
    const int64_t tiles = (z.Q + kTile - 1) / kTile;
    cudaError_t ce = cudaMemsetAsync(status, 0, sizeof(uint32_t) * (size_t)tiles * z.E, st);
    if (ce != cudaSuccess) return ce;
    ce = cudaMemsetAsync(tile_counter, 0, sizeof(uint32_t), st);
    if (ce != cudaSuccess) return ce;
    reroute_kernel<<<(unsigned)tiles, kThreads, 0, st>>>(
        idx, z.Q, z.R, z.E, z.S, plan, phys_slot, dest_row, status, tile_counter,
        spin_limit, drop_first, err);
    return cudaGetLastError();
}

}  // namespace ue
