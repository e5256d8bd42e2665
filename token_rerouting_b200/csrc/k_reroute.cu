// k_reroute.cu -- logical -> physical routing (the pages' reroute).
//
// "UltraEP" README, "Interface / 2. Forward and backward": reroute expands
// logical routing to physical replicas. Pairs are taken in global order
// (rank, token, k) and fill each expert's copies by prefix sum: the o-th pair
// of expert e (o counted in that order) goes to the copy j whose quota range
// [start_j, start_j + q_j) holds o, copies ordered master first, then replicas
// by ascending redundant slot, at dispatch row slot_offset[p] + (o - start_j).
// With the greedy plan's quotas q_j = b + [j < rem] (b = floor(L/c),
// rem = L mod c), j and the offset follow from o by one division; for any
// other quotas (the capacity planner's) j is found by a binary search over
// the copies' starts.
//
// Two more orders ("UltraEP" README, "Performance Tuning / Replication
// planning"): the interleaved order takes the pairs token-major across the
// source ranks, (t, r, k), before the prefix fill, so that each copy draws
// from every source rank; the locality order hands each source rank's pairs
// of e, in the rank's own order, to e's copies in copy order, in the counts
// the locality-aware split gave that rank (a per-(source rank, slot) table
// of first occurrence and row base, built by local_tables_kernel).
//
// Design (B200): a single-pass stable counting sort with a decoupled
// look-back. Each CTA takes a tile of 8192 pairs by an atomic ticket (so every
// tile it waits on is already running), stages the ids in shared memory and
// counts them per warp sub-range, then publishes its per-expert tile counts
// at once so that successors never wait on its later work. While its
// predecessors finish, it rebuilds the plan's copy lists (at most 512
// entries). The look-back runs H = min(4, 512/E) threads per expert column;
// each reads 16 predecessors per step with independent loads, so one step
// covers 16*H tiles, and the column adds their counts up to the nearest
// inclusive prefix. With every tile resident at once this cuts the serial
// chain of L2 round trips by the window width.
// Every wait is bounded: when it runs out the tile publishes an error flag,
// records UE_ERR_TIMEOUT and writes nothing. Finally each warp re-walks its
// 512 pairs in order, ranking equal ids within 32 lanes (the lanes holding
// the same id come from nine ballots over the id's bits), and writes the
// physical slot and dispatch row; for floor-form quotas the copy index comes
// from one exact multiply-high by a per-expert reciprocal, otherwise from the
// binary search.
// The status words carry the launch's tag, so nothing is cleared between
// launches: words of earlier launches read as "not yet published". The last
// CTA to finish resets the ticket and the counter and advances the epoch.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kTile = kRerouteTile;
constexpr int kThreads = kRerouteThreads;
constexpr int kWarps = kRerouteWarps;
constexpr int kPerWarp = kTile / kWarps;
constexpr int kRounds = kPerWarp / 32;
constexpr int kWindow = 16;  // predecessors read per thread per look-back step
constexpr int kMaxH = 4;     // threads per expert column in the look-back

__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long* p)
{
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed(unsigned long long* p, unsigned long long v)
{
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// status word of this launch: tag, flag, count
__device__ __forceinline__ unsigned long long status_word(uint32_t tag, uint32_t flag, uint32_t v)
{
    return ((unsigned long long)tag << 32) | (flag << 30) | (v & kValueMask);
}

// the lanes of the warp holding the same key (9-bit keys): one ballot per bit
__device__ __forceinline__ unsigned same_key_lanes(int key)
{
    unsigned peers = kFull;
#pragma unroll
    for (int b = 0; b < 9; ++b) {
        const bool bit = (key >> b) & 1;
        const unsigned m = __ballot_sync(kFull, bit);
        peers &= bit ? m : ~m;
    }
    return peers;
}

// per-expert data used for every pair of the tile (16-byte aligned records)
struct alignas(16) ExpA {
    int pre;   // exclusive prefix of this expert before the tile
    int L;     // total pairs of the expert (sum of its quotas)
    int thr;   // rem * (b + 1): pairs held by the copies with quota b + 1
    int rem;   // copies with quota b + 1; -1: quotas not of that form
};
struct alignas(16) ExpB {
    unsigned long long m1;  // ceil(2^64 / (b + 1))
    unsigned long long m0;  // ceil(2^64 / b) (b >= 1), unused when b == 0
};
struct alignas(8) ExpC {
    int b;   // floor(L / c); the number of copies when rem == -1
    int cb;  // first entry of the expert in the copy table
};

// order of the pairs and their mapping to copies
constexpr int kOrderPrefix = 0;      // global order (r, t, k), prefix fill
constexpr int kOrderInterleave = 1;  // (t, r, k), prefix fill
constexpr int kOrderLocal = 2;       // per source rank, locality-aware split

struct OrderArgs {
    unsigned T, K, RK, TK;                 // RK = R*K, TK = T*K
    unsigned long long mK, mRK, mTK;       // ceil(2^64 / d) of K, RK, TK
    int P;
    const int32_t* first;  // [R][P] first occurrence index (local order)
    const int32_t* rowb;   // [R][P] dispatch row minus that index
    const int32_t* quota;  // [R][P] pairs of the source rank in the slot
};

// last j in [0, n) with key(j) <= o, for keys ascending in j and key(0) <= o
template <class Key>
__device__ __forceinline__ int last_at_most(int n, int o, Key key)
{
    int j = 0;
    for (int step = n > 1 ? 1 << (31 - __clz(n - 1)) : 0; step > 0; step >>= 1)
        if (j + step < n && key(j + step) <= o) j += step;
    return j;
}

// ceil(2^64 / d) for d >= 2; floor(x / d) = umul64hi(x, m) exactly when x*d < 2^64
__device__ __forceinline__ unsigned long long recip64(unsigned d)
{
    return d <= 1u ? 0ull : (0xffffffffffffffffull / d) + 1ull;
}

__device__ __forceinline__ unsigned div_m(unsigned x, unsigned d, unsigned long long m)
{
    return d == 1u ? x : (unsigned)__umul64hi((unsigned long long)x, m);
}

// pair index of the u-th pair in the scan order
template <int kOrder>
__device__ __forceinline__ int64_t pair_at(int64_t u, const OrderArgs& o)
{
    if (kOrder != kOrderInterleave) return u;
    const unsigned uu = (unsigned)u;
    const unsigned t = div_m(uu, o.RK, o.mRK);
    const unsigned w = uu - t * o.RK;
    const unsigned r = div_m(w, o.K, o.mK);
    const unsigned k = w - r * o.K;
    return ((int64_t)r * o.T + t) * o.K + k;
}

template <int kOrder>
__global__ void __launch_bounds__(kThreads)
reroute_kernel(const int32_t* __restrict__ idx, int64_t Q, int R, int E, int S,
               ue_placement plan, OrderArgs ord, int32_t* __restrict__ phys_slot,
               int32_t* __restrict__ dest_row, unsigned long long* status,
               uint32_t* sync, int64_t spin_limit, int drop_first,
               int* err)
{
    __shared__ short s_idx[kTile];        // expert ids of the tile (-1: none)
    __shared__ short s_wh[kWarps][kMaxE]; // per-warp counts, then in-tile offsets
    __shared__ ExpA s_a[kMaxE];
    __shared__ ExpB s_bm[kMaxE];
    __shared__ ExpC s_c[kMaxE];
    __shared__ int s_cp[kMaxE + kMaxG];   // copy table: physical slot, copies of
    __shared__ int s_cr[kMaxE + kMaxG];   // each expert in order; first dispatch row;
    __shared__ int s_cs[kMaxE + kMaxG];   // first pair index o of the copy
    __shared__ union {
        struct {  // building the copy table
            int cnt[kMaxE], run[kMaxE];
            int off[kMaxE + kMaxG + 1];   // plan: slot_offset
            int se[kMaxG];                // plan: slot_expert
            int sq[kMaxE + kMaxG];        // plan: slot_quota
        } pro;
        struct {  // look-back: one window segment per (h, e)
            uint32_t part[kMaxH][kMaxE];
            unsigned char state[kMaxH][kMaxE];
            unsigned char cdone[kMaxE];  // column finished
        } lb;
    } u;
    __shared__ int s_wsum[kWarps];
    __shared__ int s_tile;
    __shared__ uint32_t s_tag;
    __shared__ int s_fail;

    const int M = E / R;
    const int G = R * S;
    const int P = R * (M + S);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;

    if (tid == 0) {
        s_tile = (int)atomicAdd(&sync[0], 1u);
        // this launch's tag; the epoch only moves after every CTA has read it
        const uint32_t epoch = *reinterpret_cast<volatile uint32_t*>(&sync[2]);
        s_tag = epoch + 1u == 0u ? 1u : epoch + 1u;
        s_fail = 0;
    }
    for (int x = tid; x < kWarps * kMaxE; x += kThreads) (&s_wh[0][0])[x] = 0;
    for (int e = tid; e < E; e += kThreads) {
        u.pro.cnt[e] = 0;
        u.pro.run[e] = 0;
    }
    __syncthreads();

    // ---- stage the tile and count it per warp sub-range ----
    const int tile = s_tile;
    const uint32_t tag = s_tag;
    const int64_t t0 = (int64_t)tile * kTile;
    const int cnt_tile = (int)min((int64_t)kTile, Q - t0);
    {
        // issue all of this thread's loads before using any of them
        constexpr int kPer = kTile / kThreads;
        int v[kPer];
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int x = tid + q * kThreads;
            v[q] = x < cnt_tile ? __ldg(idx + pair_at<kOrder>(t0 + x, ord)) : -1;
        }
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int x = tid + q * kThreads;
            int e = v[q];
            if (x < cnt_tile && (unsigned)e >= (unsigned)E) {
                raise_error(err, UE_ERR_DEVICE_BOUNDS,
                            (int)min(pair_at<kOrder>(t0 + x, ord), (int64_t)INT_MAX));
                e = -1;
            }
            s_idx[x] = (short)e;
        }
    }
    __syncthreads();
#pragma unroll 4
    for (int rd = 0; rd < kRounds; ++rd) {
        const int e = s_idx[warp * kPerWarp + rd * 32 + lane];
        if (e >= 0) atomicAdd_block(reinterpret_cast<int*>(&s_wh[warp][0]) + (e >> 1),
                                    (e & 1) ? (1 << 16) : 1);
    }
    __syncthreads();

    // ---- publish this tile's counts ----
    int acc = 0;
    unsigned long long* mine = status + (size_t)tile * E + tid;
    if (tid < E) {
        for (int w = 0; w < kWarps; ++w) {
            const int t = s_wh[w][tid];
            s_wh[w][tid] = (short)acc;
            acc += t;
        }
        if (tile == 0) {
            if (!drop_first) st_relaxed(mine, status_word(tag, kFlagPrefix, (uint32_t)acc));
        } else {
            st_relaxed(mine, status_word(tag, kFlagAggregate, (uint32_t)acc));
        }
    }

    // ---- copy table of every expert, from the plan (overlaps the wait) ----
    for (int p = tid; p <= P; p += kThreads) u.pro.off[p] = __ldg(plan.slot_offset + p);
    for (int p = tid; p < P; p += kThreads) u.pro.sq[p] = __ldg(plan.slot_quota + p);
    for (int g = tid; g < G; g += kThreads) u.pro.se[g] = __ldg(plan.slot_expert + g);
    __syncthreads();
    for (int g = tid; g < G; g += kThreads) {
        const int e = u.pro.se[g];
        if (e >= 0 && e < E) {
            atomicAdd(&u.pro.cnt[e], 1);
        } else if (e >= E) {
            raise_error(err, UE_ERR_DEVICE_BOUNDS, g);
        }
    }
    __syncthreads();
    {
        // exclusive scan of copies per expert (1 + replicas) over experts
        const int c = tid < E ? 1 + u.pro.cnt[tid] : 0;
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
            const int cb = wofs + incl - c;
            s_c[e] = ExpC{c, cb};          // completed below
            s_cp[cb] = mp;                 // copy 0: the master
            s_cr[cb] = u.pro.off[mp];
            u.pro.run[e] = cb + 1;         // next replica entry
        }
        __syncthreads();
    }
    if (warp == 0) {
        // replicas in ascending g after each expert's master
        for (int g0 = 0; g0 < G; g0 += 32) {
            const int g = g0 + lane;
            int e = -1;
            if (g < G) {
                e = u.pro.se[g];
                if (e >= E) e = -1;
            }
            const unsigned peers = __match_any_sync(kFull, e);
            if (e >= 0) {
                const int ci = u.pro.run[e] + __popc(peers & ((1u << lane) - 1u));
                const int p = (g / S) * (M + S) + M + (g % S);
                s_cp[ci] = p;
                s_cr[ci] = u.pro.off[p];
            }
            __syncwarp();
            if (e >= 0 && lane == __ffs(peers) - 1) u.pro.run[e] += __popc(peers);
            __syncwarp();
        }
    }
    __syncthreads();
    if (tid < E) {
        // the expert's load, its copies' starts, and whether the quotas have
        // the floor form b + [j < rem]
        const int e = tid;
        const ExpC c0 = s_c[e];
        const int c = c0.b, cb = c0.cb;
        int L = 0;
        for (int j = 0; j < c; ++j) {
            s_cs[cb + j] = L;
            L += u.pro.sq[s_cp[cb + j]];
        }
        const unsigned b = (unsigned)L / (unsigned)c;
        const int rem = L - (int)b * c;
        bool floor_form = kOrder != kOrderLocal;  // the local order needs the count
        for (int j = 0; j < c; ++j)
            floor_form &= u.pro.sq[s_cp[cb + j]] == (int)b + (j < rem ? 1 : 0);
        s_a[e] = ExpA{0, L, rem * (int)(b + 1u), floor_form ? rem : -1};
        s_bm[e] = ExpB{recip64(b + 1u), recip64(b)};
        s_c[e] = ExpC{floor_form ? (int)b : c, cb};
    }
    __syncthreads();  // the union switches from the copy table to look-back

    // ---- look back over predecessor tiles, publish the inclusive prefix ----
    // H threads per expert column; thread (h, e) reads predecessors
    // base - h*W .. base - h*W - (W-1) of each step, so one step covers H*W
    // tiles with independent loads.
    const int H = min(kMaxH, kThreads / E);
    const int h = tid / E;
    const int e = tid - h * E;
    const bool lb = h < H;
    uint32_t excl = 0;
    if (lb && h == 0) u.lb.cdone[e] = (tile == 0) ? 1 : 0;
    __syncthreads();
    bool done = lb ? (u.lb.cdone[e] != 0) : true;
    int base = tile - 1;  // nearest predecessor not yet added
    int64_t polls = 0;
    while (__syncthreads_or(!done)) {
        if (!done) {
            uint32_t sum = 0;
            unsigned char st = 0;  // 0: no prefix in my segment, 1: prefix, 2: error
            unsigned long long v[kWindow];
#pragma unroll
            for (int i = 0; i < kWindow; ++i) {
                const int pred = base - h * kWindow - i;
                v[i] = pred >= 0 ? ld_relaxed(status + (size_t)pred * E + e)
                                 : status_word(tag, kFlagPrefix, 0u);
            }
#pragma unroll
            for (int i = 0; i < kWindow; ++i) {
                if (st == 0) {
                    const int pred = base - h * kWindow - i;
                    unsigned long long sw = v[i];
                    // not yet published in this launch (older tag or none)
                    while (((uint32_t)(sw >> 32) != tag ||
                            (((uint32_t)sw >> 30) == kFlagInvalid)) && st == 0) {
                        if (++polls > spin_limit) {
                            raise_error(err, UE_ERR_TIMEOUT, tile);
                            st = 2;
                        } else {
                            __nanosleep(64);
                            sw = ld_relaxed(status + (size_t)pred * E + e);
                        }
                    }
                    if (st == 0) {
                        const uint32_t flag = (uint32_t)sw >> 30;
                        if (flag == kFlagError) {
                            st = 2;
                        } else {
                            if (pred >= 0) sum += (uint32_t)sw & kValueMask;
                            if (flag == kFlagPrefix) st = 1;
                        }
                    }
                }
            }
            u.lb.part[h][e] = sum;
            u.lb.state[h][e] = st;
        }
        __syncthreads();
        if (!done && h == 0) {
            // add the segments in order up to the first one holding a prefix
            bool stop = false;
            for (int hh = 0; hh < H && !stop; ++hh) {
                const unsigned char st = u.lb.state[hh][e];
                if (st == 2) {
                    atomicOr(&s_fail, 1);
                    stop = true;
                } else {
                    excl += u.lb.part[hh][e];
                    if (st == 1) stop = true;
                }
            }
            u.lb.cdone[e] = stop ? 1 : 0;
        }
        __syncthreads();
        if (!done) done = u.lb.cdone[e] != 0;
        base -= H * kWindow;
    }
    if (tid < E && tile > 0) {
        if (s_fail)
            st_relaxed(mine, status_word(tag, kFlagError, 0u));
        else
            st_relaxed(mine, status_word(tag, kFlagPrefix, excl + (uint32_t)acc));
    }
    if (tid < E) s_a[tid].pre = (int)excl;
    __syncthreads();
    const bool write_out = !s_fail;

    // ---- in-order ranks, copy, dispatch row ----
    // the o-th pair of expert e: with floor-form quotas, copy j = o / (b+1)
    // while o < rem*(b+1), else rem + (o - rem*(b+1)) / b; otherwise the
    // last copy whose start is <= o. Row = first row of the copy + (o - start).
#pragma unroll 2
    for (int rd = 0; rd < (write_out ? kRounds : 0); ++rd) {
        const int x = warp * kPerWarp + rd * 32 + lane;
        const int ex = s_idx[x];
        const unsigned peers = same_key_lanes(ex & 511);
        const int64_t i = pair_at<kOrder>(t0 + x, ord);
        int p = -1, row = -1;
        if (ex >= 0) {
            const ExpA a = s_a[ex];
            const int o = a.pre + s_wh[warp][ex] + __popc(peers & ((1u << lane) - 1u));
            const ExpC c = s_c[ex];
            if (o >= a.L) {
                // the plan does not cover this pair (plan from other ids)
                raise_error(err, UE_ERR_DEVICE_BOUNDS, (int)min(i, (int64_t)INT_MAX));
            } else if (kOrder == kOrderLocal) {
                // copies of e in copy order, as this pair's source rank
                // splits them (c.b is the number of copies here)
                const unsigned r = div_m((unsigned)i, ord.TK, ord.mTK);
                const int32_t* fr = ord.first + (size_t)r * ord.P;
                const int j = last_at_most(c.b, o, [&](int jj) { return __ldg(fr + s_cp[c.cb + jj]); });
                const int pj = s_cp[c.cb + j];
                const size_t rp = (size_t)r * ord.P + pj;
                if (o - __ldg(fr + pj) < __ldg(ord.quota + rp)) {
                    p = pj;
                    row = __ldg(ord.rowb + rp) + o;
                } else {
                    // the split does not cover this pair (split from other ids)
                    raise_error(err, UE_ERR_DEVICE_BOUNDS, (int)min(i, (int64_t)INT_MAX));
                }
            } else if (a.rem >= 0) {
                const ExpB bm = s_bm[ex];
                const bool big = o < a.thr;
                const unsigned d = big ? (unsigned)c.b + 1u : (unsigned)c.b;
                const unsigned x0 = big ? (unsigned)o : (unsigned)(o - a.thr);
                const unsigned q = div_m(x0, d, big ? bm.m1 : bm.m0);
                const int j = big ? (int)q : a.rem + (int)q;
                const int start = j * c.b + min(j, a.rem);
                const int ci = c.cb + j;
                p = s_cp[ci];
                row = s_cr[ci] + (o - start);
            } else {
                const int ci = c.cb + last_at_most(c.b, o, [&](int jj) { return s_cs[c.cb + jj]; });
                p = s_cp[ci];
                row = s_cr[ci] + (o - s_cs[ci]);
            }
        }
        __syncwarp();
        if (ex >= 0 && lane == __ffs(peers) - 1) s_wh[warp][ex] += (short)__popc(peers);
        __syncwarp();
        if (x < cnt_tile) {
            phys_slot[i] = p;
            dest_row[i] = row;
        }
    }

    // the last CTA to finish leaves the ticket, the counter and the epoch
    // ready for the next launch
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        if (atomicAdd(&sync[1], 1u) == gridDim.x - 1) {
            sync[0] = 0u;
            sync[1] = 0u;
            __threadfence();
            atomicExch(&sync[2], tag);
        }
    }
}

// First occurrence index and row base of every (source rank, copy) of one
// expert, for the locality order. Copy j of expert e receives source rank
// r's pairs of e number first .. first + quota - 1 in global order, where
// first = (pairs of e from lower ranks) + (rank r's pairs given to e's
// earlier copies); the pair with occurrence index o lands on row
// src_offset[r][p] + (o - first) = rowb + o.
__global__ void __launch_bounds__(128)
local_tables_kernel(const int32_t* __restrict__ load_re, int R, int E, int S,
                    ue_placement plan, const int32_t* __restrict__ src_quota,
                    const int32_t* __restrict__ src_offset, int32_t* __restrict__ first,
                    int32_t* __restrict__ rowb, int* err)
{
    __shared__ int s_cp[1 + kMaxG];
    __shared__ int s_pre[kMaxR + 1];
    __shared__ int s_n;
    const int e = blockIdx.x;
    const int M = E / R;
    const int G = R * S;
    const int P = R * (M + S);
    const int tid = threadIdx.x;
    if (tid < 32) {
        // copies in copy order: the master, then replicas by ascending g
        int n = 1;
        if (tid == 0) s_cp[0] = (e / M) * (M + S) + e % M;
        for (int g0 = 0; g0 < G; g0 += 32) {
            const int g = g0 + tid;
            const bool mine = g < G && __ldg(plan.slot_expert + g) == e;
            const unsigned b = __ballot_sync(kFull, mine);
            if (mine) s_cp[n + __popc(b & ((1u << tid) - 1u))] = (g / S) * (M + S) + M + g % S;
            n += __popc(b);
        }
        if (tid == 0) s_n = n;
    } else if (tid == 32) {
        int run = 0;
        for (int r = 0; r < R; ++r) {
            s_pre[r] = run;
            run += __ldg(load_re + (size_t)r * E + e);
        }
        s_pre[R] = run;
    }
    __syncthreads();
    const int n = s_n;
    for (int r = tid; r < R; r += blockDim.x) {
        int run = s_pre[r];
        for (int j = 0; j < n; ++j) {
            const size_t rp = (size_t)r * P + s_cp[j];
            first[rp] = run;
            rowb[rp] = __ldg(src_offset + rp) - run;
            run += __ldg(src_quota + rp);
        }
        // the split must give away exactly this rank's pairs of e
        if (run != s_pre[r + 1]) raise_error(err, UE_ERR_DEVICE_BOUNDS, e);
    }
}

OrderArgs make_order(const Sizes& z)
{
    auto rc = [](unsigned d) { return d <= 1u ? 0ull : (~0ull / d) + 1ull; };
    OrderArgs o{};
    o.T = (unsigned)z.T;
    o.K = (unsigned)z.K;
    o.RK = (unsigned)(z.R * z.K);
    o.TK = (unsigned)((int64_t)z.T * z.K);
    o.mK = rc(o.K);
    o.mRK = rc(o.RK);
    o.mTK = rc(o.TK);
    o.P = z.P;
    return o;
}

template <int kOrder>
cudaError_t launch_order(const Sizes& z, const int32_t* idx, const ue_placement& plan,
                         const OrderArgs& ord, int32_t* phys_slot, int32_t* dest_row,
                         unsigned long long* status, uint32_t* sync, int64_t spin_limit,
                         int drop_first, int* err, cudaStream_t st)
{
    const int64_t tiles = (z.Q + kTile - 1) / kTile;
    reroute_kernel<kOrder><<<(unsigned)tiles, kThreads, 0, st>>>(
        idx, z.Q, z.R, z.E, z.S, plan, ord, phys_slot, dest_row, status, sync, spin_limit,
        drop_first, err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_reroute(const Sizes& z, const int32_t* idx,
                           const ue_placement& plan, int32_t* phys_slot,
                           int32_t* dest_row, unsigned long long* status,
                           uint32_t* sync, int64_t spin_limit,
                           int drop_first, int* err, cudaStream_t st)
{
    return launch_reroute_order(z, idx, plan, kOrderPrefix, phys_slot, dest_row, status, sync,
                                spin_limit, drop_first, err, st);
}

cudaError_t launch_reroute_order(const Sizes& z, const int32_t* idx, const ue_placement& plan,
                                 int order, int32_t* phys_slot, int32_t* dest_row,
                                 unsigned long long* status, uint32_t* sync, int64_t spin_limit,
                                 int drop_first, int* err, cudaStream_t st)
{
    if (z.Q == 0) return cudaSuccess;
    const OrderArgs ord = make_order(z);
    if (order == kOrderInterleave)
        return launch_order<kOrderInterleave>(z, idx, plan, ord, phys_slot, dest_row, status,
                                              sync, spin_limit, drop_first, err, st);
    return launch_order<kOrderPrefix>(z, idx, plan, ord, phys_slot, dest_row, status, sync,
                                      spin_limit, drop_first, err, st);
}

cudaError_t launch_reroute_local(const Sizes& z, const int32_t* idx, const int32_t* load_re,
                                 const ue_placement& plan, const int32_t* src_quota,
                                 const int32_t* src_offset, int32_t* first, int32_t* rowb,
                                 int32_t* phys_slot, int32_t* dest_row,
                                 unsigned long long* status, uint32_t* sync, int64_t spin_limit,
                                 int drop_first, int* err, cudaStream_t st)
{
    if (z.Q == 0) return cudaSuccess;
    local_tables_kernel<<<z.E, 128, 0, st>>>(load_re, z.R, z.E, z.S, plan, src_quota, src_offset,
                                             first, rowb, err);
    const cudaError_t ce = cudaGetLastError();
    if (ce != cudaSuccess) return ce;
    OrderArgs ord = make_order(z);
    ord.first = first;
    ord.rowb = rowb;
    ord.quota = src_quota;
    return launch_order<kOrderLocal>(z, idx, plan, ord, phys_slot, dest_row, status, sync,
                                     spin_limit, drop_first, err, st);
}

}  // namespace ue
