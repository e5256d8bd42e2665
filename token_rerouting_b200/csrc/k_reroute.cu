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
// Design (B200): a single-pass stable counting sort. Each CTA takes a tile
// of 512 threads x 7 to 32 pairs by an atomic ticket (so every tile it waits
// on is already running). Its warps copy the tile's ids into shared memory
// (cp.async), count them per warp sub-range of the output phase, publish the
// tile's per-expert counts at once and arrive at its group of 16 tiles. The
// group's last arrival, whose members have all published, writes each
// member's exclusive prefix inside the group into the member's word and the
// group's sum into the group's word, then looks back over the groups before
// it (each group word is published by a tile with a lower ticket) to the
// nearest inclusive prefix, and publishes the group's inclusive prefix.
// Meanwhile every warp ranks each pair of its sub-range among the earlier
// pairs of its expert (the lanes holding the same id come from eight or nine
// ballots over the id's bits, then a running count per expert). Then, side
// by side on named barriers, warps 0-7 find the tile's exclusive prefix per
// expert: its own word plus the previous group's inclusive prefix, two loads
// per expert once they are out, so few tiles read the same words; warps 8-15
// rebuild the plan's copy table (at most 512 entries).
// Every wait is bounded: when it runs out the waiter records UE_ERR_TIMEOUT,
// publishes an error flag where others wait on it, and its tile writes
// nothing. Finally each warp takes its pairs, whose occurrence index is the
// tile's prefix plus the pair's offset in the tile, and writes the physical
// slot and dispatch row. Per expert the tile keeps the copy that holds its
// first pair of that expert; most pairs fall in it. The others find their
// copy by one exact multiply-high by a per-expert reciprocal for floor-form
// quotas, otherwise by a binary search over the copy starts.
// Only the copy table and that last phase read the plan. Launched as the
// plan kernel's programmatic dependent, the tiles copy, count, publish, rank
// and look back while the plan runs; warps 8-15 wait for the plan to
// complete before they read it.
// The status words carry the launch's tag, so nothing is cleared between
// launches: words of earlier launches read as "not yet published". The last
// CTA to finish resets the ticket and the counter and advances the epoch;
// each group's last arrival resets the group's counter.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kThreads = kRerouteThreads;
constexpr int kWarps = kRerouteWarps;
constexpr int kHalf = kThreads / 2;  // threads of each half of a tile's CTA

// asynchronous global -> shared copies (cp.async, no registers held) and the
// wait for all of this thread's copies
__device__ __forceinline__ void copy_async16(int* dst, const int32_t* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                 ::"r"((unsigned)__cvta_generic_to_shared(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void copy_async4(int* dst, const int32_t* src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;"
                 ::"r"((unsigned)__cvta_generic_to_shared(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void copy_async_wait_all()
{
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// barrier of one half of the CTA (a named barrier other than 0, which
// __syncthreads uses)
__device__ __forceinline__ void half_sync(int id)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(kHalf) : "memory");
}

__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long* p)
{
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// atomic add with release and acquire semantics at GPU scope: the arrival
// publishes what the CTA wrote before it (ordered by the barrier before) and
// sees what earlier arrivals published
__device__ __forceinline__ uint32_t add_acq_rel(uint32_t* p, uint32_t v)
{
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;"
                 : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
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

// the lanes of the warp holding the same expert id (-1 for none): one ballot
// per bit of the id, 8 bits when E <= 255 (-1 reads as 255, which no expert
// has), 9 otherwise
__device__ __forceinline__ unsigned same_key_lanes(int ex, int E)
{
    unsigned peers = kFull;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
        const bool bit = (ex >> b) & 1;
        const unsigned m = __ballot_sync(kFull, bit);
        peers &= bit ? m : ~m;
    }
    if (E > 255) {
        const bool bit = (ex >> 8) & 1;
        const unsigned m = __ballot_sync(kFull, bit);
        peers &= bit ? m : ~m;
    }
    return peers;
}

// floor(x / d) for x < 2^32 and m = ceil(2^64 / d) (d >= 2), or x when d == 1:
// the high 64 bits of x * m from two 32-bit products
__device__ __forceinline__ unsigned div_m32(unsigned x, unsigned d, unsigned long long m)
{
    const unsigned long long t =
        (unsigned long long)x * (unsigned)(m >> 32) + __umulhi(x, (unsigned)m);
    return d == 1u ? x : (unsigned)(t >> 32);
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
// (computed as floor((2^64 - 1) / d) + 1: the high half by a 32-bit division,
// the low half, a quotient below 2^32, by an fp64 estimate within one unit
// corrected with the exact remainder)
__device__ __forceinline__ unsigned long long recip64(unsigned d)
{
    if (d <= 1u) return 0ull;
    const unsigned hi = 0xffffffffu / d;
    const unsigned r1 = 0xffffffffu - hi * d;  // < d
    const unsigned long long x = ((unsigned long long)r1 << 32) | 0xffffffffull;  // < d 2^32
    unsigned long long lo = (unsigned long long)((double)x / (double)d);
    long long rem = (long long)(x - lo * d);   // small: the estimate is within one unit
#pragma unroll
    for (int k = 0; k < 2; ++k)
        if (rem < 0) {
            --lo;
            rem += d;
        }
#pragma unroll
    for (int k = 0; k < 2; ++k)
        if (rem >= (long long)d) {
            ++lo;
            rem -= d;
        }
    return ((unsigned long long)hi << 32) + lo + 1ull;
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

// the same for Q < 2^30, in 32 bits
template <int kOrder>
__device__ __forceinline__ unsigned pair_at32(unsigned u, const OrderArgs& o)
{
    if (kOrder != kOrderInterleave) return u;
    const unsigned t = div_m(u, o.RK, o.mRK);
    const unsigned w = u - t * o.RK;
    const unsigned r = div_m(w, o.K, o.mK);
    const unsigned k = w - r * o.K;
    return (r * o.T + t) * o.K + k;
}

// wait (bounded) until *p holds a word of this launch, then return it in w;
// false when the wait ran out
__device__ __forceinline__ bool wait_word(const unsigned long long* p, uint32_t tag,
                                          unsigned long long& w, int64_t& polls,
                                          int64_t spin_limit)
{
    while ((uint32_t)(w >> 32) != tag || ((uint32_t)w >> 30) == kFlagInvalid) {
        if (++polls > spin_limit) return false;
        __nanosleep(64);
        w = ld_relaxed(p);
    }
    return true;
}

template <int kOrder, int kPer>
__global__ void __launch_bounds__(kThreads, 2)
reroute_kernel(const int32_t* __restrict__ idx, int64_t Q, int R, int E, int S,
               ue_placement plan, OrderArgs ord, int32_t* __restrict__ phys_slot,
               int32_t* __restrict__ dest_row, RerouteScratch sc, int64_t spin_limit,
               int drop_first, int* err)
{
    constexpr int kTileP = kThreads * kPer;    // pairs per tile
    constexpr int kPerWarpP = kTileP / kWarps;  // pairs per warp sub-range
    extern __shared__ __align__(16) int s_idx[];  // [kTileP] expert ids of the tile (-1: none)
    __shared__ short s_wh[kWarps][kMaxE]; // per-warp counts, then in-tile offsets
    __shared__ ExpA s_a[kMaxE];
    __shared__ ExpB s_bm[kMaxE];
    __shared__ ExpC s_c[kMaxE];
    __shared__ int2 s_cpr[kMaxE + kMaxG]; // copy table, copies of each expert in
                                          // order: (physical slot, first dispatch row);
    __shared__ int s_cs[kMaxE + kMaxG + 1];  // first pair index o of the copy
    __shared__ short s_ce[kMaxE + kMaxG];    // expert of each copy-table entry
    __shared__ union {
        struct {  // building the copy table
            int se[kMaxG];                // plan: slot_expert
            unsigned char cntc[kMaxG / 32][kMaxE];  // slots of each expert per chunk of 32
            int base[kMaxE], ff[kMaxE];
            int off[kMaxE + kMaxG + 1];   // plan: slot_offset
            int sq[kMaxE + kMaxG];        // plan: slot_quota
        } pro;
    } u;
    __shared__ int s_wsum[kWarps];
    __shared__ int s_pre[kMaxE];  // the tile's exclusive prefix per expert
    __shared__ int4 s_fast[kMaxE]; // copy of each expert's first pair in the tile
    __shared__ int s_tile;
    __shared__ uint32_t s_tag;
    __shared__ int s_fail;
    __shared__ int s_fin;
    __shared__ int s_allff;  // every expert's quotas of the floor form

    const int M = E / R;
    const int G = R * S;
    const int P = R * (M + S);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int ntiles = (int)gridDim.x;

    if (tid == 0) {
        s_tile = (int)atomicAdd(&sc.sync[0], 1u);
        // this launch's tag; the epoch only moves after every CTA has read it
        const uint32_t epoch = *reinterpret_cast<volatile uint32_t*>(&sc.sync[2]);
        s_tag = epoch + 1u == 0u ? 1u : epoch + 1u;
        s_fail = 0;
        s_allff = kOrder == kOrderLocal ? 0 : 1;
    }
    __syncthreads();
    const int tile = s_tile;
    const uint32_t tag = s_tag;
    const int64_t t0 = (int64_t)tile * kTileP;
    const int cnt_tile = (int)min((int64_t)kTileP, Q - t0);
    const int grp = tile / kRerouteGroup;
    const int gfirst = grp * kRerouteGroup;
    const int members = min(kRerouteGroup, ntiles - gfirst);

    // ---- stage the tile and count it per warp sub-range (every warp) ----
    for (int x = tid; x < kWarps * kMaxE; x += kThreads) (&s_wh[0][0])[x] = 0;
    // the ids go straight to shared memory (cp.async, all copies in
    // flight at once); the count below checks them
    if (kOrder != kOrderInterleave && (reinterpret_cast<uintptr_t>(idx) & 15u) == 0) {
        for (int c4 = tid; c4 < kTileP / 4; c4 += kThreads) {
            const int x = 4 * c4;
            if (x + 4 <= cnt_tile) {
                copy_async16(&s_idx[x], idx + t0 + x);
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    s_idx[x + k] = x + k < cnt_tile ? __ldg(idx + t0 + x + k) : -1;
            }
        }
    } else {
        for (int x = tid; x < kTileP; x += kThreads) {
            if (x < cnt_tile) copy_async4(&s_idx[x], idx + pair_at<kOrder>(t0 + x, ord));
            else s_idx[x] = -1;
        }
    }
    copy_async_wait_all();
    __syncthreads();
#pragma unroll 4
    for (int rd = 0; rd < kPer; ++rd) {
        const int x = warp * kPerWarpP + rd * 32 + lane;
        int e = s_idx[x];
        if (x < cnt_tile && (unsigned)e >= (unsigned)E) {
            // an id out of range: reported and skipped from here on
            raise_error(err, UE_ERR_DEVICE_BOUNDS,
                        (int)min(pair_at<kOrder>(t0 + x, ord), (int64_t)INT_MAX));
            e = -1;
            s_idx[x] = -1;
        }
        if (e >= 0) atomicAdd_block(reinterpret_cast<int*>(&s_wh[warp][0]) + (e >> 1),
                                    (e & 1) ? (1 << 16) : 1);
    }
    __syncthreads();

    // ---- publish this tile's counts and arrive at its group ----
    if (tid < E) {
        int acc = 0;
        for (int w = 0; w < kWarps; ++w) {
            const int t = s_wh[w][tid];
            s_wh[w][tid] = (short)acc;
            acc += t;
        }
        if (!(drop_first && tile == 0))
            st_relaxed(sc.status + (size_t)tile * E + tid,
                       status_word(tag, kFlagAggregate, (uint32_t)acc));
    }
    __syncthreads();
    if (tid == 0)
        s_fin = add_acq_rel(&sc.gcount[grp], 1u) == (uint32_t)(members - 1) ? 1 : 0;
    __syncthreads();
    if (s_fin) {
        // the last tile of the group to arrive (its members published their
        // counts before they arrived): each member's exclusive prefix inside
        // the group goes into the member's own word (flag: prefix), and the
        // group's sum into the group's word (flag: aggregate)
        if (tid < E) {
            unsigned long long v[kRerouteGroup];
#pragma unroll
            for (int i = 0; i < kRerouteGroup; ++i)
                v[i] = i < members ? ld_relaxed(sc.status + (size_t)(gfirst + i) * E + tid) : 0ull;
            uint32_t run = 0, flag = kFlagAggregate;
            int64_t polls = 0;
#pragma unroll
            for (int i = 0; i < kRerouteGroup; ++i) {
                if (i < members && flag == kFlagAggregate) {
                    if (wait_word(sc.status + (size_t)(gfirst + i) * E + tid, tag, v[i], polls,
                                  spin_limit)) {
                        st_relaxed(sc.status + (size_t)(gfirst + i) * E + tid,
                                   status_word(tag, kFlagPrefix, run));
                        run += (uint32_t)v[i] & kValueMask;
                    } else {
                        raise_error(err, UE_ERR_TIMEOUT, gfirst + i);
                        flag = kFlagError;
                    }
                }
            }
            if (flag == kFlagError) {
                for (int i = 0; i < members; ++i)
                    st_relaxed(sc.status + (size_t)(gfirst + i) * E + tid,
                               status_word(tag, kFlagError, 0u));
            }
            st_relaxed(sc.gstatus + (size_t)grp * E + tid, status_word(tag, flag, run));
            // then the group's inclusive prefix: its sum plus the sums of the
            // groups before it, back to the nearest group whose inclusive
            // prefix is out (decoupled look-back over groups, each of whose
            // words is published by a tile with a lower ticket)
            if (flag == kFlagAggregate) {
                uint32_t pre = 0;
                int gb = grp - 1;
                bool done = gb < 0;
                while (!done) {
                    unsigned long long w = ld_relaxed(sc.gstatus + (size_t)gb * E + tid);
                    if (!wait_word(sc.gstatus + (size_t)gb * E + tid, tag, w, polls, spin_limit)) {
                        raise_error(err, UE_ERR_TIMEOUT, gb);
                        flag = kFlagError;
                        break;
                    }
                    const uint32_t f = (uint32_t)w >> 30;
                    if (f == kFlagError) {
                        flag = kFlagError;
                        break;
                    }
                    pre += (uint32_t)w & kValueMask;
                    done = f == kFlagPrefix || --gb < 0;
                }
                st_relaxed(sc.gstatus + (size_t)grp * E + tid,
                           status_word(tag, flag == kFlagError ? kFlagError : kFlagPrefix,
                                       pre + run));
            }
        }
        // every member has arrived: ready for the next launch
        if (tid == 0) sc.gcount[grp] = 0u;
    }

    // ---- in-tile ranks ----
    // each warp ranks its own sub-range: a pair's offset in the tile among
    // the pairs of its expert is the sub-range's offset plus the pairs of
    // that expert before it in the sub-range (the lanes holding the same id,
    // then a running count per expert); it replaces the id in shared memory
    // as (offset << 8) | id. The ranks depend on the ids alone, so they are
    // ready before the plan is read.
    {
        const unsigned lt = (1u << lane) - 1u;
#pragma unroll 2
        for (int rd = 0; rd < kPer; ++rd) {
            const int x = warp * kPerWarpP + rd * 32 + lane;
            const int e = s_idx[x];
            const unsigned peers = same_key_lanes(e, E);
            const int below = __popc(peers & lt);
            const int ev = e < 0 ? 0 : e;
            const int run = s_wh[warp][ev];
            s_idx[x] = e < 0 ? -1 : (((run + below) << 8) | e);
            __syncwarp();
            // the lowest lane of each expert's group moves its count on
            if (e >= 0 && below == 0) s_wh[warp][ev] = (short)(run + __popc(peers));
            __syncwarp();
        }
    }

    // Two halves of the CTA work side by side: warps 0-7 look back for the
    // tile's exclusive prefix per expert; warps 8-15 rebuild the copy table
    // from the plan, with their own barrier.
    if (tid < kHalf) {
        // ---- look back: this tile's exclusive prefix per expert ----
        // the tile's own word (its exclusive prefix inside its group, put there
        // by the group's last arrival) plus the inclusive prefix of the group
        // before (or, while that is not out yet, the sums of the groups before,
        // back to the nearest inclusive prefix)
        if (tid < E) {
            uint32_t excl = 0;
            bool fail = false;
            int64_t polls = 0;
            const unsigned long long* own = sc.status + (size_t)tile * E + tid;
            unsigned long long w = ld_relaxed(own);
            // wait for the prefix flag (the tile's own count is there first)
            while (!fail && ((uint32_t)(w >> 32) != tag || ((uint32_t)w >> 30) == kFlagInvalid ||
                             ((uint32_t)w >> 30) == kFlagAggregate)) {
                if (++polls > spin_limit) {
                    raise_error(err, UE_ERR_TIMEOUT, tile);
                    fail = true;
                } else {
                    __nanosleep(64);
                    w = ld_relaxed(own);
                }
            }
            if (!fail && ((uint32_t)w >> 30) == kFlagError) fail = true;
            excl = (uint32_t)w & kValueMask;
            int gb = grp - 1;
            while (!fail && gb >= 0) {
                unsigned long long gw = ld_relaxed(sc.gstatus + (size_t)gb * E + tid);
                if (!wait_word(sc.gstatus + (size_t)gb * E + tid, tag, gw, polls, spin_limit)) {
                    raise_error(err, UE_ERR_TIMEOUT, tile);
                    fail = true;
                    break;
                }
                const uint32_t f = (uint32_t)gw >> 30;
                if (f == kFlagError) {
                    fail = true;
                    break;
                }
                excl += (uint32_t)gw & kValueMask;
                gb = f == kFlagPrefix ? -1 : gb - 1;
            }
            if (fail) s_fail = 1;
            s_pre[tid] = (int)excl;
        }
    } else {
        // ---- copy table of every expert, from the plan ----
        const int bt = tid - kHalf;  // 0 .. kHalf - 1
        const int bw = bt >> 5;
        for (int x = bt; x < kMaxG / 32 * kMaxE / 4; x += kHalf)
            reinterpret_cast<int*>(&u.pro.cntc[0][0])[x] = 0;
        for (int e = bt; e < E; e += kHalf) u.pro.ff[e] = 1;
        // launched after the plan kernel as its dependent, the tile gets
        // here while the plan may still run: wait for it to complete, then
        // read the plan through L2
        pdl_wait();
        for (int x = bt; x <= P; x += kHalf) u.pro.off[x] = __ldcg(plan.slot_offset + x);
        for (int x = bt; x < P; x += kHalf) u.pro.sq[x] = __ldcg(plan.slot_quota + x);
        if (bt < G) u.pro.se[bt] = __ldcg(plan.slot_expert + bt);
        half_sync(2);
        // slot g (one per thread: G <= kMaxG <= kHalf) takes its place among
        // its expert's replicas (ascending g): its rank inside its chunk of 32
        // slots (lanes holding the same expert) plus the expert's slots in
        // the chunks below, from a per-chunk count
        int slot_e = -1, slot_rank = 0;
        if (bt < G) {
            slot_e = u.pro.se[bt];
            if (slot_e >= E) {
                raise_error(err, UE_ERR_DEVICE_BOUNDS, bt);
                slot_e = -1;
            }
        }
        if (bw * 32 < G) {  // warp-uniform
            const unsigned peers = same_key_lanes(slot_e, E);
            if (slot_e >= 0) {
                slot_rank = __popc(peers & ((1u << lane) - 1u));
                if (slot_rank == 0) u.pro.cntc[bw][slot_e] = (unsigned char)__popc(peers);
            }
        }
        half_sync(2);
        const int nchunks = (G + 31) / 32;
        if (slot_e >= 0)
            for (int ch = 0; ch < bw; ++ch) slot_rank += u.pro.cntc[ch][slot_e];
        int ncopies = 1;  // of expert bt: the master and its replicas
        if (bt < E)
            for (int ch = 0; ch < nchunks; ++ch) ncopies += u.pro.cntc[ch][bt];
        int nent;  // copy-table entries: every expert's master and replicas
        {
            // exclusive scan of copies per expert (1 + replicas) over experts
            const int c = bt < E ? ncopies : 0;
            int incl = c;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(kFull, incl, off);
                if (lane >= off) incl += o;
            }
            if (lane == 31) s_wsum[bw] = incl;
            half_sync(2);
            int wofs = 0, all = 0;
            for (int w = 0; w < kWarps / 2; ++w) {
                wofs += w < bw ? s_wsum[w] : 0;
                all += s_wsum[w];
            }
            nent = all;
            if (bt < E) {
                const int e = bt;
                const int mp = (e / M) * (M + S) + (e % M);
                const int cb = wofs + incl - c;
                s_c[e] = ExpC{c, cb};          // completed below
                s_cpr[cb] = make_int2(mp, u.pro.off[mp]);  // copy 0: the master
                s_ce[cb] = (short)e;
            }
            half_sync(2);
        }
        if (slot_e >= 0) {
            // the replicas after their expert's master, in ascending g
            const int ci = s_c[slot_e].cb + 1 + slot_rank;
            const int pp = (bt / S) * (M + S) + M + (bt % S);
            s_cpr[ci] = make_int2(pp, u.pro.off[pp]);
            s_ce[ci] = (short)slot_e;
        }
        half_sync(2);
        {
            // every copy's start: an exclusive scan of the quotas over the
            // entries (experts in order, each one's copies in copy order);
            // thread bt owns entries 2 bt and 2 bt + 1 (nent <= E + G <= 512)
            const int e0 = 2 * bt, e1 = 2 * bt + 1;
            const int q0 = e0 < nent ? u.pro.sq[s_cpr[e0].x] : 0;
            const int q1 = e1 < nent ? u.pro.sq[s_cpr[e1].x] : 0;
            const int mine = q0 + q1;
            int incl = mine;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(kFull, incl, off);
                if (lane >= off) incl += o;
            }
            if (lane == 31) s_wsum[bw] = incl;
            half_sync(2);
            int wofs = 0;
            for (int w = 0; w < bw; ++w) wofs += s_wsum[w];
            const int excl = wofs + incl - mine;
            if (e0 < nent) s_cs[e0] = excl;
            if (e1 < nent) s_cs[e1] = excl + q0;
            if (e0 == nent - 1) s_cs[nent] = excl + q0;
            if (e1 == nent - 1) s_cs[nent] = excl + mine;
            half_sync(2);
        }
        if (bt < E) {
            // the expert's load and its floor-form parameters b = floor(L/c), rem
            const ExpC c0 = s_c[bt];
            const int base = s_cs[c0.cb];
            const int L = s_cs[c0.cb + c0.b] - base;
            const unsigned b = (unsigned)L / (unsigned)c0.b;
            u.pro.base[bt] = base;
            s_a[bt] = ExpA{0, L, (L - (int)b * c0.b) * (int)(b + 1u), L - (int)b * c0.b};
        }
        half_sync(2);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int ei = 2 * bt + h;
            if (ei < nent) {
                // starts relative to the expert; quotas of the form b + [j < rem]?
                const int e = s_ce[ei];
                const ExpC c0 = s_c[e];
                const int j = ei - c0.cb;
                const int q = u.pro.sq[s_cpr[ei].x];
                const unsigned b = (unsigned)s_a[e].L / (unsigned)c0.b;
                if (kOrder == kOrderLocal || q != (int)b + (j < s_a[e].rem ? 1 : 0))
                    u.pro.ff[e] = 0;
                s_cs[ei] -= u.pro.base[e];
            }
        }
        half_sync(2);
        if (bt < E) {
            // the local order needs the number of copies, so it never takes
            // the floor form
            const ExpC c0 = s_c[bt];
            const ExpA a = s_a[bt];
            const bool floor_form = u.pro.ff[bt] != 0;
            if (!floor_form) s_allff = 0;
            const unsigned b = (unsigned)a.L / (unsigned)c0.b;
            s_a[bt] = ExpA{0, a.L, a.thr, floor_form ? a.rem : -1};
            s_bm[bt] = ExpB{recip64(b + 1u), recip64(b)};
            s_c[bt] = ExpC{floor_form ? (int)b : c0.b, c0.cb};
        }
    }
    __syncthreads();
    const bool lean = kOrder != kOrderLocal && s_allff;
    if (tid < E) {
        const int pre = s_pre[tid];
        s_a[tid].pre = pre;
        if (kOrder != kOrderLocal) {
            // the copy holding the tile's first pair of this expert (its
            // occurrence index is pre): the expert's pairs of the tile at
            // in-tile offsets below `lim` all fall in it, at row row0 + offset
            const ExpA a = s_a[tid];
            const ExpC c = s_c[tid];
            int4 f = make_int4(-1, 0, 0, 0);  // (slot, row0, lim, -)
            if (pre < a.L) {
                int j, start, end;
                if (a.rem >= 0) {
                    // floor-form quotas: the copy by one division
                    const ExpB bm = s_bm[tid];
                    const bool big = pre < a.thr;
                    const unsigned d = big ? (unsigned)c.b + 1u : (unsigned)c.b;
                    const unsigned x0 = big ? (unsigned)pre : (unsigned)(pre - a.thr);
                    const unsigned q = div_m32(x0, d, big ? bm.m1 : bm.m0);
                    j = big ? (int)q : a.rem + (int)q;
                    start = j * c.b + min(j, a.rem);
                    end = start + c.b + (j < a.rem ? 1 : 0);
                } else {
                    // other quotas (c.b copies): the last copy starting at or before pre
                    j = last_at_most(c.b, pre, [&](int jj) { return s_cs[c.cb + jj]; });
                    start = s_cs[c.cb + j];
                    end = j + 1 < c.b ? s_cs[c.cb + j + 1] : a.L;
                }
                const int2 cr = s_cpr[c.cb + j];
                f = make_int4(cr.x, cr.y + (pre - start), end - pre, 0);
            }
            s_fast[tid] = f;
        }
    }
    __syncthreads();
    const bool write_out = !s_fail;

    // ---- in-order ranks, copy, dispatch row ----
    // the o-th pair of expert e: with floor-form quotas, copy j = o / (b+1)
    // while o < rem*(b+1), else rem + (o - rem*(b+1)) / b; otherwise the
    // last copy whose start is <= o. Row = first row of the copy + (o - start).
    if (lean) {
        // every expert has floor-form quotas: most pairs take the copy of
        // their expert's first pair in the tile from one record; the others
        // (past that copy's end) find theirs by the division. A pair beyond
        // its expert's load (ids that do not match the plan) is reported,
        // and its rank is clamped so that the table reads stay inside the
        // expert's copies.
        const unsigned t0u = (unsigned)t0;
#pragma unroll 2
        for (int rd = 0; rd < (write_out ? kPer : 0); ++rd) {
            const int x = warp * kPerWarpP + rd * 32 + lane;
            const int v = s_idx[x];
            const int ex = v < 0 ? -1 : (v & 255);
            const int lo = v < 0 ? 0 : v >> 8;
            const int ev = ex < 0 ? 0 : ex;
            const unsigned i = pair_at32<kOrder>(t0u + (unsigned)x, ord);
            const int4 f = s_fast[ev];
            int p = f.x, row = f.y + lo;
            if (ex < 0 || lo >= f.z) {
                const ExpA a = s_a[ev];
                const ExpC c = s_c[ev];
                const ExpB bm = s_bm[ev];
                const int o = a.pre + lo;
                const int oc = min(o, max(a.L - 1, 0));
                const bool big = oc < a.thr;
                const unsigned d = big ? (unsigned)c.b + 1u : (unsigned)c.b;
                const unsigned x0 = big ? (unsigned)oc : (unsigned)(oc - a.thr);
                const unsigned q = div_m32(x0, d, big ? bm.m1 : bm.m0);
                const int j = big ? (int)q : a.rem + (int)q;
                const int start = j * c.b + min(j, a.rem);
                const int2 cr = s_cpr[c.cb + j];
                p = cr.x;
                row = cr.y + (oc - start);
                if (ex < 0 || o >= a.L) {
                    if (ex >= 0)
                        raise_error(err, UE_ERR_DEVICE_BOUNDS, (int)min(i, (unsigned)INT_MAX));
                    p = -1;
                    row = -1;
                }
            }
            if (x < cnt_tile) {
                phys_slot[i] = p;
                dest_row[i] = row;
            }
        }
    } else {
#pragma unroll 2
        for (int rd = 0; rd < (write_out ? kPer : 0); ++rd) {
            const int x = warp * kPerWarpP + rd * 32 + lane;
            const int v = s_idx[x];
            const int ex = v < 0 ? -1 : (v & 255);
            const int ev = ex < 0 ? 0 : ex;             // a safe index for the loads
            const int64_t i = pair_at<kOrder>(t0 + x, ord);
            const ExpA a = s_a[ev];
            const ExpC c = s_c[ev];
            const int lo = v < 0 ? 0 : v >> 8;
            const int o = a.pre + lo;
            int p = -1, row = -1;
            const int4 f = s_fast[ev];
            if (kOrder != kOrderLocal && __all_sync(kFull, ex < 0 || lo < f.z)) {
                // every pair of the round lies in the copy of its expert's
                // first pair in the tile
                if (ex >= 0) {
                    p = f.x;
                    row = f.y + lo;
                }
            } else if (kOrder != kOrderLocal &&
                       __all_sync(kFull, ex < 0 || (a.rem >= 0 && o < a.L))) {
                // every lane of the round has floor-form quotas: no branches
                const ExpB bm = s_bm[ev];
                const bool big = o < a.thr;
                const unsigned d = big ? (unsigned)c.b + 1u : (unsigned)c.b;
                const unsigned x0 = big ? (unsigned)o : (unsigned)(o - a.thr);
                const unsigned q = div_m32(x0, d, big ? bm.m1 : bm.m0);
                const int j = big ? (int)q : a.rem + (int)q;
                const int start = j * c.b + min(j, a.rem);
                const int2 cr = s_cpr[c.cb + j];
                if (ex >= 0) {
                    p = cr.x;
                    row = cr.y + (o - start);
                }
            } else if (ex >= 0) {
                if (o >= a.L) {
                    // the plan does not cover this pair (plan from other ids)
                    raise_error(err, UE_ERR_DEVICE_BOUNDS, (int)min(i, (int64_t)INT_MAX));
                } else if (kOrder == kOrderLocal) {
                    // copies of e in copy order, as this pair's source rank
                    // splits them (c.b is the number of copies here)
                    const unsigned r = div_m((unsigned)i, ord.TK, ord.mTK);
                    const int32_t* fr = ord.first + (size_t)r * ord.P;
                    const int j = last_at_most(c.b, o, [&](int jj) { return __ldg(fr + s_cpr[c.cb + jj].x); });
                    const int pj = s_cpr[c.cb + j].x;
                    const size_t rp = (size_t)r * ord.P + pj;
                    if (o - __ldg(fr + pj) < __ldg(ord.quota + rp)) {
                        p = pj;
                        row = __ldg(ord.rowb + rp) + o;
                    } else {
                        // the split does not cover this pair (split from other ids)
                        raise_error(err, UE_ERR_DEVICE_BOUNDS, (int)min(i, (int64_t)INT_MAX));
                    }
                } else if (a.rem >= 0) {
                    const ExpB bm = s_bm[ev];
                    const bool big = o < a.thr;
                    const unsigned d = big ? (unsigned)c.b + 1u : (unsigned)c.b;
                    const unsigned x0 = big ? (unsigned)o : (unsigned)(o - a.thr);
                    const unsigned q = div_m32(x0, d, big ? bm.m1 : bm.m0);
                    const int j = big ? (int)q : a.rem + (int)q;
                    const int start = j * c.b + min(j, a.rem);
                    const int2 cr = s_cpr[c.cb + j];
                    p = cr.x;
                    row = cr.y + (o - start);
                } else {
                    const int ci = c.cb + last_at_most(c.b, o, [&](int jj) { return s_cs[c.cb + jj]; });
                    p = s_cpr[ci].x;
                    row = s_cpr[ci].y + (o - s_cs[ci]);
                }
            }
            if (x < cnt_tile) {
                phys_slot[i] = p;
                dest_row[i] = row;
            }
        }
    }

    // the last CTA to finish leaves the ticket, the counter and the epoch
    // ready for the next launch
    __syncthreads();
    if (tid == 0) {
        if (add_acq_rel(&sc.sync[1], 1u) == gridDim.x - 1) {
            sc.sync[0] = 0u;
            sc.sync[1] = 0u;
            __threadfence();
            atomicExch(&sc.sync[2], tag);
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

template <int kOrder, int kPer>
cudaError_t launch_tiles(const Sizes& z, const int32_t* idx, const ue_placement& plan,
                         const OrderArgs& ord, int32_t* phys_slot, int32_t* dest_row,
                         const RerouteScratch& sc, int64_t spin_limit, int drop_first, int* err,
                         cudaStream_t st, bool pdl)
{
    const int64_t tiles = (z.Q + kThreads * kPer - 1) / (kThreads * kPer);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)tiles);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kThreads * kPer * sizeof(int);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, reroute_kernel<kOrder, kPer>, idx, z.Q, z.R, z.E, z.S, plan,
                              ord, phys_slot, dest_row, sc, spin_limit, drop_first, err);
}

// pairs per thread of the tile sizes on offer (tile = 512 * kPer)
#define UE_REROUTE_PER(X) X(7) X(8) X(10) X(12) X(14) X(16) X(18) X(20) X(24) X(28) X(32)

template <int kOrder>
cudaError_t launch_order(const Sizes& z, int tile, const int32_t* idx, const ue_placement& plan,
                         const OrderArgs& ord, int32_t* phys_slot, int32_t* dest_row,
                         const RerouteScratch& sc, int64_t spin_limit, int drop_first, int* err,
                         cudaStream_t st, bool pdl)
{
    switch (tile) {
#define UE_CASE(P)                                                                          \
    case kThreads * P:                                                                      \
        return launch_tiles<kOrder, P>(z, idx, plan, ord, phys_slot, dest_row, sc,          \
                                       spin_limit, drop_first, err, st, pdl);
        UE_REROUTE_PER(UE_CASE)
#undef UE_CASE
    default:
        return cudaErrorInvalidValue;
    }
}

template <int kPer>
cudaError_t allow_smem()
{
    const int bytes = kThreads * kPer * (int)sizeof(int);
    cudaError_t ce = cudaFuncSetAttribute(reroute_kernel<kOrderPrefix, kPer>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (ce == cudaSuccess)
        ce = cudaFuncSetAttribute(reroute_kernel<kOrderInterleave, kPer>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (ce == cudaSuccess)
        ce = cudaFuncSetAttribute(reroute_kernel<kOrderLocal, kPer>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    return ce;
}

template <int kPer>
int64_t tile_slots(int num_sms)
{
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, reroute_kernel<kOrderPrefix, kPer>,
                                                      kThreads, kThreads * kPer * sizeof(int)) !=
        cudaSuccess) {
        cudaGetLastError();
        per_sm = 1;
    }
    return (int64_t)std::max(per_sm, 1) * num_sms;
}

}  // namespace

cudaError_t reroute_setup()
{
    cudaError_t ce = cudaSuccess;
#define UE_ALLOW(P) if (ce == cudaSuccess) ce = allow_smem<P>();
    UE_REROUTE_PER(UE_ALLOW)
#undef UE_ALLOW
    return ce;
}

int reroute_tile(const Sizes& z, int num_sms)
{
    // the most tiles that are all resident at once (one wave, about the same
    // number of tiles on every SM), so that no tile waits for a CTA slot;
    // 32 pairs per thread when even those are too many
#define UE_FIT(P)                                                                        \
    if ((z.Q + kThreads * P - 1) / (kThreads * P) <= tile_slots<P>(num_sms)) return kThreads * P;
    UE_REROUTE_PER(UE_FIT)
#undef UE_FIT
    return kThreads * 32;
}

cudaError_t launch_reroute(const Sizes& z, int tile, const int32_t* idx,
                           const ue_placement& plan, int32_t* phys_slot, int32_t* dest_row,
                           const RerouteScratch& sc, int64_t spin_limit, int drop_first, int* err,
                           cudaStream_t st)
{
    return launch_reroute_order(z, tile, idx, plan, kOrderPrefix, phys_slot, dest_row, sc,
                                spin_limit, drop_first, err, st);
}

cudaError_t launch_reroute_order(const Sizes& z, int tile, const int32_t* idx,
                                 const ue_placement& plan, int order, int32_t* phys_slot,
                                 int32_t* dest_row, const RerouteScratch& sc, int64_t spin_limit,
                                 int drop_first, int* err, cudaStream_t st, bool after_plan)
{
    if (z.Q == 0) return cudaSuccess;
    const OrderArgs ord = make_order(z);
    if (order == kOrderInterleave)
        return launch_order<kOrderInterleave>(z, tile, idx, plan, ord, phys_slot, dest_row, sc,
                                              spin_limit, drop_first, err, st, after_plan);
    return launch_order<kOrderPrefix>(z, tile, idx, plan, ord, phys_slot, dest_row, sc,
                                      spin_limit, drop_first, err, st, after_plan);
}

cudaError_t launch_reroute_local(const Sizes& z, int tile, const int32_t* idx,
                                 const int32_t* load_re, const ue_placement& plan,
                                 const int32_t* src_quota, const int32_t* src_offset,
                                 int32_t* first, int32_t* rowb, int32_t* phys_slot,
                                 int32_t* dest_row, const RerouteScratch& sc, int64_t spin_limit,
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
    return launch_order<kOrderLocal>(z, tile, idx, plan, ord, phys_slot, dest_row, sc,
                                     spin_limit, drop_first, err, st, false);
}

}  // namespace ue
