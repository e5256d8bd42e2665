/*
 * oracle.c -- plain, slow, single-threaded CPU oracle for the exact-load
 * expert rebalancing hot path of UltraEP:
 *
 *   gate top-k -> exact per-expert histogram -> quota-driven replication
 *   plan -> token-to-replica reroute -> permute -> gate-weighted combine,
 *   and beside it the backward of the permute and the combine, the weight
 *   sync to replica slots, the gradient reduction to master experts, and the
 *   planner variants the pages name as knobs: a minimal load per replica in
 *   the greedy, a capacity planner by bisection on the balancing ratio, a
 *   locality-aware split of the quotas over the source ranks, and an
 *   interleaved reroute order.
 *
 * TEST INFRASTRUCTURE. Nothing in the product path links or calls this file.
 * Only the test suite, the package smoke check and the benchmark's
 * CPU-baseline leg load it. It shares no source, header, table or helper
 * with the CUDA library; the two meet only at the seeded input generator.
 *
 * Floating point is fp64 (gate weights, combine). Integer work is exact.
 * Every step is the plain definition, written in the order the pages state
 * it, without blocking, fusion or incremental tricks, so a reader can check
 * it by eye. Sources (page title, section):
 *   [P1] "UltraEP: Real-Time Load Balancing for Large-Scale MoE Training and
 *        Inference" (aikit-app weekly), sections "What Happened" and
 *        "Technical Details".
 *   [P2] "Xiaohongshu's UltraEP Balances MoE Experts in 300 us, Reaching
 *        94.3% of Ideal" (news.hamidun.com), section "How balancing in 300
 *        microseconds works".
 *   [P3] "UltraEP" project README, sections "Interface / 2. Forward and
 *        backward", "Tests" and "Performance Tuning / Replication planning".
 * The pages only sketch the scheduler. The rules written here (tie breaks,
 * quota remainders, stop test, prefix fill) are the project's fixed reading
 * of that sketch; each function states the rule it implements.
 *
 * Notation: R ranks, T tokens per rank, N = R*T tokens, E experts,
 * M = E/R masters per rank, K top-k, S redundant slots per rank,
 * G = R*S redundant slots, P = R*(M+S) physical slots, Q = N*K pairs.
 * Pair i = n*K + k; token n lives on source rank n / T.
 *
 * All entry points return 0 on success and a negative code on bad input.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

#define OR_OK 0
#define OR_EINVAL (-1)
#define OR_ENOMEM (-2)
#define OR_EDATA (-3)

/* ------------------------------------------------------------------------ */
/* gate top-k                                                                */
/* ------------------------------------------------------------------------ */

typedef struct {
    float v;
    int32_t e;
} or_item;

/* Order for the top-k: larger logit first; equal logits (IEEE ==, so
 * -0.0 and +0.0 tie) go to the lower expert id. */
static int or_item_cmp(const void* pa, const void* pb)
{
    const or_item* a = (const or_item*)pa;
    const or_item* b = (const or_item*)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    if (a->e < b->e) return -1;
    if (a->e > b->e) return 1;
    return 0;
}

/*
 * Router gating: per token, the K experts with the largest logits, listed in
 * descending logit order (ties to the lower expert id), and their gate
 * weights: the softmax taken over the K selected logits,
 *     w_k = exp(v_k - v_0) / sum_j exp(v_j - v_0),
 * which equals a softmax over all E logits restricted to the selected K and
 * renormalised. [P3] "Interface / 2. Forward and backward" (the router
 * returns probs and routing_map); [P1] "What Happened" (routing from the
 * true routing probabilities).
 * logits: fp32 [N][E] row-major. idx: int32 [N][K]. w: fp64 [N][K].
 */
int or_gate_topk(const float* logits, int64_t N, int32_t E, int32_t K,
                 int32_t* idx, double* w)
{
    if (!logits || !idx || !w || N < 0 || E < 1 || K < 1 || K > E)
        return OR_EINVAL;
    or_item* row = (or_item*)malloc(sizeof(or_item) * (size_t)E);
    if (!row) return OR_ENOMEM;
    for (int64_t n = 0; n < N; ++n) {
        for (int32_t e = 0; e < E; ++e) {
            row[e].v = logits[n * E + e];
            row[e].e = e;
        }
        qsort(row, (size_t)E, sizeof(or_item), or_item_cmp);
        double v0 = (double)row[0].v;
        double z = 0.0;
        for (int32_t k = 0; k < K; ++k) z += exp((double)row[k].v - v0);
        for (int32_t k = 0; k < K; ++k) {
            idx[n * K + k] = row[k].e;
            w[n * K + k] = exp((double)row[k].v - v0) / z;
        }
    }
    free(row);
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* exact histogram                                                           */
/* ------------------------------------------------------------------------ */

/*
 * Exact post-gating load: load_re[r][e] counts the pairs of source rank r
 * routed to expert e (the per-rank metadata the pages all-gather before
 * planning), load_e[e] = sum over r. [P3] intro (rebalances on the exact
 * post-gating load), "Performance Tuning / NVSHMEM" (global-load metadata
 * all-gather); [P1] "What Happened" (knows in advance how many tokens hit
 * each expert).
 */
int or_count(const int32_t* idx, int32_t R, int32_t T, int32_t E, int32_t K,
             int32_t* load_re, int32_t* load_e)
{
    if (!idx || !load_re || !load_e || R < 1 || T < 0 || E < 1 || K < 1)
        return OR_EINVAL;
    int64_t N = (int64_t)R * T;
    for (int64_t x = 0; x < (int64_t)R * E; ++x) load_re[x] = 0;
    for (int32_t e = 0; e < E; ++e) load_e[e] = 0;
    for (int64_t i = 0; i < N * K; ++i) {
        int32_t e = idx[i];
        if (e < 0 || e >= E) return OR_EDATA;
        int64_t n = i / K;
        int64_t r = n / T;
        load_re[r * E + e] += 1;
        load_e[e] += 1;
    }
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* replication plan                                                          */
/* ------------------------------------------------------------------------ */

/* Quota of copy j (0 = master, then replicas in ascending redundant-slot
 * index) of an expert with load L and c copies: floor(L/c), plus one for the
 * first L mod c copies. */
static int64_t or_quota(int64_t L, int64_t c, int64_t j)
{
    return L / c + (j < L % c ? 1 : 0);
}

/* Rank loads from scratch: every copy's integer quota added to the rank that
 * holds it. Master of expert e sits on rank e / M; redundant slot g = r*S + s
 * sits on rank g / S. */
static void or_rank_loads(int32_t R, int32_t E, int32_t S, const int32_t* L,
                          const int32_t* c, const int32_t* slot_expert,
                          int64_t* load)
{
    int32_t M = E / R;
    int32_t G = R * S;
    for (int32_t r = 0; r < R; ++r) load[r] = 0;
    for (int32_t e = 0; e < E; ++e) {
        int64_t j = 0;
        load[e / M] += or_quota(L[e], c[e], j);
        j = 1;
        for (int32_t g = 0; g < G; ++g) {
            if (slot_expert[g] == e) {
                load[g / S] += or_quota(L[e], c[e], j);
                j += 1;
            }
        }
    }
}

/*
 * Quota-driven replication plan ([P2] "How balancing in 300 microseconds
 * works": a quota-driven scheduler reacting right after gating; [P3]
 * "Interface / 2. Forward and backward": update_placement computes the
 * per-microbatch replication plan from the exact load).
 *
 * Rule, as fixed for this project:
 *   start with one copy per expert (its master) and every redundant slot
 *   empty; quotas and rank loads as in or_quota / or_rank_loads; then repeat:
 *     stop if 50*R*max_r load_r <= 51*Q (max <= 1.02 x mean, mean = Q/R),
 *     or if no redundant slot is free;
 *     e* = argmax_e L_e / c_e, compared as L_a*c_b > L_b*c_a, ties to the
 *          lowest e, over the experts with L_e >= min_tokens * (c_e + 1)
 *          ([P3] "Performance Tuning / Replication planning": a minimal load
 *          per replica; min_tokens = 0 takes every expert); stop if none;
 *     r* = argmin load_r over ranks with a free slot, ties to the lowest r;
 *     put the new copy of e* in r*'s lowest free slot; c_{e*} += 1.
 *
 * Outputs (caller-allocated):
 *   slot_expert[G]   expert held by redundant slot g, -1 if empty
 *   n_copies[E]      c_e
 *   slot_quota[P]    quota of physical slot p (rank-major; rank r owns
 *                    p = r*(M+S) + m for its masters m < M, then
 *                    p = r*(M+S) + M + s for its redundant slots)
 *   slot_offset[P+1] exclusive running sum of slot_quota in p order
 *   rank_load[R]     final rank loads
 *   stats[4]         {iterations, max rank load before, max rank load after,
 *                     copies placed on a rank that already held a copy of
 *                     the same expert}
 *   trace_e, trace_r (optional, [G]) the chosen e*, r* of every iteration.
 */
int or_plan(int32_t R, int32_t E, int32_t S, const int32_t* load_e,
            int32_t min_tokens,
            int32_t* slot_expert, int32_t* n_copies, int32_t* slot_quota,
            int32_t* slot_offset, int32_t* rank_load, int32_t* stats,
            int32_t* trace_e, int32_t* trace_r)
{
    if (R < 1 || E < 1 || S < 0 || E % R != 0 || min_tokens < 0 || !load_e || !n_copies ||
        !slot_quota || !slot_offset || !rank_load || !stats ||
        (S > 0 && !slot_expert))
        return OR_EINVAL;
    int32_t M = E / R;
    int32_t G = R * S;
    int32_t P = R * (M + S);
    int64_t Q = 0;
    for (int32_t e = 0; e < E; ++e) {
        if (load_e[e] < 0) return OR_EDATA;
        Q += load_e[e];
    }
    int64_t* load = (int64_t*)malloc(sizeof(int64_t) * (size_t)R);
    if (!load) return OR_ENOMEM;

    for (int32_t g = 0; g < G; ++g) slot_expert[g] = -1;
    for (int32_t e = 0; e < E; ++e) n_copies[e] = 1;

    int32_t iters = 0, colocated = 0;
    int64_t max_before = 0;
    for (;;) {
        or_rank_loads(R, E, S, load_e, n_copies, slot_expert, load);
        int64_t maxl = 0;
        for (int32_t r = 0; r < R; ++r)
            if (load[r] > maxl) maxl = load[r];
        if (iters == 0) max_before = maxl;
        if (50 * (int64_t)R * maxl <= 51 * Q) break;

        int32_t rstar = -1;
        for (int32_t r = 0; r < R; ++r) {
            int32_t used = 0;
            for (int32_t s = 0; s < S; ++s)
                if (slot_expert[r * S + s] != -1) used += 1;
            if (used < S && (rstar < 0 || load[r] < load[rstar])) rstar = r;
        }
        if (rstar < 0) break; /* no free slot anywhere */

        /* e* among the experts that may take another copy: with a minimum
         * of m pairs per replica, each of the c+1 copies must still get
         * floor(L/(c+1)) >= m pairs, i.e. L >= m*(c+1) (m = 0: every expert) */
        int32_t estar = -1;
        for (int32_t e = 0; e < E; ++e) {
            if ((int64_t)load_e[e] < (int64_t)min_tokens * (n_copies[e] + 1)) continue;
            if (estar < 0 ||
                (int64_t)load_e[e] * n_copies[estar] >
                (int64_t)load_e[estar] * n_copies[e])
                estar = e;
        }
        if (estar < 0) break; /* no expert may take another copy */

        int32_t s_free = 0;
        while (slot_expert[rstar * S + s_free] != -1) s_free += 1;

        int hosts = (estar / M == rstar);
        for (int32_t s = 0; s < S; ++s)
            if (slot_expert[rstar * S + s] == estar) hosts = 1;
        if (hosts) colocated += 1;

        if (trace_e) trace_e[iters] = estar;
        if (trace_r) trace_r[iters] = rstar;
        slot_expert[rstar * S + s_free] = estar;
        n_copies[estar] += 1;
        iters += 1;
    }

    or_rank_loads(R, E, S, load_e, n_copies, slot_expert, load);
    int64_t max_after = 0;
    for (int32_t r = 0; r < R; ++r) {
        rank_load[r] = (int32_t)load[r];
        if (load[r] > max_after) max_after = load[r];
    }

    for (int32_t p = 0; p < P; ++p) {
        int32_t r = p / (M + S);
        int32_t l = p % (M + S);
        if (l < M) {
            int32_t e = r * M + l;
            slot_quota[p] = (int32_t)or_quota(load_e[e], n_copies[e], 0);
        } else {
            int32_t g = r * S + (l - M);
            int32_t e = slot_expert[g];
            if (e < 0) {
                slot_quota[p] = 0;
            } else {
                int64_t j = 1;
                for (int32_t h = 0; h < g; ++h)
                    if (slot_expert[h] == e) j += 1;
                slot_quota[p] = (int32_t)or_quota(load_e[e], n_copies[e], j);
            }
        }
    }
    slot_offset[0] = 0;
    for (int32_t p = 0; p < P; ++p)
        slot_offset[p + 1] = slot_offset[p] + slot_quota[p];

    stats[0] = iters;
    stats[1] = (int32_t)max_before;
    stats[2] = (int32_t)max_after;
    stats[3] = colocated;
    free(load);
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* reroute                                                                   */
/* ------------------------------------------------------------------------ */

/*
 * Logical -> physical routing ([P3] "Interface / 2. Forward and backward":
 * reroute expands logical routing to physical replicas). Pairs are taken in
 * global order i = 0..Q-1 (rank, token, k); the o-th pair of expert e (o
 * counted from 0 in that order) goes to the copy j whose quota range
 * [start_j, start_j + q_j) contains o, copies ordered master first, then
 * replicas by ascending redundant-slot index. Its destination row in the
 * dispatch buffer is slot_offset[p] + (o - start_j), p the copy's slot.
 * Inputs are the plan's slot_expert, slot_quota and slot_offset.
 */
int or_reroute(const int32_t* idx, int64_t Q, int32_t R, int32_t E, int32_t S,
               const int32_t* slot_expert, const int32_t* slot_quota,
               const int32_t* slot_offset, int32_t* phys_slot,
               int32_t* dest_row)
{
    if (!idx || !phys_slot || !dest_row || !slot_quota || !slot_offset ||
        R < 1 || E < 1 || S < 0 || E % R != 0 || Q < 0 ||
        (S > 0 && !slot_expert))
        return OR_EINVAL;
    int32_t M = E / R;
    int32_t G = R * S;
    int64_t* seen = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    if (!seen) return OR_ENOMEM;
    for (int64_t i = 0; i < Q; ++i) {
        int32_t e = idx[i];
        if (e < 0 || e >= E) { free(seen); return OR_EDATA; }
        int64_t o = seen[e];
        seen[e] += 1;

        int32_t found = -1;
        int64_t start = 0;
        /* copy 0: the master */
        int32_t p = (e / M) * (M + S) + (e % M);
        if (o < start + slot_quota[p]) {
            found = p;
        } else {
            start += slot_quota[p];
            for (int32_t g = 0; g < G && found < 0; ++g) {
                if (slot_expert[g] != e) continue;
                p = (g / S) * (M + S) + M + (g % S);
                if (o < start + slot_quota[p]) found = p;
                else start += slot_quota[p];
            }
        }
        if (found < 0) { free(seen); return OR_EDATA; }
        phys_slot[i] = found;
        dest_row[i] = slot_offset[found] + (int32_t)(o - start);
    }
    free(seen);
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* capacity planner: bisection on the balancing ratio                        */
/* ------------------------------------------------------------------------ */

/*
 * Quota oracle at rank capacity C ([P3] "Performance Tuning / Replication
 * planning": the balancing binary search tests candidate ratios with a quota
 * oracle; a minimal load per replica; zero-load masters off by default). The
 * pages name these knobs only; the steps below are the project's reading.
 * H_r is the load of rank r's masters.
 *   1. Shedding. Each rank with H_r > C must hand X = H_r - C pairs to
 *      replicas. It visits its masters by load, largest first (ties to the
 *      lower e). A master e can give up to a_e = L_e - keep_e pairs, where
 *      keep_e = 1 (0 if zero-load masters are allowed, or if L_e = 0); if
 *      a_e >= m it gives s_e = max(min(X_left, a_e), m), otherwise nothing.
 *      C is infeasible if X is not covered.
 *   2. Receivers. Every rank offers spare capacity max(0, C - H_r) and its S
 *      redundant slots.
 *   3. Placement. The experts with s_e > 0, largest s_e first (ties to the
 *      lower e), are placed one at a time. While rem pairs of e are left, the
 *      receiver r* is the rank with the largest spare capacity (ties to the
 *      lower r) among those that have a free slot. Its piece is
 *      min(rem, spare_r*), cut to rem - m when it would leave
 *      0 < rem - piece < m. A piece below m, or no rank with a free slot,
 *      makes C infeasible. The replica takes r*'s lowest free slot, with the
 *      piece as its quota.
 *   Two things follow without being tested: e's master rank sheds, so its
 *   spare is 0 and it never takes a piece of e; and a piece either ends the
 *   demand or leaves its receiver less than m spare, so no rank takes two
 *   pieces of one expert.
 *   The master keeps L_e - s_e.
 * Returns 1 if C is feasible (outputs filled), 0 if not, < 0 on error.
 * Outputs: slot_expert[G] (-1 empty), slot_q[G] replica quotas, shed[E].
 */
static int or_quota_oracle(int32_t R, int32_t E, int32_t S, const int32_t* L,
                           int64_t C, int32_t m, int32_t allow_zero,
                           int32_t* slot_expert, int64_t* slot_q, int64_t* shed)
{
    int32_t M = E / R;
    int32_t G = R * S;
    int64_t* spare = (int64_t*)malloc(sizeof(int64_t) * (size_t)R);
    int32_t* nfree = (int32_t*)malloc(sizeof(int32_t) * (size_t)R);
    char* done = (char*)malloc((size_t)E);
    if (!spare || !nfree || !done) {
        free(spare); free(nfree); free(done);
        return OR_ENOMEM;
    }
    int ok = 1;
    for (int32_t g = 0; g < G; ++g) {
        slot_expert[g] = -1;
        slot_q[g] = 0;
    }
    for (int32_t e = 0; e < E; ++e) {
        shed[e] = 0;
        done[e] = 0;
    }
    for (int32_t r = 0; r < R; ++r) {
        int64_t H = 0;
        for (int32_t l = 0; l < M; ++l) H += L[r * M + l];
        spare[r] = H <= C ? C - H : 0;
        nfree[r] = S;
    }

    /* 1. shedding */
    for (int32_t r = 0; r < R && ok; ++r) {
        int64_t H = 0;
        for (int32_t l = 0; l < M; ++l) H += L[r * M + l];
        if (H <= C) continue;
        int64_t X = H - C;
        while (X > 0) {
            int32_t best = -1;
            for (int32_t l = 0; l < M; ++l) {
                int32_t e = r * M + l;
                if (!done[e] && (best < 0 || L[e] > L[best])) best = e;
            }
            if (best < 0) { ok = 0; break; }
            done[best] = 1;
            int64_t keep = (allow_zero || L[best] == 0) ? 0 : 1;
            int64_t avail = (int64_t)L[best] - keep;
            if (avail < m) continue;
            int64_t s = X < avail ? X : avail;
            if (s < m) s = m;
            shed[best] = s;
            X -= s;
        }
    }

    /* 3. placement */
    for (int32_t e = 0; e < E; ++e) done[e] = 0;
    while (ok) {
        int32_t e = -1;
        for (int32_t f = 0; f < E; ++f)
            if (!done[f] && shed[f] > 0 && (e < 0 || shed[f] > shed[e])) e = f;
        if (e < 0) break;
        done[e] = 1;
        int64_t rem = shed[e];
        while (rem > 0) {
            int32_t rs = -1;
            for (int32_t r = 0; r < R; ++r) {
                if (nfree[r] == 0) continue;
                if (rs < 0 || spare[r] > spare[rs]) rs = r;
            }
            if (rs < 0) { ok = 0; break; }
            int64_t piece = rem < spare[rs] ? rem : spare[rs];
            if (rem - piece > 0 && rem - piece < m) piece = rem - m;
            if (piece < m) { ok = 0; break; }
            int32_t g = rs * S + (S - nfree[rs]);
            slot_expert[g] = e;
            slot_q[g] = piece;
            spare[rs] -= piece;
            nfree[rs] -= 1;
            rem -= piece;
        }
    }
    free(spare);
    free(nfree);
    free(done);
    return ok;
}

/*
 * Capacity planner ([P3] "Performance Tuning / Replication planning": a
 * binary search on the balancing ratio max/mean with a numerical tolerance
 * eps, an early-stop target, and a quota oracle per candidate). Reading
 * fixed for this project: the ratio runs on the grid k/D (eps = 1/D); the
 * capacity of grid point k is C(k) = floor(k*Q / (D*R)). The search
 *   probes k = thr first and stops there if C(thr) is feasible;
 *   otherwise lo = thr, hi = the smallest k with C(k) >= max_r H_r (feasible
 *   with no replica at all), and while hi - lo > 1 it probes
 *   mid = lo + (hi - lo)/2, setting hi = mid if feasible, else lo = mid.
 * The plan is the quota oracle's result at C(hi) (at C(thr) on an early
 * stop). Copies are ordered master first, then replicas by ascending g;
 * their quotas are whatever the oracle gave them.
 * Outputs as or_plan; stats = {probes, max rank load before, max rank load
 * after, final grid point k}.
 */
int or_plan_bisect(int32_t R, int32_t E, int32_t S, const int32_t* load_e,
                   int32_t eps_inv, int32_t threshold, int32_t min_tokens,
                   int32_t allow_zero, int32_t* slot_expert, int32_t* n_copies,
                   int32_t* slot_quota, int32_t* slot_offset, int32_t* rank_load,
                   int32_t* stats)
{
    if (R < 1 || E < 1 || S < 0 || E % R != 0 || eps_inv < 1 || threshold < 0 ||
        min_tokens < 1 || !load_e || !n_copies || !slot_quota || !slot_offset ||
        !rank_load || !stats || (S > 0 && !slot_expert))
        return OR_EINVAL;
    int32_t M = E / R;
    int32_t G = R * S;
    int32_t P = R * (M + S);
    int64_t Q = 0, maxH = 0;
    for (int32_t e = 0; e < E; ++e) {
        if (load_e[e] < 0) return OR_EDATA;
        Q += load_e[e];
    }
    for (int32_t r = 0; r < R; ++r) {
        int64_t H = 0;
        for (int32_t l = 0; l < M; ++l) H += load_e[r * M + l];
        if (H > maxH) maxH = H;
    }
    int32_t* se = (int32_t*)malloc(sizeof(int32_t) * (size_t)(G > 0 ? G : 1));
    int64_t* sq = (int64_t*)malloc(sizeof(int64_t) * (size_t)(G > 0 ? G : 1));
    int64_t* shed = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
    if (!se || !sq || !shed) {
        free(se); free(sq); free(shed);
        return OR_ENOMEM;
    }
    const int64_t DR = (int64_t)eps_inv * R;
    int32_t probes = 1;
    int64_t k = threshold;
    int rc = or_quota_oracle(R, E, S, load_e, k * Q / DR, min_tokens, allow_zero, se, sq, shed);
    if (rc < 0) goto out;
    if (rc == 0) {
        int64_t lo = threshold;
        int64_t hi = (DR * maxH + Q - 1) / Q; /* Q > 0: with Q = 0 every C is feasible */
        if (hi <= lo) hi = lo + 1;
        while (hi - lo > 1) {
            int64_t mid = lo + (hi - lo) / 2;
            rc = or_quota_oracle(R, E, S, load_e, mid * Q / DR, min_tokens, allow_zero, se,
                                 sq, shed);
            probes += 1;
            if (rc < 0) goto out;
            if (rc == 1) hi = mid;
            else lo = mid;
        }
        k = hi;
        rc = or_quota_oracle(R, E, S, load_e, k * Q / DR, min_tokens, allow_zero, se, sq, shed);
        if (rc < 0) goto out;
        if (rc == 0) { rc = OR_EDATA; goto out; } /* C(hi) must be feasible */
    }

    for (int32_t g = 0; g < G; ++g) slot_expert[g] = se[g];
    for (int32_t e = 0; e < E; ++e) {
        n_copies[e] = 1;
        for (int32_t g = 0; g < G; ++g)
            if (se[g] == e) n_copies[e] += 1;
    }
    for (int32_t p = 0; p < P; ++p) {
        int32_t r = p / (M + S);
        int32_t l = p % (M + S);
        if (l < M) {
            int32_t e = r * M + l;
            slot_quota[p] = (int32_t)(load_e[e] - shed[e]);
        } else {
            slot_quota[p] = (int32_t)sq[r * S + (l - M)];
        }
    }
    slot_offset[0] = 0;
    for (int32_t p = 0; p < P; ++p) slot_offset[p + 1] = slot_offset[p] + slot_quota[p];
    int64_t max_after = 0;
    for (int32_t r = 0; r < R; ++r) {
        int64_t ld = 0;
        for (int32_t l = 0; l < M + S; ++l) ld += slot_quota[r * (M + S) + l];
        rank_load[r] = (int32_t)ld;
        if (ld > max_after) max_after = ld;
    }
    stats[0] = probes;
    stats[1] = (int32_t)maxH;
    stats[2] = (int32_t)max_after;
    stats[3] = (int32_t)k;
    rc = OR_OK;
out:
    free(se);
    free(sq);
    free(shed);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* reroute orders beyond the global prefix fill                              */
/* ------------------------------------------------------------------------ */

/* The copy of expert e that holds its o-th pair under quota-ordered prefix
 * fill (master first, then replicas by ascending g), and that copy's start. */
static int32_t or_copy_of(int32_t e, int64_t o, int32_t M, int32_t S, int32_t G,
                          const int32_t* slot_expert, const int32_t* slot_quota,
                          int64_t* start_out)
{
    int64_t start = 0;
    int32_t p = (e / M) * (M + S) + (e % M);
    if (o < start + slot_quota[p]) {
        *start_out = start;
        return p;
    }
    start += slot_quota[p];
    for (int32_t g = 0; g < G; ++g) {
        if (slot_expert[g] != e) continue;
        p = (g / S) * (M + S) + M + (g % S);
        if (o < start + slot_quota[p]) {
            *start_out = start;
            return p;
        }
        start += slot_quota[p];
    }
    return -1;
}

/*
 * Interleaved reroute ([P3] "Performance Tuning / Replication planning":
 * interleave the token order so that the dispatch that follows does not
 * congest). Reading fixed for this project: the copies are filled by prefix
 * sum exactly as in or_reroute, but the pairs are taken token-major across
 * the source ranks, in the order (t, r, k): token 0 of every rank, then token
 * 1 of every rank, and so on. Each copy then receives a contiguous range of
 * token positions from every source rank instead of whole source ranks.
 * Rows of a slot hold its pairs in that order.
 */
int or_reroute_interleave(const int32_t* idx, int32_t R, int32_t T, int32_t K, int32_t E,
                          int32_t S, const int32_t* slot_expert, const int32_t* slot_quota,
                          const int32_t* slot_offset, int32_t* phys_slot, int32_t* dest_row)
{
    if (!idx || !phys_slot || !dest_row || !slot_quota || !slot_offset || R < 1 || T < 0 ||
        K < 1 || E < 1 || S < 0 || E % R != 0 || (S > 0 && !slot_expert))
        return OR_EINVAL;
    int32_t M = E / R;
    int32_t G = R * S;
    int64_t* seen = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    if (!seen) return OR_ENOMEM;
    for (int32_t t = 0; t < T; ++t) {
        for (int32_t r = 0; r < R; ++r) {
            for (int32_t k = 0; k < K; ++k) {
                int64_t i = ((int64_t)r * T + t) * K + k;
                int32_t e = idx[i];
                if (e < 0 || e >= E) { free(seen); return OR_EDATA; }
                int64_t o = seen[e];
                seen[e] += 1;
                int64_t start = 0;
                int32_t p = or_copy_of(e, o, M, S, G, slot_expert, slot_quota, &start);
                if (p < 0) { free(seen); return OR_EDATA; }
                phys_slot[i] = p;
                dest_row[i] = slot_offset[p] + (int32_t)(o - start);
            }
        }
    }
    free(seen);
    return OR_OK;
}

/*
 * Locality-aware split of every copy's quota over the source ranks ([P3]
 * "Performance Tuning / Replication planning": a locality-aware per-rank
 * quota decomposition that cuts remote traffic). Reading fixed for this
 * project, per expert e with copies j in copy order (master, then replicas
 * by ascending g) on host ranks h_j with quotas q_j, and source loads
 * s_r = load_re[r][e] (they must sum to the quotas' sum):
 *   local pass:  every copy j, in copy order, first takes
 *                min(s_{h_j}, q_j) pairs from its own host rank;
 *   remote pass: every copy j, in copy order, fills the rest of its quota
 *                from the source ranks in ascending r.
 * Outputs ([R][P], rank-major):
 *   src_quota[r][p]   pairs of source rank r assigned to physical slot p;
 *   src_offset[r][p]  dispatch row of the first of them: a slot holds its
 *                     pairs by source rank, so this is slot_offset[p] plus
 *                     the pairs that lower source ranks send to p.
 */
int or_locality_split(int32_t R, int32_t E, int32_t S, const int32_t* load_re,
                      const int32_t* slot_expert, const int32_t* slot_quota,
                      const int32_t* slot_offset, int32_t* src_quota, int32_t* src_offset)
{
    if (R < 1 || E < 1 || S < 0 || E % R != 0 || !load_re || !slot_quota || !slot_offset ||
        !src_quota || !src_offset || (S > 0 && !slot_expert))
        return OR_EINVAL;
    int32_t M = E / R;
    int32_t G = R * S;
    int32_t P = R * (M + S);
    int64_t* s = (int64_t*)malloc(sizeof(int64_t) * (size_t)R);
    int32_t* cp = (int32_t*)malloc(sizeof(int32_t) * (size_t)(1 + G));
    int64_t* q = (int64_t*)malloc(sizeof(int64_t) * (size_t)(1 + G));
    if (!s || !cp || !q) {
        free(s); free(cp); free(q);
        return OR_ENOMEM;
    }
    for (int64_t x = 0; x < (int64_t)R * P; ++x) src_quota[x] = 0;
    int rc = OR_OK;
    for (int32_t e = 0; e < E && rc == OR_OK; ++e) {
        int32_t c = 0;
        cp[c++] = (e / M) * (M + S) + (e % M);
        for (int32_t g = 0; g < G; ++g)
            if (slot_expert[g] == e) cp[c++] = (g / S) * (M + S) + M + (g % S);
        int64_t sum_s = 0, sum_q = 0;
        for (int32_t r = 0; r < R; ++r) {
            s[r] = load_re[(int64_t)r * E + e];
            if (s[r] < 0) rc = OR_EDATA;
            sum_s += s[r];
        }
        for (int32_t j = 0; j < c; ++j) {
            q[j] = slot_quota[cp[j]];
            sum_q += q[j];
        }
        if (rc != OR_OK || sum_s != sum_q) {
            rc = OR_EDATA;
            break;
        }
        /* local pass */
        for (int32_t j = 0; j < c; ++j) {
            int32_t h = cp[j] / (M + S);
            int64_t a = s[h] < q[j] ? s[h] : q[j];
            src_quota[(int64_t)h * P + cp[j]] += (int32_t)a;
            s[h] -= a;
            q[j] -= a;
        }
        /* remote pass */
        for (int32_t j = 0; j < c; ++j) {
            for (int32_t r = 0; r < R && q[j] > 0; ++r) {
                int64_t a = s[r] < q[j] ? s[r] : q[j];
                src_quota[(int64_t)r * P + cp[j]] += (int32_t)a;
                s[r] -= a;
                q[j] -= a;
            }
        }
    }
    if (rc == OR_OK) {
        for (int32_t p = 0; p < P; ++p) {
            int64_t run = slot_offset[p];
            for (int32_t r = 0; r < R; ++r) {
                src_offset[(int64_t)r * P + p] = (int32_t)run;
                run += src_quota[(int64_t)r * P + p];
            }
        }
    }
    free(s);
    free(cp);
    free(q);
    return rc;
}

/*
 * Reroute under the locality-aware split: source rank r gives its pairs of
 * expert e, in its own order (t, k), to e's copies in copy order,
 * src_quota[r][p] pairs each; the pair's dispatch row is src_offset[r][p]
 * plus its position within that run.
 */
int or_reroute_local(const int32_t* idx, int32_t R, int32_t T, int32_t K, int32_t E,
                     int32_t S, const int32_t* slot_expert, const int32_t* src_quota,
                     const int32_t* src_offset, int32_t* phys_slot, int32_t* dest_row)
{
    if (!idx || !phys_slot || !dest_row || !src_quota || !src_offset || R < 1 || T < 0 ||
        K < 1 || E < 1 || S < 0 || E % R != 0 || (S > 0 && !slot_expert))
        return OR_EINVAL;
    int32_t M = E / R;
    int32_t G = R * S;
    int32_t P = R * (M + S);
    int64_t* seen = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
    if (!seen) return OR_ENOMEM;
    for (int32_t r = 0; r < R; ++r) {
        for (int32_t e = 0; e < E; ++e) seen[e] = 0;
        const int32_t* xr = src_quota + (int64_t)r * P;
        for (int64_t i = (int64_t)r * T * K; i < (int64_t)(r + 1) * T * K; ++i) {
            int32_t e = idx[i];
            if (e < 0 || e >= E) { free(seen); return OR_EDATA; }
            int64_t o = seen[e];
            seen[e] += 1;
            int32_t found = -1;
            int64_t start = 0;
            int32_t p = (e / M) * (M + S) + (e % M);
            if (o < start + xr[p]) {
                found = p;
            } else {
                start += xr[p];
                for (int32_t g = 0; g < G && found < 0; ++g) {
                    if (slot_expert[g] != e) continue;
                    p = (g / S) * (M + S) + M + (g % S);
                    if (o < start + xr[p]) found = p;
                    else start += xr[p];
                }
            }
            if (found < 0) { free(seen); return OR_EDATA; }
            phys_slot[i] = found;
            dest_row[i] = src_offset[(int64_t)r * P + found] + (int32_t)(o - start);
        }
    }
    free(seen);
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* permute                                                                   */
/* ------------------------------------------------------------------------ */

/*
 * Token dispatch into per-slot contiguous buffers ([P3] "Interface / 2.
 * Forward and backward": dispatch(hidden, probs, routing_map)):
 *     dispatch[dest_row[n*K + k]] = hidden[n]   for every n, k.
 * Rows are d bf16 values, copied as 16-bit payloads.
 */
int or_permute(const uint16_t* hidden, int64_t N, int32_t d, int32_t K,
               const int32_t* dest_row, uint16_t* dispatch)
{
    if (!hidden || !dest_row || !dispatch || N < 0 || d < 1 || K < 1)
        return OR_EINVAL;
    int64_t Q = N * K;
    for (int64_t i = 0; i < Q; ++i) {
        int64_t row = dest_row[i];
        if (row < 0 || row >= Q) return OR_EDATA;
        memcpy(dispatch + row * d, hidden + (i / K) * d,
               sizeof(uint16_t) * (size_t)d);
    }
    return OR_OK;
}

/*
 * The same definition, evaluated at chosen dispatch rows only: out[j] is the
 * hidden row of the pair whose destination is rows[j].
 */
int or_permute_rows(const uint16_t* hidden, int64_t N, int32_t d, int32_t K,
                    const int32_t* dest_row, const int64_t* rows,
                    int64_t nrows, uint16_t* out)
{
    if (!hidden || !dest_row || !rows || !out || N < 0 || d < 1 || K < 1 ||
        nrows < 0)
        return OR_EINVAL;
    int64_t Q = N * K;
    int64_t* pair_of_row = (int64_t*)malloc(sizeof(int64_t) * (size_t)(Q + 1));
    if (!pair_of_row) return OR_ENOMEM;
    for (int64_t r = 0; r < Q; ++r) pair_of_row[r] = -1;
    for (int64_t i = 0; i < Q; ++i) {
        int64_t row = dest_row[i];
        if (row < 0 || row >= Q) { free(pair_of_row); return OR_EDATA; }
        pair_of_row[row] = i;
    }
    for (int64_t j = 0; j < nrows; ++j) {
        int64_t r = rows[j];
        if (r < 0 || r >= Q || pair_of_row[r] < 0) {
            free(pair_of_row);
            return OR_EDATA;
        }
        memcpy(out + j * d, hidden + (pair_of_row[r] / K) * d,
               sizeof(uint16_t) * (size_t)d);
    }
    free(pair_of_row);
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* combine                                                                   */
/* ------------------------------------------------------------------------ */

/* bf16 is the upper half of an IEEE binary32 word. */
static double or_bf16_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Gate-weighted combine / unpermute ([P3] "Interface / 2. Forward and
 * backward": combine(recv_tokens) after the grouped expert GEMM):
 *     out[n][c] = sum_{k=0..K-1} w[n][k] * y[dest_row[n*K + k]][c]
 * in fp64, k ascending. y is bf16 [Q][d] (expert outputs in dispatch order).
 * tokens (optional) lists the token ids to evaluate; out then has one row
 * per listed token. With tokens == NULL every token 0..N-1 is evaluated.
 */
int or_combine(const uint16_t* y, int64_t N, int32_t d, int32_t K,
               const int32_t* dest_row, const double* w,
               const int64_t* tokens, int64_t ntok, double* out)
{
    if (!y || !dest_row || !w || !out || N < 0 || d < 1 || K < 1)
        return OR_EINVAL;
    int64_t Q = N * K;
    int64_t count = tokens ? ntok : N;
    for (int64_t j = 0; j < count; ++j) {
        int64_t n = tokens ? tokens[j] : j;
        if (n < 0 || n >= N) return OR_EDATA;
        for (int32_t c = 0; c < d; ++c) out[j * d + c] = 0.0;
        for (int32_t k = 0; k < K; ++k) {
            int64_t row = dest_row[n * K + k];
            if (row < 0 || row >= Q) return OR_EDATA;
            double wk = w[n * K + k];
            for (int32_t c = 0; c < d; ++c)
                out[j * d + c] += wk * or_bf16_to_double(y[row * d + c]);
        }
    }
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* backward of permute and combine; weight sync; gradient reduction         */
/* ------------------------------------------------------------------------ */

/*
 * Backward of the gate-weighted combine ([P3] "Interface / 2. Forward and
 * backward": reroute gathers gradients back to logical experts in backward;
 * the combine is out[n] = sum_k w[n][k] * y[dest_row[n*K+k]]):
 *     dy[dest_row[n*K+k]] = w[n][k] * dout[n]             (expert outputs)
 *     dw[n][k]            = sum_c dout[n][c] * y[dest_row[n*K+k]][c]   (gates)
 * in fp64. dout fp32 [N][d], y bf16 [Q][d], w fp32 [N][K]. Evaluated for the
 * listed tokens (all when tokens == NULL): dy_rows gets one row per (token, k)
 * in that order ([count*K][d]), dw one row per token ([count][K]).
 */
int or_combine_backward(const float* dout, const uint16_t* y, int64_t N, int32_t d,
                        int32_t K, const int32_t* dest_row, const float* w,
                        const int64_t* tokens, int64_t ntok, double* dy_rows, double* dw)
{
    if (!dout || !y || !dest_row || !w || !dy_rows || !dw || N < 0 || d < 1 || K < 1)
        return OR_EINVAL;
    int64_t Q = N * K;
    int64_t count = tokens ? ntok : N;
    for (int64_t j = 0; j < count; ++j) {
        int64_t n = tokens ? tokens[j] : j;
        if (n < 0 || n >= N) return OR_EDATA;
        for (int32_t k = 0; k < K; ++k) {
            int64_t row = dest_row[n * K + k];
            if (row < 0 || row >= Q) return OR_EDATA;
            double wk = (double)w[n * K + k];
            double dot = 0.0;
            for (int32_t c = 0; c < d; ++c) {
                double g = (double)dout[n * d + c];
                dy_rows[(j * K + k) * d + c] = wk * g;
                dot += g * or_bf16_to_double(y[row * d + c]);
            }
            dw[j * K + k] = dot;
        }
    }
    return OR_OK;
}

/*
 * Backward of the permute (dispatch[dest_row[n*K+k]] = hidden[n]): every
 * token's gradient is the sum of its K dispatched rows' gradients,
 *     dhidden[n] = sum_k ddispatch[dest_row[n*K+k]]
 * in fp64, for the listed tokens (all when tokens == NULL).
 */
int or_permute_backward(const uint16_t* ddispatch, int64_t N, int32_t d, int32_t K,
                        const int32_t* dest_row, const int64_t* tokens, int64_t ntok,
                        double* dhidden)
{
    if (!ddispatch || !dest_row || !dhidden || N < 0 || d < 1 || K < 1) return OR_EINVAL;
    int64_t Q = N * K;
    int64_t count = tokens ? ntok : N;
    for (int64_t j = 0; j < count; ++j) {
        int64_t n = tokens ? tokens[j] : j;
        if (n < 0 || n >= N) return OR_EDATA;
        for (int32_t c = 0; c < d; ++c) dhidden[j * d + c] = 0.0;
        for (int32_t k = 0; k < K; ++k) {
            int64_t row = dest_row[n * K + k];
            if (row < 0 || row >= Q) return OR_EDATA;
            for (int32_t c = 0; c < d; ++c)
                dhidden[j * d + c] += or_bf16_to_double(ddispatch[row * d + c]);
        }
    }
    return OR_OK;
}

/*
 * Weight sync on one GPU ([P3] "Interface / 2. Forward and backward":
 * weight_sync materializes the plan by distributing master weights to replica
 * slots): every redundant slot g holding expert e receives a copy of e's
 * weights, replicas[g] = master[e], bytes_per_expert bytes each; empty slots
 * are left as they are.
 */
int or_weight_sync(int32_t G, const int32_t* slot_expert, int32_t E,
                   const uint8_t* master, uint8_t* replicas, int64_t bytes_per_expert)
{
    if (G < 0 || (G > 0 && (!slot_expert || !replicas)) || !master || E < 1 ||
        bytes_per_expert < 0)
        return OR_EINVAL;
    for (int32_t g = 0; g < G; ++g) {
        int32_t e = slot_expert[g];
        if (e < 0) continue;
        if (e >= E) return OR_EDATA;
        memcpy(replicas + (int64_t)g * bytes_per_expert, master + (int64_t)e * bytes_per_expert,
               (size_t)bytes_per_expert);
    }
    return OR_OK;
}

/*
 * Gradient reduction on one GPU ([P3] "Interface / 2. Forward and backward":
 * grad_reduce reduces replica Wgrad into master-expert gradients; "Performance
 * Tuning / Expert communication": a deterministic, non-atomic reduction):
 *     master[e] + sum over the redundant slots g holding e, ascending g,
 *     of replicas[g]
 * in fp64 (fp32 inputs), written to out [E][numel].
 */
int or_grad_reduce(int32_t G, const int32_t* slot_expert, int32_t E, const float* replicas,
                   const float* master, int64_t numel, double* out)
{
    if (G < 0 || (G > 0 && (!slot_expert || !replicas)) || !master || !out || E < 1 ||
        numel < 0)
        return OR_EINVAL;
    for (int32_t e = 0; e < E; ++e)
        for (int64_t i = 0; i < numel; ++i) out[(int64_t)e * numel + i] = (double)master[(int64_t)e * numel + i];
    for (int32_t g = 0; g < G; ++g) {
        int32_t e = slot_expert[g];
        if (e < 0) continue;
        if (e >= E) return OR_EDATA;
        for (int64_t i = 0; i < numel; ++i)
            out[(int64_t)e * numel + i] += (double)replicas[(int64_t)g * numel + i];
    }
    return OR_OK;
}
