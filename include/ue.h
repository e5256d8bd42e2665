/*
 * ue.h -- C ABI of libue, the B200 (sm_100a) implementation of UltraEP's
 * per-layer, per-microbatch exact-load rebalancing hot path:
 *
 *   ue_gate_topk -> ue_count -> ue_plan -> ue_reroute -> ue_permute
 *   (experts, outside this library) -> ue_combine
 *
 * Sources (page title, section):
 *   "UltraEP" project README, "Interface / 1. Initialization" (one manager
 *     per EP group, redundant slots reserved per rank, no runtime
 *     allocation), "Interface / 2. Forward and backward" (router ->
 *     update_placement -> reroute -> dispatch -> experts -> combine),
 *     "Performance Tuning / NVSHMEM" (global-load metadata before planning);
 *   "Xiaohongshu's UltraEP Balances MoE Experts in 300 us, Reaching 94.3% of
 *     Ideal", "How balancing in 300 microseconds works" (quota-driven
 *     scheduler, rebalancing every microbatch and every layer);
 *   "UltraEP: Real-Time Load Balancing for Large-Scale MoE Training and
 *     Inference", "What Happened" (exact routing, hot experts replicated per
 *     microbatch and per layer).
 *
 * One context simulates one EP group of R ranks on one GPU. Sizes:
 *   R ranks, T tokens per rank, N = R*T tokens (token n lives on rank n/T),
 *   E experts (E % R == 0), M = E/R masters per rank (expert e's master is on
 *   rank e/M), K top-k, S redundant slots per rank, d hidden size (bf16),
 *   Q = N*K token-expert pairs (pair i = n*K + k, "global order"),
 *   G = R*S redundant slots (slot g = r*S + s lives on rank r),
 *   P = R*(M+S) physical slots, rank-major: rank r owns
 *   p = r*(M+S) + m (its masters, m < M) then p = r*(M+S) + M + s.
 *
 * Conventions, for every call below:
 *   - Pointers are device pointers unless stated otherwise. The caller owns
 *     every input and output buffer; the context owns only its scratch.
 *   - Every call is asynchronous on the given stream (0 = legacy default
 *     stream), performs no host synchronisation and allocates nothing.
 *     Output sizes never depend on the data.
 *   - Host-side errors (null or misaligned pointers, sizes out of range,
 *     a destroyed context) are returned at once and nothing is launched.
 *   - Device-side errors (an expert id out of range, a row index out of
 *     range, a wait that ran out) are recorded in the context's error word;
 *     the kernel skips the offending element or returns early. They are
 *     read (and cleared) with ue_get_error. No device code traps.
 *   - One context must not be used from two streams at once.
 */
#ifndef UE_H
#define UE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    UE_OK = 0,
    UE_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or config   */
    UE_ERR_CUDA = 2,          /* a CUDA runtime call failed               */
    UE_ERR_NOMEM = 3,         /* scratch allocation failed in ue_init     */
    UE_ERR_DEVICE_BOUNDS = 4, /* a kernel met an out-of-range id or row   */
    UE_ERR_TIMEOUT = 5,       /* a bounded device-side wait ran out       */
    UE_ERR_UNSUPPORTED = 6    /* no sm_100 device, or sizes beyond limits */
} ue_status;

/* Sizes of one simulated EP group. Limits: 1 <= R <= 128; 1 <= E <= 256;
 * E % R == 0; 1 <= K <= min(E, 32); 0 <= S <= 8 and R*S <= 256; T >= 1;
 * Q = R*T*K < 2^30; d >= 8, d % 8 == 0 (rows are whole 16-byte units) and
 * d <= 16384. */
typedef struct {
    int32_t R, T, E, K, S, d;
} ue_config;

/* The replication plan of one layer instance ("placement": the pages'
 * update_placement). All arrays are int32 device buffers owned by the
 * caller, written by ue_plan and read by ue_reroute.
 *   slot_expert [G]   expert held by redundant slot g, -1 when empty
 *   n_copies    [E]   copies of expert e (master included), >= 1
 *   slot_quota  [P]   pairs assigned to physical slot p
 *   slot_offset [P+1] exclusive running sum of slot_quota: slot p's rows in
 *                     the dispatch buffer are [slot_offset[p],
 *                     slot_offset[p+1]); rank r's receive buffer is
 *                     [slot_offset[r*(M+S)], slot_offset[(r+1)*(M+S)])
 *   rank_load   [R]   pairs each rank processes under the plan
 *   stats       [4]   {iterations, max rank load before (masters only),
 *                      max rank load after, copies placed on a rank that
 *                      already held a copy of the same expert} (ue_plan;
 *                      ue_plan_ex's capacity planner writes other stats)
 * slot_expert may be NULL when S == 0. */
typedef struct {
    int32_t* slot_expert;
    int32_t* n_copies;
    int32_t* slot_quota;
    int32_t* slot_offset;
    int32_t* rank_load;
    int32_t* stats;
} ue_placement;

typedef struct ue_ctx ue_ctx; /* opaque */

/* Create a context for `cfg` on CUDA device `device` (made current) and
 * allocate its scratch once: the error word, the reroute's look-back status
 * words (ceil(Q/tile)*E 64-bit words, a tile being 512 threads x 7 to 32
 * pairs, the smallest size whose tiles are all resident on the device at
 * once; a word per group of 16 tiles and expert, a counter per group, a
 * ticket, a counter and an epoch),
 * the locality order's two int32 [R][P] tables, a row of d zero bf16 values
 * (the combine reads it in place of a row out of range) and the gradient
 * reduction's int32 lists of replicated experts and their slots (at most
 * 3*256 + 256 + 1 words). Nothing is allocated
 * after this call ("Interface / 1. Initialization": buffers reserved up
 * front, no dynamic allocation at runtime).
 * Returns UE_ERR_INVALID_ARG for a null `out` or a config outside the
 * limits (checked before any CUDA call), UE_ERR_UNSUPPORTED if the device
 * is not compute capability 10.x, UE_ERR_CUDA / UE_ERR_NOMEM on failure.
 * On error *out is set to NULL. */
ue_status ue_init(const ue_config* cfg, int device, ue_ctx** out);

/* Free the context's scratch (synchronises the device first); the end of
 * the Manager's life ("Interface / 1. Initialization"). NULL is accepted
 * and ignored. Returns UE_OK, UE_ERR_INVALID_ARG for a pointer that is not
 * a live context, or UE_ERR_CUDA if the synchronisation failed (the
 * context is freed in every case but the first two). */
ue_status ue_destroy(ue_ctx* ctx);

/* Synchronise `stream`, then read and clear the context's device error
 * word (the pages have no counterpart: their calls raise in Python). Returns
 * UE_OK, UE_ERR_DEVICE_BOUNDS, UE_ERR_TIMEOUT, or UE_ERR_CUDA if the
 * synchronisation itself failed. */
ue_status ue_get_error(ue_ctx* ctx, void* stream);

/* Router gating ("Interface / 2. Forward and backward": probs, routing_map
 * = router(hidden); "What Happened": exact routing probabilities).
 *   logits fp32 [N][E] row-major, 4-byte aligned.
 *   idx    int32 [N][K]: per token the K experts with the largest logits,
 *          in descending logit order; equal logits (IEEE ==, -0.0 == +0.0)
 *          go to the lower expert id. Logits must be finite.
 *   w      fp32 [N][K]: softmax over the K selected logits,
 *          w_k = exp(v_k - v_0) / sum_j exp(v_j - v_0), evaluated in fp64
 *          and rounded once to fp32.
 * Errors: host-side only (null or misaligned pointers); any finite logits
 * are valid input. */
ue_status ue_gate_topk(ue_ctx* ctx, const float* logits, int32_t* idx,
                       float* w, void* stream);

/* Exact per-expert load ("UltraEP" README intro: rebalance on the exact
 * post-gating load; "Performance Tuning / NVSHMEM": per-rank load metadata
 * gathered before planning).
 *   idx     int32 [N][K] expert ids (from ue_gate_topk).
 *   load_re int32 [R][E]: pairs of source rank r routed to expert e.
 *   load_e  int32 [E]: sum over r of load_re.
 * Both outputs are overwritten: the kernel's first CTA zeroes them, and the
 * others add their counts after it (a bounded wait; UE_ERR_TIMEOUT if it
 * runs out). Uses the same context scratch as ue_gate_count (a ticket, a
 * counter, an epoch and a flag), so calls on one context must not overlap on
 * the GPU. An id outside [0, E) is skipped and sets UE_ERR_DEVICE_BOUNDS. */
ue_status ue_count(ue_ctx* ctx, const int32_t* idx, int32_t* load_re,
                   int32_t* load_e, void* stream);

/* ue_gate_topk and ue_count in one call ("Interface / 2. Forward and
 * backward": the router's routing; "UltraEP" README intro: the exact
 * post-gating load): the same idx, w, load_re and load_e as the two calls in
 * sequence (same arguments, same layouts, the same errors). For K = 8 and E a multiple of 32 from 64 to 256 the histogram is
 * taken inside the gate kernel (each CTA adds its picks to a shared
 * histogram per source rank and its bins to the outputs at the end), so
 * idx is not read back; other shapes run the two kernels. Uses context
 * scratch (a ticket, a counter, an epoch and a flag), so calls on one
 * context must not overlap on the GPU. */
ue_status ue_gate_count(ue_ctx* ctx, const float* logits, int32_t* idx, float* w,
                        int32_t* load_re, int32_t* load_e, void* stream);

/* Quota-driven replication plan ("How balancing in 300 microseconds works";
 * "Interface / 2. Forward and backward": update_placement).
 *   load_e int32 [E] exact per-expert pair counts, Q = sum(load_e).
 * Rule: start with the masters only; quota of copy j of expert e (j = 0 the
 * master, then replicas by ascending g) is floor(L_e/c_e) plus one for the
 * first L_e mod c_e copies; a rank's load is the sum of its copies' quotas.
 * Repeat: stop if 50*R*max_r load_r <= 51*Q (max <= 1.02 x mean) or no slot
 * is free; else take e* = argmax L_e/c_e (exact integer comparison, ties to
 * the lowest e) and give it a copy in the lowest free slot of the least
 * loaded rank that has one (ties to the lowest r).
 * Writes every array of `out` (device pointers, see ue_placement). Runs as
 * a single CTA. A negative entry of load_e sets UE_ERR_DEVICE_BOUNDS and
 * counts as 0. */
ue_status ue_plan(ue_ctx* ctx, const int32_t* load_e, const ue_placement* out,
                  void* stream);

/* Planner choice for ue_plan_ex. "UltraEP" README, "Performance Tuning /
 * Replication planning" names the knobs followed here (balancing binary
 * search, its early-stop target and ratio tolerance eps, minimal load per
 * replica, zero-load masters); the pages give no algorithm, and the rules
 * below are this library's reading of them. */
typedef struct {
    int32_t solver;            /* UE_SOLVER_GREEDY or UE_SOLVER_BISECT          */
    int32_t min_tokens;        /* minimal pairs per replica: >= 0 for the greedy
                                  (0: no minimum), >= 1 for the bisection
                                  (the pages' default is 1024)                  */
    int32_t eps_inv;           /* bisection: max/mean runs on the grid
                                  k / eps_inv, 1 <= eps_inv <= 10000 (the pages'
                                  default eps = 0.01 is eps_inv = 100)          */
    int32_t threshold;         /* bisection: early-stop ratio in units of
                                  1/eps_inv, >= 0 (the pages' default 1.0 is
                                  threshold = eps_inv)                          */
    int32_t allow_zero_master; /* bisection: 1 lets a master shed all its
                                  pairs (the pages' default is 0)               */
} ue_plan_opts;

enum { UE_SOLVER_GREEDY = 0, UE_SOLVER_BISECT = 1 };

/* Replication plan with a choice of planner ("Performance Tuning /
 * Replication planning"). Arguments as for ue_plan.
 *   UE_SOLVER_GREEDY: the ue_plan rule, where only experts with
 *     L_e >= min_tokens * (c_e + 1) may take a copy (each copy keeps at
 *     least min_tokens pairs); the greedy also stops when no expert may.
 *     stats as for ue_plan. min_tokens = 0 gives exactly ue_plan.
 *   UE_SOLVER_BISECT: a capacity planner. The ratio max/mean runs on the
 *     grid k/D (D = eps_inv), capacity C(k) = floor(k*Q / (D*R)); H_r is the
 *     load of rank r's masters. A quota oracle tests C: every rank with
 *     H_r > C sheds H_r - C pairs from its masters, largest load first (ties
 *     to the lower e), each giving max(min(left, L_e - keep), m) if
 *     L_e - keep >= m (keep = 1, or 0 with allow_zero_master or L_e = 0);
 *     the shed amounts, largest first (ties to the lower e), go in pieces
 *     to the rank with a free slot and the most spare capacity
 *     max(0, C - H_r) (ties to the lower r), piece = min(rem, spare), cut to
 *     rem - m if it would leave 0 < rem - piece < m; a piece below m, no
 *     receiver or uncovered excess fails C; a replica takes its rank's
 *     lowest free slot and the piece as quota; the master keeps the rest.
 *     The search probes k = threshold first and stops if it passes; else it
 *     bisects between lo = threshold and the smallest k with C(k) >= max H
 *     while hi - lo > 1 (success moves hi), and the plan is the oracle's
 *     result at hi. Quotas are then arbitrary per copy (ue_reroute handles
 *     them). stats = {probes, max rank load before, max rank load after,
 *     final grid point k}. Runs as a single CTA of 1024 threads that settles
 *     five levels of the bisection per round.
 * Invalid options return UE_ERR_INVALID_ARG. */
ue_status ue_plan_ex(ue_ctx* ctx, const int32_t* load_e, const ue_plan_opts* opts,
                     const ue_placement* out, void* stream);

/* Logical -> physical routing ("Interface / 2. Forward and backward":
 * reroute expands logical routing to physical replicas).
 *   idx       int32 [N][K] expert ids.
 *   plan      a placement written by ue_plan for the same idx.
 *   phys_slot int32 [N][K]: physical slot of each pair.
 *   dest_row  int32 [N][K]: row of each pair in the dispatch buffer.
 * Pairs in global order fill each expert's copies by prefix sum (master
 * first, then replicas by ascending g): the o-th pair of expert e goes to
 * the copy whose quota range holds o, at row slot_offset[p] + (o - start).
 * dest_row is a permutation of [0, Q). Single pass: a stable counting sort
 * with a decoupled look-back scan over tiles of 3584 to 16384 pairs (the
 * smallest size whose tiles are all resident at once); its waits are
 * bounded and end with UE_ERR_TIMEOUT. Ids outside [0, E) set
 * UE_ERR_DEVICE_BOUNDS. */
ue_status ue_reroute(ue_ctx* ctx, const int32_t* idx, const ue_placement* plan,
                     int32_t* phys_slot, int32_t* dest_row, void* stream);

/* ue_plan then ue_reroute on one stream ("Interface / 2. Forward and
 * backward": update_placement, then reroute), overlapped: the reroute kernel is
 * launched as a programmatic dependent of the plan kernel, so its tiles copy,
 * count and look back over idx on the other SMs while the plan's single CTA
 * runs, and read the plan only after the plan kernel has completed. The
 * results are exactly those of ue_plan followed by ue_reroute.
 *   load_e int32 [E] the histogram of idx (as for ue_plan).
 *   idx, phys_slot, dest_row as for ue_reroute; plan as for both (written,
 *   then read).
 * idx is read while the plan kernel runs. Whatever writes it must come
 * before this call in stream order (as ue_gate_count does); it has then
 * completed before the plan kernel starts. Errors as for ue_plan and
 * ue_reroute. */
ue_status ue_plan_reroute(ue_ctx* ctx, const int32_t* load_e, const int32_t* idx,
                          const ue_placement* plan, int32_t* phys_slot, int32_t* dest_row,
                          void* stream);

enum { UE_ORDER_PREFIX = 0, UE_ORDER_INTERLEAVE = 1 };

/* ue_reroute with a choice of pair order ("UltraEP" README, "Performance
 * Tuning / Replication planning": interleave the token order so that the
 * dispatch that follows does not congest; the reading here is a token-major
 * order across the source ranks).
 *   order UE_ORDER_PREFIX:     exactly ue_reroute (global order (r, t, k)).
 *   order UE_ORDER_INTERLEAVE: the copies are filled by prefix sum with the
 *     pairs taken in the order (t, r, k): token 0 of every rank, then token
 *     1 of every rank, ...; each copy then receives a range of token
 *     positions from every source rank. Rows of a slot hold its pairs in
 *     that order. phys_slot and dest_row are still indexed by pair i.
 * Other arguments and errors as for ue_reroute. */
ue_status ue_reroute_ex(ue_ctx* ctx, const int32_t* idx, const ue_placement* plan,
                        int32_t order, int32_t* phys_slot, int32_t* dest_row,
                        void* stream);

/* Locality-aware split of every copy's quota over the source ranks
 * ("UltraEP" README, "Performance Tuning / Replication planning": a
 * per-rank quota decomposition that cuts remote traffic; the reading here
 * is own-rank first). For expert e with copies j in copy order (master, then
 * replicas by ascending g) on host ranks h_j with quotas q_j, and the source
 * loads s_r = load_re[r][e]:
 *   local pass:  every copy j, in copy order, first takes min(s_{h_j}, q_j)
 *                pairs from its own host rank;
 *   remote pass: every copy j, in copy order, fills the rest of its quota
 *                from the source ranks in ascending r.
 *   load_re    int32 [R][E] from ue_count for the same idx as the plan.
 *   plan       a placement (slot_expert, slot_quota, slot_offset are read).
 *   src_quota  int32 [R][P]: pairs of source rank r assigned to slot p.
 *   src_offset int32 [R][P]: dispatch row of the first of them (a slot
 *              holds its pairs by source rank, then in the source's order).
 * An expert whose source loads do not sum to its quotas, or a slot_expert
 * entry >= E, sets UE_ERR_DEVICE_BOUNDS. */
ue_status ue_locality_split(ue_ctx* ctx, const int32_t* load_re, const ue_placement* plan,
                            int32_t* src_quota, int32_t* src_offset, void* stream);

/* Reroute under the locality-aware split ("Performance Tuning / Replication
 * planning": per-rank quota decomposition): source rank r hands its pairs of
 * expert e, in its own order (t, k), to e's copies in copy order,
 * src_quota[r][p] pairs each, at rows src_offset[r][p], src_offset[r][p]+1,
 * ... The arrays are those ue_locality_split wrote for this plan and load_re
 * (and load_re is ue_count's for idx). Uses the context's [R][P] tables,
 * rebuilt on every call. Other arguments and errors as for ue_reroute; a
 * pair outside its source rank's split sets UE_ERR_DEVICE_BOUNDS. */
ue_status ue_reroute_local(ue_ctx* ctx, const int32_t* idx, const int32_t* load_re,
                           const ue_placement* plan, const int32_t* src_quota,
                           const int32_t* src_offset, int32_t* phys_slot,
                           int32_t* dest_row, void* stream);

/* Token dispatch into per-slot contiguous buffers ("Interface / 2. Forward
 * and backward": dispatch(hidden, probs, routing_map), here a single-GPU
 * gather/scatter).
 *   hidden   bf16 [N][d] (raw 16-bit words), 16-byte aligned.
 *   dest_row int32 [N][K] from ue_reroute (a permutation of [0, Q)).
 *   dispatch bf16 [Q][d], 16-byte aligned, must not overlap hidden:
 *            dispatch[dest_row[n*K+k]] = hidden[n], bit for bit.
 * Rows outside [0, Q) are skipped and set UE_ERR_DEVICE_BOUNDS. */
ue_status ue_permute(ue_ctx* ctx, const uint16_t* hidden,
                     const int32_t* dest_row, uint16_t* dispatch,
                     void* stream);

/* Gate-weighted combine / unpermute ("Interface / 2. Forward and
 * backward": combine(recv_tokens)).
 *   y        bf16 [Q][d] expert outputs in dispatch order, 16-byte aligned.
 *   dest_row int32 [N][K], w fp32 [N][K].
 *   out      fp32 [N][d], 16-byte aligned:
 *            out[n] = sum_{k=0..K-1} w[n][k] * y[dest_row[n*K+k]],
 *            accumulated in fp32 with one fused multiply-add per term,
 *            k ascending, starting from 0.
 * Rows outside [0, Q) contribute nothing and set UE_ERR_DEVICE_BOUNDS. */
ue_status ue_combine(ue_ctx* ctx, const uint16_t* y, const int32_t* dest_row,
                     const float* w, float* out, void* stream);

/* Backward of the combine ("Interface / 2. Forward and backward": reroute
 * gathers gradients back to logical experts in the backward; with the
 * compact [N][K] routing each pair has one physical row, so the gradients
 * are those of the combine):
 *   dout     fp32 [N][d], 16-byte aligned: gradient of `out`.
 *   y        bf16 [Q][d]: the expert outputs the forward combined.
 *   dest_row int32 [N][K], w fp32 [N][K]: as in the forward.
 *   dy       bf16 [Q][d], 16-byte aligned: dy[dest_row[n*K+k]] =
 *            w[n][k] * dout[n], product in fp32 rounded once to bf16.
 *   dw       fp32 [N][K]: dw[n][k] = <dout[n], y[dest_row[n*K+k]]>,
 *            accumulated in fp32 in a fixed order (the same on every run).
 * Rows outside [0, Q) are skipped and set UE_ERR_DEVICE_BOUNDS. */
ue_status ue_combine_backward(ue_ctx* ctx, const float* dout, const uint16_t* y,
                              const int32_t* dest_row, const float* w, uint16_t* dy,
                              float* dw, void* stream);

/* Backward of the permute ("Interface / 2. Forward and backward": the
 * backward pass returns dispatch gradients to the tokens that sent them):
 * dhidden[n] = sum_k ddispatch[dest_row[n*K+k]],
 * fp32 [N][d] (16-byte aligned), k ascending from 0; ddispatch bf16 [Q][d].
 * Rows outside [0, Q) are skipped and set UE_ERR_DEVICE_BOUNDS. */
ue_status ue_permute_backward(ue_ctx* ctx, const uint16_t* ddispatch,
                              const int32_t* dest_row, float* dhidden, void* stream);

/* Weight sync on one GPU ("Interface / 2. Forward and backward":
 * weight_sync distributes master-expert weights to the replica slots;
 * "Interface / 1. Initialization": replica buffers reused across layers).
 *   plan             a placement from ue_plan (slot_expert is read).
 *   master           [E][bytes_per_expert] bytes, 16-byte aligned.
 *   replicas         [G][bytes_per_expert] bytes, 16-byte aligned:
 *                    replicas[g] = master[slot_expert[g]] for every used
 *                    slot; empty slots are left unchanged.
 *   bytes_per_expert > 0 and a multiple of 16 (e.g. bf16 fc1 + fc2 weights:
 *                    2 * (2*h*f + h*f) bytes).
 * A slot_expert entry >= E sets UE_ERR_DEVICE_BOUNDS. */
ue_status ue_weight_sync(ue_ctx* ctx, const ue_placement* plan, const void* master,
                         void* replicas, int64_t bytes_per_expert, void* stream);

/* Gradient reduction on one GPU ("Interface / 2. Forward and backward":
 * grad_reduce reduces replica Wgrad into master-expert gradients;
 * "Performance Tuning / Expert communication": deterministic, non-atomic).
 *   plan             a placement from ue_plan (slot_expert is read).
 *   replica_grads    fp32 [G][numel_per_expert], 16-byte aligned.
 *   master_grads     fp32 [E][numel_per_expert], 16-byte aligned, updated in
 *                    place: master[e] = master[e] + replicas[g1] + ... over
 *                    e's replica slots in ascending g, added in that order,
 *                    so the result is the same on every run.
 *   numel_per_expert > 0 and a multiple of 4.
 * A slot_expert entry >= E sets UE_ERR_DEVICE_BOUNDS and that slot is
 * skipped. */
ue_status ue_grad_reduce(ue_ctx* ctx, const ue_placement* plan, const float* replica_grads,
                         float* master_grads, int64_t numel_per_expert, void* stream);

/* ue_reroute, without a context and without allocating anything (the
 * pages have no counterpart to this call). For callers that cannot call
 * cudaMalloc: code running inside an allocator's hooks or under a memory
 * pool that forbids outside allocations, or code that keeps no context.
 * The look-back scratch is a fixed device array inside libue (about
 * 2.2 MiB, held on every GPU that loads the library until the process
 * exits): sizes with ceil(R*T*K / 8192) * E > 262144 are rejected with
 * UE_ERR_UNSUPPORTED before anything is launched. The first call made with
 * a given device current checks that the device is an sm_100 part
 * (UE_ERR_UNSUPPORTED otherwise), looks up that array's device address
 * (cudaGetSymbolAddress), caches it and sets the reroute kernel's shared
 * memory limit; make that first call before any stream capture. cudaDeviceReset makes the cached address stale: do not
 * call this entry point again in a process that has reset the device.
 * Every call shares the array and it is never cleared: its status words
 * carry the call's epoch, so words left by an earlier call read as
 * unpublished, each group of tiles' last arrival resets the group's
 * counter, and each call's last CTA resets the tile ticket, also after a
 * call that ended in a device-side error. Calls that overlap on the GPU
 * (other streams, other threads) race and give wrong results. Calls no
 * cudaMalloc or cudaFree.
 *   cfg, idx, plan, phys_slot, dest_row, stream: as for ue_init + ue_reroute
 *   (cfg is a host pointer, read during the call). idx, phys_slot,
 *   dest_row, error and the plan arrays must be memory of the current
 *   device (UE_ERR_INVALID_ARG otherwise, before any launch).
 *   error: device int32[2], zeroed by the caller, required (NULL is
 *   UE_ERR_INVALID_ARG): a device-side error writes {code, detail} into it
 *   (the first one only). After a device-side error (an expert id out of
 *   range, a look-back wait that ran out) the outputs are not valid: a pair
 *   with a bad id gets -1, and a timed-out call writes nothing.
 * Host-side errors are returned at once, as for ue_reroute. */
ue_status ue_reroute_noalloc(const ue_config* cfg, const int32_t* idx,
                             const ue_placement* plan, int32_t* phys_slot,
                             int32_t* dest_row, int32_t* error, void* stream);

/* Test hooks for the bounded waits (no counterpart on the pages).
 * ue_debug_set_lookback_limit sets the number of polls a reroute tile makes
 * on a predecessor before it gives up with UE_ERR_TIMEOUT (default 1<<22,
 * with a sleep between polls). ue_debug_drop_first_publish(ctx, 1) makes the
 * first reroute tile skip publishing its counts, so that its successor's
 * wait runs out; 0 restores normal behaviour. */
ue_status ue_debug_set_lookback_limit(ue_ctx* ctx, int64_t polls);
ue_status ue_debug_drop_first_publish(ue_ctx* ctx, int enable);

#ifdef __cplusplus
}
#endif

#endif /* UE_H */
