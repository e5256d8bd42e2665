// ue_internal.cuh -- internal declarations shared by the libue translation
// units (kernels + C ABI). Not installed, not part of the ABI.
#pragma once

#include <algorithm>
#include <climits>
#include <cstdint>
#include <cuda_runtime.h>

#include "ue.h"

namespace ue {

// Device error word layout: err[0] = first ue_status code raised,
// err[1] = a detail value (the offending index or tile).
__device__ __forceinline__ void raise_error(int* err, int code, int detail)
{
    if (atomicCAS(err, 0, code) == 0) {
        atomicExch(err + 1, detail);
    }
}

// acquire load and release store of a 32-bit flag at GPU scope
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start once the kernel before it in the stream has run
// pdl_trigger() in every CTA (or exited); pdl_wait() then blocks the calling
// thread until that kernel has completed and its writes are visible. Both
// are no-ops for kernels launched the ordinary way.
__device__ __forceinline__ void pdl_trigger()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

constexpr int kWarp = 32;
constexpr unsigned kFull = 0xffffffffu;

// Reroute tiling: threads per tile; a tile holds 8 to 32 pairs per thread
// (kRerouteTile: the 16-pair default), chosen per context so that every tile
// is resident at once. The look-back adds the counts of groups of
// kRerouteGroup tiles.
constexpr int kRerouteThreads = 512;
constexpr int kRerouteWarps = kRerouteThreads / kWarp;
constexpr int kRerouteTile = kRerouteThreads * 16;
constexpr int kRerouteGroup = 16;

// Look-back status word (64-bit): [63:32] launch tag, [31:30] flag,
// [29:0] count. A word whose tag is not the current launch's reads as
// "not yet published", so the words never need clearing between launches.
constexpr uint32_t kFlagInvalid = 0u;
constexpr uint32_t kFlagAggregate = 1u;
constexpr uint32_t kFlagPrefix = 2u;
constexpr uint32_t kFlagError = 3u;
constexpr uint32_t kValueMask = (1u << 30) - 1u;

// Upper limits of the config (checked on the host).
constexpr int kMaxR = 128;
constexpr int kMaxE = 256;
constexpr int kMaxK = 32;
constexpr int kMaxS = 8;
constexpr int kMaxG = 256;
constexpr int kMaxD = 16384;

struct Sizes {
    int R, T, E, K, S, d;
    int M, G, P;
    int64_t N, Q;
};

// The config limits every entry point checks on the host (ue.h, ue_config).
inline bool config_ok(const ue_config& c)
{
    if (c.R < 1 || c.R > kMaxR) return false;
    if (c.E < 1 || c.E > kMaxE || c.E % c.R != 0) return false;
    if (c.K < 1 || c.K > kMaxK || c.K > c.E) return false;
    if (c.S < 0 || c.S > kMaxS || c.R * c.S > kMaxG) return false;
    if (c.T < 1) return false;
    if (c.d < 8 || c.d % 8 != 0 || c.d > kMaxD) return false;
    const int64_t Q = (int64_t)c.R * c.T * c.K;
    if (Q >= (int64_t(1) << 30)) return false;
    return true;
}

inline Sizes make_sizes(const ue_config& c)
{
    Sizes s;
    s.R = c.R; s.T = c.T; s.E = c.E; s.K = c.K; s.S = c.S; s.d = c.d;
    s.M = c.E / c.R;
    s.G = c.R * c.S;
    s.P = c.R * (s.M + c.S);
    s.N = (int64_t)c.R * c.T;
    s.Q = s.N * c.K;
    return s;
}

// Launch helpers, one per kernel family. Each returns the CUDA error of the
// launch (cudaSuccess if nothing was launched because there was no work).
// Gate launch shape, fixed once per context: `fast` (K = 8, E a multiple of
// 32 from 64 to 256) uses contiguous blocks of rows_per_cta rows per CTA;
// `fused` means the exact histogram can be taken inside that kernel.
struct GateShape {
    int grid;
    int64_t rows_per_cta;
    int fast, fused;
};
// The fused histogram's outputs and scratch: sync[0..3] = {ticket, finished
// CTAs, launch epoch, zeroed-outputs flag}, zeroed once; each launch leaves
// them ready for the next one.
struct GateCount {
    int32_t* load_re;
    int32_t* load_e;
    uint32_t* sync;
    int* err;
    int T, R;
};
GateShape plan_gate_shape(const Sizes& z, int num_sms);
// cnt == nullptr: top-k and weights only; otherwise also the exact histogram
// (inside the gate kernel when the shape allows, else by launch_count)
cudaError_t launch_gate_topk(const Sizes& z, const GateShape& sh, const float* logits,
                             int32_t* idx, float* w, const GateCount* cnt, cudaStream_t st);
// sync: the same four words as GateCount's (ticket, finished CTAs, epoch,
// flag), left ready for the next launch of either kernel
cudaError_t launch_count(const Sizes& z, const int32_t* idx, int32_t* load_re,
                         int32_t* load_e, uint32_t* sync, int* err, cudaStream_t st);
// greedy plan; min_tokens = 0: every expert may take a copy
cudaError_t launch_plan(const Sizes& z, const int32_t* load_e, int min_tokens,
                        const ue_placement& out, int* err, cudaStream_t st);
// capacity planner (bisection); plan_bisect_setup sets the kernel's shared
// memory limit once per context, outside any stream capture
cudaError_t plan_bisect_setup(const Sizes& z);
cudaError_t launch_plan_bisect(const Sizes& z, const int32_t* load_e, int eps_inv, int threshold,
                               int min_tokens, int allow_zero, const ue_placement& out, int* err,
                               cudaStream_t st);
// Reroute scratch, zeroed once; each launch leaves it ready for the next one
// (the last CTA resets the ticket and the counter and advances the epoch;
// each group's last arrival resets its counter).
struct RerouteScratch {
    unsigned long long* status;   // [tiles][E] tile counts, tagged with the launch epoch
    unsigned long long* gstatus;  // [groups][E] group sums, tagged likewise
    uint32_t* gcount;             // [groups] tiles of the group that have published
    uint32_t* sync;               // [4] tile ticket, finished CTAs, launch epoch
};
inline int64_t reroute_tiles(const Sizes& z, int tile) { return (z.Q + tile - 1) / tile; }
inline int64_t reroute_groups(const Sizes& z, int tile)
{
    return (reroute_tiles(z, tile) + kRerouteGroup - 1) / kRerouteGroup;
}
// the reroute kernels' dynamic shared memory limits, set once per device
// (outside any stream capture) before the first launch
cudaError_t reroute_setup();
// pairs per tile for this GPU: the smallest size on offer whose tiles fit at
// once (call after reroute_setup)
int reroute_tile(const Sizes& z, int num_sms);
cudaError_t launch_reroute(const Sizes& z, int tile, const int32_t* idx,
                           const ue_placement& plan, int32_t* phys_slot, int32_t* dest_row,
                           const RerouteScratch& sc, int64_t spin_limit, int drop_first, int* err,
                           cudaStream_t st);
// order: 0 global (r, t, k), 1 interleaved (t, r, k). after_plan: launched
// as a programmatic dependent of the plan kernel just before it in the
// stream, so that the tiles count and look back while the plan runs and read
// the plan only once it has completed (the kernel before the plan must have
// completed ordinarily: the ids are read early).
cudaError_t launch_reroute_order(const Sizes& z, int tile, const int32_t* idx,
                                 const ue_placement& plan, int order, int32_t* phys_slot,
                                 int32_t* dest_row, const RerouteScratch& sc, int64_t spin_limit,
                                 int drop_first, int* err, cudaStream_t st,
                                 bool after_plan = false);
// locality order: builds the [R][P] tables `first` and `rowb`, then reroutes
cudaError_t launch_reroute_local(const Sizes& z, int tile, const int32_t* idx,
                                 const int32_t* load_re, const ue_placement& plan,
                                 const int32_t* src_quota, const int32_t* src_offset,
                                 int32_t* first, int32_t* rowb, int32_t* phys_slot,
                                 int32_t* dest_row, const RerouteScratch& sc, int64_t spin_limit,
                                 int drop_first, int* err, cudaStream_t st);
cudaError_t launch_locality_split(const Sizes& z, const int32_t* load_re,
                                  const ue_placement& plan, int32_t* src_quota,
                                  int32_t* src_offset, int* err, cudaStream_t st);
// Launch shapes of the row kernels, fixed once per context (ue_init) so that
// a call only enqueues work (nothing else touches the runtime, which keeps
// the calls safe under stream capture).
struct PermuteShape {
    int grid, threads, cw;  // cw: threads per token (one 16-byte chunk each)
};
struct CombineShape {
    int grid, tpt;
    int token;  // 1: one token per CTA, one chunk per thread (K = 4 or 8, 1024 <= d <= 8192)
};
cudaError_t plan_permute_shape(const Sizes& z, int num_sms, PermuteShape* out);
cudaError_t plan_combine_shape(const Sizes& z, int num_sms, CombineShape* out);

cudaError_t launch_permute(const Sizes& z, const PermuteShape& sh, const uint16_t* hidden,
                           const int32_t* dest_row, uint16_t* dispatch, int* err,
                           cudaStream_t st);
// zrow: d zero bf16 values (16-byte aligned), read in place of a row out of range
cudaError_t launch_combine(const Sizes& z, const CombineShape& sh, const uint16_t* y,
                           const int32_t* dest_row, const float* w, float* out,
                           const uint16_t* zrow, int* err, cudaStream_t st);


// Beside the forward path: backward of the combine (the permute's backward
// is launch_combine with w == nullptr), weight sync and gradient reduction.
struct BwdShape {
    int grid, threads, cw;  // cw: threads per token (whole warps)
    int single;             // 1: one chunk per thread (K = 4 or 8, d <= 8192)
};
cudaError_t plan_combine_backward_shape(const Sizes& z, BwdShape* out);
cudaError_t launch_combine_backward(const Sizes& z, const BwdShape& sh, const float* dout,
                                    const uint16_t* y, const int32_t* dest_row, const float* w,
                                    uint16_t* dy, float* dw, int* err, cudaStream_t st);
cudaError_t launch_weight_sync(const Sizes& z, const int32_t* slot_expert, const void* master,
                               void* replicas, int64_t bytes_per_expert, int num_sms, int* err,
                               cudaStream_t st);
// tables: context scratch of kGrTableWords int32 (the reduction's list of
// replicated experts and their replica slots, rebuilt by every call)
constexpr int kGrTableWords = 3 * kMaxE + kMaxG + 1;
cudaError_t launch_grad_reduce(const Sizes& z, const int32_t* slot_expert, const float* replicas,
                               float* master, int64_t numel_per_expert, int32_t* tables, int* err,
                               cudaStream_t st);

}  // namespace ue
