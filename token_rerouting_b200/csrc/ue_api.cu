// ue_api.cu -- the C ABI declared in include/ue.h: context, host-side
// argument checks, and kernel launches. See ue.h for the contract of every
// call.
#include <cstdio>
#include <cstdlib>
#include <new>

#include "ue_internal.cuh"

struct ue_ctx {
    ue_config cfg;
    ue::Sizes z;
    int device;
    int num_sms;
    ue::GateShape gate;
    ue::PermuteShape perm;
    ue::CombineShape comb;
    ue::BwdShape bwd;       // combine backward launch shape
    int* d_err;             // [2] error code, detail
    unsigned long long* d_status;  // [tiles][E] reroute tile counts
    unsigned long long* d_gstatus; // [groups][E] reroute group sums
    uint32_t* d_gcount;     // [groups] reroute group arrivals
    uint32_t* d_sync;       // [4] reroute ticket, finished CTAs, epoch
    uint32_t* d_gsync;      // [4] fused gate count: ticket, finished CTAs, epoch, flag
    int32_t* d_first;       // [R][P] locality order: first occurrence index
    int32_t* d_rowb;        // [R][P] locality order: row base
    uint16_t* d_zrow;       // [d] zeros: the combine reads it for a row out of range
    int32_t* d_grtab;       // [kGrTableWords] gradient reduction: replicated experts, their slots
    int rtile;              // reroute pairs per tile
    int64_t tiles, groups;
    int64_t spin_limit;
    int drop_first;
    uint32_t magic;
};

namespace {

constexpr uint32_t kMagic = 0x75656331u;  // "uec1"

bool ctx_ok(const ue_ctx* ctx) { return ctx != nullptr && ctx->magic == kMagic; }

bool aligned(const void* p, size_t a) { return p != nullptr && ((uintptr_t)p % a) == 0; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// make the context's device current (cheap when it already is)
ue_status use_device(const ue_ctx* ctx)
{
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return UE_ERR_CUDA;
    if (cur != ctx->device && cudaSetDevice(ctx->device) != cudaSuccess) return UE_ERR_CUDA;
    return UE_OK;
}

ue_status from_cuda(cudaError_t e) { return e == cudaSuccess ? UE_OK : UE_ERR_CUDA; }

ue::RerouteScratch rscratch(const ue_ctx* ctx)
{
    return ue::RerouteScratch{ctx->d_status, ctx->d_gstatus, ctx->d_gcount, ctx->d_sync};
}

bool placement_ok(const ue_ctx* ctx, const ue_placement* p)
{
    if (p == nullptr) return false;
    if (ctx->z.G > 0 && !aligned(p->slot_expert, 4)) return false;
    return aligned(p->n_copies, 4) && aligned(p->slot_quota, 4) && aligned(p->slot_offset, 4) &&
           aligned(p->rank_load, 4) && aligned(p->stats, 4);
}

// free every device buffer of a context (null ones are skipped)
void free_buffers(ue_ctx* ctx)
{
    cudaFree(ctx->d_err);
    cudaFree(ctx->d_status);
    cudaFree(ctx->d_gstatus);
    cudaFree(ctx->d_gcount);
    cudaFree(ctx->d_sync);
    cudaFree(ctx->d_gsync);
    cudaFree(ctx->d_first);
    cudaFree(ctx->d_rowb);
    cudaFree(ctx->d_zrow);
    cudaFree(ctx->d_grtab);
}

}  // namespace

extern "C" {

ue_status ue_init(const ue_config* cfg, int device, ue_ctx** out)
{
    if (out == nullptr) return UE_ERR_INVALID_ARG;
    *out = nullptr;
    if (cfg == nullptr || !ue::config_ok(*cfg)) return UE_ERR_INVALID_ARG;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess) return UE_ERR_CUDA;
    if (device < 0 || device >= ndev) return UE_ERR_INVALID_ARG;
    if (cudaSetDevice(device) != cudaSuccess) return UE_ERR_CUDA;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return UE_ERR_CUDA;
    if (prop.major != 10) return UE_ERR_UNSUPPORTED;

    ue_ctx* ctx = new (std::nothrow) ue_ctx();
    if (ctx == nullptr) return UE_ERR_NOMEM;
    ctx->cfg = *cfg;
    ctx->z = ue::make_sizes(*cfg);
    ctx->device = device;
    ctx->num_sms = prop.multiProcessorCount;
    ctx->gate = ue::plan_gate_shape(ctx->z, ctx->num_sms);
    if (ue::reroute_setup() != cudaSuccess) {
        delete ctx;
        cudaGetLastError();
        return UE_ERR_CUDA;
    }
    ctx->rtile = ue::reroute_tile(ctx->z, ctx->num_sms);
    ctx->tiles = ue::reroute_tiles(ctx->z, ctx->rtile);
    ctx->groups = ue::reroute_groups(ctx->z, ctx->rtile);
    ctx->spin_limit = 1LL << 22;
    ctx->drop_first = 0;

    if (ue::plan_permute_shape(ctx->z, ctx->num_sms, &ctx->perm) != cudaSuccess ||
        ue::plan_combine_shape(ctx->z, ctx->num_sms, &ctx->comb) != cudaSuccess ||
        ue::plan_combine_backward_shape(ctx->z, &ctx->bwd) != cudaSuccess ||
        ue::plan_bisect_setup(ctx->z) != cudaSuccess) {
        delete ctx;
        cudaGetLastError();
        return UE_ERR_CUDA;
    }

    const size_t status_words = (size_t)std::max<int64_t>(ctx->tiles, 1) * ctx->z.E;
    const size_t group_words = (size_t)std::max<int64_t>(ctx->groups, 1) * ctx->z.E;
    const size_t groups = (size_t)std::max<int64_t>(ctx->groups, 1);
    const size_t table_words = (size_t)ctx->z.R * ctx->z.P;
    if (cudaMalloc(&ctx->d_err, 2 * sizeof(int)) != cudaSuccess ||
        cudaMalloc(&ctx->d_status, status_words * sizeof(unsigned long long)) != cudaSuccess ||
        cudaMalloc(&ctx->d_gstatus, group_words * sizeof(unsigned long long)) != cudaSuccess ||
        cudaMalloc(&ctx->d_gcount, groups * sizeof(uint32_t)) != cudaSuccess ||
        cudaMalloc(&ctx->d_sync, 4 * sizeof(uint32_t)) != cudaSuccess ||
        cudaMalloc(&ctx->d_gsync, 4 * sizeof(uint32_t)) != cudaSuccess ||
        cudaMalloc(&ctx->d_first, table_words * sizeof(int32_t)) != cudaSuccess ||
        cudaMalloc(&ctx->d_rowb, table_words * sizeof(int32_t)) != cudaSuccess ||
        cudaMalloc(&ctx->d_zrow, (size_t)ctx->z.d * sizeof(uint16_t)) != cudaSuccess ||
        cudaMalloc(&ctx->d_grtab, ue::kGrTableWords * sizeof(int32_t)) != cudaSuccess) {
        free_buffers(ctx);
        delete ctx;
        cudaGetLastError();
        return UE_ERR_NOMEM;
    }
    if (cudaMemset(ctx->d_err, 0, 2 * sizeof(int)) != cudaSuccess ||
        cudaMemset(ctx->d_status, 0, status_words * sizeof(unsigned long long)) != cudaSuccess ||
        cudaMemset(ctx->d_gstatus, 0, group_words * sizeof(unsigned long long)) != cudaSuccess ||
        cudaMemset(ctx->d_gcount, 0, groups * sizeof(uint32_t)) != cudaSuccess ||
        cudaMemset(ctx->d_sync, 0, 4 * sizeof(uint32_t)) != cudaSuccess ||
        cudaMemset(ctx->d_gsync, 0, 4 * sizeof(uint32_t)) != cudaSuccess ||
        cudaMemset(ctx->d_zrow, 0, (size_t)ctx->z.d * sizeof(uint16_t)) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess) {
        free_buffers(ctx);
        delete ctx;
        return UE_ERR_CUDA;
    }
    ctx->magic = kMagic;
    *out = ctx;
    return UE_OK;
}

ue_status ue_destroy(ue_ctx* ctx)
{
    if (ctx == nullptr) return UE_OK;
    if (!ctx_ok(ctx)) return UE_ERR_INVALID_ARG;
    ue_status st = use_device(ctx);
    if (st == UE_OK && cudaDeviceSynchronize() != cudaSuccess) st = UE_ERR_CUDA;
    free_buffers(ctx);
    ctx->magic = 0;
    delete ctx;
    return st;
}

ue_status ue_get_error(ue_ctx* ctx, void* stream)
{
    if (!ctx_ok(ctx)) return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    int h[2] = {0, 0};
    if (cudaStreamSynchronize(st) != cudaSuccess) return UE_ERR_CUDA;
    if (cudaMemcpyAsync(h, ctx->d_err, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return UE_ERR_CUDA;
    if (cudaMemsetAsync(ctx->d_err, 0, sizeof(h), st) != cudaSuccess) return UE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return UE_ERR_CUDA;
    return (ue_status)h[0];
}

ue_status ue_gate_topk(ue_ctx* ctx, const float* logits, int32_t* idx, float* w, void* stream)
{
    if (!ctx_ok(ctx) || !aligned(logits, 4) || !aligned(idx, 4) || !aligned(w, 4))
        return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    return from_cuda(ue::launch_gate_topk(ctx->z, ctx->gate, logits, idx, w, nullptr,
                                          as_stream(stream)));
}

ue_status ue_gate_count(ue_ctx* ctx, const float* logits, int32_t* idx, float* w,
                        int32_t* load_re, int32_t* load_e, void* stream)
{
    if (!ctx_ok(ctx) || !aligned(logits, 4) || !aligned(idx, 4) || !aligned(w, 4) ||
        !aligned(load_re, 4) || !aligned(load_e, 4))
        return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    const ue::GateCount cnt{load_re, load_e, ctx->d_gsync, ctx->d_err, ctx->cfg.T, ctx->cfg.R};
    return from_cuda(ue::launch_gate_topk(ctx->z, ctx->gate, logits, idx, w, &cnt,
                                          as_stream(stream)));
}

ue_status ue_count(ue_ctx* ctx, const int32_t* idx, int32_t* load_re, int32_t* load_e,
                   void* stream)
{
    if (!ctx_ok(ctx) || !aligned(idx, 4) || !aligned(load_re, 4) || !aligned(load_e, 4))
        return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    return from_cuda(ue::launch_count(ctx->z, idx, load_re, load_e, ctx->d_gsync, ctx->d_err,
                                      as_stream(stream)));
}

ue_status ue_plan(ue_ctx* ctx, const int32_t* load_e, const ue_placement* out, void* stream)
{
    if (!ctx_ok(ctx) || !aligned(load_e, 4) || !placement_ok(ctx, out))
        return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    return from_cuda(ue::launch_plan(ctx->z, load_e, 0, *out, ctx->d_err, as_stream(stream)));
}

ue_status ue_plan_ex(ue_ctx* ctx, const int32_t* load_e, const ue_plan_opts* opts,
                     const ue_placement* out, void* stream)
{
    if (!ctx_ok(ctx) || opts == nullptr || !aligned(load_e, 4) || !placement_ok(ctx, out))
        return UE_ERR_INVALID_ARG;
    const ue_plan_opts o = *opts;
    if (o.solver == UE_SOLVER_GREEDY) {
        if (o.min_tokens < 0) return UE_ERR_INVALID_ARG;
        if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
        return from_cuda(ue::launch_plan(ctx->z, load_e, o.min_tokens, *out, ctx->d_err,
                                         as_stream(stream)));
    }
    if (o.solver != UE_SOLVER_BISECT || o.min_tokens < 1 || o.eps_inv < 1 || o.eps_inv > 10000 ||
        o.threshold < 0 || (o.allow_zero_master != 0 && o.allow_zero_master != 1))
        return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    return from_cuda(ue::launch_plan_bisect(ctx->z, load_e, o.eps_inv, o.threshold, o.min_tokens,
                                            o.allow_zero_master, *out, ctx->d_err,
                                            as_stream(stream)));
}

ue_status ue_reroute(ue_ctx* ctx, const int32_t* idx, const ue_placement* plan,
                     int32_t* phys_slot, int32_t* dest_row, void* stream)
{
    if (!ctx_ok(ctx) || !aligned(idx, 4) || !placement_ok(ctx, plan) ||
        !aligned(phys_slot, 4) || !aligned(dest_row, 4))
        return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    return from_cuda(ue::launch_reroute(ctx->z, ctx->rtile, idx, *plan, phys_slot, dest_row,
                                        rscratch(ctx), ctx->spin_limit, ctx->drop_first,
                                        ctx->d_err, as_stream(stream)));
}

ue_status ue_plan_reroute(ue_ctx* ctx, const int32_t* load_e, const int32_t* idx,
                          const ue_placement* plan, int32_t* phys_slot, int32_t* dest_row,
                          void* stream)
{
    if (!ctx_ok(ctx) || !aligned(load_e, 4) || !aligned(idx, 4) || !placement_ok(ctx, plan) ||
        !aligned(phys_slot, 4) || !aligned(dest_row, 4))
        return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    const cudaStream_t st = as_stream(stream);
    const cudaError_t ce = ue::launch_plan(ctx->z, load_e, 0, *plan, ctx->d_err, st);
    if (ce != cudaSuccess) return from_cuda(ce);
    return from_cuda(ue::launch_reroute_order(ctx->z, ctx->rtile, idx, *plan, UE_ORDER_PREFIX,
                                              phys_slot, dest_row, rscratch(ctx),
                                              ctx->spin_limit, ctx->drop_first, ctx->d_err, st,
                                              true));
}

ue_status ue_reroute_ex(ue_ctx* ctx, const int32_t* idx, const ue_placement* plan, int32_t order,
                        int32_t* phys_slot, int32_t* dest_row, void* stream)
{
    if (!ctx_ok(ctx) || !aligned(idx, 4) || !placement_ok(ctx, plan) ||
        !aligned(phys_slot, 4) || !aligned(dest_row, 4) ||
        (order != UE_ORDER_PREFIX && order != UE_ORDER_INTERLEAVE))
        return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    return from_cuda(ue::launch_reroute_order(ctx->z, ctx->rtile, idx, *plan, order, phys_slot,
                                              dest_row, rscratch(ctx), ctx->spin_limit,
                                              ctx->drop_first, ctx->d_err, as_stream(stream)));
}

ue_status ue_locality_split(ue_ctx* ctx, const int32_t* load_re, const ue_placement* plan,
                            int32_t* src_quota, int32_t* src_offset, void* stream)
{
    if (!ctx_ok(ctx) || !aligned(load_re, 4) || !placement_ok(ctx, plan) ||
        !aligned(src_quota, 4) || !aligned(src_offset, 4))
        return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    return from_cuda(ue::launch_locality_split(ctx->z, load_re, *plan, src_quota, src_offset,
                                               ctx->d_err, as_stream(stream)));
}

ue_status ue_reroute_local(ue_ctx* ctx, const int32_t* idx, const int32_t* load_re,
                           const ue_placement* plan, const int32_t* src_quota,
                           const int32_t* src_offset, int32_t* phys_slot, int32_t* dest_row,
                           void* stream)
{
    if (!ctx_ok(ctx) || !aligned(idx, 4) || !aligned(load_re, 4) || !placement_ok(ctx, plan) ||
        !aligned(src_quota, 4) || !aligned(src_offset, 4) || !aligned(phys_slot, 4) ||
        !aligned(dest_row, 4))
        return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    return from_cuda(ue::launch_reroute_local(ctx->z, ctx->rtile, idx, load_re, *plan, src_quota,
                                              src_offset, ctx->d_first, ctx->d_rowb, phys_slot,
                                              dest_row, rscratch(ctx), ctx->spin_limit,
                                              ctx->drop_first, ctx->d_err, as_stream(stream)));
}

ue_status ue_permute(ue_ctx* ctx, const uint16_t* hidden, const int32_t* dest_row,
                     uint16_t* dispatch, void* stream)
{
    if (!ctx_ok(ctx) || !aligned(hidden, 16) || !aligned(dest_row, 4) || !aligned(dispatch, 16))
        return UE_ERR_INVALID_ARG;
    const size_t hb = (size_t)ctx->z.N * ctx->z.d * 2, db = (size_t)ctx->z.Q * ctx->z.d * 2;
    const uintptr_t h0 = (uintptr_t)hidden, d0 = (uintptr_t)dispatch;
    if (h0 < d0 + db && d0 < h0 + hb) return UE_ERR_INVALID_ARG;  // overlap
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    return from_cuda(ue::launch_permute(ctx->z, ctx->perm, hidden, dest_row, dispatch,
                                        ctx->d_err, as_stream(stream)));
}

ue_status ue_combine(ue_ctx* ctx, const uint16_t* y, const int32_t* dest_row, const float* w,
                     float* out, void* stream)
{
    if (!ctx_ok(ctx) || !aligned(y, 16) || !aligned(dest_row, 4) || !aligned(w, 4) ||
        !aligned(out, 16))
        return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    return from_cuda(ue::launch_combine(ctx->z, ctx->comb, y, dest_row, w, out, ctx->d_zrow,
                                        ctx->d_err, as_stream(stream)));
}

ue_status ue_combine_backward(ue_ctx* ctx, const float* dout, const uint16_t* y,
                              const int32_t* dest_row, const float* w, uint16_t* dy, float* dw,
                              void* stream)
{
    if (!ctx_ok(ctx) || !aligned(dout, 16) || !aligned(y, 16) || !aligned(dest_row, 4) ||
        !aligned(w, 4) || !aligned(dy, 16) || !aligned(dw, 4))
        return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    return from_cuda(ue::launch_combine_backward(ctx->z, ctx->bwd, dout, y, dest_row, w, dy, dw,
                                                 ctx->d_err, as_stream(stream)));
}

ue_status ue_permute_backward(ue_ctx* ctx, const uint16_t* ddispatch, const int32_t* dest_row,
                              float* dhidden, void* stream)
{
    if (!ctx_ok(ctx) || !aligned(ddispatch, 16) || !aligned(dest_row, 4) ||
        !aligned(dhidden, 16))
        return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    // the combine with every weight equal to 1
    return from_cuda(ue::launch_combine(ctx->z, ctx->comb, ddispatch, dest_row, nullptr, dhidden,
                                        ctx->d_zrow, ctx->d_err, as_stream(stream)));
}

ue_status ue_weight_sync(ue_ctx* ctx, const ue_placement* plan, const void* master,
                         void* replicas, int64_t bytes_per_expert, void* stream)
{
    if (!ctx_ok(ctx) || plan == nullptr || !aligned(master, 16) || bytes_per_expert <= 0 ||
        bytes_per_expert % 16 != 0)
        return UE_ERR_INVALID_ARG;
    if (ctx->z.G > 0 && (!aligned(plan->slot_expert, 4) || !aligned(replicas, 16)))
        return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    return from_cuda(ue::launch_weight_sync(ctx->z, plan->slot_expert, master, replicas,
                                            bytes_per_expert, ctx->num_sms, ctx->d_err,
                                            as_stream(stream)));
}

ue_status ue_grad_reduce(ue_ctx* ctx, const ue_placement* plan, const float* replica_grads,
                         float* master_grads, int64_t numel_per_expert, void* stream)
{
    if (!ctx_ok(ctx) || plan == nullptr || !aligned(master_grads, 16) ||
        numel_per_expert <= 0 || numel_per_expert % 4 != 0)
        return UE_ERR_INVALID_ARG;
    if (ctx->z.G > 0 && (!aligned(plan->slot_expert, 4) || !aligned(replica_grads, 16)))
        return UE_ERR_INVALID_ARG;
    if (use_device(ctx) != UE_OK) return UE_ERR_CUDA;
    return from_cuda(ue::launch_grad_reduce(ctx->z, plan->slot_expert, replica_grads,
                                            master_grads, numel_per_expert, ctx->d_grtab,
                                            ctx->d_err, as_stream(stream)));
}

ue_status ue_debug_set_lookback_limit(ue_ctx* ctx, int64_t polls)
{
    if (!ctx_ok(ctx) || polls < 0) return UE_ERR_INVALID_ARG;
    ctx->spin_limit = polls;
    return UE_OK;
}

ue_status ue_debug_drop_first_publish(ue_ctx* ctx, int enable)
{
    if (!ctx_ok(ctx)) return UE_ERR_INVALID_ARG;
    ctx->drop_first = enable ? 1 : 0;
    return UE_OK;
}

}  // extern "C"
