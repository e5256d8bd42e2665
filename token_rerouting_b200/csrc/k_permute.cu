// k_permute.cu -- token dispatch into per-slot contiguous buffers.
//
// "UltraEP" README, "Interface / 2. Forward and backward":
// dispatch(hidden, probs, routing_map) after reroute. On one GPU the
// dispatch is a row scatter: dispatch[dest_row[n*K + k]] = hidden[n], bit
// for bit, so that each physical slot's rows are contiguous and in global
// pair order.
//
// Design (B200): the copy is pure HBM traffic (2*d bytes read and 2*K*d
// bytes written per token), so the data never passes through registers.
// Each warp owns a ring of shared-memory row buffers. Lane 0 brings a token's
// row in with one bulk TMA load (cp.async.bulk global->shared, completion on
// an mbarrier); then lanes 0..K-1 each issue one bulk TMA store of that
// buffer to their destination row (cp.async.bulk shared->global). A buffer is
// refilled once the stores issued from it one iteration earlier have finished
// reading it, so loads for the next tokens overlap the stores of the current
// one. Every row moves as a single 16-byte-aligned bulk copy of 2*d bytes.
// No cluster multicast is used. Every mbarrier wait is bounded; when one
// runs out the kernel records UE_ERR_TIMEOUT, waits (bounded) for its own
// loads in flight, drains its stores and returns.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kPermMaxWarps = 4;
constexpr int kBarBytes = 1024;  // mbarrier area at the start of shared memory
constexpr unsigned long long kWaitNs = 2000000000ull;  // 2 s bound on any wait

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity)
{
    uint32_t ok;
    asm volatile(
        "{\n"
        ".reg .pred p;\n"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// wait for phase `parity` of `bar` to complete, for at most kWaitNs
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > kWaitNs) return false;
    }
}

__device__ __forceinline__ void bulk_load(void* dst_smem, const void* src, unsigned bytes,
                                          uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_addr(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void bulk_store(void* dst, const void* src_smem, unsigned bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(smem_addr(src_smem)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit()
{
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_read_1()
{
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_all()
{
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__global__ void __launch_bounds__(kPermMaxWarps * 32)
permute_kernel(const uint16_t* __restrict__ hidden, const int32_t* __restrict__ dest_row,
               uint16_t* __restrict__ dispatch, int64_t N, int K, int d, int nst,
               int64_t Q, int* err)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int wpb = blockDim.x >> 5;
    const unsigned row_bytes = (unsigned)d * 2u;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem) + warp * nst;
    unsigned char* bufs = smem + kBarBytes + (size_t)warp * nst * row_bytes;

    const int64_t gw = (int64_t)blockIdx.x * wpb + warp;
    const int64_t GW = (int64_t)gridDim.x * wpb;
    if (gw >= N) return;  // warps share nothing, so a warp may leave early
    const int64_t ntok = (N - 1 - gw) / GW + 1;

    if (lane == 0) {
        for (int s = 0; s < nst; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();

    int64_t issued = 0;  // loads issued (token ordinal of the next load)
    if (lane == 0) {
        for (int s = 0; s < nst && s < ntok; ++s) {
            mbar_expect_tx(&bars[s], row_bytes);
            bulk_load(bufs + (size_t)s * row_bytes, hidden + (gw + s * GW) * (int64_t)d,
                      row_bytes, &bars[s]);
        }
    }
    issued = min((int64_t)nst, ntok);

    int64_t t = 0;
    bool ok = true;
    for (; t < ntok; ++t) {
        const int s = (int)(t % nst);
        const unsigned parity = (unsigned)((t / nst) & 1);
        const int64_t n = gw + t * GW;
        int dr = -1;
        if (lane < K) {
            dr = __ldg(dest_row + n * K + lane);
            if (dr < 0 || (int64_t)dr >= Q) {
                raise_error(err, UE_ERR_DEVICE_BOUNDS, (int)min(n * K + lane, (int64_t)INT_MAX));
                dr = -1;
            }
        }
        // every lane waits (so each sees the loaded row); the outcome is
        // made warp-uniform so that all lanes leave together on a timeout
        if (!__all_sync(kFull, mbar_wait(&bars[s], parity))) {
            ok = false;
            break;
        }
        if (dr >= 0)
            bulk_store(dispatch + (int64_t)dr * d, bufs + (size_t)s * row_bytes, row_bytes);
        bulk_commit();
        // refill the buffer whose stores were committed one iteration ago
        if (t >= 1 && issued < ntok) {
            bulk_wait_read_1();
            __syncwarp();
            if (lane == 0) {
                const int sp = (int)((t - 1) % nst);
                mbar_expect_tx(&bars[sp], row_bytes);
                bulk_load(bufs + (size_t)sp * row_bytes, hidden + (gw + issued * GW) * (int64_t)d,
                          row_bytes, &bars[sp]);
            }
            issued += 1;
        }
    }
    if (!ok) {
        raise_error(err, UE_ERR_TIMEOUT, (int)min(gw, (int64_t)INT_MAX));
        // loads t .. issued-1 are still owed to their buffers
        for (int64_t u = t; u < issued; ++u)
            mbar_wait(&bars[u % nst], (unsigned)((u / nst) & 1));
    }
    bulk_wait_all();
}

}  // namespace

cudaError_t plan_permute_shape(const Sizes& z, int num_sms, PermuteShape* out)
{
    const size_t row_bytes = (size_t)z.d * 2;
    // ring of 2..4 row buffers per warp; 4 warps per CTA unless rows are so
    // wide that two buffers for each would not fit in shared memory
    const size_t budget = 200 * 1024;
    const int warps = (int)std::max<size_t>(1, std::min<size_t>(kPermMaxWarps, budget / (2 * row_bytes)));
    int nst = (int)std::min<size_t>(4, (100 * 1024) / (warps * row_bytes));
    nst = std::max(nst, 2);
    const size_t smem = kBarBytes + (size_t)warps * nst * row_bytes;
    cudaError_t ce = cudaFuncSetAttribute(permute_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (ce != cudaSuccess) return ce;
    int per_sm = 0;
    ce = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, permute_kernel, warps * 32, smem);
    if (ce != cudaSuccess) return ce;
    per_sm = std::max(per_sm, 1);
    const int64_t need = std::max<int64_t>(1, (z.N + warps - 1) / warps);
    out->grid = (int)std::min<int64_t>(need, (int64_t)num_sms * per_sm);
    out->warps = warps;
    out->nst = nst;
    out->smem = smem;
    return cudaSuccess;
}

cudaError_t launch_permute(const Sizes& z, const PermuteShape& sh, const uint16_t* hidden,
                           const int32_t* dest_row, uint16_t* dispatch, int* err,
                           cudaStream_t st)
{
    if (z.N == 0) return cudaSuccess;
    permute_kernel<<<sh.grid, sh.warps * 32, sh.smem, st>>>(hidden, dest_row, dispatch, z.N, z.K,
                                                            z.d, sh.nst, z.Q, err);
    return cudaGetLastError();
}

}  // namespace ue
