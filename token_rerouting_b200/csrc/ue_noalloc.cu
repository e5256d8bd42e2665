// ue_noalloc.cu -- ue_reroute_noalloc: the reroute for callers that cannot
// allocate device memory.
//
// ue_init obtains the reroute's look-back scratch with cudaMalloc. Some
// callers cannot do that: code that runs where a device allocation may not
// happen (inside an allocator's own hooks, under a memory pool that forbids
// outside allocations, in a process whose device memory is reserved up front
// by another runtime) or code that has no place to keep a context. This entry
// point needs no context and allocates nothing. Its scratch (the look-back
// status words, the tile ticket, the finished-CTA counter and the launch
// epoch) is a file-scope __device__ array of fixed size, which every GPU that
// loads this library holds until the process exits. The array starts zeroed
// and is never cleared: status words carry their launch's epoch, so words
// left by an earlier call read as unpublished, and the last CTA of every
// call resets the ticket and the counter.
//
// The array's name, used in host code, is only a host-side stand-in for the
// symbol, not a device address. The device address is fetched once per
// device with cudaGetSymbolAddress (on the first call made with that device
// current) and passed to the kernel.
#include <mutex>

#include "ue_internal.cuh"

namespace {

constexpr size_t kStatusWords = size_t(1) << 18;  // 2 MiB of 64-bit look-back words
constexpr size_t kSyncWord = kStatusWords;        // ticket, counter, epoch (as 32-bit)
constexpr size_t kErrWord = kStatusWords + 16;    // error word when none is given
constexpr size_t kScratchWords = kStatusWords + 32;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned long long g_reroute_scratch[kScratchWords];

std::mutex g_mutex;
unsigned long long* g_scratch_addr[kMaxDevices] = {};

// device address of g_reroute_scratch on the current device, looked up once
ue_status scratch_address(unsigned long long** out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return UE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return UE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        const cudaError_t ce = cudaGetSymbolAddress(&p, g_reroute_scratch);
        if (ce != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return UE_ERR_CUDA;
        }
        g_scratch_addr[dev] = static_cast<unsigned long long*>(p);
    }
    *out = g_scratch_addr[dev];
    return UE_OK;
}

bool aligned4(const void* p) { return p != nullptr && ((uintptr_t)p % 4) == 0; }

}  // namespace

extern "C" ue_status ue_reroute_noalloc(const ue_config* cfg, const int32_t* idx,
                                        const ue_placement* plan, int32_t* phys_slot,
                                        int32_t* dest_row, int32_t* error, void* stream)
{
    if (cfg == nullptr || plan == nullptr) return UE_ERR_INVALID_ARG;
    const ue_config& c = *cfg;
    if (c.R < 1 || c.R > ue::kMaxR || c.E < 1 || c.E > ue::kMaxE || c.E % c.R != 0 ||
        c.K < 1 || c.K > ue::kMaxK || c.K > c.E || c.S < 0 || c.S > ue::kMaxS ||
        c.R * c.S > ue::kMaxG || c.T < 1 || c.d < 8 || c.d % 8 != 0 || c.d > ue::kMaxD ||
        (int64_t)c.R * c.T * c.K >= (int64_t(1) << 30))
        return UE_ERR_INVALID_ARG;
    const ue::Sizes z = ue::make_sizes(c);
    if ((z.G > 0 && !aligned4(plan->slot_expert)) || !aligned4(plan->n_copies) ||
        !aligned4(plan->slot_quota) || !aligned4(plan->slot_offset) ||
        !aligned4(plan->rank_load) || !aligned4(plan->stats) || !aligned4(idx) ||
        !aligned4(phys_slot) || !aligned4(dest_row) ||
        (error != nullptr && !aligned4(error)))
        return UE_ERR_INVALID_ARG;
    const int64_t tiles = (z.Q + ue::kRerouteTile - 1) / ue::kRerouteTile;
    if ((size_t)tiles * (size_t)z.E > kStatusWords) return UE_ERR_UNSUPPORTED;

    unsigned long long* base = nullptr;
    const ue_status st = scratch_address(&base);
    if (st != UE_OK) return st;
    int* err = error != nullptr ? reinterpret_cast<int*>(error)
                                : reinterpret_cast<int*>(base + kErrWord);
    uint32_t* sync = reinterpret_cast<uint32_t*>(base + kSyncWord);
    const cudaError_t ce = ue::launch_reroute(z, idx, *plan, phys_slot, dest_row, base, sync,
                                              int64_t(1) << 22, 0, err,
                                              reinterpret_cast<cudaStream_t>(stream));
    return ce == cudaSuccess ? UE_OK : UE_ERR_CUDA;
}
