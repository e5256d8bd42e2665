// ue_noalloc.cu -- ue_reroute_noalloc: the reroute for callers that cannot
// allocate device memory.
//
// ue_init obtains the reroute's look-back scratch with cudaMalloc. Some
// callers cannot do that: code that runs where a device allocation may not
// happen (inside an allocator's own hooks, under a memory pool that forbids
// outside allocations, in a process whose device memory is reserved up front
// by another runtime) or code that has no place to keep a context. This entry
// point needs no context and allocates nothing. Its scratch (the look-back
// status words of the tiles and of the groups of tiles, the groups' arrival
// counters, the tile ticket, the finished-CTA counter and the launch epoch)
// is a file-scope __device__ array of fixed size, which every GPU that loads
// this library holds until the process exits. The array starts zeroed and
// is never cleared: status words carry their launch's epoch, so words left
// by an earlier call read as unpublished, each group's last arrival resets
// its counter, and the last CTA of every call resets the ticket and the
// counter.
//
// The array's name, used in host code, is only a host-side stand-in for the
// symbol, not a device address. The device address is fetched once per
// device with cudaGetSymbolAddress (on the first call made with that device
// current, which also checks that the device is an sm_100 part) and passed
// to the kernel. cudaDeviceReset unloads the module and makes the cached
// address stale, so this entry point must not be used after a reset in the
// same process.
#include <mutex>

#include "ue_internal.cuh"

namespace {

// Layout (64-bit words): tile counts [kStatusWords], group sums
// [kGroupWords], group arrival counters [kGroupCounters as 32-bit], then the
// ticket, counter and epoch (as 32-bit).
constexpr size_t kStatusWords = size_t(1) << 18;  // 2 MiB: tiles * E <= 2^18
constexpr size_t kGroupWords = (kStatusWords / ue::kRerouteGroup) + ue::kMaxE;  // groups * E
constexpr size_t kGroupCounters = (kStatusWords / ue::kRerouteGroup) + 64;      // groups
constexpr size_t kGroupWord = kStatusWords;
constexpr size_t kCountWord = kGroupWord + kGroupWords;
constexpr size_t kSyncWord = kCountWord + kGroupCounters / 2;
constexpr size_t kScratchWords = kSyncWord + 16;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned long long g_reroute_scratch[kScratchWords];

std::mutex g_mutex;
unsigned long long* g_scratch_addr[kMaxDevices] = {};
ue_status g_device_status[kMaxDevices] = {};  // first lookup's outcome per device

// device address of g_reroute_scratch on the current device, looked up once
ue_status scratch_address(int dev, unsigned long long** out)
{
    if (dev < 0 || dev >= kMaxDevices) return UE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        if (g_device_status[dev] == UE_ERR_UNSUPPORTED) return UE_ERR_UNSUPPORTED;
        int major = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) !=
            cudaSuccess) {
            cudaGetLastError();
            return UE_ERR_CUDA;
        }
        if (major != 10) {
            g_device_status[dev] = UE_ERR_UNSUPPORTED;
            return UE_ERR_UNSUPPORTED;
        }
        void* p = nullptr;
        cudaError_t ce = ue::reroute_setup();
        if (ce == cudaSuccess) ce = cudaGetSymbolAddress(&p, g_reroute_scratch);
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

// true when p is device (or managed) memory that device dev can address as
// its own; host memory and another GPU's memory are refused
bool on_device(const void* p, int dev)
{
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (a.type == cudaMemoryTypeManaged) return true;
    return a.type == cudaMemoryTypeDevice && a.device == dev;
}

}  // namespace

extern "C" ue_status ue_reroute_noalloc(const ue_config* cfg, const int32_t* idx,
                                        const ue_placement* plan, int32_t* phys_slot,
                                        int32_t* dest_row, int32_t* error, void* stream)
{
    if (cfg == nullptr || plan == nullptr || !ue::config_ok(*cfg)) return UE_ERR_INVALID_ARG;
    const ue::Sizes z = ue::make_sizes(*cfg);
    if ((z.G > 0 && !aligned4(plan->slot_expert)) || !aligned4(plan->n_copies) ||
        !aligned4(plan->slot_quota) || !aligned4(plan->slot_offset) ||
        !aligned4(plan->rank_load) || !aligned4(plan->stats) || !aligned4(idx) ||
        !aligned4(phys_slot) || !aligned4(dest_row) || !aligned4(error))
        return UE_ERR_INVALID_ARG;
    const int64_t tiles = ue::reroute_tiles(z, ue::kRerouteTile);
    const int64_t groups = ue::reroute_groups(z, ue::kRerouteTile);
    if ((size_t)tiles * (size_t)z.E > kStatusWords ||
        (size_t)groups * (size_t)z.E > kGroupWords || (size_t)groups > kGroupCounters)
        return UE_ERR_UNSUPPORTED;

    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return UE_ERR_CUDA;
    unsigned long long* base = nullptr;
    const ue_status st = scratch_address(dev, &base);
    if (st != UE_OK) return st;
    // every buffer the kernel touches must live on the current device
    if (!on_device(idx, dev) || !on_device(phys_slot, dev) || !on_device(dest_row, dev) ||
        !on_device(error, dev) || !on_device(plan->slot_offset, dev) ||
        !on_device(plan->slot_quota, dev) || (z.G > 0 && !on_device(plan->slot_expert, dev)))
        return UE_ERR_INVALID_ARG;
    const ue::RerouteScratch sc{base, base + kGroupWord,
                                reinterpret_cast<uint32_t*>(base + kCountWord),
                                reinterpret_cast<uint32_t*>(base + kSyncWord)};
    const cudaError_t ce = ue::launch_reroute(z, ue::kRerouteTile, idx, *plan, phys_slot,
                                              dest_row, sc, int64_t(1) << 22, 0,
                                              reinterpret_cast<int*>(error),
                                              reinterpret_cast<cudaStream_t>(stream));
    return ce == cudaSuccess ? UE_OK : UE_ERR_CUDA;
}
