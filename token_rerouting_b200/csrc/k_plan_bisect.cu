// k_plan_bisect.cu -- capacity planner: bisection on the balancing ratio.
//
// "UltraEP" README, "Performance Tuning / Replication planning": the
// planner runs a binary search on the balancing ratio (max/mean rank load)
// with an early-stop target and a numerical tolerance eps, tests each
// candidate with a quota oracle, gives every replica a minimal load, and by
// default never leaves a master with zero load. The pages name these knobs
// only; the rule implemented here is this library's reading of them:
//
//   The ratio runs on the grid k/D (eps = 1/D); the capacity of grid point k
//   is C(k) = floor(k*Q / (D*R)). H_r is the load of rank r's masters.
//   Quota oracle at C:
//     1. every rank with H_r > C sheds X = H_r - C pairs: it visits its
//        masters by load, largest first (ties to the lower e); master e can
//        give a_e = L_e - keep_e (keep_e = 1, or 0 when zero-load masters
//        are allowed or L_e = 0) and, if a_e >= m, gives
//        s_e = max(min(X_left, a_e), m); C fails if X is not covered;
//     2. every rank offers spare capacity max(0, C - H_r) and S slots;
//     3. experts with s_e > 0, largest first (ties to the lower e), are
//        placed one at a time: while rem pairs are left, the receiver is the
//        rank with a free slot and the most spare capacity (ties to the lower
//        r); the piece is min(rem, spare), cut to rem - m if that would
//        leave 0 < rem - piece < m; a piece below m or no receiver fails C;
//        the replica takes the receiver's lowest free slot.
//     The master keeps L_e - s_e.
//   Search: probe k = thr (the early-stop target) and stop if it passes;
//   else lo = thr, hi = the smallest k with C(k) >= max H (passes with no
//   replica), and while hi - lo > 1 probe mid = lo + (hi - lo)/2, moving hi
//   to mid on success and lo to mid on failure. The plan is the oracle's
//   result at hi.
//
// Design (B200): the search is a chain of dependent probes, each a few
// hundred dependent warp reductions. Rather than run them one after another,
// one CTA of 32 warps evaluates a whole subtree of the bisection at once:
// warp w takes node w+1 of the complete depth-5 tree below the current
// interval (its interval follows from the path bits of the node, whatever
// the outcomes), so one round costs one oracle call and settles five levels;
// a replay of the outcomes along the real path gives exactly the probes, the
// interval and the plan the sequential search would reach. The first round
// also runs the early-stop probe (warp 31). Inside a warp the oracle keeps
// the ranks' spare capacity and free slots in registers (lane l owns ranks
// l, l+32, ...) and the experts' shed pairs in the warp's shared array (lane
// l reads experts l, l+32, ...); the demand with the largest shed and the
// receiver with the most spare are each two `redux` reductions. Each warp writes its placement into its own
// shared-memory slots; the placement of the warp whose probe became hi is
// kept. The per-rank order of masters by load does not depend on C and is
// built once.
#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kBsThreads = 1024;
constexpr int kBsWarps = kBsThreads / 32;
constexpr int kTreeDepth = 5;           // levels settled per round
constexpr int kTreeNodes = 31;          // nodes of a complete depth-5 tree
constexpr int kProbeWarp = 31;          // early-stop probe in the first round
constexpr int kMaxRounds = 16;          // 2^21 grid points need 5
constexpr int kSpareCap = 1 << 30;      // spares above any piece compare equal

struct BisectArgs {
    int eps_inv, threshold, min_tokens, allow_zero;
};

// The quota oracle at capacity C, run by one warp. Fills the warp's slot
// arrays and returns whether C is feasible.
template <int NR, int NE>
__device__ bool quota_oracle(long long C, int R, int E, int S, int M, int m, int allow_zero,
                             const int* sL, const int* sOrd, const int* sH, int* wShed,
                             int* wSlotE, int* wSlotQ, int lane)
{
    const int G = R * S;
    for (int g = lane; g < G; g += 32) {
        wSlotE[g] = -1;
        wSlotQ[g] = 0;
    }
    // 1. shedding: the lane of rank r walks r's masters by load
    int spare[NR], nfree[NR];
    bool ok = true;
#pragma unroll
    for (int u = 0; u < NR; ++u) {
        const int r = lane + 32 * u;
        spare[u] = 0;
        nfree[u] = 0;
        if (r < R) {
            const long long H = sH[r];
            spare[u] = H <= C ? (int)min(C - H, (long long)kSpareCap) : 0;
            nfree[u] = S;
            long long X = H - C;
            for (int l = 0; l < M; ++l) {
                const int e = sOrd[r * M + l];
                int s = 0;
                if (X > 0) {
                    const int keep = (allow_zero || sL[e] == 0) ? 0 : 1;
                    const int avail = sL[e] - keep;
                    if (avail >= m) {
                        s = (int)max(min(X, (long long)avail), (long long)m);
                        X -= s;
                    }
                }
                wShed[e] = s;
            }
            if (X > 0) ok = false;
        }
    }
    ok = __all_sync(kFull, ok);
    __syncwarp();
    // 3. placement, largest demand first (the demands stay in the warp's
    // shared shed array; lane l reads experts l, l+32, ...)
    while (ok) {
        int bs = 0, be = 0x7fffffff;
#pragma unroll
        for (int v = 0; v < NE; ++v) {
            const int e = lane + 32 * v;
            const int sv = e < E ? wShed[e] : 0;
            if (sv > bs) {
                bs = sv;
                be = e;
            }
        }
        const unsigned ms = __reduce_max_sync(kFull, (unsigned)bs);
        if (ms == 0u) break;
        const int estar = (int)__reduce_min_sync(kFull, (unsigned)bs == ms ? (unsigned)be : 0xffffffffu);
        if (lane == (estar & 31)) wShed[estar] = 0;
        __syncwarp();
        int rem = (int)ms;
        while (rem > 0) {
            // receiver: the most spare among ranks with a free slot (spare+1,
            // 0 = none), ties to the lower r
            unsigned bsp = 0u, br = 0xffffffffu;
#pragma unroll
            for (int u = 0; u < NR; ++u)
                if (nfree[u] > 0 && (unsigned)spare[u] + 1u > bsp) {
                    bsp = (unsigned)spare[u] + 1u;
                    br = (unsigned)(lane + 32 * u);
                }
            const unsigned mx = __reduce_max_sync(kFull, bsp);
            if (mx == 0u) {
                ok = false;
                break;
            }
            const unsigned rs = __reduce_min_sync(kFull, bsp == mx ? br : 0xffffffffu);
            int piece = min(rem, (int)(mx - 1u));
            if (rem - piece > 0 && rem - piece < m) piece = rem - m;
            if (piece < m) {
                ok = false;
                break;
            }
            if (lane == (int)(rs & 31u)) {
#pragma unroll
                for (int u = 0; u < NR; ++u)
                    if (u == (int)(rs >> 5)) {
                        const int g = (int)rs * S + (S - nfree[u]);
                        wSlotE[g] = estar;
                        wSlotQ[g] = piece;
                        spare[u] -= piece;
                        nfree[u] -= 1;
                    }
            }
            rem -= piece;
        }
    }
    __syncwarp();
    return ok;
}

template <int NR, int NE>
__global__ void __launch_bounds__(kBsThreads, 1)
plan_bisect_kernel(const int32_t* __restrict__ load_e, int R, int E, int S, BisectArgs a,
                   ue_placement out, int* err)
{
    extern __shared__ int dyn[];  // per warp: shed[E], slot expert[G], slot quota[G]
    __shared__ int sL[kMaxE];
    __shared__ int sOrd[kMaxE];          // rank r's masters by load: sOrd[r*M ..]
    __shared__ int sH[kMaxR];
    __shared__ int sBestE[kMaxG], sBestQ[kMaxG];
    __shared__ int sShed[kMaxE], sCopies[kMaxE], sRankLoad[kMaxR];
    __shared__ int sFeas[kBsWarps];
    __shared__ int sWarpSum[kBsWarps];
    __shared__ long long sLo, sHi;
    __shared__ unsigned long long sQ;
    __shared__ int sMaxH, sDone, sProbes, sBestWarp, sMaxAfter;

    const int M = E / R;
    const int G = R * S;
    const int P = R * (M + S);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int m = a.min_tokens;
    const long long DR = (long long)a.eps_inv * R;

    if (tid == 0) {
        sQ = 0ull;
        sMaxH = 0;
        sMaxAfter = 0;
    }
    for (int r = tid; r < R; r += blockDim.x) {
        sH[r] = 0;
        sRankLoad[r] = 0;
    }
    for (int e = tid; e < E; e += blockDim.x) {
        sShed[e] = 0;
        sCopies[e] = 0;
    }
    for (int g = tid; g < G; g += blockDim.x) {
        sBestE[g] = -1;  // the plan at the initial hi: no replica
        sBestQ[g] = 0;
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
        int L = __ldg(load_e + e);
        if (L < 0) {
            raise_error(err, UE_ERR_DEVICE_BOUNDS, e);
            L = 0;
        }
        sL[e] = L;
        atomicAdd(&sH[e / M], L);
        atomicAdd(&sQ, (unsigned long long)L);
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
        // position of e among its rank's masters: load descending, then id
        const int r = e / M;
        const int L = sL[e];
        int pos = 0;
        for (int l = 0; l < M; ++l) {
            const int f = r * M + l;
            const int Lf = sL[f];
            pos += (Lf > L || (Lf == L && f < e)) ? 1 : 0;
        }
        sOrd[r * M + pos] = e;
    }
    for (int r = tid; r < R; r += blockDim.x) atomicMax(&sMaxH, sH[r]);
    __syncthreads();
    const long long Q = (long long)sQ;
    if (tid == 0) {
        const long long maxH = sMaxH;
        long long top = Q > 0 ? (DR * maxH + Q - 1) / Q : 0;
        sLo = a.threshold;
        sHi = max(top, (long long)a.threshold + 1);
        sDone = 0;
        sProbes = 1;  // the early-stop probe
    }
    __syncthreads();

    int* wShed = dyn + warp * (E + 2 * G);
    int* wSlotE = wShed + E;
    int* wSlotQ = wSlotE + G;
    int rounds = 0;
    long long final_k = 0;
    while (true) {
        const long long lo = sLo, hi = sHi;
        // this warp's probe: node warp+1 of the subtree below (lo, hi), or the
        // early-stop probe
        bool probe = false;
        long long k = 0;
        if (warp < kTreeNodes) {
            const int h = warp + 1;
            const int depth = 31 - __clz(h);
            long long x = lo, y = hi;
            for (int i = depth - 1; i >= 0; --i) {
                const long long mid = x + (y - x) / 2;
                if ((h >> i) & 1) x = mid;
                else y = mid;
            }
            probe = y - x > 1;
            k = x + (y - x) / 2;
        } else if (rounds == 0) {
            probe = true;
            k = a.threshold;
        }
        bool feas = false;
        if (probe)
            feas = quota_oracle<NR, NE>(k * Q / DR, R, E, S, M, m, a.allow_zero, sL, sOrd, sH,
                                        wShed, wSlotE, wSlotQ, lane);
        if (lane == 0) sFeas[warp] = feas ? 1 : 0;
        __syncthreads();
        if (tid == 0) {
            int best = -1;
            long long x = lo, y = hi;
            if (rounds == 0 && sFeas[kProbeWarp]) {
                best = kProbeWarp;
                sDone = 1;
                final_k = a.threshold;
            } else {
                // replay the sequential search along the real path
                int h = 1;
                for (int lvl = 0; lvl < kTreeDepth && y - x > 1; ++lvl) {
                    const long long mid = x + (y - x) / 2;
                    sProbes += 1;
                    const bool f = sFeas[h - 1] != 0;
                    if (f) {
                        y = mid;
                        best = h - 1;
                    } else {
                        x = mid;
                    }
                    h = 2 * h + (f ? 0 : 1);
                }
                sLo = x;
                sHi = y;
                if (y - x <= 1) {
                    sDone = 1;
                    final_k = y;
                } else if (rounds + 1 >= kMaxRounds) {
                    raise_error(err, UE_ERR_TIMEOUT, rounds);
                    sDone = 1;
                    final_k = y;
                }
            }
            sBestWarp = best;
            if (sDone) sLo = final_k;  // the chosen grid point
        }
        __syncthreads();
        const int bw = sBestWarp;
        if (bw >= 0) {
            const int* bE = dyn + bw * (E + 2 * G) + E;
            const int* bQ = bE + G;
            for (int g = tid; g < G; g += blockDim.x) {
                sBestE[g] = bE[g];
                sBestQ[g] = bQ[g];
            }
        }
        const int done = sDone;
        __syncthreads();
        if (done) break;
        ++rounds;
    }

    // ---- the plan from the chosen placement ----
    for (int g = tid; g < G; g += blockDim.x) {
        const int e = sBestE[g];
        out.slot_expert[g] = e;
        if (e >= 0) {
            atomicAdd(&sShed[e], sBestQ[g]);
            atomicAdd(&sCopies[e], 1);
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) out.n_copies[e] = 1 + sCopies[e];
    int q = 0;
    if (tid < P) {
        const int r = tid / (M + S);
        const int l = tid - r * (M + S);
        if (l < M) {
            const int e = r * M + l;
            q = sL[e] - sShed[e];
        } else {
            q = sBestQ[r * S + (l - M)];
        }
        out.slot_quota[tid] = q;
        atomicAdd(&sRankLoad[r], q);
    }
    int incl = q;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) sWarpSum[warp] = incl;
    __syncthreads();
    int wofs = 0;
    for (int w = 0; w < warp; ++w) wofs += sWarpSum[w];
    if (tid < P) out.slot_offset[tid] = wofs + incl - q;
    if (tid == 0) out.slot_offset[P] = (int)Q;
    for (int r = tid; r < R; r += blockDim.x) {
        out.rank_load[r] = sRankLoad[r];
        atomicMax(&sMaxAfter, sRankLoad[r]);
    }
    __syncthreads();
    if (tid == 0) {
        out.stats[0] = sProbes;
        out.stats[1] = sMaxH;
        out.stats[2] = sMaxAfter;
        out.stats[3] = (int)sLo;
    }
}

template <int NR, int NE>
void* kernel_ptr()
{
    return reinterpret_cast<void*>(&plan_bisect_kernel<NR, NE>);
}

void* pick_kernel(int R, int E)
{
    const int nr = R <= 32 ? 1 : R <= 64 ? 2 : 4;
    const int ne = E <= 32 ? 1 : E <= 64 ? 2 : E <= 128 ? 4 : 8;
    switch (nr * 16 + ne) {
    case 16 + 1: return kernel_ptr<1, 1>();
    case 16 + 2: return kernel_ptr<1, 2>();
    case 16 + 4: return kernel_ptr<1, 4>();
    case 16 + 8: return kernel_ptr<1, 8>();
    case 32 + 1: return kernel_ptr<2, 1>();
    case 32 + 2: return kernel_ptr<2, 2>();
    case 32 + 4: return kernel_ptr<2, 4>();
    case 32 + 8: return kernel_ptr<2, 8>();
    case 64 + 1: return kernel_ptr<4, 1>();
    case 64 + 2: return kernel_ptr<4, 2>();
    case 64 + 4: return kernel_ptr<4, 4>();
    default: return kernel_ptr<4, 8>();
    }
}

size_t dyn_bytes(const Sizes& z) { return (size_t)kBsWarps * (z.E + 2 * z.G) * sizeof(int); }

}  // namespace

cudaError_t plan_bisect_setup(const Sizes& z)
{
    return cudaFuncSetAttribute(pick_kernel(z.R, z.E), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)dyn_bytes(z));
}

cudaError_t launch_plan_bisect(const Sizes& z, const int32_t* load_e, int eps_inv, int threshold,
                               int min_tokens, int allow_zero, const ue_placement& out, int* err,
                               cudaStream_t st)
{
    BisectArgs a{eps_inv, threshold, min_tokens, allow_zero ? 1 : 0};
    void* args[] = {(void*)&load_e, (void*)&z.R, (void*)&z.E, (void*)&z.S, (void*)&a,
                    (void*)&out, (void*)&err};
    return cudaLaunchKernel(pick_kernel(z.R, z.E), dim3(1), dim3(kBsThreads), args,
                            dyn_bytes(z), st);
}

}  // namespace ue
