// Token -> expert bucketing: a stable counting sort of the R = T*k routing
// slots (slot = t*k + j) by expert id, so that each expert's rows form one
// contiguous range [offsets[e], offsets[e+1]) ordered by slot.
//
// Three short kernels over blocks of kPermChunk slots:
//   1. count:   per-block histogram hist[b][e] (shared-memory atomics; a count
//               does not depend on the order of the adds),
//   2. scan:    offsets = exclusive scan of the totals; hist[b][e] becomes the
//               first row of block b's slots of expert e,
//   3. scatter: each warp walks a contiguous run of its block's slots in order;
//               __match_any_sync groups equal ids inside a 32-slot step, so the
//               rank of a slot among equal ids is its popcount of lower lanes.
// No global atomics decide a position, so the permutation is deterministic.
#include <mutex>

#include "moe_internal.cuh"

namespace moe {

constexpr int kPermThreads = 256;
constexpr int kPermWarps = kPermThreads / 32;

__global__ void __launch_bounds__(kPermThreads) perm_count(
        const int32_t* __restrict__ ids, int R, int E, int32_t* __restrict__ hist,
        int32_t* status) {
    __shared__ int32_t h[kMaxE];
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    const int s0 = blockIdx.x * kPermChunk;
    const int s1 = min(R, s0 + kPermChunk);
    for (int s = s0 + threadIdx.x; s < s1; s += blockDim.x) {
        int e = ids[s];
        if (e >= 0 && e < E) atomicAdd(&h[e], 1);
        else set_status(status, MOE_ERR_DEVICE_INDEX);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[size_t(blockIdx.x) * E + e] = h[e];
}

// One CTA of 1024 threads, thread e owns expert e.
__global__ void __launch_bounds__(1024) perm_scan(int32_t* __restrict__ hist, int nb, int E,
                                                 int32_t* __restrict__ offsets) {
    __shared__ int32_t wsum[32];
    const int e = threadIdx.x;
    int total = 0;
    if (e < E)
        for (int b = 0; b < nb; b++) total += hist[size_t(b) * E + e];
    // block-wide exclusive scan of total over e
    const int lane = e & 31, warp = e >> 5;
    int v = total;
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) wsum[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = wsum[lane];
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        wsum[lane] = w;
    }
    __syncthreads();
    const int incl = v + (warp > 0 ? wsum[warp - 1] : 0);
    const int excl = incl - total;
    if (e < E) {
        offsets[e] = excl;
        int run = excl;
        for (int b = 0; b < nb; b++) {
            int c = hist[size_t(b) * E + e];
            hist[size_t(b) * E + e] = run;
            run += c;
        }
    }
    if (e == E - 1) offsets[E] = incl;
}

__global__ void __launch_bounds__(kPermThreads) perm_scatter(
        const int32_t* __restrict__ ids, int R, int E, const int32_t* __restrict__ hist,
        int32_t* __restrict__ row_slot, int32_t* __restrict__ slot_row) {
    extern __shared__ int32_t wbase[];          // [kPermWarps][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int s0 = blockIdx.x * kPermChunk;
    const int s1 = min(R, s0 + kPermChunk);
    const int per_warp = kPermChunk / kPermWarps;
    const int w0 = s0 + warp * per_warp;
    const int w1 = min(s1, w0 + per_warp);
    for (int i = threadIdx.x; i < kPermWarps * E; i += blockDim.x) wbase[i] = 0;
    __syncthreads();
    int32_t* mine = wbase + warp * E;
    // pass 1: per-warp counts
    for (int s = w0; s < w1; s += 32) {
        const int si = s + lane;
        const int e = (si < w1) ? ids[si] : -1;
        const bool ok = (e >= 0 && e < E);
        const unsigned act = __ballot_sync(0xffffffffu, ok);
        const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1) & act;
        if (ok && (__ffs(peers) - 1) == lane) mine[e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // exclusive prefix over warps, on top of the block's base from the scan
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = hist[size_t(blockIdx.x) * E + e];
        for (int w = 0; w < kPermWarps; w++) {
            int c = wbase[w * E + e];
            wbase[w * E + e] = run;
            run += c;
        }
    }
    __syncthreads();
    // pass 2: stable placement
    const unsigned lt = (1u << lane) - 1u;
    for (int s = w0; s < w1; s += 32) {
        const int si = s + lane;
        const int e = (si < w1) ? ids[si] : -1;
        const bool ok = (e >= 0 && e < E);
        const unsigned act = __ballot_sync(0xffffffffu, ok);
        const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1) & act;
        int pos = 0;
        if (ok) pos = mine[e] + __popc(peers & lt);
        __syncwarp();
        if (ok && (__ffs(peers) - 1) == lane) mine[e] += __popc(peers);
        __syncwarp();
        if (si < w1) {
            if (ok) { row_slot[pos] = si; slot_row[si] = pos; }
            else slot_row[si] = -1;
        }
    }
}

int launch_permute(const int32_t* ids, int T, int k, int E, int32_t* offsets,
                   int32_t* row_slot, int32_t* slot_row, int32_t* hist, int32_t* status,
                   cudaStream_t s) {
    const int R = T * k;
    const int nb = (R + kPermChunk - 1) / kPermChunk;
    perm_count<<<nb, kPermThreads, 0, s>>>(ids, R, E, hist, status);
    count_launch();
    perm_scan<<<1, 1024, 0, s>>>(hist, nb, E, offsets);
    count_launch();
    const size_t smem = size_t(kPermWarps) * E * sizeof(int32_t);
    perm_scatter<<<nb, kPermThreads, smem, s>>>(ids, R, E, hist, row_slot, slot_row);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Bucketing without caller-provided workspace, for callers that cannot
// allocate: code running inside a fixed memory plan that has no spare buffer to
// give, or a step that must not stall on the device-wide synchronisation an
// allocation can cause.  Its scratch (a status word and the per-block expert
// histograms) is a file-scope device array, so the call allocates nothing;
// every GPU that loads this library holds the array (about 64 KB) until the
// process exits.  Calls that overlap on the GPU share the array and race.
// ---------------------------------------------------------------------------
constexpr int kNoAllocMaxSlots = 65536;                       // T * top_k
constexpr int kNoAllocBlocks = kNoAllocMaxSlots / kPermChunk;
constexpr int kNoAllocHeader = 64;                            // status word + padding (ints)
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocHeader + kNoAllocBlocks * kMaxE];

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is resolved
// with cudaGetSymbolAddress the first time a device is used and cached.
static int noalloc_scratch(int32_t** out) {
    constexpr int kMaxDevices = 64;
    static int32_t* addr[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
        addr[dev] = static_cast<int32_t*>(p);
    }
    *out = addr[dev];
    return MOE_OK;
}

int launch_permute_noalloc(const int32_t* ids, int T, int k, int E, int32_t* offsets, int32_t* row_slot,
                           int32_t* slot_row, cudaStream_t s) {
    if (size_t(T) * k > size_t(kNoAllocMaxSlots) || E > kMaxE) return MOE_ERR_UNSUPPORTED;
    int32_t* scratch = nullptr;
    const int rc = noalloc_scratch(&scratch);
    if (rc != MOE_OK) return rc;
    // the status word must start at zero; the histograms are fully rewritten
    if (cudaMemsetAsync(scratch, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
    return launch_permute(ids, T, k, E, offsets, row_slot, slot_row, scratch + kNoAllocHeader, scratch, s);
}

}  // namespace moe
