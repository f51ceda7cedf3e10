// Compressed scale format (CSF) of the NVFP4 block scales
// ("Step-5-Preview-NVFP4-Local", Format and Size).
//
// For a scale tensor u8 [E, R, C] (one E4M3 byte per 16 weights):
//   fixed       u8  [E, R/16, 16 * (1 + C/2)]: per slab of 16 rows, the 16 row
//               bases, then the rows' 4-bit codes in row order (C/2 bytes per
//               row, column 2j in the low nibble of byte j, 2j + 1 in the high);
//   exceptions  u32 [n]: (row * C + col) | byte << 24; expert 0's entries
//               first, then expert 1's and so on, each expert's in increasing
//               position;
//   starts      i64 [E + 1]: expert e's entries are exceptions[starts[e],
//               starts[e+1]).
// Decoding: byte = base(row) + code, or the stored byte of an exception.  A
// row's base is the smallest b in 0..240 that puts the largest number of the
// row's bytes inside [b, b + 15]; the code stored under an exception is 0.
//
// Decode (the serving-time step: one layer's scales are expanded into scratch
// before the layer runs, or only the experts a batch routes to):
//   csf_expand   a thread per 16 code bytes (32 scales), 16-byte loads and
//                stores; experts without routed rows are skipped when the
//                routing's expert offsets are given;
//   csf_patch    a CTA per expert writes its exceptions over the expansion.
// Encode (offline): csf_rows (a warp per row: 256-bin histogram in shared
// memory, window sums, codes, exception count), csf_scan (row offsets within
// each expert, then starts), csf_exceptions (a warp per row writes its
// exceptions in column order with a ballot prefix).
#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int kCsfWarps = 8;                          // warps per CTA of the per-row kernels

__device__ __forceinline__ uint32_t expand_nibbles(uint32_t codes16, uint32_t base4) {
    // two code bytes (4 codes, low nibble first) -> 4 scale bytes base + code
    const uint32_t lo = codes16 & 0xFFu, hi = (codes16 >> 8) & 0xFFu;
    const uint32_t v = (lo & 0xFu) | ((lo >> 4) << 8) | ((hi & 0xFu) << 16) | ((hi >> 4) << 24);
    return v + base4;                                 // no carries: base + code <= 255 per byte
}

__device__ __forceinline__ bool expert_live(const int32_t* offsets, int e) {
    return !offsets || offsets[e + 1] > offsets[e];
}

// Vector path (C % 32 == 0): thread i expands code bytes [16 i, 16 i + 16) of the tensor.
__global__ void __launch_bounds__(256) csf_expand(const uint8_t* __restrict__ fixed, int E, int R, int C,
                                                  const int32_t* __restrict__ offsets, uint8_t* __restrict__ out) {
    const int cpr = C / 32;                            // 16-byte code chunks per row
    const size_t slab = size_t(16) * (1 + C / 2);
    const size_t total = size_t(E) * R * cpr;
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += size_t(gridDim.x) * blockDim.x) {
        const size_t row = i / cpr;                    // e * R + r
        const int ch = int(i % cpr);
        const int e = int(row / R), r = int(row % R);
        if (!expert_live(offsets, e)) continue;
        const uint8_t* sl = fixed + (size_t(e) * (R / 16) + r / 16) * slab;
        const uint32_t base = sl[r % 16];
        const uint4 c = *reinterpret_cast<const uint4*>(sl + 16 + size_t(r % 16) * (C / 2) + ch * 16);
        const uint32_t b4 = base * 0x01010101u;
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
        uint32_t o[8];
#pragma unroll
        for (int j = 0; j < 4; j++) {
            o[2 * j] = expand_nibbles(w[j] & 0xFFFFu, b4);
            o[2 * j + 1] = expand_nibbles(w[j] >> 16, b4);
        }
        uint4* dst = reinterpret_cast<uint4*>(out + row * C + ch * 32);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

// Any even C: a thread per scale byte.
__global__ void __launch_bounds__(256) csf_expand_bytes(const uint8_t* __restrict__ fixed, int E, int R, int C,
                                                        const int32_t* __restrict__ offsets,
                                                        uint8_t* __restrict__ out) {
    const size_t slab = size_t(16) * (1 + C / 2);
    const size_t total = size_t(E) * R * C;
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += size_t(gridDim.x) * blockDim.x) {
        const size_t row = i / C;
        const int c = int(i % C);
        const int e = int(row / R), r = int(row % R);
        if (!expert_live(offsets, e)) continue;
        const uint8_t* sl = fixed + (size_t(e) * (R / 16) + r / 16) * slab;
        const uint32_t code = (sl[16 + size_t(r % 16) * (C / 2) + c / 2] >> (4 * (c & 1))) & 0xFu;
        out[i] = uint8_t(sl[r % 16] + code);
    }
}

// One CTA per expert: its exceptions over the expanded bytes (positions past
// R * C are ignored).
__global__ void __launch_bounds__(256) csf_patch(const uint32_t* __restrict__ exc, const int64_t* __restrict__ starts,
                                                 int R, int C, const int32_t* __restrict__ offsets,
                                                 uint8_t* __restrict__ out) {
    const int e = blockIdx.x;
    if (!expert_live(offsets, e)) return;
    const int64_t a = starts[e], b = starts[e + 1];
    const uint32_t n = uint32_t(R) * uint32_t(C);
    uint8_t* dst = out + size_t(e) * R * C;
    for (int64_t i = a + threadIdx.x; i < b; i += blockDim.x) {
        const uint32_t x = exc[i];
        const uint32_t pos = x & 0xFFFFFFu;
        if (pos < n) dst[pos] = uint8_t(x >> 24);
    }
}

// Encode, pass 1: a warp per row.  Base, codes, exception count.
__global__ void __launch_bounds__(kCsfWarps * 32) csf_rows(const uint8_t* __restrict__ sc, int E, int R, int C,
                                                          uint8_t* __restrict__ fixed, int32_t* __restrict__ rowcnt) {
    __shared__ int hist[kCsfWarps][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t row = size_t(blockIdx.x) * kCsfWarps + warp;
    if (row >= size_t(E) * R) return;                  // whole warps leave together
    const int e = int(row / R), r = int(row % R);
    const uint8_t* src = sc + row * C;
    int* h = hist[warp];
    for (int v = lane; v < 256; v += 32) h[v] = 0;
    __syncwarp();
    for (int c = lane; c < C; c += 32) atomicAdd(&h[src[c]], 1);
    __syncwarp();
    // window sums: lane covers bases 8 lane .. 8 lane + 7 (up to 240)
    int best_key = -1;
    const int b0 = lane * 8;
    if (b0 <= 240) {
        int s = 0;
        for (int v = b0; v < b0 + 16; v++) s += h[v];
        for (int b = b0; b < b0 + 8 && b <= 240; b++) {
            const int key = (s << 8) | (255 - b);      // more bytes first, then the lower base
            best_key = max(best_key, key);
            if (b + 16 <= 255) s += h[b + 16];
            s -= h[b];
        }
    }
    for (int o = 16; o > 0; o >>= 1) best_key = max(best_key, __shfl_xor_sync(0xffffffffu, best_key, o));
    const int base = 255 - (best_key & 255);
    uint8_t* sl = fixed + (size_t(e) * (R / 16) + r / 16) * (size_t(16) * (1 + C / 2));
    if (lane == 0) sl[r % 16] = uint8_t(base);
    uint8_t* codes = sl + 16 + size_t(r % 16) * (C / 2);
    int nexc = 0;
    for (int j = lane; j < C / 2; j += 32) {
        const int v0 = src[2 * j], v1 = src[2 * j + 1];
        const bool in0 = v0 >= base && v0 <= base + 15, in1 = v1 >= base && v1 <= base + 15;
        nexc += int(!in0) + int(!in1);
        codes[j] = uint8_t((in0 ? v0 - base : 0) | ((in1 ? v1 - base : 0) << 4));
    }
    for (int o = 16; o > 0; o >>= 1) nexc += __shfl_xor_sync(0xffffffffu, nexc, o);
    if (lane == 0) rowcnt[row] = nexc;
}

// Encode, pass 2: a CTA per expert turns its row counts into row offsets
// within the expert (in place) and writes the expert's total to tot[e].
__global__ void __launch_bounds__(1024) csf_scan_rows(int32_t* __restrict__ rowcnt, int R, int64_t* __restrict__ tot) {
    __shared__ int64_t s_w[32];
    const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int32_t* rc = rowcnt + size_t(e) * R;
    int64_t carry = 0;
    for (int r0 = 0; r0 < R; r0 += blockDim.x) {
        const int r = r0 + tid;
        const int64_t v = r < R ? rc[r] : 0;
        int64_t x = v;
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) s_w[warp] = x;
        __syncthreads();
        int64_t wbase = 0, all = 0;
        for (int q = 0; q < int(blockDim.x >> 5); q++) {
            if (q < warp) wbase += s_w[q];
            all += s_w[q];
        }
        if (r < R) rc[r] = int32_t(carry + wbase + x - v);     // exclusive offset within the expert
        carry += all;
        __syncthreads();
    }
    if (tid == 0) tot[e] = carry;
}

// Encode, pass 3: starts = exclusive scan of the expert totals (one CTA).
__global__ void __launch_bounds__(1024) csf_scan_experts(const int64_t* __restrict__ tot, int E,
                                                         int64_t* __restrict__ starts) {
    __shared__ int64_t s_w[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t v = tid < E ? tot[tid] : 0;
    int64_t x = v;
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_w[warp] = x;
    __syncthreads();
    int64_t wbase = 0, all = 0;
    for (int q = 0; q < int(blockDim.x >> 5); q++) {
        if (q < warp) wbase += s_w[q];
        all += s_w[q];
    }
    if (tid < E) starts[tid] = wbase + x - v;
    if (tid == 0) starts[E] = all;
}

// Encode, pass 4: a warp per row writes its exceptions in column order.
__global__ void __launch_bounds__(kCsfWarps * 32) csf_exceptions(const uint8_t* __restrict__ sc, int E, int R, int C,
                                                                const uint8_t* __restrict__ fixed,
                                                                const int32_t* __restrict__ rowoff,
                                                                const int64_t* __restrict__ starts,
                                                                uint32_t* __restrict__ exc, int64_t capacity,
                                                                int32_t* status) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t row = size_t(blockIdx.x) * kCsfWarps + warp;
    if (row >= size_t(E) * R) return;
    const int e = int(row / R), r = int(row % R);
    const uint8_t* src = sc + row * C;
    const int base = fixed[(size_t(e) * (R / 16) + r / 16) * (size_t(16) * (1 + C / 2)) + r % 16];
    int64_t idx = starts[e] + rowoff[row];
    for (int c0 = 0; c0 < C; c0 += 32) {
        const int c = c0 + lane;
        const int v = c < C ? src[c] : 0;
        const bool out = c < C && (v < base || v > base + 15);
        const uint32_t m = __ballot_sync(0xffffffffu, out);
        if (out) {
            const int64_t at = idx + __popc(m & ((1u << lane) - 1u));
            if (at < capacity) exc[at] = uint32_t(r * C + c) | (uint32_t(v) << 24);
            else set_status(status, MOE_ERR_DEVICE_INDEX);
        }
        idx += __popc(m);
    }
}

int grid_for(size_t n, int per_block) {
    const size_t b = (n + per_block - 1) / per_block;
    return int(std::min<size_t>(std::max<size_t>(b, 1), 148 * 16));
}

}  // namespace

int launch_csf_decode(const uint8_t* fixed, const uint32_t* exc, const int64_t* starts, int E, int R, int C,
                      const int32_t* offsets, uint8_t* out, cudaStream_t s) {
    const bool vec = C % 32 == 0 && (reinterpret_cast<uintptr_t>(fixed) & 15u) == 0 &&
                     (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
    if (vec) {
        csf_expand<<<grid_for(size_t(E) * R * (C / 32), 256), 256, 0, s>>>(fixed, E, R, C, offsets, out);
    } else {
        csf_expand_bytes<<<grid_for(size_t(E) * R * C, 256), 256, 0, s>>>(fixed, E, R, C, offsets, out);
    }
    count_launch();
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    if (exc) {
        csf_patch<<<E, 256, 0, s>>>(exc, starts, R, C, offsets, out);
        count_launch();
    }
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_csf_encode(const uint8_t* sc, int E, int R, int C, uint8_t* fixed, int64_t* starts, uint32_t* exc,
                      int64_t capacity, int32_t* rowcnt, int64_t* tot, int32_t* status, cudaStream_t s) {
    const size_t rows = size_t(E) * R;
    const int blocks = int((rows + kCsfWarps - 1) / kCsfWarps);
    csf_rows<<<blocks, kCsfWarps * 32, 0, s>>>(sc, E, R, C, fixed, rowcnt);
    count_launch();
    csf_scan_rows<<<E, 1024, 0, s>>>(rowcnt, R, tot);
    count_launch();
    csf_scan_experts<<<1, 1024, 0, s>>>(tot, E, starts);
    count_launch();
    if (exc) {
        csf_exceptions<<<blocks, kCsfWarps * 32, 0, s>>>(sc, E, R, C, fixed, rowcnt, starts, exc, capacity, status);
        count_launch();
    }
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
