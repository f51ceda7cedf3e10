// Weight conversion kernels (offline step): bf16 expert matrices -> the two
// 4-bit formats the layer consumes.  Every floating-point step is an explicit
// IEEE round-to-nearest operation (no contraction), so the codes and scales
// are a deterministic function of the input.
//
// int4 symmetric g128 ("Step-5-Preview-Int4-g128", Recipe): per group of 128,
// scale = bf16((r * amax) / 7) for the clip ratio r in {24/40, ..., 40/40}
// minimising sum (q*s - w)^2 (fp32, index order, ties keep the larger ratio),
// q = clamp(rint(w / s), -8, 7), stored as nibble q + 8, low nibble first.
//
// NVFP4 ("Step-5-Preview-NVFP4-Local", Format): global = amax / (6 * 448);
// block scale = E4M3(amax_block / (6 * global)); code = E2M1(w / (E4M3 * global)),
// both conversions round to nearest even and saturate (hardware cvt).
#include "moe_internal.cuh"
#include "nvfp4_block.cuh"

namespace moe {

__device__ __forceinline__ int rint_clamp_q(float w, float s) {
    double q = rint(double(w) / double(s));
    q = fmin(fmax(q, -8.0), 7.0);
    return int(q);
}

// one thread per group of 128
__global__ void quant_int4_kernel(const __nv_bfloat16* __restrict__ w, long long rows, long long cols,
                                  int32_t* __restrict__ packed, __nv_bfloat16* __restrict__ scales) {
    const long long ng = cols / 128;
    const long long gidx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gidx >= rows * ng) return;
    const long long r = gidx / ng, g = gidx % ng;
    const __nv_bfloat16* src = w + r * cols + g * 128;
    float wf[128];
    float amax = 0.f;
#pragma unroll 8
    for (int i = 0; i < 128; i += 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(src + i);
        wf[i + 0] = bf16_lo(v.x); wf[i + 1] = bf16_hi(v.x); wf[i + 2] = bf16_lo(v.y); wf[i + 3] = bf16_hi(v.y);
        wf[i + 4] = bf16_lo(v.z); wf[i + 5] = bf16_hi(v.z); wf[i + 6] = bf16_lo(v.w); wf[i + 7] = bf16_hi(v.w);
    }
    for (int i = 0; i < 128; i++) amax = fmaxf(amax, fabsf(wf[i]));
    __nv_bfloat16 best_s = __float2bfloat16_rn(0.f);
    if (amax > 0.f) {
        float best_err = INFINITY;
        for (int i = 16; i >= 0; i--) {
            const float ratio = __fdiv_rn(float(24 + i), 40.0f);
            const float sf = __fdiv_rn(__fmul_rn(ratio, amax), 7.0f);
            const __nv_bfloat16 sb = __float2bfloat16_rn(sf);
            const float s = __bfloat162float(sb);
            if (s == 0.f) continue;
            float err = 0.f;
            for (int j = 0; j < 128; j++) {
                const float d = __fsub_rn(__fmul_rn(float(rint_clamp_q(wf[j], s)), s), wf[j]);
                err = __fadd_rn(err, __fmul_rn(d, d));
            }
            if (err < best_err) { best_err = err; best_s = sb; }
        }
    }
    scales[r * ng + g] = best_s;
    const float s = __bfloat162float(best_s);
    int32_t* dst = packed + r * (cols / 8) + g * 16;
    for (int c = 0; c < 16; c++) {
        uint32_t word = 0;
        for (int j = 0; j < 8; j++) {
            const int q = (s == 0.f) ? 0 : rint_clamp_q(wf[c * 8 + j], s);
            word |= uint32_t((q + 8) & 0xF) << (4 * j);
        }
        dst[c] = int32_t(word);
    }
}

__global__ void amax_kernel(const __nv_bfloat16* __restrict__ w, long long n, uint32_t* slot) {
    float m = 0.f;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        m = fmaxf(m, fabsf(__bfloat162float(w[i])));
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) atomicMax(slot, __float_as_uint(m));   // m >= 0: bit order = value order
}

// one thread per block of 16
__global__ void quant_nvfp4_kernel(const __nv_bfloat16* __restrict__ w, long long rows, long long cols,
                                   const uint32_t* __restrict__ amax_slot, uint8_t* __restrict__ packed,
                                   uint8_t* __restrict__ scales, float* __restrict__ global_out) {
    const long long nb = cols / 16;
    const long long bidx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const float amax = __uint_as_float(*amax_slot);
    const float g = __fdiv_rn(amax, 2688.0f);
    if (bidx == 0) *global_out = g;
    if (bidx >= rows * nb) return;
    const long long r = bidx / nb, b = bidx % nb;
    const __nv_bfloat16* src = w + r * cols + b * 16;
    float wf[16];
    for (int i = 0; i < 16; i++) wf[i] = __bfloat162float(src[i]);
    uint32_t bytes[8];
    scales[r * nb + b] = uint8_t(nv_quant_block16(wf, g, bytes));
    uint8_t* dst = packed + r * (cols / 2) + b * 8;
    for (int j = 0; j < 8; j++) dst[j] = uint8_t(bytes[j]);
}

// Activations ("Step-5-Preview-NVFP4-Local", Modifications: quant_algo NVFP4
// with an input_scale): row r quantised with its own global g[r]; one thread
// per block of 16.
__global__ void quant_nvfp4_act_kernel(const __nv_bfloat16* __restrict__ x, long long rows, long long cols,
                                       const float* __restrict__ g, uint8_t* __restrict__ packed,
                                       uint8_t* __restrict__ scales) {
    const long long nb = cols / 16;
    const long long bidx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (bidx >= rows * nb) return;
    const long long r = bidx / nb, b = bidx % nb;
    const __nv_bfloat16* src = x + r * cols + b * 16;
    float xf[16];
    for (int i = 0; i < 16; i++) xf[i] = __bfloat162float(src[i]);
    uint32_t bytes[8];
    scales[r * nb + b] = uint8_t(nv_quant_block16(xf, g[r], bytes));
    uint8_t* dst = packed + r * (cols / 2) + b * 8;
    for (int j = 0; j < 8; j++) dst[j] = uint8_t(bytes[j]);
}

int launch_quant_int4(const __nv_bfloat16* w, int64_t rows, int64_t cols, int32_t* packed,
                      __nv_bfloat16* scales, cudaStream_t s) {
    const long long n = rows * (cols / 128);
    quant_int4_kernel<<<int((n + 127) / 128), 128, 0, s>>>(w, rows, cols, packed, scales);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_quant_nvfp4_act(const __nv_bfloat16* x, int64_t rows, int64_t cols, const float* g, uint8_t* packed,
                           uint8_t* scales, cudaStream_t s) {
    const long long nb = rows * (cols / 16);
    quant_nvfp4_act_kernel<<<int((nb + 255) / 256), 256, 0, s>>>(x, rows, cols, g, packed, scales);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_quant_nvfp4(const __nv_bfloat16* w, int64_t rows, int64_t cols, uint8_t* packed,
                       uint8_t* scales, float* global, uint32_t* amax_slot, cudaStream_t s) {
    if (cudaMemsetAsync(amax_slot, 0, 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    const long long n = rows * cols;
    int blocks = int(std::min<long long>((n + 255) / 256, 148 * 8));
    amax_kernel<<<blocks, 256, 0, s>>>(w, n, amax_slot);
    count_launch();
    const long long nb = rows * (cols / 16);
    quant_nvfp4_kernel<<<int((nb + 255) / 256), 256, 0, s>>>(w, rows, cols, amax_slot, packed, scales, global);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
