// Unpermute + weighted combine ("Step 5 Preview: 92 narrow layers...", The
// shape: each token's output is its shared expert plus its 8 routed experts;
// the routing weight was already applied in the down projection):
//     y[t] = bf16( shared[t] + sum_{j<k} y_perm[slot_row[t*k + j]] ),  fp32 sum
// Thread per 8 consecutive hidden elements (16-byte loads and stores).
#include <algorithm>

#include "moe_internal.cuh"

namespace moe {

template <bool F16OUT>
__global__ void __launch_bounds__(256) combine_kernel(
        const __nv_bfloat16* __restrict__ y_perm, const int32_t* __restrict__ slot_row, int T,
        int k, int H, const __nv_bfloat16* __restrict__ shared_out, __nv_bfloat16* __restrict__ y) {
    asm volatile("griddepcontrol.wait;" ::: "memory");   // y_perm / shared_out of the previous kernels
    const int per_row = H / 8;
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long long)T * per_row) return;
    const int t = int(idx / per_row), c = int(idx % per_row);
    float acc[8];
    if (shared_out) {
        const uint4 v = *reinterpret_cast<const uint4*>(shared_out + size_t(t) * H + c * 8);
        acc[0] = bf16_lo(v.x); acc[1] = bf16_hi(v.x); acc[2] = bf16_lo(v.y); acc[3] = bf16_hi(v.y);
        acc[4] = bf16_lo(v.z); acc[5] = bf16_hi(v.z); acc[6] = bf16_lo(v.w); acc[7] = bf16_hi(v.w);
    } else {
#pragma unroll
        for (int i = 0; i < 8; i++) acc[i] = 0.f;
    }
    for (int j = 0; j < k; j++) {
        const int r = slot_row[size_t(t) * k + j];
        if (r < 0) continue;                          // dropped slot (invalid expert id)
        const uint4 v = *reinterpret_cast<const uint4*>(y_perm + size_t(r) * H + c * 8);
        acc[0] += bf16_lo(v.x); acc[1] += bf16_hi(v.x); acc[2] += bf16_lo(v.y); acc[3] += bf16_hi(v.y);
        acc[4] += bf16_lo(v.z); acc[5] += bf16_hi(v.z); acc[6] += bf16_lo(v.w); acc[7] += bf16_hi(v.w);
    }
    uint4 o;
    if constexpr (F16OUT) {                  // fp16 activation mode: y in fp16
        __half2 p;
        p = __floats2half2_rn(acc[0], acc[1]); o.x = *reinterpret_cast<uint32_t*>(&p);
        p = __floats2half2_rn(acc[2], acc[3]); o.y = *reinterpret_cast<uint32_t*>(&p);
        p = __floats2half2_rn(acc[4], acc[5]); o.z = *reinterpret_cast<uint32_t*>(&p);
        p = __floats2half2_rn(acc[6], acc[7]); o.w = *reinterpret_cast<uint32_t*>(&p);
    } else {
        __nv_bfloat162 p;
        p = __floats2bfloat162_rn(acc[0], acc[1]); o.x = *reinterpret_cast<uint32_t*>(&p);
        p = __floats2bfloat162_rn(acc[2], acc[3]); o.y = *reinterpret_cast<uint32_t*>(&p);
        p = __floats2bfloat162_rn(acc[4], acc[5]); o.z = *reinterpret_cast<uint32_t*>(&p);
        p = __floats2bfloat162_rn(acc[6], acc[7]); o.w = *reinterpret_cast<uint32_t*>(&p);
    }
    *reinterpret_cast<uint4*>(y + size_t(t) * H + c * 8) = o;
}

int launch_combine(const __nv_bfloat16* y_perm, const int32_t* slot_row, int T, int k, int H,
                   const __nv_bfloat16* shared_out, __nv_bfloat16* y, cudaStream_t s, bool pdl, int y_f16) {
    const long long n = (long long)T * (H / 8);
    const int blocks = int((n + 255) / 256);
    auto kern = y_f16 ? combine_kernel<true> : combine_kernel<false>;
    if (pdl) {
        if (launch_pdl(kern, dim3(blocks), dim3(256), 0, s, y_perm, slot_row, T, k, H, shared_out, y) != cudaSuccess)
            return MOE_ERR_CUDA;
    } else {
        kern<<<blocks, 256, 0, s>>>(y_perm, slot_row, T, k, H, shared_out, y);
        count_launch();
    }
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

__global__ void __launch_bounds__(256) f16_to_bf16_kernel(const __half* __restrict__ src,
                                                         __nv_bfloat16* __restrict__ dst, size_t n8) {
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += size_t(gridDim.x) * blockDim.x) {
        const uint4 v = reinterpret_cast<const uint4*>(src)[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const __half2 h = *reinterpret_cast<const __half2*>(&w[j]);
            __nv_bfloat162 b = __floats2bfloat162_rn(__low2float(h), __high2float(h));
            o[j] = *reinterpret_cast<uint32_t*>(&b);
        }
        reinterpret_cast<uint4*>(dst)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

int launch_f16_to_bf16(const __half* src, __nv_bfloat16* dst, size_t n, cudaStream_t s) {
    const size_t n8 = n / 8;
    const int blocks = int(std::min<size_t>((n8 + 255) / 256, 148 * 8));
    f16_to_bf16_kernel<<<blocks > 0 ? blocks : 1, 256, 0, s>>>(src, dst, n8);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// The shared expert runs through the grouped kernels as one expert that
// owns every token: offsets = {0, T}, row i <- slot i*k (token i).
__global__ void shared_routing_kernel(int T, int k, int32_t* sh_offsets, int32_t* sh_rowslot) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i == 0) { sh_offsets[0] = 0; sh_offsets[1] = T; }
    if (i < T) sh_rowslot[i] = i * k;
}

int launch_shared_routing(int T, int k, int32_t* sh_offsets, int32_t* sh_rowslot, cudaStream_t s) {
    shared_routing_kernel<<<(T + 255) / 256, 256, 0, s>>>(T, k, sh_offsets, sh_rowslot);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// One 64-bit word of the workspace control block (moe_set_wait_limit).
__global__ void set_u64_kernel(unsigned long long* dst, unsigned long long v) { *dst = v; }

int launch_set_u64(unsigned long long* dst, unsigned long long v, cudaStream_t s) {
    set_u64_kernel<<<1, 1, 0, s>>>(dst, v);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// One 32-bit word of the workspace control block (moe_set_wait_hold).
__global__ void set_u32_kernel(uint32_t* dst, uint32_t v) { *dst = v; }

int launch_set_u32(uint32_t* dst, uint32_t v, cudaStream_t s) {
    set_u32_kernel<<<1, 1, 0, s>>>(dst, v);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
