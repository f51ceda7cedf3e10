// One NVFP4 block of 16 values ("Step-5-Preview-NVFP4-Local", Format: E2M1
// codes with one E4M3 scale per 16, times a global fp32 scale g):
//   sb = e4m3_rne_sat(amax / (6 g)),  code = e2m1_rne_sat(x / (e4m3(sb) g)),
// every step in fp32 with the hardware conversions (round to nearest even,
// saturating).  Shared by the weight quantiser and the activation quantisers.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace moe {

__device__ __forceinline__ uint32_t nv_f32_to_e4m3_rn_sat(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.f), "f"(v));
    return r & 0xffu;
}

__device__ __forceinline__ float nv_e4m3_val(uint32_t b) {
    uint32_t h;
    asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h) : "r"(b));
    return __half2float(__ushort_as_half(uint16_t(h & 0xffffu)));
}

__device__ __forceinline__ uint32_t nv_f32x2_to_e2m1x2(float lo, float hi) {
    uint16_t r;
    asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u16.u8 %0, t; }" : "=h"(r) : "f"(hi), "f"(lo));
    return r & 0xffu;
}

// Quantise x[0..16) with global g: the block's E4M3 scale byte and its eight
// code bytes (even element in the low nibble).
__device__ __forceinline__ uint32_t nv_quant_block16(const float (&x)[16], float g, uint32_t (&bytes)[8]) {
    float amax_b = 0.f;
#pragma unroll
    for (int i = 0; i < 16; i++) amax_b = fmaxf(amax_b, fabsf(x[i]));
    uint32_t sb = 0;
    if (g > 0.f) sb = nv_f32_to_e4m3_rn_sat(__fdiv_rn(amax_b, __fmul_rn(6.0f, g)));
    const float eff = __fmul_rn(nv_e4m3_val(sb), g);
#pragma unroll
    for (int j = 0; j < 8; j++)
        bytes[j] = eff > 0.f ? nv_f32x2_to_e2m1x2(__fdiv_rn(x[2 * j], eff), __fdiv_rn(x[2 * j + 1], eff)) : 0u;
    return sb;
}

}  // namespace moe
