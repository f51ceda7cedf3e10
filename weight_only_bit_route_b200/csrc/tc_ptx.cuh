// PTX wrappers shared by the tcgen05 kernels of libmoe (sm_100a): mbarriers
// with bounded waits, TMA copies, tcgen05 MMA / commit / TMEM load and store,
// shared-memory matrix descriptors, and the host-side tensor-map encoder.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "moe_internal.cuh"

namespace moe {

constexpr unsigned long long G_WAIT_NS = 2000000000ull;   // default bound on every device-side wait

// Per-CTA abort state of the warp-specialised kernels: the flag a role sets
// when one of its waits runs out (the other roles then stop issuing work),
// and the bound on each wait, read from the workspace control block (words
// 4-5, 0 = the default G_WAIT_NS; moe_set_wait_limit writes it).
struct GAbort {
    int flag;
    unsigned long long limit_ns;
};
// The configured wait bound (status = the control block, may be null).  Read
// it after griddepcontrol.wait: the word may come from the previous kernel.
__device__ __forceinline__ unsigned long long g_limit_from(const int32_t* status) {
    if (!status) return G_WAIT_NS;
    const unsigned long long v = *reinterpret_cast<const volatile unsigned long long*>(status + 4);
    return v ? v : G_WAIT_NS;
}

// Failure-testing hold: word 6 of the control block (moe_set_wait_hold).
__device__ __forceinline__ int g_hold_from(const int32_t* status) {
    return status ? *reinterpret_cast<const volatile int32_t*>(status + 6) : 0;
}

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t g_smem(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ unsigned long long g_timer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ bool g_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
// Bounded wait: false once the configured bound has passed, or as soon as
// another role has aborted.  Roles off the critical path back off with a
// short sleep between polls so that they leave issue slots to the
// dequantisation warps.
__device__ __forceinline__ bool g_wait(uint32_t bar, uint32_t parity, volatile GAbort* ab, int sleep_ns = 0) {
    if (g_try(bar, parity)) return true;
    const unsigned long long t0 = g_timer();
    while (true) {
        if (sleep_ns) __nanosleep(sleep_ns);
        if (g_try(bar, parity)) return true;
        if (ab->flag || g_timer() - t0 > ab->limit_ns) return false;
    }
}
// Warp-wide bounded wait: every lane observes the phase (so whichever lane
// is elected to issue has acquired it); the outcome is warp-uniform, so the
// warp stays converged for the .sync.aligned instructions that follow.
__device__ __forceinline__ bool g_wait_w(uint32_t bar, uint32_t parity, volatile GAbort* ab, int sleep_ns = 0) {
    const bool ok = g_wait(bar, parity, ab, sleep_ns);
    return __all_sync(0xffffffffu, ok);
}
// Warp-uniform test of the abort flag (loop conditions of whole-warp roles).
__device__ __forceinline__ bool g_aborted(volatile GAbort* ab) { return __any_sync(0xffffffffu, ab->flag != 0); }
// Bounded wait that ignores the abort flag (draining work already in flight).
__device__ __forceinline__ void g_drain_wait(uint32_t bar, uint32_t parity) {
    const unsigned long long t0 = g_timer();
    while (!g_try(bar, parity) && g_timer() - t0 < G_WAIT_NS) {
    }
}
// One lane of a converged warp (warp-uniform code keeps the operands of the
// tcgen05 and TMA instructions in uniform registers; issuing from inside a
// lane-0 branch costs tens of cycles per instruction).
__device__ __forceinline__ bool g_elect() {
    uint32_t pred = 0;
    asm volatile("{ .reg .pred p; elect.sync _|p, 0xffffffff; selp.u32 %0, 1, 0, p; }" : "=r"(pred));
    return pred != 0;
}
__device__ __forceinline__ void g_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void g_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void g_tma2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}
__device__ __forceinline__ void g_bulk(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}
// K-major operand, 128-byte swizzle, 8-row groups 1024 bytes apart
__device__ __forceinline__ uint64_t g_desc(uint32_t saddr) {
    return uint64_t((saddr >> 4) & 0x3FFF) | (uint64_t(1) << 16) | (uint64_t(64) << 32) | (uint64_t(1) << 46) |
           (uint64_t(2) << 61);
}
// kind::f16 instruction descriptor: fp32 accumulate, A/B bf16 (or f16), both K-major, M x N
__device__ __forceinline__ uint32_t g_idesc(int n, bool f16, int m = 128) {
    const uint32_t ab = f16 ? 0u : 1u;
    return (1u << 4) | (ab << 7) | (ab << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}
__device__ __forceinline__ void g_mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile("{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }"
                 ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void g_mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile("{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }"
                 ::"r"(d), "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
// kind::i8: D s32, A u8 (bits 7-9 = 0), B s8 (bits 10-12 = 1), K = 32 per instruction
__device__ __forceinline__ uint32_t g_idesc_i8(int n, int m = 128) {
    return (2u << 4) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}
__device__ __forceinline__ void g_mma_ts_i8(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile("{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p; }"
                 ::"r"(d), "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
// kind::mxf4nvf4 block-scaled instruction descriptor: A and B E2M1 (format 1), UE4M3 scale
// factors (scale format 0, factor ids 0), K-major, M = 128, N = n, dense K = 64
__device__ __forceinline__ uint32_t g_idesc_mxf4(int n, int m = 128) {
    return (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}
// D (+)= A (E2M1, shared memory) x B (E2M1, shared memory), each 16-element block scaled by its
// E4M3 factor from tensor memory (sfa: the A rows' four factors of this K 64, sfb: B's)
__device__ __forceinline__ void g_mma_mxf4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc,
                                           uint32_t sfa, uint32_t sfb) {
    asm volatile("{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
                 "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p; }"
                 ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb) : "memory");
}
// Shared-memory descriptor of a 32-row x 16-byte scale-factor chunk (rows 16 bytes apart, no
// swizzle: 8-row core matrices 128 bytes apart)
__device__ __forceinline__ uint64_t g_desc_sf(uint32_t saddr) {
    return uint64_t((saddr >> 4) & 0x3FFF) | (uint64_t(128 >> 4) << 16) | (uint64_t(128 >> 4) << 32) |
           (uint64_t(1) << 46);
}
// Copy one scale-factor chunk into four tensor-memory columns, broadcast to the four lane
// quarters: lane 32 q + m0 then holds the factors of rows m0, m0 + 32, m0 + 64, m0 + 96
__device__ __forceinline__ void g_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void g_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void g_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void g_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void g_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
}
__device__ __forceinline__ void g_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void g_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                 ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
                   "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
                 : "memory");
}
__device__ __forceinline__ void g_fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void g_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ uint32_t g_e2m1x2_f16x2(uint32_t byte) {
    uint32_t h;
    asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h) : "r"(byte));
    return h;
}
// The four bytes of a word, each a pair of E2M1 codes (low nibble first), as four f16 pairs.
__device__ __forceinline__ void g_e2m1x8_f16x2(uint32_t w, uint32_t (&h)[4]) {
    asm("{ .reg .b8 b0, b1, b2, b3; mov.b32 {b0, b1, b2, b3}, %4;\n"
        " cvt.rn.f16x2.e2m1x2 %0, b0; cvt.rn.f16x2.e2m1x2 %1, b1;\n"
        " cvt.rn.f16x2.e2m1x2 %2, b2; cvt.rn.f16x2.e2m1x2 %3, b3; }"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(w));
}
__device__ __forceinline__ uint32_t g_e4m3_f16x2(uint32_t byte) {          // {s, s} in f16
    uint32_t h;
    asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h) : "r"(byte | (byte << 8)));
    return h;
}
// byte offset of 16-byte chunk c of row r in a 128-byte-swizzled tile (1024-byte aligned)
__device__ __forceinline__ uint32_t g_swz(int r, int c) { return uint32_t(r * 128 + ((c ^ (r & 7)) << 4)); }

// ---------------------------------------------------------------------------
// Host: 2D tensor maps (cuTensorMapEncodeTiled through the runtime's driver
// entry point, so the library links no driver library)
// ---------------------------------------------------------------------------
inline PFN_cuTensorMapEncodeTiled& g_encode_fn_ref() {
    static PFN_cuTensorMapEncodeTiled fn = nullptr;
    return fn;
}

// Resolves cuTensorMapEncodeTiled through the runtime once per process.
inline int g_encoder() {
    static std::once_flag once;
    std::call_once(once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode_fn_ref() = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(fn);
    });
    return g_encode_fn_ref() ? MOE_OK : MOE_ERR_CUDA;
}

// 2D map over [outer rows][inner elements] of 1- or 2-byte elements; pitch in bytes.
inline int g_map(CUtensorMap* m, bool two_byte, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch,
                 uint32_t box_in, uint32_t box_out, bool swz) {
    if ((reinterpret_cast<uintptr_t>(base) & 15u) || (pitch & 15u)) return MOE_ERR_INVALID_ARG;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {pitch};
    cuuint32_t box[2] = {box_in, box_out};
    cuuint32_t es[2] = {1, 1};
    const CUresult r = g_encode_fn_ref()(m, two_byte ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                                   const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                   swz ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
