// Router logits on the tensor cores for prefill-sized batches:
//     l[t, e] = sum_h x[t, h] * Wr[e, h]       (fp32)
// for the sigmoid router over the routed experts ("Step-5-Preview-Spark", At a
// glance).  The bias and the sigmoid / top-k follow in router_topk.
//
// x is bf16, so every x[t, h] is exact in bf16.  The fp32 router weights are
// split once per call into three bf16 planes, Wr = hi + mid + lo, with hi the
// nearest bf16 to Wr, mid the nearest to Wr - hi and lo the nearest to
// Wr - hi - mid; the three planes hold Wr to within 2^-26 relative.  A bf16 x
// bf16 product has at most 16 significant bits, so each product is exact in
// fp32, and the tensor core accumulates in fp32: the result differs from a
// sequential fp32 dot product only in the order and rounding of the sums.
// The tensor core's fp32 accumulation does not round to nearest, and over the
// 768 MMAs of a 4096-long dot product its error grows to a few 1e-5 of the
// logit.  So each K = 64 stage (12 MMAs) accumulates into a fresh tensor-memory
// buffer, and the epilogue warps add the stage sums into fp32 registers with
// ordinary round-to-nearest adds, overlapped with the next stage's MMAs.
//
// One CTA per (128 experts, 64 tokens) tile.  Warp 4 streams K = 64 stages by
// TMA (the three weight planes and the token rows, 128-byte swizzled), warp 5
// issues three tcgen05.mma per K = 16 step (one per plane) into one of two
// accumulator buffers, and warps 0-3 drain the buffers with tcgen05.ld.  Every
// wait is bounded and reports MOE_ERR_TIMEOUT.
#include <cstring>

#include "moe_internal.cuh"
#include "tc_ptx.cuh"

namespace moe {

constexpr int RT_M = 128;          // experts per tile (MMA M)
constexpr int RT_BN = 64;          // tokens per tile (MMA N)
constexpr int RT_STAGES = 3;
constexpr int RT_THREADS = 192;
constexpr int RT_PLANE = RT_M * 128;   // one weight plane of a K = 64 stage: 16 KB
constexpr int RT_STAGE = 3 * RT_PLANE + RT_BN * 128;

struct RtArgs {
    CUtensorMap tm_w;    // planes [3 * E, H] bf16
    CUtensorMap tm_x;    // x [T, H] bf16
    float* logits;       // [T, E]
    int32_t* status;
    int T, E, H;
};

__global__ void __launch_bounds__(RT_THREADS, 1) router_tc(const __grid_constant__ RtArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ __align__(8) uint64_t full[RT_STAGES], empty[RT_STAGES], acc_full[2], acc_empty[2], done;
    __shared__ uint32_t s_tmem;
    __shared__ volatile GAbort s_ab;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * RT_M, n0 = blockIdx.y * RT_BN;
    const int KB = a.H / 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < RT_STAGES; s++) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(g_smem(&full[s])));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(g_smem(&empty[s])));
        }
        for (int b = 0; b < 2; b++) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(g_smem(&acc_full[b])));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 4;" ::"r"(g_smem(&acc_empty[b])));
        }
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(g_smem(&done)));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_ab.flag = 0;
        s_ab.limit_ns = G_WAIT_NS;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 128;" ::"r"(g_smem(&s_tmem)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0) s_ab.limit_ns = g_limit_from(a.status);
    g_fence_before();
    __syncthreads();
    g_fence_after();
    const uint32_t tmem = s_tmem;
    uint8_t* ring = smem + ((1024u - (g_smem(smem) & 1023u)) & 1023u);
    auto fail = [&]() {
        set_status(a.status, MOE_ERR_TIMEOUT);
        s_ab.flag = 1;
    };

    if (warp == 4) {
        // TMA producer: three weight planes (rows p*E + m0 ...) and 64 token rows per stage
        int kb = 0;
        for (; kb < KB && !g_aborted(&s_ab); kb++) {
            const int s = kb % RT_STAGES;
            if (kb >= RT_STAGES && !g_wait_w(g_smem(&empty[s]), ((kb / RT_STAGES) - 1) & 1, &s_ab, 32)) {
                fail();
                break;
            }
            const uint32_t st = g_smem(ring + s * RT_STAGE), bar = g_smem(&full[s]);
            if (g_elect()) {
                g_expect(bar, RT_STAGE);
#pragma unroll
                for (int p = 0; p < 3; p++) g_tma2d(st + p * RT_PLANE, &a.tm_w, kb * 64, p * a.E + m0, bar);
                g_tma2d(st + 3 * RT_PLANE, &a.tm_x, kb * 64, n0, bar);
            }
            __syncwarp();
        }
        if (lane == 0)
            for (int n = kb > RT_STAGES ? kb - RT_STAGES : 0; n < kb; n++)
                g_drain_wait(g_smem(&full[n % RT_STAGES]), (n / RT_STAGES) & 1);
        __syncwarp();
    } else if (warp == 5) {
        // MMA issuer: stage kb accumulates (from zero) into buffer kb & 1
        const uint32_t idesc = g_idesc(RT_BN, false, RT_M);
        for (int kb = 0; kb < KB && !g_aborted(&s_ab); kb++) {
            const int s = kb % RT_STAGES, b = kb & 1;
            if (kb >= 2 && !g_wait_w(g_smem(&acc_empty[b]), ((kb >> 1) - 1) & 1, &s_ab)) {
                fail();
                break;
            }
            if (!g_wait_w(g_smem(&full[s]), (kb / RT_STAGES) & 1, &s_ab)) {
                fail();
                break;
            }
            g_fence_after();
            const uint32_t st = g_smem(ring + s * RT_STAGE);
            const uint32_t d = tmem + b * RT_BN;
            if (g_elect()) {
#pragma unroll
                for (int ks = 0; ks < 4; ks++) {
                    const uint64_t bd = g_desc(st + 3 * RT_PLANE + ks * 32);
#pragma unroll
                    for (int p = 0; p < 3; p++)
                        g_mma_ss(d, g_desc(st + p * RT_PLANE + ks * 32), bd, idesc, (ks | p) != 0);
                }
                g_commit(g_smem(&empty[s]));
                g_commit(g_smem(&acc_full[b]));
            }
            __syncwarp();
        }
        if (g_elect()) g_commit(g_smem(&done));     // drains the MMAs in flight
        __syncwarp();
        if (lane == 0) g_drain_wait(g_smem(&done), 0);
        __syncwarp();
    } else {
        // warps 0-3: add every stage's partial logits into fp32 registers;
        // thread (warp w, lane l) holds expert m0 + 32w + l for the tile's 64 tokens
        float acc[RT_BN];
#pragma unroll
        for (int j = 0; j < RT_BN; j++) acc[j] = 0.f;
        const uint32_t taddr = tmem + (uint32_t(warp * 32) << 16);
        bool ok = true;
        for (int kb = 0; kb < KB; kb++) {
            const int b = kb & 1;
            if (!g_wait_w(g_smem(&acc_full[b]), (kb >> 1) & 1, &s_ab, 32)) {
                ok = false;
                break;
            }
            g_fence_after();
#pragma unroll
            for (int c = 0; c < RT_BN; c += 16) {
                uint32_t v[16];
                g_ld16(taddr + b * RT_BN + c, v);
                g_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; j++) acc[c + j] += __uint_as_float(v[j]);
            }
            g_fence_before();
            __syncwarp();
            if (lane == 0) g_arrive(g_smem(&acc_empty[b]));
        }
        if (ok) {
            const int e = m0 + warp * 32 + lane;
#pragma unroll
            for (int j = 0; j < RT_BN; j++) {
                const int t = n0 + j;
                if (t < a.T && e < a.E) a.logits[size_t(t) * a.E + e] = acc[j];
            }
        } else {
            fail();
        }
    }
    g_fence_before();
    __syncthreads();
    g_fence_after();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 128;" ::"r"(tmem));
}

// Wr (fp32, n elements) -> planes[0..2][n] bf16 with Wr = hi + mid + lo (round to nearest at each step).
__global__ void __launch_bounds__(256) router_split(const float4* __restrict__ w, size_t n4,
                                                    __nv_bfloat16* __restrict__ planes) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const size_t n = n4 * 4;
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += size_t(gridDim.x) * blockDim.x) {
        const float4 v = w[i];
        const float f[4] = {v.x, v.y, v.z, v.w};
        __nv_bfloat16 hi[4], mid[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; j++) {
            hi[j] = __float2bfloat16_rn(f[j]);
            const float r1 = f[j] - __bfloat162float(hi[j]);          // exact
            mid[j] = __float2bfloat16_rn(r1);
            lo[j] = __float2bfloat16_rn(r1 - __bfloat162float(mid[j]));   // exact subtraction
        }
        *reinterpret_cast<uint2*>(planes + 4 * i) = *reinterpret_cast<uint2*>(hi);
        *reinterpret_cast<uint2*>(planes + n + 4 * i) = *reinterpret_cast<uint2*>(mid);
        *reinterpret_cast<uint2*>(planes + 2 * n + 4 * i) = *reinterpret_cast<uint2*>(lo);
    }
}

static int rt_launch(const RtArgs& a, cudaStream_t s) {
    constexpr int smem = RT_STAGES * RT_STAGE + 1024;
    if (cudaFuncSetAttribute(router_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return MOE_ERR_CUDA;
    dim3 grid((a.E + RT_M - 1) / RT_M, (a.T + RT_BN - 1) / RT_BN);
    return launch_pdl(router_tc, grid, dim3(RT_THREADS), size_t(smem), s, a) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_router_logits_tc(const __nv_bfloat16* x, int T, int H, const float* Wr, int E, float* logits,
                            __nv_bfloat16* planes, int32_t* status, cudaStream_t s) {
    if (H % 64 || T <= 0 || E <= 0) return MOE_ERR_UNSUPPORTED;
    if (int rc = g_encoder(); rc != MOE_OK) return rc;
    const size_t n = size_t(E) * H;
    router_split<<<std::min<size_t>((n / 4 + 255) / 256, 148 * 8), 256, 0, s>>>(
        reinterpret_cast<const float4*>(Wr), n / 4, planes);
    count_launch();
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    RtArgs a;
    memset(&a, 0, sizeof(a));
    int rc = g_map(&a.tm_w, true, planes, uint64_t(H), uint64_t(3) * E, uint64_t(H) * 2, 64, RT_M, true);
    if (rc == MOE_OK) rc = g_map(&a.tm_x, true, x, uint64_t(H), uint64_t(T), uint64_t(H) * 2, 64, RT_BN, true);
    if (rc != MOE_OK) return rc;
    a.logits = logits;
    a.status = status;
    a.T = T;
    a.E = E;
    a.H = H;
    return rt_launch(a, s);
}

}  // namespace moe
