// Sigmoid top-k router ("Step-5-Preview-Spark", At a glance: 352 routed
// experts, top-8, sigmoid router).
//
//   l[t,e] = sum_h x[t,h] * Wr[e,h] (+ bias[e])   fp32
//   s      = 1 / (1 + exp(-l))                     fp32
//   ids    = top_k of s, ties to the lower expert id, by descending s
//   w      = s_sel / sum(s_sel)                     fp32
//
// Two logit kernels: for few tokens (decode) one warp streams one router row
// (16 KB at H = 4096) against every token, so the 5.8 MB of router weights
// are read once across ~100 CTAs; for many tokens a register-tiled fp32 SIMT
// GEMM.  A warp-per-token kernel then does the sigmoid, selection and
// renormalisation.
#include "moe_internal.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Logits, few tokens: warp per expert, NT tokens per pass.
// ---------------------------------------------------------------------------
template <int NT>
__global__ void __launch_bounds__(256) router_logits_rows(
        const __nv_bfloat16* __restrict__ x, int T, int H, const float* __restrict__ Wr, int E,
        float* __restrict__ logits) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * (blockDim.x >> 5) + warp;
    const int t0 = blockIdx.y * NT;
    if (e >= E) return;
    const float* wrow = Wr + size_t(e) * H;
    float acc[NT];
#pragma unroll
    for (int i = 0; i < NT; i++) acc[i] = 0.f;
    // lane covers h = 8*lane + 256*i .. +8
    for (int h = lane * 8; h < H; h += 256) {
        const float4 w0 = __ldg(reinterpret_cast<const float4*>(wrow + h));
        const float4 w1 = __ldg(reinterpret_cast<const float4*>(wrow + h + 4));
#pragma unroll
        for (int i = 0; i < NT; i++) {
            if (t0 + i < T) {
                const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + size_t(t0 + i) * H + h));
                float a = acc[i];
                a = fmaf(bf16_lo(xv.x), w0.x, a); a = fmaf(bf16_hi(xv.x), w0.y, a);
                a = fmaf(bf16_lo(xv.y), w0.z, a); a = fmaf(bf16_hi(xv.y), w0.w, a);
                a = fmaf(bf16_lo(xv.z), w1.x, a); a = fmaf(bf16_hi(xv.z), w1.y, a);
                a = fmaf(bf16_lo(xv.w), w1.z, a); a = fmaf(bf16_hi(xv.w), w1.w, a);
                acc[i] = a;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NT; i++) {
        float v = warp_sum(acc[i], 32);
        if (lane == 0 && t0 + i < T) logits[size_t(t0 + i) * E + e] = v;
    }
}

// ---------------------------------------------------------------------------
// Logits, many tokens: 64 x 64 output tile per CTA, 256 threads, 4 x 4 per
// thread, K step 32, operands staged in shared memory as fp32.
// ---------------------------------------------------------------------------
constexpr int RT_BM = 64, RT_BN = 64, RT_BK = 32;

__global__ void __launch_bounds__(256) router_logits_tiled(
        const __nv_bfloat16* __restrict__ x, int T, int H, const float* __restrict__ Wr, int E,
        float* __restrict__ logits) {
    __shared__ float xs[RT_BK][RT_BM + 4];
    __shared__ float ws[RT_BK][RT_BN + 4];
    const int tid = threadIdx.x;
    const int m0 = blockIdx.y * RT_BM, n0 = blockIdx.x * RT_BN;
    const int tm = (tid / 16) * 4, tn = (tid % 16) * 4;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < H; k0 += RT_BK) {
        // x tile: 64 rows x 32 k = 2048 bf16; each thread loads 8 (one uint4)
        {
            int r = tid / 4, c = (tid % 4) * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (m0 + r < T) v = __ldg(reinterpret_cast<const uint4*>(x + size_t(m0 + r) * H + k0 + c));
            xs[c + 0][r] = bf16_lo(v.x); xs[c + 1][r] = bf16_hi(v.x);
            xs[c + 2][r] = bf16_lo(v.y); xs[c + 3][r] = bf16_hi(v.y);
            xs[c + 4][r] = bf16_lo(v.z); xs[c + 5][r] = bf16_hi(v.z);
            xs[c + 6][r] = bf16_lo(v.w); xs[c + 7][r] = bf16_hi(v.w);
        }
        // Wr tile: 64 experts x 32 k fp32; each thread loads 8 (two float4)
        {
            int r = tid / 4, c = (tid % 4) * 8;
            float4 a = make_float4(0, 0, 0, 0), b = a;
            if (n0 + r < E) {
                a = __ldg(reinterpret_cast<const float4*>(Wr + size_t(n0 + r) * H + k0 + c));
                b = __ldg(reinterpret_cast<const float4*>(Wr + size_t(n0 + r) * H + k0 + c + 4));
            }
            ws[c + 0][r] = a.x; ws[c + 1][r] = a.y; ws[c + 2][r] = a.z; ws[c + 3][r] = a.w;
            ws[c + 4][r] = b.x; ws[c + 5][r] = b.y; ws[c + 6][r] = b.z; ws[c + 7][r] = b.w;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < RT_BK; kk++) {
            const float4 av = *reinterpret_cast<const float4*>(&xs[kk][tm]);
            const float4 bv = *reinterpret_cast<const float4*>(&ws[kk][tn]);
            const float a[4] = {av.x, av.y, av.z, av.w};
            const float b[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < 4; i++)
#pragma unroll
                for (int j = 0; j < 4; j++) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) {
            int t = m0 + tm + i, e = n0 + tn + j;
            if (t < T && e < E) logits[size_t(t) * E + e] = acc[i][j];
        }
}

// ---------------------------------------------------------------------------
// Sigmoid + top-k + renormalisation: warp per token.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) router_topk(
        const float* __restrict__ logits, const float* __restrict__ bias, int T, int E, int k,
        int32_t* __restrict__ ids, float* __restrict__ wout) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + warp;
    if (t >= T) return;
    constexpr int PER = kMaxE / 32;
    float s[PER];
#pragma unroll
    for (int i = 0; i < PER; i++) {
        int e = lane + 32 * i;
        float v = -INFINITY;
        if (e < E) {
            float l = logits[size_t(t) * E + e];
            if (bias) l = l + bias[e];
            v = 1.0f / (1.0f + expf(-l));
        }
        s[i] = v;
    }
    float sel[kMaxTopK];
    int sel_id[kMaxTopK];
    float sum = 0.f;
    for (int j = 0; j < k; j++) {
        // local best: largest s, lowest id on ties (ids grow with i)
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < PER; i++) {
            int e = lane + 32 * i;
            if (e < E && (s[i] > bv || (s[i] == bv && e < bi))) { bv = s[i]; bi = e; }
        }
        for (int o = 16; o > 0; o >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        // the owner removes the winner from its candidates
        if ((bi & 31) == lane) {
#pragma unroll
            for (int i = 0; i < PER; i++)
                if (lane + 32 * i == bi) s[i] = -INFINITY;
        }
        sel[j] = bv;
        sel_id[j] = bi;
        sum = sum + bv;
    }
    if (lane == 0) {
        for (int j = 0; j < k; j++) {
            ids[size_t(t) * k + j] = sel_id[j];
            wout[size_t(t) * k + j] = sel[j] / sum;
        }
    }
}

int launch_route(const __nv_bfloat16* x, int T, int H, const float* Wr, const float* bias,
                 int E, int k, int32_t* ids, float* w, float* logits, int32_t* status,
                 cudaStream_t s) {
    (void)status;
    if (T <= 32) {
        dim3 block(256);
        int epb = 8;
        if (T <= 8) {
            dim3 grid((E + epb - 1) / epb, 1);
            router_logits_rows<8><<<grid, block, 0, s>>>(x, T, H, Wr, E, logits);
        } else {
            dim3 grid((E + epb - 1) / epb, (T + 7) / 8);
            router_logits_rows<8><<<grid, block, 0, s>>>(x, T, H, Wr, E, logits);
        }
    } else {
        dim3 grid((E + RT_BN - 1) / RT_BN, (T + RT_BM - 1) / RT_BM);
        router_logits_tiled<<<grid, 256, 0, s>>>(x, T, H, Wr, E, logits);
    }
    router_topk<<<(T + 7) / 8, 256, 0, s>>>(logits, bias, T, E, k, ids, w);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
