// Sigmoid top-k router ("Step-5-Preview-Spark", At a glance: a sigmoid router
// keeps 8 of the 352 routed experts per token).
//
//   l[t,e] = sum_h x[t,h] * Wr[e,h] (+ bias[e])   fp32
//   s      = 1 / (1 + exp(-l))                     fp32
//   ids    = top_k of s, ties to the lower expert id, by descending s
//   w      = s_sel / sum(s_sel)                     fp32
//
// Decode (T <= 16): one fused kernel, see router_decode below.  Otherwise two
// logit kernels (warp per router row for T <= 32, a register-tiled fp32 SIMT
// GEMM above) and a warp-per-token kernel for the sigmoid, selection and
// renormalisation.
#include <algorithm>
#include <mutex>

#include "moe_internal.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Logits, few tokens: warp per expert, NT tokens per pass.
// ---------------------------------------------------------------------------
template <int NT, bool F16>
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
                a = fmaf(act_lo<F16>(xv.x), w0.x, a); a = fmaf(act_hi<F16>(xv.x), w0.y, a);
                a = fmaf(act_lo<F16>(xv.y), w0.z, a); a = fmaf(act_hi<F16>(xv.y), w0.w, a);
                a = fmaf(act_lo<F16>(xv.z), w1.x, a); a = fmaf(act_hi<F16>(xv.z), w1.y, a);
                a = fmaf(act_lo<F16>(xv.w), w1.z, a); a = fmaf(act_hi<F16>(xv.w), w1.w, a);
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

template <bool F16>
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
            xs[c + 0][r] = act_lo<F16>(v.x); xs[c + 1][r] = act_hi<F16>(v.x);
            xs[c + 2][r] = act_lo<F16>(v.y); xs[c + 3][r] = act_hi<F16>(v.y);
            xs[c + 4][r] = act_lo<F16>(v.z); xs[c + 5][r] = act_hi<F16>(v.z);
            xs[c + 6][r] = act_lo<F16>(v.w); xs[c + 7][r] = act_hi<F16>(v.w);
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
// Sigmoid + top-k + renormalisation for one token, by one warp.  PER is the
// number of experts each lane holds (ceil(E / 32) rounded to a supported size).
// Each expert is a 64-bit key: the score's bits (s >= 0, so they order like the
// score) above the complement of its id (so equal scores prefer the lower id);
// 0 marks an empty or taken slot.  A lane keeps the largest of its keys; a pick
// is one warp-wide maximum, after which only the lane that owned the winner
// rescans its keys.  STAGED: lrow holds the scores s themselves (sigmoid of
// the biased logits, computed where the logits were), in shared memory, and
// the ids also go to ids_s.
// ---------------------------------------------------------------------------
template <int PER, bool STAGED = false>
__device__ __forceinline__ void topk_warp(const float* __restrict__ lrow, const float* __restrict__ bias, int E,
                                          int k, int32_t* __restrict__ ids, float* __restrict__ wout, int lane,
                                          int32_t* ids_s = nullptr) {
    unsigned long long key[PER];
#pragma unroll
    for (int i = 0; i < PER; i++) {
        const int e = lane + 32 * i;
        key[i] = 0ull;
        if (e < E) {
            float v;
            if constexpr (STAGED) {
                v = lrow[e];
            } else {
                float l = lrow[e];
                if (bias) l = l + bias[e];
                v = 1.0f / (1.0f + expf(-l));
            }
            key[i] = (static_cast<unsigned long long>(__float_as_uint(v)) << 32) | static_cast<uint32_t>(~e);
        }
    }
    unsigned long long lmax = 0ull;
#pragma unroll
    for (int i = 0; i < PER; i++) lmax = key[i] > lmax ? key[i] : lmax;
    float sum = 0.f, my_s = 0.f;
    int my_id = 0;
    for (int j = 0; j < k; j++) {
        unsigned long long m = lmax;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long om = __shfl_xor_sync(0xffffffffu, m, o);
            m = om > m ? om : m;
        }
        const int bi = static_cast<int>(~static_cast<uint32_t>(m));
        const float bv = __uint_as_float(static_cast<uint32_t>(m >> 32));
        if ((bi & 31) == lane) {
            lmax = 0ull;
#pragma unroll
            for (int i = 0; i < PER; i++) {
                if (i == (bi >> 5)) key[i] = 0ull;
                lmax = key[i] > lmax ? key[i] : lmax;
            }
        }
        if (lane == j) { my_s = bv; my_id = bi; }
        sum = sum + bv;
    }
    if (lane < k) {
        ids[lane] = my_id;
        wout[lane] = my_s / sum;
        if constexpr (STAGED) ids_s[lane] = my_id;
    }
}

__global__ void __launch_bounds__(256) router_topk(
        const float* __restrict__ logits, const float* __restrict__ bias, int T, int E, int k,
        int32_t* __restrict__ ids, float* __restrict__ wout) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + warp;
    if (t >= T) return;
    if (E <= 384) topk_warp<12>(logits + size_t(t) * E, bias, E, k, ids + size_t(t) * k, wout + size_t(t) * k, lane);
    else topk_warp<kMaxE / 32>(logits + size_t(t) * E, bias, E, k, ids + size_t(t) * k, wout + size_t(t) * k, lane);
}

// ---------------------------------------------------------------------------
// Fused decode router (T <= 16).  Each CTA takes two experts, a warp per
// quarter of H of one of them, against every token's activations (staged once
// per CTA in shared memory), and writes the two experts' scores
// s = sigmoid(l + b); the router weights are read once in total.  The last CTA
// to finish (an arrival counter in the workspace, no waiting; it leaves the
// counter at zero for the next call) stages all scores in shared memory and
// does the top-k of every token, the stable bucketing of the T*k slots and
// the shared expert's routing.
// ---------------------------------------------------------------------------
constexpr unsigned long long kRouterWaitNs = 2000000000ull;   // default bound of a wait
// Bound on the fused router's wait: words 4-5 of the workspace control block
// (moe_set_wait_limit), 0 = the default.  Read after griddepcontrol.wait.
__device__ __forceinline__ unsigned long long router_wait_limit(const int32_t* status) {
    if (!status) return kRouterWaitNs;
    const unsigned long long v = *reinterpret_cast<const volatile unsigned long long*>(status + 4);
    return v ? v : kRouterWaitNs;
}
constexpr int RD_WARPS = 8;          // 2 experts x 4 quarters of H per CTA
constexpr int RD_EPC = 2;            // experts per CTA
constexpr int RD_TMAX = 16;          // tokens (kRouterDecodeMaxT)

template <bool F16>
__global__ void __launch_bounds__(RD_WARPS * 32) router_decode(RouterDecodeArgs a) {
    extern __shared__ __align__(16) uint8_t rsm[];
    __shared__ int s_last;
    __shared__ float s_part[RD_EPC][4][RD_TMAX];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int el = warp >> 2, kq = warp & 3;                 // expert of the CTA, quarter of H
    const int e = blockIdx.x * RD_EPC + el;
    const int hq = a.H / 4;                                  // elements per quarter (a multiple of 32)
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(rsm);
    __shared__ __align__(8) uint64_t bar;
    const uint32_t bar_a = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
    const uint32_t xs_a = static_cast<uint32_t>(__cvta_generic_to_shared(xs));
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_a));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");      // x may come from the previous kernel
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0) {                                  // all token rows, one bulk copy
        const uint32_t bytes = uint32_t(a.T) * a.H * 2;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_a), "r"(bytes) : "memory");
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                     ::"r"(xs_a), "l"(a.x), "r"(bytes), "r"(bar_a) : "memory");
    }
    // this warp's quarter of its router row: every load issued before any math
    const float* wq = a.Wr + size_t(e < a.E ? e : 0) * a.H + kq * hq;
    float4 wv[8];
    const int nq = hq / 128;                                 // float4 steps of the warp (8 at H = 4096)
#pragma unroll
    for (int q = 0; q < 8; q++)
        wv[q] = (q < nq) ? __ldg(reinterpret_cast<const float4*>(wq + q * 128 + lane * 4)) : make_float4(0, 0, 0, 0);
    {   // activations landed (bounded wait; the bound comes from the workspace control block)
        const unsigned long long limit = router_wait_limit(a.status);
        uint32_t ok = 0;
        unsigned long long t_start, t_now;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_start));
        while (!ok) {
            asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0; selp.u32 %0, 1, 0, p; }"
                         : "=r"(ok) : "r"(bar_a) : "memory");
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_now));
            if (!ok && t_now - t_start > limit) {
                set_status(a.status, MOE_ERR_TIMEOUT);
                // the copy is still in flight: wait for it (at most the default bound) before this
                // CTA's shared memory is read or released
                while (!ok) {
                    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0; selp.u32 %0, 1, 0, p; }"
                                 : "=r"(ok) : "r"(bar_a) : "memory");
                    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_now));
                    if (t_now - t_start > kRouterWaitNs) break;
                }
                break;
            }
        }
    }
    float acc[RD_TMAX];
#pragma unroll
    for (int t = 0; t < RD_TMAX; t++) acc[t] = 0.f;
#pragma unroll
    for (int q = 0; q < 8; q++) {
        if (q < nq) {
            const int h = kq * hq + q * 128 + lane * 4;
#pragma unroll
            for (int t = 0; t < RD_TMAX; t++) {
                if (t < a.T) {
                    const uint2 xv = *reinterpret_cast<const uint2*>(xs + t * a.H + h);
                    float v = acc[t];
                    v = fmaf(act_lo<F16>(xv.x), wv[q].x, v); v = fmaf(act_hi<F16>(xv.x), wv[q].y, v);
                    v = fmaf(act_lo<F16>(xv.y), wv[q].z, v); v = fmaf(act_hi<F16>(xv.y), wv[q].w, v);
                    acc[t] = v;
                }
            }
        }
    }
    // larger H: the rest of the quarter, 4 floats per lane per step
    for (int h0 = 8 * 128; h0 < hq; h0 += 128) {
        const float4 w4 = __ldg(reinterpret_cast<const float4*>(wq + h0 + lane * 4));
        const int h = kq * hq + h0 + lane * 4;
#pragma unroll
        for (int t = 0; t < RD_TMAX; t++) {
            if (t < a.T) {
                const uint2 xv = *reinterpret_cast<const uint2*>(xs + t * a.H + h);
                float v = acc[t];
                v = fmaf(act_lo<F16>(xv.x), w4.x, v); v = fmaf(act_hi<F16>(xv.x), w4.y, v);
                v = fmaf(act_lo<F16>(xv.y), w4.z, v); v = fmaf(act_hi<F16>(xv.y), w4.w, v);
                acc[t] = v;
            }
        }
    }
#pragma unroll
    for (int t = 0; t < RD_TMAX; t++) {
        if (t < a.T) {                                       // uniform: only the tokens present
            const float v = warp_sum(acc[t], 32);
            if (lane == 0) s_part[el][kq][t] = v;
        }
    }
    __syncthreads();
    // quarters in a fixed order; the CTA's experts' scores s = sigmoid(l + b) go out (into the
    // logits region) for the last CTA's selection
    for (int i = threadIdx.x; i < RD_EPC * a.T; i += blockDim.x) {
        const int ee = i / a.T, t = i % a.T, eg = blockIdx.x * RD_EPC + ee;
        if (eg < a.E) {
            float l = ((s_part[ee][0][t] + s_part[ee][1][t]) + s_part[ee][2][t]) + s_part[ee][3][t];
            if (a.bias) l = l + a.bias[eg];
            a.logits[size_t(t) * a.E + eg] = 1.0f / (1.0f + expf(-l));
        }
    }
    // last CTA to arrive continues: the CTA's stores are ordered before its arrival by the barrier
    // and thread 0's release fence; the last CTA acquires everyone's before it reads them
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("fence.acq_rel.gpu;" ::: "memory");
        const int last = atomicAdd(a.counter, 1) == int(gridDim.x) - 1;
        if (last) asm volatile("fence.acq_rel.gpu;" ::: "memory");
        s_last = last;
    }
    __syncthreads();
    if (!s_last) return;
    // Every token's scores (written by the other CTAs: read at L2) into shared memory, each
    // thread's loads all issued before its stores, so the tail waits for one round of loads
    float* lg = reinterpret_cast<float*>(rsm);               // [T][E] (x staging is no longer needed)
    int32_t* ids_s = reinterpret_cast<int32_t*>(lg + a.T * a.E);   // [T][k]
    int32_t* cnt = ids_s + a.T * a.k;                        // [E]
    {
        constexpr int LPT = 16;
        const int n = a.T * a.E;
        for (int i0 = 0; i0 < n; i0 += LPT * RD_WARPS * 32) {
            float v[LPT];
#pragma unroll
            for (int j = 0; j < LPT; j++) {
                const int i = i0 + j * RD_WARPS * 32 + threadIdx.x;
                v[j] = i < n ? __ldcg(a.logits + i) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < LPT; j++) {
                const int i = i0 + j * RD_WARPS * 32 + threadIdx.x;
                if (i < n) lg[i] = v[j];
            }
        }
    }
    __syncthreads();
    for (int t = warp; t < a.T; t += RD_WARPS) {
        if (a.E <= 384)
            topk_warp<12, true>(lg + t * a.E, nullptr, a.E, a.k, a.ids + size_t(t) * a.k, a.w + size_t(t) * a.k,
                                lane, ids_s + t * a.k);
        else
            topk_warp<kMaxE / 32, true>(lg + t * a.E, nullptr, a.E, a.k, a.ids + size_t(t) * a.k,
                                        a.w + size_t(t) * a.k, lane, ids_s + t * a.k);
    }
    if (threadIdx.x == 0) *a.counter = 0;
    if (a.sh_offsets) {
        if (threadIdx.x == 0) { a.sh_offsets[0] = 0; a.sh_offsets[1] = a.T; }
        for (int i = threadIdx.x; i < a.T; i += blockDim.x) a.sh_rowslot[i] = i * a.k;
    }
    if (!a.offsets) return;
    __syncthreads();                       // ids of every token in ids_s
    // stable counting sort of the R <= T * k slots by expert id
    __shared__ int s_wsum[RD_WARPS];
    const int R = a.T * a.k;
    for (int i = threadIdx.x; i < a.E; i += blockDim.x) cnt[i] = 0;
    __syncthreads();
    for (int sl = threadIdx.x; sl < R; sl += blockDim.x) {
        const int id = ids_s[sl];
        if (id >= 0 && id < a.E) atomicAdd(&cnt[id], 1);
        else set_status(a.status, MOE_ERR_DEVICE_INDEX);
    }
    __syncthreads();
    // exclusive scan of cnt over E: each thread a contiguous run of experts
    const int per = (a.E + blockDim.x - 1) / blockDim.x;
    const int b0 = threadIdx.x * per, b1 = min(a.E, b0 + per);
    int local = 0;
    for (int i = b0; i < b1; i++) local += cnt[i];
    int v = local;
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) s_wsum[warp] = v;
    __syncthreads();
    int base = 0;
    for (int q = 0; q < warp; q++) base += s_wsum[q];
    int run = base + v - local;
    for (int i = b0; i < b1; i++) {
        const int c = cnt[i];
        a.offsets[i] = run;
        cnt[i] = run;                        // becomes the next free row of expert i
        run += c;
    }
    if (threadIdx.x == blockDim.x - 1) a.offsets[a.E] = base + v;
    __syncthreads();
    if (warp == 0) {
        const unsigned lt = (1u << lane) - 1u;
        for (int s0 = 0; s0 < R; s0 += 32) {
            const int sl = s0 + lane;
            const int id = (sl < R) ? ids_s[sl] : -1;
            const bool ok = id >= 0 && id < a.E;
            const unsigned act = __ballot_sync(0xffffffffu, ok);
            const unsigned peers = __match_any_sync(0xffffffffu, ok ? id : -1) & act;
            int pos = 0;
            if (ok) pos = cnt[id] + __popc(peers & lt);
            __syncwarp();
            if (ok && (__ffs(peers) - 1) == lane) cnt[id] += __popc(peers);
            __syncwarp();
            if (sl < R) {
                if (ok) { a.row_slot[pos] = sl; a.slot_row[sl] = pos; }
                else a.slot_row[sl] = -1;
            }
        }
    }
}

int launch_route_decode(const RouterDecodeArgs& a, cudaStream_t s) {
    // x staging, then (the last CTA) scores, ids and the bucket counters
    const size_t smem = std::max<size_t>(size_t(a.T) * a.H * 2, (size_t(a.T) * a.E + size_t(a.E) + size_t(a.T) * a.k) * 4);
    if (a.T > RD_TMAX || a.H % 512) return MOE_ERR_UNSUPPORTED;
    auto k = a.x_f16 ? router_decode<true> : router_decode<false>;
    // the attribute is set to this call's size and the launch follows under one lock, so that another host
    // thread cannot lower it in between
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
        return MOE_ERR_UNSUPPORTED;
    return launch_pdl(k, dim3((a.E + RD_EPC - 1) / RD_EPC), dim3(RD_WARPS * 32), smem, s, a) == cudaSuccess
               ? MOE_OK : MOE_ERR_CUDA;
}

int launch_route(const __nv_bfloat16* x, int T, int H, const float* Wr, const float* bias,
                 int E, int k, int32_t* ids, float* w, float* logits, __nv_bfloat16* planes,
                 int32_t* status, int32_t* counter, cudaStream_t s, int x_f16) {
    if (T <= kRouterDecodeMaxT && counter && router_decode_ok(H)) {
        RouterDecodeArgs a{};
        a.x = x; a.T = T; a.H = H; a.Wr = Wr; a.bias = bias; a.E = E; a.k = k;
        a.logits = logits; a.ids = ids; a.w = w; a.counter = counter; a.status = status; a.x_f16 = x_f16;
        return launch_route_decode(a, s);
    }
    auto rows8 = x_f16 ? router_logits_rows<8, true> : router_logits_rows<8, false>;
    auto tiled = x_f16 ? router_logits_tiled<true> : router_logits_tiled<false>;
    if (T <= 32) {
        dim3 block(256);
        int epb = 8;
        if (T <= 8) {
            dim3 grid((E + epb - 1) / epb, 1);
            rows8<<<grid, block, 0, s>>>(x, T, H, Wr, E, logits);
            count_launch();
        } else {
            dim3 grid((E + epb - 1) / epb, (T + 7) / 8);
            rows8<<<grid, block, 0, s>>>(x, T, H, Wr, E, logits);
            count_launch();
        }
    } else if (T >= kRouterTcMinT && planes && !x_f16) {     // (bf16 planes: x must be bf16)
        const int rc = launch_router_logits_tc(x, T, H, Wr, E, logits, planes, status, s);
        if (rc != MOE_OK) return rc;
    } else {
        dim3 grid((E + RT_BN - 1) / RT_BN, (T + RT_BM - 1) / RT_BM);
        tiled<<<grid, 256, 0, s>>>(x, T, H, Wr, E, logits);
        count_launch();
    }
    router_topk<<<(T + 7) / 8, 256, 0, s>>>(logits, bias, T, E, k, ids, w);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
