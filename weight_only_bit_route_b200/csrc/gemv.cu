// Decode-shaped grouped GEMV over 4-bit expert weights.
//
// For every expert with at least one routed row the kernel streams that
// expert's packed weights once (128-bit loads, no L1 allocation), dequantises
// them in registers and multiplies them with the expert's few activation rows
// (staged in shared memory).  Only touched experts are read; the list of
// touched experts is built on the device from expert_offsets, so no host
// round trip is needed.
//
// Work: item = (touched expert, block of output rows).  A CTA of 8 warps takes
// a contiguous range of items (consecutive items usually share an expert, so
// the staged activations are reused).  Inside a warp, groups of LPR lanes own 4
// "row vectors" (gate: 2 rows x {gate, up}; down: 4 rows) and split the
// reduction dimension: lane i of a group handles 16-byte chunks i, i+LPR, ...;
// partial sums meet in a shuffle reduction (split-K within the warp).
//
// Dequantisation in registers:
//   int4   ("Step-5-Preview-Int4-g128", Recipe): nibble u -> the fp32 value
//          128 + u built by one byte permute (bits 0x43 | u << 16), so
//          sum x*q = sum x*(128+u) - 136 * sum x; sum x per 32-element chunk is
//          precomputed when the activations are staged; one bf16 scale per 128.
//   NVFP4  ("Step-5-Preview-NVFP4-Local", Format): E2M1 pairs converted by the
//          hardware cvt to f16x2 (exact), E4M3 block scale per 16, fp32
//          global scale per expert.
//   BF16   (shared expert): bf16 -> fp32 by shifting.
// All products accumulate in fp32.
#include <cuda_fp16.h>

#include <algorithm>

#include "moe_internal.cuh"

namespace moe {

constexpr int GV_THREADS = 256;
constexpr int GV_WARPS = GV_THREADS / 32;
constexpr int GV_RV = 4;     // row vectors per lane group
constexpr int GV_NT = 4;     // activation rows per pass

__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// weights per 16-byte chunk
template <int FMT> struct Kw { static constexpr int v = 32; };
template <> struct Kw<MOE_FMT_BF16> { static constexpr int v = 8; };

struct GvShape {
    int lpr;          // lanes per group
    int ngrp;         // groups per warp
    int rows_grp;     // output rows per group
    int rows_item;    // output rows per CTA item
    int items_per_e;  // items per expert
    int nchunks;      // 16-byte chunks per row
};

__host__ __device__ inline GvShape gv_shape(int fmt, bool gateup, int in_dim, int out_dim) {
    GvShape s;
    const int kw = (fmt == MOE_FMT_BF16) ? 8 : 32;
    s.nchunks = in_dim / kw;
    int lpr = 32;
    while (lpr > 1 && (s.nchunks % lpr) != 0) lpr >>= 1;
    s.lpr = lpr;
    s.ngrp = 32 / lpr;
    s.rows_grp = gateup ? GV_RV / 2 : GV_RV;
    s.rows_item = GV_WARPS * s.ngrp * s.rows_grp;
    s.items_per_e = (out_dim + s.rows_item - 1) / s.rows_item;
    return s;
}

// int4: float 128 + u for byte b of t (t holds 4 nibbles, one per byte)
__device__ __forceinline__ float i4f(uint32_t t, int b) {
    return __uint_as_float(__byte_perm(t, 0x43000000u, 0x7044u | (uint32_t(b) << 8)));
}

__device__ __forceinline__ void e2m1x2_to_f32(uint32_t byte, float& lo, float& hi) {
    uint32_t h;
    asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h) : "r"(byte));
    __half2 hv = *reinterpret_cast<__half2*>(&h);
    float2 f = __half22float2(hv);
    lo = f.x;
    hi = f.y;
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
    uint32_t h;
    asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h) : "r"(byte));
    __half2 hv = *reinterpret_cast<__half2*>(&h);
    return __low2float(hv);
}

struct GvCtx {
    GemvProblem p;
    GvShape sh;
    const uint8_t* xs;    // staged activations (pieces of 16 B)
    const float* xsum;    // [GV_NT][nchunks] (int4 only)
};

// Compute GV_RV row vectors for NP staged activation rows.
template <int FMT, bool GATEUP, int NP>
__device__ __forceinline__ void gv_rows(const GvCtx& c, int e, int row0, int r0,
                                        int lane_g, const uint8_t* __restrict__ rvp[GV_RV],
                                        bool rv_ok[GV_RV], int srow[GV_RV]) {
    constexpr int KW = Kw<FMT>::v;
    constexpr int PIECES = KW / 8;                 // 16-B activation pieces per chunk
    const int nchunks = c.sh.nchunks;
    const int lpr = c.sh.lpr;
    const int cpl = nchunks / lpr;                 // chunks per lane
    float acc[GV_RV][NP];
#pragma unroll
    for (int v = 0; v < GV_RV; v++)
#pragma unroll
        for (int t = 0; t < NP; t++) acc[v][t] = 0.f;

    uint4 cur[GV_RV], nxt[GV_RV];
#pragma unroll
    for (int v = 0; v < GV_RV; v++)
        nxt[v] = rv_ok[v] ? ld_stream(rvp[v] + size_t(lane_g) * 16) : make_uint4(0, 0, 0, 0);

    for (int i = 0; i < cpl; i++) {
        const int ch = lane_g + i * lpr;
#pragma unroll
        for (int v = 0; v < GV_RV; v++) cur[v] = nxt[v];
        if (i + 1 < cpl) {
#pragma unroll
            for (int v = 0; v < GV_RV; v++)
                nxt[v] = rv_ok[v] ? ld_stream(rvp[v] + size_t(ch + lpr) * 16) : make_uint4(0, 0, 0, 0);
        }
        if (FMT == MOE_FMT_INT4_G128) {
            float d[GV_RV][NP];
#pragma unroll
            for (int v = 0; v < GV_RV; v++)
#pragma unroll
                for (int t = 0; t < NP; t++) d[v][t] = 0.f;
#pragma unroll
            for (int j = 0; j < 4; j++) {
                float xv[NP][8];
#pragma unroll
                for (int t = 0; t < NP; t++) {
                    const uint4 xq = *reinterpret_cast<const uint4*>(
                        c.xs + (size_t(t) * PIECES * nchunks + size_t(j) * nchunks + ch) * 16);
                    xv[t][0] = bf16_lo(xq.x); xv[t][1] = bf16_hi(xq.x);
                    xv[t][2] = bf16_lo(xq.y); xv[t][3] = bf16_hi(xq.y);
                    xv[t][4] = bf16_lo(xq.z); xv[t][5] = bf16_hi(xq.z);
                    xv[t][6] = bf16_lo(xq.w); xv[t][7] = bf16_hi(xq.w);
                }
#pragma unroll
                for (int v = 0; v < GV_RV; v++) {
                    const uint32_t w = (j == 0) ? cur[v].x : (j == 1) ? cur[v].y : (j == 2) ? cur[v].z : cur[v].w;
                    const uint32_t t0 = w & 0x0F0F0F0Fu;
                    const uint32_t t1 = (w >> 4) & 0x0F0F0F0Fu;
                    float f[8];
                    f[0] = i4f(t0, 0); f[1] = i4f(t1, 0); f[2] = i4f(t0, 1); f[3] = i4f(t1, 1);
                    f[4] = i4f(t0, 2); f[5] = i4f(t1, 2); f[6] = i4f(t0, 3); f[7] = i4f(t1, 3);
#pragma unroll
                    for (int t = 0; t < NP; t++) {
                        float a = d[v][t];
#pragma unroll
                        for (int m = 0; m < 8; m++) a = fmaf(xv[t][m], f[m], a);
                        d[v][t] = a;
                    }
                }
            }
#pragma unroll
            for (int v = 0; v < GV_RV; v++) {
                float s = 0.f;
                if (rv_ok[v]) {
                    const __nv_bfloat16* sp = reinterpret_cast<const __nv_bfloat16*>(
                        (v & 1) && GATEUP ? c.p.s1 : c.p.s0);
                    s = __bfloat162float(sp[size_t(srow[v]) * (c.p.in_dim / 128) + (ch >> 2)]);
                }
#pragma unroll
                for (int t = 0; t < NP; t++)
                    acc[v][t] = fmaf(s, d[v][t] - 136.f * c.xsum[t * nchunks + ch], acc[v][t]);
            }
        } else if (FMT == MOE_FMT_NVFP4) {
#pragma unroll
            for (int jb = 0; jb < 2; jb++) {       // two blocks of 16 per chunk
                float d[GV_RV][NP];
#pragma unroll
                for (int v = 0; v < GV_RV; v++)
#pragma unroll
                    for (int t = 0; t < NP; t++) d[v][t] = 0.f;
#pragma unroll
                for (int jj = 0; jj < 2; jj++) {
                    const int j = jb * 2 + jj;
                    float xv[NP][8];
#pragma unroll
                    for (int t = 0; t < NP; t++) {
                        const uint4 xq = *reinterpret_cast<const uint4*>(
                            c.xs + (size_t(t) * PIECES * nchunks + size_t(j) * nchunks + ch) * 16);
                        xv[t][0] = bf16_lo(xq.x); xv[t][1] = bf16_hi(xq.x);
                        xv[t][2] = bf16_lo(xq.y); xv[t][3] = bf16_hi(xq.y);
                        xv[t][4] = bf16_lo(xq.z); xv[t][5] = bf16_hi(xq.z);
                        xv[t][6] = bf16_lo(xq.w); xv[t][7] = bf16_hi(xq.w);
                    }
#pragma unroll
                    for (int v = 0; v < GV_RV; v++) {
                        const uint32_t w = (j == 0) ? cur[v].x : (j == 1) ? cur[v].y : (j == 2) ? cur[v].z : cur[v].w;
                        float f[8];
                        e2m1x2_to_f32(w & 0xffu, f[0], f[1]);
                        e2m1x2_to_f32((w >> 8) & 0xffu, f[2], f[3]);
                        e2m1x2_to_f32((w >> 16) & 0xffu, f[4], f[5]);
                        e2m1x2_to_f32(w >> 24, f[6], f[7]);
#pragma unroll
                        for (int t = 0; t < NP; t++) {
                            float a = d[v][t];
#pragma unroll
                            for (int m = 0; m < 8; m++) a = fmaf(xv[t][m], f[m], a);
                            d[v][t] = a;
                        }
                    }
                }
#pragma unroll
                for (int v = 0; v < GV_RV; v++) {
                    float s = 0.f;
                    if (rv_ok[v]) {
                        const uint8_t* sp = reinterpret_cast<const uint8_t*>((v & 1) && GATEUP ? c.p.s1 : c.p.s0);
                        s = e4m3_to_f32(sp[size_t(srow[v]) * (c.p.in_dim / 16) + 2 * ch + jb]);
                    }
#pragma unroll
                    for (int t = 0; t < NP; t++) acc[v][t] = fmaf(s, d[v][t], acc[v][t]);
                }
            }
        } else {   // BF16
            float xv[NP][8];
#pragma unroll
            for (int t = 0; t < NP; t++) {
                const uint4 xq = *reinterpret_cast<const uint4*>(c.xs + (size_t(t) * nchunks + ch) * 16);
                xv[t][0] = bf16_lo(xq.x); xv[t][1] = bf16_hi(xq.x);
                xv[t][2] = bf16_lo(xq.y); xv[t][3] = bf16_hi(xq.y);
                xv[t][4] = bf16_lo(xq.z); xv[t][5] = bf16_hi(xq.z);
                xv[t][6] = bf16_lo(xq.w); xv[t][7] = bf16_hi(xq.w);
            }
#pragma unroll
            for (int v = 0; v < GV_RV; v++) {
                float f[8];
                f[0] = bf16_lo(cur[v].x); f[1] = bf16_hi(cur[v].x);
                f[2] = bf16_lo(cur[v].y); f[3] = bf16_hi(cur[v].y);
                f[4] = bf16_lo(cur[v].z); f[5] = bf16_hi(cur[v].z);
                f[6] = bf16_lo(cur[v].w); f[7] = bf16_hi(cur[v].w);
#pragma unroll
                for (int t = 0; t < NP; t++) {
                    float a = acc[v][t];
#pragma unroll
                    for (int m = 0; m < 8; m++) a = fmaf(xv[t][m], f[m], a);
                    acc[v][t] = a;
                }
            }
        }
    }
    // split-K reduction across the group's lanes
#pragma unroll
    for (int v = 0; v < GV_RV; v++)
#pragma unroll
        for (int t = 0; t < NP; t++) acc[v][t] = warp_sum(acc[v][t], lpr);

    if (lane_g != 0) return;
    if (GATEUP) {
#pragma unroll
        for (int q = 0; q < 2; q++) {
            const int row = row0 + q;
            if (row >= c.p.out_dim) continue;
#pragma unroll
            for (int t = 0; t < NP; t++) {
                float g = acc[2 * q][t], u = acc[2 * q + 1][t];
                if (FMT == MOE_FMT_NVFP4) { g *= c.p.g0[e]; u *= c.p.g1[e]; }
                const float h = g / (1.0f + expf(-g)) * u;
                c.p.out[size_t(r0 + t) * c.p.out_dim + row] = __float2bfloat16_rn(h);
            }
        }
    } else {
#pragma unroll
        for (int t = 0; t < NP; t++) {
            float wt = 1.f;
            if (c.p.topk_w) wt = c.p.topk_w[c.p.row_slot[r0 + t]];
            if (FMT == MOE_FMT_NVFP4) wt *= c.p.g0[e];
#pragma unroll
            for (int q = 0; q < GV_RV; q++) {
                const int row = row0 + q;
                if (row < c.p.out_dim)
                    c.p.out[size_t(r0 + t) * c.p.out_dim + row] = __float2bfloat16_rn(wt * acc[q][t]);
            }
        }
    }
}

template <int FMT, bool GATEUP>
__global__ void __launch_bounds__(GV_THREADS, 2) grouped_gemv(GemvProblem p, GvShape sh) {
    extern __shared__ __align__(16) uint8_t smem[];
    constexpr int KW = Kw<FMT>::v;
    constexpr int PIECES = KW / 8;
    __shared__ int s_active[kMaxE];
    __shared__ int s_nactive;
    __shared__ int s_wsum[GV_WARPS];

    // 1. touched experts, in expert order
    {
        const int tid = threadIdx.x;
        int cnt[kMaxE / GV_THREADS];
        int local = 0;
#pragma unroll
        for (int i = 0; i < kMaxE / GV_THREADS; i++) {
            const int e = tid * (kMaxE / GV_THREADS) + i;
            cnt[i] = (e < p.E) ? (p.offsets[e + 1] > p.offsets[e]) : 0;
            local += cnt[i];
        }
        const int lane = tid & 31, warp = tid >> 5;
        int v = local;
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += n;
        }
        if (lane == 31) s_wsum[warp] = v;
        __syncthreads();
        int base = 0;
        for (int w = 0; w < warp; w++) base += s_wsum[w];
        int pos = base + v - local;
#pragma unroll
        for (int i = 0; i < kMaxE / GV_THREADS; i++) {
            const int e = tid * (kMaxE / GV_THREADS) + i;
            if (cnt[i]) s_active[pos++] = e;
        }
        if (tid == GV_THREADS - 1) s_nactive = base + v;
        __syncthreads();
    }
    const int nact = s_nactive;
    const int total = nact * sh.items_per_e;
    const int per_cta = (total + gridDim.x - 1) / gridDim.x;
    const int i0 = blockIdx.x * per_cta;
    const int i1 = min(total, i0 + per_cta);

    uint8_t* xs = smem;
    float* xsum = reinterpret_cast<float*>(smem + size_t(GV_NT) * p.in_dim * 2);
    GvCtx c{p, sh, xs, xsum};

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = lane / sh.lpr, lane_g = lane % sh.lpr;
    int cur_e = -1, cur_pass = -1;

    for (int it = i0; it < i1; it++) {
        const int a = it / sh.items_per_e;
        const int blk = it % sh.items_per_e;
        const int e = s_active[a];
        const int rbeg = p.offsets[e];
        const int n = p.offsets[e + 1] - rbeg;
        for (int ps = 0; ps < n; ps += GV_NT) {
            const int np = min(GV_NT, n - ps);
            if (e != cur_e || ps != cur_pass) {
                __syncthreads();
                // stage np activation rows as 16-byte pieces: piece (j, ch) -> (j*nchunks + ch)
                const int qpr = p.in_dim / 8;          // pieces per row
                for (int idx = threadIdx.x; idx < np * qpr; idx += GV_THREADS) {
                    const int t = idx / qpr, q = idx % qpr;
                    const int r = rbeg + ps + t;
                    const int arow = p.act_by_token ? (p.row_slot[r] / p.top_k) : r;
                    const uint4 v = *reinterpret_cast<const uint4*>(p.act + size_t(arow) * p.in_dim + q * 8);
                    const int ch = q / PIECES, j = q % PIECES;
                    *reinterpret_cast<uint4*>(xs + (size_t(t) * PIECES * sh.nchunks + size_t(j) * sh.nchunks + ch) * 16) = v;
                }
                __syncthreads();
                if (FMT == MOE_FMT_INT4_G128) {
                    for (int idx = threadIdx.x; idx < np * sh.nchunks; idx += GV_THREADS) {
                        const int t = idx / sh.nchunks, ch = idx % sh.nchunks;
                        float sum = 0.f;
#pragma unroll
                        for (int j = 0; j < PIECES; j++) {
                            const uint4 v = *reinterpret_cast<const uint4*>(
                                xs + (size_t(t) * PIECES * sh.nchunks + size_t(j) * sh.nchunks + ch) * 16);
                            sum += bf16_lo(v.x) + bf16_hi(v.x) + bf16_lo(v.y) + bf16_hi(v.y) +
                                   bf16_lo(v.z) + bf16_hi(v.z) + bf16_lo(v.w) + bf16_hi(v.w);
                        }
                        xsum[t * sh.nchunks + ch] = sum;
                    }
                    __syncthreads();
                }
                cur_e = e;
                cur_pass = ps;
            }
            // this group's rows
            const int row0 = blk * sh.rows_item + (warp * sh.ngrp + grp) * sh.rows_grp;
            const uint8_t* rvp[GV_RV];
            bool ok[GV_RV];
            int srow[GV_RV];
            const size_t row_bytes = (FMT == MOE_FMT_BF16) ? size_t(p.in_dim) * 2 : size_t(p.in_dim) / 2;
#pragma unroll
            for (int v = 0; v < GV_RV; v++) {
                const int row = GATEUP ? row0 + v / 2 : row0 + v;
                const void* base = (GATEUP && (v & 1)) ? p.p1 : p.p0;
                ok[v] = row < p.out_dim;
                srow[v] = e * p.out_dim + (ok[v] ? row : 0);
                rvp[v] = reinterpret_cast<const uint8_t*>(base) + size_t(srow[v]) * row_bytes;
            }
            const int r0 = rbeg + ps;
            switch (np) {
                case 1: gv_rows<FMT, GATEUP, 1>(c, e, row0, r0, lane_g, rvp, ok, srow); break;
                case 2: gv_rows<FMT, GATEUP, 2>(c, e, row0, r0, lane_g, rvp, ok, srow); break;
                case 3: gv_rows<FMT, GATEUP, 3>(c, e, row0, r0, lane_g, rvp, ok, srow); break;
                default: gv_rows<FMT, GATEUP, 4>(c, e, row0, r0, lane_g, rvp, ok, srow); break;
            }
        }
    }
}

template <int FMT, bool GATEUP>
static int launch_gv(const GemvProblem& p, int max_touched, cudaStream_t s) {
    const GvShape sh = gv_shape(FMT, GATEUP, p.in_dim, p.out_dim);
    const size_t smem = size_t(GV_NT) * p.in_dim * 2 + size_t(GV_NT) * sh.nchunks * 4;
    auto kern = grouped_gemv<FMT, GATEUP>;
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
            return MOE_ERR_UNSUPPORTED;
    }
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, GV_THREADS, smem);
    if (per_sm < 1) per_sm = 1;
    const long long items_bound = (long long)std::min(p.E, max_touched) * sh.items_per_e;
    int grid = sms * per_sm;
    if (items_bound < grid) grid = int(items_bound);
    if (grid < 1) grid = 1;
    kern<<<grid, GV_THREADS, smem, s>>>(p, sh);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_grouped_gemv(const GemvProblem& p, bool gateup, int max_touched,
                        cudaStream_t s) {
    switch (p.fmt) {
        case MOE_FMT_INT4_G128:
            return gateup ? launch_gv<MOE_FMT_INT4_G128, true>(p, max_touched, s)
                          : launch_gv<MOE_FMT_INT4_G128, false>(p, max_touched, s);
        case MOE_FMT_NVFP4:
            return gateup ? launch_gv<MOE_FMT_NVFP4, true>(p, max_touched, s)
                          : launch_gv<MOE_FMT_NVFP4, false>(p, max_touched, s);
        case MOE_FMT_BF16:
            return gateup ? launch_gv<MOE_FMT_BF16, true>(p, max_touched, s)
                          : launch_gv<MOE_FMT_BF16, false>(p, max_touched, s);
    }
    return MOE_ERR_UNSUPPORTED;
}

}  // namespace moe
