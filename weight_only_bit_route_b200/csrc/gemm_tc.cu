// Prefill-shaped grouped GEMM on the 5th-generation tensor cores (tcgen05).
//
// Per expert e with n_e routed rows, gate/up computes
//     G = X_e Wg_e^T, U = X_e Wu_e^T, h = bf16(silu(G) * U)      (K = H)
// and down computes
//     Y = w * (Hp_e Wd_e^T)                                         (K = F)
// with the 4-bit weights dequantised inside the kernel
// ("Step-5-Preview-Int4-g128", Recipe; "Step-5-Preview-NVFP4-Local", Format).
//
// Tiles are swapped (weights are the M = 128 operand, tokens the N operand),
// because an expert sees few tokens (about 47 at 2048 tokens): a tile is
// (expert, n-tile of up to 256 rows, m-tile of 128 weight rows).  A persistent
// CTA per SM walks the tile list (built on the device from expert_offsets).
// For each 64-wide K block all eight warps
//   - dequantise the 128 x 64 weight tile(s) into bf16 (int4: q*s rounded
//     once; NVFP4: e2m1 * e4m3 exactly, in f16 with f16 activations) laid out
//     K-major with the 128-byte swizzle the MMA descriptors expect, and
//   - gather the tile's activation rows into the same layout,
// then one thread issues tcgen05.mma (M = 128, N = tile rows, K = 16, fp32
// accumulation in tensor memory; gate and up are two accumulators sharing the
// activation operand) and tcgen05.commit arrives on the stage's mbarrier.  A
// ring of three stages lets the next blocks be produced while the MMAs run.
// The epilogue reads the accumulators with tcgen05.ld and fuses SwiGLU (gate/up)
// or the routing weight (down); NVFP4 global and activation row scales are
// applied there too.  Waits are bounded (about 2 s) and report MOE_ERR_TIMEOUT.
#include <cuda_fp16.h>

#include <algorithm>
#include <type_traits>

#include "moe_internal.cuh"

namespace moe {

constexpr int TC_BM = 128;
constexpr int TC_BK = 64;
constexpr int TC_BN_MAX = 256;
constexpr int TC_STAGES = 3;
constexpr int TC_THREADS = 256;
constexpr int TC_A_BYTES = TC_BM * TC_BK * 2;          // 16 KB per weight matrix
constexpr int TC_B_BYTES = TC_BN_MAX * TC_BK * 2;      // 32 KB
constexpr int TC_STAGE_BYTES = 2 * TC_A_BYTES + TC_B_BYTES;
constexpr unsigned long long TC_WAIT_NS = 2000000000ull;

struct TcArgs {
    int fmt, gateup, E, out_dim, in_dim, top_k, act_by_token;
    const uint8_t* p0; const uint8_t* s0; const float* g0;
    const uint8_t* p1; const uint8_t* s1; const float* g1;
    const int32_t* offsets;
    const int32_t* row_slot;
    const float* topk_w;        // down: routing weight by slot (nullable)
    const uint8_t* act;         // bf16 rows (int4, bf16) or f16 rows (NVFP4, pre-scaled)
    const float* act_scale;     // NVFP4: activation row scale [act rows]
    __nv_bfloat16* out;
    int32_t* status;
};

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t tc_smem(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ unsigned long long tc_timer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok = 0;
    const unsigned long long t0 = tc_timer();
    while (true) {
        asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
                     : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
        if (ok) return true;
        if (tc_timer() - t0 > TC_WAIT_NS) return false;
    }
}
// K-major operand, 128-byte swizzle, 8-row groups 1024 bytes apart
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr) {
    return uint64_t((saddr >> 4) & 0x3FFF) | (uint64_t(1) << 16) | (uint64_t(64) << 32) | (uint64_t(1) << 46) |
           (uint64_t(2) << 61);
}
// kind::f16 instruction descriptor: fp32 accumulate, A/B bf16 (or f16), K-major, M = 128
__device__ __forceinline__ uint32_t tc_idesc(int n, bool f16) {
    const uint32_t ab = f16 ? 0u : 1u;
    return (1u << 4) | (ab << 7) | (ab << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(TC_BM >> 4) << 24);
}
__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile("{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }"
                 ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
}
__device__ __forceinline__ void tc_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ uint32_t tc_e2m1x2_f16x2(uint32_t byte) {
    uint32_t h;
    asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h) : "r"(byte));
    return h;
}
__device__ __forceinline__ uint32_t tc_e4m3_f16x2(uint32_t byte) {          // {s, s} in f16
    uint32_t h;
    asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h) : "r"(byte | (byte << 8)));
    return h;
}

// byte offset of 16-byte chunk c of row r inside a K-major, 128B-swizzled tile
__device__ __forceinline__ uint32_t tc_swz(int r, int c) {
    return uint32_t((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// ---------------------------------------------------------------------------
// Weight unit: 32 consecutive K elements of one row of one matrix -> 4 chunks
// ---------------------------------------------------------------------------
struct TcWUnit { uint4 w[4]; uint32_t sc; };     // packed weights (int4/NVFP4 use w[0]) and scale bits

template <int FMT>
__device__ __forceinline__ void tc_load_wunit(const TcArgs& a, int mi, size_t wrow, int k, TcWUnit& u) {
    const uint8_t* p = mi ? a.p1 : a.p0;
    const uint8_t* sp = mi ? a.s1 : a.s0;
    if (FMT == MOE_FMT_INT4_G128) {
        u.w[0] = __ldg(reinterpret_cast<const uint4*>(p + wrow * (a.in_dim / 2) + k / 2));
        u.sc = __ldg(reinterpret_cast<const uint16_t*>(sp) + wrow * (a.in_dim / 128) + k / 128);
    } else if (FMT == MOE_FMT_NVFP4) {
        u.w[0] = __ldg(reinterpret_cast<const uint4*>(p + wrow * (a.in_dim / 2) + k / 2));
        u.sc = __ldg(reinterpret_cast<const uint16_t*>(sp + wrow * (a.in_dim / 16) + k / 16));   // two E4M3 bytes
    } else {
        const uint4* q = reinterpret_cast<const uint4*>(p + (wrow * a.in_dim + k) * 2);
        u.w[0] = __ldg(q); u.w[1] = __ldg(q + 1); u.w[2] = __ldg(q + 2); u.w[3] = __ldg(q + 3);
    }
}

// Dequantise a unit and store its 4 chunks (row r, chunks c0..c0+3) into a swizzled tile.
template <int FMT>
__device__ __forceinline__ void tc_store_wunit(uint8_t* tile, int r, int c0, const TcWUnit& u) {
    if (FMT == MOE_FMT_INT4_G128) {
        const __nv_bfloat162 s2 = __bfloat162bfloat162(__ushort_as_bfloat16(static_cast<unsigned short>(u.sc)));
        const __nv_bfloat162 off = __floats2bfloat162_rn(136.f, 136.f);
        const uint32_t ws[4] = {u.w[0].x, u.w[0].y, u.w[0].z, u.w[0].w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const uint32_t w = ws[j];
            uint32_t pr[4];
#pragma unroll
            for (int p = 0; p < 4; p++) {
                // nibbles (p, p+4) -> bf16 {128+u}; minus 136 -> q exactly; times s (one rounding)
                uint32_t v = ((w >> (4 * p)) & 0x000F000Fu) | 0x43004300u;
                __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&v);
                h = __hmul2(__hsub2(h, off), s2);
                pr[p] = *reinterpret_cast<uint32_t*>(&h);
            }
            uint4 o;   // natural order: (x0,x1) (x2,x3) (x4,x5) (x6,x7)
            o.x = __byte_perm(pr[0], pr[1], 0x5410);
            o.y = __byte_perm(pr[2], pr[3], 0x5410);
            o.z = __byte_perm(pr[0], pr[1], 0x7632);
            o.w = __byte_perm(pr[2], pr[3], 0x7632);
            *reinterpret_cast<uint4*>(tile + tc_swz(r, c0 + j)) = o;
        }
    } else if (FMT == MOE_FMT_NVFP4) {
        const uint32_t ws[4] = {u.w[0].x, u.w[0].y, u.w[0].z, u.w[0].w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            uint32_t sv = tc_e4m3_f16x2((u.sc >> (8 * (j >> 1))) & 0xffu);
            const __half2 s2 = *reinterpret_cast<__half2*>(&sv);
            const uint32_t w = ws[j];
            uint32_t o[4];
#pragma unroll
            for (int b = 0; b < 4; b++) {
                uint32_t hv = tc_e2m1x2_f16x2((w >> (8 * b)) & 0xffu);
                __half2 h = __hmul2(*reinterpret_cast<__half2*>(&hv), s2);       // exact
                o[b] = *reinterpret_cast<uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(tile + tc_swz(r, c0 + j)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 4; j++) *reinterpret_cast<uint4*>(tile + tc_swz(r, c0 + j)) = u.w[j];
    }
}

// ---------------------------------------------------------------------------
// Kernel
// ---------------------------------------------------------------------------
template <int FMT>
__global__ void __launch_bounds__(TC_THREADS, 1) tc_grouped_gemm(TcArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[TC_STAGES];
    __shared__ uint32_t s_tmem;
    __shared__ int s_active[kMaxE];
    __shared__ int s_prefix[kMaxE];
    __shared__ int s_wsum[TC_THREADS / 32];
    __shared__ int s_nact, s_total, s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int MT = a.out_dim / TC_BM;
    const int KB = a.in_dim / TC_BK;

    if (tid == 0) {
        for (int s = 0; s < TC_STAGES; s++) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tc_smem(&bars[s])));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_abort = 0;
    }
    if (warp == 0) {   // 512 TMEM columns: gate accumulator at 0, up at 256
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(tc_smem(&s_tmem)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // tile list: active experts, tiles per expert = ceil(n / 256) * MT
    {
        constexpr int PER = kMaxE / TC_THREADS;
        int cnt[PER], nt[PER], local = 0, ltiles = 0;
#pragma unroll
        for (int i = 0; i < PER; i++) {
            const int e = tid * PER + i;
            const int n = (e < a.E) ? a.offsets[e + 1] - a.offsets[e] : 0;
            cnt[i] = n > 0;
            nt[i] = n > 0 ? ((n + TC_BN_MAX - 1) / TC_BN_MAX) * MT : 0;
            local += cnt[i];
            ltiles += nt[i];
        }
        int v = local, w = ltiles;
        for (int o = 1; o < 32; o <<= 1) {
            const int n1 = __shfl_up_sync(0xffffffffu, v, o), n2 = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) { v += n1; w += n2; }
        }
        __shared__ int s_wt[TC_THREADS / 32];
        if (lane == 31) { s_wsum[warp] = v; s_wt[warp] = w; }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        int base = 0, tbase = 0, tot = 0, ttot = 0;
        for (int q = 0; q < TC_THREADS / 32; q++) {
            if (q < warp) { base += s_wsum[q]; tbase += s_wt[q]; }
            tot += s_wsum[q];
            ttot += s_wt[q];
        }
        int pos = base + v - local, tpos = tbase + w - ltiles;
#pragma unroll
        for (int i = 0; i < PER; i++)
            if (cnt[i]) { s_active[pos] = tid * PER + i; s_prefix[pos] = tpos; pos++; tpos += nt[i]; }
        if (tid == 0) { s_nact = tot; s_total = ttot; }
        __syncthreads();
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t tmem = s_tmem;
    const int ntiles = s_total;
    // stage ring on a 1024-byte boundary (128B-swizzle atoms)
    uint8_t* ring = smem + ((1024u - (tc_smem(smem) & 1023u)) & 1023u);
    uint32_t kcount = 0;            // K blocks issued by this CTA (stage / phase counter)

    for (int tile = blockIdx.x; tile < ntiles && !s_abort; tile += gridDim.x) {
        // tile -> (expert, n-tile, m-tile)
        int lo = 0, hi = s_nact - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
        }
        const int e = s_active[lo];
        const int local = tile - s_prefix[lo];
        const int nti = local / MT, m0 = (local % MT) * TC_BM;
        const int ebase = a.offsets[e], n_e = a.offsets[e + 1] - ebase;
        const int ntile = (n_e + TC_BN_MAX - 1) / TC_BN_MAX;
        const int per = (n_e + ntile - 1) / ntile;                 // balanced rows per n-tile
        const int n0 = nti * per;
        const int nval = min(per, n_e - n0);
        const int bn = (nval + 15) & ~15;                            // MMA N: multiple of 16
        const uint32_t idesc = tc_idesc(bn, FMT == MOE_FMT_NVFP4);

        // Register double buffer: the global loads of block kb+1 are issued
        // before block kb is dequantised and stored.  Per thread: up to 2
        // weight units and up to 8 activation chunks per block.
        const int nunits = (a.gateup ? 2 : 1) * TC_BM * 2;
        const int nchunks = bn * 8;
        TcWUnit wu[2][2];
        uint4 xv[2][8];
        auto load_block = [&](int kb, auto bufc) {
            constexpr int buf = decltype(bufc)::value;
            const int k0 = kb * TC_BK;
#pragma unroll
            for (int q = 0; q < 2; q++) {
                const int uidx = tid + q * TC_THREADS;
                if (uidx < nunits) {
                    const int mi = uidx / (TC_BM * 2), rr = (uidx / 2) % TC_BM, half = uidx & 1;
                    tc_load_wunit<FMT>(a, mi, size_t(e) * a.out_dim + m0 + rr, k0 + half * 32, wu[buf][q]);
                }
            }
#pragma unroll
            for (int q = 0; q < 8; q++) {
                const int cidx = tid + q * TC_THREADS;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (cidx < nchunks) {
                    const int n = cidx >> 3, c = cidx & 7;
                    if (n < nval) {
                        const int r = ebase + n0 + n;
                        const int arow = a.act_by_token ? a.row_slot[r] / a.top_k : r;
                        v = __ldg(reinterpret_cast<const uint4*>(a.act + (size_t(arow) * a.in_dim + k0 + c * 8) * 2));
                    }
                }
                xv[buf][q] = v;
            }
        };
        load_block(0, std::integral_constant<int, 0>{});
        auto step = [&](int kb, auto bufc) {
            constexpr int buf = decltype(bufc)::value;
            const int s = kcount % TC_STAGES;
            uint8_t* A0 = ring + s * TC_STAGE_BYTES;
            uint8_t* A1 = A0 + TC_A_BYTES;
            uint8_t* B = A0 + 2 * TC_A_BYTES;
            if (kb + 1 < KB) load_block(kb + 1, std::integral_constant<int, buf ^ 1>{});
            if (kcount >= TC_STAGES && !s_abort) {                  // the MMAs that read this stage are done
                if (!tc_wait(tc_smem(&bars[s]), ((kcount / TC_STAGES) - 1) & 1)) {
                    set_status(a.status, MOE_ERR_TIMEOUT);
                    s_abort = 1;
                }
            }
#pragma unroll
            for (int q = 0; q < 2; q++) {
                const int uidx = tid + q * TC_THREADS;
                if (uidx < nunits) {
                    const int mi = uidx / (TC_BM * 2), rr = (uidx / 2) % TC_BM, half = uidx & 1;
                    tc_store_wunit<FMT>(mi ? A1 : A0, rr, half * 4, wu[buf][q]);
                }
            }
#pragma unroll
            for (int q = 0; q < 8; q++) {
                const int cidx = tid + q * TC_THREADS;
                if (cidx < nchunks) *reinterpret_cast<uint4*>(B + tc_swz(cidx >> 3, cidx & 7)) = xv[buf][q];
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncthreads();
            if (tid == 0 && !s_abort) {
                tc_fence_after();
                const uint32_t a0 = tc_smem(A0), a1 = tc_smem(A1), b0 = tc_smem(B);
#pragma unroll
                for (int ks = 0; ks < TC_BK / 16; ks++) {
                    const uint32_t acc = (kb > 0 || ks > 0) ? 1u : 0u;
                    tc_mma(tmem, tc_desc(a0 + ks * 32), tc_desc(b0 + ks * 32), idesc, acc);
                    if (a.gateup) tc_mma(tmem + 256, tc_desc(a1 + ks * 32), tc_desc(b0 + ks * 32), idesc, acc);
                }
                tc_commit(tc_smem(&bars[s]));
            }
            kcount++;
        };
        for (int kb = 0; kb < KB; kb += 2) {
            step(kb, std::integral_constant<int, 0>{});
            if (kb + 1 < KB) step(kb + 1, std::integral_constant<int, 1>{});
        }
        // epilogue: wait for the tile's last commit, read the accumulators
        {
            const uint32_t last = kcount - 1;
            if (!s_abort && !tc_wait(tc_smem(&bars[last % TC_STAGES]), (last / TC_STAGES) & 1)) {
                set_status(a.status, MOE_ERR_TIMEOUT);
                s_abort = 1;
            }
            tc_fence_after();
            const int quarter = warp & 3, chalf = warp >> 2;
            const int f = m0 + quarter * 32 + lane;            // output feature of this thread
            const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
            float gsc = 1.f, usc = 1.f;
            if (FMT == MOE_FMT_NVFP4) { gsc = a.g0[e]; usc = a.gateup ? a.g1[e] : 1.f; }
            for (int cc = chalf; cc * 16 < bn; cc += 2) {
                uint32_t g[16], uvals[16];
                tc_ld16(tmem + lane_addr + cc * 16, g);
                if (a.gateup) tc_ld16(tmem + 256 + lane_addr + cc * 16, uvals);
                tc_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; j++) {
                    const int n = cc * 16 + j;
                    if (n >= nval) break;
                    const int r = ebase + n0 + n;
                    float rs = 1.f;
                    if (FMT == MOE_FMT_NVFP4) rs = a.act_scale[a.act_by_token ? a.row_slot[r] / a.top_k : r];
                    float v;
                    if (a.gateup) {
                        const float gg = __uint_as_float(g[j]) * gsc * rs, uu = __uint_as_float(uvals[j]) * usc * rs;
                        v = gg / (1.0f + expf(-gg)) * uu;
                    } else {
                        const float wt = a.topk_w ? a.topk_w[a.row_slot[r]] : 1.f;
                        v = wt * (__uint_as_float(g[j]) * gsc * rs);
                    }
                    a.out[size_t(r) * a.out_dim + f] = __float2bfloat16_rn(v);
                }
            }
            tc_fence_before();
            __syncthreads();          // accumulators free for the next tile
        }
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
}

// NVFP4: activations as f16 rows times 2^-e (e >= 0 least with |x| * 2^-e <= 16384), scale 2^e.
__global__ void __launch_bounds__(256) tc_act_f16(const __nv_bfloat16* __restrict__ act, int rows, int in_dim,
                                                  __half* __restrict__ out, float* __restrict__ scale) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= rows) return;
    const __nv_bfloat16* row = act + size_t(warp) * in_dim;
    float amax = 0.f;
    for (int i = lane * 8; i < in_dim; i += 256) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + i);
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))), fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y)))));
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))), fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w)))));
    }
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int e = 0;
    while (e < 126 && ldexpf(amax, -e) > 16384.f) e++;
    const float down = ldexpf(1.f, -e);
    for (int i = lane * 8; i < in_dim; i += 256) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + i);
        __half2 h[4];
        h[0] = __floats2half2_rn(bf16_lo(v.x) * down, bf16_hi(v.x) * down);
        h[1] = __floats2half2_rn(bf16_lo(v.y) * down, bf16_hi(v.y) * down);
        h[2] = __floats2half2_rn(bf16_lo(v.z) * down, bf16_hi(v.z) * down);
        h[3] = __floats2half2_rn(bf16_lo(v.w) * down, bf16_hi(v.w) * down);
        *reinterpret_cast<uint4*>(out + size_t(warp) * in_dim + i) = *reinterpret_cast<uint4*>(h);
    }
    if (lane == 0) scale[warp] = ldexpf(1.f, e);
}

template <int FMT>
static cudaError_t tc_launch(const TcArgs& a, cudaStream_t s) {
    static int sms = 0;
    static bool attr = false;
    auto k = tc_grouped_gemm<FMT>;
    if (sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    const int smem = TC_STAGES * TC_STAGE_BYTES + 1024;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    k<<<sms, TC_THREADS, smem, s>>>(a);
    return cudaGetLastError();
}

static int tc_run(const GemvProblem& p, bool gateup, int act_rows, void* prep_ws, cudaStream_t s) {
    if (p.out_dim % TC_BM || p.in_dim % TC_BK) return MOE_ERR_UNSUPPORTED;
    TcArgs a{};
    a.fmt = p.fmt; a.gateup = gateup; a.E = p.E; a.out_dim = p.out_dim; a.in_dim = p.in_dim;
    a.top_k = p.top_k; a.act_by_token = p.act_by_token;
    a.p0 = reinterpret_cast<const uint8_t*>(p.p0); a.s0 = reinterpret_cast<const uint8_t*>(p.s0); a.g0 = p.g0;
    a.p1 = reinterpret_cast<const uint8_t*>(p.p1); a.s1 = reinterpret_cast<const uint8_t*>(p.s1); a.g1 = p.g1;
    a.offsets = p.offsets; a.row_slot = p.row_slot; a.topk_w = p.topk_w; a.out = p.out; a.status = p.status;
    a.act = reinterpret_cast<const uint8_t*>(p.act);
    if (p.fmt == MOE_FMT_NVFP4) {
        float* scale = reinterpret_cast<float*>(prep_ws);
        __half* act16 = reinterpret_cast<__half*>(reinterpret_cast<uint8_t*>(prep_ws) + align256(size_t(act_rows) * 4));
        tc_act_f16<<<(act_rows * 32 + 255) / 256, 256, 0, s>>>(p.act, act_rows, p.in_dim, act16, scale);
        a.act = reinterpret_cast<const uint8_t*>(act16);
        a.act_scale = scale;
    }
    cudaError_t e;
    if (p.fmt == MOE_FMT_INT4_G128) e = tc_launch<MOE_FMT_INT4_G128>(a, s);
    else if (p.fmt == MOE_FMT_NVFP4) e = tc_launch<MOE_FMT_NVFP4>(a, s);
    else e = tc_launch<MOE_FMT_BF16>(a, s);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_grouped_gemm(const GemvProblem& routed, const GemvProblem* shared, bool gateup, int act_rows,
                        void* prep_ws, int32_t* tile_ws, cudaStream_t s) {
    (void)tile_ws;
    int rc = tc_run(routed, gateup, act_rows, prep_ws, s);
    if (rc != MOE_OK || !shared) return rc;
    const int sh_rows = act_rows;   // the shared expert sees every token (gate/up) or every shared row (down)
    (void)sh_rows;
    return tc_run(*shared, gateup, 0, nullptr, s);
}

}  // namespace moe
