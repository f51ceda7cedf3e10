// Decode-shaped grouped GEMV over 4-bit expert weights (streaming kernel).
//
// Only experts with at least one routed row are read; their list is built on
// the device from expert_offsets, so no host round trip is needed.  Work is a
// list of items, item = (expert, pass over at most two activation rows, block
// of output rows); an item covers up to ~64 KB of packed weights, so items
// cost about the same and a persistent grid (one CTA per SM) takes a
// contiguous range of them.  The shared expert (BF16 weights) is appended to
// the same item list, so it streams in the same launch.
//
// Per CTA, warp 16 is a producer: for each item it issues TMA bulk copies
// (cp.async.bulk, completion counted on an mbarrier) of the item's weight rows,
// scales, activation rows and activation sums into one stage of a shared-
// memory ring.  Warps 0..15 consume stages: a group of LPT lanes owns a
// (row, K-segment) task and splits its 16-byte chunks; partial sums meet in a
// shuffle reduction (split-K inside the warp) or, when a row's segments belong
// to different warps, in shared memory.  The bytes in flight per SM are the
// ring, not registers.
//
// Dequantisation in registers (products exact, accumulation in fp32):
//   int4   ("Step-5-Preview-Int4-g128", Recipe): nibble pair (m, m+4) of a
//          word becomes bf16x2 {128+u, 128+u'} with one LOP3; fma.rn.f32.bf16
//          multiplies it with the activation pair (x_m, x_m+4), which the
//          pre-pass stored in that order; then sum x*q = sum x*(128+u) -
//          136 * sum x, with sum x per 32-element chunk from the pre-pass;
//          one bf16 scale per 128.
//   NVFP4  ("Step-5-Preview-NVFP4-Local", Format): cvt.rn.f16x2.e2m1x2 gives
//          two exact f16 weights per byte; fma.rn.f32.f16 with f16
//          activations (the pre-pass converts them with a per-row power-of-two
//          scale); E4M3 block scale per 16; fp32 global scale per expert.
//   BF16   (shared expert): fma.rn.f32.bf16 on the raw weights.
// Every mbarrier wait is bounded (about 2 s); on expiry the kernel records
// MOE_ERR_TIMEOUT in the status word and returns.
#include <cuda_fp16.h>

#include <algorithm>
#include <mutex>

#include "moe_internal.cuh"

namespace moe {

constexpr int SV_CONSUMERS = 16;                 // consumer warps
constexpr int SV_GROUPS = 1;                     // consumer groups, taking alternate stages
constexpr int SV_GWARPS = SV_CONSUMERS / SV_GROUPS;
constexpr int SV_THREADS = (SV_CONSUMERS + 1) * 32;
constexpr int SV_NT = 2;                         // activation rows per pass
constexpr int SV_STAGE_TARGET = 64 * 1024;       // weight bytes per item
constexpr int SV_PREFETCH = 0;                   // items prefetched into L2 beyond the ring (measured: no gain)
constexpr int SV_SMEM_MAX = 192 * 1024;          // ring; tables ~24 KB and static ~9 KB follow (227 KB max)
constexpr int SV_META_ROWS = 512;                // rows whose metadata is tabled in shared memory
constexpr int SV_MAX_STAGES = 8;
constexpr unsigned long long SV_WAIT_NS = 2000000000ull;

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ unsigned long long gtimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait: true on completion, false after SV_WAIT_NS.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = gtimer();
    while (!mbar_try(bar, parity))
        if (gtimer() - t0 > SV_WAIT_NS) return false;
    return true;
}
__device__ __forceinline__ void l2_prefetch(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void tma_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}
__device__ __forceinline__ void group_sync(int group) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + group), "n"(SV_GWARPS * 32) : "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// fp32 += bf16 * bf16 on the low / high halves of two packed registers (exact product)
__device__ __forceinline__ float fma_bf16_lo(uint32_t a, uint32_t b, float c) {
    float d;
    asm("{.reg .b16 al, ah, bl, bh; mov.b32 {al, ah}, %1; mov.b32 {bl, bh}, %2; fma.rn.f32.bf16 %0, al, bl, %3;}"
        : "=f"(d) : "r"(a), "r"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float fma_bf16_hi(uint32_t a, uint32_t b, float c) {
    float d;
    asm("{.reg .b16 al, ah, bl, bh; mov.b32 {al, ah}, %1; mov.b32 {bl, bh}, %2; fma.rn.f32.bf16 %0, ah, bh, %3;}"
        : "=f"(d) : "r"(a), "r"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float fma_f16_lo(uint32_t a, uint32_t b, float c) {
    float d;
    asm("{.reg .b16 al, ah, bl, bh; mov.b32 {al, ah}, %1; mov.b32 {bl, bh}, %2; fma.rn.f32.f16 %0, al, bl, %3;}"
        : "=f"(d) : "r"(a), "r"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float fma_f16_hi(uint32_t a, uint32_t b, float c) {
    float d;
    asm("{.reg .b16 al, ah, bl, bh; mov.b32 {al, ah}, %1; mov.b32 {bl, bh}, %2; fma.rn.f32.f16 %0, ah, bh, %3;}"
        : "=f"(d) : "r"(a), "r"(b), "f"(c));
    return d;
}
__device__ __forceinline__ uint32_t e2m1x2_f16x2(uint32_t byte) {
    uint32_t h;
    asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h) : "r"(byte));
    return h;
}
__device__ __forceinline__ float e4m3_f32(uint32_t byte) {
    uint32_t h;
    asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h) : "r"(byte));
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xffffu)));
}

// ---------------------------------------------------------------------------
// Problem description
// ---------------------------------------------------------------------------
struct SvGeom {
    int rv_bytes;      // packed bytes of one row vector
    int sc_bytes;      // scale bytes of one row vector
    int act_bytes;     // bytes of one staged activation row
    int aux_bytes;     // bytes of one row's staged chunk sums (int4)
    int nchunks;       // 16-byte chunks per row vector
    int seg;           // K segments per row
    int cpt;           // chunks per task (= nchunks / seg)
    int lpt;           // lanes per task
    int tpw;           // tasks per warp per item
    int rows_item;     // output rows per item
    int items_per_pass;
};

struct SvBank {
    int fmt, gateup, E, out_dim, in_dim, top_k, act_by_token;
    const uint8_t* p0; const uint8_t* s0; const float* g0;
    const uint8_t* p1; const uint8_t* s1; const float* g1;
    const int32_t* offsets;
    const int32_t* row_slot;
    const uint8_t* act;        // staged activation rows (layout per format, see header)
    const float* act_aux;      // int4: chunk sums [rows, in/32]; nvfp4: row scale [rows]
    const float* topk_w;       // down: weight by slot (nullable)
    __nv_bfloat16* out;
    SvGeom g;
};

struct SvStageLayout {
    int w0, w1, s0, s1, act, aux, red, meta, bytes;
};

// Per-stage item description, written by the producer before it arrives on
// the stage's full barrier (so the consumers see it once the stage is full).
struct SvMeta {
    int bank, e, np, row0, nrows;
    int r[2];          // output rows of the pass
    float wt[2];       // down: routing weight x global scale; gate/up: unused
    float rs[2];       // activation row scale (NVFP4 pre-pass), else 1
    float g0, g1;      // NVFP4 global scales of the expert (gate/up or down)
};

__host__ __device__ inline SvStageLayout sv_layout(const SvGeom& g, int gateup) {
    SvStageLayout L;
    int o = 0;
    auto take = [&](int n) { int r = o; o += (n + 127) & ~127; return r; };
    L.meta = take(int(sizeof(SvMeta)));          // first, at the same offset for every bank
    L.w0 = take(g.rows_item * g.rv_bytes);
    L.w1 = take(gateup ? g.rows_item * g.rv_bytes : 0);
    L.s0 = take(g.rows_item * g.sc_bytes);
    L.s1 = take(gateup ? g.rows_item * g.sc_bytes : 0);
    L.act = take(SV_NT * g.act_bytes);
    L.aux = take(SV_NT * g.aux_bytes);
    L.red = take(SV_GWARPS * SV_NT * 2 * 4);
    L.bytes = o;
    return L;
}

struct SvArgs {
    SvBank b[2];         // [0] routed, [1] shared (E = 0 when absent)
    int stage_bytes;
    int nstages;
    int32_t* status;
};

struct SvItems {
    int n_active;        // routed experts with rows
    int routed_items;
    int total;
    int tabled;          // 1: per-row metadata lives in the shared-memory tables
};

// Metadata tables in shared memory (after the stage ring), filled once in the
// prologue so that the producer's per-item work reads no global memory.
struct SvTables {
    int* eoff;           // [SV_TE] first row of active expert a (bank 0); [kMaxE] bank 1
    int* en;             // [SV_TE] rows of active expert a; [kMaxE] bank 1
    float* g0;           // [kMaxE] NVFP4 global scale (gate or down) of active expert a
    float* g1;           // [kMaxE] NVFP4 global scale (up)
    int* arow0;          // [SV_META_ROWS] activation row of bank-0 row r
    float* wt0;          // [SV_META_ROWS] routing weight of bank-0 row r (1 if none)
    float* rs0;          // [SV_META_ROWS] activation row scale of bank-0 row r
    int* arow1;          // [SV_META_ROWS] activation row of bank-1 row r
};
constexpr int SV_TE = kMaxE + 1;                // per-expert entries; [kMaxE] is bank 1
constexpr int SV_TABLE_BYTES = SV_TE * 4 * 4 + SV_META_ROWS * 4 * 4;

__device__ __forceinline__ SvTables sv_tables(uint8_t* base) {
    SvTables t;
    t.eoff = reinterpret_cast<int*>(base);
    t.en = t.eoff + SV_TE;
    t.g0 = reinterpret_cast<float*>(t.en + SV_TE);
    t.g1 = t.g0 + SV_TE;
    t.arow0 = reinterpret_cast<int*>(t.g1 + SV_TE);
    t.wt0 = reinterpret_cast<float*>(t.arow0 + SV_META_ROWS);
    t.rs0 = t.wt0 + SV_META_ROWS;
    t.arow1 = reinterpret_cast<int*>(t.rs0 + SV_META_ROWS);
    return t;
}

struct SvItem {
    int bank, a, e, r0, np, row0, nrows;     // a: index among active experts (bank 0)
};

// Item i -> (bank, expert, first row of the pass, rows in the pass, output rows)
__device__ __forceinline__ SvItem sv_item(const SvArgs& a, const int* s_active, const int* s_prefix,
                                          const SvTables& tb, const SvItems& it, int i) {
    SvItem m;
    int local, base_row, n;
    if (i < it.routed_items) {
        m.bank = 0;
        int lo = 0, hi = it.n_active - 1;           // largest a with s_prefix[a] <= i
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_prefix[mid] <= i) lo = mid; else hi = mid - 1;
        }
        m.a = lo;
        m.e = s_active[lo];
        local = i - s_prefix[lo];
        base_row = tb.eoff[lo];
        n = tb.en[lo];
    } else {
        m.bank = 1;
        m.a = 0;
        m.e = 0;
        local = i - it.routed_items;
        base_row = tb.eoff[kMaxE];
        n = tb.en[kMaxE];
    }
    const SvBank& b = a.b[m.bank];
    const int pass_idx = local / b.g.items_per_pass;
    const int blk = local - pass_idx * b.g.items_per_pass;
    m.r0 = base_row + pass_idx * SV_NT;
    m.np = min(SV_NT, n - pass_idx * SV_NT);
    m.row0 = blk * b.g.rows_item;
    m.nrows = min(b.g.rows_item, b.out_dim - m.row0);
    return m;
}

// ---------------------------------------------------------------------------
// Consumer math for one (row, segment) task.  NRV row vectors (gate and up, or
// down), NP activation rows.  CPL (chunks per lane), LPT (lanes per task) and
// NCH (chunks per row vector) are compile-time for the layer's own shapes and
// 0 ("read from the geometry") otherwise.
// ---------------------------------------------------------------------------
template <int FMT, int NP, int NRV, int CPL, int LPT, int NCH>
__device__ __forceinline__ void sv_task(const SvBank& b, const uint8_t* st, const SvStageLayout& L, int task_row,
                                        int seg_idx, int lane_t, float acc[2][SV_NT]) {
    const SvGeom& g = b.g;
    const int lpt = LPT ? LPT : g.lpt;
    const int cpl = CPL ? CPL : g.cpt / g.lpt;
    const int nch = NCH ? NCH : g.nchunks;
    const int cpt = CPL ? CPL * LPT : g.cpt;
    const int rvb = NCH ? NCH * 16 : g.rv_bytes;
#pragma unroll
    for (int v = 0; v < 2; v++)
#pragma unroll
        for (int t = 0; t < SV_NT; t++) acc[v][t] = 0.f;
    const int ch0 = seg_idx * cpt + lane_t;                      // first chunk of this lane
    const uint8_t* wr0 = st + L.w0 + size_t(task_row) * rvb + ch0 * 16;
    const uint8_t* wr1 = st + L.w1 + size_t(task_row) * rvb + ch0 * 16;
    const uint8_t* act = st + L.act + ch0 * 16;
    const int abytes = g.act_bytes;
#pragma unroll
    for (int i = 0; i < (CPL ? CPL : 64); i++) {
        if (!CPL && i >= cpl) break;
        const int ch = ch0 + i * lpt;
        uint4 w4[2];
        w4[0] = *reinterpret_cast<const uint4*>(wr0 + i * lpt * 16);
        if (NRV > 1) w4[1] = *reinterpret_cast<const uint4*>(wr1 + i * lpt * 16);
        if (FMT == MOE_FMT_INT4_G128) {
            float d[NRV][NP][2];
#pragma unroll
            for (int v = 0; v < NRV; v++)
#pragma unroll
                for (int t = 0; t < NP; t++) d[v][t][0] = d[v][t][1] = 0.f;
#pragma unroll
            for (int j = 0; j < 4; j++) {
                uint32_t p[NRV][4];
#pragma unroll
                for (int v = 0; v < NRV; v++) {
                    const uint32_t w = (j == 0) ? w4[v].x : (j == 1) ? w4[v].y : (j == 2) ? w4[v].z : w4[v].w;
                    p[v][0] = (w & 0x000F000Fu) | 0x43004300u;             // nibbles (0, 4)
                    p[v][1] = ((w >> 4) & 0x000F000Fu) | 0x43004300u;      // (1, 5)
                    p[v][2] = ((w >> 8) & 0x000F000Fu) | 0x43004300u;      // (2, 6)
                    p[v][3] = ((w >> 12) & 0x000F000Fu) | 0x43004300u;     // (3, 7)
                }
#pragma unroll
                for (int t = 0; t < NP; t++) {
                    // piece j of chunk ch: (x0,x4) (x1,x5) (x2,x6) (x3,x7)
                    const uint4 q = *reinterpret_cast<const uint4*>(act + t * abytes + (j * nch + i * lpt) * 16);
#pragma unroll
                    for (int v = 0; v < NRV; v++) {
                        float s0 = d[v][t][j & 1];
                        s0 = fma_bf16_lo(p[v][0], q.x, s0); s0 = fma_bf16_hi(p[v][0], q.x, s0);
                        s0 = fma_bf16_lo(p[v][1], q.y, s0); s0 = fma_bf16_hi(p[v][1], q.y, s0);
                        s0 = fma_bf16_lo(p[v][2], q.z, s0); s0 = fma_bf16_hi(p[v][2], q.z, s0);
                        s0 = fma_bf16_lo(p[v][3], q.w, s0); s0 = fma_bf16_hi(p[v][3], q.w, s0);
                        d[v][t][j & 1] = s0;
                    }
                }
            }
            const float* xs = reinterpret_cast<const float*>(st + L.aux);
#pragma unroll
            for (int v = 0; v < NRV; v++) {
                const __nv_bfloat16* sc = reinterpret_cast<const __nv_bfloat16*>(
                    st + (v ? L.s1 : L.s0) + size_t(task_row) * g.sc_bytes);
                const float scale = __bfloat162float(sc[ch >> 2]);
#pragma unroll
                for (int t = 0; t < NP; t++)
                    acc[v][t] = fmaf(scale, (d[v][t][0] + d[v][t][1]) - 136.f * xs[t * nch + ch], acc[v][t]);
            }
        } else if (FMT == MOE_FMT_NVFP4) {
#pragma unroll
            for (int blk = 0; blk < 2; blk++) {
                float d[NRV][NP][2];
#pragma unroll
                for (int v = 0; v < NRV; v++)
#pragma unroll
                    for (int t = 0; t < NP; t++) d[v][t][0] = d[v][t][1] = 0.f;
#pragma unroll
                for (int jj = 0; jj < 2; jj++) {
                    const int j = blk * 2 + jj;
                    uint32_t h[NRV][4];
#pragma unroll
                    for (int v = 0; v < NRV; v++) {
                        const uint32_t w = (j == 0) ? w4[v].x : (j == 1) ? w4[v].y : (j == 2) ? w4[v].z : w4[v].w;
                        h[v][0] = e2m1x2_f16x2(w & 0xffu);
                        h[v][1] = e2m1x2_f16x2((w >> 8) & 0xffu);
                        h[v][2] = e2m1x2_f16x2((w >> 16) & 0xffu);
                        h[v][3] = e2m1x2_f16x2(w >> 24);
                    }
#pragma unroll
                    for (int t = 0; t < NP; t++) {
                        const uint4 xv = *reinterpret_cast<const uint4*>(act + t * abytes + (j * nch + i * lpt) * 16);
#pragma unroll
                        for (int v = 0; v < NRV; v++) {
                            float s0 = d[v][t][jj];
                            s0 = fma_f16_lo(h[v][0], xv.x, s0); s0 = fma_f16_hi(h[v][0], xv.x, s0);
                            s0 = fma_f16_lo(h[v][1], xv.y, s0); s0 = fma_f16_hi(h[v][1], xv.y, s0);
                            s0 = fma_f16_lo(h[v][2], xv.z, s0); s0 = fma_f16_hi(h[v][2], xv.z, s0);
                            s0 = fma_f16_lo(h[v][3], xv.w, s0); s0 = fma_f16_hi(h[v][3], xv.w, s0);
                            d[v][t][jj] = s0;
                        }
                    }
                }
#pragma unroll
                for (int v = 0; v < NRV; v++) {
                    const uint8_t* sc = st + (v ? L.s1 : L.s0) + size_t(task_row) * g.sc_bytes;
                    const float sb = e4m3_f32(sc[2 * ch + blk]);
#pragma unroll
                    for (int t = 0; t < NP; t++) acc[v][t] = fmaf(sb, d[v][t][0] + d[v][t][1], acc[v][t]);
                }
            }
        } else {   // BF16: 8 weights per chunk, elements 8ch .. 8ch+7
#pragma unroll
            for (int t = 0; t < NP; t++) {
                const uint4 xv = *reinterpret_cast<const uint4*>(act + t * abytes + i * lpt * 16);
#pragma unroll
                for (int v = 0; v < NRV; v++) {
                    float s0 = 0.f, s1 = 0.f;
                    s0 = fma_bf16_lo(w4[v].x, xv.x, s0); s1 = fma_bf16_hi(w4[v].x, xv.x, s1);
                    s0 = fma_bf16_lo(w4[v].y, xv.y, s0); s1 = fma_bf16_hi(w4[v].y, xv.y, s1);
                    s0 = fma_bf16_lo(w4[v].z, xv.z, s0); s1 = fma_bf16_hi(w4[v].z, xv.z, s1);
                    s0 = fma_bf16_lo(w4[v].w, xv.w, s0); s1 = fma_bf16_hi(w4[v].w, xv.w, s1);
                    acc[v][t] += s0 + s1;
                }
            }
        }
    }
#pragma unroll
    for (int v = 0; v < NRV; v++)
#pragma unroll
        for (int t = 0; t < NP; t++)
            for (int o = lpt / 2; o > 0; o >>= 1) acc[v][t] += __shfl_xor_sync(0xffffffffu, acc[v][t], o);
}

// Epilogue for one finished output row (all segments summed).
__device__ __forceinline__ void sv_store(const SvBank& b, const SvMeta& m, int row, const float gs[SV_NT],
                                         const float us[SV_NT]) {
    for (int t = 0; t < m.np; t++) {
        float v;
        if (b.gateup) {
            const float gg = gs[t] * m.rs[t] * m.g0, uu = us[t] * m.rs[t] * m.g1;
            v = gg / (1.0f + expf(-gg)) * uu;
        } else {
            v = m.wt[t] * (gs[t] * m.rs[t]);
        }
        b.out[size_t(m.r[t]) * b.out_dim + row] = __float2bfloat16_rn(v);
    }
}

template <int FMT, int NP, int NRV, int CPL, int LPT, int NCH>
__device__ __forceinline__ void sv_consume(const SvBank& b, const SvMeta& m, const uint8_t* st,
                                           const SvStageLayout& L, int warp, int lane, int warp_group) {
    const SvGeom& g = b.g;
    const int lpt = LPT ? LPT : g.lpt;
    const int tps = 32 / lpt;                      // tasks per warp step
    const int lane_t = lane % lpt;
    const int sub = lane / lpt;
    float acc[2][SV_NT];
    if (g.tpw % (g.seg * tps) == 0) {
        // this warp owns whole rows
        const int rows_w = g.tpw / g.seg;
        for (int q = 0; q < rows_w; q += tps) {
            const int rloc = warp * rows_w + q + sub;
            float gs[SV_NT] = {0.f, 0.f}, us[SV_NT] = {0.f, 0.f};
            for (int sgi = 0; sgi < g.seg; sgi++) {
                sv_task<FMT, NP, NRV, CPL, LPT, NCH>(b, st, L, rloc < m.nrows ? rloc : 0, sgi, lane_t, acc);
#pragma unroll
                for (int t = 0; t < SV_NT; t++) { gs[t] += acc[0][t]; us[t] += acc[1][t]; }
            }
            if (lane_t == 0 && rloc < m.nrows) sv_store(b, m, m.row0 + rloc, gs, us);
        }
    } else {
        // one task per warp; seg warps share a row and meet in shared memory
        const int rloc = warp / g.seg, sgi = warp % g.seg;
        sv_task<FMT, NP, NRV, CPL, LPT, NCH>(b, st, L, rloc < m.nrows ? rloc : 0, sgi, lane_t, acc);
        float* red = reinterpret_cast<float*>(const_cast<uint8_t*>(st) + L.red);
        if (lane == 0) {
#pragma unroll
            for (int t = 0; t < SV_NT; t++) {
                red[(warp * SV_NT + t) * 2] = acc[0][t];
                red[(warp * SV_NT + t) * 2 + 1] = acc[1][t];
            }
        }
        group_sync(warp_group);
        if (sgi == 0 && lane == 0 && rloc < m.nrows) {
            float gs[SV_NT] = {0.f, 0.f}, us[SV_NT] = {0.f, 0.f};
            for (int k = 0; k < g.seg; k++)
#pragma unroll
                for (int t = 0; t < SV_NT; t++) {
                    gs[t] += red[((warp + k) * SV_NT + t) * 2];
                    us[t] += red[((warp + k) * SV_NT + t) * 2 + 1];
                }
            sv_store(b, m, m.row0 + rloc, gs, us);
        }
    }
}

template <int FMT, int NRV, int CPL, int LPT, int NCH>
__device__ __forceinline__ void sv_consume_np(const SvBank& b, const SvMeta& m, const uint8_t* st,
                                              const SvStageLayout& L, int warp, int lane, int group) {
    if (m.np == 1) sv_consume<FMT, 1, NRV, CPL, LPT, NCH>(b, m, st, L, warp, lane, group);
    else sv_consume<FMT, 2, NRV, CPL, LPT, NCH>(b, m, st, L, warp, lane, group);
}

// Compile-time instances for the layer's shapes (hidden 4096, width 1536);
// any other shape takes the runtime-geometry instance.
template <int FMT>
__device__ __forceinline__ void sv_dispatch(const SvBank& b, const SvMeta& m, const uint8_t* st,
                                            const SvStageLayout& L, int warp, int lane, int group) {
    const SvGeom& g = b.g;
    const int cpl = g.cpt / g.lpt;
    if (b.gateup) {
        constexpr int NCH_H = (FMT == MOE_FMT_BF16) ? 512 : 128;       // hidden 4096
        if (cpl == 4 && g.lpt == 32 && g.nchunks == NCH_H) sv_consume_np<FMT, 2, 4, 32, NCH_H>(b, m, st, L, warp, lane, group);
        else sv_consume_np<FMT, 2, 0, 0, 0>(b, m, st, L, warp, lane, group);
    } else {
        if (FMT != MOE_FMT_BF16 && cpl == 3 && g.lpt == 16 && g.nchunks == 48)        // width 1536
            sv_consume_np<FMT, 1, 3, 16, 48>(b, m, st, L, warp, lane, group);
        else if (FMT == MOE_FMT_BF16 && cpl == 3 && g.lpt == 32 && g.nchunks == 192)
            sv_consume_np<FMT, 1, 3, 32, 192>(b, m, st, L, warp, lane, group);
        else sv_consume_np<FMT, 1, 0, 0, 0>(b, m, st, L, warp, lane, group);
    }
}

template <int FMT0>
__global__ void __launch_bounds__(SV_THREADS, 1) stream_gemv(SvArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[2 * SV_MAX_STAGES];
    __shared__ int s_active[kMaxE];
    __shared__ int s_prefix[kMaxE];
    __shared__ int s_wcnt[SV_THREADS / 32], s_witems[SV_THREADS / 32];
    __shared__ SvItems s_it;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NS = a.nstages;
    const SvTables tb = sv_tables(smem + size_t(NS) * a.stage_bytes);
    if (tid == 0) {
        for (int s = 0; s < NS; s++) {
            mbar_init(smem_u32(&bars[s]), 1);                              // full
            mbar_init(smem_u32(&bars[SV_MAX_STAGES + s]), SV_GWARPS);      // empty: the consuming group
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    pdl_wait();       // routing results of the previous kernel are read from here on

    // touched routed experts, in expert order, and the first item of each
    {
        const SvBank& b = a.b[0];
        constexpr int PER = (kMaxE + SV_THREADS - 1) / SV_THREADS;
        int cnt[PER], nit[PER];
        int local = 0, local_items = 0;
#pragma unroll
        for (int i = 0; i < PER; i++) {
            const int e = tid * PER + i;
            const int n = (e < b.E) ? b.offsets[e + 1] - b.offsets[e] : 0;
            cnt[i] = n > 0;
            nit[i] = n > 0 ? ((n + SV_NT - 1) / SV_NT) * b.g.items_per_pass : 0;
            local += cnt[i];
            local_items += nit[i];
        }
        int v = local, w = local_items;
        for (int o = 1; o < 32; o <<= 1) {
            const int n1 = __shfl_up_sync(0xffffffffu, v, o), n2 = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) { v += n1; w += n2; }
        }
        if (lane == 31) { s_wcnt[warp] = v; s_witems[warp] = w; }
        __syncthreads();
        int base = 0, ibase = 0, tot = 0, itot = 0;
        for (int q = 0; q < SV_THREADS / 32; q++) {
            if (q < warp) { base += s_wcnt[q]; ibase += s_witems[q]; }
            tot += s_wcnt[q];
            itot += s_witems[q];
        }
        int pos = base + v - local, ipos = ibase + w - local_items;
#pragma unroll
        for (int i = 0; i < PER; i++) {
            const int e = tid * PER + i;
            if (cnt[i]) { s_active[pos] = e; s_prefix[pos] = ipos; pos++; ipos += nit[i]; }
        }
        int sh_rows = 0;
        if (a.b[1].E > 0) sh_rows = a.b[1].offsets[1] - a.b[1].offsets[0];
        const int rows0 = b.offsets[b.E];
        const bool tabled = rows0 <= SV_META_ROWS && sh_rows <= SV_META_ROWS;
        if (tid == 0) {
            s_it.n_active = tot;
            s_it.routed_items = itot;
            s_it.total = itot + ((sh_rows + SV_NT - 1) / SV_NT) * a.b[1].g.items_per_pass * (a.b[1].E > 0);
            s_it.tabled = tabled;
            tb.eoff[kMaxE] = (a.b[1].E > 0) ? a.b[1].offsets[0] : 0;
            tb.en[kMaxE] = sh_rows;
        }
        __syncthreads();
        // per active expert
        for (int q = tid; q < tot; q += SV_THREADS) {
            const int e = s_active[q];
            tb.eoff[q] = b.offsets[e];
            tb.en[q] = b.offsets[e + 1] - b.offsets[e];
            tb.g0[q] = (b.fmt == MOE_FMT_NVFP4) ? b.g0[e] : 1.f;
            tb.g1[q] = (b.fmt == MOE_FMT_NVFP4 && b.gateup) ? b.g1[e] : 1.f;
        }
        // per row
        if (tabled) {
            for (int r = tid; r < rows0; r += SV_THREADS) {
                const int slot = b.row_slot[r];
                const int arow = b.act_by_token ? slot / b.top_k : r;
                tb.arow0[r] = arow;
                tb.wt0[r] = b.topk_w ? b.topk_w[slot] : 1.f;
                tb.rs0[r] = (b.fmt == MOE_FMT_NVFP4) ? b.act_aux[arow] : 1.f;
            }
            const SvBank& b1 = a.b[1];
            for (int r = tid; r < sh_rows; r += SV_THREADS) {
                const int rr = tb.eoff[kMaxE] + r;
                tb.arow1[r] = b1.act_by_token ? b1.row_slot[rr] / b1.top_k : rr;
            }
        }
        __syncthreads();
    }
    pdl_trigger();
    const SvItems it = s_it;
    const int per_cta = (it.total + gridDim.x - 1) / gridDim.x;
    const int i0 = min(it.total, blockIdx.x * per_cta);
    const int i1 = min(it.total, i0 + per_cta);
    const uint32_t smem0 = smem_u32(smem);

    if (warp == SV_CONSUMERS) {
        // ------------------------------ producer ------------------------------
        if (lane != 0) return;
        // weights of item j into L2 ahead of the ring (DRAM keeps streaming
        // while the shared-memory stages are busy)
        auto prefetch = [&](int j) {
            if (j >= i1) return;
            const SvItem m = sv_item(a, s_active, s_prefix, tb, it, j);
            const SvBank& b = a.b[m.bank];
            const size_t wrow = size_t(m.e) * b.out_dim + m.row0;
            l2_prefetch(b.p0 + wrow * b.g.rv_bytes, m.nrows * b.g.rv_bytes);
            if (b.gateup) l2_prefetch(b.p1 + wrow * b.g.rv_bytes, m.nrows * b.g.rv_bytes);
            if (b.g.sc_bytes) {
                l2_prefetch(b.s0 + wrow * b.g.sc_bytes, m.nrows * b.g.sc_bytes);
                if (b.gateup) l2_prefetch(b.s1 + wrow * b.g.sc_bytes, m.nrows * b.g.sc_bytes);
            }
        };
        if (SV_PREFETCH > 0)
            for (int j = i0 + NS; j < i0 + NS + SV_PREFETCH; j++) prefetch(j);
        for (int i = i0; i < i1; i++) {
            const int k = i - i0, s = k % NS;
            if (k >= NS && !mbar_wait(smem_u32(&bars[SV_MAX_STAGES + s]), ((k / NS) - 1) & 1)) {
                set_status(a.status, MOE_ERR_TIMEOUT);
                return;
            }
            if (SV_PREFETCH > 0) prefetch(i + NS + SV_PREFETCH);
            const SvItem m = sv_item(a, s_active, s_prefix, tb, it, i);
            const SvBank& b = a.b[m.bank];
            const SvStageLayout L = sv_layout(b.g, b.gateup);
            const uint32_t st = smem0 + s * a.stage_bytes;
            const uint32_t full = smem_u32(&bars[s]);
            const size_t wrow = size_t(m.e) * b.out_dim + m.row0;
            const uint32_t wbytes = m.nrows * b.g.rv_bytes, sbytes = m.nrows * b.g.sc_bytes;
            const int nbank = b.gateup ? 2 : 1;
            const uint32_t tx = (wbytes + sbytes) * nbank + m.np * (b.g.act_bytes + b.g.aux_bytes);
            SvMeta* meta = reinterpret_cast<SvMeta*>(smem + size_t(s) * a.stage_bytes + L.meta);
            meta->bank = m.bank; meta->e = m.e; meta->np = m.np; meta->row0 = m.row0; meta->nrows = m.nrows;
            meta->g0 = m.bank == 0 ? tb.g0[m.a] : 1.f;
            meta->g1 = m.bank == 0 ? tb.g1[m.a] : 1.f;
            int arows[SV_NT];
            for (int t = 0; t < SV_NT; t++) {
                const int r = m.r0 + min(t, m.np - 1);
                float wt, rs;
                if (it.tabled) {
                    if (m.bank == 0) { arows[t] = tb.arow0[r]; wt = tb.wt0[r]; rs = tb.rs0[r]; }
                    else { arows[t] = tb.arow1[r - tb.eoff[kMaxE]]; wt = 1.f; rs = 1.f; }
                } else {
                    const int slot = b.row_slot[r];
                    arows[t] = b.act_by_token ? slot / b.top_k : r;
                    wt = b.topk_w ? b.topk_w[slot] : 1.f;
                    rs = (b.fmt == MOE_FMT_NVFP4) ? b.act_aux[arows[t]] : 1.f;
                }
                meta->r[t] = r;
                meta->rs[t] = rs;
                meta->wt[t] = b.gateup ? meta->g0 : wt * meta->g0;
            }
            mbar_expect_tx(full, tx);
            tma_load(st + L.w0, b.p0 + wrow * b.g.rv_bytes, wbytes, full);
            if (b.gateup) tma_load(st + L.w1, b.p1 + wrow * b.g.rv_bytes, wbytes, full);
            if (sbytes) {
                tma_load(st + L.s0, b.s0 + wrow * b.g.sc_bytes, sbytes, full);
                if (b.gateup) tma_load(st + L.s1, b.s1 + wrow * b.g.sc_bytes, sbytes, full);
            }
            for (int t = 0; t < m.np; t++) {
                const int arow = arows[t];
                tma_load(st + L.act + t * b.g.act_bytes, b.act + size_t(arow) * b.g.act_bytes, b.g.act_bytes, full);
                if (b.g.aux_bytes)
                    tma_load(st + L.aux + t * b.g.aux_bytes,
                             reinterpret_cast<const uint8_t*>(b.act_aux) + size_t(arow) * b.g.aux_bytes,
                             b.g.aux_bytes, full);
            }
        }
        // drain: every stage released (bounded), so no copy is in flight at exit
        const int n = i1 - i0;
        for (int k = max(0, n - NS); k < n; k++)
            if (!mbar_wait(smem_u32(&bars[SV_MAX_STAGES + (k % NS)]), (k / NS) & 1)) {
                set_status(a.status, MOE_ERR_TIMEOUT);
                return;
            }
        return;
    }

    // ------------------------------ consumers ------------------------------
    // group g takes items g, g + SV_GROUPS, ...; lw is the warp's rank in its group
    const int group = warp / SV_GWARPS, lw = warp % SV_GWARPS;
    for (int i = i0 + group; i < i1; i += SV_GROUPS) {
        const int k = i - i0, s = k % NS;
        if (!mbar_wait(smem_u32(&bars[s]), (k / NS) & 1)) {
            set_status(a.status, MOE_ERR_TIMEOUT);
            return;
        }
        const uint8_t* st = smem + size_t(s) * a.stage_bytes;
        const int bank = reinterpret_cast<const SvMeta*>(st)->bank;     // metadata is first in a stage
        if (bank == 0) {
            const SvStageLayout L = sv_layout(a.b[0].g, a.b[0].gateup);
            sv_dispatch<FMT0>(a.b[0], *reinterpret_cast<const SvMeta*>(st + L.meta), st, L, lw, lane, group);
        } else {
            const SvStageLayout L = sv_layout(a.b[1].g, a.b[1].gateup);
            sv_dispatch<MOE_FMT_BF16>(a.b[1], *reinterpret_cast<const SvMeta*>(st + L.meta), st, L, lw, lane, group);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars[SV_MAX_STAGES + s]));
    }
}

// ---------------------------------------------------------------------------
// Activation pre-pass, warp per row.  A row's 32-element chunk c holds four
// 16-byte pieces j = 0..3 (elements 32c + 8j .. +7); piece (j, c) is stored at
// (j * in/32 + c) * 16 bytes, so lanes reading consecutive chunks touch
// consecutive shared-memory words.
//   int4:  each piece holds the pairs (x0,x4) (x1,x5) (x2,x6) (x3,x7) (bf16),
//          matching the nibble pairs of a packed word; aux = sum per chunk.
//   NVFP4: each piece holds the f16 values x * 2^-e in order; aux = 2^e, with
//          e >= 0 the least exponent that keeps every element at or below 16384.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) act_prep(const __nv_bfloat16* __restrict__ act, int rows, int in_dim,
                                                int fmt, float* __restrict__ aux, uint8_t* __restrict__ act_out) {
    pdl_wait();
    pdl_trigger();
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= rows) return;
    const __nv_bfloat16* row = act + size_t(warp) * in_dim;
    if (fmt == MOE_FMT_INT4_G128) {
        const int nch = in_dim / 32;
        uint32_t* out = reinterpret_cast<uint32_t*>(act_out + size_t(warp) * in_dim * 2);
        for (int c = lane; c < nch; c += 32) {
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const uint4 v = *reinterpret_cast<const uint4*>(row + c * 32 + j * 8);
                s += bf16_lo(v.x) + bf16_hi(v.x) + bf16_lo(v.y) + bf16_hi(v.y) +
                     bf16_lo(v.z) + bf16_hi(v.z) + bf16_lo(v.w) + bf16_hi(v.w);
                uint4 q;
                q.x = __byte_perm(v.x, v.z, 0x5410);
                q.y = __byte_perm(v.x, v.z, 0x7632);
                q.z = __byte_perm(v.y, v.w, 0x5410);
                q.w = __byte_perm(v.y, v.w, 0x7632);
                *reinterpret_cast<uint4*>(out + (j * nch + c) * 4) = q;
            }
            aux[size_t(warp) * nch + c] = s;
        }
    } else {
        float amax = 0.f;
        for (int i = lane * 8; i < in_dim; i += 256) {
            const uint4 v = *reinterpret_cast<const uint4*>(row + i);
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))),
                                     fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y)))));
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))),
                                     fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w)))));
        }
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        int e = 0;
        while (e < 126 && ldexpf(amax, -e) > 16384.f) e++;
        const float down = ldexpf(1.f, -e);
        __half* out = reinterpret_cast<__half*>(act_out) + size_t(warp) * in_dim;
        const int nch = in_dim / 32;
        for (int i = lane * 8; i < in_dim; i += 256) {
            const uint4 v = *reinterpret_cast<const uint4*>(row + i);
            const int c = i / 32, j = (i % 32) / 8;
            __half2 h[4];
            h[0] = __floats2half2_rn(bf16_lo(v.x) * down, bf16_hi(v.x) * down);
            h[1] = __floats2half2_rn(bf16_lo(v.y) * down, bf16_hi(v.y) * down);
            h[2] = __floats2half2_rn(bf16_lo(v.z) * down, bf16_hi(v.z) * down);
            h[3] = __floats2half2_rn(bf16_lo(v.w) * down, bf16_hi(v.w) * down);
            *reinterpret_cast<uint4*>(out + (j * nch + c) * 8) = *reinterpret_cast<uint4*>(h);
        }
        if (lane == 0) aux[warp] = ldexpf(1.f, e);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static bool sv_geometry(int fmt, bool gateup, int in_dim, int out_dim, SvGeom& g) {
    const int nrv = gateup ? 2 : 1;
    g.rv_bytes = (fmt == MOE_FMT_BF16) ? in_dim * 2 : in_dim / 2;
    g.sc_bytes = (fmt == MOE_FMT_INT4_G128) ? (in_dim / 128) * 2 : (fmt == MOE_FMT_NVFP4 ? in_dim / 16 : 0);
    g.act_bytes = in_dim * 2;
    g.aux_bytes = (fmt == MOE_FMT_INT4_G128) ? (in_dim / 32) * 4 : 0;
    g.nchunks = g.rv_bytes / 16;
    g.seg = 1;
    while (g.rv_bytes / g.seg > 2048 || g.nchunks % g.seg) {
        if (++g.seg > SV_GWARPS) return false;
    }
    g.cpt = g.nchunks / g.seg;
    g.lpt = 32;
    while (g.lpt > 1 && g.cpt % g.lpt) g.lpt >>= 1;
    const int tps = 32 / g.lpt;
    int best = -1;
    for (int tpw = 1; tpw <= 512; tpw++) {
        const bool whole = tpw % (g.seg * tps) == 0;
        const bool shared_row = tpw == 1 && tps == 1 && g.seg > 1 && SV_GWARPS % g.seg == 0;
        if (!whole && !shared_row) continue;
        const long long rows = (long long)SV_GWARPS * tpw / g.seg;
        if (rows * nrv * g.rv_bytes > SV_STAGE_TARGET && best > 0) break;
        best = tpw;
        if (rows >= out_dim) break;
    }
    if (best < 0) return false;
    g.tpw = best;
    g.rows_item = SV_GWARPS * best / g.seg;
    g.items_per_pass = (out_dim + g.rows_item - 1) / g.rows_item;
    // TMA bulk copies: sizes and addresses in multiples of 16 bytes
    const int tail = out_dim % g.rows_item;
    if ((g.rows_item * g.sc_bytes) % 16 || (size_t(out_dim) * g.sc_bytes) % 16 || (tail * g.sc_bytes) % 16)
        return false;
    if (g.rv_bytes % 16 || g.act_bytes % 16 || g.aux_bytes % 16) return false;
    return true;
}

size_t stream_prep_bytes(int fmt, int rows, int in_dim) {
    if (fmt == MOE_FMT_BF16) return 0;
    const size_t aux = (fmt == MOE_FMT_INT4_G128) ? size_t(rows) * (in_dim / 32) * 4 : size_t(rows) * 4;
    return align256(aux) + size_t(rows) * in_dim * 2;
}

static void fill_bank(SvBank& b, const GemvProblem& p, bool gateup, const uint8_t* act, const float* aux) {
    b.fmt = p.fmt; b.gateup = gateup; b.E = p.E; b.out_dim = p.out_dim; b.in_dim = p.in_dim;
    b.top_k = p.top_k; b.act_by_token = p.act_by_token;
    b.p0 = reinterpret_cast<const uint8_t*>(p.p0); b.s0 = reinterpret_cast<const uint8_t*>(p.s0); b.g0 = p.g0;
    b.p1 = reinterpret_cast<const uint8_t*>(p.p1); b.s1 = reinterpret_cast<const uint8_t*>(p.s1); b.g1 = p.g1;
    b.offsets = p.offsets; b.row_slot = p.row_slot; b.topk_w = p.topk_w; b.out = p.out;
    b.act = act;
    b.act_aux = aux;
}

template <typename K, typename... Args>
static cudaError_t launch_ex(K kern, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl, Args... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (e == cudaSuccess) count_launch();
    return e;
}

template <int FMT>
static cudaError_t launch_sv(const SvArgs& a, size_t smem, cudaStream_t s, bool pdl) {
    // per device (a kernel's shared memory limit is a per-device attribute): the SM count, read once, and
    // the dynamic shared memory granted so far, raised under a lock when a call needs more
    struct Dev {
        std::once_flag once;
        int sms = 0;
        std::mutex mu;
        size_t granted = 0;
    };
    static Dev devs[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    Dev& d = devs[dev];
    std::call_once(d.once, [&] {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) d.sms = 0;
    });
    if (d.sms <= 0) return cudaErrorInvalidDevice;
    auto k = stream_gemv<FMT>;
    {
        std::lock_guard<std::mutex> lock(d.mu);
        if (smem > d.granted) {
            cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            if (e != cudaSuccess) return e;
            d.granted = smem;
        }
    }
    return launch_ex(k, dim3(d.sms), dim3(SV_THREADS), smem, s, pdl, a);
}

int launch_stream_gemv(const GemvProblem& routed, const GemvProblem* shared, bool gateup, int act_rows,
                       void* prep_ws, cudaStream_t s, bool pdl) {
    SvArgs a{};
    a.status = routed.status;
    const uint8_t* act = reinterpret_cast<const uint8_t*>(routed.act);
    float* aux = nullptr;
    if (routed.fmt != MOE_FMT_BF16) {
        aux = reinterpret_cast<float*>(prep_ws);
        const size_t aux_bytes = (routed.fmt == MOE_FMT_INT4_G128) ? size_t(act_rows) * (routed.in_dim / 32) * 4
                                                                   : size_t(act_rows) * 4;
        uint8_t* act_out = reinterpret_cast<uint8_t*>(prep_ws) + align256(aux_bytes);
        const int blocks = (act_rows * 32 + 255) / 256;
        if (launch_ex(act_prep, dim3(blocks), dim3(256), 0, s, pdl, routed.act, act_rows, routed.in_dim,
                      routed.fmt, aux, act_out) != cudaSuccess)
            return MOE_ERR_CUDA;
        act = act_out;
        pdl = true;
    }
    fill_bank(a.b[0], routed, gateup, act, aux);
    if (!sv_geometry(routed.fmt, gateup, routed.in_dim, routed.out_dim, a.b[0].g)) return MOE_ERR_UNSUPPORTED;
    int stage = sv_layout(a.b[0].g, gateup).bytes;
    if (shared) {
        fill_bank(a.b[1], *shared, gateup, reinterpret_cast<const uint8_t*>(shared->act), nullptr);
        if (shared->fmt != MOE_FMT_BF16) return MOE_ERR_UNSUPPORTED;
        if (!sv_geometry(shared->fmt, gateup, shared->in_dim, shared->out_dim, a.b[1].g)) return MOE_ERR_UNSUPPORTED;
        stage = std::max(stage, sv_layout(a.b[1].g, gateup).bytes);
    } else {
        a.b[1] = SvBank{};
    }
    stage = (stage + 127) & ~127;
    a.stage_bytes = stage;
    a.nstages = std::min(SV_MAX_STAGES, SV_SMEM_MAX / stage);
    if (a.nstages < 2) return MOE_ERR_UNSUPPORTED;
    const size_t smem = size_t(a.nstages) * stage + SV_TABLE_BYTES;
    cudaError_t e;
    if (routed.fmt == MOE_FMT_INT4_G128) e = launch_sv<MOE_FMT_INT4_G128>(a, smem, s, pdl);
    else if (routed.fmt == MOE_FMT_NVFP4) e = launch_sv<MOE_FMT_NVFP4>(a, smem, s, pdl);
    else e = launch_sv<MOE_FMT_BF16>(a, smem, s, pdl);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
