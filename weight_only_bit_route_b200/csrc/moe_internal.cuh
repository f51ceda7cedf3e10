// Internal declarations of libmoe (sm_100a).  Kernels and host helpers share
// this header; the public boundary is include/moe_w4a16.h.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "../../include/moe_w4a16.h"

namespace moe {

constexpr int kMaxE = 1024;
constexpr int kMaxTopK = 8;
constexpr int kMaxDecodeT = 64;

// ---------------------------------------------------------------------------
// Workspace layout.  Every region starts on a 256-byte boundary.
// ctrl (1 KB): [0] status word, [1] router arrival counter, [2] quantiser
//              amax (float bits), [3] reserved, [4..5] bound on every
//              device wait in ns (uint64, 0 = the default of about 2 s),
//              [6] failure-testing hold (non-zero: each tensor-core GEMM
//              first waits on a barrier nothing completes), [7] reserved,
//              [8..9] the routed GEMMs' tile scheduler (next tile, CTAs
//              done), [10..15] reserved, [16..255] split-K tile arrival
//              counters (counters are left at zero by every call that
//              completes).
// ---------------------------------------------------------------------------
struct WsLayout {
    size_t ctrl, logits, wsplit, hist, offsets, row_slot, slot_row, ids, tw;
    size_t sh_offsets, sh_rowslot, h_perm, y_perm, ys, tiles, prep, shpart, total;
};

constexpr int kPermChunk = 4096;   // slots handled by one bucketing block

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// ---------------------------------------------------------------------------
// Device status word: the first error recorded wins.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }
// The layer's input activations: bf16, or fp16 in the fp16 activation mode (both exact in fp32).
template <bool F16>
__device__ __forceinline__ float act_lo(uint32_t v) {
    if constexpr (F16) return __half2float(__ushort_as_half(static_cast<unsigned short>(v & 0xffffu)));
    else return bf16_lo(v);
}
template <bool F16>
__device__ __forceinline__ float act_hi(uint32_t v) {
    if constexpr (F16) return __half2float(__ushort_as_half(static_cast<unsigned short>(v >> 16)));
    else return bf16_hi(v);
}

__device__ __forceinline__ float warp_sum(float v, int width) {
    for (int o = width / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Step-level calls use the workspace as [ctrl 1 KB][their own scratch].
constexpr size_t kStepScratch = 1024;
// router: logits [T, E] fp32, then the three bf16 planes of the router weights
// used by the tensor-core path (3 * E * H bf16)
inline size_t route_scratch(int T, int E, int H) { return align256(size_t(T) * E * 4) + align256(size_t(E) * H * 6); }
inline size_t permute_scratch(int T, int k, int E) {
    size_t R = size_t(T) * k;
    size_t nb = (R + kPermChunk - 1) / kPermChunk;
    return (nb ? nb : 1) * E * 4;
}
// Activation pre-pass output of the streaming GEMV (largest over formats):
// int4 chunk sums [rows, in/32] fp32 + a reordered bf16 copy [rows, in].
inline size_t prep_scratch(int rows, int in_dim) {
    return align256(size_t(rows) * (in_dim / 32) * 4) + align256(size_t(rows) * in_dim * 2);
}
// int4 routed problems with at most this many rows take the 8-bit int4 GEMM
constexpr int kI8Int4MaxRows = 512;
// Row stride (floats) of the 8-bit int4 group sums: in/128 rounded up to a
// multiple of 4, so that a tile's rows are one 16-byte aligned block.
inline int zsum_stride(int in_dim) { return ((in_dim / 128) + 3) & ~3; }
// 8-bit int4 row record (floats): group sums [zst], group factors [zst], the row factor, padding to 16 bytes
inline int zrow_floats(int in_dim) { return 2 * zsum_stride(in_dim) + 4; }
// GEMM pre-pass output: row scales [rows] fp32, the 8-bit path's row records
// [rows][zrow_floats] fp32, then the gathered rows: 16-bit [rows][in], or
// three int8 digit rows per row when the 8-bit int4 GEMM can take the problem.
inline size_t gemm_prep_bytes(int rows, int in_dim) {
    return align256(size_t(rows) * 4) + align256(size_t(rows) * zrow_floats(in_dim) * 4) +
           align256(size_t(rows) * in_dim * (rows <= kI8Int4MaxRows ? 3 : 2));
}
// Step-level scratch of a grouped call: tile metadata, then the pre-pass of
// act_rows rows (GEMV or GEMM).
inline size_t grouped_scratch(int E, int act_rows, int in_dim) {
    return align256(size_t(E + 2) * 16) + std::max(prep_scratch(act_rows, in_dim), gemm_prep_bytes(act_rows, in_dim));
}

// The BF16 shared expert at a small batch has few (m, n) tiles (12 for gate/up,
// 32 for down); split K so that the weight stream spreads over more SMs (48 and
// 64 tiles: at decode sizes it runs beside the routed chain on at most 64 SMs).
inline int shared_ksplit(int E, int fmt, bool gateup, int rows, int in_dim) {
    if (E != 1 || fmt != MOE_FMT_BF16 || rows > 64) return 1;
    int ks = gateup ? 4 : 2;
    while (ks > 1 && in_dim % (ks * 128)) ks >>= 1;
    return ks;
}
inline size_t split_bytes(int ksplit, bool gateup, int rows, int out_dim) {
    return ksplit > 1 ? align256(size_t(ksplit) * (gateup ? 2 : 1) * rows * out_dim * 4) : 0;
}

inline WsLayout ws_layout(int T, int H, int E, int F, int k) {
    WsLayout L{};
    size_t R = size_t(T) * k;
    size_t nb = (R + kPermChunk - 1) / kPermChunk;
    if (nb == 0) nb = 1;
    size_t o = 0;
    L.ctrl = o;       o = align256(o + kStepScratch);
    L.logits = o;     o = align256(o + size_t(T) * E * 4);
    L.wsplit = o;     o = align256(o + size_t(E) * H * 6);
    L.hist = o;       o = align256(o + nb * E * 4);
    L.offsets = o;    o = align256(o + size_t(E + 1) * 4);
    L.row_slot = o;   o = align256(o + R * 4);
    L.slot_row = o;   o = align256(o + R * 4);
    L.ids = o;        o = align256(o + R * 4);
    L.tw = o;         o = align256(o + R * 4);
    L.sh_offsets = o; o = align256(o + 2 * 4);
    L.sh_rowslot = o; o = align256(o + size_t(T) * 4);
    L.h_perm = o;     o = align256(o + (R + T) * size_t(F) * 2);
    L.y_perm = o;     o = align256(o + R * size_t(H) * 2);
    L.ys = o;         o = align256(o + size_t(T) * H * 2);
    L.tiles = o;      o = align256(o + size_t(E + 2) * 4 * 4);
    L.prep = o;       o = align256(o + std::max(std::max(prep_scratch(T, H), prep_scratch(int(R), F)),
                                            std::max(gemm_prep_bytes(int(R), H), gemm_prep_bytes(int(R), F))));
    L.shpart = o;     o = align256(o + std::max(split_bytes(shared_ksplit(1, MOE_FMT_BF16, true, T, H), true, T, F),
                                                split_bytes(shared_ksplit(1, MOE_FMT_BF16, false, T, F), false, T, H)));
    L.total = o;
    return L;
}

// Host-side count of successful kernel launches (moe_launch_count).
void count_launch();

// Launch with programmatic dependent launch allowed: the kernel may start
// while the previous kernel on the stream finishes, and must execute
// griddepcontrol.wait before it reads anything that kernel wrote.
template <typename K, typename... Args>
inline cudaError_t launch_pdl(K kern, dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (e == cudaSuccess) count_launch();
    return e;
}

// ---------------------------------------------------------------------------
// Host-side launchers (defined in the .cu files).
// ---------------------------------------------------------------------------
constexpr int kRouterDecodeMaxT = 16;
// the fused decode router splits H into four quarters of whole 128-wide steps
inline bool router_decode_ok(int H) { return H % 512 == 0; }
constexpr int kRouterTcMinT = 64;      // from this many tokens the router logits run on the tensor cores

// Router: logits + sigmoid top-k.  counter: a zeroed int in the workspace
// (enables the fused decode router for T <= kRouterDecodeMaxT), or null.
// planes: 3 * E * H bf16 of scratch for the tensor-core logits (used when T >= 64).
int launch_route(const __nv_bfloat16* x, int T, int H, const float* Wr, const float* bias,
                 int E, int k, int32_t* ids, float* w, float* logits, __nv_bfloat16* planes,
                 int32_t* status, int32_t* counter, cudaStream_t s, int x_f16 = 0);
// Router logits l = x Wr^T (fp32) on the tensor cores (Wr split into three bf16 planes).
int launch_router_logits_tc(const __nv_bfloat16* x, int T, int H, const float* Wr, int E, float* logits,
                            __nv_bfloat16* planes, int32_t* status, cudaStream_t s);

struct RouterDecodeArgs {
    const __nv_bfloat16* x; int T, H; const float* Wr; const float* bias; int E, k;
    int x_f16;                                                  // x holds fp16 values (fp16 activation mode)
    float* logits; int32_t* ids; float* w;
    int32_t* counter; int32_t* status;
    int32_t* offsets; int32_t* row_slot; int32_t* slot_row;     // bucketing (nullable: skip)
    int32_t* sh_offsets; int32_t* sh_rowslot;                   // shared routing (nullable: skip)
};
// Fused decode router: logits, top-k, bucketing and shared routing in one launch.
int launch_route_decode(const RouterDecodeArgs& a, cudaStream_t s);

int launch_permute(const int32_t* ids, int T, int k, int E, int32_t* offsets,
                   int32_t* row_slot, int32_t* slot_row, int32_t* hist, int32_t* status,
                   cudaStream_t s);
int launch_permute_noalloc(const int32_t* ids, int T, int k, int E, int32_t* offsets, int32_t* row_slot,
                           int32_t* slot_row, cudaStream_t s);

struct GemvProblem {
    const __nv_bfloat16* act;  // gate/up: x [T, in]; down: h_perm [rows, in]
    int act_by_token;          // 1: activation row = row_slot[r] / top_k; 0: row r
    int top_k;
    const int32_t* offsets;    // [E+1]
    const int32_t* row_slot;   // [rows]
    int E;
    const float* topk_w;       // down only: weight by slot (nullable)
    int fmt, out_dim, in_dim;
    const void* p0; const void* s0; const float* g0;   // gate (or down)
    const void* p1; const void* s1; const float* g1;   // up (gate/up only)
    __nv_bfloat16* out;        // [rows, out_dim]
    int32_t* status;
    const float* in_scale;     // NVFP4 W4A4: activation global scale by expert [E] (nullable)
    int act_f16;               // act holds fp16 values (fp16 activation mode; 4-bit formats on the GEMM)
};

// Streaming grouped GEMV (decode): routed bank plus an optional BF16 shared
// bank in one launch.  act_rows: activation rows of the routed problem (T for
// gate/up, rows for down); prep_ws: prep_scratch(act_rows, in_dim) bytes.
int launch_stream_gemv(const GemvProblem& routed, const GemvProblem* shared, bool gateup, int act_rows,
                       void* prep_ws, cudaStream_t s, bool pdl);

int launch_combine(const __nv_bfloat16* y_perm, const int32_t* slot_row, int T, int k, int H,
                   const __nv_bfloat16* shared_out, __nv_bfloat16* y, cudaStream_t s, bool pdl = true,
                   int y_f16 = 0);
// fp16 -> bf16 (round to nearest even), n elements, n % 8 == 0: the BF16 shared expert's input
// in the fp16 activation mode.
int launch_f16_to_bf16(const __half* src, __nv_bfloat16* dst, size_t n, cudaStream_t s);

int launch_quant_int4(const __nv_bfloat16* w, int64_t rows, int64_t cols, int32_t* packed,
                      __nv_bfloat16* scales, cudaStream_t s);
int launch_quant_nvfp4_act(const __nv_bfloat16* x, int64_t rows, int64_t cols, const float* g, uint8_t* packed,
                           uint8_t* scales, cudaStream_t s);
int launch_quant_nvfp4(const __nv_bfloat16* w, int64_t rows, int64_t cols, uint8_t* packed,
                       uint8_t* scales, float* global, uint32_t* amax_slot, cudaStream_t s);

int launch_shared_routing(int T, int k, int32_t* sh_offsets, int32_t* sh_rowslot,
                          cudaStream_t s);
// Compressed scale format (csf.cu).
int launch_csf_decode(const uint8_t* fixed, const uint32_t* exc, const int64_t* starts, int E, int R, int C,
                      const int32_t* offsets, uint8_t* out, cudaStream_t s);
int launch_csf_encode(const uint8_t* sc, int E, int R, int C, uint8_t* fixed, int64_t* starts, uint32_t* exc,
                      int64_t capacity, int32_t* rowcnt, int64_t* tot, int32_t* status, cudaStream_t s);
inline size_t csf_encode_scratch(int E, int R) { return align256(size_t(E) * R * 4) + align256(size_t(E) * 8); }

// Writes one 64-bit word of device memory in stream order.
int launch_set_u64(unsigned long long* dst, unsigned long long v, cudaStream_t s);
// Writes one 32-bit word of device memory in stream order.
int launch_set_u32(uint32_t* dst, uint32_t v, cudaStream_t s);

// Activation operand of the tcgen05 grouped GEMM.  A pre-pass gathers the
// problem's rows (row r reads activation row row_slot[r] / top_k when
// act_by_token, else row r) into act_buf ([rows, in] 16-bit) in the kernel's
// operand order: f16 with a power-of-two row scale (scale_buf, [rows] fp32)
// for the 4-bit formats (int4: its pairs (0,4) (1,5) (2,6) (3,7) in every 8;
// NVFP4 W4A4: the NVFP4-quantised values e2m1 x e4m3, exact in f16, with the
// expert's input scale as the row scale),
// a plain copy for BF16; the 8-bit int4 path writes three int8 digit rows
// per row instead.  act_ready (BF16 only): the rows are already in place
// (row r is row r), no pre-pass runs.
struct GemmBuffers {
    void* act_buf;
    float* scale_buf;
    int act_ready;
    int ksplit;          // > 1: split K into this many slices (BF16 only); fp32 partial sums go to partial
    float* partial;      // split_bytes(...) bytes
    int i8;              // int4 on the 8-bit MMA with per-group accumulation (small batches)
    float* zbuf;         // i8: row records [rows][zrow_floats(in)] (group sums, group factors, row factor)
    int* tile_cnt;       // split-K: kTileCounters zeroed ints (the control block's [16..255])
    int max_ctas;        // > 0: at most this many CTAs (a side-stream problem leaves the other SMs free)
    int no_pdl;          // launch without programmatic dependent launch (its CTAs hold no SM while waiting)
    int* sched;          // tensor-core GEMM: {next, done} tile counters (zero), or null for a static tile order;
                         // problems that may run at the same time need their own
    int max_expert_rows; // > 0: no expert holds more rows than this (the batch's token count); 0: unknown
};
constexpr int kTileCounters = 240;


// Prefill-shaped grouped GEMM (tcgen05) for one problem; rows: activation
// (and output) rows of the problem.
int launch_grouped_gemm(const GemvProblem& p, bool gateup, int rows, const GemmBuffers& buf, cudaStream_t s);

}  // namespace moe
