/*
 * moe_w4a16.h -- C ABI of libmoe: the routed-expert MoE layer of Step-5-Preview
 * run directly on 4-bit weights, on one NVIDIA B200 (sm_100a).
 *
 * The layer ("Step-5-Preview-Spark", At a glance; "Step 5 Preview: 92 narrow
 * layers, and a sparse indexer that scores blocks of 8", The shape): hidden
 * size H = 4096, E = 352 routed experts chosen top-8 by a sigmoid router, each
 * a SwiGLU of width F = 1536, plus one shared SwiGLU expert of the same width:
 *
 *     y[t] = FFN_shared(x[t]) + sum_{j<k} w[t,j] * FFN_{e[t,j]}(x[t]),
 *     FFN(x) = W_down (silu(W_gate x) * (W_up x)).
 *
 * Routed expert weights come in the pages' fused layout [E, out, in] in one of
 * two 4-bit formats:
 *   MOE_FMT_INT4_G128 -- "Step-5-Preview-Int4-g128", Recipe / Tensor layout:
 *       int4 symmetric, group 128 along `in`, one bf16 scale per group.
 *       packed: int32 [E, out, in/8]; element in = 8c + j is bits 4j..4j+3 of
 *       word c, stored offset-binary (nibble u = q + 8, q in [-8, 7]).
 *       scales: bf16 [E, out, in/128].  w = q * scale.
 *   MOE_FMT_NVFP4 -- "Step-5-Preview-NVFP4-Local", Modifications item 2 and
 *       Format (W4A16_NVFP4, activations stay bf16): packed: uint8
 *       [E, out, in/2], two E2M1 codes per byte, even element in the low nibble;
 *       scales: uint8 E4M3 [E, out, in/16]; global_scale: fp32 [E]
 *       (weight_scale_2).  w = e2m1(code) * e4m3(scale) * global_scale[e].
 *       With input_scale (W4A4, layers 3-87 of the pages' model): the
 *       activation entering the projection is quantised to NVFP4 on the fly,
 *       per 16 elements, with the expert's input_scale as its global scale
 *       (block scale e4m3_rne_sat(amax / (6 g)), codes e2m1_rne_sat(x / (e4m3 g))),
 *       and the product runs on the quantised values.  Gate and up read the
 *       same activation, quantised once with gate.input_scale (up.input_scale
 *       must be NULL or the same pointer); the down projection's input is h
 *       rounded to bf16, quantised with down.input_scale.
 *   MOE_FMT_BF16 -- plain bf16 [E, out, in] (used for the shared expert).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are caller-owned DEVICE memory on the current device.
 *     The library never allocates, frees, or synchronises the stream, except
 *     moe_read_status(), which synchronises to read the status word.
 *   - Calls are asynchronous and stream-ordered on `stream` (a cudaStream_t;
 *     NULL = legacy default stream).
 *   - The return value reports argument and launch errors only (moe_status).
 *     On an argument error nothing is launched.  Conditions found on the device
 *     (an expert id out of range, a bounded wait that ran out) are recorded in
 *     the status word at the start of the workspace; read it with
 *     moe_read_status().
 *   - Weight, activation and output pointers must be 16-byte aligned.
 *     H, F must be multiples of 128; 1 <= top_k <= 8; 1 <= E <= 1024.
 *     Other shapes return MOE_ERR_UNSUPPORTED.  T = 0 is a no-op (MOE_OK).
 *   - bf16 tensors are passed as `void*` (2 bytes per element, IEEE bfloat16).
 *   - Intermediates: h_perm is bf16 [rows, F]; y_perm is bf16 [rows, H].
 *   - The workspace `ws` (ws_bytes bytes, 256-byte aligned) must be zero-filled
 *     once before first use (moe_workspace_init); kernels leave their counters
 *     at zero again when they finish.  Its first 1024 bytes hold the status
 *     word and those counters; the step calls use the bytes after them as
 *     scratch (sizes below),
 *     the layer entries the whole of moe_workspace_bytes().  A workspace of
 *     moe_workspace_bytes(T, H, E, F, top_k) bytes serves every call at those
 *     sizes.  Calls that share a workspace must not run concurrently.
 *   - Host threads: calls from several threads are safe when they use separate
 *     workspaces (moe_permute_noalloc excepted: its calls share one scratch
 *     array).  The library's launch-time state (per-device kernel attributes,
 *     the shared expert's side stream) is taken under locks; no lock is held
 *     while the GPU is waited on.
 */
#ifndef MOE_W4A16_H
#define MOE_W4A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* same type as cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1, /* null pointer, negative size, misalignment   */
    MOE_ERR_UNSUPPORTED = -2, /* valid but unsupported shape / format         */
    MOE_ERR_CUDA = -3,        /* a CUDA call or kernel launch failed          */
    MOE_ERR_TIMEOUT = -4,     /* device status: a bounded wait ran out        */
    MOE_ERR_WORKSPACE = -5,   /* workspace missing or too small               */
    MOE_ERR_DEVICE_INDEX = -6,/* device status: an index was out of range     */
    MOE_ERR_NONFINITE = -7    /* device status: an activation row held an inf
                                 or NaN where the kernel needs a finite row
                                 maximum; that row's outputs are NaN        */
} moe_status;

typedef enum { MOE_FMT_INT4_G128 = 0, MOE_FMT_NVFP4 = 1, MOE_FMT_BF16 = 2 } moe_wfmt;

/* One projection bank in the pages' fused layout [num_experts, out_dim, in_dim]. */
typedef struct {
    int32_t fmt;              /* moe_wfmt                                          */
    int32_t num_experts;      /* E (1 for the shared expert)                      */
    int32_t out_dim;          /* rows: F for gate/up, H for down                  */
    int32_t in_dim;           /* reduction length: H for gate/up, F for down      */
    const void* packed;       /* INT4: int32[E,out,in/8]; NVFP4: u8[E,out,in/2]; BF16: bf16[E,out,in] */
    const void* scales;       /* INT4: bf16[E,out,in/128]; NVFP4: u8 E4M3[E,out,in/16]; BF16: NULL   */
    const float* global_scale;/* NVFP4: fp32[E]; otherwise NULL                    */
    const float* input_scale; /* NVFP4 W4A4: fp32[E], the activation global scale of
                                 each expert (quant_algo NVFP4 with an input_scale,
                                 "Step-5-Preview-NVFP4-Local", Modifications); NULL:
                                 W4A16 (activations stay bf16).  Only NVFP4 banks
                                 on the tensor-core GEMM take it.               */
} moe_qweight;

/* A whole MoE layer.  sh_gate/sh_up/sh_down: MOE_FMT_BF16 banks with
 * num_experts = 1, or all three with packed = NULL for no shared expert.
 * router_w: fp32 [E, H]; router_bias: fp32 [E] added to the logits before
 * the sigmoid, or NULL.  swiglu_limit must be 0 (the pages give no value or
 * definition for a SwiGLU limit, so none is applied).
 * act_f16: 0 = x and y are bf16; 1 = x and y are IEEE fp16 ("Step-5-Preview-
 * Spark", At a glance and Quality: the release runs activations in fp16, since
 * bf16 rounding of the routing input changed far more top-8 sets).  The router
 * and the routed experts read the fp16 x exactly; the BF16 shared expert reads x
 * rounded to bf16 (its MMA takes bf16 operands); the intermediates h and
 * y_perm stay bf16.  Requires the routed banks in a 4-bit format with both
 * projections on the tensor-core GEMM (H and F multiples of 256); from 64
 * tokens the router logits run on the fp32 SIMT kernel (the tensor-core router
 * splits bf16 operands). */
typedef struct {
    moe_qweight gate, up, down;
    moe_qweight sh_gate, sh_up, sh_down;
    const float* router_w;
    const float* router_bias;
    int32_t E, H, F, top_k;
    float swiglu_limit;
    int32_t act_f16;
} moe_layer;

/* ---------------------------------------------------------------------- */
/* Workspace and status                                                    */
/* ---------------------------------------------------------------------- */

/* Bytes of workspace sufficient for every entry point below at these sizes
 * (T tokens), including the intermediates of moe_layer_decode and
 * moe_layer_forward.  Returns 0 for invalid sizes. */
size_t moe_workspace_bytes(int T, int H, int E, int F, int top_k);

/* Zero-fill a workspace (cudaMemsetAsync on `stream`). */
int moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream);

/* Synchronise `stream`, copy the workspace's device status word to
 * *status_out (MOE_OK or a negative moe_status; the first condition recorded
 * wins), and clear it.  When it was not MOE_OK, the arrival counters of the
 * control block are cleared too (a kernel that stopped early may have left
 * them set), so the workspace serves the next call. */
int moe_read_status(void* ws, moe_stream_t stream, int32_t* status_out);

/* Bound, in nanoseconds, on each device-side wait of the tensor-core kernels
 * and the fused router when they run with this workspace (stream-ordered: a
 * one-thread kernel writes words 4-5 of the control block).  0 restores the
 * default of about 2 s, which a zero-filled workspace starts with.  A wait
 * that runs out records MOE_ERR_TIMEOUT, the kernel stops issuing work,
 * waits (bounded by the default) for the copies and MMAs it has in flight,
 * releases its tensor memory and returns; its outputs are then undefined.
 * A wait polls with mbarrier try_wait, which may itself suspend until the
 * barrier completes, so a wait that the hardware completes within that
 * suspension never times out, however short the bound.  The pages have no
 * counterpart to this call. */
int moe_set_wait_limit(void* ws, uint64_t limit_ns, moe_stream_t stream);

/* Failure testing: while `hold` is non-zero (word 6 of the control block,
 * stream-ordered), the MMA warp of every tensor-core GEMM launched with this
 * workspace first waits on a barrier that nothing completes, so that wait
 * runs out after the configured bound (moe_set_wait_limit) with the kernel's
 * copies in flight, and the kernel takes its abort path (MOE_ERR_TIMEOUT,
 * drain, return).  No other call is affected.  hold = 0 ends it.  The pages
 * have no counterpart to this call. */
int moe_set_wait_hold(void* ws, int hold, moe_stream_t stream);

/* Static description of a status code. */
const char* moe_status_string(int status);

/* Number of kernels this library has launched in this process since it was
 * loaded (a host-side count of successful launch calls, over every stream
 * and device).  Launches recorded by moe_layer_graph_create are not counted;
 * each moe_layer_graph_launch adds the graph's kernels.  For measurement; no
 * part of the layer's arithmetic. */
uint64_t moe_launch_count(void);

/* ---------------------------------------------------------------------- */
/* Hot-path steps                                                          */
/* ---------------------------------------------------------------------- */

/* Router ("Step-5-Preview-Spark", At a glance: sigmoid router, top-8).
 *   l[t,e] = sum_h x[t,h] * router_w[e,h] (+ router_bias[e]), fp32;
 *   s = 1 / (1 + exp(-l)), fp32; the top_k largest s per token, ties to the
 *   lower expert id, listed by descending s; topk_w = s / sum(selected s).
 * x: bf16 [T, H]; router_w: fp32 [E, H]; router_bias: fp32 [E] or NULL;
 * topk_ids: int32 [T, top_k] (out); topk_w: fp32 [T, top_k] (out).
 * From 64 tokens the logits run on the tensor cores: router_w is split into
 * three bf16 planes (hi + mid + lo) whose bf16 x bf16 products are exact in
 * fp32, accumulated in fp32.
 * ws (256-byte aligned): at least 1024 + a(4*T*E) + a(6*E*H) bytes, a()
 * rounding up to a multiple of 256. */
int moe_route_topk(const void* x, int T, int H, const float* router_w,
                   const float* router_bias, int E, int top_k, int32_t* topk_ids,
                   float* topk_w, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Token -> expert bucketing ("Step 5 Preview: 92 narrow layers...", The
 * shape: each token goes to its 8 routed experts, whose weights sit in the
 * fused [E, out, in] banks of "Step-5-Preview-Int4-g128", Tensor layout, so
 * each expert's tokens are gathered into one contiguous block of rows): a
 * stable counting sort of the R = T*top_k slots (slot = t*top_k + j) by
 * expert id.
 * topk_ids: int32 [T, top_k], each in [0, E) (an id outside sets the device
 * status MOE_ERR_DEVICE_INDEX and is dropped);
 * expert_offsets: int32 [E+1] (out), exclusive prefix sum of per-expert counts;
 * row_slot: int32 [R] (out), the slot placed at permuted row r;
 * slot_row: int32 [R] (out), its inverse.
 * Rows of one expert are ordered by slot (token, then rank j).
 * ws: at least 1024 + 4*E*ceil(T*top_k / 4096) bytes. */
int moe_permute(const int32_t* topk_ids, int T, int top_k, int E,
                int32_t* expert_offsets, int32_t* row_slot, int32_t* slot_row,
                void* ws, size_t ws_bytes, moe_stream_t stream);

/* Bucketing for callers that cannot allocate device memory.  Some callers run
 * inside another runtime's fixed memory plan (an engine that reserves the GPU's
 * memory up front and hands out no extra buffers), or cannot afford the
 * device-wide synchronisation that an allocation can cause in the middle of a
 * step; they cannot supply the workspace moe_permute needs.  This call
 * computes exactly what moe_permute computes (same arguments and outputs,
 * minus the workspace) and allocates nothing: its scratch is a file-scope device array of about 64 KB that every
 * GPU loading the library keeps until the process exits.
 * Limits: T*top_k <= 65536 and E <= 1024; larger sizes return
 * MOE_ERR_UNSUPPORTED.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress), so make one call on each device before any
 * stream capture.  All calls share the array and each call overwrites it:
 * calls that may overlap on the GPU (different streams with no ordering
 * between them) race.  An expert id outside [0, E) is dropped and its slot_row
 * entry is -1; that condition is not reported (no caller can read the static
 * array's status word), and row_slot past expert_offsets[E] is left
 * unwritten.  The model pages describe no counterpart to this call. */
int moe_permute_noalloc(const int32_t* topk_ids, int T, int top_k, int E,
                        int32_t* expert_offsets, int32_t* row_slot, int32_t* slot_row,
                        moe_stream_t stream);

/* Grouped gate/up projection with fused SwiGLU, weights dequantised in-kernel
 * ("Step 5 Preview: 92 narrow layers...", The shape: routed SwiGLU experts of
 * width 1536 at hidden 4096; weights as "Step-5-Preview-Int4-g128", Recipe /
 * Tensor layout, or "Step-5-Preview-NVFP4-Local", Format):
 * for each expert e and row r in [expert_offsets[e], expert_offsets[e+1]),
 * with token t = row_slot[r] / top_k:
 *     h_perm[r, f] = bf16( silu(g) * u ),  g = x[t] . Wg[e,f,:],  u = x[t] . Wu[e,f,:]
 * (fp32 accumulation).  x: bf16 [T, H]; gate/up: banks [E, F, H] of the same
 * format; h_perm: bf16 [T*top_k, F] (out).  swiglu_limit must be 0.
 * For the shared expert pass BF16 banks with E = 1, expert_offsets = {0, T}
 * and row_slot[i] = i * top_k.  rows = T*top_k (T for E = 1).  With H a
 * multiple of 256 and F of 128 the call runs the tcgen05 grouped GEMM: int4
 * banks with E > 1 and rows <= 512 on the 8-bit tensor-core path (x as three
 * 8-bit digits of a 24-bit fixed point with an exponent per row and scale
 * group, exact integer sums per scale group), everything else on the 16-bit
 * one; other shapes stream the weights with a GEMV.
 * ws (256-byte aligned): at least 1024 + a(16*(E+2)) + max(a(rows*H/8) +
 * a(2*rows*H), a(4*rows) + a(rows*(8*z+16)) + a(c*rows*H)) bytes, z = H/128
 * rounded up to a multiple of 4, c = 3 for rows <= 512 and 2 above, plus
 * a(8*k*rows*F) for a BF16 bank with E = 1 and rows <= 64 (split-K partial
 * sums, k = 4 halved while H is not a multiple of 128*k); a() rounds up to a
 * multiple of 256.  moe_workspace_bytes(T, H, E, F,
 * top_k) is always enough. */
int moe_grouped_w4a16_swiglu(const void* x, int T, int H,
                             const int32_t* expert_offsets, const int32_t* row_slot,
                             int top_k, const moe_qweight* gate, const moe_qweight* up,
                             float swiglu_limit, void* h_perm,
                             void* ws, size_t ws_bytes, moe_stream_t stream);

/* Grouped down projection with the routing weight fused ("Step 5 Preview:
 * 92 narrow layers...", The shape: the down projection of each routed SwiGLU
 * expert, [E, 4096, 1536] in the banks of "Step-5-Preview-Int4-g128", Tensor
 * layout / "Step-5-Preview-NVFP4-Local", Format; the token's output weighs
 * each routed expert by its renormalised sigmoid score, "Step-5-Preview-Spark",
 * At a glance):
 *     y_perm[r, :] = bf16( topk_w[row_slot[r]] * (h_perm[r] . Wd[e]^T) )
 * for rows r of expert e (fp32 accumulation).  h_perm: bf16 [rows, F];
 * topk_w: fp32 [rows] indexed by slot, or NULL for weight 1;
 * down: bank [E, H, F]; y_perm: bf16 [rows, H] (out).  The path follows the
 * gate/up call's rule with the roles of H and F exchanged (F a multiple of
 * 256, H of 128 for the GEMM).
 * ws (256-byte aligned): at least 1024 + a(16*(E+2)) + max(a(rows*F/8) +
 * a(2*rows*F), a(4*rows) + a(rows*(8*z+16)) + a(c*rows*F)) bytes, z = F/128
 * rounded up to a multiple of 4, c = 3 for rows <= 512 and 2 above, plus
 * a(4*k*rows*H) for a BF16 bank with E = 1 and rows <= 64 (k = 2 halved while
 * F is not a multiple of 128*k); a() rounds up to a multiple of 256.  moe_workspace_bytes(T, H, E, F, top_k) with
 * rows = T*top_k is always enough. */
int moe_grouped_w4a16_down(const void* h_perm, const int32_t* expert_offsets,
                           const int32_t* row_slot, const float* topk_w, int rows,
                           const moe_qweight* down, void* y_perm,
                           void* ws, size_t ws_bytes, moe_stream_t stream);

/* Unpermute and combine ("Step 5 Preview: 92 narrow layers...", The shape:
 * a token's output is its shared expert plus its 8 routed experts; the
 * routing weight was applied by the down projection):
 *     y[t, :] = bf16( shared_out[t, :] + sum_{j<top_k} y_perm[slot_row[t*top_k + j], :] )
 * summed in fp32 in the order shared, j = 0..top_k-1.  y_perm: bf16 [T*top_k, H];
 * shared_out: bf16 [T, H] or NULL; y: bf16 [T, H] (out). */
int moe_unpermute_combine(const void* y_perm, const int32_t* slot_row, int T,
                          int top_k, int H, const void* shared_out, void* y,
                          moe_stream_t stream);

/* The whole layer for decode-sized batches (1 <= T <= 64): router, bucketing,
 * gate/up + SwiGLU, down with routing weights, shared expert and combine, on
 * device with no host synchronisation ("Step-5-Preview-Spark", At a glance and
 * How it was made: the decode path of the layer, 8 routed experts plus one
 * shared per token; "Step 5 Preview: 92 narrow layers...", The shape).
 * x: bf16 [T, H]; y: bf16 [T, H] (out).  The shared expert runs on a
 * per-device side stream that the caller's stream forks to and joins; calls
 * from several host threads are safe with separate workspaces (their
 * shared-expert work is serialised on that side stream). */
int moe_layer_decode(const void* x, int T, const moe_layer* L, void* y,
                     void* ws, size_t ws_bytes, moe_stream_t stream);

/* The whole layer for any T >= 1 (prefill-sized batches use the tcgen05
 * grouped GEMM; "Step-5-Preview-Spark", Serving on 4 x DGX Spark, which
 * reports prefill and decode separately).  Same arguments and result as
 * moe_layer_decode; T = 0 does nothing and returns 0. */
int moe_layer_forward(const void* x, int T, const moe_layer* L, void* y,
                      void* ws, size_t ws_bytes, moe_stream_t stream);

/* A layer call recorded once as a CUDA graph and replayed (no page has a
 * counterpart: it removes the host's launch work from a decode step, which
 * on this path is a large share of the layer's time): the same kernels
 * as moe_layer_forward(x, T, L, y, ws, ws_bytes, .) with these exact
 * pointers, without the host's per-call launch work (argument checks, tensor
 * map encoding, about ten kernel launches).  The graph reads x and the banks
 * and writes y and ws at every launch, so the caller refills x in place
 * between launches and keeps every buffer (and the banks' contents, which may
 * change) alive until moe_layer_graph_destroy.  One launch at a time per
 * workspace.  create: checks as moe_layer_forward and refuses T = 0 (nothing
 * to record), records on a private
 * stream (the caller's stream is not touched), returns the handle in *out
 * (NULL on error).  launch: enqueues one layer on `stream`.  The recording
 * uses the per-device side stream of the shared expert, so create must not
 * overlap a layer call of another host thread on the same device. */
typedef struct moe_layer_graph_s* moe_layer_graph_t;
int moe_layer_graph_create(const void* x, int T, const moe_layer* L, void* y,
                           void* ws, size_t ws_bytes, moe_layer_graph_t* out);
int moe_layer_graph_launch(moe_layer_graph_t graph, moe_stream_t stream);
int moe_layer_graph_destroy(moe_layer_graph_t graph);

/* ---------------------------------------------------------------------- */
/* Weight conversion (offline step, not on the hot path)                   */
/* ---------------------------------------------------------------------- */

/* NVFP4 activation quantiser (W4A4 inputs, "Step-5-Preview-NVFP4-Local",
 * Modifications: quant_algo NVFP4, group size 16, with an input_scale): row r
 * of x (bf16 [rows, cols], cols % 16 == 0) with global g[r] (device fp32
 * [rows]): scales[r, b] = e4m3_rne_sat(amax_b / (6 g[r])), codes
 * e2m1_rne_sat(x / (e4m3(scale) g[r])); packed: u8 [rows, cols/2] (even
 * element in the low nibble), scales: u8 [rows, cols/16] (out).  The layer
 * paths quantise the same way inside their activation pre-pass. */
int moe_quantize_nvfp4_act(const void* x, int64_t rows, int64_t cols, const float* g,
                           uint8_t* packed, uint8_t* scales, moe_stream_t stream);

/* int4 symmetric g128 quantiser ("Step-5-Preview-Int4-g128", Recipe): per row
 * and group of 128, the scale is bf16((r * amax) / 7) for the clip ratio r in
 * {24/40, 25/40, ..., 40/40} that minimises sum (q*s - w)^2 (fp32, index
 * order; ties keep the larger ratio); q = clamp(rint(w / s), -8, 7).
 * w: bf16 [rows, cols] (cols % 128 == 0); packed: int32 [rows, cols/8] (out);
 * scales: bf16 [rows, cols/128] (out). */
int moe_quantize_int4_g128(const void* w, int64_t rows, int64_t cols, int32_t* packed,
                           void* scales, moe_stream_t stream);

/* NVFP4 quantiser ("Step-5-Preview-NVFP4-Local", Format): per matrix,
 * global = amax / (6 * 448) (fp32); per block of 16 along cols,
 * scale = e4m3_rne(amax_block / (6 * global)); code = e2m1_rne(w / (e4m3(scale) * global)).
 * w: bf16 [rows, cols] (one expert matrix, cols % 16 == 0); packed: uint8
 * [rows, cols/2] (out); scales: uint8 [rows, cols/16] (out); global_scale:
 * fp32 [1] (out).  ws: at least 256 bytes of zero-filled workspace. */
int moe_quantize_nvfp4(const void* w, int64_t rows, int64_t cols, uint8_t* packed,
                       uint8_t* scales, float* global_scale, void* ws, size_t ws_bytes,
                       moe_stream_t stream);

/* ---------------------------------------------------------------------- */
/* Compressed scale format of the NVFP4 block scales                       */
/* ---------------------------------------------------------------------- */

/* CSF ("Step-5-Preview-NVFP4-Local", Format): a scale tensor u8 [E, R, C]
 * (one E4M3 byte per 16 weights; gate/up R = 1536, C = 256, down R = 4096,
 * C = 96) is stored as
 *   fixed       u8 [E, R/16, 16 * (1 + C/2)]: a slab of 16 rows is their 16
 *               bases followed by their 4-bit codes (C/2 bytes per row, rows
 *               in order; column 2j in the low nibble of byte j);
 *   exceptions  u32 [n]: (row * C + col) | byte << 24 (row counts from 0 in
 *               each expert); expert 0's entries first, then expert 1's and
 *               so on, each expert's in increasing position;
 *   starts      i64 [E + 1]: expert e's entries are exceptions[starts[e],
 *               starts[e+1]).
 * Decoding: byte = base(row) + code, or the stored byte of an exception.  A
 * row's base is the smallest b in 0..240 that puts the largest number of the
 * row's bytes inside [b, b + 15]; the code stored under an exception is 0.
 * Requirements: R % 16 == 0, C even, R * C < 2^24, 1 <= E <= 1024. */

/* Expand CSF planes into scale bytes u8 [E, R, C] (scales, out), e.g. one
 * layer's scales into scratch before the layer runs, which is how the page's
 * loader uses the format ("Step-5-Preview-NVFP4-Local", Size).  expert_offsets:
 * int32 [E+1] of a routing (moe_permute), or NULL; when given, only experts
 * with at least one routed row are expanded and the other experts' bytes are
 * left as they were.  exceptions and starts are both given or both NULL (no
 * exceptions); an exception whose position is R * C or more is ignored.
 * Two kernels (expansion, then the exceptions), stream-ordered. */
int moe_csf_decode(const uint8_t* fixed, const uint32_t* exceptions, const int64_t* starts,
                   int E, int R, int C, const int32_t* expert_offsets, uint8_t* scales,
                   moe_stream_t stream);

/* Workspace bytes moe_csf_encode needs for E experts of R rows (0 if invalid). */
size_t moe_csf_encode_workspace_bytes(int E, int R);

/* Encode scale bytes u8 [E, R, C] into CSF ("Step-5-Preview-NVFP4-Local",
 * Format: per 16 rows a slab of row bases and 4-bit codes, exceptions where
 * a byte is not base + code; an offline step).  Always writes
 * fixed and starts (device memory); with exceptions non-NULL it also writes
 * the exceptions, at most exceptions_capacity of them (a larger count records
 * MOE_ERR_DEVICE_INDEX in the workspace status word).  To size the
 * exceptions, call once with exceptions = NULL and read starts[E].
 * ws: moe_csf_encode_workspace_bytes(E, R) bytes, 256-byte aligned, its first
 * 1024 bytes zero-filled (moe_workspace_init). */
int moe_csf_encode(const uint8_t* scales, int E, int R, int C, uint8_t* fixed, int64_t* starts,
                   uint32_t* exceptions, int64_t exceptions_capacity, void* ws, size_t ws_bytes,
                   moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_W4A16_H */
