// C ABI entry points of libmoe (declared in include/moe_w4a16.h): argument
// validation, workspace carving and kernel composition.  Nothing here touches
// the data; every step runs in the kernels of this library.
#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "moe_internal.cuh"

using namespace moe;

namespace {

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t cs(moe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

template <typename T>
inline T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(ws) + off);
}

int check_dims(int T, int H, int E, int F, int k) {
    if (T < 0 || H <= 0 || E <= 0 || F <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    if (H % 128 || F % 128 || k > kMaxTopK || E > kMaxE || k > E) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

int check_bank(const moe_qweight* b, int E, int out, int in) {
    if (!b) return MOE_ERR_INVALID_ARG;
    if (b->input_scale && b->fmt != MOE_FMT_NVFP4) return MOE_ERR_UNSUPPORTED;   // W4A4 is NVFP4 only
    if (b->fmt != MOE_FMT_INT4_G128 && b->fmt != MOE_FMT_NVFP4 && b->fmt != MOE_FMT_BF16)
        return MOE_ERR_UNSUPPORTED;
    if (b->num_experts != E || b->out_dim != out || b->in_dim != in) return MOE_ERR_INVALID_ARG;
    if (in % 128 || out <= 0) return MOE_ERR_UNSUPPORTED;
    if (!b->packed || !al16(b->packed)) return MOE_ERR_INVALID_ARG;
    if (b->fmt != MOE_FMT_BF16 && !b->scales) return MOE_ERR_INVALID_ARG;
    if (b->fmt == MOE_FMT_NVFP4 && !b->global_scale) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

int check_ws(void* ws, size_t ws_bytes, size_t need) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_WORKSPACE;
    if (ws_bytes < need) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

#define MOE_TRY(x)                     \
    do {                               \
        int _rc = (x);                 \
        if (_rc != MOE_OK) return _rc; \
    } while (0)

// Routed experts run on the tcgen05 grouped GEMM whenever its shape rules
// hold (input dimension a multiple of 256, output a multiple of 128), at any
// batch size; other shapes take the streaming GEMV.  The BF16 shared expert at
// a small batch splits K across tiles (shared_ksplit) so that its weight
// stream spreads over the GPU; partial is split_bytes() of scratch for that.
bool gemm_shape_ok(int in_dim, int out_dim) { return in_dim % 256 == 0 && out_dim % 128 == 0; }

// The grouped GEMM raises its kernel's shared-memory attribute the first time a launch needs more; two host
// threads doing that at once for one kernel could leave the smaller value set last.  Every grouped GEMM
// launch of this library is therefore made under one process-wide lock (host launch work only: nothing
// waits on the GPU while it is held).
int grouped_gemm(const GemvProblem& p, bool gateup, int rows, const GemmBuffers& b, cudaStream_t s) {
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    return launch_grouped_gemm(p, gateup, rows, b, s);
}

int run_problem(const GemvProblem& p, bool gateup, int rows, int act_rows, void* prep, const GemmBuffers& gb,
                float* partial, cudaStream_t s) {
    if (!gemm_shape_ok(p.in_dim, p.out_dim)) {
        if (p.in_scale) return MOE_ERR_UNSUPPORTED;     // W4A4 runs on the GEMM only
        return launch_stream_gemv(p, nullptr, gateup, act_rows, prep, s, true);
    }
    GemmBuffers b = gb;
    b.ksplit = shared_ksplit(p.E, p.fmt, gateup, rows, p.in_dim);
    b.partial = partial;
    b.tile_cnt = p.status + 16;            // the control block's split-K counters
    return grouped_gemm(p, gateup, rows, b, s);
}

// The step-level calls' scratch: the GEMV or GEMM pre-pass of rows rows, then
// the shared expert's split-K partial sums.
// GEMM pre-pass layout in a scratch region of gemm_prep_bytes(rows, in_dim):
// row scales [rows], row records [rows][zrow_floats(in_dim)] (8-bit int4),
// gathered rows.
GemmBuffers gemm_buffers(void* base, int rows, int in_dim, bool act_ready, bool i8) {
    uint8_t* p = reinterpret_cast<uint8_t*>(base);
    GemmBuffers b{};
    b.scale_buf = reinterpret_cast<float*>(p);
    b.zbuf = reinterpret_cast<float*>(p + align256(size_t(rows) * 4));
    b.act_buf = p + align256(size_t(rows) * 4) + align256(size_t(rows) * zrow_floats(in_dim) * 4);
    b.act_ready = act_ready;
    b.i8 = i8;
    return b;
}
bool i8_int4(const GemvProblem& p, int rows) {
    return p.fmt == MOE_FMT_INT4_G128 && p.E > 1 && rows <= kI8Int4MaxRows;
}
size_t step_scratch(int E, int fmt, bool gateup, int rows, int in_dim, int out_dim) {
    return grouped_scratch(E, rows, in_dim) + split_bytes(shared_ksplit(E, fmt, gateup, rows, in_dim), gateup, rows, out_dim);
}
float* step_partial(void* ws, int E, int rows, int in_dim) {
    return at<float>(ws, kStepScratch + grouped_scratch(E, rows, in_dim));
}

int layer_checks(const void* x, int T, const moe_layer* L, void* y, void* ws, size_t ws_bytes) {
    if (!L) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_dims(T, L->H, L->E, L->F, L->top_k));
    if (T == 0) return MOE_OK;
    if (!x || !y) return MOE_ERR_INVALID_ARG;
    if (!al16(x) || !al16(y) || !L->router_w || !al16(L->router_w)) return MOE_ERR_INVALID_ARG;
    if (L->swiglu_limit != 0.0f) return MOE_ERR_UNSUPPORTED;
    MOE_TRY(check_bank(&L->gate, L->E, L->F, L->H));
    MOE_TRY(check_bank(&L->up, L->E, L->F, L->H));
    MOE_TRY(check_bank(&L->down, L->E, L->H, L->F));
    if (L->gate.fmt == MOE_FMT_BF16 || L->gate.fmt != L->up.fmt || L->gate.fmt != L->down.fmt)
        return MOE_ERR_UNSUPPORTED;
    if (L->act_f16 && !(gemm_shape_ok(L->H, L->F) && gemm_shape_ok(L->F, L->H))) return MOE_ERR_UNSUPPORTED;
    // gate and up share one quantised activation (the gate's input scale)
    if (L->up.input_scale && L->up.input_scale != L->gate.input_scale) return MOE_ERR_UNSUPPORTED;
    if ((L->gate.input_scale || L->down.input_scale) && !(gemm_shape_ok(L->H, L->F) && gemm_shape_ok(L->F, L->H)))
        return MOE_ERR_UNSUPPORTED;
    const bool has_sh = L->sh_gate.packed || L->sh_up.packed || L->sh_down.packed;
    if (has_sh) {
        MOE_TRY(check_bank(&L->sh_gate, 1, L->F, L->H));
        MOE_TRY(check_bank(&L->sh_up, 1, L->F, L->H));
        MOE_TRY(check_bank(&L->sh_down, 1, L->H, L->F));
        if (L->sh_gate.fmt != MOE_FMT_BF16 || L->sh_up.fmt != MOE_FMT_BF16 || L->sh_down.fmt != MOE_FMT_BF16)
            return MOE_ERR_UNSUPPORTED;
    }
    return check_ws(ws, ws_bytes, ws_layout(T, L->H, L->E, L->F, L->top_k).total);
}

// A non-blocking stream per device for the shared expert, with fork/join
// events, created on first use.  A layer call holds `call` from its fork
// record until its stream's wait on the join event is enqueued, so calls
// from several host threads cannot interleave their records on the shared
// events (their shared-expert work then runs one after another on the side
// stream).
struct SideStream {
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    std::mutex call;
};
int side_stream(SideStream** out) {
    static std::mutex mu;
    static SideStream per_dev[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    SideStream& st = per_dev[dev];
    if (!st.s) {
        if (cudaStreamCreateWithFlags(&st.s, cudaStreamNonBlocking) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaEventCreateWithFlags(&st.fork, cudaEventDisableTiming) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaEventCreateWithFlags(&st.join, cudaEventDisableTiming) != cudaSuccess) return MOE_ERR_CUDA;
    }
    *out = &st;
    return MOE_OK;
}

// SMs the BF16 shared expert's GEMMs may take at decode sizes (T <= 16), beside the routed chain
// (measured on the decode workloads: 32 to 148 give the layer within 1 %, 64 the best).
constexpr int kSharedDecodeCtas = 64;

int layer_run(const void* x, int T, const moe_layer* L, void* y, void* ws, cudaStream_t s) {
    const int H = L->H, E = L->E, F = L->F, k = L->top_k;
    const WsLayout W = ws_layout(T, H, E, F, k);
    const int R = T * k;
    int32_t* status = at<int32_t>(ws, W.ctrl);
    int32_t* ids = at<int32_t>(ws, W.ids);
    float* tw = at<float>(ws, W.tw);
    int32_t* offsets = at<int32_t>(ws, W.offsets);
    int32_t* row_slot = at<int32_t>(ws, W.row_slot);
    int32_t* slot_row = at<int32_t>(ws, W.slot_row);
    __nv_bfloat16* h_perm = at<__nv_bfloat16>(ws, W.h_perm);
    __nv_bfloat16* y_perm = at<__nv_bfloat16>(ws, W.y_perm);
    __nv_bfloat16* ys = at<__nv_bfloat16>(ws, W.ys);
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);

    const bool has_sh = L->sh_gate.packed != nullptr;
    const int x_f16 = L->act_f16 ? 1 : 0;
    int32_t* sh_off = at<int32_t>(ws, W.sh_offsets);
    int32_t* sh_rs = at<int32_t>(ws, W.sh_rowslot);
    int32_t* counter = status + 1;
    void* prep = at<void>(ws, W.prep);
    __nv_bfloat16* h_sh = h_perm + size_t(R) * F;

    // The shared expert needs x only: it runs on a side stream while the
    // router, the bucketing and the routed experts run on `s`, and `s` waits
    // for it before the combine.  The routed chain is launched first (it is
    // the critical path, and the host's launch work for the shared expert would
    // otherwise delay it); the shared expert's own routing (offsets {0, T}, row
    // i at slot i * top_k) comes first on its stream.  At decode sizes its GEMMs
    // take at most kSharedDecodeCtas SMs and no early launch, so that no waiting
    // CTA holds an SM; the routed GEMMs hand out their tiles dynamically around
    // them.
    SideStream* side = nullptr;
    std::unique_lock<std::mutex> side_lock;
    // An error return after the fork still joins the side stream back into `s` (and so into a recording
    // in progress), before the lock is released; the normal path joins explicitly and disarms it.
    struct JoinOnExit {
        SideStream* side = nullptr;
        cudaStream_t s = nullptr;
        ~JoinOnExit() {
            if (side && cudaEventRecord(side->join, side->s) == cudaSuccess) cudaStreamWaitEvent(s, side->join, 0);
        }
    } join_on_exit;
    if (has_sh) {
        MOE_TRY(side_stream(&side));
        side_lock = std::unique_lock<std::mutex>(side->call);
        if (cudaEventRecord(side->fork, s) != cudaSuccess || cudaStreamWaitEvent(side->s, side->fork, 0) != cudaSuccess)
            return MOE_ERR_CUDA;
        join_on_exit.side = side;
        join_on_exit.s = s;
    }

    if (T <= kRouterDecodeMaxT && router_decode_ok(H)) {
        // router, top-k and bucketing in one launch
        RouterDecodeArgs ra{};
        ra.x = xb; ra.T = T; ra.H = H; ra.Wr = L->router_w; ra.bias = L->router_bias; ra.E = E; ra.k = k;
        ra.logits = at<float>(ws, W.logits); ra.ids = ids; ra.w = tw; ra.counter = counter; ra.status = status;
        ra.offsets = offsets; ra.row_slot = row_slot; ra.slot_row = slot_row;
        ra.sh_offsets = nullptr; ra.sh_rowslot = nullptr; ra.x_f16 = x_f16;
        MOE_TRY(launch_route_decode(ra, s));
    } else {
        MOE_TRY(launch_route(xb, T, H, L->router_w, L->router_bias, E, k, ids, tw, at<float>(ws, W.logits),
                             at<__nv_bfloat16>(ws, W.wsplit), status, counter, s, x_f16));
        MOE_TRY(launch_permute(ids, T, k, E, offsets, row_slot, slot_row, at<int32_t>(ws, W.hist), status, s));
    }

    const bool routed_gemm = gemm_shape_ok(H, F) && gemm_shape_ok(F, H);

    GemvProblem gu{};
    gu.act = xb; gu.act_by_token = 1; gu.top_k = k; gu.offsets = offsets; gu.row_slot = row_slot;
    gu.E = E; gu.topk_w = nullptr; gu.fmt = L->gate.fmt; gu.out_dim = F; gu.in_dim = H;
    gu.p0 = L->gate.packed; gu.s0 = L->gate.scales; gu.g0 = L->gate.global_scale;
    gu.p1 = L->up.packed; gu.s1 = L->up.scales; gu.g1 = L->up.global_scale;
    gu.out = h_perm; gu.status = status; gu.in_scale = L->gate.input_scale; gu.act_f16 = x_f16;
    GemvProblem dn{};
    dn.act = h_perm; dn.act_by_token = 0; dn.top_k = k; dn.offsets = offsets; dn.row_slot = row_slot;
    dn.E = E; dn.topk_w = tw; dn.fmt = L->down.fmt; dn.out_dim = H; dn.in_dim = F;
    dn.p0 = L->down.packed; dn.s0 = L->down.scales; dn.g0 = L->down.global_scale;
    dn.out = y_perm; dn.status = status; dn.in_scale = L->down.input_scale;
    // routed experts: both projections on one path
    const bool i8 = routed_gemm && i8_int4(gu, R);
    if (routed_gemm) {
        // 16-bit gate/up activation rows are gathered into the y_perm region,
        // free until the down projection writes it
        GemmBuffers gb = gemm_buffers(prep, R, H, false, i8);
        gb.sched = status + 8;             // tiles handed out as CTAs get SMs (the shared expert may hold some)
        gb.max_expert_rows = T;            // a token routes to an expert at most once
        if (!i8) gb.act_buf = y_perm;
        MOE_TRY(grouped_gemm(gu, true, R, gb, s));
    } else {
        MOE_TRY(launch_stream_gemv(gu, nullptr, true, T, prep, s, true));
    }
    if (routed_gemm) {
        GemmBuffers db = gemm_buffers(prep, R, F, false, i8);
        db.sched = status + 8;
        db.max_expert_rows = T;
        MOE_TRY(grouped_gemm(dn, false, R, db, s));
    } else {
        MOE_TRY(launch_stream_gemv(dn, nullptr, false, R, prep, s, true));
    }
    if (has_sh) {
        // fp16 mode: the BF16 shared expert reads x rounded to bf16, staged in its output region (the
        // down projection overwrites it only after the gate/up projection has read it)
        const __nv_bfloat16* xs = xb;
        if (x_f16) {
            MOE_TRY(launch_f16_to_bf16(reinterpret_cast<const __half*>(x), ys, size_t(T) * H, side->s));
            xs = ys;
        }
        GemvProblem sg{};
        sg.act = xs; sg.act_by_token = 1; sg.top_k = k; sg.offsets = sh_off; sg.row_slot = sh_rs;
        sg.E = 1; sg.fmt = MOE_FMT_BF16; sg.out_dim = F; sg.in_dim = H;
        sg.p0 = L->sh_gate.packed; sg.p1 = L->sh_up.packed; sg.out = h_sh; sg.status = status;
        GemvProblem sd{};
        sd.act = h_sh; sd.act_by_token = 0; sd.top_k = k; sd.offsets = sh_off; sd.row_slot = sh_rs;
        sd.E = 1; sd.fmt = MOE_FMT_BF16; sd.out_dim = H; sd.in_dim = F;
        sd.p0 = L->sh_down.packed; sd.out = ys; sd.status = status;
        // the shared expert reads x and its own h directly (identity routing, natural order)
        GemmBuffers direct{};
        direct.act_ready = 1;
        direct.max_expert_rows = T;
        if (T <= kRouterDecodeMaxT) {
            direct.max_ctas = kSharedDecodeCtas;
            direct.no_pdl = 1;
        }
        float* shpart = at<float>(ws, W.shpart);
        MOE_TRY(launch_shared_routing(T, k, sh_off, sh_rs, side->s));
        MOE_TRY(run_problem(sg, true, T, T, nullptr, direct, shpart, side->s));
        MOE_TRY(run_problem(sd, false, T, T, nullptr, direct, shpart, side->s));
        join_on_exit.side = nullptr;
        if (cudaEventRecord(side->join, side->s) != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (has_sh && cudaStreamWaitEvent(s, side->join, 0) != cudaSuccess) return MOE_ERR_CUDA;

    // after a join with the side stream the combine starts only when both inputs are complete (no
    // early launch of a dependent grid across an event wait)
    return launch_combine(y_perm, slot_row, T, k, H, has_sh ? ys : nullptr,
                          reinterpret_cast<__nv_bfloat16*>(y), s, !has_sh, x_f16);
}

}  // namespace

namespace moe {
namespace {
std::atomic<uint64_t> g_launches{0};
thread_local uint64_t t_launches = 0;      // this thread's share, so a recording can take back its own
}
void count_launch() {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    t_launches++;
}
}  // namespace moe

extern "C" {

size_t moe_workspace_bytes(int T, int H, int E, int F, int top_k) {
    if (check_dims(T, H, E, F, top_k) != MOE_OK) return 0;
    return ws_layout(std::max(T, 1), H, E, F, top_k).total;
}

int moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (!ws) return MOE_ERR_INVALID_ARG;
    return cudaMemsetAsync(ws, 0, ws_bytes, cs(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_read_status(void* ws, moe_stream_t stream, int32_t* status_out) {
    if (!ws || !status_out) return MOE_ERR_INVALID_ARG;
    int32_t v = 0;
    if (cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, cs(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(cs(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    *status_out = v;
    if (v != 0) {
        // a kernel that stopped early may have left its arrival counters (router word 1, tile
        // scheduler words 8-9, split-K words 16..255) non-zero: clear them with the status word
        if (cudaMemsetAsync(ws, 0, 8, cs(stream)) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemsetAsync(at<int32_t>(ws, 32), 0, 8, cs(stream)) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemsetAsync(at<int32_t>(ws, 64), 0, kStepScratch - 64, cs(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

int moe_set_wait_limit(void* ws, uint64_t limit_ns, moe_stream_t stream) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_WORKSPACE;
    return launch_set_u64(at<unsigned long long>(ws, 16), limit_ns, cs(stream));
}

int moe_set_wait_hold(void* ws, int hold, moe_stream_t stream) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_WORKSPACE;
    return launch_set_u32(at<uint32_t>(ws, 24), hold ? 1u : 0u, cs(stream));
}

uint64_t moe_launch_count(void) { return moe::g_launches.load(std::memory_order_relaxed); }

const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape or format";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_TIMEOUT: return "device wait timed out";
        case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case MOE_ERR_DEVICE_INDEX: return "index out of range on device";
        case MOE_ERR_NONFINITE: return "non-finite activation on device";
    }
    return "unknown status";
}

int moe_route_topk(const void* x, int T, int H, const float* router_w, const float* router_bias,
                   int E, int top_k, int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes,
                   moe_stream_t stream) {
    if (T < 0 || H <= 0 || E <= 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
    if (H % 128 || E > kMaxE || top_k > kMaxTopK || top_k > E) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!x || !router_w || !topk_ids || !topk_w || !al16(x) || !al16(router_w)) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_ws(ws, ws_bytes, kStepScratch + route_scratch(T, E, H)));
    return launch_route(reinterpret_cast<const __nv_bfloat16*>(x), T, H, router_w, router_bias, E,
                        top_k, topk_ids, topk_w, at<float>(ws, kStepScratch),
                        at<__nv_bfloat16>(ws, kStepScratch + align256(size_t(T) * E * 4)), at<int32_t>(ws, 0),
                        at<int32_t>(ws, 4), cs(stream));
}

int moe_permute(const int32_t* topk_ids, int T, int top_k, int E, int32_t* expert_offsets,
                int32_t* row_slot, int32_t* slot_row, void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (T < 0 || top_k <= 0 || E <= 0) return MOE_ERR_INVALID_ARG;
    if (E > kMaxE || top_k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
    if (!expert_offsets) return MOE_ERR_INVALID_ARG;
    if (T == 0) {
        return cudaMemsetAsync(expert_offsets, 0, size_t(E + 1) * 4, cs(stream)) == cudaSuccess
                   ? MOE_OK : MOE_ERR_CUDA;
    }
    if (!topk_ids || !row_slot || !slot_row) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_ws(ws, ws_bytes, kStepScratch + permute_scratch(T, top_k, E)));
    return launch_permute(topk_ids, T, top_k, E, expert_offsets, row_slot, slot_row,
                          at<int32_t>(ws, kStepScratch), at<int32_t>(ws, 0), cs(stream));
}

int moe_permute_noalloc(const int32_t* topk_ids, int T, int top_k, int E, int32_t* expert_offsets,
                        int32_t* row_slot, int32_t* slot_row, moe_stream_t stream) {
    if (T < 0 || top_k <= 0 || E <= 0) return MOE_ERR_INVALID_ARG;
    if (E > kMaxE || top_k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
    if (!expert_offsets) return MOE_ERR_INVALID_ARG;
    if (T == 0) {
        return cudaMemsetAsync(expert_offsets, 0, size_t(E + 1) * 4, cs(stream)) == cudaSuccess
                   ? MOE_OK : MOE_ERR_CUDA;
    }
    if (!topk_ids || !row_slot || !slot_row) return MOE_ERR_INVALID_ARG;
    return launch_permute_noalloc(topk_ids, T, top_k, E, expert_offsets, row_slot, slot_row, cs(stream));
}

int moe_grouped_w4a16_swiglu(const void* x, int T, int H, const int32_t* expert_offsets,
                             const int32_t* row_slot, int top_k, const moe_qweight* gate,
                             const moe_qweight* up, float swiglu_limit, void* h_perm, void* ws,
                             size_t ws_bytes, moe_stream_t stream) {
    if (T < 0 || H <= 0 || top_k <= 0 || !gate || !up) return MOE_ERR_INVALID_ARG;
    if (swiglu_limit != 0.0f) return MOE_ERR_UNSUPPORTED;
    if (top_k > kMaxTopK || H % 128) return MOE_ERR_UNSUPPORTED;
    const int E = gate->num_experts, F = gate->out_dim;
    if (E <= 0 || E > kMaxE) return MOE_ERR_UNSUPPORTED;
    MOE_TRY(check_bank(gate, E, F, H));
    MOE_TRY(check_bank(up, E, F, H));
    if (gate->fmt != up->fmt || F % 128) return MOE_ERR_UNSUPPORTED;
    if (up->input_scale && up->input_scale != gate->input_scale) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!x || !al16(x) || !expert_offsets || !row_slot || !h_perm || !al16(h_perm)) return MOE_ERR_INVALID_ARG;
    // rows present: T * top_k routed slots, or T for a single shared expert
    const int rows = (E == 1) ? T : T * top_k;
    MOE_TRY(check_ws(ws, ws_bytes, kStepScratch + step_scratch(E, gate->fmt, true, rows, H, F)));
    GemvProblem p{};
    p.act = reinterpret_cast<const __nv_bfloat16*>(x); p.act_by_token = 1; p.top_k = top_k;
    p.offsets = expert_offsets; p.row_slot = row_slot; p.E = E; p.fmt = gate->fmt;
    p.out_dim = F; p.in_dim = H;
    p.p0 = gate->packed; p.s0 = gate->scales; p.g0 = gate->global_scale;
    p.p1 = up->packed; p.s1 = up->scales; p.g1 = up->global_scale;
    p.out = reinterpret_cast<__nv_bfloat16*>(h_perm); p.status = at<int32_t>(ws, 0);
    p.in_scale = gate->input_scale;
    void* prep = at<void>(ws, kStepScratch + align256(size_t(E + 2) * 16));
    GemmBuffers b = gemm_buffers(prep, rows, H, false, i8_int4(p, rows));
    b.sched = p.status + 8;
    b.max_expert_rows = T;
    return run_problem(p, true, rows, T, prep, b, step_partial(ws, E, rows, H), cs(stream));
}

int moe_grouped_w4a16_down(const void* h_perm, const int32_t* expert_offsets, const int32_t* row_slot,
                           const float* topk_w, int rows, const moe_qweight* down, void* y_perm,
                           void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (rows < 0 || !down) return MOE_ERR_INVALID_ARG;
    const int E = down->num_experts, H = down->out_dim, F = down->in_dim;
    if (E <= 0 || E > kMaxE) return MOE_ERR_UNSUPPORTED;
    MOE_TRY(check_bank(down, E, H, F));
    if (H % 128) return MOE_ERR_UNSUPPORTED;
    if (rows == 0) return MOE_OK;
    if (!h_perm || !al16(h_perm) || !expert_offsets || !row_slot || !y_perm || !al16(y_perm))
        return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_ws(ws, ws_bytes, kStepScratch + step_scratch(E, down->fmt, false, rows, F, H)));
    GemvProblem p{};
    p.act = reinterpret_cast<const __nv_bfloat16*>(h_perm); p.act_by_token = 0; p.top_k = 1;
    p.offsets = expert_offsets; p.row_slot = row_slot; p.E = E; p.topk_w = topk_w;
    p.fmt = down->fmt; p.out_dim = H; p.in_dim = F;
    p.p0 = down->packed; p.s0 = down->scales; p.g0 = down->global_scale;
    p.out = reinterpret_cast<__nv_bfloat16*>(y_perm); p.status = at<int32_t>(ws, 0);
    p.in_scale = down->input_scale;
    void* prep = at<void>(ws, kStepScratch + align256(size_t(E + 2) * 16));
    // BF16 rows are read in place (row r is activation row r)
    GemmBuffers b = gemm_buffers(prep, rows, F, down->fmt == MOE_FMT_BF16, i8_int4(p, rows));
    b.sched = p.status + 8;
    b.max_expert_rows = rows;
    return run_problem(p, false, rows, rows, prep, b, step_partial(ws, E, rows, F), cs(stream));
}

int moe_unpermute_combine(const void* y_perm, const int32_t* slot_row, int T, int top_k, int H,
                          const void* shared_out, void* y, moe_stream_t stream) {
    if (T < 0 || top_k <= 0 || H <= 0) return MOE_ERR_INVALID_ARG;
    if (H % 128 || top_k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!y_perm || !slot_row || !y || !al16(y_perm) || !al16(y) || (shared_out && !al16(shared_out)))
        return MOE_ERR_INVALID_ARG;
    return launch_combine(reinterpret_cast<const __nv_bfloat16*>(y_perm), slot_row, T, top_k, H,
                          reinterpret_cast<const __nv_bfloat16*>(shared_out),
                          reinterpret_cast<__nv_bfloat16*>(y), cs(stream));
}

int moe_layer_decode(const void* x, int T, const moe_layer* L, void* y, void* ws, size_t ws_bytes,
                     moe_stream_t stream) {
    MOE_TRY(layer_checks(x, T, L, y, ws, ws_bytes));
    if (T > kMaxDecodeT) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    return layer_run(x, T, L, y, ws, cs(stream));
}

int moe_layer_forward(const void* x, int T, const moe_layer* L, void* y, void* ws, size_t ws_bytes,
                      moe_stream_t stream) {
    MOE_TRY(layer_checks(x, T, L, y, ws, ws_bytes));
    if (T == 0) return MOE_OK;
    return layer_run(x, T, L, y, ws, cs(stream));
}

}  // extern "C"

struct moe_layer_graph_s {
    cudaGraphExec_t exec = nullptr;
    uint64_t kernels = 0;             // kernel nodes: added to the launch count at every replay
};

extern "C" {

int moe_layer_graph_create(const void* x, int T, const moe_layer* L, void* y, void* ws, size_t ws_bytes,
                           moe_layer_graph_t* out) {
    if (!out) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    MOE_TRY(layer_checks(x, T, L, y, ws, ws_bytes));
    if (T == 0) return MOE_ERR_INVALID_ARG;
    if (L->sh_gate.packed) {                 // the side stream and its events exist before the recording
        SideStream* side = nullptr;
        MOE_TRY(side_stream(&side));
    }
    cudaStream_t cap = nullptr;
    if (cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking) != cudaSuccess) return MOE_ERR_CUDA;
    const uint64_t counted_before = moe::t_launches;
    cudaGraph_t graph = nullptr;
    int rc = MOE_OK;
    if (cudaStreamBeginCapture(cap, cudaStreamCaptureModeRelaxed) != cudaSuccess) {
        rc = MOE_ERR_CUDA;
    } else {
        rc = layer_run(x, T, L, y, ws, cap);
        // the capture is ended whatever happened inside it
        if (cudaStreamEndCapture(cap, &graph) != cudaSuccess && rc == MOE_OK) rc = MOE_ERR_CUDA;
    }
    moe_layer_graph_s* g = nullptr;
    if (rc == MOE_OK) {
        g = new moe_layer_graph_s();
        size_t n = 0;
        if (cudaGraphGetNodes(graph, nullptr, &n) != cudaSuccess) rc = MOE_ERR_CUDA;
        std::vector<cudaGraphNode_t> nodes(n);
        if (rc == MOE_OK && n && cudaGraphGetNodes(graph, nodes.data(), &n) != cudaSuccess) rc = MOE_ERR_CUDA;
        for (size_t i = 0; rc == MOE_OK && i < n; i++) {
            cudaGraphNodeType t;
            if (cudaGraphNodeGetType(nodes[i], &t) != cudaSuccess) rc = MOE_ERR_CUDA;
            else if (t == cudaGraphNodeTypeKernel) g->kernels++;
        }
        if (rc == MOE_OK && cudaGraphInstantiate(&g->exec, graph, 0) != cudaSuccess) rc = MOE_ERR_CUDA;
    }
    if (graph) cudaGraphDestroy(graph);
    cudaStreamDestroy(cap);
    // the launches recorded above ran nothing, whether or not the recording succeeded: take them back (the
    // graph's kernels are counted when it is launched)
    moe::g_launches.fetch_sub(moe::t_launches - counted_before, std::memory_order_relaxed);
    moe::t_launches = counted_before;
    if (rc != MOE_OK) {
        cudaGetLastError();
        delete g;
        return rc;
    }
    *out = g;
    return MOE_OK;
}

int moe_layer_graph_launch(moe_layer_graph_t graph, moe_stream_t stream) {
    if (!graph || !graph->exec) return MOE_ERR_INVALID_ARG;
    if (cudaGraphLaunch(graph->exec, cs(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    moe::g_launches.fetch_add(graph->kernels, std::memory_order_relaxed);
    return MOE_OK;
}

int moe_layer_graph_destroy(moe_layer_graph_t graph) {
    if (!graph) return MOE_OK;
    const int rc = (graph->exec && cudaGraphExecDestroy(graph->exec) != cudaSuccess) ? MOE_ERR_CUDA : MOE_OK;
    delete graph;
    return rc;
}

int moe_csf_decode(const uint8_t* fixed, const uint32_t* exceptions, const int64_t* starts, int E, int R, int C,
                   const int32_t* expert_offsets, uint8_t* scales, moe_stream_t stream) {
    if (E <= 0 || R <= 0 || C <= 0) return MOE_ERR_INVALID_ARG;
    if (E > kMaxE || R % 16 || C % 2 || int64_t(R) * C >= (int64_t(1) << 24)) return MOE_ERR_UNSUPPORTED;
    if (!fixed || !scales || (!exceptions) != (!starts)) return MOE_ERR_INVALID_ARG;
    return launch_csf_decode(fixed, exceptions, starts, E, R, C, expert_offsets, scales, cs(stream));
}

size_t moe_csf_encode_workspace_bytes(int E, int R) {
    if (E <= 0 || R <= 0 || E > kMaxE) return 0;
    return kStepScratch + csf_encode_scratch(E, R);
}

int moe_csf_encode(const uint8_t* scales, int E, int R, int C, uint8_t* fixed, int64_t* starts,
                   uint32_t* exceptions, int64_t exceptions_capacity, void* ws, size_t ws_bytes,
                   moe_stream_t stream) {
    if (E <= 0 || R <= 0 || C <= 0 || exceptions_capacity < 0) return MOE_ERR_INVALID_ARG;
    if (E > kMaxE || R % 16 || C % 2 || int64_t(R) * C >= (int64_t(1) << 24)) return MOE_ERR_UNSUPPORTED;
    if (!scales || !fixed || !starts) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_ws(ws, ws_bytes, kStepScratch + csf_encode_scratch(E, R)));
    int32_t* rowcnt = at<int32_t>(ws, kStepScratch);
    int64_t* tot = at<int64_t>(ws, kStepScratch + align256(size_t(E) * R * 4));
    return launch_csf_encode(scales, E, R, C, fixed, starts, exceptions, exceptions_capacity, rowcnt, tot,
                             at<int32_t>(ws, 0), cs(stream));
}

int moe_quantize_int4_g128(const void* w, int64_t rows, int64_t cols, int32_t* packed, void* scales,
                           moe_stream_t stream) {
    if (rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
    if (cols % 128) return MOE_ERR_UNSUPPORTED;
    if (rows == 0 || cols == 0) return MOE_OK;
    if (!w || !packed || !scales || !al16(w) || !al16(packed)) return MOE_ERR_INVALID_ARG;
    return launch_quant_int4(reinterpret_cast<const __nv_bfloat16*>(w), rows, cols, packed,
                             reinterpret_cast<__nv_bfloat16*>(scales), cs(stream));
}

int moe_quantize_nvfp4_act(const void* x, int64_t rows, int64_t cols, const float* g, uint8_t* packed,
                           uint8_t* scales, moe_stream_t stream) {
    if (rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
    if (cols % 16) return MOE_ERR_UNSUPPORTED;
    if (rows == 0 || cols == 0) return MOE_OK;
    if (!x || !g || !packed || !scales) return MOE_ERR_INVALID_ARG;
    return launch_quant_nvfp4_act(reinterpret_cast<const __nv_bfloat16*>(x), rows, cols, g, packed, scales,
                                  cs(stream));
}

int moe_quantize_nvfp4(const void* w, int64_t rows, int64_t cols, uint8_t* packed, uint8_t* scales,
                       float* global_scale, void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
    if (cols % 16) return MOE_ERR_UNSUPPORTED;
    if (rows == 0 || cols == 0) return MOE_OK;
    if (!w || !packed || !scales || !global_scale || !al16(w)) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_ws(ws, ws_bytes, 256));                 // uses only the control block's amax word
    return launch_quant_nvfp4(reinterpret_cast<const __nv_bfloat16*>(w), rows, cols, packed, scales,
                              global_scale, at<uint32_t>(ws, 8), cs(stream));
}

}  // extern "C"
