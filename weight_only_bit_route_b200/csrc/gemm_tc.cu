// Prefill-shaped grouped GEMM entry.  Until the tcgen05 kernel is in place the
// streaming GEMV serves every size (it loops over rows in passes of two).
#include "moe_internal.cuh"

namespace moe {

int launch_grouped_gemm(const GemvProblem& routed, const GemvProblem* shared, bool gateup, int act_rows,
                        void* prep_ws, int32_t* tile_ws, cudaStream_t s) {
    (void)tile_ws;
    return launch_stream_gemv(routed, shared, gateup, act_rows, prep_ws, s, false);
}

}  // namespace moe
