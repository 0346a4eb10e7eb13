// Prefill path (M > 16). Placeholder: runs the decode GEMV on 16-row chunks of x.
#include "tern_internal.cuh"

namespace tern {

size_t gemm_workspace_bytes(const tern_weight& w, int64_t M) {
    return gemv_workspace_bytes(w, M < 16 ? M : 16);
}

tern_status gemm_launch(const tern_weight& w, const __half* x, int64_t M, __half* y, void* workspace,
                        cudaStream_t stream) {
    for (int64_t m0 = 0; m0 < M; m0 += 16) {
        const int mc = int(M - m0 < 16 ? M - m0 : 16);
        const tern_status st = gemv_launch(w, x + m0 * w.K, mc, y + m0 * w.N, static_cast<float*>(workspace), stream);
        if (st != TERN_OK) return st;
    }
    return TERN_OK;
}

}  // namespace tern
