// tl_gemm.cuh -- batched / prefill ternary linear layer (M >= 16).
#pragma once
#include "tl_common.cuh"

namespace tlk {

inline int launch_gemm(int fmt, const uint8_t *dT, int64_t ldp, float alpha, const uint16_t *dX,
                       int64_t ldx, uint16_t *dY, int64_t ldy, int M, int N, int K,
                       cudaStream_t stream, int *last_cuda_error) {
    (void)fmt; (void)dT; (void)ldp; (void)alpha; (void)dX; (void)ldx; (void)dY; (void)ldy;
    (void)M; (void)N; (void)K; (void)stream; (void)last_cuda_error;
    return 7;  // TL_ERR_UNSUPPORTED until the tensor-core kernel lands
}

}  // namespace tlk
