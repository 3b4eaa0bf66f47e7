// Grouped expert GEMM (prefill).  Placeholder dispatch until the tcgen05
// kernel lands: runs the CUDA-core expert kernels over 16-token sub-chunks.
#include "common.cuh"
#include "kernels.h"

namespace moe {

size_t gemm_ws_bytes(int bits, int T, int k, int H, int I, int E) {
    (void)bits; (void)H; (void)E;
    return gemv_ws_bytes(T, k, I);
}

int launch_gemm(int bits, const uint8_t *const *blobs, const int32_t *offsets, const int32_t *active,
                const int32_t *perm_src, const void *x, int x_dtype, int T, int k, int H, int I, int E,
                const uint8_t *shared_blob, float *y_perm, float *y_shared, void *ws, unsigned *err, cudaStream_t s) {
    return launch_gemv(bits, blobs, offsets, active, perm_src, x, x_dtype, T, k, H, I, E, shared_blob, y_perm,
                       y_shared, ws, err, s);
}

}  // namespace moe
