// Internal launchers of libmoe (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

void launch_router_logits(const void *x, int x_dtype, const void *w, int w_dtype, const float *bias, int T, int H,
                          int E, float *out, cudaStream_t s);
bool router_mma_supported(int x_dtype, int w_dtype, int T, int H);
int launch_router_mma(const void *x, const void *w, const float *bias, int T, int H, int E, float *out,
                      unsigned *err, cudaStream_t s);
void launch_topk(const float *logits, int T, int E, int k, int32_t *ids, float *w, unsigned *err, void *cand_ws,
                 cudaStream_t s);
// E > 1024: the chunk candidates' place in the route workspace and their size
size_t topk_chunk_ws_offset(int T, int E);
size_t topk_chunk_ws_bytes(int T, int E, int k);

size_t permute_ws_bytes(int T, int k, int E);
int launch_permute(const int32_t *ids, int T, int k, int E, int32_t *offsets, int32_t *perm_src, int32_t *perm_dst,
                   int32_t *active, void *ws, unsigned *err, cudaStream_t s);

size_t gemv_ws_bytes(int T, int k, int I);
bool gemv_supported(int bits, int H, int I);
int launch_gemv(int bits, const uint8_t *const *blobs, const int32_t *offsets, const int32_t *active,
                const int32_t *perm_src, const void *x, int x_dtype, int T, int k, int H, int I, int E,
                const uint8_t *shared_blob, float *y_perm, float *y_shared, void *ws, unsigned *err, cudaStream_t s);

size_t gemm_ws_bytes(int bits, int T, int k, int H, int I, int E);
bool gemm_supported(int bits, int T, int k, int H, int I, int E);
int launch_gemm(int bits, const uint8_t *const *blobs, const int32_t *offsets, const int32_t *active,
                const int32_t *perm_src, const void *x, int x_dtype, int T, int k, int H, int I, int E,
                const uint8_t *shared_blob, float *y_perm, float *y_shared, void *ws, unsigned *err, cudaStream_t s);

size_t decode_ws_bytes(int E, int k, int I);
bool decode_supported(int bits, int H, int I, int E, int k);
int launch_decode(int bits, const void *x, int x_dtype, const void *w_router, int w_dtype, const float *bias,
                  const float *logits_in, const uint8_t *const *blobs, const uint8_t *shared, int H, int I, int E,
                  int k, int32_t *ids, float *w, float *logits_out, float *y, void *ws, unsigned *err,
                  cudaStream_t s);

bool decode_step_supported(int bits, int H, int I, int E, int k, bool shared);
int launch_decode_step(int bits, const void *x, int x_dtype, const void *w_router, int w_dtype, const float *bias,
                       const float *logits_in, const uint8_t *const *blobs, const uint8_t *shared, int H, int I,
                       int E, int k, int32_t *ids, float *w, float *logits_out, float *y, float *logits_ws,
                       float *h_ws, unsigned *bar, unsigned *err, cudaStream_t s);

// Test hooks (moe_test_hook): the current value of a hook, 0 when unset.
long long test_hook_value(int which);

int launch_combine(const float *y_perm, const int32_t *perm_dst, const float *w, const float *y_shared, int T, int k,
                   int H, float *y, unsigned *err, cudaStream_t s);

// expert-cache device table patch: table[ids[i]] = ptrs[i]
struct TablePatch {
    int n;
    int32_t ids[64];
    const void *ptrs[64];
};
int launch_table_patch(const void **table, const TablePatch &p, cudaStream_t s);

}  // namespace moe
