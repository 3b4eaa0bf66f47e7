// Weighted combine of the expert rows back into token order:
//   y[t] = sum_j w[t,j] * y_perm[perm_dst[t,j]] (+ y_shared[t]), slot order, fp32.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kCombineBatch = 8;

__global__ void __launch_bounds__(256) k_combine(const float *__restrict__ y_perm, const int32_t *__restrict__ perm_dst,
                                                  const float *__restrict__ w, const float *__restrict__ y_shared,
                                                  int T, int k, int H, float *__restrict__ y, unsigned *err) {
    const int h4n = H / 4;
    const long total = static_cast<long>(T) * h4n;
    for (long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<long>(gridDim.x) * blockDim.x) {
        const int t = static_cast<int>(i / h4n), h4 = static_cast<int>(i % h4n);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        // kCombineBatch slots at a time: their rows and gates, then their rows'
        // values, each batch's loads in flight together (summed in slot order)
        for (int j0 = 0; j0 < k; j0 += kCombineBatch) {
            int rr[kCombineBatch];
            float gg[kCombineBatch];
#pragma unroll
            for (int u = 0; u < kCombineBatch; ++u) {
                const int j = j0 + u;
                rr[u] = j < k ? perm_dst[static_cast<size_t>(t) * k + j] : -1;
                gg[u] = j < k ? w[static_cast<size_t>(t) * k + j] : 0.f;
            }
            float4 v[kCombineBatch];
#pragma unroll
            for (int u = 0; u < kCombineBatch; ++u) {
                const bool ok = rr[u] >= 0 && rr[u] < T * k;   // never read outside y_perm
                if (j0 + u < k && !ok) report(err, MOE_DEVERR_BAD_ROW);
                v[u] = ok ? reinterpret_cast<const float4 *>(y_perm + static_cast<size_t>(rr[u]) * H)[h4]
                          : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < kCombineBatch; ++u) {
                if (j0 + u >= k || rr[u] < 0 || rr[u] >= T * k) continue;
                acc.x = fmaf(gg[u], v[u].x, acc.x);
                acc.y = fmaf(gg[u], v[u].y, acc.y);
                acc.z = fmaf(gg[u], v[u].z, acc.z);
                acc.w = fmaf(gg[u], v[u].w, acc.w);
            }
        }
        if (y_shared) {
            const float4 v = reinterpret_cast<const float4 *>(y_shared + static_cast<size_t>(t) * H)[h4];
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        reinterpret_cast<float4 *>(y + static_cast<size_t>(t) * H)[h4] = acc;
    }
}

int launch_combine(const float *y_perm, const int32_t *perm_dst, const float *w, const float *y_shared, int T, int k,
                   int H, float *y, unsigned *err, cudaStream_t s) {
    const long total = static_cast<long>(T) * (H / 4);
    long blocks = (total + 255) / 256;
    const long cap = static_cast<long>(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    k_combine<<<blocks, 256, 0, s>>>(y_perm, perm_dst, w, y_shared, T, k, H, y, err); count_launches(1);
    return cuda_status(cudaGetLastError(), "combine launch");
}

}  // namespace moe
