// Router logits of a prefill chunk on the 5th-generation tensor cores.
//
// Strata article, summary table and section 2 item 1: every token scores all
// experts of the layer before the top-k.  For a chunk of thousands of tokens
// that is a dense bf16 contraction, logits[t, e] = x[t] . W_r[e] (+ b_e),
// with fp32 accumulation: tcgen05.mma kind::f16 with both operands bf16.
//
// One CTA per (128 experts) x (128 tokens) tile; K in steps of 64 through a
// ring of shared-memory stages in the 128-byte-swizzled K-major layout.
//   warps 0-3  copy W_r rows (A) and x rows (B) with cp.async a few k-steps
//              ahead; each warp publishes a stage with one barrier arrival
//              once its copies have landed;
//   warp  8    allocates 128 TMEM columns and issues the MMAs (one thread);
//   warps 4-7  read the fp32 accumulators (tcgen05.ld) and write logits.
// Every mbarrier wait is bounded; a timeout sets MOE_DEVERR_TIMEOUT.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace moe {
using namespace sm100;

namespace {
constexpr int kRM = 128;            // experts per tile (MMA M)
constexpr int kRN = 128;            // tokens per tile (MMA N)
constexpr int kRK = 64;             // K per stage (128 bytes of bf16)
constexpr int kRS = 3;              // stages
constexpr int kRThreads = 288;      // 4 loader, 4 epilogue, 1 MMA warp
constexpr long kRSpin = 1L << 22;
constexpr size_t kRStage = static_cast<size_t>(kRM + kRN) * 128;
constexpr size_t kROffBar = kRS * kRStage;
constexpr size_t kRSmem = kROffBar + 16 * 8 + 16 + 1024;

// bf16 A and B, fp32 D, both K-major
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}
}  // namespace

__global__ void __launch_bounds__(kRThreads) k_router_mma(const __nv_bfloat16 *__restrict__ x,
                                                           const __nv_bfloat16 *__restrict__ w,
                                                           const float *__restrict__ bias, int T, int H, int E,
                                                           float *__restrict__ logits, unsigned *err) {
    extern __shared__ __align__(1024) uint8_t rsmem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(rsmem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kROffBar);
    uint64_t *full = bars, *empty = bars + kRS, *accF = bars + 2 * kRS;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 16);
    volatile int &abort_s = *(reinterpret_cast<int *>(bars + 16) + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int e0 = blockIdx.x * kRM, t0 = blockIdx.y * kRN;
    const int nk = H / kRK;
    if (tid == 0) {
        abort_s = 0;
        for (int i = 0; i < kRS; ++i) {
            mbar_init(full + i, 4);                              // one arrival per loader warp
            mbar_init(empty + i, 1);
        }
        mbar_init(accF, 1);
        fence_barrier_init();
    }
    if (warp == 8) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto fail = [&]() {
        report(err, MOE_DEVERR_TIMEOUT);
        abort_s = 1;
    };

    if (warp < 4) {
        // ----------------------------------------------------- loaders
        const int c = lane & 7;
        constexpr int D = kRS / 2;                               // k-steps of copies in flight per thread
        for (int s = 0; s < nk + D; ++s) {
            if (__shfl_sync(0xffffffffu, abort_s, 0)) break;
            if (s < nk) {
                const int st = s % kRS;
                int ok = 1;
                if (lane == 0) ok = mbar_wait(empty + st, static_cast<uint32_t>(((s / kRS) & 1) ^ 1), kRSpin);
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    fail();
                    break;
                }
                const uint32_t sa = smem_addr(smem + st * kRStage), sb = sa + kRM * 128;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = warp * 32 + i * 4 + (lane >> 3);   // row of the tile
                    const int e = e0 + r, t = t0 + r;
                    const uint32_t sw = static_cast<uint32_t>(((c ^ (r & 7)) << 4));
                    cp_async16(sa + r * 128 + sw, w + static_cast<size_t>(e < E ? e : 0) * H + s * kRK + c * 8,
                               e < E ? 16u : 0u);
                    cp_async16(sb + r * 128 + sw, x + static_cast<size_t>(t < T ? t : 0) * H + s * kRK + c * 8,
                               t < T ? 16u : 0u);
                }
            }
            cp_async_commit();
            if (s >= D) {                                        // publish k-step s - D
                cp_async_wait<D>();
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(full + (s - D) % kRS);
            }
        }
        cp_async_wait<0>();
    } else if (warp < 8) {
        // ----------------------------------------------------- epilogue
        const int q = warp & 3;
        const int e = e0 + 32 * q + lane;
        if (mbar_wait(accF, 0, kRSpin)) {
            tc_fence_after();
            const float b = (bias && e < E) ? bias[e] : 0.f;
            const uint32_t base = tmem + (static_cast<uint32_t>(32 * q) << 16);
            for (int c0 = 0; c0 < kRN; c0 += 16) {
                if (t0 + c0 >= T) break;                             // uniform over the warp
                float v[16];
                tmem_ld16(base + c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int t = t0 + c0 + j;
                    if (t < T && e < E) logits[static_cast<size_t>(t) * E + e] = v[j] + b;
                }
            }
        } else {
            fail();
        }
    } else if (warp == 8) {
        // ---------------------------------------------------------- MMA
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kRM, kRN);
            for (int s = 0; s < nk && !abort_s; ++s) {
                const int st = s % kRS;
                if (!mbar_wait(full + st, static_cast<uint32_t>((s / kRS) & 1), kRSpin)) {
                    fail();
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_addr(smem + st * kRStage), sb = sa + kRM * 128;
#pragma unroll
                for (int kk = 0; kk < kRK / 16; ++kk)
                    mma_f16(tmem, desc_sw128(sa + kk * 32), desc_sw128(sb + kk * 32), idesc, (s | kk) != 0);
                mma_commit(empty + st);
            }
            mma_commit(accF);                                        // also when aborted: the epilogue waits on it
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

bool router_mma_supported(int x_dtype, int w_dtype, int T, int H) {
    return x_dtype == MOE_BF16 && w_dtype == MOE_BF16 && T >= 64 && H % kRK == 0;
}

int launch_router_mma(const void *x, const void *w, const float *bias, int T, int H, int E, float *out,
                      unsigned *err, cudaStream_t s) {
    int rc = cuda_status(cudaFuncSetAttribute(k_router_mma, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(kRSmem)),
                         "router smem attribute");
    if (rc) return rc;
    const dim3 grid((E + kRM - 1) / kRM, (T + kRN - 1) / kRN);
    k_router_mma<<<grid, kRThreads, kRSmem, s>>>(static_cast<const __nv_bfloat16 *>(x),
                                                 static_cast<const __nv_bfloat16 *>(w), bias, T, H, E, out, err);
    count_launches(1);
    return cuda_status(cudaGetLastError(), "router launch");
}

}  // namespace moe
