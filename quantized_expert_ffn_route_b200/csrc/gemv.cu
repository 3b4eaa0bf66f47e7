// Expert FFN on CUDA cores for a few tokens per expert (decode and verify
// windows of 1-16 tokens).  HBM-bound at one token: each packed weight is
// read once with 16-byte loads and dequantised in registers.
// The packed-code dot product (qdot.cuh) dequantises in registers.
#include "common.cuh"
#include "kernels.h"
#include "qdot.cuh"

namespace moe {

struct Group {
    const uint8_t *blob;
    int n;          // tokens (rows) of the group
    int row0;       // first row in y_perm / h (routed), or -1 for the shared expert
};

__device__ __forceinline__ bool group_of(int g, int n_act, const int32_t *active, const int32_t *offsets,
                                         const uint8_t *const *blobs, const uint8_t *shared_blob, int T, int k,
                                         int E, unsigned *err, Group &G) {
    if (g < n_act) {
        const int e = active[1 + g];
        if (e < 0 || e >= E) {
            if (threadIdx.x == 0) report(err, MOE_DEVERR_BAD_EXPERT);
            return false;
        }
        const int r0 = offsets[e], r1 = offsets[e + 1];
        if (r0 < 0 || r1 < r0 || r1 > T * k) {
            if (threadIdx.x == 0) report(err, MOE_DEVERR_BAD_ROW);
            return false;
        }
        G.blob = blobs[e];
        if (!G.blob) {
            if (threadIdx.x == 0) report(err, MOE_DEVERR_NULL_BLOB);
            return false;
        }
        G.n = r1 - r0;
        G.row0 = r0;
    } else {
        G.blob = shared_blob;
        G.n = T;
        G.row0 = -1;
    }
    return G.n > 0;
}

constexpr int kWarps = 8;
constexpr int kRowsPerWarpGU = 2;
constexpr int kNTS = 16;   // most tokens staged at once

// ---------------------------------------------------------------- gate/up
template <int BITS, int NT>
__device__ __forceinline__ void rows_gateup(const BlobView &bv, int H, int I, int i0, const float4 *xs,
                                            const float *cs, int nt, float *hrow0, size_t hld, int lane) {
    using Q = QT<BITS>;
    const int nch = H / Q::EPC;
    const size_t rowbytes = static_cast<size_t>(H) * BITS / 8;
    const int nsc = H / 32;
    constexpr int SPL = 2;     // chunks per lane: H <= 64 chunks (q4: 2048, q2: 4096)
    uint4 cg[kRowsPerWarpGU][SPL], cu[kRowsPerWarpGU][SPL];
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarpGU; ++rr)
#pragma unroll
        for (int s = 0; s < SPL; ++s) {
            const int c = lane + 32 * s;
            const size_t off = static_cast<size_t>(i0 + rr) * rowbytes + static_cast<size_t>(c) * 16;
            if (c < nch) {
                cg[rr][s] = ldg_stream(bv.cg + off);
                cu[rr][s] = ldg_stream(bv.cu + off);
            } else {
                cg[rr][s] = cu[rr][s] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarpGU; ++rr) {
        float dg[NT], du[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) dg[t] = du[t] = 0.f;
#pragma unroll
        for (int s = 0; s < SPL; ++s) {
            const int c = lane + 32 * s;
            const bool valid = c < nch;
            float sg[Q::BPC], su[Q::BPC];
            load_scales<BITS>(bv.sg + static_cast<size_t>(i0 + rr) * nsc, c, valid, sg);
            load_scales<BITS>(bv.su + static_cast<size_t>(i0 + rr) * nsc, c, valid, su);
            if (valid) {
                chunk_dot<BITS, NT>(cg[rr][s], sg, xs, cs, nch, c, dg);
                chunk_dot<BITS, NT>(cu[rr][s], su, xs, cs, nch, c, du);
            }
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const float g = warp_sum(dg[t]);
            const float u = warp_sum(du[t]);
            if (lane == t && t < nt) hrow0[static_cast<size_t>(t) * hld + i0 + rr] = g / (1.0f + expf(-g)) * u;
        }
    }
}

template <int BITS, int NT>
__global__ void __launch_bounds__(256) k_gemv_gateup(const uint8_t *const *__restrict__ blobs,
                                                      const int32_t *__restrict__ offsets,
                                                      const int32_t *__restrict__ active,
                                                      const int32_t *__restrict__ perm_src,
                                                      const void *__restrict__ x, int x_bf16, int T, int k, int H,
                                                      int I, int E,
                                                      const uint8_t *__restrict__ shared_blob,
                                                      float *__restrict__ hbuf, int NTS, unsigned *err) {
    using Q = QT<BITS>;
    extern __shared__ float4 smem[];
    float4 *xs = smem;
    float *cs = reinterpret_cast<float *>(smem + static_cast<size_t>(NTS) * (H / 4));
    __shared__ const void *rows[kNTS];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n_act = min(max(active[0], 0), min(E, T * k));   // a corrupt count cannot run past `active`
    const int n_groups = n_act + (shared_blob ? 1 : 0);
    const int rows_per_block = kWarps * kRowsPerWarpGU;
    const size_t xrow = static_cast<size_t>(H) * (x_bf16 ? 2 : 4);
    const int row_blocks = I / rows_per_block;
    for (int task = blockIdx.x; task < n_groups * row_blocks; task += gridDim.x) {
        const int g = task / row_blocks, rb = task % row_blocks;
        Group G;
        if (!group_of(g, n_act, active, offsets, blobs, shared_blob, T, k, E, err, G)) continue;
        const BlobView bv = blob_view(G.blob, BITS, H, I);
        const int i0 = rb * rows_per_block + warp * kRowsPerWarpGU;
        for (int sub = 0; sub < G.n; sub += NTS) {
            const int nt = min(NTS, G.n - sub);
            if (threadIdx.x < NTS) {
                const int r = sub + static_cast<int>(threadIdx.x);
                const int tok = r < G.n ? (G.row0 >= 0 ? perm_src[G.row0 + r] : r) : 0;
                rows[threadIdx.x] = static_cast<const uint8_t *>(x) + static_cast<size_t>(tok < 0 || tok >= T ? 0 : tok) * xrow;
            }
            __syncthreads();
            stage_rows<BITS>(xs, cs, NTS, nt, H, rows, x_bf16);
            float *hrow0 = hbuf + static_cast<size_t>(G.row0 >= 0 ? G.row0 + sub : T * k + sub) * I;
            if (NT == 1 || nt == 1) rows_gateup<BITS, 1>(bv, H, I, i0, xs, cs, nt, hrow0, I, lane);
            else rows_gateup<BITS, NT>(bv, H, I, i0, xs, cs, nt, hrow0, I, lane);
            __syncthreads();
        }
    }
}

// ------------------------------------------------------------------- down
constexpr int kRowPassesD = 2;

template <int BITS, int NT>
__device__ __forceinline__ void rows_down(const BlobView &bv, int H, int I, int r0, int lpr, const float4 *hs,
                                          const float *cs, int nt, float *yrow0, int lane) {
    using Q = QT<BITS>;
    const int nch = I / Q::EPC;
    const size_t rowbytes = static_cast<size_t>(I) * BITS / 8;
    const int nsc = I / 32;
    const int seg = lane % lpr;
    const int rpp = 32 / lpr;
    const int spl = (nch + lpr - 1) / lpr;
    uint4 code[kRowPassesD][2];
#pragma unroll
    for (int pp = 0; pp < kRowPassesD; ++pp) {
        const int r = r0 + pp * rpp + lane / lpr;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            const int c = seg + lpr * s;
            code[pp][s] = (s < spl && c < nch && r < H)
                              ? ldg_stream(bv.cd + static_cast<size_t>(r) * rowbytes + static_cast<size_t>(c) * 16)
                              : make_uint4(0, 0, 0, 0);
        }
    }
#pragma unroll
    for (int pp = 0; pp < kRowPassesD; ++pp) {
        const int r = r0 + pp * rpp + lane / lpr;
        float dot[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) dot[t] = 0.f;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            const int c = seg + lpr * s;
            const bool valid = s < spl && c < nch && r < H;
            float d[Q::BPC];
            load_scales<BITS>(bv.sd + static_cast<size_t>(r < H ? r : 0) * nsc, c, valid, d);
            if (valid) chunk_dot<BITS, NT>(code[pp][s], d, hs, cs, nch, c, dot);
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            float v = dot[t];
            for (int o = lpr >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            dot[t] = v;
        }
        if (r < H) {
#pragma unroll
            for (int t = 0; t < NT; ++t)
                if (t % lpr == seg && t < nt) yrow0[static_cast<size_t>(t) * H + r] = dot[t];
        }
    }
}

template <int BITS, int NT>
__global__ void __launch_bounds__(256) k_gemv_down(const uint8_t *const *__restrict__ blobs,
                                                    const int32_t *__restrict__ offsets,
                                                    const int32_t *__restrict__ active,
                                                    const float *__restrict__ hbuf, int T, int k, int H, int I,
                                                    int E, const uint8_t *__restrict__ shared_blob,
                                                    float *__restrict__ y_perm, float *__restrict__ y_shared,
                                                    int NTS, int lpr, unsigned *err) {
    using Q = QT<BITS>;
    extern __shared__ float4 smem[];
    float4 *hs = smem;
    float *cs = reinterpret_cast<float *>(smem + static_cast<size_t>(NTS) * (I / 4));
    __shared__ const void *rows[kNTS];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n_act = min(max(active[0], 0), min(E, T * k));   // a corrupt count cannot run past `active`
    const int n_groups = n_act + (shared_blob ? 1 : 0);
    const int rpp = 32 / lpr;
    const int rows_per_block = kWarps * kRowPassesD * rpp;
    const int row_blocks = (H + rows_per_block - 1) / rows_per_block;
    for (int task = blockIdx.x; task < n_groups * row_blocks; task += gridDim.x) {
        const int g = task / row_blocks, rb = task % row_blocks;
        Group G;
        if (!group_of(g, n_act, active, offsets, blobs, shared_blob, T, k, E, err, G)) continue;
        const BlobView bv = blob_view(G.blob, BITS, H, I);
        const int r0 = rb * rows_per_block + warp * kRowPassesD * rpp;
        for (int sub = 0; sub < G.n; sub += NTS) {
            const int nt = min(NTS, G.n - sub);
            const size_t hrow = static_cast<size_t>(G.row0 >= 0 ? G.row0 + sub : T * k + sub);
            if (threadIdx.x < NTS) rows[threadIdx.x] = hbuf + (hrow + min(static_cast<int>(threadIdx.x), nt - 1)) * I;
            __syncthreads();
            stage_rows<BITS>(hs, cs, NTS, nt, I, rows, 0);
            float *yrow0 = G.row0 >= 0 ? y_perm + static_cast<size_t>(G.row0 + sub) * H
                                       : y_shared + static_cast<size_t>(sub) * H;
            if (NT == 1 || nt == 1) rows_down<BITS, 1>(bv, H, I, r0, lpr, hs, cs, nt, yrow0, lane);
            else rows_down<BITS, NT>(bv, H, I, r0, lpr, hs, cs, nt, yrow0, lane);
            __syncthreads();
        }
    }
}

// --------------------------------------------------------------- launcher
size_t gemv_ws_bytes(int T, int k, int I) {
    return static_cast<size_t>(T) * (k + 1) * I * sizeof(float);
}

template <int BITS, int NT>
static void launch_gemv_nt(const uint8_t *const *blobs, const int32_t *offsets, const int32_t *active,
                           const int32_t *perm_src, const void *x, int x_bf16, int T, int k, int H, int I, int E,
                           const uint8_t *shared_blob, float *y_perm, float *y_shared, float *hbuf, unsigned *err,
                           cudaStream_t s) {
    using Q = QT<BITS>;
    const int NTS = NT;
    const int max_groups = (T * k < E ? T * k : E) + (shared_blob ? 1 : 0);
    const int sms = num_sms();
    {
        const size_t smem = static_cast<size_t>(NTS) * H * 4 + static_cast<size_t>(NTS) * (H / 32) * 4;
        const int row_blocks = I / (kWarps * kRowsPerWarpGU);
        long blocks = static_cast<long>(max_groups) * row_blocks;
        if (blocks > sms * 8L) blocks = sms * 8L;
        cudaFuncSetAttribute(k_gemv_gateup<BITS, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        k_gemv_gateup<BITS, NT><<<blocks, 256, smem, s>>>(blobs, offsets, active, perm_src, x, x_bf16, T, k, H, I, E,
                                                          shared_blob, hbuf, NTS, err); count_launches(1);
    }
    {
        const int nch = I / Q::EPC;
        int lpr = 1;
        while (lpr * 2 <= nch && lpr * 2 <= 32) lpr *= 2;
        const size_t smem = static_cast<size_t>(NTS) * I * 4 + static_cast<size_t>(NTS) * (I / 32) * 4;
        const int rows_per_block = kWarps * kRowPassesD * (32 / lpr);
        const int row_blocks = (H + rows_per_block - 1) / rows_per_block;
        long blocks = static_cast<long>(max_groups) * row_blocks;
        if (blocks > sms * 8L) blocks = sms * 8L;
        cudaFuncSetAttribute(k_gemv_down<BITS, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        k_gemv_down<BITS, NT><<<blocks, 256, smem, s>>>(blobs, offsets, active, hbuf, T, k, H, I, E, shared_blob,
                                                        y_perm, y_shared, NTS, lpr, err); count_launches(1);
    }
}

template <int BITS>
static int launch_gemv_t(const uint8_t *const *blobs, const int32_t *offsets, const int32_t *active,
                         const int32_t *perm_src, const void *x, int x_bf16, int T, int k, int H, int I, int E,
                         const uint8_t *shared_blob, float *y_perm, float *y_shared, float *hbuf, unsigned *err,
                         cudaStream_t s) {
#define MOE_GEMV_NT(N) \
    launch_gemv_nt<BITS, N>(blobs, offsets, active, perm_src, x, x_bf16, T, k, H, I, E, shared_blob, y_perm, y_shared, \
                            hbuf, err, s)
    if (T <= 1) MOE_GEMV_NT(1);
    else if (T <= 2) MOE_GEMV_NT(2);
    else if (T <= 4) MOE_GEMV_NT(4);
    else if (T <= 8) MOE_GEMV_NT(8);
    else MOE_GEMV_NT(16);
#undef MOE_GEMV_NT
    return cuda_status(cudaGetLastError(), "expert GEMV launch");
}

int launch_gemv(int bits, const uint8_t *const *blobs, const int32_t *offsets, const int32_t *active,
                const int32_t *perm_src, const void *x, int x_dtype, int T, int k, int H, int I, int E,
                const uint8_t *shared_blob, float *y_perm, float *y_shared, void *ws, unsigned *err,
                cudaStream_t s) {
    float *hbuf = static_cast<float *>(ws);
    const int xb = x_dtype == MOE_BF16;
    if (bits == 4)
        return launch_gemv_t<4>(blobs, offsets, active, perm_src, x, xb, T, k, H, I, E, shared_blob, y_perm, y_shared,
                                hbuf, err, s);
    return launch_gemv_t<2>(blobs, offsets, active, perm_src, x, xb, T, k, H, I, E, shared_blob, y_perm, y_shared,
                            hbuf, err, s);
}

}  // namespace moe
