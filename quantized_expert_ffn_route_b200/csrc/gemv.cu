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

constexpr int kGvThreads = 256;
constexpr int kGvWarps = kGvThreads / 32;
constexpr int kGvRows = 16;      // gate/up rows per task (2 per warp)
constexpr int kGvNT = 8;         // token rows staged per pass (8: two CTAs fit an SM)
// down: row groups per warp (4-bit codes need more registers per chunk)
template <int BITS>
struct GvTPW { static constexpr int value = BITS == 4 ? 2 : 4; };

// ---------------------------------------------------------------- gate/up
// Task = (group, 16 rows).  The codes of a warp's four row vectors (gate and
// up of two rows) stay in registers while the group's tokens are staged 16
// at a time and streamed past them, one token per pass over the codes.
template <int BITS>
__global__ void __launch_bounds__(kGvThreads, 2) k_gemv_gateup(const uint8_t *const *__restrict__ blobs,
                                                               const int32_t *__restrict__ offsets,
                                                               const int32_t *__restrict__ active,
                                                               const int32_t *__restrict__ perm_src,
                                                               const void *__restrict__ x, int x_bf16, int T, int k,
                                                               int H, int I, int E,
                                                               const uint8_t *__restrict__ shared_blob,
                                                               float *__restrict__ hbuf, unsigned *err) {
    using Q = QT<BITS>;
    extern __shared__ float4 smem[];
    float4 *xs = smem;
    float *cs = reinterpret_cast<float *>(smem + static_cast<size_t>(kGvNT) * (H / 4));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n_act = guard_count(active[0], min(E, T * k), err);   // a corrupt count cannot run past `active`
    const int n_groups = n_act + (shared_blob ? 1 : 0);
    const int row_blocks = I / kGvRows;
    const int nch = H / Q::EPC, nblk = H / 32, nsc = H / 32;
    const size_t xrowb = static_cast<size_t>(H) * BITS / 8;
    const size_t xrow = static_cast<size_t>(H) * (x_bf16 ? 2 : 4);
    constexpr int S = 2048 / Q::EPC / 32;               // chunks per lane (H <= 2048)
    for (int task = blockIdx.x; task < n_groups * row_blocks; task += gridDim.x) {
        const int g = task / row_blocks, rb = task - g * row_blocks;
        Group G;
        if (!group_of(g, n_act, active, offsets, blobs, shared_blob, T, k, E, err, G)) continue;
        const BlobView bv = blob_view(G.blob, BITS, H, I);
        const int i0 = rb * kGvRows + warp * 2;
        uint4 code[4][S];
        float dsc[4][S][Q::BPC];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int i = i0 + (v >> 1);
            const uint8_t *cbase = (v & 1) ? bv.cu : bv.cg;
            const __half *sbase = (v & 1) ? bv.su : bv.sg;
#pragma unroll
            for (int s = 0; s < S; ++s) {
                const int cc = lane + 32 * s;
                const bool valid = cc < nch;
                code[v][s] = valid ? ldg_stream(cbase + static_cast<size_t>(i) * xrowb + static_cast<size_t>(cc) * 16)
                                   : make_uint4(0, 0, 0, 0);
                load_scales<BITS>(sbase + static_cast<size_t>(i) * nsc, cc, valid, dsc[v][s]);
            }
        }
        const size_t hrow0 = static_cast<size_t>(G.row0 >= 0 ? G.row0 : T * k);
#pragma unroll 1
        for (int sub = 0; sub < G.n; sub += kGvNT) {
            const int nt = min(kGvNT, G.n - sub);
            const int row0 = G.row0;
            stage_rows_fn<BITS>(
                xs, cs, nt, nt, H,
                [=](int t) {
                    const int r = sub + t;
                    const int tok = row0 >= 0 ? guard_index(perm_src[row0 + r], T, err, MOE_DEVERR_BAD_ROW) : r;
                    return static_cast<const void *>(static_cast<const uint8_t *>(x) + static_cast<size_t>(tok) * xrow);
                },
                x_bf16);
#pragma unroll 1
            for (int t = 0; t < nt; ++t) {
                float dot[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    const int cc = lane + 32 * s;
                    if (cc < nch) {
                        float csum[Q::BPC];
#pragma unroll
                        for (int b = 0; b < Q::BPC; ++b) csum[b] = cs[t * nblk + cc * Q::BPC + b];
                        uint4 cv[4] = {code[0][s], code[1][s], code[2][s], code[3][s]};
#pragma unroll
                        for (int v = 0; v < 4; ++v) opaque(cv[v]);
                        float fx[4][Q::BPC];
                        rows_fx<BITS, 4>(cv, xs + static_cast<size_t>(t) * Q::PPC * nch + cc, nch, fx);
#pragma unroll
                        for (int v = 0; v < 4; ++v) dot[v] = chunk_finish<BITS>(fx[v], dsc[v][s], csum, dot[v]);
                    }
                }
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const float gv = warp_sum(dot[2 * j]);
                    const float uv = warp_sum(dot[2 * j + 1]);
                    if (lane == 0) hbuf[(hrow0 + sub + t) * I + i0 + j] = gv / (1.0f + expf(-gv)) * uv;
                }
            }
            __syncthreads();                             // before the next pass restages
        }
    }
}

// ------------------------------------------------------------------- down
// Task = (group, RB output rows): each lane one 16-byte chunk of one row
// (LPR lanes per row), GvTPW rows per lane kept in registers; the group's
// h rows are staged 16 at a time.
template <int BITS, int LPR>
__global__ void __launch_bounds__(kGvThreads, 2) k_gemv_down(const uint8_t *const *__restrict__ blobs,
                                                             const int32_t *__restrict__ offsets,
                                                             const int32_t *__restrict__ active,
                                                             const float *__restrict__ hbuf, int T, int k, int H,
                                                             int E, const uint8_t *__restrict__ shared_blob,
                                                             float *__restrict__ y_perm, float *__restrict__ y_shared,
                                                             unsigned *err) {
    using Q = QT<BITS>;
    constexpr int kGvTPW = GvTPW<BITS>::value;
    constexpr int RPP = 32 / LPR;                        // rows per warp pass
    constexpr int RB = kGvWarps * kGvTPW * RPP;          // rows per task
    constexpr int IL = LPR * Q::EPC;                     // the intermediate size I
    constexpr int nblk = IL / 32;
    constexpr size_t drowb = static_cast<size_t>(IL) * BITS / 8;
    extern __shared__ float4 smem[];
    float4 *hs = smem;
    float *hcs = reinterpret_cast<float *>(smem + static_cast<size_t>(kGvNT) * (IL / 4));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int seg = lane % LPR, subr = lane / LPR;
    const int n_act = guard_count(active[0], min(E, T * k), err);
    const int n_groups = n_act + (shared_blob ? 1 : 0);
    const int row_blocks = (H + RB - 1) / RB;
    for (int task = blockIdx.x; task < n_groups * row_blocks; task += gridDim.x) {
        const int g = task / row_blocks, rb = task - g * row_blocks;
        Group G;
        if (!group_of(g, n_act, active, offsets, blobs, shared_blob, T, k, E, err, G)) continue;
        const BlobView bv = blob_view(G.blob, BITS, H, IL);
        uint4 code[kGvTPW];
        float dsc[kGvTPW][Q::BPC];
        int rows[kGvTPW];
#pragma unroll
        for (int tt = 0; tt < kGvTPW; ++tt) {
            const int r = rb * RB + (warp * kGvTPW + tt) * RPP + subr;
            rows[tt] = r;
            const bool valid = r < H;
            code[tt] = valid ? ldg_stream(bv.cd + static_cast<size_t>(r) * drowb + static_cast<size_t>(seg) * 16)
                             : make_uint4(0, 0, 0, 0);
            load_scales<BITS>(bv.sd + static_cast<size_t>(valid ? r : 0) * nblk, seg, valid, dsc[tt]);
        }
        const size_t hrow0 = static_cast<size_t>(G.row0 >= 0 ? G.row0 : T * k);
        float *yrow0 = G.row0 >= 0 ? y_perm + static_cast<size_t>(G.row0) * H : y_shared;
#pragma unroll 1
        for (int sub = 0; sub < G.n; sub += kGvNT) {
            const int nt = min(kGvNT, G.n - sub);
            stage_rows_fn<BITS>(
                hs, hcs, nt, nt, IL,
                [=](int t) { return static_cast<const void *>(hbuf + (hrow0 + sub + t) * IL); }, 0);
#pragma unroll 1
            for (int t = 0; t < nt; ++t) {
                float csum[Q::BPC];
#pragma unroll
                for (int b = 0; b < Q::BPC; ++b) csum[b] = hcs[t * nblk + seg * Q::BPC + b];
                float fx[kGvTPW][Q::BPC];
#pragma unroll
                for (int tt = 0; tt < kGvTPW; ++tt) opaque(code[tt]);
                rows_fx<BITS, kGvTPW>(code, hs + static_cast<size_t>(t) * Q::PPC * LPR + seg, LPR, fx);
#pragma unroll
                for (int tt = 0; tt < kGvTPW; ++tt) {
                    float v = chunk_finish<BITS>(fx[tt], dsc[tt], csum, 0.f);
#pragma unroll
                    for (int o = LPR >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                    if (seg == 0 && rows[tt] < H) yrow0[static_cast<size_t>(sub + t) * H + rows[tt]] = v;
                }
            }
            __syncthreads();
        }
    }
}

// --------------------------------------------------------------- launcher
size_t gemv_ws_bytes(int T, int k, int I) {
    return static_cast<size_t>(T) * (k + 1) * I * sizeof(float);
}

bool gemv_supported(int bits, int H, int I) {
    const int lpr = I / (bits == 4 ? 32 : 64);
    return H >= 128 && H <= 2048 && H % 128 == 0 && I % 128 == 0 &&
           (lpr == 2 || lpr == 4 || lpr == 8 || lpr == 16 || lpr == 32);
}

template <int BITS, int LPR>
static void launch_down(const uint8_t *const *blobs, const int32_t *offsets, const int32_t *active, const float *hbuf,
                        int T, int k, int H, int E, const uint8_t *shared_blob, float *y_perm, float *y_shared,
                        unsigned *err, int max_groups, cudaStream_t s) {
    using Q = QT<BITS>;
    constexpr int IL = LPR * Q::EPC;
    constexpr int RB = kGvWarps * GvTPW<BITS>::value * (32 / LPR);
    const size_t smem = static_cast<size_t>(kGvNT) * IL * 4 + static_cast<size_t>(kGvNT) * (IL / 32) * 4;
    long blocks = static_cast<long>(max_groups) * ((H + RB - 1) / RB);
    if (blocks > num_sms() * 8L) blocks = num_sms() * 8L;
    cudaFuncSetAttribute(k_gemv_down<BITS, LPR>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    k_gemv_down<BITS, LPR><<<blocks, kGvThreads, smem, s>>>(blobs, offsets, active, hbuf, T, k, H, E, shared_blob,
                                                            y_perm, y_shared, err);
    count_launches(1);
}

template <int BITS>
static int launch_gemv_t(const uint8_t *const *blobs, const int32_t *offsets, const int32_t *active,
                         const int32_t *perm_src, const void *x, int x_bf16, int T, int k, int H, int I, int E,
                         const uint8_t *shared_blob, float *y_perm, float *y_shared, float *hbuf, unsigned *err,
                         cudaStream_t s) {
    using Q = QT<BITS>;
    const int max_groups = (T * k < E ? T * k : E) + (shared_blob ? 1 : 0);
    {
        const size_t smem = static_cast<size_t>(kGvNT) * H * 4 + static_cast<size_t>(kGvNT) * (H / 32) * 4;
        long blocks = static_cast<long>(max_groups) * (I / kGvRows);
        if (blocks > num_sms() * 8L) blocks = num_sms() * 8L;
        cudaFuncSetAttribute(k_gemv_gateup<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        k_gemv_gateup<BITS><<<blocks, kGvThreads, smem, s>>>(blobs, offsets, active, perm_src, x, x_bf16, T, k, H, I,
                                                             E, shared_blob, hbuf, err);
        count_launches(1);
    }
    switch (I / Q::EPC) {
        case 2: launch_down<BITS, 2>(blobs, offsets, active, hbuf, T, k, H, E, shared_blob, y_perm, y_shared, err, max_groups, s); break;
        case 4: launch_down<BITS, 4>(blobs, offsets, active, hbuf, T, k, H, E, shared_blob, y_perm, y_shared, err, max_groups, s); break;
        case 8: launch_down<BITS, 8>(blobs, offsets, active, hbuf, T, k, H, E, shared_blob, y_perm, y_shared, err, max_groups, s); break;
        case 16: launch_down<BITS, 16>(blobs, offsets, active, hbuf, T, k, H, E, shared_blob, y_perm, y_shared, err, max_groups, s); break;
        default: launch_down<BITS, 32>(blobs, offsets, active, hbuf, T, k, H, E, shared_blob, y_perm, y_shared, err, max_groups, s); break;
    }
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
