// Grouped expert GEMM on the 5th-generation tensor cores (prefill chunks).
//
// Strata article, section 2 item 3 and section 4: prompts are read in chunks
// of up to 8,192 tokens, and reading touches all the experts, so the expert
// step becomes a dense contraction per expert: D = W_e (dequantised) x X_e^T.
//
// Per tile: 128 weight rows (MMA M) x up to 256 of the expert's tokens (MMA N),
// K in steps of 64.  Weights are the A operand, so small token groups still
// fill the M = 128 datapath ("swap AB").  Roles of one persistent CTA per SM:
//   warps 0-3  producers: copy raw codes + scales (cp.async, two steps ahead),
//              dequantise them to fp16 into the 128-byte-swizzled A tile, and
//              gather the tile's token rows (fp16) into the B tile;
//   warp  8    allocates 512 TMEM columns and issues tcgen05.mma (one thread);
//   warps 4-7  epilogue: tcgen05.ld the fp32 accumulators and write
//              gate/up -> h = silu(g) * u (fp16) or down -> y rows (fp32).
// Every mbarrier wait is bounded; a timeout sets MOE_DEVERR_TIMEOUT and all
// roles leave their loops, after which TMEM is freed.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace moe {
using namespace sm100;

constexpr int kBM = 128;            // weight rows per tile
constexpr int kBK = 64;             // K per stage: one 128-byte row of fp16
constexpr int kMaxN = 256;          // tokens per tile
constexpr int kStA = 2;             // A operand stages
constexpr int kStB = 3;             // B operand stages = raw-code ring slots
constexpr int kLook = kStB - 1;     // copies run this many k-steps ahead
constexpr int kGemmThreads = 288;   // 4 producer warps, 4 epilogue warps, 1 MMA warp
constexpr long kSpin = 1L << 22;    // polls before a wait gives up (about a second)
constexpr int kMaxGroups = 2048;

template <int BITS, bool GATEUP>
struct GemmCfg {
    static constexpr int NA = GATEUP ? 2 : 1;                 // weight matrices per tile (gate, up)
    static constexpr int RAW_CODE = kBK * BITS / 8;           // code bytes of a row per k-step
    static constexpr int SEG = (RAW_CODE + 4 + 15) / 16 * 16; // codes + 2 fp16 scales, 16-byte aligned
    static constexpr int RAW_ROW = NA * SEG;
    static constexpr size_t A_STAGE = static_cast<size_t>(NA) * kBM * 128;
    static constexpr size_t B_STAGE = static_cast<size_t>(kMaxN) * 128;
    static constexpr size_t RAW_STAGE = static_cast<size_t>(kBM) * RAW_ROW;
    // shared-memory plan
    static constexpr size_t OFF_A = 0;
    static constexpr size_t OFF_B = OFF_A + kStA * A_STAGE;
    static constexpr size_t OFF_RAW = OFF_B + kStB * B_STAGE;
    static constexpr size_t OFF_TOK = OFF_RAW + kStB * RAW_STAGE;
    static constexpr size_t OFF_GS = OFF_TOK + kMaxN * 4;
    static constexpr size_t OFF_BAR = (OFF_GS + (kMaxGroups + 1) * 4 + 15) / 16 * 16;
    static constexpr size_t SMEM = OFF_BAR + 16 * 8 + 16 + 1024;   // + slack for 1024-byte alignment
};

struct GemmArgs {
    const uint8_t *const *blobs;
    const int32_t *offsets;
    const int32_t *active;
    const int32_t *perm_src;
    const uint8_t *shared;
    const __half *x16;      // [T, H]
    __half *h16;            // [T*k + T, I]
    float *y_perm;          // [T*k, H]
    float *y_shared;        // [T, H]
    int T, k, H, I, E;
    unsigned *err;
};

struct GroupInfo {
    const uint8_t *blob;
    int n;       // rows (tokens) of the group
    int row0;    // first permuted row (routed), or -1 for the shared expert
};

__device__ __forceinline__ GroupInfo group_info(const GemmArgs &a, int g, int n_act) {
    GroupInfo G;
    if (g < n_act) {
        const int e = a.active[1 + g];
        const bool ok = e >= 0 && e < a.E;
        G.row0 = ok ? a.offsets[e] : 0;
        G.n = ok ? a.offsets[e + 1] - G.row0 : 0;
        G.blob = ok ? a.blobs[e] : nullptr;
        if (G.row0 < 0 || G.n < 0 || G.row0 + G.n > a.T * a.k) G.n = 0;
    } else {
        G.row0 = -1;
        G.n = a.T;
        G.blob = a.shared;
    }
    if (!G.blob) G.n = 0;
    return G;
}

// fp16 weights of 8 consecutive elements from 4 packed code bytes (q4: the
// low or high nibbles of 8 bytes) -- returned as 4 half2 words.
__device__ __forceinline__ uint32_t pair16(uint32_t bytes, uint32_t sel) {
    // bytes hold one code (0..15) per byte; builds half2 (1024 + q_a, 1024 + q_b)
    return __byte_perm(bytes, 0x64646464u, sel);
}
__device__ __forceinline__ uint32_t dq2(uint32_t magic_pair, __half2 offset, __half2 d2) {
    __half2 h = *reinterpret_cast<__half2 *>(&magic_pair);
    h = __hmul2(__hsub2(h, offset), d2);       // (q - offset) exact, then one rounding of d * (q - offset)
    return *reinterpret_cast<uint32_t *>(&h);
}

// Dequantises one row's k-step (64 elements) into the swizzled A row.
template <int BITS>
__device__ __forceinline__ void dequant_row(const uint8_t *raw_seg, uint32_t a_row_addr, int row) {
    constexpr int RAW_CODE = kBK * BITS / 8;
    const uint4 *cw = reinterpret_cast<const uint4 *>(raw_seg);
    const __half2 *sc = reinterpret_cast<const __half2 *>(raw_seg + RAW_CODE);
    const __half2 s01 = *sc;
    const int sw = row & 7;
    if constexpr (BITS == 4) {
        const __half2 off = __float2half2_rn(1032.0f);
#pragma unroll
        for (int b = 0; b < 2; ++b) {                              // quant block b: elements 32b..32b+31
            const uint4 w = cw[b];
            const __half2 d2 = b == 0 ? __low2half2(s01) : __high2half2(s01);
            const uint32_t lo0 = w.x & 0x0F0F0F0Fu, lo1 = w.y & 0x0F0F0F0Fu;
            const uint32_t lo2 = w.z & 0x0F0F0F0Fu, lo3 = w.w & 0x0F0F0F0Fu;
            const uint32_t hi0 = (w.x >> 4) & 0x0F0F0F0Fu, hi1 = (w.y >> 4) & 0x0F0F0F0Fu;
            const uint32_t hi2 = (w.z >> 4) & 0x0F0F0F0Fu, hi3 = (w.w >> 4) & 0x0F0F0F0Fu;
            // chunk j (8 elements): 0 = low nibbles of bytes 0-7, 1 = low of 8-15,
            //                       2 = high nibbles of bytes 0-7, 3 = high of 8-15
            const uint32_t src[4][2] = {{lo0, lo1}, {lo2, lo3}, {hi0, hi1}, {hi2, hi3}};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t v0 = dq2(pair16(src[j][0], 0x5140u), off, d2);
                const uint32_t v1 = dq2(pair16(src[j][0], 0x5342u), off, d2);
                const uint32_t v2 = dq2(pair16(src[j][1], 0x5140u), off, d2);
                const uint32_t v3 = dq2(pair16(src[j][1], 0x5342u), off, d2);
                const int c = 4 * b + j;                               // 16-byte chunk of the 128-byte row
                const uint32_t dst = a_row_addr + static_cast<uint32_t>(((c ^ sw) << 4));
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(v0), "r"(v1), "r"(v2),
                             "r"(v3)
                             : "memory");
            }
        }
    } else {
        const __half2 off = __float2half2_rn(1026.0f);
        const uint4 w = cw[0];
        const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int b = 0; b < 2; ++b) {                              // quant block b: 8 bytes = words 2b, 2b+1
            const __half2 d2 = b == 0 ? __low2half2(s01) : __high2half2(s01);
#pragma unroll
            for (int j = 0; j < 4; ++j) {                          // crumb level j: elements 8j..8j+7 of the block
                const uint32_t c0 = (words[2 * b] >> (2 * j)) & 0x03030303u;
                const uint32_t c1 = (words[2 * b + 1] >> (2 * j)) & 0x03030303u;
                const uint32_t v0 = dq2(pair16(c0, 0x5140u), off, d2);
                const uint32_t v1 = dq2(pair16(c0, 0x5342u), off, d2);
                const uint32_t v2 = dq2(pair16(c1, 0x5140u), off, d2);
                const uint32_t v3 = dq2(pair16(c1, 0x5342u), off, d2);
                const int c = 4 * b + j;
                const uint32_t dst = a_row_addr + static_cast<uint32_t>(((c ^ sw) << 4));
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(v0), "r"(v1), "r"(v2),
                             "r"(v3)
                             : "memory");
            }
        }
    }
}

template <int BITS, bool GATEUP>
__global__ void __launch_bounds__(kGemmThreads, 1) k_gemm(GemmArgs a) {
    using Cfg = GemmCfg<BITS, GATEUP>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment of the operand tiles (swizzle atoms)
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + Cfg::OFF_A;
    uint8_t *sB = smem + Cfg::OFF_B;
    uint8_t *sRaw = smem + Cfg::OFF_RAW;
    int32_t *sTok = reinterpret_cast<int32_t *>(smem + Cfg::OFF_TOK);
    int32_t *gstart = reinterpret_cast<int32_t *>(smem + Cfg::OFF_GS);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *fullA = bars, *emptyA = bars + 2, *fullB = bars + 4, *emptyB = bars + 7;
    uint64_t *acc_full = bars + 10, *acc_empty = bars + 11, *drain = bars + 12;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 13);
    __shared__ int abort_sh;
    __shared__ int total_tiles_s;
    volatile int &abort_s = abort_sh;            // read in loop conditions: never cached

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = GATEUP ? a.H : a.I;           // reduction length
    const int Mtot = GATEUP ? a.I : a.H;        // weight rows
    const int MT = Mtot / kBM;
    const int nk = K / kBK;
    const int n_act = min(max(a.active[0], 0), min(a.E, a.T * a.k));
    const int ng = n_act + (a.shared ? 1 : 0);

    if (tid == 0) {
        abort_s = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(fullA + i, 128);
            mbar_init(emptyA + i, 1);
        }
        for (int i = 0; i < 3; ++i) {
            mbar_init(fullB + i, 128);
            mbar_init(emptyB + i, 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 128);
        mbar_init(drain, 1);
        fence_barrier_init();
        fence_proxy_async();
    }
    // tile prefix sums over the groups (one warp)
    if (warp == 0) {
        int run = 0;
        for (int base = 0; base < ng; base += 32) {
            const int g = base + lane;
            int t = 0;
            if (g < ng) {
                const GroupInfo G = group_info(a, g, n_act);
                t = ((G.n + kMaxN - 1) / kMaxN) * MT;
            }
            int incl = t;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (g < ng) gstart[g] = run + incl - t;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            gstart[ng] = run;
            total_tiles_s = run;
        }
    }
    if (warp == 8) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int total = total_tiles_s;

    auto decode_tile = [&](int t, int &g, int &n0, int &m0) {
        int lo = 0, hi = ng;                      // largest g with gstart[g] <= t
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (gstart[mid] <= t) lo = mid;
            else hi = mid;
        }
        g = lo;
        const int local = t - gstart[g];
        n0 = (local / MT) * kMaxN;
        m0 = (local % MT) * kBM;
    };

    if (warp < 4) {
        // ------------------------------------------------------- producers
        long it = 0;                              // global k-step counter of this CTA
        const int row = tid;                      // weight row within the tile
        for (int t = blockIdx.x; t < total && !abort_s; t += gridDim.x) {
            int g, n0, m0;
            decode_tile(t, g, n0, m0);
            const GroupInfo G = group_info(a, g, n_act);
            const int nvalid = min(kMaxN, G.n - n0);
            const int N = (nvalid + 15) & ~15;
            const BlobView bv = blob_view(G.blob, BITS, a.H, a.I);
            // token rows (gate/up: x16 rows; down: h16 rows) of this tile
            asm volatile("bar.sync 1, 128;" ::: "memory");
            for (int n = tid; n < N; n += 128) {
                int r = 0;
                if (n < nvalid) {
                    if (GATEUP) r = min(max(G.row0 >= 0 ? a.perm_src[G.row0 + n0 + n] : n0 + n, 0), a.T - 1);
                    else r = (G.row0 >= 0 ? G.row0 : a.T * a.k) + n0 + n;
                }
                sTok[n] = r;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            const uint8_t *codes[2];
            const __half *scl[2];
            codes[0] = GATEUP ? bv.cg : bv.cd;
            codes[1] = bv.cu;
            scl[0] = GATEUP ? bv.sg : bv.sd;
            scl[1] = bv.su;
            const size_t rowbytes = static_cast<size_t>(K) * BITS / 8;
            const int nsc = K / 32;
            const uint8_t *bsrc = GATEUP ? reinterpret_cast<const uint8_t *>(a.x16)
                                         : reinterpret_cast<const uint8_t *>(a.h16);
            const size_t brow = static_cast<size_t>(K) * 2;
            auto issue = [&](int s, long j) {
                const int sb = static_cast<int>(j % kStB);
                if (!mbar_wait(emptyB + sb, static_cast<uint32_t>(((j / kStB) & 1) ^ 1), kSpin)) {
                    report(a.err, MOE_DEVERR_TIMEOUT);
                    abort_s = 1;
                }
                // raw codes + scales of this thread's row
                const uint32_t raw = smem_addr(sRaw + sb * Cfg::RAW_STAGE + static_cast<size_t>(row) * Cfg::RAW_ROW);
#pragma unroll
                for (int mat = 0; mat < Cfg::NA; ++mat) {
                    const uint8_t *src = codes[mat] + static_cast<size_t>(m0 + row) * rowbytes +
                                         static_cast<size_t>(s) * Cfg::RAW_CODE;
#pragma unroll
                    for (int q = 0; q < Cfg::RAW_CODE / 16; ++q)
                        cp_async16(raw + mat * Cfg::SEG + q * 16, src + q * 16, 16);
                    cp_async4(raw + mat * Cfg::SEG + Cfg::RAW_CODE,
                              scl[mat] + static_cast<size_t>(m0 + row) * nsc + 2 * s);
                }
                // token rows of the B tile, 16 bytes per copy, swizzled
                const uint32_t bdst = smem_addr(sB + sb * Cfg::B_STAGE);
                for (int idx = tid; idx < N * 8; idx += 128) {
                    const int n = idx >> 3, c = idx & 7;
                    const uint8_t *src = bsrc + static_cast<size_t>(sTok[n]) * brow + static_cast<size_t>(s) * 128 + c * 16;
                    cp_async16(bdst + n * 128 + ((c ^ (n & 7)) << 4), src, n < nvalid ? 16u : 0u);
                }
                cp_async_commit();
            };
            const long j0 = it;
            for (int s = 0; s < kLook && s < nk; ++s) issue(s, j0 + s);
            for (int s = 0; s < nk && !abort_s; ++s) {
                const long j = j0 + s;
                if (s + 1 < nk) cp_async_wait<1>();
                else cp_async_wait<0>();
                const int sa = static_cast<int>(j % kStA), sb = static_cast<int>(j % kStB);
                if (!mbar_wait(emptyA + sa, static_cast<uint32_t>(((j / kStA) & 1) ^ 1), kSpin)) {
                    report(a.err, MOE_DEVERR_TIMEOUT);
                    abort_s = 1;
                    break;
                }
                const uint8_t *raw = sRaw + sb * Cfg::RAW_STAGE + static_cast<size_t>(row) * Cfg::RAW_ROW;
#pragma unroll
                for (int mat = 0; mat < Cfg::NA; ++mat)
                    dequant_row<BITS>(raw + mat * Cfg::SEG,
                                      smem_addr(sA + sa * Cfg::A_STAGE + static_cast<size_t>(mat) * kBM * 128 +
                                                static_cast<size_t>(row) * 128),
                                      row);
                fence_proxy_async();
                mbar_arrive(fullA + sa);
                mbar_arrive(fullB + sb);
                if (s + kLook < nk) issue(s + kLook, j + kLook);
            }
            it = j0 + nk;
        }
        cp_async_wait<0>();
    } else if (warp < 8) {
        // -------------------------------------------------------- epilogue
        const int q = warp & 3;                   // TMEM lanes 32q .. 32q+31
        const int m = 32 * q + lane;              // weight row within the tile
        long tile_it = 0;
        for (int t = blockIdx.x; t < total && !abort_s; t += gridDim.x, ++tile_it) {
            int g, n0, m0;
            decode_tile(t, g, n0, m0);
            const GroupInfo G = group_info(a, g, n_act);
            const int nvalid = min(kMaxN, G.n - n0);
            if (!mbar_wait(acc_full, static_cast<uint32_t>(tile_it & 1), kSpin)) {
                report(a.err, MOE_DEVERR_TIMEOUT);
                abort_s = 1;
                break;
            }
            tc_fence_after();
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
            for (int c0 = 0; c0 < nvalid; c0 += 16) {
                float gv[16], uv[16];
                tmem_ld16(lane_base + c0, gv);
                if (GATEUP) tmem_ld16(lane_base + 256 + c0, uv);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int n = c0 + i;
                    if (n >= nvalid) break;
                    if (GATEUP) {
                        const float h = gv[i] / (1.0f + expf(-gv[i])) * uv[i];
                        const size_t r = static_cast<size_t>(G.row0 >= 0 ? G.row0 : a.T * a.k) + n0 + n;
                        a.h16[r * a.I + m0 + m] = __float2half_rn(h);
                    } else {
                        float *dst = G.row0 >= 0 ? a.y_perm + (static_cast<size_t>(G.row0) + n0 + n) * a.H
                                                 : a.y_shared + (static_cast<size_t>(n0) + n) * a.H;
                        dst[m0 + m] = gv[i];
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(acc_empty);
        }
    } else {
        // ------------------------------------------------------ MMA issuer
        long it = 0, tile_it = 0;
        for (int t = blockIdx.x; t < total && !abort_s; t += gridDim.x, ++tile_it) {
            int g, n0, m0;
            decode_tile(t, g, n0, m0);
            const GroupInfo G = group_info(a, g, n_act);
            const int nvalid = min(kMaxN, G.n - n0);
            const int N = (nvalid + 15) & ~15;
            const uint32_t idesc = idesc_f16_f32(kBM, N);
            if (lane == 0) {
                if (!mbar_wait(acc_empty, static_cast<uint32_t>((tile_it & 1) ^ 1), kSpin)) {
                    report(a.err, MOE_DEVERR_TIMEOUT);
                    abort_s = 1;
                }
                tc_fence_after();
                for (int s = 0; s < nk && !abort_s; ++s) {
                    const long j = it + s;
                    const int sa = static_cast<int>(j % kStA), sb = static_cast<int>(j % kStB);
                    if (!mbar_wait(fullA + sa, static_cast<uint32_t>((j / kStA) & 1), kSpin) ||
                        !mbar_wait(fullB + sb, static_cast<uint32_t>((j / kStB) & 1), kSpin)) {
                        report(a.err, MOE_DEVERR_TIMEOUT);
                        abort_s = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t b_addr = smem_addr(sB + sb * Cfg::B_STAGE);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t bdesc = desc_sw128(b_addr + kk * 32);
#pragma unroll
                        for (int mat = 0; mat < Cfg::NA; ++mat) {
                            const uint32_t a_addr =
                                smem_addr(sA + sa * Cfg::A_STAGE + static_cast<size_t>(mat) * kBM * 128) + kk * 32;
                            mma_f16(tmem + mat * 256, desc_sw128(a_addr), bdesc, idesc, (s | kk) != 0);
                        }
                    }
                    mma_commit(emptyA + sa);
                    mma_commit(emptyB + sb);
                }
                mma_commit(acc_full);
            }
            __syncwarp();
            it += nk;
        }
        // every MMA issued has completed before TMEM is released
        if (lane == 0) {
            mma_commit(drain);
            if (!mbar_wait(drain, 0, kSpin)) report(a.err, MOE_DEVERR_TIMEOUT);
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// x (bf16 or f32) [T, H] -> fp16 [T, H]
__global__ void k_to_half(const void *x, int bf16, long n, __half *out) {
    for (long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n / 4;
         i += static_cast<long>(gridDim.x) * blockDim.x) {
        const float4 v = bf16 ? load4(static_cast<const __nv_bfloat16 *>(x) + 4 * i)
                              : load4(static_cast<const float *>(x) + 4 * i);
        __half2 lo = __floats2half2_rn(v.x, v.y), hi = __floats2half2_rn(v.z, v.w);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t *>(&lo);
        u.y = *reinterpret_cast<uint32_t *>(&hi);
        reinterpret_cast<uint2 *>(out)[i] = u;
    }
}

// ------------------------------------------------------------------ host
static size_t align256(size_t v) { return (v + 255) / 256 * 256; }

size_t gemm_ws_bytes(int bits, int T, int k, int H, int I, int E) {
    (void)bits;
    (void)E;
    return align256(static_cast<size_t>(T) * H * 2) + align256(static_cast<size_t>(T) * (k + 1) * I * 2);
}

bool gemm_supported(int T, int k, int E) { return (T * k < E ? T * k : E) + 1 <= kMaxGroups; }

template <int BITS, bool GATEUP>
static int launch_k_gemm(const GemmArgs &a, cudaStream_t s) {
    using Cfg = GemmCfg<BITS, GATEUP>;
    int rc = cuda_status(cudaFuncSetAttribute(k_gemm<BITS, GATEUP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(Cfg::SMEM)),
                         "gemm smem attribute");
    if (rc) return rc;
    k_gemm<BITS, GATEUP><<<num_sms(), kGemmThreads, Cfg::SMEM, s>>>(a);
    count_launches(1);
    return cuda_status(cudaGetLastError(), "gemm launch");
}

int launch_gemm(int bits, const uint8_t *const *blobs, const int32_t *offsets, const int32_t *active,
                const int32_t *perm_src, const void *x, int x_dtype, int T, int k, int H, int I, int E,
                const uint8_t *shared_blob, float *y_perm, float *y_shared, void *ws, unsigned *err, cudaStream_t s) {
    uint8_t *p = static_cast<uint8_t *>(ws);
    GemmArgs a;
    a.blobs = blobs;
    a.offsets = offsets;
    a.active = active;
    a.perm_src = perm_src;
    a.shared = shared_blob;
    a.x16 = reinterpret_cast<__half *>(p);
    a.h16 = reinterpret_cast<__half *>(p + align256(static_cast<size_t>(T) * H * 2));
    a.y_perm = y_perm;
    a.y_shared = y_shared;
    a.T = T;
    a.k = k;
    a.H = H;
    a.I = I;
    a.E = E;
    a.err = err;
    {
        const long n = static_cast<long>(T) * H;
        long blocks = (n / 4 + 255) / 256;
        if (blocks > num_sms() * 8L) blocks = num_sms() * 8L;
        k_to_half<<<blocks, 256, 0, s>>>(x, x_dtype == MOE_BF16, n, const_cast<__half *>(a.x16));
        count_launches(1);
    }
    int rc = bits == 4 ? launch_k_gemm<4, true>(a, s) : launch_k_gemm<2, true>(a, s);
    if (rc) return rc;
    return bits == 4 ? launch_k_gemm<4, false>(a, s) : launch_k_gemm<2, false>(a, s);
}

}  // namespace moe
