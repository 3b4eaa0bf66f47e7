// Grouped expert GEMM on the 5th-generation tensor cores (prefill chunks).
//
// Strata article, section 2 item 3 and section 4: prompts are read in chunks
// of up to 8,192 tokens, and reading touches all the experts, so the expert
// step becomes a dense contraction per expert: D = W_e (dequantised) x X_e^T.
//
// Per tile: 128 weight rows (MMA M) x up to 256 of the expert's tokens (MMA N),
// K in steps of 64.  Weights are the A operand, so small token groups still
// fill the M = 128 datapath ("swap AB").  Roles of one persistent CTA per SM:
//   warps 0-7   copy their raw codes + scales a few k-steps ahead (cp.async
//               into private slots) and dequantise them to fp16 into the
//               128-byte-swizzled A stages;
//   warps 13-14 gather the tile's token rows (fp16) into the B stages with
//               cp.async, each thread arriving on the stage's barrier when
//               its copies land (cp.async.mbarrier.arrive.noinc);
//   warp  12    allocates TMEM and issues tcgen05.mma (one thread);
//   warps 8-11  epilogue: tcgen05.ld the fp32 accumulators and write
//               gate/up -> h = silu(g) * u (fp16) or down -> y rows (fp32).
// Every mbarrier wait is bounded; a timeout sets MOE_DEVERR_TIMEOUT and all
// roles leave their loops, after which TMEM is freed.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace moe {
using namespace sm100;

constexpr int kBM = 128;            // weight rows per tile
constexpr int kBK = 64;             // K per stage: one 128-byte row of fp16
constexpr int kProd = 256;          // dequantising threads: 128 rows x 2 parts
constexpr int kLoad = 64;           // token-row loader threads
constexpr int kGemmThreads = 480;   // 8 dequant warps, 4 epilogue warps, 1 MMA warp, 2 loader warps
constexpr long kSpin = 1L << 22;    // polls before a wait gives up (about a second)
constexpr int kMaxGroups = 2048;

// MAXN: tokens per tile.  Small tiles (64) leave room for deep rings (the
// HBM-bound regime: few tokens per expert); large tiles (256) fill the
// tensor cores when experts hold hundreds of tokens.
template <int BITS, bool GATEUP, int MAXN>
struct GemmCfg {
    static constexpr int NA = GATEUP ? 2 : 1;                 // weight matrices per tile (gate, up)
    static constexpr int ELEMS = GATEUP ? 64 : 32;            // elements one producer thread dequantises per k-step
    static constexpr int RAW_CODE = ELEMS * BITS / 8;         // its code bytes per k-step
    static constexpr int SEG = (RAW_CODE + 4 + 15) / 16 * 16; // codes + two fp16 scales, 16-byte aligned
    static constexpr int SA = GATEUP ? 3 : 4;                 // A (dequantised weight) stages
    static constexpr int SB = MAXN > 128 ? (GATEUP ? 3 : 4) : 8;   // B (token row) stages
    static constexpr int L = MAXN > 128 ? (GATEUP ? 2 : 3) : 4;    // k-steps the code copies run ahead (= slots)
    static constexpr int ACC = NA * MAXN * 2 <= 512 ? 2 : 1;  // TMEM accumulator buffers
    static constexpr int TMEM_COLS = ACC * NA * MAXN <= 128 ? 128 : (ACC * NA * MAXN <= 256 ? 256 : 512);
    static constexpr size_t A_STAGE = static_cast<size_t>(NA) * kBM * 128;
    static constexpr size_t B_STAGE = static_cast<size_t>(MAXN) * 128;
    static constexpr size_t RAW_STAGE = static_cast<size_t>(kProd) * SEG;
    static constexpr size_t OFF_A = 0;
    static constexpr size_t OFF_B = OFF_A + SA * A_STAGE;
    static constexpr size_t OFF_RAW = OFF_B + SB * B_STAGE;
    static constexpr size_t OFF_TOK = OFF_RAW + L * RAW_STAGE;
    static constexpr size_t OFF_GS = OFF_TOK + MAXN * 4;
    static constexpr size_t OFF_BAR = (OFF_GS + (kMaxGroups + 1) * 4 + 15) / 16 * 16;
    static constexpr size_t SMEM = OFF_BAR + 32 * 8 + 16 + 1024;   // bars, TMEM address, tile count, abort
                                                                   // flag; + slack for 1024-byte alignment
    static_assert(2 * SA + 2 * SB + 5 <= 32, "barrier slots");
    static_assert(SMEM <= 232448, "shared memory per block (no static shared memory is used)");
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

// One tile of this CTA's sequence: group, first token, first weight row.
struct TileInfo {
    GroupInfo G;
    int n0, m0, nvalid, N;
};

// bytes hold one code per byte; builds the half2 (1024 + q_a, 1024 + q_b)
__device__ __forceinline__ uint32_t pair16(uint32_t bytes, uint32_t sel) { return __byte_perm(bytes, 0x64646464u, sel); }
__device__ __forceinline__ uint32_t dq2(uint32_t magic_pair, __half2 offset, __half2 d2) {
    __half2 h = *reinterpret_cast<__half2 *>(&magic_pair);
    h = __hmul2(__hsub2(h, offset), d2);       // (q - offset) exact, then one rounding of d * (q - offset)
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ void st_shared16(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Dequantises one quant block (32 elements) into chunks chunk0..chunk0+3 of a
// swizzled 128-byte A row (chunk c stored at c ^ (row % 8)).
template <int BITS>
__device__ __forceinline__ void dequant_block(const uint8_t *codes, __half2 d2, uint32_t a_row, int chunk0, int sw) {
    if constexpr (BITS == 4) {
        const __half2 off = __float2half2_rn(1032.0f);
        const uint4 w = *reinterpret_cast<const uint4 *>(codes);
        // chunk j (8 elements): 0 = low nibbles of bytes 0-7, 1 = low of 8-15,
        //                       2 = high nibbles of bytes 0-7, 3 = high of 8-15
        const uint32_t src[4][2] = {{w.x & 0x0F0F0F0Fu, w.y & 0x0F0F0F0Fu},
                                    {w.z & 0x0F0F0F0Fu, w.w & 0x0F0F0F0Fu},
                                    {(w.x >> 4) & 0x0F0F0F0Fu, (w.y >> 4) & 0x0F0F0F0Fu},
                                    {(w.z >> 4) & 0x0F0F0F0Fu, (w.w >> 4) & 0x0F0F0F0Fu}};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            st_shared16(a_row + ((((chunk0 + j) ^ sw)) << 4), dq2(pair16(src[j][0], 0x5140u), off, d2),
                        dq2(pair16(src[j][0], 0x5342u), off, d2), dq2(pair16(src[j][1], 0x5140u), off, d2),
                        dq2(pair16(src[j][1], 0x5342u), off, d2));
    } else {
        const __half2 off = __float2half2_rn(1026.0f);
        const uint2 w = *reinterpret_cast<const uint2 *>(codes);
#pragma unroll
        for (int j = 0; j < 4; ++j) {            // crumb level j: elements 8j..8j+7 of the block
            const uint32_t c0 = (w.x >> (2 * j)) & 0x03030303u, c1 = (w.y >> (2 * j)) & 0x03030303u;
            st_shared16(a_row + ((((chunk0 + j) ^ sw)) << 4), dq2(pair16(c0, 0x5140u), off, d2),
                        dq2(pair16(c0, 0x5342u), off, d2), dq2(pair16(c1, 0x5140u), off, d2),
                        dq2(pair16(c1, 0x5342u), off, d2));
        }
    }
}

template <int BITS, bool GATEUP, int MAXN>
__global__ void __launch_bounds__(kGemmThreads, 1) k_gemm(GemmArgs a) {
    using Cfg = GemmCfg<BITS, GATEUP, MAXN>;
    constexpr int SA = Cfg::SA, SB = Cfg::SB, L = Cfg::L, ACC = Cfg::ACC, NA = Cfg::NA;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + Cfg::OFF_A;
    uint8_t *sB = smem + Cfg::OFF_B;
    uint8_t *sRaw = smem + Cfg::OFF_RAW;
    int32_t *tok_s = reinterpret_cast<int32_t *>(smem + Cfg::OFF_TOK);
    int32_t *gstart = reinterpret_cast<int32_t *>(smem + Cfg::OFF_GS);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *fullA = bars, *emptyA = bars + SA, *fullB = bars + 2 * SA, *emptyB = bars + 2 * SA + SB;
    uint64_t *accF = bars + 2 * SA + 2 * SB, *accE = accF + 2, *drain = accF + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 32);
    int *total_tiles_p = reinterpret_cast<int *>(bars + 32) + 1;
    volatile int &abort_s = *(reinterpret_cast<int *>(bars + 32) + 2);   // read in loop conditions: never cached

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = GATEUP ? a.H : a.I;           // reduction length
    const int Mtot = GATEUP ? a.I : a.H;        // weight rows
    const int MT = Mtot / kBM;
    const int nk = K / kBK;
    const int n_act = min(max(a.active[0], 0), min(a.E, a.T * a.k));
    const int ng = n_act + (a.shared ? 1 : 0);

    if (tid == 0) {
        abort_s = 0;
        for (int i = 0; i < SA; ++i) {
            mbar_init(fullA + i, kProd);
            mbar_init(emptyA + i, 1);
        }
        for (int i = 0; i < SB; ++i) {
            mbar_init(fullB + i, kLoad);
            mbar_init(emptyB + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(accF + i, 1);
            mbar_init(accE + i, 128);
        }
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
                t = ((G.n + MAXN - 1) / MAXN) * MT;
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
            *total_tiles_p = run;
        }
    }
    if (warp == 12) {
        tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int total = *total_tiles_p;
    const int n_my = blockIdx.x < total ? (total - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1 : 0;
    const long J = static_cast<long>(n_my) * nk;   // k-steps of this CTA

    auto tile_of = [&](int i) {                  // i-th tile of this CTA
        const int t = blockIdx.x + i * gridDim.x;
        int lo = 0, hi = ng;                     // largest g with gstart[g] <= t
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (gstart[mid] <= t) lo = mid;
            else hi = mid;
        }
        TileInfo ti;
        ti.G = group_info(a, lo, n_act);
        const int local = t - gstart[lo];
        ti.n0 = (local / MT) * MAXN;
        ti.m0 = (local % MT) * kBM;
        ti.nvalid = min(MAXN, ti.G.n - ti.n0);
        ti.N = (ti.nvalid + 15) & ~15;
        return ti;
    };
    auto fail = [&]() {
        report(a.err, MOE_DEVERR_TIMEOUT);
        abort_s = 1;
    };

    if (warp < 8) {
        // ------------------------------------------------- dequantisation
        const int row = tid & 127, part = tid >> 7;
        const size_t rowbytes = static_cast<size_t>(K) * BITS / 8;
        const int nsc = K / 32;
        int raw_tile = -1;
        TileInfo rt{};
        // copies of this thread's codes + scales of k-step jr into its slot jr % L
        auto issue_raw = [&](long jr) {
            if (jr >= J) return;
            const int i = static_cast<int>(jr / nk), s = static_cast<int>(jr % nk);
            if (i != raw_tile) {
                rt = tile_of(i);
                raw_tile = i;
            }
            const BlobView bv = blob_view(rt.G.blob, BITS, a.H, a.I);
            const uint8_t *codes = GATEUP ? (part ? bv.cu : bv.cg) : bv.cd;
            const __half *scl = GATEUP ? (part ? bv.su : bv.sg) : bv.sd;
            const size_t m = static_cast<size_t>(rt.m0 + row);
            const uint8_t *src = codes + m * rowbytes + static_cast<size_t>(s) * (kBK * BITS / 8) +
                                 (GATEUP ? 0 : part * Cfg::RAW_CODE);
            const uint32_t dst = smem_addr(sRaw + (jr % L) * Cfg::RAW_STAGE + static_cast<size_t>(tid) * Cfg::SEG);
            if constexpr (Cfg::RAW_CODE >= 16) {
#pragma unroll
                for (int q = 0; q < Cfg::RAW_CODE / 16; ++q) cp_async16(dst + q * 16, src + q * 16, 16);
            } else {
                asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
            }
            cp_async4(dst + Cfg::RAW_CODE, scl + m * nsc + 2 * s);
        };
        for (int p = 0; p < L; ++p) {             // prologue: one commit group per k-step
            issue_raw(p);
            cp_async_commit();
        }
        for (long j = 0; j < J && !abort_s; ++j) {
            cp_async_wait<L - 1>();              // this thread's codes of k-step j have landed
            const int sa = static_cast<int>(j % SA);
            if (!mbar_wait(emptyA + sa, static_cast<uint32_t>(((j / SA) & 1) ^ 1), kSpin)) {
                fail();
                break;
            }
            const uint8_t *raw = sRaw + (j % L) * Cfg::RAW_STAGE + static_cast<size_t>(tid) * Cfg::SEG;
            const __half2 s01 = *reinterpret_cast<const __half2 *>(raw + Cfg::RAW_CODE);
            const uint32_t a_row = smem_addr(sA + sa * Cfg::A_STAGE +
                                             static_cast<size_t>(GATEUP ? part : 0) * kBM * 128 +
                                             static_cast<size_t>(row) * 128);
            if (GATEUP) {
                dequant_block<BITS>(raw, __low2half2(s01), a_row, 0, row & 7);
                dequant_block<BITS>(raw + 4 * BITS, __high2half2(s01), a_row, 4, row & 7);
            } else {
                dequant_block<BITS>(raw, part ? __high2half2(s01) : __low2half2(s01), a_row, 4 * part, row & 7);
            }
            fence_proxy_async();
            mbar_arrive(fullA + sa);
            issue_raw(j + L);                    // into the slot just read
            cp_async_commit();
        }
        cp_async_wait<0>();
    } else if (warp >= 13) {
        // --------------------------------------------------- token rows
        // Loader warp lw copies rows lw*MAXN/2 .. of each tile: lane = 8 x row
        // + 16-byte chunk.  Its token indices live in a warp-private table.
        const int lw = warp - 13;
        constexpr int HALF = MAXN / 2;
        int32_t *tok = tok_s + lw * HALF;
        const uint8_t *bsrc = GATEUP ? reinterpret_cast<const uint8_t *>(a.x16)
                                     : reinterpret_cast<const uint8_t *>(a.h16);
        const size_t brow = static_cast<size_t>(K) * 2;
        const int c = lane & 7;
        int cur = -1;
        TileInfo bt{};
        for (long j = 0; j < J && !abort_s; ++j) {
            const int i = static_cast<int>(j / nk), s = static_cast<int>(j % nk);
            if (i != cur) {
                bt = tile_of(i);
                cur = i;
                __syncwarp();
                for (int nl = lane; nl < HALF; nl += 32) {
                    const int n = lw * HALF + nl;
                    int v = 0;
                    if (n < bt.nvalid) {
                        if (GATEUP)
                            v = min(max(bt.G.row0 >= 0 ? a.perm_src[bt.G.row0 + bt.n0 + n] : bt.n0 + n, 0), a.T - 1);
                        else
                            v = (bt.G.row0 >= 0 ? bt.G.row0 : a.T * a.k) + bt.n0 + n;
                    }
                    tok[nl] = v;
                }
                __syncwarp();
            }
            const int sb = static_cast<int>(j % SB);
            if (!mbar_wait(emptyB + sb, static_cast<uint32_t>(((j / SB) & 1) ^ 1), kSpin)) {
                fail();
                break;
            }
            const uint32_t bdst = smem_addr(sB + sb * Cfg::B_STAGE);
#pragma unroll 4
            for (int nl = lane >> 3; nl < HALF; nl += 4) {
                const int n = lw * HALF + nl;
                if (n < bt.N) {
                    const uint8_t *src = bsrc + static_cast<size_t>(tok[nl]) * brow + static_cast<size_t>(s) * 128 + c * 16;
                    cp_async16(bdst + n * 128 + ((c ^ (n & 7)) << 4), src, n < bt.nvalid ? 16u : 0u);
                }
            }
            asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(fullB + sb))
                         : "memory");
        }
        cp_async_wait<0>();
    } else if (warp < 12) {
        // -------------------------------------------------------- epilogue
        const int q = warp & 3;                   // TMEM lanes 32q .. 32q+31
        const int m = 32 * q + lane;              // weight row within the tile
        for (int i = 0; i < n_my && !abort_s; ++i) {
            const TileInfo ti = tile_of(i);
            const int b = i % ACC;
            if (!mbar_wait(accF + b, static_cast<uint32_t>((i / ACC) & 1), kSpin)) {
                fail();
                break;
            }
            tc_fence_after();
            const uint32_t base = tmem + (static_cast<uint32_t>(32 * q) << 16) + b * NA * MAXN;
            for (int c0 = 0; c0 < ti.nvalid; c0 += 16) {
                float gv[16], uv[16];
                tmem_ld16(base + c0, gv);
                if (GATEUP) tmem_ld16(base + MAXN + c0, uv);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int n = c0 + e;
                    if (n >= ti.nvalid) break;
                    if (GATEUP) {
                        const float h = gv[e] / (1.0f + expf(-gv[e])) * uv[e];
                        const size_t r = static_cast<size_t>(ti.G.row0 >= 0 ? ti.G.row0 : a.T * a.k) + ti.n0 + n;
                        a.h16[r * a.I + ti.m0 + m] = __float2half_rn(h);
                    } else {
                        float *dst = ti.G.row0 >= 0 ? a.y_perm + (static_cast<size_t>(ti.G.row0) + ti.n0 + n) * a.H
                                                    : a.y_shared + (static_cast<size_t>(ti.n0) + n) * a.H;
                        dst[ti.m0 + m] = gv[e];
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(accE + b);
        }
    } else {
        // ------------------------------------------------------ MMA issuer
        for (int i = 0; i < n_my && !abort_s; ++i) {
            const TileInfo ti = tile_of(i);
            const uint32_t idesc = idesc_f16_f32(kBM, ti.N);
            const int b = i % ACC;
            if (lane == 0) {
                if (!mbar_wait(accE + b, static_cast<uint32_t>(((i / ACC) & 1) ^ 1), kSpin)) fail();
                tc_fence_after();
                for (int s = 0; s < nk && !abort_s; ++s) {
                    const long j = static_cast<long>(i) * nk + s;
                    const int sa = static_cast<int>(j % SA), sb = static_cast<int>(j % SB);
                    if (!mbar_wait(fullA + sa, static_cast<uint32_t>((j / SA) & 1), kSpin) ||
                        !mbar_wait(fullB + sb, static_cast<uint32_t>((j / SB) & 1), kSpin)) {
                        fail();
                        break;
                    }
                    tc_fence_after();
                    const uint32_t b_addr = smem_addr(sB + sb * Cfg::B_STAGE);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t bdesc = desc_sw128(b_addr + kk * 32);
#pragma unroll
                        for (int mat = 0; mat < NA; ++mat) {
                            const uint32_t a_addr =
                                smem_addr(sA + sa * Cfg::A_STAGE + static_cast<size_t>(mat) * kBM * 128) + kk * 32;
                            mma_f16(tmem + b * NA * MAXN + mat * MAXN, desc_sw128(a_addr), bdesc, idesc,
                                    (s | kk) != 0);
                        }
                    }
                    mma_commit(emptyA + sa);
                    mma_commit(emptyB + sb);
                }
                mma_commit(accF + b);
            }
            __syncwarp();
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
    if (warp == 12) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::TMEM_COLS);
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

template <int BITS, bool GATEUP, int MAXN>
static int launch_k_gemm(const GemmArgs &a, cudaStream_t s) {
    using Cfg = GemmCfg<BITS, GATEUP, MAXN>;
    int rc = cuda_status(cudaFuncSetAttribute(k_gemm<BITS, GATEUP, MAXN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(Cfg::SMEM)),
                         "gemm smem attribute");
    if (rc) return rc;
    k_gemm<BITS, GATEUP, MAXN><<<num_sms(), kGemmThreads, Cfg::SMEM, s>>>(a);
    count_launches(1);
    return cuda_status(cudaGetLastError(), "gemm launch");
}

template <int BITS>
static int launch_pair(const GemmArgs &a, bool large, cudaStream_t s) {
    int rc = large ? launch_k_gemm<BITS, true, 256>(a, s) : launch_k_gemm<BITS, true, 64>(a, s);
    if (rc) return rc;
    return large ? launch_k_gemm<BITS, false, 256>(a, s) : launch_k_gemm<BITS, false, 64>(a, s);
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
    // tiles of 256 tokens once experts hold more than ~48 tokens on average, else 64
    const int groups = T * k < E ? T * k : E;
    const bool large = static_cast<long>(T) * k > 48L * (groups > 0 ? groups : 1);
    return bits == 4 ? launch_pair<4>(a, large, s) : launch_pair<2>(a, large, s);
}

}  // namespace moe
