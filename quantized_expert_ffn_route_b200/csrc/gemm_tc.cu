// Grouped expert GEMM on the 5th-generation tensor cores (prefill chunks).
//
// Strata article, section 2 item 3 and section 4: prompts are read in chunks
// of up to 8,192 tokens, and reading touches all the experts, so the expert
// step becomes a dense contraction per expert: D = W_e (dequantised) x X_e^T.
//
// Per tile: two 128-row weight matrices (gate and up rows m0..m0+127, or down
// rows m0..m0+255 as two halves) x up to MAXN of the expert's tokens, K in
// steps of 64.  Weights are the MMA's A operand (M = 128), tokens the N side,
// so a group of ten tokens still fills the datapath ("swap AB"); both
// matrices share the token tile.  Roles of one persistent CTA per SM:
//   warps 0-15  copy the weight codes of a tile's rows, a few k-steps at a
//               time, into raw slots (each row's span is contiguous, so the
//               copies are whole lines), then each thread dequantises one
//               32-weight block per k-step to fp16 into a 128-byte-swizzled
//               A stage;
//   warps 21+ gather the tile's token rows (fp16) into the B stages with
//               cp.async, a few k-steps ahead; each warp publishes a stage
//               with one barrier arrival once its copies have landed (eight
//               warps: with two, the gather set the pace of every k-step);
//   warp  20    allocates TMEM and issues tcgen05.mma (one thread);
//   warps 16-19 epilogue: tcgen05.ld the fp32 accumulators and write
//               gate/up -> h = silu(g) * u (fp16) or down -> y rows (fp32).
// The CTA's tile list (expert blob, token range, weight rows) is built once
// in shared memory.  Every mbarrier wait is bounded; a timeout sets
// MOE_DEVERR_TIMEOUT and all roles leave their loops, after which TMEM is
// freed.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace moe {
using namespace sm100;

constexpr int kBM = 128;            // weight rows per matrix of a tile (MMA M)
constexpr int kBK = 64;             // K per stage: one 128-byte row of fp16
constexpr int kDeq = 512;           // dequantising threads: 128 rows x 2 matrices x 2 blocks
// Token-row loader threads: 8 warps for 256-token tiles (there the gather
// sets the pace of every k-step), 2 for 64-token tiles (there the weights do).
__host__ __device__ constexpr int gemm_loaders(int maxn) { return maxn > 64 ? 256 : 64; }
__host__ __device__ constexpr int gemm_threads(int maxn) { return 672 + gemm_loaders(maxn); }
constexpr int kEpiWarp0 = 16, kMmaWarp = 20, kLoadWarp0 = 21;
// threads: 16 dequant, 4 epilogue, 1 MMA and gemm_loaders / 32 loader warps
constexpr long kSpin = 1L << 22;    // polls before a wait gives up (about a second); the test hook may lower it
constexpr int kMaxGroups = 4096;    // groups (active experts + shared) one launch may hold
constexpr size_t kSmemLimit = 232448;

// One tile of a CTA's list.
struct TileEntry {
    const uint8_t *blob;
    int row0;     // first permuted row of the group, or -1 for the shared expert
    int n0;       // first token of the tile within the group
    int m0;       // first weight row
    int nvalid;   // tokens in the tile
};

// MAXN: tokens per tile.  Small tiles (64) leave room for deep rings (the
// HBM-bound regime: few tokens per expert); large tiles (256) fill the
// tensor cores when experts hold hundreds of tokens.
template <int BITS, bool GATEUP, int MAXN>
struct GemmCfg {
    static constexpr int CODE = 32 * BITS / 8;                // code bytes of one block
    static constexpr int CBK = 2 * CODE;                      // code bytes of one row per k-step
    static constexpr int SA = MAXN > 128 ? 2 : 3;             // A (dequantised weight) stages
    static constexpr int SB = MAXN > 128 ? 3 : 4;             // B (token row) stages
    static constexpr int R = 2;                               // raw-code slots
    static constexpr int KSMAX = MAXN > 128 ? 2 : 4;          // k-steps per raw slot
    static constexpr int CS = KSMAX * CBK + 16;               // padded row stride of a slot's codes
    static constexpr int ACC = 2 * MAXN * 2 <= 512 ? 2 : 1;   // TMEM accumulator buffers
    static constexpr int TMEM_COLS = ACC * 2 * MAXN <= 128 ? 128 : (ACC * 2 * MAXN <= 256 ? 256 : 512);
    static constexpr size_t A_STAGE = static_cast<size_t>(2) * kBM * 128;
    static constexpr size_t B_STAGE = static_cast<size_t>(MAXN) * 128;
    static constexpr size_t RAW_CODES = static_cast<size_t>(2 * kBM) * CS;
    static constexpr size_t RAW_SLOT = RAW_CODES + static_cast<size_t>(2 * kBM) * 16;   // + 16 B of scales per row
    static constexpr size_t OFF_A = 0;
    static constexpr size_t OFF_B = OFF_A + SA * A_STAGE;
    static constexpr size_t OFF_RAW = OFF_B + SB * B_STAGE;
    static constexpr size_t OFF_TOK = OFF_RAW + R * RAW_SLOT;
    static constexpr size_t OFF_BAR = (OFF_TOK + MAXN * 4 + 15) / 16 * 16;
    static constexpr size_t OFF_TILES = OFF_BAR + 32 * 8 + 16;   // bars, TMEM address, tile count, abort flag
    static constexpr size_t FIXED = OFF_TILES + 1024;            // + slack for 1024-byte alignment
    static size_t smem(int cap) { return FIXED + static_cast<size_t>(cap) * sizeof(TileEntry); }
    static_assert(2 * SA + 2 * SB + 5 + 2 * R <= 32, "barrier slots");
    static_assert(SB * B_STAGE >= (kMaxGroups + 1) * 4, "group scratch fits the B ring");
    static_assert(KSMAX * 4 <= 16, "scale bytes of a row per slot");
    static_assert(FIXED <= kSmemLimit, "shared memory per block");
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
    long spin;              // polls before a pipeline wait gives up (the drain before TMEM is freed keeps kSpin)
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
        const bool rows_ok = G.row0 >= 0 && G.n >= 0 && G.row0 + G.n <= a.T * a.k;
#ifdef MOE_DEBUG
        if (!ok) report(a.err, MOE_DEVERR_BAD_EXPERT);
        else if (!rows_ok) report(a.err, MOE_DEVERR_BAD_ROW);
        else if (!G.blob) report(a.err, MOE_DEVERR_NULL_BLOB);
#endif
        if (!rows_ok) G.n = 0;
    } else {
        G.row0 = -1;
        G.n = a.T;
        G.blob = a.shared;
    }
    if (!G.blob) G.n = 0;
    return G;
}

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
__global__ void __launch_bounds__(gemm_threads(MAXN), 1) k_gemm(GemmArgs a, int tile_cap) {
    using Cfg = GemmCfg<BITS, GATEUP, MAXN>;
    constexpr int SA = Cfg::SA, SB = Cfg::SB, R = Cfg::R, ACC = Cfg::ACC;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + Cfg::OFF_A;
    uint8_t *sB = smem + Cfg::OFF_B;
    uint8_t *sRaw = smem + Cfg::OFF_RAW;
    int32_t *tok_s = reinterpret_cast<int32_t *>(smem + Cfg::OFF_TOK);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *fullA = bars, *emptyA = bars + SA, *fullB = bars + 2 * SA, *emptyB = bars + 2 * SA + SB;
    uint64_t *accF = bars + 2 * SA + 2 * SB, *accE = accF + 2, *drain = accF + 4;
    uint64_t *rawFull = drain + 1, *rawEmpty = rawFull + R;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 32);
    volatile int &abort_s = *(reinterpret_cast<int *>(bars + 32) + 2);   // read in loop conditions: never cached
    TileEntry *tiles = reinterpret_cast<TileEntry *>(smem + Cfg::OFF_TILES);
    int32_t *gcnt = reinterpret_cast<int32_t *>(sB);   // per-group tile counts while the tile list is built

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = GATEUP ? a.H : a.I;                  // reduction length
    const int Mtot = GATEUP ? a.I : a.H;               // weight rows
    const int MROWS = GATEUP ? kBM : 2 * kBM;          // weight rows a tile advances by
    const int MT = (Mtot + MROWS - 1) / MROWS;
    const int nk = K / kBK;
    // k-steps per raw-code slot: the largest of KSMAX, 2, 1 dividing nk (a
    // slot never spans two tiles)
    const int KS = nk % Cfg::KSMAX == 0 ? Cfg::KSMAX : (nk % 2 == 0 ? 2 : 1);
    const int n_act = guard_count(a.active[0], min(a.E, a.T * a.k), a.err);
    const int ng = min(n_act + (a.shared ? 1 : 0), kMaxGroups);

    if (tid == 0) {
        abort_s = 0;
        for (int i = 0; i < SA; ++i) {
            mbar_init(fullA + i, kDeq / 32);           // one arrival per dequantising warp
            mbar_init(emptyA + i, 1);
        }
        for (int i = 0; i < SB; ++i) {
            mbar_init(fullB + i, gemm_loaders(MAXN) / 32);   // one arrival per loader warp
            mbar_init(emptyB + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(accF + i, 1);
            mbar_init(accE + i, 4);                     // one arrival per epilogue warp
        }
        mbar_init(drain, 1);
        for (int i = 0; i < R; ++i) {
            mbar_init(rawFull + i, kDeq / 32);         // one arrival per dequantising warp
            mbar_init(rawEmpty + i, kDeq / 32);
        }
        fence_barrier_init();
        fence_proxy_async();
    }
    // ---- the CTA's tile list: tiles are numbered group by group, m-tile
    // fastest, and dealt to CTAs round robin (tile t -> CTA t % grid)
    for (int g = tid; g < ng; g += blockDim.x) {
        const GroupInfo G = group_info(a, g, n_act);
        gcnt[g] = ((G.n + MAXN - 1) / MAXN) * MT;
    }
    __syncthreads();
    if (warp == 0) {                                   // exclusive prefix sum, in place
        int run = 0;
        for (int base = 0; base < ng; base += 32) {
            const int g = base + lane;
            const int t = g < ng ? gcnt[g] : 0;
            int incl = t;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (g < ng) gcnt[g] = run + incl - t;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) gcnt[ng] = run;
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    __syncthreads();
    const int total = gcnt[ng];
    const int grid = static_cast<int>(gridDim.x), bid = static_cast<int>(blockIdx.x);
    int n_my = bid < total ? (total - 1 - bid) / grid + 1 : 0;
    for (int g = tid; g < ng; g += blockDim.x) {
        const int start = gcnt[g], cnt = gcnt[g + 1] - start;
        if (cnt <= 0) continue;
        const GroupInfo G = group_info(a, g, n_act);
        for (int tt = start + ((bid - start) % grid + grid) % grid; tt < start + cnt; tt += grid) {
            const int i = (tt - bid) / grid, local = tt - start;
            if (i >= tile_cap) break;
            TileEntry te;
            te.blob = G.blob;
            te.row0 = G.row0;
            te.n0 = (local / MT) * MAXN;
            te.m0 = (local % MT) * MROWS;
            te.nvalid = min(MAXN, G.n - te.n0);
            tiles[i] = te;
        }
    }
    if (n_my > tile_cap) {                             // offsets inconsistent with T*k: do nothing
        if (tid == 0) report(a.err, MOE_DEVERR_BAD_ROW);
        n_my = 0;
    }
    tc_fence_before();
    __syncthreads();                                   // tile list final; the B ring is free again
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const long J = static_cast<long>(n_my) * nk;      // k-steps of this CTA
    auto fail = [&]() {
        report(a.err, MOE_DEVERR_TIMEOUT);
        abort_s = 1;
    };
    auto aborted = [&]() { return __shfl_sync(0xffffffffu, abort_s, 0) != 0; };   // the same answer on every lane

    if (warp < kEpiWarp0) {
        // ------------------------------------------------- dequantisation
        // The 512 threads first copy, together, the codes of KS k-steps of the
        // tile's 256 weight rows into a raw slot: each row's span is
        // contiguous in the blob, so eight lanes cover 128 bytes of one row
        // and a warp instruction touches four whole lines.  Slots are handed
        // over with (bounded) barriers: rawFull when every warp's copies
        // landed, rawEmpty when every warp has read the slot.  Then each
        // thread dequantises one 32-weight block per k-step, thread -> (row,
        // matrix, block), from the slot into a 128-byte-swizzled A stage.
        const int row = tid & 127, mat = (tid >> 7) & 1, half = tid >> 8;
        const int r = mat * kBM + row;
        const size_t rowbytes = static_cast<size_t>(K) * BITS / 8;
        const int nsc = K / 32;
        const long U = J / KS;
        auto issue = [&](long u) {                     // copies of slot u (all threads)
            if (u >= U) return;
            const long j0 = u * KS;
            const TileEntry te = tiles[j0 / nk];
            const int s0 = static_cast<int>(j0 % nk);
            const BlobView bv = blob_view(te.blob, BITS, a.H, a.I);
            uint8_t *raw = sRaw + (u % R) * Cfg::RAW_SLOT;
            const int cpr = KS * Cfg::CBK / 16;        // 16-byte chunks of one row
            for (int q = tid; q < 2 * kBM * cpr; q += kDeq) {
                const int rr = q / cpr, c = q - rr * cpr;
                const int mt = rr >> 7, m = te.m0 + (GATEUP ? 0 : kBM * mt) + (rr & 127);
                const bool ok = m < Mtot;
                const uint8_t *codes = GATEUP ? (mt ? bv.cu : bv.cg) : bv.cd;
                cp_async16(smem_addr(raw + rr * Cfg::CS + c * 16),
                           codes + (ok ? static_cast<size_t>(m) : 0) * rowbytes + s0 * Cfg::CBK + c * 16, ok ? 16u : 0u);
            }
            if (tid < 2 * kBM) {                       // one row's scales: 4*KS bytes
                const int mt = tid >> 7, m = te.m0 + (GATEUP ? 0 : kBM * mt) + (tid & 127);
                const bool ok = m < Mtot;
                const __half *scl = (GATEUP ? (mt ? bv.su : bv.sg) : bv.sd) + (ok ? static_cast<size_t>(m) : 0) * nsc +
                                    2 * s0;
                const uint32_t dst = smem_addr(raw + Cfg::RAW_CODES + tid * 16);
                if (KS == 4) cp_async16(dst, scl, ok ? 16u : 0u);
                else if (KS == 2) cp_async8z(dst, scl, ok ? 8u : 0u);
                else cp_async4z(dst, scl, ok ? 4u : 0u);
            }
        };
        issue(0);
        cp_async_commit();
        for (long j = 0; j < J && !aborted(); ++j) {
            const long u = j / KS;
            const int sl = static_cast<int>(j - u * KS), slot = static_cast<int>(u % R);
            if (sl == 0) {
                // the next slot: wait until every warp has read its previous
                // contents (slot u + 1 - R), then copy
                int ok = 1;
                if (lane == 0 && u + 1 >= R)
                    ok = mbar_wait(rawEmpty + (u + 1) % R, static_cast<uint32_t>(((u + 1 - R) / R) & 1), a.spin);
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    fail();
                    break;
                }
                issue(u + 1);
                cp_async_commit();
                cp_async_wait<1>();                    // this thread's copies of slot u have landed
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(rawFull + slot);
                    ok = mbar_wait(rawFull + slot, static_cast<uint32_t>((u / R) & 1), a.spin);
                }
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    fail();
                    break;
                }
                __syncwarp();                          // the lanes read the slot after lane 0's acquire
            }
            const int sa = static_cast<int>(j % SA);
            // one lane per warp polls the stage barrier; the warp follows it
            int ok = 1;
            if (lane == 0) ok = mbar_wait(emptyA + sa, static_cast<uint32_t>(((j / SA) & 1) ^ 1), a.spin);
            if (!__shfl_sync(0xffffffffu, ok, 0)) {
                fail();
                break;
            }
            const uint8_t *raw = sRaw + slot * Cfg::RAW_SLOT;
            const __half2 s01 = *reinterpret_cast<const __half2 *>(raw + Cfg::RAW_CODES + r * 16 + sl * 4);
            const uint32_t a_row = smem_addr(sA + sa * Cfg::A_STAGE + static_cast<size_t>(mat) * kBM * 128 +
                                             static_cast<size_t>(row) * 128);
            dequant_block<BITS>(raw + r * Cfg::CS + sl * Cfg::CBK + half * Cfg::CODE,
                                half ? __high2half2(s01) : __low2half2(s01), a_row, 4 * half, row & 7);
            fence_proxy_async();                       // this thread's A writes -> async proxy
            __syncwarp();                              // ... ordered before lane 0's release-arrive
            if (lane == 0) {
                mbar_arrive(fullA + sa);
                if (sl == KS - 1) mbar_arrive(rawEmpty + slot);   // this warp is done with slot u
            }
        }
        cp_async_wait<0>();
    } else if (warp >= kLoadWarp0) {
        // --------------------------------------------------- token rows
        // Loader warp lw copies rows lw * HALF .. of each tile: lane = 8 x row
        // + 16-byte chunk.  Its token indices live in a warp-private table.
        const int lw = warp - kLoadWarp0;
        constexpr int HALF = MAXN / (gemm_loaders(MAXN) / 32);   // rows of each tile this warp copies
        int32_t *tok = tok_s + lw * HALF;
        const uint8_t *bsrc = GATEUP ? reinterpret_cast<const uint8_t *>(a.x16)
                                     : reinterpret_cast<const uint8_t *>(a.h16);
        const size_t brow = static_cast<size_t>(K) * 2;
        const int c = lane & 7;
        int cur = -1, N = 0, nvalid = 0;
        // Copies of k-step j are issued at iteration j and published at
        // iteration j + D, after this thread's cp.async group for j has
        // landed: wait, proxy fence, then one arrival per warp.
        constexpr int D = SB / 2;                  // leaves SB - D stages for the MMAs to overlap with
        for (long j = 0; j < J + D; ++j) {
            if (aborted()) break;
            if (j < J) {
                const int i = static_cast<int>(j / nk), s = static_cast<int>(j % nk);
                if (i != cur) {
                    const TileEntry te = tiles[i];
                    cur = i;
                    nvalid = te.nvalid;
                    N = (nvalid + 15) & ~15;
                    __syncwarp();
                    for (int nl = lane; nl < HALF; nl += 32) {
                        const int n = lw * HALF + nl;
                        int v = 0;
                        if (n < nvalid) {
                            if (GATEUP)
                                v = te.row0 >= 0 ? guard_index(a.perm_src[te.row0 + te.n0 + n], a.T, a.err, MOE_DEVERR_BAD_ROW)
                                                 : te.n0 + n;
                            else
                                v = (te.row0 >= 0 ? te.row0 : a.T * a.k) + te.n0 + n;
                        }
                        tok[nl] = v;
                    }
                    __syncwarp();
                }
                const int sb = static_cast<int>(j % SB);
                int ok = 1;
                if (lane == 0) ok = mbar_wait(emptyB + sb, static_cast<uint32_t>(((j / SB) & 1) ^ 1), a.spin);
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    fail();
                    break;
                }
                const uint32_t bdst = smem_addr(sB + sb * Cfg::B_STAGE);
#pragma unroll 4
                for (int nl = lane >> 3; nl < HALF; nl += 4) {
                    const int n = lw * HALF + nl;
                    if (n < N) {
                        const uint8_t *src =
                            bsrc + static_cast<size_t>(tok[nl]) * brow + static_cast<size_t>(s) * 128 + c * 16;
                        cp_async16(bdst + n * 128 + ((c ^ (n & 7)) << 4), src, n < nvalid ? 16u : 0u);
                    }
                }
            }
            cp_async_commit();                         // one group per iteration (empty while draining)
            if (j >= D) {
                cp_async_wait<D>();                    // this thread's copies of k-step j - D have landed
                fence_proxy_async();                   // ... and are visible to the tensor cores
                __syncwarp();
                if (lane == 0) mbar_arrive(fullB + (j - D) % SB);
            }
        }
        cp_async_wait<0>();
    } else if (warp < kMmaWarp) {
        // -------------------------------------------------------- epilogue
        const int q = warp & 3;                        // TMEM lanes 32q .. 32q+31
        const int m = 32 * q + lane;                   // weight row within a matrix of the tile
        for (int i = 0; i < n_my && !aborted(); ++i) {
            const TileEntry te = tiles[i];
            const int b = i % ACC;
            int ok = 1;
            if (lane == 0) ok = mbar_wait(accF + b, static_cast<uint32_t>((i / ACC) & 1), a.spin);
            if (!__shfl_sync(0xffffffffu, ok, 0)) {
                fail();
                break;
            }
            tc_fence_after();
            const uint32_t base = tmem + (static_cast<uint32_t>(32 * q) << 16) + b * 2 * MAXN;
            const size_t rbase = static_cast<size_t>(te.row0 >= 0 ? te.row0 : a.T * a.k) + te.n0;
            if (GATEUP) {
                for (int c0 = 0; c0 < te.nvalid; c0 += 16) {
                    float gv[16], uv[16];
                    tmem_ld16(base + c0, gv);
                    tmem_ld16(base + MAXN + c0, uv);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int n = c0 + e;
                        if (n >= te.nvalid) break;
                        const float h = __fdividef(gv[e], 1.0f + __expf(-gv[e])) * uv[e];
                        a.h16[(rbase + n) * a.I + te.m0 + m] = __float2half_rn(h);
                    }
                }
            } else {
                for (int mat = 0; mat < 2; ++mat) {
                    const int mrow = te.m0 + kBM * mat + m;
                    if (te.m0 + kBM * mat >= a.H) break;     // ragged last tile: one matrix
                    for (int c0 = 0; c0 < te.nvalid; c0 += 16) {
                        float v[16];
                        tmem_ld16(base + mat * MAXN + c0, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int n = c0 + e;
                            if (n >= te.nvalid) break;
                            float *dst = te.row0 >= 0 ? a.y_perm + (rbase + n) * a.H
                                                      : a.y_shared + (static_cast<size_t>(te.n0) + n) * a.H;
                            if (mrow < a.H) dst[mrow] = v[e];
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(accE + b);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------ MMA issuer
        for (int i = 0; i < n_my && !aborted(); ++i) {
            const TileEntry te = tiles[i];
            const int N = (te.nvalid + 15) & ~15;
            const uint32_t idesc = idesc_f16_f32(kBM, N);
            const int nmat = (GATEUP || te.m0 + kBM < a.H) ? 2 : 1;
            const int b = i % ACC;
            if (lane == 0) {
                if (!mbar_wait(accE + b, static_cast<uint32_t>(((i / ACC) & 1) ^ 1), a.spin)) fail();
                tc_fence_after();
                for (int s = 0; s < nk && !abort_s; ++s) {
                    const long j = static_cast<long>(i) * nk + s;
                    const int sa = static_cast<int>(j % SA), sb = static_cast<int>(j % SB);
                    if (!mbar_spin(fullA + sa, static_cast<uint32_t>((j / SA) & 1), a.spin * 16) ||
                        !mbar_spin(fullB + sb, static_cast<uint32_t>((j / SB) & 1), a.spin * 16)) {
                        fail();
                        break;
                    }
                    tc_fence_after();
                    const uint32_t b_addr = smem_addr(sB + sb * Cfg::B_STAGE);
                    const uint32_t a_addr = smem_addr(sA + sa * Cfg::A_STAGE);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t bdesc = desc_sw128(b_addr + kk * 32);
                        for (int mat = 0; mat < nmat; ++mat)
                            mma_f16(tmem + b * 2 * MAXN + mat * MAXN, desc_sw128(a_addr + mat * kBM * 128 + kk * 32),
                                    bdesc, idesc, (s | kk) != 0);
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
    if (warp == kMmaWarp) {
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

// Upper bound on the tiles of one launch: a group of n tokens has
// ceil(n / maxn) <= n / maxn + 1 token tiles, the shared expert ceil(T / maxn).
static long tiles_bound(int T, int k, int E, int MT, int maxn) {
    const long rows = static_cast<long>(T) * k;
    const long groups = rows < E ? rows : E;
    return (rows / maxn + groups + (T + maxn - 1) / maxn) * static_cast<long>(MT);
}

struct GemmPlan {
    bool large;      // 256-token tiles (else 64)
    int cap_gu;      // tile-list capacity per CTA, gate/up launch
    int cap_dn;      // same, down launch
};

template <int BITS>
static bool make_plan(int T, int k, int H, int I, int E, GemmPlan &p) {
    const long groups = static_cast<long>(T) * k < E ? static_cast<long>(T) * k : E;
    if (groups + 1 > kMaxGroups || H % kBK != 0 || I % kBM != 0) return false;
    // tiles of 256 tokens once experts hold more than ~48 tokens on average
    p.large = static_cast<long>(T) * k > 48L * (groups > 0 ? groups : 1);
    const int maxn = p.large ? 256 : 64;
    const long grid = num_sms();
    const long bg = tiles_bound(T, k, E, I / kBM, maxn), bd = tiles_bound(T, k, E, (H + 2 * kBM - 1) / (2 * kBM), maxn);
    const long cg = (bg + grid - 1) / grid, cd = (bd + grid - 1) / grid;
    if (cg > 65536 || cd > 65536) return false;
    p.cap_gu = static_cast<int>(cg > 0 ? cg : 1);
    p.cap_dn = static_cast<int>(cd > 0 ? cd : 1);
    if (p.large)
        return GemmCfg<BITS, true, 256>::smem(p.cap_gu) <= kSmemLimit &&
               GemmCfg<BITS, false, 256>::smem(p.cap_dn) <= kSmemLimit;
    return GemmCfg<BITS, true, 64>::smem(p.cap_gu) <= kSmemLimit && GemmCfg<BITS, false, 64>::smem(p.cap_dn) <= kSmemLimit;
}

bool gemm_supported(int bits, int T, int k, int H, int I, int E) {
    GemmPlan p;
    return bits == 4 ? make_plan<4>(T, k, H, I, E, p) : make_plan<2>(T, k, H, I, E, p);
}

template <int BITS, bool GATEUP, int MAXN>
static int launch_k_gemm(const GemmArgs &a, int cap, cudaStream_t s) {
    using Cfg = GemmCfg<BITS, GATEUP, MAXN>;
    const size_t smem = Cfg::smem(cap);
    int rc = cuda_status(cudaFuncSetAttribute(k_gemm<BITS, GATEUP, MAXN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(smem)),
                         "gemm smem attribute");
    if (rc) return rc;
    k_gemm<BITS, GATEUP, MAXN><<<num_sms(), gemm_threads(MAXN), smem, s>>>(a, cap);
    count_launches(1);
    return cuda_status(cudaGetLastError(), "gemm launch");
}

template <int BITS>
static int launch_pair(const GemmArgs &a, const GemmPlan &p, cudaStream_t s) {
    int rc = p.large ? launch_k_gemm<BITS, true, 256>(a, p.cap_gu, s) : launch_k_gemm<BITS, true, 64>(a, p.cap_gu, s);
    if (rc) return rc;
    return p.large ? launch_k_gemm<BITS, false, 256>(a, p.cap_dn, s) : launch_k_gemm<BITS, false, 64>(a, p.cap_dn, s);
}

int launch_gemm(int bits, const uint8_t *const *blobs, const int32_t *offsets, const int32_t *active,
                const int32_t *perm_src, const void *x, int x_dtype, int T, int k, int H, int I, int E,
                const uint8_t *shared_blob, float *y_perm, float *y_shared, void *ws, unsigned *err, cudaStream_t s) {
    GemmPlan plan;
    if (!(bits == 4 ? make_plan<4>(T, k, H, I, E, plan) : make_plan<2>(T, k, H, I, E, plan)))
        return cuda_status(cudaErrorInvalidConfiguration, "gemm plan");
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
    const long hook = test_hook_value(MOE_HOOK_GEMM_SPIN);
    a.spin = hook > 0 ? hook : kSpin;
    {
        const long n = static_cast<long>(T) * H;
        long blocks = (n / 4 + 255) / 256;
        if (blocks > num_sms() * 8L) blocks = num_sms() * 8L;
        k_to_half<<<blocks, 256, 0, s>>>(x, x_dtype == MOE_BF16, n, const_cast<__half *>(a.x16));
        count_launches(1);
    }
    return bits == 4 ? launch_pair<4>(a, plan, s) : launch_pair<2>(a, plan, s);
}

}  // namespace moe
