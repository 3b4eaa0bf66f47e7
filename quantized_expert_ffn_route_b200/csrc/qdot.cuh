// Packed-code dot products shared by the CUDA-core expert kernels.
//
// Dequantisation without int->float conversions: a byte 0x80|q placed in bits
// 16..23 of 0x3F000000 is the float 1 + q/128, so
//   sum_i (q_i - half) x_i = 128 * sum_i f_i x_i - (128 + half) * sum_i x_i,
// where the per-block activation sums are computed once per token when the
// activations are staged in shared memory.  All arithmetic is fp32.
#pragma once

#include "common.cuh"

namespace moe {

template <int BITS> struct QT;
template <> struct QT<4> {
    static constexpr int EPC = 32;    // elements per 16-byte code chunk
    static constexpr int BPC = 1;     // quant blocks (scales) per chunk
    static constexpr int PPC = 8;     // float4 pieces per chunk
    static constexpr int HALF = 8;
};
template <> struct QT<2> {
    static constexpr int EPC = 64;
    static constexpr int BPC = 2;
    static constexpr int PPC = 16;
    static constexpr int HALF = 2;
};

__device__ __forceinline__ float magic(uint32_t bytes, int b) {
    // bytes hold 0x80|q in every byte; select byte b into bits 16..23 of 0x3F000000
    return __uint_as_float(__byte_perm(bytes, 0x3F000000u, 0x7054u | (static_cast<unsigned>(b) << 8)));
}

__device__ __forceinline__ uint4 ldg_stream(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

template <int BITS>
__device__ __forceinline__ void load_scales(const __half *row_scales, int c, bool valid, float (&d)[QT<BITS>::BPC]) {
    if constexpr (BITS == 4) {
        d[0] = valid ? __half2float(row_scales[c]) : 0.f;
    } else {
        if (valid) {
            const __half2 s2 = *reinterpret_cast<const __half2 *>(row_scales + 2 * c);
            d[0] = __low2float(s2);
            d[1] = __high2float(s2);
        } else {
            d[0] = d[1] = 0.f;
        }
    }
}

// Stages nt activation rows (fp32 or bf16, row_of(t) -> row t) as fp32
// pieces plus the pre-scaled block sums; rows nt..NTS-1 are zero.
template <int BITS, class RowOf>
__device__ void stage_rows_fn(float4 *xs, float *cs, int NTS, int nt, int K, RowOf row_of, int bf16) {
    using Q = QT<BITS>;
    const int nch = K / Q::EPC;
    const int g4n = K / 4;
#pragma unroll 1
    for (int t = 0; t < NTS; ++t) {                 // divisors below are compile-time constants
        const void *row = t < nt ? row_of(t) : nullptr;
        for (int g4 = threadIdx.x; g4 < g4n; g4 += blockDim.x) {
            const int c = g4 / Q::PPC, q = g4 % Q::PPC;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (row)
                v = bf16 ? load4(static_cast<const __nv_bfloat16 *>(row) + 4 * g4)
                         : load4(static_cast<const float *>(row) + 4 * g4);
            xs[(t * Q::PPC + q) * nch + c] = v;
        }
    }
    __syncthreads();
    const int nblk = K / 32;
#pragma unroll 1
    for (int t = 0; t < NTS; ++t)
        for (int b = threadIdx.x; b < nblk; b += blockDim.x) {
            const int c = b / Q::BPC, beta = b % Q::BPC;
            float s = 0.f;
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const float4 v = xs[(t * Q::PPC + 8 * beta + p) * nch + c];
                s += (v.x + v.y) + (v.z + v.w);
            }
            cs[t * nblk + b] = static_cast<float>(128 + Q::HALF) * s;
        }
    __syncthreads();
}


}  // namespace moe

namespace moe {

// ---------------------------------------------------------------------------
// Single-token variant with the activation pieces of one chunk in registers,
// so several weight rows can reuse them: returns, per quant block of the
// chunk, sum_i f_i x_i with f_i = 1 + q_i/128, accumulated with packed fp32
// FMAs (two lanes of a float2 per instruction).
template <int BITS>
__device__ __forceinline__ void chunk_fx(const uint4 &code, const float4 (&xp)[QT<BITS>::PPC],
                                         float (&out)[QT<BITS>::BPC]) {
    const uint32_t words[4] = {code.x, code.y, code.z, code.w};
    // Each packed FMA pairs neighbouring elements (j, j+1) of one code word
    // with the neighbouring x values of one float4, so operands sit in
    // register pairs as loaded.
    if constexpr (BITS == 4) {
        // four independent accumulators (one per code word), so consecutive
        // packed FMAs do not wait on each other
        float2 acc[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const uint32_t L = (words[m] & 0x0F0F0F0Fu) | 0x80808080u;
            const uint32_t Hh = ((words[m] >> 4) & 0x0F0F0F0Fu) | 0x80808080u;
            const float4 a = xp[m], b = xp[4 + m];   // elements 4m..4m+3 (low nibbles), 16+4m.. (high)
            acc[m] = __fmul2_rn(make_float2(magic(L, 0), magic(L, 1)), make_float2(a.x, a.y));
            acc[m] = __ffma2_rn(make_float2(magic(L, 2), magic(L, 3)), make_float2(a.z, a.w), acc[m]);
            acc[m] = __ffma2_rn(make_float2(magic(Hh, 0), magic(Hh, 1)), make_float2(b.x, b.y), acc[m]);
            acc[m] = __ffma2_rn(make_float2(magic(Hh, 2), magic(Hh, 3)), make_float2(b.z, b.w), acc[m]);
        }
        out[0] = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) + ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
    } else {
        float2 acc[2][2] = {{make_float2(0.f, 0.f), make_float2(0.f, 0.f)},
                            {make_float2(0.f, 0.f), make_float2(0.f, 0.f)}};
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            const int beta = wi >> 1, m = wi & 1;
#pragma unroll
            for (int s = 0; s < 4; ++s) {            // crumb level s: elements 8s + 4m + j of block beta
                const uint32_t Ls = ((words[wi] >> (2 * s)) & 0x03030303u) | 0x80808080u;
                const float4 a = xp[8 * beta + 2 * s + m];
                float2 &v = acc[beta][s & 1];
                v = __ffma2_rn(make_float2(magic(Ls, 0), magic(Ls, 1)), make_float2(a.x, a.y), v);
                v = __ffma2_rn(make_float2(magic(Ls, 2), magic(Ls, 3)), make_float2(a.z, a.w), v);
            }
        }
        out[0] = (acc[0][0].x + acc[0][0].y) + (acc[0][1].x + acc[0][1].y);
        out[1] = (acc[1][0].x + acc[1][0].y) + (acc[1][1].x + acc[1][1].y);
    }
}

// chunk_fx for NV weight rows that share one chunk of x: the x pieces are
// read from shared memory (piece q at xs[q * stride]) one code word at a
// time and applied to all NV rows, so only two or four pieces are live.
template <int BITS, int NV>
__device__ __forceinline__ void rows_fx(const uint4 (&code)[NV], const float4 *xs, int stride,
                                        float (&out)[NV][QT<BITS>::BPC]) {
    if constexpr (BITS == 4) {
        float2 acc[NV];
#pragma unroll
        for (int v = 0; v < NV; ++v) acc[v] = make_float2(0.f, 0.f);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 a = xs[m * stride], b = xs[(4 + m) * stride];
#pragma unroll
            for (int v = 0; v < NV; ++v) {
                const uint32_t w = m == 0 ? code[v].x : m == 1 ? code[v].y : m == 2 ? code[v].z : code[v].w;
                const uint32_t L = (w & 0x0F0F0F0Fu) | 0x80808080u;
                const uint32_t Hh = ((w >> 4) & 0x0F0F0F0Fu) | 0x80808080u;
                acc[v] = __ffma2_rn(make_float2(magic(L, 0), magic(L, 1)), make_float2(a.x, a.y), acc[v]);
                acc[v] = __ffma2_rn(make_float2(magic(L, 2), magic(L, 3)), make_float2(a.z, a.w), acc[v]);
                acc[v] = __ffma2_rn(make_float2(magic(Hh, 0), magic(Hh, 1)), make_float2(b.x, b.y), acc[v]);
                acc[v] = __ffma2_rn(make_float2(magic(Hh, 2), magic(Hh, 3)), make_float2(b.z, b.w), acc[v]);
            }
        }
#pragma unroll
        for (int v = 0; v < NV; ++v) out[v][0] = acc[v].x + acc[v].y;
    } else {
        float2 acc[NV][2];
#pragma unroll
        for (int v = 0; v < NV; ++v) acc[v][0] = acc[v][1] = make_float2(0.f, 0.f);
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            const int beta = wi >> 1, m = wi & 1;
            float4 xq[4];                            // crumb level s: elements 8s + 4m + j of block beta
#pragma unroll
            for (int sl = 0; sl < 4; ++sl) xq[sl] = xs[(8 * beta + 2 * sl + m) * stride];
#pragma unroll
            for (int v = 0; v < NV; ++v) {
                const uint32_t w = wi == 0 ? code[v].x : wi == 1 ? code[v].y : wi == 2 ? code[v].z : code[v].w;
#pragma unroll
                for (int sl = 0; sl < 4; ++sl) {
                    const uint32_t Ls = ((w >> (2 * sl)) & 0x03030303u) | 0x80808080u;
                    acc[v][beta] = __ffma2_rn(make_float2(magic(Ls, 0), magic(Ls, 1)), make_float2(xq[sl].x, xq[sl].y),
                                              acc[v][beta]);
                    acc[v][beta] = __ffma2_rn(make_float2(magic(Ls, 2), magic(Ls, 3)), make_float2(xq[sl].z, xq[sl].w),
                                              acc[v][beta]);
                }
            }
        }
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            out[v][0] = acc[v][0].x + acc[v][0].y;
            out[v][1] = acc[v][1].x + acc[v][1].y;
        }
    }
}

// Makes the compiler treat a code chunk as changed here, so the dequantised
// values derived from it are rebuilt per token instead of being hoisted out
// of a token loop (hoisting them would need 32-64 registers per chunk).
__device__ __forceinline__ void opaque(uint4 &c) {
    asm volatile("" : "+r"(c.x), "+r"(c.y), "+r"(c.z), "+r"(c.w));
}

// dot += sum over the chunk's blocks of d_b * (128 * fx_b - cs_b)
template <int BITS>
__device__ __forceinline__ float chunk_finish(const float (&fx)[QT<BITS>::BPC], const float (&d)[QT<BITS>::BPC],
                                              const float (&cs)[QT<BITS>::BPC], float dot) {
#pragma unroll
    for (int b = 0; b < QT<BITS>::BPC; ++b) dot = fmaf(d[b], fmaf(128.f, fx[b], -cs[b]), dot);
    return dot;
}

}  // namespace moe
