// Selection keys and the gate softmax shared by the top-k kernels.
// Order: larger logit first, equal logits by lower expert id, NaN below -inf.
#pragma once

#include "common.cuh"

namespace moe {

// Order-preserving 32-bit key of a float: larger float -> larger key,
// -0 and +0 equal, every NaN -> 0 (below -inf, whose key is 0x007fffff).
__device__ __forceinline__ uint32_t float_key(float v) {
    if (v != v) return 0u;
    if (v == 0.0f) v = 0.0f;
    uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
    if (k == 0u) return __uint_as_float(0x7fc00000u);
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}
// 64-bit selection key: value key, then the larger the lower the id.
__device__ __forceinline__ uint64_t sel_key(float v, int e) {
    return (static_cast<uint64_t>(float_key(v)) << 32) | static_cast<uint32_t>(0xffffffffu - static_cast<uint32_t>(e));
}
__device__ __forceinline__ uint64_t shfl_max64(uint64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        uint64_t w = __shfl_xor_sync(0xffffffffu, v, o);
        v = w > v ? w : v;
    }
    return v;
}

// ------------------------------------------------------------- gate math
// Every lane holds (v_j, id_j) for slot j = lane (< k).  Writes ids and gates.
__device__ __forceinline__ void write_gates(int lane, int k, float my_v, int my_id, int32_t *ids, float *w,
                                            unsigned *err) {
    const float v0 = __shfl_sync(0xffffffffu, my_v, 0);
    const bool bad = lane < k && (my_v != my_v || my_v == __int_as_float(0x7f800000));
    const bool any_bad = __any_sync(0xffffffffu, bad);
    float ex = lane < k ? expf(my_v - v0) : 0.f;
    float s = 0.f;
    for (int j = 0; j < k; ++j) s += __shfl_sync(0xffffffffu, ex, j);   // slot order
    if (lane < k) {
        ids[lane] = my_id;
        w[lane] = any_bad ? __int_as_float(0x7fc00000) : ex / s;
    }
    if (any_bad && lane == 0) report(err, MOE_DEVERR_NONFINITE);
}

}  // namespace moe
