// Shared device/host helpers of libmoe (not shared with the oracle).
#pragma once

#include <nvtx3/nvToolsExt.h>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// ---------------------------------------------------------------- host side
void set_error(const char *fmt, ...);
int cuda_status(cudaError_t e, const char *what);   // MOE_OK or MOE_ECUDA (+ message)

unsigned *device_error_word();                       // this device's error word, or nullptr
int num_sms();                                       // SMs of the current device (cached)
void count_launches(int n);                          // adds to the library's launch counter

// Argument check of a C-ABI call: sets the error message, returns MOE_EINVAL.
#define REQUIRE(cond, ...)            \
    do {                              \
        if (!(cond)) {                \
            set_error(__VA_ARGS__);   \
            return MOE_EINVAL;        \
        }                             \
    } while (0)

// Makes a device current for the scope and restores the caller's.
struct DeviceGuard {
    int prev = -1;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) cudaSetDevice(dev);
    }
    ~DeviceGuard() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

// Names the enclosing C-ABI call in profiler timelines (NVTX range; a no-op
// when no tool is attached).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// -------------------------------------------------------------- device side
__device__ __forceinline__ void report(unsigned *err, unsigned bits) {
    if (err) atomicOr(err, bits);
}

// An index read from a caller's buffer (a permutation entry, an active-expert
// count) before it addresses memory: every build keeps it inside [0, n) --
// out-of-range values become 0 -- and a MOE_DEBUG build also sets `bits` in
// the device error word, so that a corrupt buffer is reported instead of
// silently folded onto row 0.
__device__ __forceinline__ int guard_index(int v, int n, unsigned *err, unsigned bits) {
    const bool bad = v < 0 || v >= n;
#ifdef MOE_DEBUG
    if (bad) report(err, bits);
#else
    (void)err;
    (void)bits;
#endif
    return bad ? 0 : v;
}

// The active-expert count active[0], kept inside [0, cap]; MOE_DEBUG builds
// report a count outside it.
__device__ __forceinline__ int guard_count(int v, int cap, unsigned *err) {
#ifdef MOE_DEBUG
    if (v < 0 || v > cap) report(err, MOE_DEVERR_BAD_ROW);
#else
    (void)err;
#endif
    return min(max(v, 0), cap);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

// Four consecutive activations as floats (16-byte aligned f32 or 8-byte aligned bf16).
__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    uint2 u = *reinterpret_cast<const uint2 *>(p);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                       __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Byte offsets inside an expert blob (codes Wg, Wu, Wd, then fp16 scales).
struct BlobView {
    const uint8_t *cg, *cu, *cd;
    const __half *sg, *su, *sd;
};

__device__ __forceinline__ BlobView blob_view(const uint8_t *b, int bits, int H, int I) {
    size_t cb = static_cast<size_t>(I) * H * bits / 8;      // code bytes per matrix
    size_t sb = static_cast<size_t>(I) * H / 32;            // scales per matrix
    BlobView v;
    v.cg = b;
    v.cu = b + cb;
    v.cd = b + 2 * cb;
    v.sg = reinterpret_cast<const __half *>(b + 3 * cb);
    v.su = v.sg + sb;
    v.sd = v.su + sb;
    return v;
}

inline size_t blob_bytes_host(int bits, int H, int I) {
    return 3 * static_cast<size_t>(I) * H * bits / 8 + 3 * static_cast<size_t>(I) * H / 32 * 2;
}

}  // namespace moe
