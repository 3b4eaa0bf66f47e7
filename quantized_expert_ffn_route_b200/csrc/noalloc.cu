// Allocation-free variant of the expert FFN (CUDA-core GEMV kernels).
//
// Some callers cannot allocate device memory at the point where they run the
// expert step: engines that must stay inside a device-memory budget fixed at
// start-up, plain C hosts that have no device allocator of their own to hand
// out a workspace, and latency-critical loops where an allocation could
// synchronise the device.  For them, this entry point takes its scratch (the SwiGLU
// intermediate h, fp32) from a fixed array compiled into the library instead
// of a caller-provided workspace.
//
// The array below is a file-scope __device__ object: every GPU that loads the
// library holds it (kNoAllocScratchBytes) until the process exits.  Its name
// is only a host-side stand-in for the symbol; the device address comes from
// cudaGetSymbolAddress, taken once per device with that device current.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr size_t kNoAllocScratchBytes = 8u << 20;   // 8 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

static std::mutex g_noalloc_mu;
static void *g_noalloc_ptr[64];

// Device address of the scratch array on the current device (set up on the
// first call per device); nullptr and an error message on failure.
static void *noalloc_scratch() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        set_error("no current CUDA device");
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) {
            cudaGetLastError();
            set_error("cudaGetSymbolAddress of the scratch array failed: %s", cudaGetErrorString(e));
            return nullptr;
        }
        g_noalloc_ptr[dev] = p;
    }
    return g_noalloc_ptr[dev];
}

}  // namespace moe

using namespace moe;

extern "C" size_t moe_expert_ffn_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }

extern "C" int moe_expert_ffn_noalloc(int bits, const void *const *expert_blobs, const int32_t *expert_offsets,
                                      const int32_t *active, const int32_t *perm_src, const void *x, int x_dtype,
                                      int T, int k, int H, int I, int E, const void *shared_blob, float *y_perm,
                                      float *y_shared, moe_stream_t s) {
    moe::NvtxRange nvtx_range("moe_expert_ffn_noalloc");
    set_error("%s", "");
#define NA_REQUIRE(cond, ...)      \
    do {                           \
        if (!(cond)) {             \
            set_error(__VA_ARGS__); \
            return MOE_EINVAL;     \
        }                          \
    } while (0)
    NA_REQUIRE(bits == 4 || bits == 2, "bits must be 4 or 2 (got %d)", bits);
    NA_REQUIRE(T >= 0, "T must be >= 0 (got %d)", T);
    NA_REQUIRE(E >= 1 && E <= 32768, "E must be in [1, 32768] (got %d)", E);
    NA_REQUIRE(k >= 1 && k <= 32 && k <= E, "k must be in [1, min(E, 32)] (got k=%d, E=%d)", k, E);
    NA_REQUIRE(H >= 128 && H % 128 == 0 && H <= 2048, "H must be a multiple of 128 in [128, 2048] (got %d)", H);
    NA_REQUIRE(I >= 128 && I % 128 == 0 && I <= 2048, "I must be a multiple of 128 in [128, 2048] (got %d)", I);
    NA_REQUIRE(gemv_supported(bits, H, I), "I/32 (4-bit) or I/64 (2-bit) must be 2, 4, 8, 16 or 32 (got I=%d)", I);
    if (T == 0) return MOE_OK;
    NA_REQUIRE(x_dtype == MOE_F32 || x_dtype == MOE_BF16, "x_dtype must be MOE_F32 or MOE_BF16");
    NA_REQUIRE(expert_blobs && expert_offsets && active && perm_src && x && y_perm,
               "expert_blobs/expert_offsets/active/perm_src/x/y_perm must not be NULL");
    NA_REQUIRE(!shared_blob || y_shared, "y_shared is NULL while shared_blob is set");
    NA_REQUIRE(aligned16(x) && aligned16(y_perm) && (!y_shared || aligned16(y_shared)) &&
                   (!shared_blob || aligned16(shared_blob)) && aligned16(expert_blobs),
               "x/y_perm/y_shared/shared_blob/expert_blobs must be 16-byte aligned");
    const size_t need = gemv_ws_bytes(T, k, I);
    NA_REQUIRE(need <= kNoAllocScratchBytes,
               "call needs %zu bytes of scratch, more than the built-in %zu (T*(k+1)*I*4 must fit)", need,
               kNoAllocScratchBytes);
#undef NA_REQUIRE
    void *scratch = noalloc_scratch();
    if (!scratch) return MOE_ECUDA;
    unsigned *err = device_error_word();
    if (!err) return cuda_status(cudaErrorInvalidDevice, "device error word");
    // The intermediate rows are fully written by the gate/up kernel before the
    // down kernel reads them, so nothing in the scratch needs clearing.
    return launch_gemv(bits, reinterpret_cast<const uint8_t *const *>(expert_blobs), expert_offsets, active, perm_src,
                       x, x_dtype, T, k, H, I, E, static_cast<const uint8_t *>(shared_blob), y_perm, y_shared,
                       scratch, err, reinterpret_cast<cudaStream_t>(s));
}
