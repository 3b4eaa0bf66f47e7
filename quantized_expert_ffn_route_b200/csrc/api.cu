// C ABI of libmoe: argument validation, workspace sizing and dispatch.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "common.cuh"
#include "kernels.h"

__device__ unsigned g_moe_device_error;

namespace moe {

static thread_local std::string t_err;

void set_error(const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    t_err = buf;
}

int cuda_status(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return MOE_OK;
    set_error("%s: %s", what, cudaGetErrorString(e));
    (void)cudaGetLastError();   // a non-sticky error is reported here, not to the caller's next CUDA call
    return MOE_ECUDA;
}

static std::mutex g_dev_mu;
static unsigned *g_err_ptr[64];
static int g_sms[64];

unsigned *device_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!g_err_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_moe_device_error) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_err_ptr[dev] = static_cast<unsigned *>(p);
    }
    return g_err_ptr[dev];
}

int num_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!g_sms[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        g_sms[dev] = n;
    }
    return g_sms[dev];
}

static std::atomic<long long> g_hooks[5];
long long test_hook_value(int which) {
    return which >= 1 && which <= 4 ? g_hooks[which].load(std::memory_order_relaxed) : 0;
}

static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

static bool check_dtype(int dt) { return dt == MOE_F32 || dt == MOE_BF16; }

}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_last_error(void) { return t_err.c_str(); }

int moe_version(void) { return 100; }

int moe_build_flags(void) {
#ifdef MOE_DEBUG
    return MOE_BUILD_DEBUG;
#else
    return 0;
#endif
}

uint64_t moe_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

int moe_device_error(uint32_t *bits_out, int clear, moe_stream_t s) {
    t_err.clear();
    REQUIRE(bits_out != nullptr, "bits_out is NULL");
    unsigned *p = device_error_word();
    if (!p) return cuda_status(cudaErrorInvalidDevice, "device error word");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(s);
    int rc = cuda_status(cudaStreamSynchronize(st), "moe_device_error sync");
    if (rc) return rc;
    unsigned v = 0;
    rc = cuda_status(cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost), "moe_device_error read");
    if (rc) return rc;
    if (clear && v) {
        rc = cuda_status(cudaMemset(p, 0, sizeof v), "moe_device_error clear");
        if (rc) return rc;
    }
    *bits_out = v;
    if (v) {
        set_error("device error word 0x%x", v);
        return MOE_EDEVICE;
    }
    return MOE_OK;
}

int moe_test_hook(int which, int64_t value) {
    t_err.clear();
    REQUIRE(which >= 1 && which <= 4, "unknown test hook %d", which);
    REQUIRE(value >= 0, "test hook value must be >= 0");
    g_hooks[which].store(value, std::memory_order_relaxed);
    return MOE_OK;
}

size_t moe_expert_blob_bytes(int bits, int H, int I) {
    if ((bits != 2 && bits != 4) || H <= 0 || I <= 0 || H % 32 || I % 32) return 0;
    return blob_bytes_host(bits, H, I);
}

// ------------------------------------------------------------------ route
size_t moe_route_ws_size(int T, int E, int k) {
    if (T <= 0 || E <= 0) return 0;
    if (E <= 1024) return static_cast<size_t>(T) * E * sizeof(float);
    k = k < 1 ? 1 : (k > 32 ? 32 : k);
    return topk_chunk_ws_offset(T, E) + topk_chunk_ws_bytes(T, E, k);   // logits, then the chunk candidates
}

int moe_route_topk(const void *x, int x_dtype, const void *w_router, int w_dtype, const float *logits_in,
                   const float *bias, int T, int H, int E, int k, int32_t *topk_ids, float *topk_w,
                   float *logits_out, void *ws, size_t ws_bytes, moe_stream_t s) {
    moe::NvtxRange nvtx_range("moe_route_topk");
    t_err.clear();
    REQUIRE(T >= 0, "T must be >= 0 (got %d)", T);
    REQUIRE(E >= 1 && E <= 32768, "E must be in [1, 32768] (got %d)", E);
    REQUIRE(k >= 1 && k <= 32 && k <= E, "k must be in [1, min(E, 32)] (got k=%d, E=%d)", k, E);
    if (T == 0) return MOE_OK;
    REQUIRE(topk_ids && topk_w, "topk_ids/topk_w are NULL");
    REQUIRE(aligned16(topk_ids) && aligned16(topk_w), "topk_ids/topk_w must be 16-byte aligned");
    REQUIRE(!logits_out || aligned16(logits_out), "logits_out must be 16-byte aligned");
    if (w_router) {
        REQUIRE(x != nullptr, "x is NULL");
        REQUIRE(check_dtype(x_dtype) && check_dtype(w_dtype), "x_dtype/w_dtype must be MOE_F32 or MOE_BF16");
        REQUIRE(H >= 8 && H % 8 == 0, "H must be a positive multiple of 8 (got %d)", H);
        REQUIRE(aligned16(x) && aligned16(w_router), "x/w_router must be 16-byte aligned");
        REQUIRE(!bias || aligned16(bias), "bias must be 16-byte aligned");
        REQUIRE(logits_out || (ws && ws_bytes >= moe_route_ws_size(T, E, k) && aligned16(ws)),
                "workspace too small: need %zu bytes", moe_route_ws_size(T, E, k));
    } else {
        REQUIRE(logits_in != nullptr, "w_router and logits_in are both NULL");
        REQUIRE(aligned16(logits_in), "logits_in must be 16-byte aligned");
    }
    REQUIRE(E <= 1024 || (ws && ws_bytes >= moe_route_ws_size(T, E, k) && aligned16(ws)),
            "E > 1024 needs the workspace (the chunked top-k keeps its candidates there): need %zu bytes",
            moe_route_ws_size(T, E, k));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(s);
    unsigned *err = device_error_word();
    if (!err) return cuda_status(cudaErrorInvalidDevice, "device error word");
    const float *logits = nullptr;
    if (w_router) {
        float *out = logits_out ? logits_out : static_cast<float *>(ws);
        if (router_mma_supported(x_dtype, w_dtype, T, H)) {
            int rc = launch_router_mma(x, w_router, bias, T, H, E, out, err, st);
            if (rc) return rc;
        } else {
            launch_router_logits(x, x_dtype, w_router, w_dtype, bias, T, H, E, out, st);
        }
        logits = out;
    } else {
        logits = logits_in;
        if (logits_out && logits_out != logits_in) {
            int rc = cuda_status(cudaMemcpyAsync(logits_out, logits_in, static_cast<size_t>(T) * E * sizeof(float),
                                                 cudaMemcpyDeviceToDevice, st),
                                 "logits copy");
            if (rc) return rc;
        }
    }
    launch_topk(logits, T, E, k, topk_ids, topk_w, err,
                E > 1024 ? static_cast<uint8_t *>(ws) + topk_chunk_ws_offset(T, E) : nullptr, st);
    return cuda_status(cudaGetLastError(), "route launch");
}

// ---------------------------------------------------------------- permute
size_t moe_permute_ws_size(int T, int k, int E) {
    if (T <= 0 || k <= 0 || E <= 0) return 0;
    return permute_ws_bytes(T, k, E);
}

int moe_permute(const int32_t *topk_ids, int T, int k, int E, int32_t *expert_offsets, int32_t *perm_src,
                int32_t *perm_dst, int32_t *active, void *ws, size_t ws_bytes, moe_stream_t s) {
    moe::NvtxRange nvtx_range("moe_permute");
    t_err.clear();
    REQUIRE(T >= 0, "T must be >= 0 (got %d)", T);
    REQUIRE(E >= 1 && E <= 32768, "E must be in [1, 32768] (got %d)", E);
    REQUIRE(k >= 1 && k <= 32 && k <= E, "k must be in [1, min(E, 32)] (got k=%d, E=%d)", k, E);
    REQUIRE(static_cast<long>(T) * k <= (1L << 30), "T*k too large");
    REQUIRE(expert_offsets != nullptr, "expert_offsets is NULL");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(s);
    if (T == 0) {
        int rc = cuda_status(cudaMemsetAsync(expert_offsets, 0, (E + 1) * sizeof(int32_t), st), "offsets memset");
        if (!rc && active) rc = cuda_status(cudaMemsetAsync(active, 0, sizeof(int32_t), st), "active memset");
        return rc;
    }
    REQUIRE(topk_ids && perm_src && perm_dst, "topk_ids/perm_src/perm_dst are NULL");
    REQUIRE(aligned16(topk_ids) && aligned16(expert_offsets) && aligned16(perm_src) && aligned16(perm_dst) &&
                (!active || aligned16(active)),
            "permute buffers must be 16-byte aligned");
    const size_t need = permute_ws_bytes(T, k, E);
    REQUIRE(need == 0 || (ws && ws_bytes >= need && aligned16(ws)), "workspace too small: need %zu bytes", need);
    unsigned *err = device_error_word();
    if (!err) return cuda_status(cudaErrorInvalidDevice, "device error word");
    return launch_permute(topk_ids, T, k, E, expert_offsets, perm_src, perm_dst, active, ws, err, st);
}

// ------------------------------------------------------------- expert FFN
static int resolve_mode(int mode, int T, int bits, int H, int I) {
    if (mode == MOE_MODE_AUTO) return T <= 16 && gemv_supported(bits, H, I) ? MOE_MODE_GEMV : MOE_MODE_GEMM;
    return mode;
}

size_t moe_expert_ffn_ws_size(int bits, int T, int k, int H, int I, int E, int mode) {
    if ((bits != 2 && bits != 4) || T <= 0 || k <= 0 || H <= 0 || I <= 0 || E <= 0) return 0;
    mode = resolve_mode(mode, T, bits, H, I);
    if (mode == MOE_MODE_GEMM) return gemm_ws_bytes(bits, T, k, H, I, E);
    return gemv_ws_bytes(T, k, I);
}

static int expert_ffn(int bits, const void *const *expert_blobs, const int32_t *expert_offsets,
                      const int32_t *active, const int32_t *perm_src, const void *x, int x_dtype, int T, int k, int H,
                      int I, int E, const void *shared_blob, float *y_perm, float *y_shared, int mode, void *ws,
                      size_t ws_bytes, moe_stream_t s) {
    moe::NvtxRange nvtx_range("moe_expert_ffn");
    t_err.clear();
    REQUIRE(T >= 0, "T must be >= 0 (got %d)", T);
    REQUIRE(E >= 1 && E <= 32768, "E must be in [1, 32768] (got %d)", E);
    REQUIRE(k >= 1 && k <= 32 && k <= E, "k must be in [1, min(E, 32)] (got k=%d, E=%d)", k, E);
    REQUIRE(H >= 128 && H % 128 == 0 && H <= 8192, "H must be a multiple of 128 in [128, 8192] (got %d)", H);
    REQUIRE(I >= 128 && I % 128 == 0 && I <= 4096, "I must be a multiple of 128 in [128, 4096] (got %d)", I);
    REQUIRE(mode == MOE_MODE_AUTO || mode == MOE_MODE_GEMV || mode == MOE_MODE_GEMM, "bad mode %d", mode);
    if (T == 0) return MOE_OK;
    REQUIRE(check_dtype(x_dtype), "x_dtype must be MOE_F32 or MOE_BF16");
    REQUIRE(expert_blobs && expert_offsets && active && perm_src && x && y_perm,
            "expert_blobs/expert_offsets/active/perm_src/x/y_perm must not be NULL");
    REQUIRE(!shared_blob || y_shared, "y_shared is NULL while shared_blob is set");
    REQUIRE(aligned16(x) && aligned16(y_perm) && (!y_shared || aligned16(y_shared)) &&
                (!shared_blob || aligned16(shared_blob)) && aligned16(expert_blobs),
            "x/y_perm/y_shared/shared_blob/expert_blobs must be 16-byte aligned");
    mode = resolve_mode(mode, T, bits, H, I);
    if (mode == MOE_MODE_GEMV) {
        REQUIRE(gemv_supported(bits, H, I),
                "GEMV mode needs H <= 2048 and I/32 (4-bit) or I/64 (2-bit) in {2, 4, 8, 16, 32} (got H=%d, I=%d)",
                H, I);
    } else {
        REQUIRE(gemm_supported(bits, T, k, H, I, E), "GEMM mode supports at most 4095 active experts (min(E, T*k))");
    }
    const size_t need = moe_expert_ffn_ws_size(bits, T, k, H, I, E, mode);
    REQUIRE(ws && ws_bytes >= need && aligned16(ws), "workspace too small: need %zu bytes", need);
    unsigned *err = device_error_word();
    if (!err) return cuda_status(cudaErrorInvalidDevice, "device error word");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(s);
    auto blobs = reinterpret_cast<const uint8_t *const *>(expert_blobs);
    auto sh = static_cast<const uint8_t *>(shared_blob);
    if (mode == MOE_MODE_GEMM)
        return launch_gemm(bits, blobs, expert_offsets, active, perm_src, x, x_dtype, T, k, H, I, E, sh, y_perm,
                           y_shared, ws, err, st);
    return launch_gemv(bits, blobs, expert_offsets, active, perm_src, x, x_dtype, T, k, H, I, E, sh, y_perm, y_shared,
                       ws, err, st);
}

int moe_expert_ffn_q4(const void *const *expert_blobs, const int32_t *expert_offsets, const int32_t *active,
                      const int32_t *perm_src, const void *x, int x_dtype, int T, int k, int H, int I, int E,
                      const void *shared_blob, float *y_perm, float *y_shared, int mode, void *ws, size_t ws_bytes,
                      moe_stream_t s) {
    return expert_ffn(4, expert_blobs, expert_offsets, active, perm_src, x, x_dtype, T, k, H, I, E, shared_blob,
                      y_perm, y_shared, mode, ws, ws_bytes, s);
}

int moe_expert_ffn_q2(const void *const *expert_blobs, const int32_t *expert_offsets, const int32_t *active,
                      const int32_t *perm_src, const void *x, int x_dtype, int T, int k, int H, int I, int E,
                      const void *shared_blob, float *y_perm, float *y_shared, int mode, void *ws, size_t ws_bytes,
                      moe_stream_t s) {
    return expert_ffn(2, expert_blobs, expert_offsets, active, perm_src, x, x_dtype, T, k, H, I, E, shared_blob,
                      y_perm, y_shared, mode, ws, ws_bytes, s);
}

// ------------------------------------------------------- fused decode step
size_t moe_layer_decode_ws_size(int E, int k, int I) {
    if (E <= 0 || k <= 0 || I <= 0) return 0;
    return decode_ws_bytes(E, k, I);
}

int moe_layer_decode(int bits, const void *x, int x_dtype, const void *w_router, int w_dtype, const float *bias,
                     const float *logits_in, const void *const *expert_blobs, const void *shared_blob, int H, int I,
                     int E, int k, int32_t *topk_ids, float *topk_w, float *logits_out, float *y, void *ws,
                     size_t ws_bytes, moe_stream_t s) {
    moe::NvtxRange nvtx_range("moe_layer_decode");
    t_err.clear();
    REQUIRE(bits == 4 || bits == 2, "bits must be 4 or 2 (got %d)", bits);
    REQUIRE(E >= 1 && k >= 1 && k <= E, "need 1 <= k <= E (got k=%d, E=%d)", k, E);
    REQUIRE(H >= 128 && H % 128 == 0 && I >= 128 && I % 128 == 0, "H and I must be multiples of 128");
    REQUIRE(decode_supported(bits, H, I, E, k),
            "fused decode supports E <= 1024, k <= 32, H, I <= 2048, I %% 256 == 0 (got H=%d I=%d E=%d k=%d)", H, I,
            E, k);
    REQUIRE(check_dtype(x_dtype), "x_dtype must be MOE_F32 or MOE_BF16");
    REQUIRE(x && expert_blobs && topk_ids && topk_w && y, "x/expert_blobs/topk_ids/topk_w/y must not be NULL");
    REQUIRE(w_router || logits_in, "w_router and logits_in are both NULL");
    REQUIRE(!w_router || check_dtype(w_dtype), "w_dtype must be MOE_F32 or MOE_BF16");
    REQUIRE(aligned16(x) && aligned16(y) && aligned16(expert_blobs) && (!w_router || aligned16(w_router)) &&
                (!logits_in || aligned16(logits_in)) && (!logits_out || aligned16(logits_out)) &&
                (!shared_blob || aligned16(shared_blob)),
            "x/y/expert_blobs/w_router/logits/shared_blob must be 16-byte aligned");
    REQUIRE(ws && ws_bytes >= decode_ws_bytes(E, k, I) && aligned16(ws), "workspace too small: need %zu bytes",
            decode_ws_bytes(E, k, I));
    unsigned *err = device_error_word();
    if (!err) return cuda_status(cudaErrorInvalidDevice, "device error word");
    return launch_decode(bits, x, x_dtype, w_router, w_dtype, bias, logits_in,
                         reinterpret_cast<const uint8_t *const *>(expert_blobs),
                         static_cast<const uint8_t *>(shared_blob), H, I, E, k, topk_ids, topk_w, logits_out, y, ws,
                         err, reinterpret_cast<cudaStream_t>(s));
}

// ---------------------------------------------------------------- combine
int moe_combine(const float *y_perm, const int32_t *perm_dst, const float *topk_w, const float *y_shared, int T, int k,
                int H, float *y, moe_stream_t s) {
    moe::NvtxRange nvtx_range("moe_combine");
    t_err.clear();
    REQUIRE(T >= 0, "T must be >= 0 (got %d)", T);
    REQUIRE(k >= 1 && k <= 32, "k must be in [1, 32] (got %d)", k);
    REQUIRE(H >= 4 && H % 4 == 0, "H must be a positive multiple of 4 (got %d)", H);
    if (T == 0) return MOE_OK;
    REQUIRE(y_perm && perm_dst && topk_w && y, "y_perm/perm_dst/topk_w/y must not be NULL");
    REQUIRE(aligned16(y_perm) && aligned16(y) && (!y_shared || aligned16(y_shared)),
            "y_perm/y/y_shared must be 16-byte aligned");
    unsigned *err = device_error_word();
    if (!err) return cuda_status(cudaErrorInvalidDevice, "device error word");
    return launch_combine(y_perm, perm_dst, topk_w, y_shared, T, k, H, y, err, reinterpret_cast<cudaStream_t>(s));
}

}  // extern "C"
