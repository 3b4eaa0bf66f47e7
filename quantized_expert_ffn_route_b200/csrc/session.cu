// A prepared one-token decode step with host buffers: the host->device copy
// of x, the fused step (route -> gate/up -> down + combine) and the
// device->host copy of y, recorded once into a CUDA graph and replayed by one
// C call per token.  A serving loop then pays one graph launch and one
// synchronisation per token instead of a copy, three kernel launches and a
// copy issued one by one.
#include "common.cuh"
#include "kernels.h"

using namespace moe;

struct moe_decode_session {
    cudaStream_t stream = nullptr;
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
    int device = 0;
};

void moe_decode_session_destroy(moe_decode_session *ds) {
    if (!ds) return;
    if (ds->exec) cudaGraphExecDestroy(ds->exec);
    if (ds->graph) cudaGraphDestroy(ds->graph);
    delete ds;
}

int moe_decode_session_create(int bits, const void *x_host, int x_dtype, const void *w_router, int w_dtype,
                              const float *bias, const void *const *expert_blobs, const void *shared_blob, int H,
                              int I, int E, int k, float *y_host, int32_t *ids_host, void *x_dev, int32_t *ids_dev,
                              float *w_dev, float *y_dev, void *ws, size_t ws_bytes, moe_stream_t s,
                              moe_decode_session **out) {
    moe::NvtxRange nvtx_range("moe_decode_session_create");
    REQUIRE(out, "out is NULL");
    *out = nullptr;
    REQUIRE(x_host && y_host && x_dev && y_dev && ids_dev && w_dev && ws, "buffers must not be NULL");
    REQUIRE(w_router, "the session computes the router logits: w_router must not be NULL");
    REQUIRE(s != nullptr, "the session needs a non-default stream (graph capture)");
    const size_t xb = static_cast<size_t>(H) * (x_dtype == MOE_BF16 ? 2 : 4);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(s);
    // zero-filled workspace, then one eager call: it checks every argument
    // (MOE_EINVAL before anything is recorded) and loads the kernels
    int rc = cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, st), "session workspace");
    if (rc) return rc;
    rc = cuda_status(cudaMemcpyAsync(x_dev, x_host, xb, cudaMemcpyHostToDevice, st), "session x copy");
    if (rc) return rc;
    rc = moe_layer_decode(bits, x_dev, x_dtype, w_router, w_dtype, bias, nullptr, expert_blobs, shared_blob, H, I, E,
                          k, ids_dev, w_dev, nullptr, y_dev, ws, ws_bytes, s);
    if (rc) return rc;
    rc = cuda_status(cudaStreamSynchronize(st), "session warm-up");
    if (rc) return rc;
    auto *ds = new moe_decode_session();
    ds->stream = st;
    cudaGetDevice(&ds->device);
    rc = cuda_status(cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal), "session capture");
    if (!rc) {
        int r1 = cuda_status(cudaMemcpyAsync(x_dev, x_host, xb, cudaMemcpyHostToDevice, st), "session x copy");
        int r2 = r1 ? r1 : moe_layer_decode(bits, x_dev, x_dtype, w_router, w_dtype, bias, nullptr, expert_blobs,
                                            shared_blob, H, I, E, k, ids_dev, w_dev, nullptr, y_dev, ws, ws_bytes, s);
        int r3 = r2 ? r2 : cuda_status(cudaMemcpyAsync(y_host, y_dev, static_cast<size_t>(H) * sizeof(float),
                                                       cudaMemcpyDeviceToHost, st), "session y copy");
        if (!r3 && ids_host)
            r3 = cuda_status(cudaMemcpyAsync(ids_host, ids_dev, static_cast<size_t>(k) * sizeof(int32_t),
                                             cudaMemcpyDeviceToHost, st), "session ids copy");
        const int re = cuda_status(cudaStreamEndCapture(st, &ds->graph), "session capture end");
        rc = r3 ? r3 : re;
    }
    if (!rc) rc = cuda_status(cudaGraphInstantiate(&ds->exec, ds->graph, 0), "session graph instantiate");
    if (!rc) rc = cuda_status(cudaGraphUpload(ds->exec, st), "session graph upload");
    if (rc) {
        moe_decode_session_destroy(ds);
        return rc;
    }
    *out = ds;
    return MOE_OK;
}

int moe_decode_session_run(moe_decode_session *ds) {
    REQUIRE(ds, "session is NULL");
    int rc = cuda_status(cudaGraphLaunch(ds->exec, ds->stream), "session launch");
    count_launches(3);
    if (!rc) rc = cuda_status(cudaStreamSynchronize(ds->stream), "session sync");
    return rc;
}
