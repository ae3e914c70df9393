// The whole layer forward behind one C call, and a host-data runner that
// overlaps the uploads and downloads of consecutive batches with the forward.
//
// The forward chains the library's own entry points in the order of the
// "DeepSeek-V3 technical report" walkthrough (2kiu.com), sections 3.2 and 4.1
// (route -> dispatch -> expert MLP -> combine) with the FP8 steps of section
// 4.3; the shared expert is one more group of the two grouped GEMMs.  All
// launches go to the caller's stream; nothing here allocates device memory.
#include "common.cuh"

using namespace moe;

MOE_API int moe_layer_forward(const moe_layer *L, const void *x, void *out, void *stream) {
    if (!L || !x || !out) return MOE_ERR_INVALID_ARG;
    const moe_dims *d = &L->dims;
    if (d->T < 0 || d->E <= 0 || d->K <= 0 || d->H <= 0 || d->I <= 0) return MOE_ERR_INVALID_ARG;
    if (d->T == 0) return MOE_OK;
    const int64_t T = d->T, H = d->H, K = d->K, I = d->I, E = d->E;
    const int64_t TK = T * K, M = TK + T;
    uint8_t *xq = L->aq + TK * H;             // the quantised tokens: the last T rows of A
    float *xs = L->as + TK * (H / 128);
    int rc = moe_route_pieces(d, x, L->w_pieces, L->e_bias, L->router_offset, L->topk_idx, L->topk_w, L->scores,
                              L->ws, L->ws_bytes, L->status, stream);
    if (rc != MOE_OK) return rc;
    if ((rc = fp8_quant_1x128(x, T, H, xq, xs, L->status, stream)) != MOE_OK) return rc;
    rc = moe_permute(d, L->topk_idx, xq, xs, L->load, L->offsets, L->tok_of, L->row_of, L->aq, L->as, L->ws,
                     L->ws_bytes, L->status, stream);
    if (rc != MOE_OK) return rc;
    rc = fp8_grouped_gemm_blockscaled(static_cast<int32_t>(E + 1), L->offsets, M, 2 * I, H, L->aq, L->as, L->w13,
                                      L->s13, MOE_EPI_SWIGLU_REQUANT, L->actq, L->acts, L->status, stream);
    if (rc != MOE_OK) return rc;
    rc = fp8_grouped_gemm_blockscaled(static_cast<int32_t>(E + 1), L->offsets, M, H, I, L->actq, L->acts, L->w2,
                                      L->s2, MOE_EPI_BF16, L->yperm, nullptr, L->status, stream);
    if (rc != MOE_OK) return rc;
    const void *ysh = static_cast<const uint8_t *>(L->yperm) + TK * H * 2;
    rc = moe_combine(d, L->yperm, L->row_of, L->topk_w, ysh, out, nullptr, stream);
    if (rc != MOE_OK) return rc;
    if (L->bias_out) rc = moe_bias_update(static_cast<int32_t>(E), T, static_cast<int32_t>(K), L->gamma, L->load,
                                          L->bias_out, stream);
    return rc;
}

MOE_API int moe_layer_run_host(const moe_layer *L, const void *const *x_host, void *const *out_host, int32_t n,
                               void *const *x_dev, void *const *out_dev, void *stream) {
    if (!L || n < 0) return MOE_ERR_INVALID_ARG;
    if (n == 0 || L->dims.T == 0) return MOE_OK;
    if (!x_host || !out_host || !x_dev || !out_dev || !x_dev[0] || !x_dev[1] || !out_dev[0] || !out_dev[1])
        return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i)
        if (!x_host[i] || !out_host[i]) return MOE_ERR_INVALID_ARG;
    const size_t bytes = static_cast<size_t>(L->dims.T) * L->dims.H * 2;
    cudaStream_t st = as_stream(stream), up = nullptr, down = nullptr;
    cudaEvent_t in_done[2] = {}, fwd_done[2] = {}, out_done[2] = {}, start = nullptr;
    int rc = MOE_OK;
    auto fail = [&](int code) { rc = code; };
    if (cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&down, cudaStreamNonBlocking) != cudaSuccess)
        fail(MOE_ERR_CUDA);
    // the copies start after the work already on `stream` (e.g. an earlier call
    // whose forwards still read x_dev or write out_dev)
    if (rc == MOE_OK && (cudaEventCreateWithFlags(&start, cudaEventDisableTiming) != cudaSuccess ||
                         cudaEventRecord(start, st) != cudaSuccess || cudaStreamWaitEvent(up, start, 0) != cudaSuccess ||
                         cudaStreamWaitEvent(down, start, 0) != cudaSuccess))
        fail(MOE_ERR_CUDA);
    for (int b = 0; b < 2 && rc == MOE_OK; ++b)
        if (cudaEventCreateWithFlags(&in_done[b], cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&fwd_done[b], cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&out_done[b], cudaEventDisableTiming) != cudaSuccess)
            fail(MOE_ERR_CUDA);
    // batch i uses buffer pair b = i % 2: its upload waits for the forward that
    // last read x_dev[b] (batch i - 2), its forward for its upload and for the
    // download that last read out_dev[b] (batch i - 2)
    for (int i = 0; i < n && rc == MOE_OK; ++i) {
        const int b = i & 1;
        if (i >= 2 && cudaStreamWaitEvent(up, fwd_done[b], 0) != cudaSuccess) { fail(MOE_ERR_CUDA); break; }
        if (cudaMemcpyAsync(x_dev[b], x_host[i], bytes, cudaMemcpyHostToDevice, up) != cudaSuccess ||
            cudaEventRecord(in_done[b], up) != cudaSuccess || cudaStreamWaitEvent(st, in_done[b], 0) != cudaSuccess) {
            fail(MOE_ERR_CUDA);
            break;
        }
        if (i >= 2 && cudaStreamWaitEvent(st, out_done[b], 0) != cudaSuccess) { fail(MOE_ERR_CUDA); break; }
        const int r = moe_layer_forward(L, x_dev[b], out_dev[b], st);
        if (r != MOE_OK) { fail(r); break; }
        if (cudaEventRecord(fwd_done[b], st) != cudaSuccess || cudaStreamWaitEvent(down, fwd_done[b], 0) != cudaSuccess ||
            cudaMemcpyAsync(out_host[i], out_dev[b], bytes, cudaMemcpyDeviceToHost, down) != cudaSuccess ||
            cudaEventRecord(out_done[b], down) != cudaSuccess) {
            fail(MOE_ERR_CUDA);
            break;
        }
    }
    // the caller's stream ends after the last downloads
    if (rc == MOE_OK) {
        for (int b = 0; b < 2 && b < n; ++b)
            if (cudaStreamWaitEvent(st, out_done[b], 0) != cudaSuccess) fail(MOE_ERR_CUDA);
    } else if (up && down) {
        // an enqueue failed: let the streams' work finish before they go away
        cudaStreamSynchronize(up);
        cudaStreamSynchronize(down);
    }
    // released once their work completes
    if (start) cudaEventDestroy(start);
    for (int b = 0; b < 2; ++b) {
        if (in_done[b]) cudaEventDestroy(in_done[b]);
        if (fwd_done[b]) cudaEventDestroy(fwd_done[b]);
        if (out_done[b]) cudaEventDestroy(out_done[b]);
    }
    if (up) cudaStreamDestroy(up);
    if (down) cudaStreamDestroy(down);
    return rc;
}
