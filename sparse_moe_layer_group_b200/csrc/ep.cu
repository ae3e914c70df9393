// Expert-parallel placement helpers.
//
// "DeepSeek-V3 technical report" walkthrough (2kiu.com), section 4.1: with
// expert parallelism each device holds a subset of the routed experts; tokens
// are dispatched to the devices that hold their experts, processed there and
// combined back (dispatch -> expert MLP -> combine).  Placement used here:
// routed expert e lives on rank e % world as that rank's local expert e / world.
//
// moe_ep_split turns routing indices into (destination rank, local expert id)
// pairs; moe_ep_scatter moves per-pair values into the order of a permutation
// (out[row_of[i]] = values[i]), e.g. the local expert ids into send order.
// The row grouping itself is moe_permute with the destination ranks as groups.
#include "common.cuh"

namespace moe {

__global__ void ep_split_kernel(const int32_t *__restrict__ idx, int64_t n, int E, int world,
                                int32_t *__restrict__ dest, int32_t *__restrict__ local, int32_t *status) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int e = idx[i];
    if (e < 0 || e >= E) {
        set_flag(status, MOE_FLAG_BAD_INDEX);
        dest[i] = -1;
        local[i] = -1;
        return;
    }
    dest[i] = e % world;
    local[i] = e / world;
}

__global__ void ep_scatter_kernel(const int32_t *__restrict__ row_of, const int32_t *__restrict__ vals, int64_t n,
                                  int32_t *__restrict__ out) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int r = row_of[i];
    if (r >= 0) out[r] = vals[i];
}

// One thread per token: the (token, rank) dispatch plan.  Slot k of token t is
// the first of its rank among the token's slots, or a repeat; only first slots
// are dispatched (dest >= 0), each carrying the local expert ids and gates of
// every slot of the token that lives on that rank (-1 / 0 elsewhere).
__global__ void ep_plan_kernel(const int32_t *__restrict__ idx, const float *__restrict__ w, int T, int K, int E,
                               int world, int block, int32_t *__restrict__ dest, int32_t *__restrict__ meta_ids,
                               float *__restrict__ meta_w, int32_t *status) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    const int El = E / world;
    int rk[32], lk[32];
    for (int k = 0; k < K; ++k) {
        const int e = idx[static_cast<int64_t>(t) * K + k];
        if (e < 0 || e >= E) {
            set_flag(status, MOE_FLAG_BAD_INDEX);
            rk[k] = -1;
            lk[k] = -1;
        } else {
            rk[k] = block ? e / El : e % world;
            lk[k] = block ? e % El : e / world;
        }
    }
    for (int k = 0; k < K; ++k) {
        const int64_t i = static_cast<int64_t>(t) * K + k;
        bool first = rk[k] >= 0;
        for (int j = 0; j < k && first; ++j) first = rk[j] != rk[k];
        dest[i] = first ? rk[k] : -1;
        for (int j = 0; j < K; ++j) {
            const bool mine = first && rk[j] == rk[k];
            meta_ids[i * K + j] = mine ? lk[j] : -1;
            meta_w[i * K + j] = mine ? w[static_cast<int64_t>(t) * K + j] : 0.0f;
        }
    }
}

__global__ void ep_scatter_rows_kernel(const int32_t *__restrict__ row_of, const int32_t *__restrict__ vals,
                                       int64_t n, int width, int32_t *__restrict__ out) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n * width) return;
    const int64_t p = i / width;
    const int r = row_of[p];
    if (r >= 0) out[static_cast<int64_t>(r) * width + (i - p * width)] = vals[i];
}

}  // namespace moe

using namespace moe;

MOE_API int moe_ep_split(const int32_t *topk_idx, int64_t n, int32_t E, int32_t world, int32_t *dest_rank,
                         int32_t *local_idx, int32_t *status, void *stream) {
    if (n < 0 || E <= 0 || world <= 0) return MOE_ERR_INVALID_ARG;
    if (n == 0) return MOE_OK;
    if (!topk_idx || !dest_rank || !local_idx) return MOE_ERR_INVALID_ARG;
    if (n > 0x7fffffffLL * 256) return MOE_ERR_UNSUPPORTED;
    const int64_t blocks = (n + 255) / 256;
    ep_split_kernel<<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(topk_idx, n, E, world, dest_rank,
                                                                                 local_idx, status);
    return launch_status();
}

MOE_API int moe_ep_scatter(const int32_t *row_of, const int32_t *values, int64_t n, int32_t *out, void *stream) {
    if (n < 0) return MOE_ERR_INVALID_ARG;
    if (n == 0) return MOE_OK;
    if (!row_of || !values || !out) return MOE_ERR_INVALID_ARG;
    if (n > 0x7fffffffLL * 256) return MOE_ERR_UNSUPPORTED;
    const int64_t blocks = (n + 255) / 256;
    ep_scatter_kernel<<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(row_of, values, n, out);
    return launch_status();
}

MOE_API int moe_ep_plan(const int32_t *topk_idx, const float *topk_w, int64_t T, int32_t K, int32_t E, int32_t world,
                        int32_t placement, int32_t *dest_rank, int32_t *meta_ids, float *meta_w, int32_t *status,
                        void *stream) {
    if (T < 0 || K <= 0 || K > 32 || E <= 0 || world <= 0 || E % world != 0) return MOE_ERR_INVALID_ARG;
    if (placement != MOE_EP_CYCLIC && placement != MOE_EP_BLOCK) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!topk_idx || !topk_w || !dest_rank || !meta_ids || !meta_w) return MOE_ERR_INVALID_ARG;
    if (T > 0x7fffffffLL - 255) return MOE_ERR_UNSUPPORTED;
    const int64_t blocks = (T + 127) / 128;
    ep_plan_kernel<<<static_cast<unsigned>(blocks), 128, 0, as_stream(stream)>>>(
        topk_idx, topk_w, static_cast<int>(T), K, E, world, placement == MOE_EP_BLOCK ? 1 : 0, dest_rank, meta_ids,
        meta_w, status);
    return launch_status();
}

MOE_API int moe_ep_scatter_rows(const int32_t *row_of, const int32_t *values, int64_t n, int32_t width, int32_t *out,
                                void *stream) {
    if (n < 0 || width <= 0) return MOE_ERR_INVALID_ARG;
    if (n == 0) return MOE_OK;
    if (!row_of || !values || !out) return MOE_ERR_INVALID_ARG;
    if (n * width > 0x7fffffffLL * 256) return MOE_ERR_UNSUPPORTED;
    const int64_t blocks = (n * width + 255) / 256;
    ep_scatter_rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(row_of, values, n, width,
                                                                                          out);
    return launch_status();
}
