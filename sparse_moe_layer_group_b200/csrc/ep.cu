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
