// Library-level entry points: status strings, ABI version, workspace query.
#include "common.cuh"

namespace moe {
size_t route_workspace_bytes(const moe_dims *d);
size_t permute_workspace_bytes(const moe_dims *d);
}  // namespace moe

MOE_API const char *moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: bad size, NULL or misaligned pointer";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: valid arguments outside the kernels' limits";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing or smaller than moe_workspace_size()";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA runtime or launch error";
        case MOE_ERR_TOO_LARGE:
            return "MOE_ERR_TOO_LARGE: the problem needs more than the no-allocation call's static scratch";
        default: return "unknown moe_status";
    }
}

MOE_API int moe_abi_version(void) { return 1; }

MOE_API size_t moe_workspace_size(const moe_dims *d) {
    if (!d || d->T < 0 || d->E <= 0) return 0;
    const size_t a = moe::route_workspace_bytes(d), b = moe::permute_workspace_bytes(d);
    return a > b ? a : b;
}
