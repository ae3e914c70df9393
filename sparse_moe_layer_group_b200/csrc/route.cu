// Router: sigmoid affinities and group-limited, bias-ranked top-K with gates.
//
// "DeepSeek-V3 technical report" walkthrough (2kiu.com), section 3.2: the
// affinity is s = sigmoid(h W_router) (sigmoid, not softmax); the top-K ranks
// s + b, where b is the per-expert balancing bias, but the gate values come
// from s alone, normalised over the K selected; section 3.4: a token may reach
// at most M nodes, picked by the sum of the highest affinities of each node's
// experts (here: n_group equal groups, topk_group kept, top-2 sum).  Gating stays
// in fp32 ("From technical report to a runnable config", lpnh.cn, section 3:
// keep_bf16 moe_gating); routed_scaling_factor multiplies the gates.
//
// Kernels:
//   router_split_kernel / router_tc_kernel (router_tc.cu)  fp32-exact logits on
//                         the tensor cores, split over K into partial sums.
//   route_select_kernel   one warp per token: adds the partial logits in split
//                         order, offset, sigmoid; group scores, group pick, top-K,
//                         gates in float64 (exact sum of <= 32 fp32 values).
#include <cfloat>

#include "common.cuh"

namespace moe {

// (value, index) order used for every ranking: larger value first, then the
// lower index.
__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
    return v > bv || (v == bv && i < bi);
}

__device__ __forceinline__ void warp_best(float &v, int &i) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (better(ov, oi, v, i)) { v = ov; i = oi; }
    }
}

constexpr int SEL_WARPS = 8;
constexpr int SEL_MAX_E = 1024;

// One warp per token.  The affinities come either given (s_in [T, E]) or as
// n_split fp32 partial logits [n_split, T, E] from the tensor-core router, which
// are added in split order (a fixed order, so results are deterministic), offset
// and passed through the sigmoid here.  r = s + b is formed where it is used.
__global__ void __launch_bounds__(SEL_WARPS * 32) route_select_kernel(
    const float *__restrict__ s_in, const float *__restrict__ partial, int n_split,
    const float *__restrict__ offset, float *__restrict__ s_out, const float *__restrict__ bias,
    int32_t *__restrict__ topk_idx, float *__restrict__ topk_w, int T, int E, int K, int n_group,
    int topk_group, float rho) {
    extern __shared__ float sh[];   // SEL_WARPS * E affinities
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int t = blockIdx.x * SEL_WARPS + wid;
    if (t >= T) return;
    float *srow = sh + wid * E;
    if (partial) {
        const int64_t plane = static_cast<int64_t>(T) * E;
        const float *base = partial + static_cast<int64_t>(t) * E;
        // eight experts per lane at a time: the eight loads of one split are
        // independent, so a split costs one memory round trip; every logit is
        // still summed in split order
        for (int e0 = 0; e0 < E; e0 += 256) {
            float l[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int e = e0 + lane + 32 * j;
                l[j] = e < E ? base[e] : 0.0f;
            }
#pragma unroll 4
            for (int q = 1; q < n_split; ++q) {
                const float *pq = base + q * plane;
                float v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int e = e0 + lane + 32 * j;
                    v[j] = e < E ? pq[e] : 0.0f;
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) l[j] = __fadd_rn(l[j], v[j]);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int e = e0 + lane + 32 * j;
                if (e < E) {
                    const float lj = offset ? __fadd_rn(l[j], __ldg(offset + e)) : l[j];
                    const float sv = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-lj)));
                    srow[e] = sv;
                    if (s_out) s_out[static_cast<int64_t>(t) * E + e] = sv;
                }
            }
        }
    } else {
        for (int e = lane; e < E; e += 32) srow[e] = s_in[static_cast<int64_t>(t) * E + e];
    }
    __syncwarp();
    const int gs = E / n_group;
    // group scores: lane g scans its group for the two largest values of r
    float gscore = -FLT_MAX;
    const bool gvalid = lane < n_group;
    if (gvalid) {
        float m1 = -FLT_MAX, m2 = -FLT_MAX;
        for (int j = 0; j < gs; ++j) {
            const int e = lane * gs + j;
            const float v = __fadd_rn(srow[e], __ldg(bias + e));
            if (v > m1) { m2 = m1; m1 = v; } else if (v > m2) { m2 = v; }
        }
        gscore = gs == 1 ? m1 : __fadd_rn(m1, m2);
    }
    // keep the topk_group best groups (ties to the lower group)
    uint32_t kept = 0;
    bool taken_g = !gvalid;
    for (int round = 0; round < topk_group; ++round) {
        float v = taken_g ? -INFINITY : gscore;
        int i = taken_g ? 0x7fffffff : lane;
        warp_best(v, i);
        kept |= 1u << i;
        if (lane == i) taken_g = true;
    }
    // top-K over the kept groups' experts
    uint32_t taken = 0;   // bit j: expert lane + 32 j already chosen (E <= 1024)
    float my_s = 0.0f;
    int my_i = -1;
    const int per_lane = (E + 31) / 32;
    for (int k = 0; k < K; ++k) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int j = 0; j < per_lane; ++j) {
            const int e = lane + 32 * j;
            if (e >= E || (taken >> j & 1u) || !(kept >> (e / gs) & 1u)) continue;
            const float v = __fadd_rn(srow[e], __ldg(bias + e));
            if (better(v, e, bv, bi)) { bv = v; bi = e; }
        }
        warp_best(bv, bi);
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == k) { my_i = bi; my_s = srow[bi]; }
    }
    // gates: (rho * s_k) / sum s_j in float64 (the sum of <= 32 fp32 values in (0,1) is exact)
    double sum = lane < K ? static_cast<double>(my_s) : 0.0;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane < K) {
        topk_idx[static_cast<int64_t>(t) * K + lane] = my_i;
        topk_w[static_cast<int64_t>(t) * K + lane] =
            static_cast<float>((static_cast<double>(rho) * static_cast<double>(my_s)) / sum);
    }
}

static int check_route_dims(const moe_dims *d) {
    if (!d) return MOE_ERR_INVALID_ARG;
    if (d->T < 0 || d->H <= 0 || d->E <= 0 || d->K <= 0 || d->n_group <= 0 || d->topk_group <= 0)
        return MOE_ERR_INVALID_ARG;
    if (d->H % 128 != 0 || d->E % d->n_group != 0 || d->topk_group > d->n_group) return MOE_ERR_INVALID_ARG;
    if (static_cast<int64_t>(d->topk_group) * (d->E / d->n_group) < d->K) return MOE_ERR_INVALID_ARG;
    if (d->E > SEL_MAX_E || d->n_group > 32 || d->K > 32) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

static int launch_select(const moe_dims *d, const float *s_in, const float *partial, int n_split,
                         const float *offset, float *s_out, const float *e_bias, int32_t *idx, float *w,
                         cudaStream_t st) {
    const int blocks = (d->T + SEL_WARPS - 1) / SEL_WARPS;
    const size_t smem = static_cast<size_t>(SEL_WARPS) * d->E * sizeof(float);
    route_select_kernel<<<blocks, SEL_WARPS * 32, smem, st>>>(s_in, partial, n_split, offset, s_out, e_bias, idx,
                                                              w, d->T, d->E, d->K, d->n_group, d->topk_group,
                                                              d->routed_scaling_factor);
    return launch_status();
}

int router_splits(int T, int E, int H);
size_t router_tc_ws_bytes(int T, int E, int H);
int launch_router_split(const float *w, int E, int H, void *pieces_out, cudaStream_t st);
int launch_router_tc(const void *x, const void *pieces, int T, int E, int H, void *ws, float **partial_out,
                     int *n_split_out, int32_t *status, cudaStream_t st);

size_t route_workspace_bytes(const moe_dims *d) {
    // three bf16 pieces of W_r and the split-K partial logits
    return router_tc_ws_bytes(d->T, d->E, d->H);
}

}  // namespace moe

using namespace moe;

MOE_API int moe_route(const moe_dims *d, const void *x, const float *w_router, const float *e_bias,
                      const float *router_offset, int32_t *topk_idx, float *topk_w, float *scores,
                      void *ws, size_t ws_bytes, int32_t *status, void *stream) {
    int rc = check_route_dims(d);
    if (rc != MOE_OK) return rc;
    if (d->T == 0) return MOE_OK;
    if (!x || !w_router || !e_bias || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router)) return MOE_ERR_INVALID_ARG;
    if (!ws || ws_bytes < route_workspace_bytes(d) || (reinterpret_cast<uintptr_t>(ws) & 255)) return MOE_ERR_WORKSPACE;
    cudaStream_t st = as_stream(stream);
    // the pieces go to the front of the workspace, the partial sums after them
    rc = launch_router_split(w_router, d->E, d->H, ws, st);
    if (rc != MOE_OK) return rc;
    float *partial = nullptr;
    int n_split = 0;
    rc = launch_router_tc(x, ws, d->T, d->E, d->H, ws, &partial, &n_split, status, st);
    if (rc != MOE_OK) return rc;
    return launch_select(d, nullptr, partial, n_split, router_offset, scores, e_bias, topk_idx, topk_w, st);
}

MOE_API size_t moe_router_pieces_bytes(int32_t E, int32_t H) {
    if (E <= 0 || H <= 0) return 0;
    return static_cast<size_t>(3) * E * H * 2;
}

MOE_API int moe_router_split(const float *w_router, int32_t E, int32_t H, void *w_pieces, void *stream) {
    if (E <= 0 || H <= 0 || H % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (E > SEL_MAX_E) return MOE_ERR_UNSUPPORTED;
    if (!w_router || !w_pieces || !aligned16(w_router) || !aligned16(w_pieces)) return MOE_ERR_INVALID_ARG;
    return launch_router_split(w_router, E, H, w_pieces, as_stream(stream));
}

MOE_API int moe_route_pieces(const moe_dims *d, const void *x, const void *w_pieces, const float *e_bias,
                             const float *router_offset, int32_t *topk_idx, float *topk_w, float *scores,
                             void *ws, size_t ws_bytes, int32_t *status, void *stream) {
    int rc = check_route_dims(d);
    if (rc != MOE_OK) return rc;
    if (d->T == 0) return MOE_OK;
    if (!x || !w_pieces || !e_bias || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_pieces)) return MOE_ERR_INVALID_ARG;
    if (!ws || ws_bytes < route_workspace_bytes(d) || (reinterpret_cast<uintptr_t>(ws) & 255)) return MOE_ERR_WORKSPACE;
    cudaStream_t st = as_stream(stream);
    float *partial = nullptr;
    int n_split = 0;
    rc = launch_router_tc(x, w_pieces, d->T, d->E, d->H, ws, &partial, &n_split, status, st);
    if (rc != MOE_OK) return rc;
    return launch_select(d, nullptr, partial, n_split, router_offset, scores, e_bias, topk_idx, topk_w, st);
}

MOE_API int moe_route_select(const moe_dims *d, const float *scores, const float *e_bias,
                             int32_t *topk_idx, float *topk_w, void *stream) {
    int rc = check_route_dims(d);
    if (rc != MOE_OK) return rc;
    if (d->T == 0) return MOE_OK;
    if (!scores || !e_bias || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    return launch_select(d, scores, nullptr, 0, nullptr, nullptr, e_bias, topk_idx, topk_w, as_stream(stream));
}
