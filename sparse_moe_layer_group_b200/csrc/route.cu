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
//                         order, offset, sigmoid; group scores, group pick, top-K
//                         (warp max/min reductions over order-preserving keys),
//                         gates in float64 (exact sum of <= 32 fp32 values).
#include <cfloat>

#include "common.cuh"

namespace moe {

constexpr int SEL_WARPS = 8;
constexpr int SEL_MAX_E = 1024;

// Order-preserving map of an fp32 value to uint32 (larger value -> larger
// key); NaN maps below every number, so it is never preferred.
__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v);
    if (v != v) return 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Best (largest value, then lowest index) of one candidate per lane, by two
// warp reductions: the largest key, then the lowest index holding it.
__device__ __forceinline__ int warp_best_index(float v, int i) {
    const uint32_t k = order_key(v);
    const uint32_t mx = __reduce_max_sync(0xffffffffu, k);
    return static_cast<int>(__reduce_min_sync(0xffffffffu, k == mx ? static_cast<uint32_t>(i) : 0xffffffffu));
}

// One warp per token; lane l holds experts l + 32 j, j < PER (PER >= ceil(E/32)).
// The affinities come either given (s_in [T, E]) or as n_split fp32 partial
// logits [n_split, T, E] from the tensor-core router, which are added in split
// order (a fixed order, so results are deterministic), offset and passed through
// the sigmoid here.  r = s + b is kept in registers; every ranking orders by
// value, then by the lower index.
template <int PER>
__global__ void __launch_bounds__(SEL_WARPS * 32) route_select_kernel(
    const float *__restrict__ s_in, const float *__restrict__ partial, int n_split,
    const float *__restrict__ offset, float *__restrict__ s_out, const float *__restrict__ bias,
    int32_t *__restrict__ topk_idx, float *__restrict__ topk_w, int T, int E, int K, int n_group,
    int topk_group, float rho) {
    extern __shared__ float sh[];   // SEL_WARPS * 2 * E: affinities s, then r = s + b
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int t = blockIdx.x * SEL_WARPS + wid;
    if (t >= T) return;
    float *srow = sh + wid * 2 * E;
    float *rrow = srow + E;
    float r[PER];
    if (partial) {
        const int64_t plane = static_cast<int64_t>(T) * E;
        const float *base = partial + static_cast<int64_t>(t) * E;
        float l[PER];
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int e = lane + 32 * j;
            l[j] = e < E ? base[e] : 0.0f;
        }
        // four splits' loads in flight at a time; each logit still sums in split order
        int q = 1;
        for (; q + 3 < n_split; q += 4) {
            float v[4][PER];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int j = 0; j < PER; ++j) {
                    const int e = lane + 32 * j;
                    v[u][j] = e < E ? base[(q + u) * plane + e] : 0.0f;
                }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int j = 0; j < PER; ++j) l[j] = __fadd_rn(l[j], v[u][j]);
        }
        for (; q < n_split; ++q) {
#pragma unroll
            for (int j = 0; j < PER; ++j) {
                const int e = lane + 32 * j;
                l[j] = __fadd_rn(l[j], e < E ? base[q * plane + e] : 0.0f);
            }
        }
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int e = lane + 32 * j;
            if (e < E) {
                const float lj = offset ? __fadd_rn(l[j], __ldg(offset + e)) : l[j];
                const float sv = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-lj)));
                srow[e] = sv;
                if (s_out) s_out[static_cast<int64_t>(t) * E + e] = sv;
                r[j] = __fadd_rn(sv, __ldg(bias + e));
                rrow[e] = r[j];
            } else {
                r[j] = -INFINITY;
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int e = lane + 32 * j;
            if (e < E) {
                const float sv = s_in[static_cast<int64_t>(t) * E + e];
                srow[e] = sv;
                r[j] = __fadd_rn(sv, __ldg(bias + e));
                rrow[e] = r[j];
            } else {
                r[j] = -INFINITY;
            }
        }
    }
    __syncwarp();
    const int gs = E / n_group;
    // group scores: lane g takes the two largest r of its group (a repeated
    // maximum counts twice) from shared memory
    float gscore = -FLT_MAX;
    const bool gvalid = lane < n_group;
    if (gvalid) {
        float m1 = -FLT_MAX, m2 = -FLT_MAX;
        const float *gr = rrow + lane * gs;
#pragma unroll 8
        for (int j = 0; j < gs; ++j) {
            const float v = gr[j];
            if (v > m1) { m2 = m1; m1 = v; } else if (v > m2) { m2 = v; }
        }
        gscore = gs == 1 ? m1 : __fadd_rn(m1, m2);
    }
    // keep the topk_group best groups (ties to the lower group): a group's rank
    // is the number of groups ahead of it
    int rank = 0;
    for (int h = 0; h < n_group; ++h) {
        const float o = __shfl_sync(0xffffffffu, gscore, h);
        rank += (o > gscore || (o == gscore && h < lane)) ? 1 : 0;
    }
    const uint32_t kept = __ballot_sync(0xffffffffu, gvalid && rank < topk_group);
    // top-K over the kept groups' experts: each lane keeps its own best
    // candidate; per round the warp's best is taken and only its lane rescans
    uint32_t taken = 0;   // bit j: expert lane + 32 j chosen, or not selectable
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        const int e = lane + 32 * j;
        if (e >= E || !(kept >> (e / gs) & 1u)) taken |= 1u << j;
    }
    auto local_best = [&](float &bv, int &bi) {
        bv = -INFINITY;
        bi = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const float v = r[j];
            const int e = lane + 32 * j;
            if (!(taken >> j & 1u) && (v > bv || (v == bv && e < bi) || bi == 0x7fffffff)) { bv = v; bi = e; }
        }
    };
    float bv;
    int bi;
    local_best(bv, bi);
    float my_s = 0.0f;
    int my_i = -1;
    for (int k = 0; k < K; ++k) {
        const int w = warp_best_index(bv, bi);
        if ((w & 31) == lane) {
            taken |= 1u << (w >> 5);
            local_best(bv, bi);
        }
        if (lane == k) { my_i = w; my_s = srow[w]; }
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
    const size_t smem = static_cast<size_t>(SEL_WARPS) * 2 * d->E * sizeof(float);
    const int per = (d->E + 31) / 32;
    auto go = [&](auto kern) -> int {
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
                cudaSuccess)
            return MOE_ERR_CUDA;
        kern<<<blocks, SEL_WARPS * 32, smem, st>>>(s_in, partial, n_split, offset, s_out, e_bias, idx, w, d->T, d->E,
                                                   d->K, d->n_group, d->topk_group, d->routed_scaling_factor);
        return launch_status();
    };
    if (per <= 1) return go(route_select_kernel<1>);
    if (per <= 2) return go(route_select_kernel<2>);
    if (per <= 4) return go(route_select_kernel<4>);
    if (per <= 8) return go(route_select_kernel<8>);
    if (per <= 16) return go(route_select_kernel<16>);
    return go(route_select_kernel<32>);
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
