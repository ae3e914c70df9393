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
//   router_logits_kernel  SIMT fp32 GEMM x[T,H] (bf16) . W_r[E,H]^T, epilogue
//                         adds the optional offset and applies the sigmoid.
//   route_select_kernel   one warp per token: group scores, group pick, top-K,
//                         gates in float64 (exact sum of <= 32 fp32 values).
#include <cfloat>

#include "common.cuh"

namespace moe {

namespace rt {
constexpr int BT = 64;      // tokens per CTA tile
constexpr int BE = 64;      // experts per CTA tile
constexpr int BK = 32;      // H chunk
constexpr int THREADS = 256;
}  // namespace rt

// Each thread owns a 4 (tokens) x 4 (experts) block of the 64x64 tile.
__global__ void __launch_bounds__(rt::THREADS) router_logits_kernel(
    const __nv_bfloat16 *__restrict__ x, const float *__restrict__ w, const float *__restrict__ offset,
    float *__restrict__ s_out, int T, int H, int E) {
    __shared__ float xs[rt::BK][rt::BT + 4];
    __shared__ float ws[rt::BK][rt::BE + 4];
    const int tid = threadIdx.x;
    const int t0 = blockIdx.x * rt::BT, e0 = blockIdx.y * rt::BE;
    const int tr = tid / 16, tc = tid % 16;     // 16 x 16 threads
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

    // load mapping: x tile 64 tokens x 32 h = 256 x (8 bf16); w tile 64 x 32 fp32 = 256 x 8 fp32
    const int lrow = tid / 4, lcol = (tid % 4) * 8;
    for (int k0 = 0; k0 < H; k0 += rt::BK) {
        {
            const int t = t0 + lrow;
            float v[8];
            if (t < T) {
                const uint4 u = __ldg(reinterpret_cast<const uint4 *>(x + static_cast<int64_t>(t) * H + k0 + lcol));
                v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
                v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = 0.0f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) xs[lcol + i][lrow] = v[i];
        }
        {
            const int e = e0 + lrow;
            float4 a = make_float4(0, 0, 0, 0), b = make_float4(0, 0, 0, 0);
            if (e < E) {
                const float4 *p = reinterpret_cast<const float4 *>(w + static_cast<int64_t>(e) * H + k0 + lcol);
                a = __ldg(p);
                b = __ldg(p + 1);
            }
            ws[lcol + 0][lrow] = a.x; ws[lcol + 1][lrow] = a.y; ws[lcol + 2][lrow] = a.z; ws[lcol + 3][lrow] = a.w;
            ws[lcol + 4][lrow] = b.x; ws[lcol + 5][lrow] = b.y; ws[lcol + 6][lrow] = b.z; ws[lcol + 7][lrow] = b.w;
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < rt::BK; ++k) {
            float xa[4], wb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) xa[i] = xs[k][tr + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) wb[j] = ws[k][tc + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xa[i], wb[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + tr + 16 * i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + tc + 16 * j;
            if (e >= E) continue;
            float l = acc[i][j];
            if (offset) l = __fadd_rn(l, __ldg(offset + e));
            s_out[static_cast<int64_t>(t) * E + e] = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-l)));
        }
    }
}

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

// One warp per token.  Per-warp shared row of r = s + b.
__global__ void __launch_bounds__(SEL_WARPS * 32) route_select_kernel(
    const float *__restrict__ s, const float *__restrict__ bias, int32_t *__restrict__ topk_idx,
    float *__restrict__ topk_w, int T, int E, int K, int n_group, int topk_group, float rho) {
    extern __shared__ float sh[];   // SEL_WARPS * E floats
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int t = blockIdx.x * SEL_WARPS + wid;
    if (t >= T) return;
    float *r = sh + wid * E;
    const float *srow = s + static_cast<int64_t>(t) * E;
    for (int e = lane; e < E; e += 32) r[e] = __fadd_rn(srow[e], __ldg(bias + e));
    __syncwarp();
    const int gs = E / n_group;
    // group scores: lane g scans its group for the two largest values
    float gscore = -FLT_MAX;
    bool gvalid = false;
    if (lane < n_group) {
        float m1 = -FLT_MAX, m2 = -FLT_MAX;
        for (int j = 0; j < gs; ++j) {
            const float v = r[lane * gs + j];
            if (v > m1) { m2 = m1; m1 = v; } else if (v > m2) { m2 = v; }
        }
        gscore = gs == 1 ? m1 : __fadd_rn(m1, m2);
        gvalid = true;
    }
    // keep the topk_group best groups (ties to the lower group)
    uint32_t kept = 0;
    bool taken_g = !gvalid;
    for (int round = 0; round < topk_group; ++round) {
        float v = taken_g ? -FLT_MAX : gscore;
        int i = taken_g ? 0x7fffffff : lane;
        if (taken_g) v = -INFINITY;
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
            const float v = r[e];
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

static int launch_select(const moe_dims *d, const float *scores, const float *e_bias, int32_t *idx,
                         float *w, cudaStream_t st) {
    const int blocks = (d->T + SEL_WARPS - 1) / SEL_WARPS;
    const size_t smem = static_cast<size_t>(SEL_WARPS) * d->E * sizeof(float);
    route_select_kernel<<<blocks, SEL_WARPS * 32, smem, st>>>(scores, e_bias, idx, w, d->T, d->E, d->K,
                                                              d->n_group, d->topk_group,
                                                              d->routed_scaling_factor);
    return launch_status();
}

size_t route_workspace_bytes(const moe_dims *d) {
    // the [T, E] fp32 affinities when the caller does not want them
    return (static_cast<size_t>(d->T) * d->E * sizeof(float) + 255) & ~static_cast<size_t>(255);
}

}  // namespace moe

using namespace moe;

MOE_API int moe_route(const moe_dims *d, const void *x, const float *w_router, const float *e_bias,
                      const float *router_offset, int32_t *topk_idx, float *topk_w, float *scores,
                      void *ws, size_t ws_bytes, int32_t *status, void *stream) {
    (void)status;
    int rc = check_route_dims(d);
    if (rc != MOE_OK) return rc;
    if (d->T == 0) return MOE_OK;
    if (!x || !w_router || !e_bias || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router)) return MOE_ERR_INVALID_ARG;
    float *s = scores;
    if (!s) {
        if (!ws || ws_bytes < route_workspace_bytes(d)) return MOE_ERR_WORKSPACE;
        s = reinterpret_cast<float *>(ws);
    }
    cudaStream_t st = as_stream(stream);
    dim3 grid((d->T + rt::BT - 1) / rt::BT, (d->E + rt::BE - 1) / rt::BE);
    router_logits_kernel<<<grid, rt::THREADS, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(x), w_router,
                                                       router_offset, s, d->T, d->H, d->E);
    rc = launch_status();
    if (rc != MOE_OK) return rc;
    return launch_select(d, s, e_bias, topk_idx, topk_w, st);
}

MOE_API int moe_route_select(const moe_dims *d, const float *scores, const float *e_bias,
                             int32_t *topk_idx, float *topk_w, void *stream) {
    int rc = check_route_dims(d);
    if (rc != MOE_OK) return rc;
    if (d->T == 0) return MOE_OK;
    if (!scores || !e_bias || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    return launch_select(d, scores, e_bias, topk_idx, topk_w, as_stream(stream));
}
