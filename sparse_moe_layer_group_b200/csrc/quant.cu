// FP8 (E4M3) quantisers: 1x128 activation tiles, 128x128 weight blocks, and the
// stand-alone SwiGLU + 1x128 requantisation.
//
// Scaling follows the "DeepSeek-V3 technical report" walkthrough (2kiu.com),
// section 4.3 (per-block scales so an outlier only spoils its own block), with
// the granularities of the "From technical report to a runnable config" guide
// (lpnh.cn), section 3: inputs tile-wise 1x128, weights block-wise 128x128, e4m3.
//
// All three kernels are HBM-bound streams: 16-byte vector loads, a group of
// lanes per tile, shuffles for the tile amax.
#include "common.cuh"

namespace moe {

// 8 lanes own one 1x128 tile: lane l holds columns 16l .. 16l+15 (two 16-byte
// loads, one 16-byte store of codes).  Each trip handles Q tiles per 8-lane
// group with all loads issued first, so several loads per thread are in flight.
template <int Q>
__device__ __forceinline__ void quant_tiles(const uint4 *__restrict__ x, uint4 *__restrict__ q,
                                            float *__restrict__ scales, int64_t first, int64_t stride,
                                            int64_t n_tiles, int lane8, int32_t *status) {
    uint4 v[Q][2];
#pragma unroll
    for (int u = 0; u < Q; ++u) {
        const int64_t tile = first + u * stride;
#pragma unroll
        for (int h = 0; h < 2; ++h)
            v[u][h] = tile < n_tiles ? __ldg(x + tile * 16 + lane8 * 2 + h) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < Q; ++u) {
        const int64_t tile = first + u * stride;
        float f[16];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            f[8 * h + 0] = bf16_lo(v[u][h].x); f[8 * h + 1] = bf16_hi(v[u][h].x);
            f[8 * h + 2] = bf16_lo(v[u][h].y); f[8 * h + 3] = bf16_hi(v[u][h].y);
            f[8 * h + 4] = bf16_lo(v[u][h].z); f[8 * h + 5] = bf16_hi(v[u][h].z);
            f[8 * h + 6] = bf16_lo(v[u][h].w); f[8 * h + 7] = bf16_hi(v[u][h].w);
        }
        // max |v| as the max of the magnitude bit patterns (ordered like the
        // values); a pattern >= 0x7f800000 is an Inf or NaN in the tile
        uint32_t um[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 16; ++i) um[i & 1] = max(um[i & 1], __float_as_uint(f[i]) & 0x7fffffffu);
        uint32_t umax = max(um[0], um[1]);
#pragma unroll
        for (int o = 4; o >= 1; o >>= 1) umax = max(umax, __shfl_xor_sync(0xffffffffu, umax, o));
        if (tile >= n_tiles) continue;
        const bool finite = umax < 0x7f800000u;
        const float sc = tile_scale(__uint_as_float(umax), finite);
        // codes of the correctly rounded quotients v / scale, two at a time
        // (e4m3x2_div: the product with the reciprocal wherever it provably
        // rounds like the quotient, else the division)
        const float inv = __frcp_rn(sc);
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = finite ? e4m3x2_div(f[4 * i], f[4 * i + 1], sc, inv) | e4m3x2_div(f[4 * i + 2], f[4 * i + 3], sc, inv) << 16
                          : 0x7F7F7F7Fu;
        q[tile * 8 + lane8] = make_uint4(w[0], w[1], w[2], w[3]);
        if (lane8 == 0) {
            scales[tile] = sc;
            if (!finite) set_flag(status, MOE_FLAG_NONFINITE);
        }
    }
}

constexpr int QUANT_Q = 2;

__global__ void __launch_bounds__(256) quant_1x128_kernel(const uint4 *__restrict__ x,
                                                          uint4 *__restrict__ q,
                                                          float *__restrict__ scales,
                                                          int64_t n_tiles, int32_t *status) {
    const int lane8 = threadIdx.x & 7;
    const int64_t group = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 3;
    const int64_t n_groups = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 3;
    // every 8-lane group runs the same trip count so the shuffles stay converged
    const int64_t per_trip = n_groups * QUANT_Q;
    const int64_t trips = (n_tiles + per_trip - 1) / per_trip;
    for (int64_t it = 0; it < trips; ++it)
        quant_tiles<QUANT_Q>(x, q, scales, group + it * per_trip, n_groups, n_tiles, lane8, status);
}

// One CTA per 128x128 block: 256 threads, each row of the block is 16 lanes x 16 B.
__global__ void __launch_bounds__(256) quant_128x128_kernel(const uint4 *__restrict__ w,
                                                            uint2 *__restrict__ q,
                                                            float *__restrict__ scales,
                                                            int64_t rows, int64_t cols,
                                                            int32_t *status) {
    const int64_t rb_n = rows / 128, cb_n = cols / 128;
    const int64_t blk = blockIdx.x;
    const int64_t b = blk / (rb_n * cb_n);
    const int64_t rb = (blk / cb_n) % rb_n, cb = blk % cb_n;
    const int64_t vec_per_row = cols / 8;
    const int tid = threadIdx.x;
    const int c16 = tid & 15;       // 16-byte column chunk within the block row
    const int r0 = tid >> 4;        // 0..15
    float f[8][8];
    float amax = 0.0f;
    bool fin = true;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const int64_t row = b * rows + rb * 128 + r0 + 16 * p;
        uint4 v = __ldg(w + row * vec_per_row + cb * 16 + c16);
        f[p][0] = bf16_lo(v.x); f[p][1] = bf16_hi(v.x); f[p][2] = bf16_lo(v.y); f[p][3] = bf16_hi(v.y);
        f[p][4] = bf16_lo(v.z); f[p][5] = bf16_hi(v.z); f[p][6] = bf16_lo(v.w); f[p][7] = bf16_hi(v.w);
#pragma unroll
        for (int i = 0; i < 8; ++i) amax_step(f[p][i], amax, fin);
    }
    __shared__ float s_amax[8];
    __shared__ int s_fin[8];
    int fin_i = fin ? 1 : 0;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        fin_i &= __shfl_xor_sync(0xffffffffu, fin_i, o);
    }
    if ((tid & 31) == 0) { s_amax[tid >> 5] = amax; s_fin[tid >> 5] = fin_i; }
    __syncthreads();
    amax = 0.0f;
    fin_i = 1;
#pragma unroll
    for (int i = 0; i < 8; ++i) { amax = fmaxf(amax, s_amax[i]); fin_i &= s_fin[i]; }
    const bool finite = fin_i != 0;
    const float s = tile_scale(amax, finite);
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const int64_t row = b * rows + rb * 128 + r0 + 16 * p;
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) lo |= static_cast<uint32_t>(quant_code(f[p][i], s, finite)) << (8 * i);
#pragma unroll
        for (int i = 0; i < 4; ++i) hi |= static_cast<uint32_t>(quant_code(f[p][4 + i], s, finite)) << (8 * i);
        q[row * vec_per_row + cb * 16 + c16] = make_uint2(lo, hi);
    }
    if (tid == 0) {
        scales[blk] = s;   // [batch, rows/128, cols/128] flattened == blk
        if (!finite) set_flag(status, MOE_FLAG_NONFINITE);
    }
}

// One warp per (row, 128-wide act tile): lane l owns act columns 4l .. 4l+3.
__global__ void __launch_bounds__(256) swiglu_requant_kernel(const float *__restrict__ gu,
                                                             uint32_t *__restrict__ q,
                                                             float *__restrict__ s, int64_t M,
                                                             int64_t I, int32_t *status) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t tiles_per_row = I / 128;
    const int64_t n_tiles = M * tiles_per_row;
    for (int64_t tile = warp; tile < n_tiles; tile += n_warps) {
        const int64_t row = tile / tiles_per_row, j = tile % tiles_per_row;
        const float *grow = gu + row * 2 * I;
        const float4 g = __ldg(reinterpret_cast<const float4 *>(grow + 128 * j) + lane);
        const float4 u = __ldg(reinterpret_cast<const float4 *>(grow + I + 128 * j) + lane);
        float a[4] = {swiglu_act(g.x, u.x), swiglu_act(g.y, u.y), swiglu_act(g.z, u.z),
                      swiglu_act(g.w, u.w)};
        float amax = 0.0f;
        bool fin = true;
#pragma unroll
        for (int i = 0; i < 4; ++i) amax_step(a[i], amax, fin);
        int fin_i = fin ? 1 : 0;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            fin_i &= __shfl_xor_sync(0xffffffffu, fin_i, o);
        }
        const bool finite = fin_i != 0;
        const float sc = tile_scale(amax, finite);
        const float inv = __frcp_rn(sc);
        const uint32_t packed =
            finite ? e4m3x2_div(a[0], a[1], sc, inv) | e4m3x2_div(a[2], a[3], sc, inv) << 16 : 0x7F7F7F7Fu;
        q[(row * I + 128 * j) / 4 + lane] = packed;
        if (lane == 0) {
            s[tile] = sc;
            if (!finite) set_flag(status, MOE_FLAG_NONFINITE);
        }
    }
}

}  // namespace moe

using namespace moe;

MOE_API int fp8_quant_1x128(const void *x, int64_t rows, int64_t cols, uint8_t *q, float *scales,
                            int32_t *status, void *stream) {
    if (rows < 0 || cols < 0 || cols % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return MOE_OK;
    if (!x || !q || !scales || !aligned16(x) || !aligned16(q) || !aligned16(scales))
        return MOE_ERR_INVALID_ARG;
    const int64_t n_tiles = rows * (cols / 128);
    // one trip per half-warp up to a million blocks (the hardware schedules the
    // blocks as SMs free up, so no trip is left mostly idle); beyond that the
    // half-warps loop over further trips
    const int64_t tiles_per_block = 256 / 8 * QUANT_Q;
    int64_t blocks = (n_tiles + tiles_per_block - 1) / tiles_per_block;
    const int64_t cap = int64_t(1) << 20;
    if (blocks > cap) blocks = cap;
    quant_1x128_kernel<<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(
        reinterpret_cast<const uint4 *>(x), reinterpret_cast<uint4 *>(q), scales, n_tiles, status);
    return launch_status();
}

MOE_API int fp8_quant_128x128(const void *w, int64_t batch, int64_t rows, int64_t cols, uint8_t *q,
                              float *scales, int32_t *status, void *stream) {
    if (batch < 0 || rows < 0 || cols < 0 || rows % 128 != 0 || cols % 128 != 0)
        return MOE_ERR_INVALID_ARG;
    if (batch == 0 || rows == 0 || cols == 0) return MOE_OK;
    if (!w || !q || !scales || !aligned16(w) || !aligned16(q)) return MOE_ERR_INVALID_ARG;
    const int64_t blocks = batch * (rows / 128) * (cols / 128);
    if (blocks > 0x7fffffff) return MOE_ERR_UNSUPPORTED;
    quant_128x128_kernel<<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(
        reinterpret_cast<const uint4 *>(w), reinterpret_cast<uint2 *>(q), scales, rows, cols, status);
    return launch_status();
}

MOE_API int swiglu_requant(const float *gu, int64_t M, int64_t I, uint8_t *q, float *s,
                           int32_t *status, void *stream) {
    if (M < 0 || I < 0 || I % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (M == 0 || I == 0) return MOE_OK;
    if (!gu || !q || !s || !aligned16(gu) || !aligned16(q)) return MOE_ERR_INVALID_ARG;
    const int64_t n_tiles = M * (I / 128);
    int64_t blocks = (n_tiles + 7) / 8;
    const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    swiglu_requant_kernel<<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(
        gu, reinterpret_cast<uint32_t *>(q), s, M, I, status);
    return launch_status();
}
