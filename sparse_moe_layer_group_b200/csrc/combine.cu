// Gated combine with the shared expert, and the auxiliary-loss-free bias update.
//
// "DeepSeek-V3 technical report" walkthrough (2kiu.com), section 3.2: the layer
// output is y = sum_j gate_j * ffn_{idx_j}(h) (plus the always-on shared expert,
// section 1 / "DeepSeek-V3 MoE architecture and FP8 training" (0539edu.com):
// 1 shared + 256 routed experts); after each step the per-expert load is compared
// with the batch mean T*K/N_r and the bias moves by gamma against the imbalance
// (a feedback thermostat with no gradient; rate 0.001 in the lpnh.cn guide's
// section 3 config).
#include "common.cuh"

namespace moe {

// One CTA per token; each thread owns 8 consecutive columns per step.
__global__ void __launch_bounds__(128) combine_kernel(const uint4 *__restrict__ yperm,
                                                      const int32_t *__restrict__ row_of,
                                                      const float *__restrict__ topk_w,
                                                      const uint4 *__restrict__ yshared,
                                                      uint4 *__restrict__ out, float4 *__restrict__ out_f32,
                                                      int H, int K) {
    const int t = blockIdx.x;
    __shared__ int32_t rows[32];
    __shared__ float wts[32];
    if (threadIdx.x < K) {
        rows[threadIdx.x] = row_of[static_cast<int64_t>(t) * K + threadIdx.x];
        wts[threadIdx.x] = topk_w[static_cast<int64_t>(t) * K + threadIdx.x];
    }
    __syncthreads();
    const int nv = H / 8;
    for (int v = threadIdx.x; v < nv; v += blockDim.x) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        for (int k = 0; k < K; ++k) {
            const int r = rows[k];
            if (r < 0) continue;
            const float w = wts[k];
            const uint4 y = __ldg(yperm + static_cast<int64_t>(r) * nv + v);
            acc[0] = fmaf(w, bf16_lo(y.x), acc[0]); acc[1] = fmaf(w, bf16_hi(y.x), acc[1]);
            acc[2] = fmaf(w, bf16_lo(y.y), acc[2]); acc[3] = fmaf(w, bf16_hi(y.y), acc[3]);
            acc[4] = fmaf(w, bf16_lo(y.z), acc[4]); acc[5] = fmaf(w, bf16_hi(y.z), acc[5]);
            acc[6] = fmaf(w, bf16_lo(y.w), acc[6]); acc[7] = fmaf(w, bf16_hi(y.w), acc[7]);
        }
        if (yshared) {
            const uint4 y = __ldg(yshared + static_cast<int64_t>(t) * nv + v);
            acc[0] = __fadd_rn(acc[0], bf16_lo(y.x)); acc[1] = __fadd_rn(acc[1], bf16_hi(y.x));
            acc[2] = __fadd_rn(acc[2], bf16_lo(y.y)); acc[3] = __fadd_rn(acc[3], bf16_hi(y.y));
            acc[4] = __fadd_rn(acc[4], bf16_lo(y.z)); acc[5] = __fadd_rn(acc[5], bf16_hi(y.z));
            acc[6] = __fadd_rn(acc[6], bf16_lo(y.w)); acc[7] = __fadd_rn(acc[7], bf16_hi(y.w));
        }
        uint4 o;
        __nv_bfloat162 p;
        p = __floats2bfloat162_rn(acc[0], acc[1]); o.x = *reinterpret_cast<uint32_t *>(&p);
        p = __floats2bfloat162_rn(acc[2], acc[3]); o.y = *reinterpret_cast<uint32_t *>(&p);
        p = __floats2bfloat162_rn(acc[4], acc[5]); o.z = *reinterpret_cast<uint32_t *>(&p);
        p = __floats2bfloat162_rn(acc[6], acc[7]); o.w = *reinterpret_cast<uint32_t *>(&p);
        out[static_cast<int64_t>(t) * nv + v] = o;
        if (out_f32) {
            float4 *dst = out_f32 + (static_cast<int64_t>(t) * nv + v) * 2;
            dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
    }
}

// 8 values per thread: two 16-byte loads, one 16-byte bf16 store.
__global__ void combine_finish_kernel(float4 *__restrict__ acc, uint4 *__restrict__ out, float4 *__restrict__ f32,
                                      int64_t n8, int zero) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n8) return;
    const float4 a = acc[2 * i], b = acc[2 * i + 1];
    const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    out[i] = bf16x8(f);
    if (f32) {
        f32[2 * i] = a;
        f32[2 * i + 1] = b;
    }
    if (zero) {
        acc[2 * i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        acc[2 * i + 1] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
}

__global__ void bias_update_kernel(int E, int64_t TK, float gamma, const int32_t *__restrict__ load,
                                   float *__restrict__ bias) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    const int64_t diff = TK - static_cast<int64_t>(E) * load[e];
    if (diff > 0) bias[e] = __fadd_rn(bias[e], gamma);
    else if (diff < 0) bias[e] = __fsub_rn(bias[e], gamma);
}

}  // namespace moe

using namespace moe;

MOE_API int moe_combine(const moe_dims *d, const void *yperm, const int32_t *row_of, const float *topk_w,
                        const void *yshared, void *out, float *out_f32, void *stream) {
    if (!d || d->T < 0 || d->H < 0 || d->K <= 0 || d->H % 8 != 0) return MOE_ERR_INVALID_ARG;
    if (d->K > 32) return MOE_ERR_UNSUPPORTED;
    if (d->T == 0 || d->H == 0) return MOE_OK;
    if (!yperm || !row_of || !topk_w || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(yperm) || !aligned16(out) || (yshared && !aligned16(yshared)) ||
        (out_f32 && !aligned16(out_f32)))
        return MOE_ERR_INVALID_ARG;
    combine_kernel<<<d->T, 128, 0, as_stream(stream)>>>(
        reinterpret_cast<const uint4 *>(yperm), row_of, topk_w, reinterpret_cast<const uint4 *>(yshared),
        reinterpret_cast<uint4 *>(out), reinterpret_cast<float4 *>(out_f32), d->H, d->K);
    return launch_status();
}

MOE_API int moe_bias_update(int32_t E, int64_t T, int32_t K, float gamma, const int32_t *expert_load,
                            float *e_bias, void *stream) {
    if (E <= 0 || T < 0 || K <= 0) return MOE_ERR_INVALID_ARG;
    if (!expert_load || !e_bias) return MOE_ERR_INVALID_ARG;
    bias_update_kernel<<<(E + 255) / 256, 256, 0, as_stream(stream)>>>(E, T * K, gamma, expert_load, e_bias);
    return launch_status();
}

MOE_API int moe_combine_finish(float *acc, int64_t n, void *out_bf16, float *out_f32, int32_t zero, void *stream) {
    if (n < 0 || n % 8 != 0) return MOE_ERR_INVALID_ARG;
    if (n == 0) return MOE_OK;
    if (!acc || !out_bf16 || !aligned16(acc) || !aligned16(out_bf16) || (out_f32 && !aligned16(out_f32)))
        return MOE_ERR_INVALID_ARG;
    const int64_t n8 = n / 8;
    if ((n8 + 255) / 256 > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
    combine_finish_kernel<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, as_stream(stream)>>>(
        reinterpret_cast<float4 *>(acc), static_cast<uint4 *>(out_bf16), reinterpret_cast<float4 *>(out_f32), n8,
        zero ? 1 : 0);
    return launch_status();
}
