// Shared device/host helpers of the sm_100a kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe_b200.h"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace moe {

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

inline int num_sms() {
    static int cached = 0;
    if (cached == 0) {
        int dev = 0, n = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached = n > 0 ? n : 148;
    }
    return cached;
}

__device__ __forceinline__ void set_flag(int32_t *status, int32_t bit) {
    if (status) atomicOr(status, bit);
}

// ------------------------------------------------------------- E4M3 rule
// One correctly rounded fp32 division and the hardware's round-to-nearest-even
// saturating conversion (cvt.rn.satfinite.e4m3x2.f32).
__device__ __forceinline__ uint8_t e4m3_of(float v) {
    return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

// Scale of one tile/block from its max |v|; finite == false for a tile
// holding NaN/Inf.  amax == 0 gives 1; otherwise fp32(amax / 448).
__device__ __forceinline__ float tile_scale(float amax, bool finite) {
    if (!finite) return __int_as_float(0x7fc00000);
    return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
}

__device__ __forceinline__ uint8_t quant_code(float v, float scale, bool finite) {
    return finite ? e4m3_of(__fdiv_rn(v, scale)) : static_cast<uint8_t>(0x7F);
}

// |v| folded into a running max, tracking non-finite values separately
// (fmaxf alone would drop NaN).
__device__ __forceinline__ void amax_step(float v, float &amax, bool &finite) {
    finite = finite && isfinite(v);
    amax = fmaxf(amax, fabsf(v));
}

// SwiGLU activation silu(g) * u = g / (1 + exp(-g)) * u in fp32, with the
// hardware exp2 approximation (__expf) and approximate division (__fdividef):
// a few fp32 ulps from the exact value wherever the result is large enough to
// set a tile's scale (the error of __expf grows with |g| only where exp(-g)
// dominates the denominator, i.e. where the activation is near zero).
__device__ __forceinline__ float swiglu_act(float g, float u) {
    return __fmul_rn(__fdividef(g, __fadd_rn(1.0f, __expf(-g))), u);
}

// E4M3 codes of two activation values against one tile scale, given as its
// correctly rounded reciprocal (the requantisation of the SwiGLU output:
// fp32(v * (1/s)) differs from fp32(v / s) by at most one ulp, below the error
// the activation already carries).  Low byte = a.
__device__ __forceinline__ uint32_t e4m3x2_rcp(float a, float b, float inv) {
    return static_cast<uint32_t>(
        __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(a, inv), __fmul_rn(b, inv)), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

}  // namespace moe
