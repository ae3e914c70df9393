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

// SwiGLU of one (gate, up) pair in fp32, every operation rounded as written:
// silu(g) = g / (1 + exp(-g)), act = silu(g) * u.
__device__ __forceinline__ float swiglu_act(float g, float u) {
    float den = __fadd_rn(1.0f, expf(-g));
    return __fmul_rn(__fdiv_rn(g, den), u);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

}  // namespace moe
