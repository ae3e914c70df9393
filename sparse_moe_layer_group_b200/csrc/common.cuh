// Shared device/host helpers of the sm_100a kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/moe_b200.h"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace moe {

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

constexpr int MAX_DEVICES = 64;

// The current device, or -1 when it cannot be queried.
inline int current_device() {
    int dev = -1;
    return cudaGetDevice(&dev) == cudaSuccess ? dev : -1;
}

// Per-device, once-only set-up (kernel attributes, occupancy queries): runs
// `fn` for the current device the first time and returns its cached result
// afterwards.  `state` and `mu` belong to one call site; thread-safe.  fn
// returns a positive value on success; a non-positive result is not cached.
template <typename F>
inline int once_per_device(int (&state)[MAX_DEVICES], std::mutex &mu, F fn) {
    const int dev = current_device();
    if (dev < 0 || dev >= MAX_DEVICES) return fn();
    std::lock_guard<std::mutex> lock(mu);
    if (state[dev] <= 0) state[dev] = fn();
    return state[dev];
}

// Number of SMs of the current device (cached per device).
inline int num_sms() {
    static int state[MAX_DEVICES] = {};
    static std::mutex mu;
    return once_per_device(state, mu, []() {
        int dev = 0, n = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        return n > 0 ? n : 148;
    });
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

// E4M3 codes of fp32(a / s) and fp32(b / s), the correctly rounded quotients
// of the quantisation rule, for a tile whose scale s has the correctly rounded
// reciprocal inv = 1/s.  Low byte = a.
//
// q = fp32(v * inv) differs from v / s by at most 2^-24 |v/s| (the reciprocal)
// plus half an ulp (the product), so the correctly rounded quotient lies
// within three steps of the fp32 grid from q, on q's side of zero.  For |q| in
// the E4M3 normal range (>= 2^-6) the E4M3 rounding boundaries of q's binade
// are the fp32 values whose 20 bits below E4M3's three mantissa bits read
// 0x80000 (binade edges are E4M3 values), and E4M3 rounding is monotone; so
// when those 20 bits of q are more than four steps from 0x80000, the quotient
// rounds to q's code.  Otherwise (a quotient within a few fp32 ulps of a
// boundary, |q| below 2^-6 where E4M3 is subnormal, or a reciprocal that
// overflowed) the quotient is computed by the correctly rounded division.
__device__ __forceinline__ uint32_t e4m3x2_cvt(float a, float b) {
    return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}
__device__ __forceinline__ bool e4m3_near_boundary(float q) {
    const uint32_t u = __float_as_uint(q) & 0x7fffffffu;
    return (u != 0u && u < 0x3C800000u) || ((u & 0xFFFFFu) - 0x7FFFCu) <= 8u;
}
// E4M3 codes of fp32(a * inv) and fp32(b * inv), inv the correctly rounded
// reciprocal of the tile scale: the fast form of the requantisation, within 1.5
// fp32 ulps of the quotient before the E4M3 rounding.  Low byte = a.
__device__ __forceinline__ uint32_t e4m3x2_rcp(float a, float b, float inv) {
    return e4m3x2_cvt(__fmul_rn(a, inv), __fmul_rn(b, inv));
}
__device__ __forceinline__ uint32_t e4m3x2_div(float a, float b, float s, float inv) {
    if (isfinite(inv)) {
        const float qa = __fmul_rn(a, inv), qb = __fmul_rn(b, inv);
        if (!e4m3_near_boundary(qa) && !e4m3_near_boundary(qb)) return e4m3x2_cvt(qa, qb);
    }
    return e4m3x2_cvt(__fdiv_rn(a, s), __fdiv_rn(b, s));
}

// Eight fp32 values rounded (RN) to bf16 and packed into 16 bytes, f[0] lowest.
__device__ __forceinline__ uint4 bf16x8(const float *f) {
    const __nv_bfloat162 p0 = __floats2bfloat162_rn(f[0], f[1]), p1 = __floats2bfloat162_rn(f[2], f[3]);
    const __nv_bfloat162 p2 = __floats2bfloat162_rn(f[4], f[5]), p3 = __floats2bfloat162_rn(f[6], f[7]);
    return make_uint4(*reinterpret_cast<const uint32_t *>(&p0), *reinterpret_cast<const uint32_t *>(&p1),
                      *reinterpret_cast<const uint32_t *>(&p2), *reinterpret_cast<const uint32_t *>(&p3));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

}  // namespace moe
