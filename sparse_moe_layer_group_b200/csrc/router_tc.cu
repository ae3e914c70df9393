// Router logits on the tensor cores with fp32 weights, exactly.
//
// The router stays in high precision ("From technical report to a runnable
// config" guide (lpnh.cn), section 3: keep_bf16 moe_gating; "DeepSeek-V3
// technical report" walkthrough (2kiu.com), section 3.2: s = sigmoid(h W_router)).
// x is bf16 and W_r is fp32.  Every fp32 weight is the exact sum of three bf16
// pieces, W = W0 + W1 + W2 (W0 = bf16(W), W1 = bf16(W - W0), W2 = W - W0 - W1,
// which has at most 8 significant bits), so
//     x W^T = x W0^T + x W1^T + x W2^T
// where every product x * Wj is exact in fp32 and the tensor core accumulates in
// fp32: the fp32 dot product, computed as a bf16 GEMM with K = 3H.
//
// router_split_kernel  W fp32 [E, H] -> pieces bf16 [3, E, H]
// router_tc_kernel     one 128 x 256 tile of logits per CTA over one K split
//                      (two CTAs per SM, 256 TMEM columns each):
//                      warp 0 TMA (x tile 128 x 64 bf16, two 128-row W halves),
//                      warp 1 TMEM (256 columns) + tcgen05.mma kind::f16,
//                      warps 2-5 read TMEM and store the fp32 partial sums
//                      [split, T, E]; route_select_kernel adds the splits in
//                      a fixed order (deterministic), applies the sigmoid and
//                      selects.
#include "tc_util.cuh"

namespace moe {
namespace rtc {

using namespace moe::tc;

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BKE = 64;                 // bf16 elements per 128-byte swizzle row
constexpr int STAGES = 2;               // 2 x 48 KB: two CTAs share an SM
constexpr uint32_t A_BYTES = BM * 128;
constexpr uint32_t B_HALF = 128 * 128;
constexpr uint32_t STAGE_BYTES = A_BYTES + 2 * B_HALF;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t OFF_BARS = STAGES * STAGE_BYTES;
constexpr uint32_t OFF_MISC = OFF_BARS + 128;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 32 + 1024;
// D fp32, A and B bf16, both K-major, N = 256, M = 128
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                           (static_cast<uint32_t>(BM >> 4) << 24);
constexpr int MAX_SPLIT = 32;

__global__ void __launch_bounds__(256) router_split_kernel(const float4 *__restrict__ w, uint2 *__restrict__ p0,
                                                           uint2 *__restrict__ p1, uint2 *__restrict__ p2,
                                                           int64_t n4) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n4) return;
    const float4 v = __ldg(w + i);
    const float f[4] = {v.x, v.y, v.z, v.w};
    uint16_t a[4], b[4], c[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const __nv_bfloat16 h0 = __float2bfloat16_rn(f[k]);
        const float r1 = __fsub_rn(f[k], __bfloat162float(h0));      // exact
        const __nv_bfloat16 h1 = __float2bfloat16_rn(r1);
        const float r2 = __fsub_rn(r1, __bfloat162float(h1));        // exact, <= 8 significant bits
        const __nv_bfloat16 h2 = __float2bfloat16_rn(r2);            // exact
        a[k] = __bfloat16_as_ushort(h0);
        b[k] = __bfloat16_as_ushort(h1);
        c[k] = __bfloat16_as_ushort(h2);
    }
    p0[i] = make_uint2(a[0] | (uint32_t(a[1]) << 16), a[2] | (uint32_t(a[3]) << 16));
    p1[i] = make_uint2(b[0] | (uint32_t(b[1]) << 16), b[2] | (uint32_t(b[3]) << 16));
    p2[i] = make_uint2(c[0] | (uint32_t(c[1]) << 16), c[2] | (uint32_t(c[3]) << 16));
}

__global__ void __launch_bounds__(THREADS, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, int T, int E,
                 int H, int kb_per_split, float *__restrict__ partial, int32_t *status) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
    const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    const uint32_t sbase = raw_addr + pad;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar0 = sbase + OFF_BARS;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    const uint32_t tfull_bar = bar0 + 8u * (2 * STAGES);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);

    const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN, split = blockIdx.z;
    const int kb_h = H / BKE;                 // K blocks per piece
    const int kb_total = 3 * kb_h;
    const int kb_begin = split * kb_per_split;
    const int kb_end = min(kb_total, kb_begin + kb_per_split);
    const int n_kb = kb_end > kb_begin ? kb_end - kb_begin : 0;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
        mbar_init(tfull_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sbase + OFF_MISC),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // TMA producer: the whole warp runs the loop, lane 0 issues
        const uint32_t one = lane == 0 ? 1u : 0u;
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        for (int kb = kb_begin; kb < kb_end; ++kb) {
            if (!__all_sync(0xffffffffu, mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, status))) break;
            const int piece = kb / kb_h, k0 = (kb % kb_h) * BKE;
            const uint32_t sa = sbase + stage * STAGE_BYTES;
            mbar_expect_tx_if(full_bar(stage), STAGE_BYTES, one);
            tma_load_2d(sa, &tmX, k0, m0, full_bar(stage), one);
            tma_load_3d(sa + A_BYTES, &tmW, k0, n0, piece, full_bar(stage), one);
            tma_load_3d(sa + A_BYTES + B_HALF, &tmW, k0, n0 + 128, piece, full_bar(stage), one);
            __syncwarp();
            ++issued;
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (lane == 0) {
            const int tail = issued < STAGES ? issued : STAGES;
            for (int i = 0; i < tail; ++i) {
                if (stage == 0) { stage = STAGES - 1; phase ^= 1u; } else { --stage; }
                mbar_wait(full_bar(stage), phase, abort_flag, status, true);
            }
        }
    } else if (warp == 1) {
        // MMA issuer: the whole warp runs the loop, lane 0 issues
        const uint32_t one = lane == 0 ? 1u : 0u;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int i = 0; i < n_kb; ++i) {
            if (!__all_sync(0xffffffffu, mbar_wait(full_bar(stage), phase, abort_flag, status))) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = sbase + stage * STAGE_BYTES;
            const uint64_t ad = sw128_desc(sa), bd = sw128_desc(sa + A_BYTES);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_f16(tmem, ad + 2u * k, bd + 2u * k, IDESC, (i > 0 || k > 0) ? 1u : 0u, one);
            mma_commit(empty_bar(stage), one);
            __syncwarp();
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        // tfull also serves as the drain: it fires once every MMA issued above is done
        mma_commit(tfull_bar, one);
        __syncwarp();
        if (!ok && lane == 0) mbar_wait(tfull_bar, 0, abort_flag, status, true);
    } else {
        // epilogue: warps 2..5 cover TMEM lane quarters 2, 3, 0, 1
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const int t = m0 + row;
        const bool ok = mbar_wait(tfull_bar, 0, abort_flag, status);
        tc_fence_after();
        if (ok) {
            float *dst = partial + (static_cast<int64_t>(split) * T + t) * E;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + 32u * c, r);
                const int e0 = n0 + 32 * c;
                if (t >= T || e0 >= E) continue;
                if (n_kb == 0) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = 0u;
                }
                if (e0 + 32 <= E && (E % 4) == 0) {
                    float4 *d4 = reinterpret_cast<float4 *>(dst + e0);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        d4[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                            __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
                } else {
                    for (int j = 0; j < 32 && e0 + j < E; ++j) dst[e0 + j] = __uint_as_float(r[j]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
                     : "memory");
    }
}

}  // namespace rtc

// Number of K splits for T tokens and E experts: enough CTAs to fill every SM
// with two CTAs, at least 8 K blocks per split.
int router_splits(int T, int E, int H) {
    const int tiles = ((T + rtc::BM - 1) / rtc::BM) * ((E + rtc::BN - 1) / rtc::BN);
    const int kb_total = 3 * (H / rtc::BKE);
    int s = 2 * num_sms() / (tiles > 0 ? tiles : 1);
    if (s > rtc::MAX_SPLIT) s = rtc::MAX_SPLIT;
    if (s > kb_total / 8) s = kb_total / 8;
    return s < 1 ? 1 : s;
}

size_t router_tc_ws_bytes(int T, int E, int H) {
    const size_t pieces = (static_cast<size_t>(3) * E * H * 2 + 255) & ~size_t(255);
    const size_t part = (static_cast<size_t>(router_splits(T, E, H)) * T * E * 4 + 255) & ~size_t(255);
    return pieces + part;
}

// W fp32 [E, H] -> three exact bf16 pieces [3, E, H] (the per-weight-set step).
int launch_router_split(const float *w, int E, int H, void *pieces_out, cudaStream_t st) {
    using namespace rtc;
    const size_t piece_elems = static_cast<size_t>(E) * H;
    __nv_bfloat16 *pieces = reinterpret_cast<__nv_bfloat16 *>(pieces_out);
    const int64_t n4 = static_cast<int64_t>(piece_elems / 4);
    router_split_kernel<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, st>>>(
        reinterpret_cast<const float4 *>(w), reinterpret_cast<uint2 *>(pieces),
        reinterpret_cast<uint2 *>(pieces + piece_elems), reinterpret_cast<uint2 *>(pieces + 2 * piece_elems), n4);
    return launch_status();
}

// Tensor-core logits from the pieces; the split-K partial sums land in ws after
// the space a per-call split would use (so both routes share one workspace size).
int launch_router_tc(const void *x, const void *pieces_in, int T, int E, int H, void *ws, float **partial_out,
                     int *n_split_out, int32_t *status, cudaStream_t st) {
    using namespace rtc;
    static int state[MAX_DEVICES] = {};
    static std::mutex mu;
    const int ready = once_per_device(state, mu, []() {
        return cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(SMEM_BYTES)) == cudaSuccess
                   ? 1
                   : -MOE_ERR_CUDA;
    });
    if (ready <= 0) return MOE_ERR_CUDA;
    auto enc = encode_fn();
    if (!enc) return MOE_ERR_CUDA;
    uint8_t *base = static_cast<uint8_t *>(ws);
    const size_t piece_elems = static_cast<size_t>(E) * H;
    const void *pieces = pieces_in;
    float *partial = reinterpret_cast<float *>(base + ((3 * piece_elems * 2 + 255) & ~size_t(255)));
    CUtensorMap tmX, tmW;
    {
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(H) * 2};
        cuuint32_t box[2] = {BKE, BM};
        cuuint32_t es[2] = {1, 1};
        if (enc(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MOE_ERR_CUDA;
    }
    {
        cuuint64_t dims[3] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(E), 3};
        cuuint64_t strides[2] = {static_cast<cuuint64_t>(H) * 2, static_cast<cuuint64_t>(piece_elems) * 2};
        cuuint32_t box[3] = {BKE, 128, 1};
        cuuint32_t es[3] = {1, 1, 1};
        if (enc(&tmW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(pieces), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MOE_ERR_CUDA;
    }
    const int n_split = router_splits(T, E, H);
    const int kb_total = 3 * (H / BKE);
    const int kb_per_split = (kb_total + n_split - 1) / n_split;
    dim3 grid((T + BM - 1) / BM, (E + BN - 1) / BN, n_split);
    router_tc_kernel<<<grid, THREADS, SMEM_BYTES, st>>>(tmX, tmW, T, E, H, kb_per_split, partial, status);
    *partial_out = partial;
    *n_split_out = n_split;
    return launch_status();
}

}  // namespace moe
