// Weight gradient of the expert GEMMs in FP8 (E4M3): the 128x1 grouped
// quantiser and the grouped wgrad GEMM on the sm_100a tensor cores.
//
// What it computes (the lpnh.cn guide "From technical report to a runnable
// config", section 3: gemm_fprop, gemm_dgrad and gemm_wgrad all in e4m3 with
// tile-wise 1x128 input scaling; the Zhihu infrastructure answer on
// DeepSeek-V3: E4M3 in the forward and the backward pass, partial sums
// promoted because the tensor cores apply no per-tile scales).  For expert g
// with rows m in [offsets[g], offsets[g+1]) of dY [M, N] and X [M, K]:
//   dW[g, n, k] = sum_t  sdy[t, n] * sx[t, k] * sum_{m in tile t} e4m3(dY[m, n]) e4m3(X[m, k])
// The contraction runs over the expert's rows, so the 1x128 input tiling is
// taken along it: tiles of 128 consecutive rows of one column (128x1), never
// crossing the expert's row range (the last tile of a ragged range is shorter),
// each with its own scale (amax / 448, the forward rule).
//
// Layout.  The quantiser writes both operands transposed and row-padded: code
// q_t[c, 128 t + r] for row r of tile t (tiles numbered in group order, rows
// beyond a short tile are code 0), so each operand is K-major along the
// contraction, which is what tcgen05 reads, and each tile is one 128-wide K
// block of the GEMM.  Scales are [tile, column].
//
// The GEMM is the forward grouped kernel's pipeline (persistent CTAs, TMA
// loads, tcgen05.mma into two 256-column TMEM buffers, promotion in the
// epilogue warps) with two differences: a tile's K-block count is its group's
// tile count (an empty group writes zeros), and the promotion scale is an
// outer product -- a row scale sdy[t, n] per thread and a column scale
// sx[t, k] per accumulator column, the latter copied into shared memory with
// each stage (the stage is released only after the MMA and all epilogue
// threads are done with it).
#include "tc_util.cuh"

namespace moe {
namespace wg {

using namespace moe::tc;

constexpr int MAX_G = 2048;
constexpr int BN = 256;                      // output columns (k) per tile
constexpr uint32_t A_BYTES = 128 * 128;      // 128 rows of dY^T x one tile of 128 rows
constexpr uint32_t B_BYTES = 256 * 128;      // 256 rows of X^T
constexpr uint32_t SX_BYTES = 256 * 4;       // the tile's column scales of X
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + SX_BYTES;   // 49 KB, 1 KB aligned
constexpr int STAGES = 3;
constexpr int THREADS = 384;
constexpr int EPI_THREADS = 256;
constexpr uint32_t TMEM_COLS = 512;
constexpr int LAUNCH_REGS = 168;
constexpr uint32_t EPI_BOX = 32 * 128;          // one TMA-store box: 32 rows x 32 fp32, 128-byte swizzle
constexpr uint32_t EPI_STG = 2 * EPI_BOX;       // per epilogue warp: two boxes in flight
constexpr uint32_t OFF_EPI = STAGES * STAGE_BYTES;
constexpr uint32_t OFF_BARS = OFF_EPI + 8 * EPI_STG;
constexpr uint32_t OFF_MISC = OFF_BARS + 128;
constexpr uint32_t OFF_TSTART = OFF_MISC + 32;   // int32 [G + 1]
constexpr uint32_t SMEM_BYTES = OFF_TSTART + (MAX_G + 1) * 4 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "wgrad shared memory");
static_assert(STAGE_BYTES % 1024 == 0, "stages stay 1 KB aligned (128-byte swizzle atoms)");
// D fp32, A/B e4m3, K-major both, N = 256, M = 128
constexpr uint32_t IDESC = (1u << 4) | (static_cast<uint32_t>(BN >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);

// tstart[g] = number of 128-row tiles of groups 0..g-1 (tstart[G] = all tiles),
// by one warp; *bad is set for decreasing or out-of-range offsets.
__device__ __forceinline__ void group_tiles(const int32_t *__restrict__ offs, int G, int64_t M, int32_t *tstart,
                                            int lane, int *bad) {
    int carry = 0;
    for (int base = 0; base < G; base += 32) {
        const int g = base + lane;
        int v = 0;
        if (g < G) {
            const int a = __ldg(offs + g), b = __ldg(offs + g + 1);
            if (b < a || a < 0 || static_cast<int64_t>(b) > M) *bad = 1;
            v = b > a ? (b - a + 127) / 128 : 0;
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += n;
        }
        if (g < G) tstart[g + 1] = v + carry;
        carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) tstart[0] = 0;
}

// ---------------------------------------------------------------- quantiser
// CTA = (tile t, a strided set of 128-column blocks: gridDim.y of them apart),
// so the group-table scan is paid once per several blocks.  Each 128 x 128 bf16
// block is staged in shared memory with 16-byte loads (eight per thread, all
// issued before use); then thread (column c, half h) owns rows 64h..64h+63 of
// column c.
__global__ void __launch_bounds__(256) quant_128x1_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t C,
                                                          const int32_t *__restrict__ offs, int G,
                                                          uint8_t *__restrict__ q_t, int64_t p_cap,
                                                          float *__restrict__ scales, int64_t t_cap,
                                                          int32_t *status) {
    __shared__ int32_t tstart[MAX_G + 1];
    __shared__ __align__(16) uint16_t blk[128 * 128];   // the tile's rows x 128 columns
    __shared__ float s_amax[2][128];
    __shared__ int s_fin[2][128];
    __shared__ int bad;
    const int tid = threadIdx.x, lane = tid & 31;
    if (tid == 0) bad = 0;
    __syncthreads();
    if (tid < 32) group_tiles(offs, G, M, tstart, lane, &bad);
    __syncthreads();
    const int n_tiles = tstart[G];
    if (bad || n_tiles > t_cap || static_cast<int64_t>(n_tiles) * 128 > p_cap) {
        if (blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) set_flag(status, MOE_FLAG_BAD_OFFSETS);
        return;
    }
    const int t = blockIdx.x;
    if (t >= n_tiles) return;
    int lo = 0, hi = G;          // the group of tile t: tstart[lo] <= t < tstart[lo + 1]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tstart[mid] <= t) lo = mid; else hi = mid;
    }
    const int g = lo;
    const int64_t r0 = __ldg(offs + g) + static_cast<int64_t>(t - tstart[g]) * 128;
    const int64_t r1 = min(r0 + 128, static_cast<int64_t>(__ldg(offs + g + 1)));
    const int nrows = static_cast<int>(r1 - r0);
    const int cl = tid & 127, h = tid >> 7;
    for (int64_t cb = blockIdx.y; cb < C / 128; cb += gridDim.y) {
    const int64_t c0 = cb * 128;
    const int64_t c = c0 + cl;
    __syncthreads();   // the previous block's reads of blk and s_amax are done
    {
        // 128 rows x 256 bytes: 16 lanes per row, 16 rows per pass, 8 passes
        uint4 ld[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const int r = 16 * p + (tid >> 4), seg = tid & 15;
            ld[p] = r < nrows ? __ldg(reinterpret_cast<const uint4 *>(x + (r0 + r) * C + c0) + seg)
                              : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const int r = 16 * p + (tid >> 4), seg = tid & 15;
            reinterpret_cast<uint4 *>(blk + r * 128)[seg] = ld[p];
        }
    }
    __syncthreads();
    float v[64];
    float amax = 0.0f;
    bool fin = true;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        v[i] = __uint_as_float(static_cast<uint32_t>(blk[(64 * h + i) * 128 + cl]) << 16);
        amax_step(v[i], amax, fin);
    }
    s_amax[h][cl] = amax;
    s_fin[h][cl] = fin ? 1 : 0;
    __syncthreads();
    const bool finite = s_fin[0][cl] && s_fin[1][cl];
    const float sc = tile_scale(fmaxf(s_amax[0][cl], s_amax[1][cl]), finite);
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        uint32_t p = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = 64 * h + 4 * i + j;
            const uint32_t code = r < nrows ? quant_code(v[4 * i + j], sc, finite) : 0u;
            p |= code << (8 * j);
        }
        w[i] = p;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(q_t + c * p_cap + static_cast<int64_t>(t) * 128 + 64 * h);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    if (h == 0) {
        scales[static_cast<int64_t>(t) * C + c] = sc;
        if (!finite) set_flag(status, MOE_FLAG_NONFINITE);
    }
    }
}

// ---------------------------------------------------------------- GEMM
struct Tile {
    int g, n0, k0, ts, kb;   // group, first output row / column, first tile, tile count
};

__device__ __forceinline__ Tile decode(int t, int NTn, int NTk, const int32_t *tstart) {
    Tile r;
    const int per = NTn * NTk;
    r.g = t / per;
    const int local = t - r.g * per;
    r.n0 = (local / NTk) * 128;
    r.k0 = (local % NTk) * BN;
    r.ts = tstart[r.g];
    r.kb = tstart[r.g + 1] - r.ts;
    return r;
}

__global__ void __launch_bounds__(THREADS, 1)
wgrad_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
             const __grid_constant__ CUtensorMap tmD, const int32_t *__restrict__ offs, int G, int64_t M, int N, int K, const float *__restrict__ sdy,
             const float *__restrict__ sx, int64_t t_cap, int64_t p_cap, float *__restrict__ dW, int32_t *status,
             uint64_t wait_ns) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
    const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    const uint32_t sbase = raw_addr + pad;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar0 = sbase + OFF_BARS;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
    int *bad_flag = reinterpret_cast<int *>(smem + OFF_MISC + 8);
    int32_t *tstart = reinterpret_cast<int32_t *>(smem + OFF_TSTART);

    const int NTn = N / 128, NTk = (K + BN - 1) / BN;

    if (threadIdx.x == 0) { *abort_flag = 0; *bad_flag = 0; }
    __syncthreads();
    if (warp == 0) {
        group_tiles(offs, G, M, tstart, lane, bad_flag);
    } else if (warp == 2 && lane == 0) {
        // the empty barrier of a stage also waits for every epilogue thread,
        // which reads the stage's column scales while promoting
        for (int s = 0; s < STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1 + EPI_THREADS); }
        for (int b = 0; b < 2; ++b) { mbar_init(tfull_bar(b), 1); mbar_init(tempty_bar(b), EPI_THREADS); }
        mbar_init(drain_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    } else if (warp == 3 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmD)) : "memory");
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
    const uint32_t tmem_base = *tmem_holder;
    const bool bad = *bad_flag || tstart[G] > t_cap || static_cast<int64_t>(tstart[G]) * 128 > p_cap;
    const int num_tiles = bad ? 0 : G * NTn * NTk;
    if (blockIdx.x == 0 && threadIdx.x == 0 && bad) set_flag(status, MOE_FLAG_BAD_OFFSETS);

    __syncwarp();
    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 40;" ::: "memory");
        if (warp == 0) {
            // ------------------------------------------------ TMA producer
            const uint32_t one = lane == 0 ? 1u : 0u;
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
                const Tile tl = decode(t, NTn, NTk, tstart);
                const uint32_t sx_bytes = static_cast<uint32_t>(min(BN, K - tl.k0)) * 4u;
                for (int kb = 0; kb < tl.kb; ++kb) {
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, status, false, wait_ns));
                    if (!ok) break;
                    const uint32_t sa = sbase + stage * STAGE_BYTES;
                    const int xk = (tl.ts + kb) * 128;       // contraction coordinate (padded row)
                    mbar_expect_tx_if(full_bar(stage), A_BYTES + B_BYTES + sx_bytes, one);
                    tma_load_2d(sa, &tmA, xk, tl.n0, full_bar(stage), one);
                    tma_load_2d(sa + A_BYTES, &tmB, xk, tl.k0, full_bar(stage), one);
                    tma_load_2d(sa + A_BYTES + B_BYTES / 2, &tmB, xk, tl.k0 + 128, full_bar(stage), one);
                    bulk_load(sa + A_BYTES + B_BYTES, sx + static_cast<int64_t>(tl.ts + kb) * K + tl.k0, sx_bytes,
                              full_bar(stage), one);
                    __syncwarp();
                    ++issued;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (lane == 0) {
                const int tail = issued < STAGES ? issued : STAGES;
                for (int i = 0; i < tail; ++i) {
                    if (stage == 0) { stage = STAGES - 1; phase ^= 1u; } else { --stage; }
                    mbar_wait(full_bar(stage), phase, abort_flag, status, true);
                }
            }
        } else if (warp == 1) {
            // ------------------------------------------------ MMA issuer
            const uint32_t one = lane == 0 ? 1u : 0u;
            int stage = 0;
            uint32_t phase = 0, kc = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
                const Tile tl = decode(t, NTn, NTk, tstart);
                for (int kb = 0; kb < tl.kb; ++kb, ++kc) {
                    const uint32_t buf = kc & 1u, use = kc >> 1;
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait(tempty_bar(buf), (use & 1u) ^ 1u, abort_flag, status, false, wait_ns));
                    if (!ok) break;
                    ok = __all_sync(0xffffffffu, mbar_wait(full_bar(stage), phase, abort_flag, status, false, wait_ns));
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t sa = sbase + stage * STAGE_BYTES;
                    const uint64_t ad = sw128_desc(sa), bd = sw128_desc(sa + A_BYTES);
                    const uint32_t d = tmem_base + buf * 256u;
#pragma unroll
                    for (int k = 0; k < 4; ++k) mma_f8(d, ad + 2u * k, bd + 2u * k, IDESC, k > 0 ? 1u : 0u, one);
                    mma_commit(empty_bar(stage), one);
                    mma_commit(tfull_bar(buf), one);
                    __syncwarp();
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            mma_commit(drain_bar, one);
            __syncwarp();
            mbar_wait(drain_bar, 0, abort_flag, status, true);
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 232;" ::: "memory");
        // ---------------------------------------------------- epilogue
        const int q = warp & 3, half = (warp - 4) >> 2;
        const int row = q * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
        uint32_t kc = 0, sphase = 0;
        int stage = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
            const Tile tl = decode(t, NTn, NTk, tstart);
            const int n = tl.n0 + row;
            float acc[128];
#pragma unroll
            for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
            float ns = tl.kb > 0 ? __ldg(sdy + static_cast<int64_t>(tl.ts) * N + n) : 0.0f;
            for (int kb = 0; kb < tl.kb; ++kb, ++kc) {
                const float s_row = ns;
                if (kb + 1 < tl.kb) ns = __ldg(sdy + static_cast<int64_t>(tl.ts + kb + 1) * N + n);
                const uint32_t buf = kc & 1u, use = kc >> 1;
                if (!__all_sync(0xffffffffu, mbar_wait(tfull_bar(buf), use & 1u, abort_flag, status, false, wait_ns))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // the stage's TMA bytes (column scales) are visible to this thread
                // once it has seen the stage's full phase (completed long ago; the
                // stage cannot be refilled before this thread releases it)
                mbar_wait(full_bar(stage), sphase, abort_flag, status, true);
                const float *sxs = reinterpret_cast<const float *>(smem + stage * STAGE_BYTES + A_BYTES + B_BYTES) +
                                   128 * half;
                const float2 sr2 = make_float2(s_row, s_row);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t r[32];
                    tmem_ld32(lane_base + buf * 256u + 128u * half + 32u * c, r);
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const float4 cs = *reinterpret_cast<const float4 *>(sxs + 32 * c + j);
                        // scale of each column: sdy[t, n] * sx[t, k], one rounding
                        const float2 s01 = __fmul2_rn(sr2, make_float2(cs.x, cs.y));
                        const float2 s23 = __fmul2_rn(sr2, make_float2(cs.z, cs.w));
                        const float2 a01 = __ffma2_rn(s01, make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])),
                                                      make_float2(acc[32 * c + j], acc[32 * c + j + 1]));
                        const float2 a23 =
                            __ffma2_rn(s23, make_float2(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3])),
                                       make_float2(acc[32 * c + j + 2], acc[32 * c + j + 3]));
                        acc[32 * c + j] = a01.x;
                        acc[32 * c + j + 1] = a01.y;
                        acc[32 * c + j + 2] = a23.x;
                        acc[32 * c + j + 3] = a23.y;
                    }
                }
                tc_fence_before();
                mbar_arrive(tempty_bar(buf));
                // done with the stage's column scales: order these generic-proxy reads
                // before the bulk copy (async proxy) that will refill the stage (without
                // the fence a later copy was seen to land under a pending read)
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(empty_bar(stage));
                if (++stage == STAGES) { stage = 0; sphase ^= 1u; }
            }
            if (!ok) break;
            const int k = tl.k0 + 128 * half;
            if (k < K) {
                // the warp's 32 rows (n0 + 32 q ..) x this half's 128 columns as four
                // 32 x 32 fp32 TMA-store boxes from two alternating staging boxes (row r's
                // 16-byte chunk i at i ^ (r % 8): the 128-byte swizzle)
                uint8_t *stg = smem + OFF_EPI + (warp - 4) * EPI_STG;
                const uint32_t stg_s = sbase + OFF_EPI + (warp - 4) * EPI_STG;
                const int32_t drow = tl.g * N + tl.n0 + 32 * q;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t bsel = (c & 1) * EPI_BOX;
                    if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float *f = acc + 32 * c + 4 * i;
                        *reinterpret_cast<uint4 *>(stg + bsel + lane * 128 + ((i ^ (lane & 7)) << 4)) =
                            make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                                       __float_as_uint(f[3]));
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    tma_store_2d(&tmD, stg_s + bsel, k + 32 * c, drow, lane == 0 ? 1u : 0u);
                    if (lane == 0) bulk_commit();
                }
            }
        }
        // this warp's TMA stores are complete before the CTA exits
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
    }
}

static int prepare() {
    static int state[MAX_DEVICES] = {};
    static std::mutex mu;
    const int r = once_per_device(state, mu, []() {
        cudaFuncAttributes attr;
        if (cudaFuncGetAttributes(&attr, wgrad_kernel) != cudaSuccess) return -MOE_ERR_CUDA;
        if (attr.numRegs != LAUNCH_REGS) return -MOE_ERR_UNSUPPORTED;   // the setmaxnreg split needs 168
        if (cudaFuncSetAttribute(wgrad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(SMEM_BYTES)) != cudaSuccess)
            return -MOE_ERR_CUDA;
        return 1;
    });
    return r > 0 ? MOE_OK : -r;
}

}  // namespace wg
}  // namespace moe

using namespace moe;

MOE_API int fp8_quant_128x1_grouped(const void *x, int64_t M, int64_t C, int32_t G, const int32_t *group_offsets,
                                    uint8_t *q_t, int64_t p_capacity, float *scales, int64_t t_capacity,
                                    int32_t *status, void *stream) {
    if (M < 0 || C < 0 || G < 0 || p_capacity < 0 || t_capacity < 0) return MOE_ERR_INVALID_ARG;
    if (C % 128 != 0 || p_capacity % 16 != 0) return MOE_ERR_INVALID_ARG;
    if (G == 0 || C == 0 || t_capacity == 0) return MOE_OK;
    if (G > wg::MAX_G || t_capacity > 0x7fffffffLL || C / 128 > 65535) return MOE_ERR_UNSUPPORTED;
    if (!x || !group_offsets || !q_t || !scales || !aligned16(x) || !aligned16(q_t)) return MOE_ERR_INVALID_ARG;
    const int64_t cblocks = C / 128;
    dim3 grid(static_cast<unsigned>(t_capacity), static_cast<unsigned>(cblocks < 8 ? cblocks : 8), 1);
    wg::quant_128x1_kernel<<<grid, 256, 0, as_stream(stream)>>>(
        static_cast<const uint16_t *>(x), M, C, group_offsets, G, q_t, p_capacity, scales, t_capacity, status);
    return launch_status();
}

MOE_API int fp8_grouped_gemm_wgrad(int32_t G, const int32_t *group_offsets, int64_t M, int64_t N, int64_t K,
                                   const uint8_t *dy_t, const float *sdy, const uint8_t *x_t, const float *sx,
                                   int64_t p_capacity, int64_t t_capacity, float *dW, int32_t *status,
                                   void *stream) {
    using namespace moe::wg;
    if (G < 0 || M < 0 || N < 0 || K < 0 || p_capacity < 0 || t_capacity < 0) return MOE_ERR_INVALID_ARG;
    if (N % 128 != 0 || K % 128 != 0 || p_capacity % 16 != 0) return MOE_ERR_INVALID_ARG;
    if (G == 0 || N == 0 || K == 0) return MOE_OK;
    if (G > MAX_G || N > 0x7fffffffLL || K > 0x7fffffffLL || p_capacity > 0x7fffffffLL ||
        static_cast<int64_t>(G) * (N / 128) * ((K + BN - 1) / BN) > 0x7fffffffLL ||
        static_cast<int64_t>(G) * N > 0x7fffffffLL)
        return MOE_ERR_UNSUPPORTED;
    if (!group_offsets || !dy_t || !sdy || !x_t || !sx || !dW) return MOE_ERR_INVALID_ARG;
    if (p_capacity == 0) return MOE_ERR_INVALID_ARG;
    if (!aligned16(dy_t) || !aligned16(x_t) || !aligned16(sx) || !aligned16(dW) ||
        (reinterpret_cast<uintptr_t>(sdy) & 3))
        return MOE_ERR_INVALID_ARG;
    int rc = prepare();
    if (rc != MOE_OK) return rc;
    auto enc = encode_fn();
    if (!enc) return MOE_ERR_CUDA;
    CUtensorMap tmA, tmB;
    {
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(p_capacity), static_cast<cuuint64_t>(N)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(p_capacity)};
        cuuint32_t box[2] = {128, 128};
        cuuint32_t es[2] = {1, 1};
        if (enc(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(dy_t), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MOE_ERR_CUDA;
    }
    {
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(p_capacity), static_cast<cuuint64_t>(K)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(p_capacity)};
        cuuint32_t box[2] = {128, 128};
        cuuint32_t es[2] = {1, 1};
        if (enc(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(x_t), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MOE_ERR_CUDA;
    }
    CUtensorMap tmD;   // dW viewed as [G * N rows, K] fp32, stored in 32 x 32 boxes
    {
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(G) * static_cast<cuuint64_t>(N)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 4};
        cuuint32_t box[2] = {32, 32};
        cuuint32_t es[2] = {1, 1};
        if (enc(&tmD, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, dW, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MOE_ERR_CUDA;
    }
    wgrad_kernel<<<num_sms(), THREADS, SMEM_BYTES, as_stream(stream)>>>(
        tmA, tmB, tmD, group_offsets, G, M, static_cast<int>(N), static_cast<int>(K), sdy, sx, t_capacity, p_capacity, dW,
        status, wait_limit_ns());
    return launch_status();
}
