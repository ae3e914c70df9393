// Grouped FP8 (E4M3) GEMM with 1x128 / 128x128 block scales, promoted every 128
// of K, on the sm_100a tensor cores (tcgen05 + TMEM, operands staged by TMA).
//
// What it computes ("DeepSeek-V3 technical report" walkthrough (2kiu.com),
// section 4.3; the Zhihu infrastructure answer on DeepSeek-V3: per-tile 1x128
// activation scales and per-block 128x128 weight scales are not supported by the
// tensor cores, so the product is formed as partial sums that are promoted):
//   C[m, n] = sum_kb  sA[m, kb] * sB[g, n/128, kb] * P_kb[m, n],
//   P_kb    = sum_{k in kb} e4m3(A[m, k]) * e4m3(B[g, n, k])   (fp32, tensor core)
// for the rows m of group g.  Each 128-wide K block is accumulated by the tensor
// core into a fresh TMEM buffer; the epilogue warps read it (tcgen05.ld), scale it
// and add it to fp32 registers.  Two TMEM buffers (2 x 256 columns) let the
// tensor core run block kb+1 while the epilogue promotes block kb.
//
// Two variants share the code (template parameter PAIR):
//   single  one CTA per SM, tile 128 rows x 256 columns; each stage holds the A
//           tile (128 x 128 B) and the whole B tile (256 x 128 B).
//   pair    clusters of two CTAs on two SMs share one tcgen05.mma.cta_group::2
//           of M = 256: each CTA stages its own 128 rows of A and HALF of the
//           B tile (128 of 256 rows), the leader CTA issues the MMA, and each
//           CTA's TMEM receives its own 128 rows x 256 columns.  A weight tile is
//           therefore streamed once for 256 rows, and each SM moves 32 KB per K
//           block instead of 48 KB.  Transaction bytes of both CTAs' TMA loads and
//           both CTAs' TMEM releases land on the leader's barriers; the leader's
//           commits arrive on both CTAs' barriers.
//
// CTA organisation (persistent, 384 threads):
//   warp 0        TMA producer
//   warp 1        TMEM allocator and MMA issuer (the leader CTA only in the pair
//                 variant); both role warps run converged, lane 0 issues
//   warps 2-3     idle (complete warpgroup 0 for setmaxnreg)
//   warps 4-11    epilogue: warp w reads TMEM lanes 32*(w%4).., the two
//                 warpgroups split the 256 accumulator columns; at a tile's end
//                 each warp writes its 32 output rows through its own shared
//                 staging tile (TMA store when all 32 rows are the group's)
// The tile list (group-major, then N tile, then M tile so that CTAs working at
// the same time share weight tiles through L2; the last group cut into two
// chunks, see remap_tile) is derived on the device from group_offsets, so no
// host synchronisation is needed.
//
// Gather variant (template parameter GATHER, single tiles only): A is not given
// in group order but as the source rows it is made of, with a map from GEMM row
// m to source row a_map[m] (the layer's permutation: A row m of expert g is
// token tok_of[m]'s quantised activation row), so the permuted copy of the
// activations is never written.  The producer warp loads each stage's A tile
// with 32 TMA row gathers (tile::gather4), one per lane: lane l fetches tile rows
// 4l..4l+3 (their source rows read from a_map once per tile) into bytes
// 512l..512l+511 of the tile, in the same 128-byte swizzle as a tiled load.  Rows
// outside the group read source row 0 (computed, never stored).  The epilogue
// reads the A row scales through the same map.
//
// Combine variant (template parameter COMBINE, single tiles, the W2 GEMM of the
// layer): instead of storing row m, the epilogue adds c_gate[m] * bf16(C[m, :])
// into the fp32 row c_tok[m] of an output accumulator with vector reductions at
// the L2 (red.global.add.v4.f32): the gated combine of the routed rows (and, with
// gate 1, of the shared expert's rows) happens inside the GEMM, and the permuted
// rows are never written.  The additions to one output row come from different
// CTAs in no fixed order, so the fp32 sums are not reproducible bit for bit.
//
// No TMA multicast: every CTA loads its own tiles.  Every work wait is bounded
// (by default 2 s, see wait_limit_ns); on expiry the CTA raises MOE_FLAG_TIMEOUT,
// drains its own outstanding TMA loads and MMAs (waits of up to 2 s each), frees
// its TMEM and returns.
#include "tc_util.cuh"

namespace moe {
namespace gg {

using namespace moe::tc;

constexpr int BN = 256;
constexpr int BK = 128;          // bytes == e4m3 elements == one 128B swizzle row
constexpr uint32_t A_BYTES = 128 * BK;
constexpr uint32_t B_HALF = 128 * BK;
constexpr int THREADS = 384;
constexpr int EPI_THREADS = 256;
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAX_G = 4000;
constexpr uint32_t SMEM_LIMIT = 227 * 1024;   // dynamic shared memory per CTA on sm_100
constexpr int LAUNCH_REGS = 168;   // 384 threads x 168 = 128 x 40 + 256 x 232
constexpr int EPI_ROW_PITCH = 144;  // 128 data bytes + 16 pad: 16-byte staging stores without bank conflicts
constexpr uint32_t EPI_STAGE_BYTES = 8192;   // per epilogue warp: 32 rows x 256 B (TMA-store layout)
static_assert(32 * EPI_ROW_PITCH <= EPI_STAGE_BYTES, "row-store staging fits the warp's buffer");

// Row stores through the warp's shared staging buffer: each thread holds bytes of
// its own row (the warp owns 32 consecutive rows); they are written to shared
// memory row by row and read back so that consecutive lanes cover one row, so a
// global store instruction writes whole row segments (4 rows x 128 bytes, or
// 8 rows x 64 bytes) rather than 32 rows x 16 bytes.  Rows >= nvalid are not
// written.  Warp-collective.
template <int NV>   // 16-byte vectors per thread: 8 (128 bytes) or 4 (64 bytes)
__device__ __forceinline__ void warp_store_rows(uint8_t *stg, const uint4 (&v)[NV], uint8_t *dst, int64_t pitch,
                                                int nvalid, int lane) {
    static_assert(NV == 4 || NV == 8, "row chunk of 64 or 128 bytes");
    uint4 *mine = reinterpret_cast<uint4 *>(stg + lane * EPI_ROW_PITCH);
#pragma unroll
    for (int i = 0; i < NV; ++i) mine[i] = v[i];
    __syncwarp();
    constexpr int ROWS_PER_PASS = 32 / NV;   // lanes per row = NV
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int r = ROWS_PER_PASS * i + lane / NV, seg = lane % NV;
        const uint4 w = *reinterpret_cast<const uint4 *>(stg + r * EPI_ROW_PITCH + seg * 16);
        if (r < nvalid) *reinterpret_cast<uint4 *>(dst + r * pitch + seg * 16) = w;
    }
    __syncwarp();
}

template <bool PAIR>
struct Cfg {
    static constexpr int TM = PAIR ? 256 : 128;                     // rows per tile (whole pair)
    static constexpr int STAGES = PAIR ? 4 : 3;     // 3 x 48 KB: a fourth stage measured no faster
    static constexpr uint32_t STAGE_BYTES = PAIR ? A_BYTES + B_HALF : A_BYTES + 2 * B_HALF;
    static constexpr uint32_t OFF_EPI = STAGES * STAGE_BYTES;        // per epilogue warp: store staging (1 KB aligned)
    static constexpr uint32_t OFF_BARS = OFF_EPI + 8 * EPI_STAGE_BYTES;
    static constexpr uint32_t OFF_MISC = OFF_BARS + 256;             // tmem holder, abort, bad
    static constexpr uint32_t OFF_RED = OFF_MISC + 32;               // [2 parity][2 half][128] fp32
    static constexpr uint32_t OFF_MSTART = OFF_RED + 2 * 2 * 128 * 4;  // int32 [G + 1]
    // launched with smem_bytes(G) <= SMEM_LIMIT (the attribute is set once to the limit)
    static constexpr uint32_t SMEM_BYTES = SMEM_LIMIT;
    static constexpr int G_LIMIT = static_cast<int>((SMEM_LIMIT - OFF_MSTART - 1024) / 4) - 1;
    static constexpr int MAX_GROUPS = G_LIMIT < MAX_G ? G_LIMIT : MAX_G;
    static_assert(MAX_GROUPS >= 1024, "shared memory layout leaves too little room for the group table");
    static constexpr uint32_t smem_bytes(int G) { return OFF_MSTART + static_cast<uint32_t>(G + 1) * 4u + 1024u; }
    // instruction descriptor: D fp32, A/B e4m3, K-major both, N = 256, M = 128 or 256
    static constexpr uint32_t IDESC = (1u << 4) | (static_cast<uint32_t>(BN >> 3) << 17) |
                                      (static_cast<uint32_t>(TM >> 4) << 24);
    static constexpr uint32_t TEMPTY_COUNT = PAIR ? 2 * EPI_THREADS : EPI_THREADS;
};

struct Tile {
    int g, m0, m_end, nt;
};

// Tile t -> (group, first row, group end, N tile).  Group g owns the tiles
// [NT*mstart[g], NT*mstart[g+1]), ordered N-tile-major, M tile innermost.
__device__ __forceinline__ Tile decode_tile(int t, const int32_t *mstart, int G, int NT, int TM,
                                            const int32_t *__restrict__ offs) {
    int lo = 0, hi = G;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (NT * mstart[mid] <= t) lo = mid; else hi = mid;
    }
    const int mcount = mstart[lo + 1] - mstart[lo];
    const int local = t - NT * mstart[lo];
    Tile r;
    r.g = lo;
    r.nt = local / mcount;
    const int mt = local % mcount;
    r.m0 = __ldg(offs + lo) + mt * TM;
    r.m_end = __ldg(offs + lo + 1);
    return r;
}

// Tile order seen by the CTAs.  The last group's tiles (the shared expert in the
// layer: all T rows, so many M tiles per weight tile and little weight traffic
// per FLOP) are cut into C chunks of whole N columns placed evenly between the
// other groups' tiles (which stream weights), so that tensor-bound and
// HBM-bound tiles run side by side instead of one after the other.  Measured on
// B200 at the DeepSeek-V3 layer shape with C = 2: W2 1.043 -> 1.015 ms, W13
// unchanged.  R = tiles of groups 0..G-2, S = tiles of group G-1 (S % C == 0).
__device__ __forceinline__ int remap_tile(int v, int R, int S, int C) {
    if (C <= 1) return v;
    const int sc = S / C;
    for (int i = C - 1; i >= 0; --i) {
        const int rb = static_cast<int>(static_cast<long long>(i) * R / C);
        const int st = rb + i * sc;
        if (v >= st) {
            const int rlen = static_cast<int>(static_cast<long long>(i + 1) * R / C) - rb;
            const int off = v - st;
            return off < rlen ? rb + off : R + i * sc + (off - rlen);
        }
    }
    return v;
}

template <bool PAIR, bool GATHER, bool COMBINE>
__global__ void __launch_bounds__(THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC,
                    const int32_t *__restrict__ offs, int G, int64_t m_cap, int N, int K,
                    const float *__restrict__ sA, const float *__restrict__ sB, int epi,
                    void *__restrict__ C, float *__restrict__ sC, int32_t *status, uint64_t wait_ns,
                    int stall, const int32_t *__restrict__ a_map, int64_t a_rows,
                    const int32_t *__restrict__ c_tok, const float *__restrict__ c_gate, int64_t c_rows) {
    static_assert(!(PAIR && GATHER), "the gather variant runs single tiles");
    static_assert(!(PAIR && COMBINE), "the combine variant runs single tiles");
    using Cf = Cfg<PAIR>;
    constexpr int STAGES = Cf::STAGES;
    constexpr uint32_t STAGE_BYTES = Cf::STAGE_BYTES;
    constexpr int TM = Cf::TM;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
    const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    const uint32_t sbase = raw_addr + pad;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;   // 0 = leader of the pair
    const bool leader = rank == 0;
    const int unit = PAIR ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
    const int n_units = PAIR ? static_cast<int>(n_clusters_x()) : static_cast<int>(gridDim.x);

    const uint32_t bar0 = sbase + Cf::OFF_BARS;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
    auto xchg_bar = [&](int p) { return bar0 + 8u * (2 * STAGES + 5 + p); };

    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + Cf::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cf::OFF_MISC + 4);
    int *bad_flag = reinterpret_cast<int *>(smem + Cf::OFF_MISC + 8);
    float *red = reinterpret_cast<float *>(smem + Cf::OFF_RED);
    int32_t *mstart = reinterpret_cast<int32_t *>(smem + Cf::OFF_MSTART);

    const bool swiglu = epi == MOE_EPI_SWIGLU_REQUANT;
    const int I = N / 2;
    const int NT = swiglu ? I / 128 : (N + BN - 1) / BN;
    const int KB = K / BK;
    const int NB = N / 128;

    // ---- setup: per-group M-tile counts -> prefix; barriers; TMEM
    if (threadIdx.x == 0) { *abort_flag = 0; *bad_flag = 0; }
    __syncthreads();
    for (int g = threadIdx.x; g < G; g += THREADS) {
        const int a = __ldg(offs + g), b = __ldg(offs + g + 1);
        if (b < a || a < 0 || static_cast<int64_t>(b) > m_cap) *bad_flag = 1;
        mstart[g + 1] = b > a ? (b - a + TM - 1) / TM : 0;
    }
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < G; base += 32) {
            const int g = base + lane;
            int v = g < G ? mstart[g + 1] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += n;
            }
            if (g < G) mstart[g + 1] = v + carry;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) mstart[0] = 0;
    } else if (warp == 2 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(tfull_bar(b), 1); mbar_init(tempty_bar(b), Cf::TEMPTY_COUNT); }
        mbar_init(drain_bar, 1);
        for (int p = 0; p < 2; ++p) mbar_init(xchg_bar(p), EPI_THREADS);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    } else if (warp == 3 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmC)) : "memory");
    }
    if (warp == 1) {
        __syncwarp();
        if constexpr (PAIR) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             sbase + Cf::OFF_MISC),
                         "r"(TMEM_COLS)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             sbase + Cf::OFF_MISC),
                         "r"(TMEM_COLS)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();   // the peer's barriers and TMEM exist before any cross-CTA use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int num_tiles = *bad_flag ? 0 : NT * mstart[G];
    const int R_t = NT * mstart[G - 1], S_t = NT * (mstart[G] - mstart[G - 1]);
    const int C_t = (NT % 2 == 0 && mstart[G] - mstart[G - 1] >= 8) ? 2 : 1;   // chunks of the last group
    if (blockIdx.x == 0 && threadIdx.x == 0 && *bad_flag) set_flag(status, MOE_FLAG_BAD_OFFSETS);
    // the leader's barriers as seen from this CTA (its own in the single variant)
    const uint32_t lead_bar0 = PAIR ? mapa_shared(bar0, 0) : bar0;

    __syncwarp();
    if (warp < 4) {
        // warpgroup 0 gives registers away to the two epilogue warpgroups
        asm volatile("setmaxnreg.dec.sync.aligned.u32 40;" ::: "memory");
    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        // (the whole warp runs the loop; lane 0 issues)
        const uint32_t one = lane == 0 ? 1u : 0u;
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        bool ok = true;
        for (int t = unit; ok && t < num_tiles; t += n_units) {
            const Tile tl = decode_tile(remap_tile(t, R_t, S_t, C_t), mstart, G, NT, TM, offs);
            const int r0 = swiglu ? 128 * tl.nt : BN * tl.nt;            // B rows of columns 0..127
            const int r1 = swiglu ? I + 128 * tl.nt : BN * tl.nt + 128;  // B rows of columns 128..255
            const int arow = tl.m0 + 128 * static_cast<int>(rank);
            int src[4] = {0, 0, 0, 0};   // gather: source rows of tile rows 4 lane .. 4 lane + 3
            if (GATHER) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int m = tl.m0 + 4 * lane + i;
                    if (m < tl.m_end) {
                        const int v = __ldg(a_map + m);
                        if (v >= 0 && v < a_rows) src[i] = v;
                        else set_flag(status, MOE_FLAG_BAD_INDEX);
                    }
                }
            }
            for (int kb = 0; kb < KB; ++kb) {
                ok = __all_sync(0xffffffffu, mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, status, false, wait_ns));
                if (!ok) break;
                if (!PAIR && stall && blockIdx.x == 0 && t == unit && kb == 0) {
                    // test hook: CTA 0 never fills its first stage, so the MMA
                    // warp's wait for it runs out (nothing is in flight for it)
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                    continue;
                }
                const uint32_t sa = sbase + stage * STAGE_BYTES;
                if constexpr (PAIR) {
                    const uint32_t fb = lead_bar0 + 8u * stage;
                    mbar_expect_tx_if(full_bar(stage), 2 * STAGE_BYTES, leader ? one : 0u);
                    tma_load_2d_pair(sa, &tmA, kb * BK, arow, fb, one);
                    tma_load_3d_pair(sa + A_BYTES, &tmB, kb * BK, leader ? r0 : r1, tl.g, fb, one);
                } else {
                    mbar_expect_tx_if(full_bar(stage), STAGE_BYTES, one);
                    if (GATHER)
                        tma_gather4(sa + 512u * lane, &tmA, kb * BK, src[0], src[1], src[2], src[3], full_bar(stage));
                    else
                        tma_load_2d(sa, &tmA, kb * BK, arow, full_bar(stage), one);
                    tma_load_3d(sa + A_BYTES, &tmB, kb * BK, r0, tl.g, full_bar(stage), one);
                    tma_load_3d(sa + A_BYTES + B_HALF, &tmB, kb * BK, r1, tl.g, full_bar(stage), one);
                }
                __syncwarp();
                ++issued;
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
        }
        // no TMA write may land after the CTAs exit: wait for the last loads
        // (in a pair the leader's full barriers count both CTAs' bytes; a stage
        // skipped by the test hook is the oldest slot and outside this tail,
        // because `issued` counts real loads only)
        if (leader && lane == 0) {
            const int tail = issued < STAGES ? issued : STAGES;
            for (int i = 0; i < tail; ++i) {
                if (stage == 0) { stage = STAGES - 1; phase ^= 1u; } else { --stage; }
                mbar_wait(full_bar(stage), phase, abort_flag, status, true);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        // (the whole warp runs the loop; lane 0 issues)
        if (leader) {
            const uint32_t one = lane == 0 ? 1u : 0u;
            int stage = 0;
            uint32_t phase = 0, kc = 0;
            bool ok = true;
            for (int t = unit; ok && t < num_tiles; t += n_units) {
                for (int kb = 0; kb < KB; ++kb, ++kc) {
                    const uint32_t buf = kc & 1u, use = kc >> 1;
                    ok = __all_sync(0xffffffffu, mbar_wait(tempty_bar(buf), (use & 1u) ^ 1u, abort_flag, status, false, wait_ns));
                    if (!ok) break;
                    ok = __all_sync(0xffffffffu, mbar_wait(full_bar(stage), phase, abort_flag, status, false, wait_ns));
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t sa = sbase + stage * STAGE_BYTES;
                    const uint64_t ad = sw128_desc(sa), bd = sw128_desc(sa + A_BYTES);
                    const uint32_t d = tmem_base + buf * 256u;
                    if constexpr (PAIR) {
#pragma unroll
                        for (int k = 0; k < BK / 32; ++k)
                            mma_f8_pair(d, ad + 2u * k, bd + 2u * k, Cf::IDESC, k > 0 ? 1u : 0u, one);
                        mma_commit_pair(empty_bar(stage), 0x3, one);
                        mma_commit_pair(tfull_bar(buf), 0x3, one);
                    } else {
#pragma unroll
                        for (int k = 0; k < BK / 32; ++k)
                            mma_f8(d, ad + 2u * k, bd + 2u * k, Cf::IDESC, k > 0 ? 1u : 0u, one);
                        mma_commit(empty_bar(stage), one);
                        mma_commit(tfull_bar(buf), one);
                    }
                    __syncwarp();
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // every MMA of this CTA (pair) has completed before TMEM is released
            if constexpr (PAIR) mma_commit_pair(drain_bar, 0x1, one);
            else mma_commit(drain_bar, one);
            __syncwarp();
            mbar_wait(drain_bar, 0, abort_flag, status, true);
        }
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 232;" ::: "memory");
        // ------------------------------------------------------ epilogue
        const int q = warp & 3;               // TMEM lane quarter
        const int half = (warp - 4) >> 2;     // column half of the 256-wide tile
        const int row = q * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
        uint32_t kc = 0, xphase0 = 0, xphase1 = 0;
        int iter = 0;
        bool ok = true;
        for (int t = unit; ok && t < num_tiles; t += n_units, ++iter) {
            const Tile tl = decode_tile(remap_tile(t, R_t, S_t, C_t), mstart, G, NT, TM, offs);
            const int64_t grow = static_cast<int64_t>(tl.m0) + 128 * static_cast<int>(rank) + row;
            int64_t arow = grow;          // row of A (and sA) this output row is made of
            if (GATHER) {
                arow = -1;
                if (grow < tl.m_end) {
                    const int v = __ldg(a_map + grow);
                    if (v >= 0 && v < a_rows) arow = v;
                }
            }
            const bool row_ok = GATHER ? arow >= 0 : grow < m_cap;
            const float *sa_row = sA + (row_ok ? arow : 0) * KB;
            // scale rows of B for the two column halves of this thread
            int nb0, nb1;
            bool nb1_ok = true;
            if (swiglu) { nb0 = tl.nt; nb1 = I / 128 + tl.nt; }
            else { nb0 = 2 * tl.nt + half; nb1 = nb0; nb1_ok = nb0 < NB; }
            const float *sb0 = sB + (static_cast<int64_t>(tl.g) * NB + (nb1_ok ? nb0 : 0)) * KB;
            const float *sb1 = sB + (static_cast<int64_t>(tl.g) * NB + (nb1_ok ? nb1 : 0)) * KB;
            float acc[128];
#pragma unroll
            for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
            // the three scales of K block kb + 1 are loaded while block kb is promoted
            float na = row_ok ? __ldg(sa_row) : 0.0f;
            float nb0v = nb1_ok ? __ldg(sb0) : 0.0f, nb1v = nb1_ok ? __ldg(sb1) : 0.0f;
            for (int kb = 0; kb < KB; ++kb, ++kc) {
                const float s0 = __fmul_rn(na, nb0v);
                const float s1 = __fmul_rn(na, nb1v);
                if (kb + 1 < KB) {
                    na = row_ok ? __ldg(sa_row + kb + 1) : 0.0f;
                    nb0v = nb1_ok ? __ldg(sb0 + kb + 1) : 0.0f;
                    nb1v = nb1_ok ? __ldg(sb1 + kb + 1) : 0.0f;
                }
                const uint32_t buf = kc & 1u, use = kc >> 1;
                if (!__all_sync(0xffffffffu, mbar_wait(tfull_bar(buf), use & 1u, abort_flag, status, false, wait_ns))) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    // SwiGLU: chunks 0,1 gate columns 64*half + 32c; chunks 2,3 up columns 128 + 64*half + 32(c-2)
                    // plain : chunk c columns 128*half + 32c
                    const uint32_t col = swiglu ? (c < 2 ? 64u * half + 32u * c : 128u + 64u * half + 32u * (c - 2))
                                                : 128u * half + 32u * c;
                    uint32_t r[32];
                    tmem_ld32(lane_base + buf * 256u + col, r);
                    const float sc = (swiglu && c >= 2) ? s1 : s0;
                    const float2 sc2 = make_float2(sc, sc);
                    // packed dual fp32 FMA: the same round-to-nearest FMA per element, half the issues
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        const float2 a2 = __ffma2_rn(sc2, make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])),
                                                     make_float2(acc[32 * c + j], acc[32 * c + j + 1]));
                        acc[32 * c + j] = a2.x;
                        acc[32 * c + j + 1] = a2.y;
                    }
                }
                tc_fence_before();
                if constexpr (PAIR) mbar_arrive_cluster(lead_bar0 + 8u * (2 * STAGES + 2 + buf));
                else mbar_arrive(tempty_bar(buf));
            }
            if (!ok) break;
            const bool store_row = grow < tl.m_end;
            // this warp's 32 rows start at wrow0; the first nvalid of them belong to the group
            const int64_t wrow0 = static_cast<int64_t>(tl.m0) + 128 * static_cast<int>(rank) + 32 * q;
            const int64_t left = static_cast<int64_t>(tl.m_end) - wrow0;
            const int nvalid = left <= 0 ? 0 : (left >= 32 ? 32 : static_cast<int>(left));
            uint8_t *stg = smem + Cf::OFF_EPI + (warp - 4) * EPI_STAGE_BYTES;
            const uint32_t stg_s = sbase + Cf::OFF_EPI + (warp - 4) * EPI_STAGE_BYTES;
            // a warp whose 32 rows all belong to the group stores them with TMA from
            // a swizzled staging tile; others store row segments themselves.  Either
            // way the staging buffer is reused only after the previous TMA store of
            // this warp has read it.
            const bool full_warp = nvalid == 32;
            if (lane == 0) bulk_wait_read();
            __syncwarp();
            if (COMBINE) {
                // the gated row, bf16-rounded as a stored expert row would be, added into
                // its token's fp32 output row
                const int64_t n0 = static_cast<int64_t>(tl.nt) * BN + 128 * half;
                if (n0 < N && store_row) {
                    const int tok = __ldg(c_tok + grow);
                    const float gate = __ldg(c_gate + grow);
                    if (tok >= 0 && tok < c_rows) {
                        float *dst = reinterpret_cast<float *>(C) + static_cast<int64_t>(tok) * N + n0;
#pragma unroll
                        for (int j = 0; j < 128; j += 4) {
                            float v[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                v[q] = __fmul_rn(gate, __bfloat162float(__float2bfloat16_rn(acc[j + q])));
                            red_add_f32x4(dst + j, v[0], v[1], v[2], v[3]);
                        }
                    } else {
                        set_flag(status, MOE_FLAG_BAD_INDEX);
                    }
                }
            } else if (!swiglu) {
                const int64_t n0 = static_cast<int64_t>(tl.nt) * BN + 128 * half;
                if (n0 < N) {
                    if (epi == MOE_EPI_BF16) {
                        uint8_t *dst = reinterpret_cast<uint8_t *>(C) + (wrow0 * N + n0) * 2;
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            uint4 v[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float *f = acc + 64 * c + 8 * i;
                                __nv_bfloat162 p0 = __floats2bfloat162_rn(f[0], f[1]);
                                __nv_bfloat162 p1 = __floats2bfloat162_rn(f[2], f[3]);
                                __nv_bfloat162 p2 = __floats2bfloat162_rn(f[4], f[5]);
                                __nv_bfloat162 p3 = __floats2bfloat162_rn(f[6], f[7]);
                                v[i] = make_uint4(*reinterpret_cast<uint32_t *>(&p0), *reinterpret_cast<uint32_t *>(&p1),
                                                  *reinterpret_cast<uint32_t *>(&p2), *reinterpret_cast<uint32_t *>(&p3));
                            }
                            if (full_warp) {
                                // box c: 32 rows x 128 B, 128-byte swizzle (chunk i of row r at i ^ (r % 8))
#pragma unroll
                                for (int i = 0; i < 8; ++i)
                                    *reinterpret_cast<uint4 *>(stg + c * 4096 + lane * 128 + ((i ^ (lane & 7)) << 4)) = v[i];
                            } else {
                                warp_store_rows<8>(stg, v, dst + 128 * c, 2 * static_cast<int64_t>(N), nvalid, lane);
                            }
                        }
                        if (full_warp) {
                            fence_proxy_async_smem();
                            __syncwarp();
                            const uint32_t one = lane == 0 ? 1u : 0u;
                            tma_store_2d(&tmC, stg_s, static_cast<int32_t>(n0), static_cast<int32_t>(wrow0), one);
                            tma_store_2d(&tmC, stg_s + 4096, static_cast<int32_t>(n0 + 64), static_cast<int32_t>(wrow0), one);
                            if (lane == 0) bulk_commit();
                        }
                    } else {
                        uint8_t *dst = reinterpret_cast<uint8_t *>(C) + (wrow0 * N + n0) * 4;
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            uint4 v[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float *f = acc + 32 * c + 4 * i;
                                v[i] = make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                                                  __float_as_uint(f[3]));
                            }
                            warp_store_rows<8>(stg, v, dst + 128 * c, 4 * static_cast<int64_t>(N), nvalid, lane);
                        }
                    }
                }
            } else {
                // act = silu(g) * u on this thread's 64 columns, amax over the full
                // 128-column tile via the partner warpgroup (same row, other half)
                // eight independent running maxima (max is exact in any order), so
                // the 64 steps do not form one dependency chain
                float am[8];
                bool fn[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) { am[i] = 0.0f; fn[i] = true; }
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    acc[j] = swiglu_act(acc[j], acc[64 + j]);
                    amax_step(acc[j], am[j & 7], fn[j & 7]);
                }
                float amax = am[0];
                bool fin = fn[0];
#pragma unroll
                for (int i = 1; i < 8; ++i) { amax = fmaxf(amax, am[i]); fin = fin && fn[i]; }
                const int p = iter & 1;
                float *rp = red + p * 256;
                rp[half * 128 + row] = fin ? amax : __int_as_float(0x7fc00000);
                mbar_arrive(xchg_bar(p));
                uint32_t &xph = p ? xphase1 : xphase0;
                // warp-uniform outcome: the staged store below is warp-collective
                if (!__all_sync(0xffffffffu, mbar_wait(xchg_bar(p), xph, abort_flag, status, false, wait_ns))) { ok = false; break; }
                xph ^= 1u;
                const float mine = rp[half * 128 + row], other = rp[(half ^ 1) * 128 + row];
                const bool finite = !isnan(mine) && !isnan(other);
                const float sc = tile_scale(fmaxf(mine, other), finite);
                const float inv = __frcp_rn(sc);
                // codes of fp32(act * (1/scale)): within 1.5 fp32 ulps of the
                // correctly rounded quotient, so a code can differ from the
                // division rule's only where act/scale lies that close to an E4M3
                // rounding boundary (the exact quotient would double the cost of
                // this tile-end step on the critical path)
                uint4 v[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float *f = acc + 16 * i;
                    v[i] = finite ? make_uint4(e4m3x2_rcp(f[0], f[1], inv) | e4m3x2_rcp(f[2], f[3], inv) << 16,
                                               e4m3x2_rcp(f[4], f[5], inv) | e4m3x2_rcp(f[6], f[7], inv) << 16,
                                               e4m3x2_rcp(f[8], f[9], inv) | e4m3x2_rcp(f[10], f[11], inv) << 16,
                                               e4m3x2_rcp(f[12], f[13], inv) | e4m3x2_rcp(f[14], f[15], inv) << 16)
                                  : make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
                }
                if (full_warp) {
                    // one box of 32 rows x 64 B, 64-byte swizzle (chunk i of row r at i ^ ((r / 2) % 4))
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        *reinterpret_cast<uint4 *>(stg + lane * 64 + ((i ^ ((lane >> 1) & 3)) << 4)) = v[i];
                    fence_proxy_async_smem();
                    __syncwarp();
                    tma_store_2d(&tmC, stg_s, 128 * tl.nt + 64 * half, static_cast<int32_t>(wrow0), lane == 0 ? 1u : 0u);
                    if (lane == 0) bulk_commit();
                } else {
                    warp_store_rows<4>(stg, v, reinterpret_cast<uint8_t *>(C) + wrow0 * I + 128 * tl.nt + 64 * half,
                                       static_cast<int64_t>(I), nvalid, lane);
                }
                if (store_row && half == 0) {
                    sC[grow * (I / 128) + tl.nt] = sc;
                    if (!finite) set_flag(status, MOE_FLAG_NONFINITE);
                }
            }
        }
        // this warp's TMA stores are complete before the CTA exits
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    // the leader's MMAs into the peer's TMEM, the peer's TMA bytes and TMEM
    // releases on the leader's barriers: all done before either CTA frees or exits
    if constexpr (PAIR) cluster_sync();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        if constexpr (PAIR)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                         : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                         : "memory");
    }
}

// Once per device and kernel variant: check the register split and raise the
// dynamic shared-memory limit.  Returns a moe_status.
template <bool PAIR, bool GATHER, bool COMBINE>
static int prepare_kernel() {
    static int state[MAX_DEVICES] = {};
    static std::mutex mu;
    const int r = once_per_device(state, mu, []() {
        cudaFuncAttributes attr;
        if (cudaFuncGetAttributes(&attr, grouped_gemm_kernel<PAIR, GATHER, COMBINE>) != cudaSuccess)
            return -MOE_ERR_CUDA;
        // setmaxnreg moves registers inside the launch's allotment: the split
        // 128 x 40 + 256 x 232 must equal 384 x (registers at launch)
        if (attr.numRegs != LAUNCH_REGS) return -MOE_ERR_UNSUPPORTED;
        if (cudaFuncSetAttribute(grouped_gemm_kernel<PAIR, GATHER, COMBINE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(Cfg<PAIR>::SMEM_BYTES)) != cudaSuccess)
            return -MOE_ERR_CUDA;
        return 1;
    });
    return r > 0 ? MOE_OK : -r;
}

// Co-resident CTA pairs for one wave of the persistent pair kernel (per device).
static int pair_clusters() {
    static int state[MAX_DEVICES] = {};
    static std::mutex mu;
    return once_per_device(state, mu, []() {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(num_sms() / 2 * 2), 1, 1);
        cfg.blockDim = dim3(THREADS, 1, 1);
        cfg.dynamicSmemBytes = Cfg<true>::SMEM_BYTES;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, grouped_gemm_kernel<true, false, false>, &cfg) == cudaSuccess && n > 0)
            return n;
        return num_sms() / 2;
    });
}

// Both public entry points.  a_map == nullptr: A is [m_capacity, K] in group
// order (TMA loads); otherwise A is [a_rows, K] and GEMM row m reads A row
// a_map[m] (gather variant, single tiles).
static int grouped_gemm(int32_t G, const int32_t *group_offsets, int64_t m_capacity, int64_t N, int64_t K,
                        const uint8_t *A, const float *sA, const int32_t *a_map, int64_t a_rows, const uint8_t *B,
                        const float *sB, int32_t epilogue, void *C, float *sC, int32_t *status, void *stream,
                        const int32_t *c_tok = nullptr, const float *c_gate = nullptr, int64_t c_rows = 0) {
    const bool gather = a_map != nullptr;
    const bool combine = c_tok != nullptr;
    if (gather && combine) return MOE_ERR_UNSUPPORTED;
    // tile mode: one-SM tiles unless CTA pairs are asked for (measured on B200:
    // pairs are 25 % slower at 128 tokens per expert, where 256-row tiles are
    // mostly padding, and about 1 % faster at 1024 tokens per expert)
    const bool single = gather || combine || (epilogue & MOE_GEMM_PAIR_CTA) == 0 ||
                        (epilogue & MOE_GEMM_SINGLE_CTA) != 0;
    epilogue &= ~(MOE_GEMM_SINGLE_CTA | MOE_GEMM_PAIR_CTA);
    if (G < 0 || m_capacity < 0 || N < 0 || K < 0 || a_rows < 0 || c_rows < 0) return MOE_ERR_INVALID_ARG;
    if (N % 128 != 0 || K % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (combine ? epilogue != MOE_EPI_COMBINE_F32
                : (epilogue != MOE_EPI_BF16 && epilogue != MOE_EPI_F32 && epilogue != MOE_EPI_SWIGLU_REQUANT))
        return MOE_ERR_INVALID_ARG;
    if (epilogue == MOE_EPI_SWIGLU_REQUANT && (N % 256 != 0 || !sC)) return MOE_ERR_INVALID_ARG;
    if (G == 0 || m_capacity == 0 || N == 0) return MOE_OK;
    if (K == 0) return MOE_ERR_UNSUPPORTED;   // an empty reduction is not a GEMM this kernel runs
    if (gather && a_rows == 0) return MOE_ERR_INVALID_ARG;
    if (combine && (c_rows == 0 || !c_gate || (reinterpret_cast<uintptr_t>(c_tok) & 3) ||
                    (reinterpret_cast<uintptr_t>(c_gate) & 3) || c_rows > 0x7fffffffLL))
        return MOE_ERR_INVALID_ARG;
    const int max_groups = single ? Cfg<false>::MAX_GROUPS : Cfg<true>::MAX_GROUPS;
    if (G > max_groups || m_capacity > 0x7fffffffLL || N > 0x7fffffffLL || K > 0x7fffffffLL ||
        a_rows > 0x7fffffffLL)
        return MOE_ERR_UNSUPPORTED;
    if (!group_offsets || !A || !sA || !B || !sB || !C) return MOE_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(B) || !aligned16(C) || (reinterpret_cast<uintptr_t>(sA) & 3) ||
        (reinterpret_cast<uintptr_t>(sB) & 3) || (sC && (reinterpret_cast<uintptr_t>(sC) & 3)) ||
        (reinterpret_cast<uintptr_t>(a_map) & 3))
        return MOE_ERR_INVALID_ARG;
    int rc = gather ? prepare_kernel<false, true, false>()
             : combine ? prepare_kernel<false, false, true>()
             : single ? prepare_kernel<false, false, false>() : prepare_kernel<true, false, false>();
    if (rc != MOE_OK) return rc;
    auto enc = encode_fn();
    if (!enc) return MOE_ERR_CUDA;

    CUtensorMap tmA, tmB, tmC;
    if (!gather) {
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(m_capacity)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
        cuuint32_t box[2] = {128, 128};
        cuuint32_t es[2] = {1, 1};
        if (enc(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(A), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MOE_ERR_CUDA;
    }
    // 256-byte L2 promotion of weight rows: measured on B200 at the layer shapes, it
    // makes the K = 7168 GEMM 2 % faster and makes the K = 2048 GEMM fetch 0.65 GB
    // it never uses (1.5 % slower), so long rows only
    const CUtensorMapL2promotion b_promotion =
        K >= 4096 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_NONE;
    {
        cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(G)};
        cuuint64_t strides[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N * K)};
        cuuint32_t box[3] = {128, 128, 1};
        cuuint32_t es[3] = {1, 1, 1};
        if (enc(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(B), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, b_promotion,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MOE_ERR_CUDA;
    }
    // output tiles stored by TMA from the epilogue: bf16 rows in boxes of 32 rows x
    // 64 columns (128-byte swizzle), SwiGLU codes in boxes of 32 rows x 64 columns
    // (64-byte swizzle); the fp32 epilogue stores directly (tmC unused)
    if (gather) {
        // source rows of A, gathered four at a time: box one row high
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(a_rows)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
        cuuint32_t box[2] = {128, 1};
        cuuint32_t es[2] = {1, 1};
        if (enc(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(A), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MOE_ERR_CUDA;
    }
    if (epilogue == MOE_EPI_F32 || epilogue == MOE_EPI_COMBINE_F32) {
        tmC = tmA;   // unused: these epilogues write without TMA
    } else {
        const bool codes = epilogue == MOE_EPI_SWIGLU_REQUANT;
        const int64_t cols = codes ? N / 2 : N;
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(m_capacity)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(codes ? cols : 2 * cols)};
        cuuint32_t box[2] = {64, 32};
        cuuint32_t es[2] = {1, 1};
        if (enc(&tmC, codes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, C, dims, strides,
                box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                codes ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MOE_ERR_CUDA;
    }
    cudaStream_t st = as_stream(stream);
    const int n = static_cast<int>(N), k = static_cast<int>(K);
    const uint64_t wait_ns = wait_limit_ns();
    const int stall = test_stall() ? 1 : 0;
    if (gather) {
        grouped_gemm_kernel<false, true, false><<<num_sms(), THREADS, Cfg<false>::smem_bytes(G), st>>>(
            tmA, tmB, tmC, group_offsets, G, m_capacity, n, k, sA, sB, epilogue, C, sC, status, wait_ns, stall,
            a_map, a_rows, nullptr, nullptr, 0);
        return launch_status();
    }
    if (combine) {
        grouped_gemm_kernel<false, false, true><<<num_sms(), THREADS, Cfg<false>::smem_bytes(G), st>>>(
            tmA, tmB, tmC, group_offsets, G, m_capacity, n, k, sA, sB, epilogue, C, sC, status, wait_ns, stall,
            nullptr, 0, c_tok, c_gate, c_rows);
        return launch_status();
    }
    if (single) {
        grouped_gemm_kernel<false, false, false><<<num_sms(), THREADS, Cfg<false>::smem_bytes(G), st>>>(
            tmA, tmB, tmC, group_offsets, G, m_capacity, n, k, sA, sB, epilogue, C, sC, status, wait_ns, stall,
            nullptr, 0, nullptr, nullptr, 0);
        return launch_status();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pair_clusters()), 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = Cfg<true>::smem_bytes(G);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<true, false, false>, tmA, tmB, tmC, group_offsets, G, m_capacity,
                           n, k, sA, sB, static_cast<int>(epilogue), C, sC, status, wait_ns, 0,
                           static_cast<const int32_t *>(nullptr), static_cast<int64_t>(0),
                           static_cast<const int32_t *>(nullptr), static_cast<const float *>(nullptr),
                           static_cast<int64_t>(0)) != cudaSuccess)
        return MOE_ERR_CUDA;
    return launch_status();
}

}  // namespace gg
}  // namespace moe

using namespace moe;

MOE_API int fp8_grouped_gemm_blockscaled(int32_t G, const int32_t *group_offsets, int64_t m_capacity,
                                         int64_t N, int64_t K, const uint8_t *A, const float *sA,
                                         const uint8_t *B, const float *sB, int32_t epilogue, void *C,
                                         float *sC, int32_t *status, void *stream) {
    return gg::grouped_gemm(G, group_offsets, m_capacity, N, K, A, sA, nullptr, 0, B, sB, epilogue, C, sC, status,
                            stream);
}

MOE_API int fp8_grouped_gemm_blockscaled_gather(int32_t G, const int32_t *group_offsets, int64_t m_capacity,
                                                int64_t N, int64_t K, const uint8_t *A, const float *sA,
                                                int64_t a_rows, const int32_t *a_map, const uint8_t *B,
                                                const float *sB, int32_t epilogue, void *C, float *sC,
                                                int32_t *status, void *stream) {
    if (!a_map) return MOE_ERR_INVALID_ARG;
    return gg::grouped_gemm(G, group_offsets, m_capacity, N, K, A, sA, a_map, a_rows, B, sB, epilogue, C, sC, status,
                            stream);
}

MOE_API int fp8_grouped_gemm_blockscaled_combine(int32_t G, const int32_t *group_offsets, int64_t m_capacity,
                                                 int64_t N, int64_t K, const uint8_t *A, const float *sA,
                                                 const uint8_t *B, const float *sB, const int32_t *row_token,
                                                 const float *row_gate, int64_t out_rows, float *out_f32,
                                                 int32_t *status, void *stream) {
    if (!row_token) return MOE_ERR_INVALID_ARG;
    return gg::grouped_gemm(G, group_offsets, m_capacity, N, K, A, sA, nullptr, 0, B, sB, MOE_EPI_COMBINE_F32,
                            out_f32, nullptr, status, stream, row_token, row_gate, out_rows);
}
