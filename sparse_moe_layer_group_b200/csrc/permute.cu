// Dispatch: stable counting sort of the (token, slot) pairs by expert and the
// gather of the quantised token rows into per-expert segments.
//
// The pages give the semantics (every token reaches all K of its experts, no
// capacity factor and no dropping: "DeepSeek-V3 technical report" walkthrough
// (2kiu.com), sections 3.2 and 3.4; dispatch -> expert MLP -> combine, section
// 4.1) but no layout.  Layout: experts in ascending order, each expert's rows in
// ascending token order, which makes the result deterministic.
//
// Four launches, no atomics on the data path and no inter-CTA spin-waits:
//   count   CTA b (a chunk of PERM_CHUNK tokens), thread e: #pairs of e in chunk b
//   scan    one CTA: per-expert prefix over chunks, load, exclusive offsets
//   place   CTA b, thread e: walks its chunk in (t, k) order, writes maps
//   gather  one CTA per token: reads the token's e4m3 row and scales once and
//           writes them to its K rows (16-byte vectors)
// Scratch: ws holds counts[n_chunks][E] int32.
#include "common.cuh"

namespace moe {

constexpr int PERM_CHUNK = 32;
constexpr int PERM_MAX_E = 1024;

__global__ void perm_count_kernel(const int32_t *__restrict__ idx, int32_t *__restrict__ counts, int T,
                                  int K, int E, int32_t *status) {
    extern __shared__ int32_t chunk[];   // PERM_CHUNK * K
    const int b = blockIdx.x;
    const int t0 = b * PERM_CHUNK;
    const int n = min(PERM_CHUNK, T - t0) * K;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int v = idx[static_cast<int64_t>(t0) * K + i];
        if (v < 0 || v >= E) set_flag(status, MOE_FLAG_BAD_INDEX);
        chunk[i] = v;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c = 0;
        for (int i = 0; i < n; ++i) c += chunk[i] == e;
        counts[static_cast<int64_t>(b) * E + e] = c;
    }
}

// One CTA of SCAN_THREADS threads.  Thread (p, e) owns expert e's chunks
// [p*n/P, (p+1)*n/P): pass 1 sums them (loads batched), the P partial sums of
// each expert are scanned in shared memory, pass 2 writes the exclusive
// per-chunk prefixes.  Then the per-expert totals are scanned into offsets.
constexpr int SCAN_THREADS = 1024;

__global__ void __launch_bounds__(SCAN_THREADS) perm_scan_kernel(int32_t *__restrict__ counts, int n_chunks,
                                                                 int E, int P, int32_t *__restrict__ load,
                                                                 int32_t *__restrict__ offsets) {
    __shared__ int32_t part[SCAN_THREADS];
    __shared__ int32_t sums[PERM_MAX_E];
    const int tid = threadIdx.x;
    const int Ep = blockDim.x / P;             // experts per pass (>= E)
    const int e = tid % Ep, p = tid / Ep;
    const int per = (n_chunks + P - 1) / P;
    const int b0 = p * per, b1 = min(n_chunks, b0 + per);
    int local = 0;
    if (e < E) {
        int b = b0;
        for (; b + 8 <= b1; b += 8) {
            int v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = counts[static_cast<int64_t>(b + u) * E + e];
#pragma unroll
            for (int u = 0; u < 8; ++u) local += v[u];
        }
        for (; b < b1; ++b) local += counts[static_cast<int64_t>(b) * E + e];
    }
    part[tid] = local;
    __syncthreads();
    // exclusive prefix over p for this expert (P is small)
    int run = 0;
    for (int pp = 0; pp < p; ++pp) run += part[pp * Ep + e];
    if (e < E) {
        int b = b0;
        for (; b + 8 <= b1; b += 8) {
            int v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = counts[static_cast<int64_t>(b + u) * E + e];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                counts[static_cast<int64_t>(b + u) * E + e] = run;
                run += v[u];
            }
        }
        for (; b < b1; ++b) {
            const int c = counts[static_cast<int64_t>(b) * E + e];
            counts[static_cast<int64_t>(b) * E + e] = run;
            run += c;
        }
        if (p == P - 1) load[e] = run;
    }
    __syncthreads();
    // exclusive scan of the expert totals into offsets (totals = last pass's run)
    if (tid < Ep) sums[tid] = 0;
    __syncthreads();
    if (p == P - 1 && e < E) sums[e] = run;
    __syncthreads();
    for (int o = 1; o < Ep; o <<= 1) {
        const int v = (tid < Ep && tid >= o) ? sums[tid - o] : 0;
        __syncthreads();
        if (tid < Ep) sums[tid] += v;
        __syncthreads();
    }
    if (tid < E) offsets[tid + 1] = sums[tid];
    if (tid == 0) offsets[0] = 0;
}

__global__ void perm_place_kernel(const int32_t *__restrict__ idx, const int32_t *__restrict__ counts,
                                  const int32_t *__restrict__ offsets, int32_t *__restrict__ tok_of,
                                  int32_t *__restrict__ row_of, int T, int K, int E) {
    extern __shared__ int32_t chunk[];
    const int b = blockIdx.x;
    const int t0 = b * PERM_CHUNK;
    const int n = min(PERM_CHUNK, T - t0) * K;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int v = idx[static_cast<int64_t>(t0) * K + i];
        chunk[i] = v;
        if (v < 0 || v >= E) row_of[static_cast<int64_t>(t0) * K + i] = -1;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int row = offsets[e] + counts[static_cast<int64_t>(b) * E + e];
        for (int i = 0; i < n; ++i) {
            if (chunk[i] != e) continue;
            tok_of[row] = t0 + i / K;
            row_of[static_cast<int64_t>(t0) * K + i] = row;
            ++row;
        }
    }
}

// One CTA per token: H/16 16-byte vectors of codes plus H/128 scales.
constexpr int GATHER_V = 4;
__global__ void __launch_bounds__(128) perm_gather_kernel(const uint4 *__restrict__ xq,
                                                          const float *__restrict__ xs,
                                                          const int32_t *__restrict__ row_of,
                                                          uint4 *__restrict__ aq, float *__restrict__ as,
                                                          int H, int K) {
    const int t = blockIdx.x;
    __shared__ int32_t rows[32];
    if (threadIdx.x < K) rows[threadIdx.x] = row_of[static_cast<int64_t>(t) * K + threadIdx.x];
    __syncthreads();
    const int nv = H / 16;
    const uint4 *src = xq + static_cast<int64_t>(t) * nv;
    // issue GATHER_V loads per thread before any store, then fan each out to the K rows
    for (int v0 = threadIdx.x; v0 < nv; v0 += GATHER_V * blockDim.x) {
        uint4 d[GATHER_V];
#pragma unroll
        for (int u = 0; u < GATHER_V; ++u) {
            const int v = v0 + u * blockDim.x;
            d[u] = v < nv ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
        }
        for (int k = 0; k < K; ++k) {
            const int r = rows[k];
            if (r < 0) continue;
            uint4 *dst = aq + static_cast<int64_t>(r) * nv;
#pragma unroll
            for (int u = 0; u < GATHER_V; ++u) {
                const int v = v0 + u * blockDim.x;
                if (v < nv) dst[v] = d[u];
            }
        }
    }
    const int ns = H / 128;
    for (int j = threadIdx.x; j < ns * K; j += blockDim.x) {
        const int k = j / ns, c = j % ns;
        const int r = rows[k];
        if (r >= 0) as[static_cast<int64_t>(r) * ns + c] = __ldg(xs + static_cast<int64_t>(t) * ns + c);
    }
}

size_t permute_workspace_bytes(const moe_dims *d) {
    const size_t n_chunks = (static_cast<size_t>(d->T) + PERM_CHUNK - 1) / PERM_CHUNK;
    return (n_chunks * d->E * sizeof(int32_t) + 255) & ~static_cast<size_t>(255);
}

static inline int threads_for(int E) {
    int t = ((E + 31) / 32) * 32;
    return t < 32 ? 32 : t;
}

}  // namespace moe

using namespace moe;

MOE_API int moe_permute(const moe_dims *d, const int32_t *topk_idx, const uint8_t *xq, const float *xs,
                        int32_t *expert_load, int32_t *expert_offsets, int32_t *tok_of, int32_t *row_of,
                        uint8_t *aq, float *as, void *ws, size_t ws_bytes, int32_t *status, void *stream) {
    if (!d || d->T < 0 || d->E <= 0 || d->K <= 0 || d->H < 0) return MOE_ERR_INVALID_ARG;
    if (d->E > PERM_MAX_E || d->K > 32) return MOE_ERR_UNSUPPORTED;
    if (!expert_load || !expert_offsets) return MOE_ERR_INVALID_ARG;
    const bool gather = xq || xs || aq || as;
    if (gather && (!xq || !xs || !aq || !as || d->H % 128 != 0 || !aligned16(xq) || !aligned16(aq)))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    if (d->T == 0) {
        // empty batch: zero loads and offsets
        if (cudaMemsetAsync(expert_load, 0, sizeof(int32_t) * d->E, st) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (d->E + 1), st) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (!topk_idx || !tok_of || !row_of) return MOE_ERR_INVALID_ARG;
    if (!ws || ws_bytes < permute_workspace_bytes(d)) return MOE_ERR_WORKSPACE;
    int32_t *counts = reinterpret_cast<int32_t *>(ws);
    const int n_chunks = (d->T + PERM_CHUNK - 1) / PERM_CHUNK;
    const int thr = threads_for(d->E);
    const size_t smem = static_cast<size_t>(PERM_CHUNK) * d->K * sizeof(int32_t);
    perm_count_kernel<<<n_chunks, thr, smem, st>>>(topk_idx, counts, d->T, d->K, d->E, status);
    {
        const int P = SCAN_THREADS / thr;      // chunk partitions per expert
        perm_scan_kernel<<<1, P * thr, 0, st>>>(counts, n_chunks, d->E, P, expert_load, expert_offsets);
    }
    perm_place_kernel<<<n_chunks, thr, smem, st>>>(topk_idx, counts, expert_offsets, tok_of, row_of, d->T,
                                                  d->K, d->E);
    if (gather && d->H > 0)
        perm_gather_kernel<<<d->T, 128, 0, st>>>(reinterpret_cast<const uint4 *>(xq), xs, row_of,
                                                reinterpret_cast<uint4 *>(aq), as, d->H, d->K);
    return launch_status();
}

// ---------------------------------------------------------------------------
// moe_permute_noalloc: the same permutation for callers that cannot allocate
// device memory.  Its per-chunk expert counts live in the file-scope array
// below instead of a caller workspace.  The array is a fixed part of every
// device image of this library, so each GPU that loads the library holds its
// 1 MiB until the process exits.
// ---------------------------------------------------------------------------
#include <mutex>

namespace moe {

constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(1) << 20;   // 1 MiB: counts[ceil(T/32)][E] int32
constexpr int NOALLOC_MAX_DEVICES = 64;

static __device__ __align__(256) int32_t g_perm_noalloc_scratch[NOALLOC_SCRATCH_BYTES / sizeof(int32_t)];

// Device address of the scratch array, looked up once per device.  In host code
// g_perm_noalloc_scratch names a host-side stand-in, not device memory, so the
// kernels must be given the address cudaGetSymbolAddress returns.
static int noalloc_scratch(int32_t **out) {
    static std::mutex mu;
    static int32_t *addr[NOALLOC_MAX_DEVICES] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= NOALLOC_MAX_DEVICES) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_perm_noalloc_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
        addr[dev] = static_cast<int32_t *>(p);
    }
    *out = addr[dev];
    return MOE_OK;
}

}  // namespace moe

MOE_API size_t moe_permute_noalloc_max_scratch(void) { return moe::NOALLOC_SCRATCH_BYTES; }

MOE_API int moe_permute_noalloc(const moe_dims *d, const int32_t *topk_idx, const uint8_t *xq, const float *xs,
                                int32_t *expert_load, int32_t *expert_offsets, int32_t *tok_of,
                                int32_t *row_of, uint8_t *aq, float *as, int32_t *status, void *stream) {
    if (!d || d->T < 0 || d->E <= 0 || d->K <= 0 || d->H < 0) return MOE_ERR_INVALID_ARG;
    if (d->E > PERM_MAX_E || d->K > 32) return MOE_ERR_UNSUPPORTED;
    if (!expert_load || !expert_offsets) return MOE_ERR_INVALID_ARG;
    const bool gather = xq || xs || aq || as;
    if (gather && (!xq || !xs || !aq || !as || d->H % 128 != 0 || !aligned16(xq) || !aligned16(aq)))
        return MOE_ERR_INVALID_ARG;
    // the per-chunk counts must fit the static scratch
    if (permute_workspace_bytes(d) > NOALLOC_SCRATCH_BYTES) return MOE_ERR_TOO_LARGE;
    int32_t *counts = nullptr;
    int rc = noalloc_scratch(&counts);
    if (rc != MOE_OK) return rc;
    cudaStream_t st = as_stream(stream);
    if (d->T == 0) {
        if (cudaMemsetAsync(expert_load, 0, sizeof(int32_t) * d->E, st) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (d->E + 1), st) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (!topk_idx || !tok_of || !row_of) return MOE_ERR_INVALID_ARG;
    // every count the later kernels read is written by perm_count_kernel first
    // in this call, so the scratch needs no clearing between calls
    const int n_chunks = (d->T + PERM_CHUNK - 1) / PERM_CHUNK;
    const int thr = threads_for(d->E);
    const size_t smem = static_cast<size_t>(PERM_CHUNK) * d->K * sizeof(int32_t);
    perm_count_kernel<<<n_chunks, thr, smem, st>>>(topk_idx, counts, d->T, d->K, d->E, status);
    {
        const int P = SCAN_THREADS / thr;      // chunk partitions per expert
        perm_scan_kernel<<<1, P * thr, 0, st>>>(counts, n_chunks, d->E, P, expert_load, expert_offsets);
    }
    perm_place_kernel<<<n_chunks, thr, smem, st>>>(topk_idx, counts, expert_offsets, tok_of, row_of, d->T,
                                                  d->K, d->E);
    if (gather && d->H > 0)
        perm_gather_kernel<<<d->T, 128, 0, st>>>(reinterpret_cast<const uint4 *>(xq), xs, row_of,
                                                reinterpret_cast<uint4 *>(aq), as, d->H, d->K);
    return launch_status();
}
