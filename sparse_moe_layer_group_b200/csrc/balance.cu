// Sequence-wise balance loss and expert-load entropy.
//
// "DeepSeek-V3 technical report" walkthrough (2kiu.com), section 3.3: besides the
// batch-level bias, a complementary sequence-wise balance loss is kept as a safety
// valve -- per sequence, the sum over experts of each expert's share of the
// sequence's assignments times its mean affinity, times a very small alpha
// (aux_loss_alpha 0.001 in the lpnh.cn guide's section 3 config).  The load
// entropy is the observability metric of the same section's balance discussion.
//
//   f_i = (#slots of the sequence routed to i) / (S * K),  P_i = (1/S) sum_t s[t, i]
//   seq_loss[q] = alpha * sum_i f_i * P_i
//   entropy     = -sum_i p_i ln p_i,  p_i = load_i / sum_j load_j
// Every sum runs in float64 in a fixed order (token order, then a fixed tree over
// experts), so the result does not depend on scheduling.
#include "common.cuh"

namespace moe {

constexpr int BAL_THREADS = 256;

__device__ double block_sum_fixed(double v, double *sh) {
    const int tid = threadIdx.x;
    sh[tid] = v;
    __syncthreads();
    for (int o = BAL_THREADS / 2; o > 0; o >>= 1) {
        if (tid < o) sh[tid] += sh[tid + o];
        __syncthreads();
    }
    const double r = sh[0];
    __syncthreads();
    return r;
}

// one CTA per sequence
__global__ void __launch_bounds__(BAL_THREADS) seq_balance_kernel(const float *__restrict__ s,
                                                                  const int32_t *__restrict__ idx, int E, int K,
                                                                  int S, double alpha, double *__restrict__ out) {
    __shared__ double sh[BAL_THREADS];
    const int q = blockIdx.x;
    const int64_t t0 = static_cast<int64_t>(q) * S;
    double part = 0.0;
    for (int e = threadIdx.x; e < E; e += BAL_THREADS) {
        int cnt = 0;
        double psum = 0.0;
        for (int t = 0; t < S; ++t) {
            psum += static_cast<double>(s[(t0 + t) * E + e]);
            const int32_t *row = idx + (t0 + t) * K;
            for (int k = 0; k < K; ++k) cnt += row[k] == e;
        }
        const double f = static_cast<double>(cnt) / (static_cast<double>(S) * K);
        part += f * (psum / S);
    }
    const double tot = block_sum_fixed(part, sh);
    if (threadIdx.x == 0) out[q] = alpha * tot;
}

__global__ void __launch_bounds__(BAL_THREADS) load_entropy_kernel(const int32_t *__restrict__ load, int E,
                                                                   double *__restrict__ out) {
    __shared__ double sh[BAL_THREADS];
    double c = 0.0;
    for (int e = threadIdx.x; e < E; e += BAL_THREADS) c += static_cast<double>(load[e]);
    const double tot = block_sum_fixed(c, sh);
    double h = 0.0;
    if (tot > 0.0) {
        for (int e = threadIdx.x; e < E; e += BAL_THREADS) {
            const double p = static_cast<double>(load[e]) / tot;
            if (p > 0.0) h -= p * log(p);
        }
    }
    const double H = block_sum_fixed(h, sh);
    if (threadIdx.x == 0) *out = H;
}

}  // namespace moe

using namespace moe;

MOE_API int moe_balance_stats(const moe_dims *d, const float *scores, const int32_t *topk_idx,
                              const int32_t *expert_load, int32_t seq_len, double alpha, double *seq_loss,
                              double *entropy, void *stream) {
    if (!d || d->T < 0 || d->E <= 0 || d->K <= 0) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    if (seq_loss) {
        if (seq_len <= 0 || d->T % seq_len != 0 || !scores || !topk_idx) return MOE_ERR_INVALID_ARG;
        if (d->T > 0) {
            seq_balance_kernel<<<d->T / seq_len, BAL_THREADS, 0, st>>>(scores, topk_idx, d->E, d->K, seq_len, alpha,
                                                                       seq_loss);
        }
    }
    if (entropy) {
        if (!expert_load) return MOE_ERR_INVALID_ARG;
        load_entropy_kernel<<<1, BAL_THREADS, 0, st>>>(expert_load, d->E, entropy);
    }
    return launch_status();
}
