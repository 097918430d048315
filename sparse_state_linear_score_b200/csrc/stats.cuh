// Memory-utilisation diagnostics over post-softmax selected-slot weights (Appendix D.1
// "Memory Utilization and Access" of the pages: cumulative top-k mass and an entropy-based
// effective-key measure, summarised by the mean and by token-level quantiles over batch,
// head and time).
//
// Rows w[r][0..K) are given best first, as the scoring writes them:
//   cum[r][k] = w[r][0] + ... + w[r][k]        eff[r] = exp(H_r) / K,  H_r = -sum w ln w
// (0 ln 0 = 0).  Means over rows (deterministic: per-block sums in a fixed order, then the
// blocks in order) and exact order statistics of eff at floor(p (rows-1)) by a 4-pass radix
// select on the float bits (eff > 0, so the bits order like the values).
#pragma once

#include <math.h>

#include "common.cuh"

namespace sdm {

constexpr int STATS_THREADS = 256;
constexpr int STATS_MAXK = 64;
constexpr int STATS_MAXP = 16;

// One thread per row; block b writes its sums of cum[.][k] (k < K) and of eff to
// part[b][0..K].
__global__ void __launch_bounds__(STATS_THREADS) weight_stats_rows_kernel(
    const float* __restrict__ w, long long rows, int K, float* __restrict__ cum,
    float* __restrict__ eff, float* __restrict__ part) {
    __shared__ float s_warp[STATS_THREADS / 32][STATS_MAXK + 1];
    const long long r = (long long)blockIdx.x * STATS_THREADS + threadIdx.x;
    const bool in = r < rows;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float* wr = w + (in ? r : 0) * K;
    float c = 0.f, H = 0.f;
    for (int k = 0; k < K; ++k) {
        const float x = in ? wr[k] : 0.f;
        c += x;
        if (x > 0.f) H -= x * logf(x);
        if (in && cum) cum[r * K + k] = c;
        float s = in ? c : 0.f;
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
        if (lane == 0) s_warp[warp][k] = s;
    }
    const float e = expf(H) / (float)K;
    if (in) eff[r] = e;
    float s = in ? e : 0.f;
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
    if (lane == 0) s_warp[warp][K] = s;
    __syncthreads();
    for (int k = threadIdx.x; k <= K; k += STATS_THREADS) {
        float t = 0.f;
        for (int q = 0; q < STATS_THREADS / 32; ++q) t += s_warp[q][k];
        part[(size_t)blockIdx.x * (K + 1) + k] = t;
    }
}

struct StatsProbs {
    double p[STATS_MAXP];
};

// One block: means from the block sums (blocks in order), then the order statistics.
__global__ void __launch_bounds__(1024) weight_stats_summary_kernel(
    const float* __restrict__ part, int nblocks, long long rows, int K,
    const float* __restrict__ eff, float* __restrict__ mean, int nprobs, StatsProbs probs,
    float* __restrict__ quant) {
    __shared__ unsigned s_hist[256];
    __shared__ unsigned s_prefix, s_mask;
    __shared__ long long s_rank;
    const int tid = threadIdx.x;
    for (int k = tid; k <= K; k += blockDim.x) {
        double t = 0.0;
        for (int b = 0; b < nblocks; ++b) t += (double)part[(size_t)b * (K + 1) + k];
        mean[k] = (float)(t / (double)rows);
    }
    for (int q = 0; q < nprobs; ++q) {
        if (tid == 0) {
            s_prefix = 0u;
            s_mask = 0u;
            s_rank = (long long)floor(probs.p[q] * (double)(rows - 1));
        }
        __syncthreads();
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += blockDim.x) s_hist[i] = 0u;
            __syncthreads();
            const unsigned prefix = s_prefix, mask = s_mask;
            for (long long i = tid; i < rows; i += blockDim.x) {
                const unsigned key = __float_as_uint(eff[i]);
                if ((key & mask) == prefix) atomicAdd(&s_hist[(key >> shift) & 255u], 1u);
            }
            __syncthreads();
            if (tid == 0) {  // the bin holding the rank-th smallest remaining key
                long long rank = s_rank, below = 0;
                int bin = 255;
                for (int b = 0; b < 256; ++b) {
                    if (below + s_hist[b] > rank) {
                        bin = b;
                        break;
                    }
                    below += s_hist[b];
                }
                s_rank = rank - below;
                s_prefix = prefix | ((unsigned)bin << shift);
                s_mask = mask | (255u << shift);
            }
            __syncthreads();
        }
        if (tid == 0) quant[q] = __uint_as_float(s_prefix);
        __syncthreads();
    }
}

}  // namespace sdm
