// The two sides of an SDM layer around the memory.
//
// Output side (§3 Method "Sparse retrieval": the read result is
// RMS-normalised, elementwise gated and mixed across the SDM heads by the output
// projection):
//   a[b,t][h*d_v + c] = x[c] / sqrt(mean_c x^2 + eps) * wn[c] * swish(g[b,t][h*d_v + c]),
//                       x = o[b][h][t][0..d_v),  swish(z) = z * sigmoid(z)
//   y[b,t][:]         = a[b,t][:] @ Wo            (Wo given transposed: Wo_t [d_model][H*d_v])
// The first line is layer_prologue_kernel (one warp per (b,t,h) row, a stored as bf16, the
// tensor cores' operand type); the second is the tcgen05 GEMM of gemm_tc.cuh.
#pragma once

#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"

namespace sdm {

constexpr int LAYER_THREADS = 256;

template <int PER>  // d_v / 32 values per lane
__global__ void __launch_bounds__(LAYER_THREADS) layer_prologue_kernel(
    const float* __restrict__ o, const __nv_bfloat16* __restrict__ g,
    const float* __restrict__ wn, float eps, int B, int H, int T, int d_v,
    __nv_bfloat16* __restrict__ a) {
    const long long wid = ((long long)blockIdx.x * LAYER_THREADS + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long rows = (long long)B * T * H;
    if (wid >= rows) return;  // whole warps leave together
    const int h = (int)(wid % H);
    const long long bt = wid / H;  // b*T + t
    const int t = (int)(bt % T);
    const int b = (int)(bt / T);
    const float* x = o + (((size_t)b * H + h) * T + t) * d_v;
    const __nv_bfloat16* gr = g + (size_t)bt * H * d_v + (size_t)h * d_v;
    __nv_bfloat16* ar = a + (size_t)bt * H * d_v + (size_t)h * d_v;
    float v[PER];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int c = lane + 32 * i;
        v[i] = c < d_v ? x[c] : 0.f;
        ss = fmaf(v[i], v[i], ss);
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    const float r = rsqrtf(ss / (float)d_v + eps);
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int c = lane + 32 * i;
        if (c < d_v) {
            const float z = __bfloat162float(gr[c]);
            const float sw = z / (1.f + expf(-z));
            ar[c] = __float2bfloat16_rn(v[i] * r * wn[c] * sw);
        }
    }
}

// Input side: P = x Win (the tcgen05 GEMM), then this kernel splits each row of P into the
// per-head q, k, v, the output-gate pre-activation g and the gates
//   alpha = exp(-exp(A_log[h]) * softplus(a + dt_bias[h])),  beta = sigmoid(b),
// with P's columns per head laid out as [q (dk) | k (dk) | v (dv) | g (dv) | a | b].
// One thread per (row b*T+t, head, column of the head's block).
template <typename VT>
__global__ void __launch_bounds__(LAYER_THREADS) layer_in_split_kernel(
    const float* __restrict__ P, const float* __restrict__ A_log,
    const float* __restrict__ dt_bias, int B, int H, int T, int dk, int dv,
    __nv_bfloat16* __restrict__ q, __nv_bfloat16* __restrict__ k, VT* __restrict__ v,
    __nv_bfloat16* __restrict__ g, float* __restrict__ alpha, float* __restrict__ beta) {
    const int hs = 2 * dk + 2 * dv + 2;
    const long long total = (long long)B * T * H * hs;
    for (long long i = (long long)blockIdx.x * LAYER_THREADS + threadIdx.x; i < total;
         i += (long long)gridDim.x * LAYER_THREADS) {
        const int c = (int)(i % hs);
        const long long rh = i / hs;
        const int h = (int)(rh % H);
        const long long bt = rh / H;
        const int t = (int)(bt % T), b = (int)(bt / T);
        const float p = P[i];
        const size_t bht = ((size_t)b * H + h) * T + t;
        if (c < dk) {
            q[bht * dk + c] = __float2bfloat16_rn(p);
        } else if (c < 2 * dk) {
            k[bht * dk + (c - dk)] = __float2bfloat16_rn(p);
        } else if (c < 2 * dk + dv) {
            const float x = p;
            if constexpr (sizeof(VT) == 2) v[bht * dv + (c - 2 * dk)] = __float2bfloat16_rn(x);
            else v[bht * dv + (c - 2 * dk)] = x;
        } else if (c < 2 * dk + 2 * dv) {
            g[(size_t)bt * H * dv + (size_t)h * dv + (c - 2 * dk - dv)] = __float2bfloat16_rn(p);
        } else if (c == 2 * dk + 2 * dv) {
            const float z = p + dt_bias[h];
            const float sp = z > 20.f ? z : log1pf(expf(z));
            alpha[bht] = expf(-expf(A_log[h]) * sp);
        } else {
            beta[bht] = 1.f / (1.f + expf(-p));
        }
    }
}

}  // namespace sdm
