// Output side of an SDM layer (§3 Method "Sparse retrieval": the read result is
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

}  // namespace sdm
