// State kernels: reset (all slots pristine) and materialisation of the dense memory.
#pragma once

#include <math.h>

#include "common.cuh"

namespace sdm {

// stamp[:] = NaN (pristine: the slot still holds M0), Lambda[:] = 0.
// A sequence starts from the initial memory M0 (§3 Method, "Learned initial state");
// marking slots pristine stands for copying M0 into every sequence's table.
__global__ void state_reset_kernel(double* __restrict__ stamp, size_t n_stamp,
                                   double* __restrict__ lambda, int n_lambda) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    const double nan = __longlong_as_double(0x7ff8000000000000ULL);
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_stamp; i += stride)
        stamp[i] = nan;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < (size_t)n_lambda; i += stride)
        lambda[i] = 0.0;
}

// Dense memory: out[b,h,s,:] = M[b,h,s,:] * exp(Lambda - stamp) or M0[h,s,:] * exp(Lambda)
// for a pristine slot (touched-slots decay: M[b,h,s,:], or M0[h,s,:] while pristine).  One
// thread per float4 of a row.
__global__ void state_materialize_kernel(const float* __restrict__ M, const double* __restrict__ stamp,
                                         const double* __restrict__ lambda,
                                         const float* __restrict__ M0, int H, int N, int d_v,
                                         size_t n_rows, int touched, float* __restrict__ out) {
    const int q_per_row = d_v / 4;
    const size_t total = n_rows * q_per_row;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        const size_t row = i / q_per_row;  // (b*H + h)*N + s
        const int q = (int)(i % q_per_row);
        const size_t bh = row / N;
        const int s = (int)(row % N);
        const int h = (int)(bh % H);
        const double st = stamp[row];
        const double L = lambda[bh];
        float4 val;
        float f;
        if (isnan(st)) {
            val = reinterpret_cast<const float4*>(M0 + ((size_t)h * N + s) * d_v)[q];
            f = touched ? 1.f : (float)exp(L);
        } else {
            val = reinterpret_cast<const float4*>(M + row * d_v)[q];
            f = touched ? 1.f : (float)exp(L - st);
        }
        val.x *= f;
        val.y *= f;
        val.z *= f;
        val.w *= f;
        reinterpret_cast<float4*>(out + row * d_v)[q] = val;
    }
}

}  // namespace sdm
