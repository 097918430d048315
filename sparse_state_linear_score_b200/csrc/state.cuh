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

// Call log: what a forward call (or decode step) overwrites in the state, so that the state at
// its start can be put back once it has run -- the in-place undo of the Sparse Delta Memory
// summary's appendix A.3 "Memory-Efficient Backward", taken across calls: a sequence run as
// several calls is differentiated call by call from the last one back, each call's start
// state rebuilt from the state after it and its log (O(T*W*d) per call, no copy of the N*d
// table).  A call writes only the rows and stamps of its write slots and Lambda, so the log
// holds, per write occurrence o (token-major, [BH][T*W]), the raw row and the stamp of o's
// slot before the call, and Lambda per sequence.  Occurrences of the same slot log the same
// values, so the restore's duplicate stores write equal bytes.  Layout of the log:
//   rows  [BH][T*W][d_v] fp32, stamps [BH][T*W] fp64, Lambda [BH] fp64 (16-byte sections).
// One thread per float4 of a logged row; SAVE copies state -> log, otherwise log -> state.
template <bool SAVE>
__global__ void call_log_kernel(const int32_t* __restrict__ widx, float* __restrict__ M,
                                double* __restrict__ stamp, double* __restrict__ lambda,
                                float* __restrict__ lrows, double* __restrict__ lstamp,
                                double* __restrict__ llam, size_t n_occ, int TW, int N, int d_v,
                                int BH) {
    const int Q = d_v / 4;
    const size_t total = n_occ * (size_t)Q;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += stride) {
        const size_t occ = e / Q;
        const int q = (int)(e - occ * Q);
        const size_t bh = occ / (size_t)TW;
        const int sl = widx[occ];
        if (!slot_ok(sl, N)) {
            if (q == 0) raise_err(SDM_DEVERR_SLOT_RANGE);
            continue;
        }
        const size_t row = bh * (size_t)N + (size_t)sl;
        float4* m = reinterpret_cast<float4*>(M + row * d_v) + q;
        float4* l = reinterpret_cast<float4*>(lrows + occ * d_v) + q;
        if (SAVE) {
            *l = *m;
            if (q == 0) lstamp[occ] = stamp[row];
        } else {
            *m = *l;
            if (q == 0) stamp[row] = lstamp[occ];
        }
    }
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < (size_t)BH; i += stride) {
        if (SAVE) llam[i] = lambda[i];
        else lambda[i] = llam[i];
    }
}

}  // namespace sdm
