// Gradient through the scoring with the selected slots held fixed (the top-k choice is
// piecewise constant): for one role, with the selection weights w = softmax of the selected
// scores as the forward produced them and their gradient dw (§2 Background "Product Key
// Memory", §3 Method "Sparse addressing", §4 "SDM Configuration"):
//   dscore_q = w_q (dw_q - sum_r w_r dw_r)
//   dx[0:h]  = sum_q dscore_q C1[i_q],       dx[h:2h] = sum_q dscore_q C2[j_q]
//   dC1[i]  += sum_{q: i_q = i} dscore_q x[0:h],   dC2[j] likewise with x[h:2h]
// (slot = i*n + j).  One warp per row (token of one head), lanes over the half width; the
// table gradient is accumulated with atomic adds (rows of the same head share the tables).
#pragma once

#include "common.cuh"

namespace sdm {

constexpr int SBWD_THREADS = 256;
constexpr int SBWD_ROWS = SBWD_THREADS / 32;

// HPL: half-width elements per lane (ceil(h / 32)); TPL: selected slots per lane.
template <typename XT, int HPL, int TPL>
__global__ void __launch_bounds__(SBWD_THREADS) score_backward_kernel(
    const XT* __restrict__ x, const XT* __restrict__ sk, const int32_t* __restrict__ idx,
    const float* __restrict__ w, const float* __restrict__ dw, int B, int H, int T, int d_k,
    int n, int top, float* __restrict__ dx, float* __restrict__ dsk) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y, hd = d_k >> 1;
    const long long r = (long long)blockIdx.x * SBWD_ROWS + warp;
    if (r >= (long long)B * T) return;  // whole warps leave together
    const long long b = r / T, t = r - b * T;
    const size_t ro = ((size_t)b * H + h) * T + (size_t)t;
    // dscore for the lane's selected slots
    float ds[TPL], wq[TPL], dq[TPL];
    int sq[TPL];
    float part = 0.f;
#pragma unroll
    for (int k = 0; k < TPL; ++k) {
        const int q = lane + 32 * k;
        const bool in = q < top;
        wq[k] = in ? w[ro * top + q] : 0.f;
        dq[k] = in ? dw[ro * top + q] : 0.f;
        const int s = in ? idx[ro * top + q] : 0;
        sq[k] = slot_ok(s, n * n) ? s : -1;
        part = fmaf(wq[k], dq[k], part);
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) part += __shfl_xor_sync(0xffffffffu, part, m);
#pragma unroll
    for (int k = 0; k < TPL; ++k) ds[k] = wq[k] * (dq[k] - part);
    // the row's two halves, lane-wise
    float xv[2][HPL], gx[2][HPL];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int e = 0; e < HPL; ++e) {
            const int dd = lane + 32 * e;
            xv[hf][e] = dd < hd ? to_f32(x[ro * d_k + hf * hd + dd]) : 0.f;
            gx[hf][e] = 0.f;
        }
    const XT* tab = sk + (size_t)h * 2 * n * hd;
    float* gtab = dsk + (size_t)h * 2 * n * hd;
    for (int q = 0; q < top; ++q) {
        const int k = q >> 5, src = q & 31;
        float dsq = 0.f;
        int s = -1;
#pragma unroll
        for (int kk = 0; kk < TPL; ++kk)
            if (kk == k) {
                dsq = __shfl_sync(0xffffffffu, ds[kk], src);
                s = __shfl_sync(0xffffffffu, sq[kk], src);
            }
        if (s < 0) continue;  // warp-uniform
        const int ij[2] = {s / n, s % n};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const size_t row = ((size_t)hf * n + ij[hf]) * hd;
#pragma unroll
            for (int e = 0; e < HPL; ++e) {
                const int dd = lane + 32 * e;
                if (dd < hd) {
                    gx[hf][e] = fmaf(dsq, to_f32(tab[row + dd]), gx[hf][e]);
                    atomicAdd(gtab + row + dd, dsq * xv[hf][e]);
                }
            }
        }
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int e = 0; e < HPL; ++e) {
            const int dd = lane + 32 * e;
            if (dd < hd) dx[ro * d_k + hf * hd + dd] = gx[hf][e];
        }
}

}  // namespace sdm
