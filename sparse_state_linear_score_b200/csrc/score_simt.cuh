// Product-key scoring on CUDA cores: one warp per (row, role).  Used for fp32 inputs
// (exact fp32 FMA accumulation) and as the generic path for any shape the tensor-core
// kernel does not take.
//
// Per row x (a key for the write role, a query for the read role), following
// §2 Background "Product Key Memory" and §3 Method "Sparse addressing":
//   s1[i] = <x[0:h], C1[i]>,  s2[j] = <x[h:2h], C2[j]>        (fp32 FMA, d ascending)
//   keep the k_half best of each half (best first; ties to the lower sub-index)
//   rank the pairs (a, b) of those lists with (a+1)(b+1) <= top by s1 + s2
//     (any other pair has >= top pairs that beat it componentwise)
//   slot = i*n + j; weights = softmax of the `top` selected scores (§4 "SDM Configuration")
#pragma once

#include <float.h>
#include <limits.h>

#include "common.cuh"

namespace sdm {

SDM_DEV void warp_best(float& v, int& i) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, v, off);
        const int i2 = __shfl_xor_sync(0xffffffffu, i, off);
        if (better(v2, i2, v, i)) {
            v = v2;
            i = i2;
        }
    }
}

// Number of (a, b) pairs with a, b < k and (a+1)(b+1) <= top.
__host__ __device__ inline int pk_candidates(int k, int top) {
    int c = 0;
    for (int a = 0; a < k; ++a) {
        int m = top / (a + 1);
        c += m < k ? m : k;
    }
    return c;
}

// Per-warp shared memory (floats): x row, n scores, 2 x k_half (value, index), candidates.
__host__ __device__ inline int score_simt_warp_floats(int d_k, int n, int k_half, int top) {
    return d_k + n + 4 * k_half + 2 * pk_candidates(k_half, top) + 2 * top;
}

// One row scored by one warp: xr is the row [d_k], tab the head's two sub-key tables
// [2][n][d_k/2]; the selected slots and weights go to idx_row / w_row [top].  ws is this
// warp's shared scratch of score_simt_warp_floats(d_k, n, k_half, top) floats.  The scores
// are fp32 FMA sums in d order.
template <typename XT>
SDM_DEV void simt_score_row(const XT* __restrict__ xr, const XT* __restrict__ tab, int d_k, int n,
                            int k_half, int top, float* ws, int32_t* __restrict__ idx_row,
                            float* __restrict__ w_row) {
    const int lane = threadIdx.x & 31;
    const int hd = d_k / 2;
    float* xs = ws;
    float* sc = xs + d_k;
    float* tv = sc + n;                                       // [2][k_half] values
    int* ti = reinterpret_cast<int*>(tv + 2 * k_half);        // [2][k_half] sub-indices
    const int ncand = pk_candidates(k_half, top);
    float* cv = reinterpret_cast<float*>(ti + 2 * k_half);    // candidate sums
    int* cs = reinterpret_cast<int*>(cv + ncand);             // candidate slots
    float* sv = reinterpret_cast<float*>(cs + ncand);         // selected scores
    int* ss = reinterpret_cast<int*>(sv + top);               // selected slots

    for (int d = lane; d < d_k; d += 32) xs[d] = to_f32(xr[d]);
    __syncwarp();
    for (int hf = 0; hf < 2; ++hf) {
        const XT* th = tab + (size_t)hf * n * hd;
        const float* xh = xs + hf * hd;
        for (int i = lane; i < n; i += 32) {
            const XT* row = th + (size_t)i * hd;
            float s = 0.f;
            for (int d = 0; d < hd; ++d) s = fmaf(xh[d], to_f32(row[d]), s);
            sc[i] = s;
        }
        __syncwarp();
        for (int q = 0; q < k_half; ++q) {  // k_half rounds of warp argmax
            float bv = -INFINITY;
            int bi = INT_MAX;
            for (int i = lane; i < n; i += 32) {
                const float v = sc[i];
                if (better(v, i, bv, bi)) {
                    bv = v;
                    bi = i;
                }
            }
            warp_best(bv, bi);
            if (lane == 0) {
                tv[hf * k_half + q] = bv;
                ti[hf * k_half + q] = bi;
                if (bi >= 0 && bi < n) sc[bi] = -INFINITY;  // taken (NaN rows select nothing)
            }
            __syncwarp();
        }
    }
    // k x k combine over the pairs that can still reach the top
    int base = 0;
    for (int a = 0; a < k_half; ++a) {
        const int m = min(k_half, top / (a + 1));
        for (int bb = lane; bb < m; bb += 32) {
            cv[base + bb] = tv[a] + tv[k_half + bb];
            cs[base + bb] = ti[a] * n + ti[k_half + bb];
        }
        base += m;
    }
    __syncwarp();
    for (int q = 0; q < top; ++q) {
        float bv = -INFINITY;
        int bi = INT_MAX, bp = -1;
        for (int c = lane; c < ncand; c += 32) {
            const float v = cv[c];
            if (better(v, cs[c], bv, bi)) {
                bv = v;
                bi = cs[c];
                bp = c;
            }
        }
        // reduce carrying the candidate position
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float v2 = __shfl_xor_sync(0xffffffffu, bv, off);
            const int i2 = __shfl_xor_sync(0xffffffffu, bi, off);
            const int p2 = __shfl_xor_sync(0xffffffffu, bp, off);
            if (better(v2, i2, bv, bi)) {
                bv = v2;
                bi = i2;
                bp = p2;
            }
        }
        if (lane == 0) {
            sv[q] = bv;
            ss[q] = bi;
            if (bp >= 0) {
                cv[bp] = -INFINITY;
                cs[bp] = INT_MAX;
            }
        }
        __syncwarp();
    }
    // softmax over the selected scores (sv[0] is the largest)
    const float mx = sv[0];
    float z = 0.f;
    for (int q = 0; q < top; ++q) z += expf(sv[q] - mx);
    for (int q = lane; q < top; q += 32) {
        idx_row[q] = ss[q];
        w_row[q] = expf(sv[q] - mx) / z;
    }
    __syncwarp();
}

template <typename XT>
__global__ void __launch_bounds__(128) score_simt_kernel(
    const XT* __restrict__ x, const XT* __restrict__ sk, int B, int H, int T, int d_k, int n,
    int k_half, int top, int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
    extern __shared__ float smem[];
    const int warps = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5;
    const int h = blockIdx.y;
    float* ws = smem + (size_t)warp * score_simt_warp_floats(d_k, n, k_half, top);
    const XT* tab = sk + (size_t)h * 2 * n * (d_k / 2);
    const long long rows = (long long)B * T;
    for (long long r = (long long)blockIdx.x * warps + warp; r < rows;
         r += (long long)gridDim.x * warps) {
        const int b = (int)(r / T), t = (int)(r % T);
        const size_t row_off = (((size_t)b * H + h) * T + t);
        simt_score_row<XT>(x + row_off * d_k, tab, d_k, n, k_half, top, ws, idx_out + row_off * top,
                           w_out + row_off * top);
    }
}

}  // namespace sdm
