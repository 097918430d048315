// Single-token step for every (b,h): one CTA per sequence owns full slot rows, so it
// reads and writes the stamps directly (no plan needed).
//
// Per sequence, following §2 Background "Gated DeltaNet" and §3 Method:
//   Lambda' = Lambda + log(alpha)
//   seen(s) = M[s] e^{Lambda' - stamp[s]}   (M0[s] e^{Lambda'} while pristine)
//   p = sum_i w_i seen(s_i);  d = beta (v - p)
//   M[s_i] = seen(s_i) + w_i d,  stamp[s_i] = Lambda'
//   out = sum_j u_j (value of r_j after the write)
#pragma once

#include <math.h>

#include "common.cuh"

namespace sdm {

constexpr int DECODE_THREADS = 256;

__host__ __device__ inline size_t decode_smem_bytes(int W, int R, int d_v) {
    return (size_t)(W + R) * d_v * 4 + (size_t)d_v * 4 + (size_t)(W + R) * 4 * 3 + (size_t)R * 4;
}

template <typename VT>
__global__ void __launch_bounds__(DECODE_THREADS) decode_kernel(
    const VT* __restrict__ v, const float* __restrict__ alpha, const float* __restrict__ beta,
    const int32_t* __restrict__ widx, const float* __restrict__ ww,
    const int32_t* __restrict__ ridx, const float* __restrict__ rw, float* __restrict__ M,
    double* __restrict__ stamp, double* __restrict__ lambda, const float* __restrict__ M0,
    float* __restrict__ out, int H, int N, int d_v, int W, int R) {
    extern __shared__ __align__(16) unsigned char dec_smem[];
    const size_t bh = blockIdx.x;
    const int h = (int)(bh % H);
    const int tid = threadIdx.x;
    const int no = W + R;
    const int Q = d_v / 4;
    float* s_rows = reinterpret_cast<float*>(dec_smem);        // [W+R][d_v]
    float* s_d = s_rows + (size_t)no * d_v;                    // [d_v]
    int* s_slot = reinterpret_cast<int*>(s_d + d_v);           // [W+R]
    float* s_w = reinterpret_cast<float*>(s_slot + no);        // [W+R]
    float* s_fe = s_w + no;                                    // [W+R], sign: pristine
    int* s_match = reinterpret_cast<int*>(s_fe + no);          // [R]

    float* Mb = M + bh * (size_t)N * d_v;
    const float* M0h = M0 + (size_t)h * N * d_v;
    double* stb = stamp + bh * (size_t)N;
    const float a = alpha[bh];
    double la = 0.0;
    if (a > 0.f) la = log((double)a);
    else if (tid == 0) raise_err(SDM_DEVERR_ALPHA);
    const double Lnew = lambda[bh] + la;

    if (tid < no) {
        int s;
        float w;
        if (tid < W) {
            s = widx[bh * W + tid];
            w = ww[bh * W + tid];
        } else {
            s = ridx[bh * R + (tid - W)];
            w = rw[bh * R + (tid - W)];
        }
        float f = 0.f;
        if (!slot_ok(s, N)) {
            raise_err(SDM_DEVERR_SLOT_RANGE);
            s = -1;
        } else {
            const double st = stb[s];
            f = isnan(st) ? -(float)exp(Lnew) : (float)exp(Lnew - st);
        }
        s_slot[tid] = s;
        s_w[tid] = w;
        s_fe[tid] = f;
    }
    __syncthreads();
    if (tid < W) {
        const int s = s_slot[tid];
        for (int i = 0; i < tid; ++i)
            if (s >= 0 && s_slot[i] == s) raise_err(SDM_DEVERR_DUP_WRITE);
    }
    if (tid < R) {
        const int s = s_slot[W + tid];
        int m = -1;
        for (int i = 0; i < W; ++i)
            if (s >= 0 && s_slot[i] == s) m = i;
        s_match[tid] = m;
    }
    for (int e = tid; e < no * Q; e += DECODE_THREADS) {
        const int o = e / Q, q = e % Q;
        const int s = s_slot[o];
        float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
        if (s >= 0) {
            const float* src = signbit(s_fe[o]) ? M0h : Mb;
            val = reinterpret_cast<const float4*>(src + (size_t)s * d_v)[q];
        }
        reinterpret_cast<float4*>(s_rows + (size_t)o * d_v)[q] = val;
    }
    __syncthreads();
    for (int c = tid; c < d_v; c += DECODE_THREADS) {
        float p = 0.f;
        for (int i = 0; i < W; ++i) p = fmaf(s_w[i] * fabsf(s_fe[i]), s_rows[(size_t)i * d_v + c], p);
        s_d[c] = beta[bh] * (to_f32(v[bh * d_v + c]) - p);
    }
    __syncthreads();
    for (int e = tid; e < W * Q; e += DECODE_THREADS) {
        const int i = e / Q, q = e % Q;
        const int s = s_slot[i];
        const float f = fabsf(s_fe[i]), w = s_w[i];
        float4 r = reinterpret_cast<const float4*>(s_rows + (size_t)i * d_v)[q];
        const float4 dd = reinterpret_cast<const float4*>(s_d)[q];
        r.x = fmaf(f, r.x, w * dd.x);
        r.y = fmaf(f, r.y, w * dd.y);
        r.z = fmaf(f, r.z, w * dd.z);
        r.w = fmaf(f, r.w, w * dd.w);
        reinterpret_cast<float4*>(s_rows + (size_t)i * d_v)[q] = r;  // now the written value
        if (s >= 0) reinterpret_cast<float4*>(Mb + (size_t)s * d_v)[q] = r;
    }
    if (tid < W && s_slot[tid] >= 0) stb[s_slot[tid]] = Lnew;
    __syncthreads();
    for (int c = tid; c < d_v; c += DECODE_THREADS) {
        float o = 0.f;
        for (int j = 0; j < R; ++j) {
            const int m = s_match[j];
            const float val = m >= 0 ? s_rows[(size_t)m * d_v + c]
                                     : fabsf(s_fe[W + j]) * s_rows[(size_t)(W + j) * d_v + c];
            o = fmaf(s_w[W + j], val, o);
        }
        out[bh * d_v + c] = o;
    }
    if (tid == 0) lambda[bh] = Lnew;
}

}  // namespace sdm
