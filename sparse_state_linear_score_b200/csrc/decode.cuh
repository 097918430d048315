// Single-token step for every (b,h): one CTA per sequence owns full slot rows, so it
// reads and writes the stamps directly (no plan needed).
//
// Per sequence, following §2 Background "Gated DeltaNet" and §3 Method:
//   Lambda' = Lambda + log(alpha)
//   seen(s) = M[s] e^{Lambda' - stamp[s]}   (M0[s] e^{Lambda'} while pristine)
//             [touched-slots decay: alpha M[s] for a write slot, M[s] for a read slot]
//   p = sum_i w_i seen(s_i);  d = beta (v - p)
//   M[s_i] = seen(s_i) + w_i d,  stamp[s_i] = Lambda'
//   out = sum_j u_j (value of r_j after the write)
#pragma once

#include <math.h>

#include "common.cuh"

namespace sdm {

constexpr int DECODE_THREADS = 256;
constexpr int DECODE_WARPS = DECODE_THREADS / 32;

// Layout of one CTA: warp w owns write rows i = w, w+8, ... and read rows j = w, w+8, ...;
// lane l owns the float4 columns q = l (+32) of d_v.  The rows live in registers: every
// row load of a warp is issued before the first is used, and the cross-warp sums (p, then
// the output) go through two [8][d_v] partial arrays in shared memory.  A read slot that is
// also written this step takes the written row: its weight is added to that write row's
// output weight (read slots are distinct, so at most one read lands on a write row).
__host__ __device__ inline size_t decode_smem_bytes(int W, int R, int d_v) {
    return (size_t)2 * DECODE_WARPS * d_v * 4 + (size_t)(W + R) * 12 + (size_t)W * 4 +
           (size_t)R * 4;
}

template <typename VT>
SDM_DEV float4 load_v4(const VT* p);
template <>
SDM_DEV float4 load_v4<float>(const float* p) {
    return __ldg(reinterpret_cast<const float4*>(p));
}
template <>
SDM_DEV float4 load_v4<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                       __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}

SDM_DEV void fma4(float4& acc, float c, const float4& x) {
    acc.x = fmaf(c, x.x, acc.x);
    acc.y = fmaf(c, x.y, acc.y);
    acc.z = fmaf(c, x.z, acc.z);
    acc.w = fmaf(c, x.w, acc.w);
}

// RPW: rows of each role per warp (ceil(max(W, R) / 8)); QPL: float4 columns per lane.
template <typename VT, int RPW, int QPL>
__global__ void __launch_bounds__(DECODE_THREADS) decode_kernel(
    const VT* __restrict__ v, const float* __restrict__ alpha, const float* __restrict__ beta,
    const int32_t* __restrict__ widx, const float* __restrict__ ww,
    const int32_t* __restrict__ ridx, const float* __restrict__ rw, float* __restrict__ M,
    double* __restrict__ stamp, double* __restrict__ lambda, const float* __restrict__ M0,
    float* __restrict__ out, int H, int N, int d_v, int W, int R, int touched) {
    extern __shared__ __align__(16) unsigned char dec_smem[];
    const size_t bh = blockIdx.x;
    const int h = (int)(bh % H);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int no = W + R;
    const int Q = d_v / 4;
    float* s_pp = reinterpret_cast<float*>(dec_smem);              // [8][d_v] partial p
    float* s_po = s_pp + DECODE_WARPS * d_v;                       // [8][d_v] partial out
    int* s_slot = reinterpret_cast<int*>(s_po + DECODE_WARPS * d_v);  // [W+R]
    float* s_w = reinterpret_cast<float*>(s_slot + no);            // [W+R]
    float* s_f = s_w + no;                                         // [W+R], sign: pristine
    float* s_uw = s_f + no;                                        // [W] read weight on row i
    int* s_rm = reinterpret_cast<int*>(s_uw + W);                  // [R] read j is written

    float* Mb = M + bh * (size_t)N * d_v;
    const float* M0h = M0 + (size_t)h * N * d_v;
    double* stb = stamp + bh * (size_t)N;
    // inputs that do not come from the scoring launch before this one: read them while it
    // finishes (programmatic dependent launch), then wait for its indices and weights
    const float bt = beta[bh];
    float4 vv[QPL];
#pragma unroll
    for (int c = 0; c < QPL; ++c) {
        const int q = lane + 32 * c;
        vv[c] = q < Q ? load_v4<VT>(v + bh * d_v + 4 * q) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    double Lnew;  // Lambda'
    const float a_t = alpha[bh];
    {
        double la = 0.0;
        if (a_t > 0.f) la = log((double)a_t);
        else if (tid == 0) raise_err(SDM_DEVERR_ALPHA);
        Lnew = lambda[bh] + la;
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---- this warp's rows: lane k fetches write row w + 8k, lane 16 + k read row w + 8k
    //      (slot, weight, decay factor from the stamp), the warp shares them by shuffles and
    //      puts every row load in flight before the first block barrier --------------------
    int my_s = -1;
    float my_f = 0.f;
    {
        const bool rl = lane >= 16;
        const int k = lane & 15, i = warp + DECODE_WARPS * k;
        if (k < RPW && i < (rl ? R : W)) {
            int sl = rl ? ridx[bh * R + i] : widx[bh * W + i];
            const float w = rl ? rw[bh * R + i] : ww[bh * W + i];
            float f = 0.f;
            if (!slot_ok(sl, N)) {
                raise_err(SDM_DEVERR_SLOT_RANGE);
                sl = -1;
            } else {
                const double st = stb[sl];
                if (touched) {  // alpha scales the write slots only
                    const float fv = rl ? 1.f : a_t;
                    f = isnan(st) ? -fv : fv;
                } else {
                    f = isnan(st) ? -(float)exp(Lnew) : (float)exp(Lnew - st);
                }
            }
            my_s = sl;
            my_f = f;
            const int o = rl ? W + i : i;
            s_slot[o] = sl;
            s_w[o] = w;
            s_f[o] = f;
        }
    }
    float4 wr[RPW][QPL], rd[RPW][QPL];
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
        const int si = __shfl_sync(0xffffffffu, my_s, k);
        const int sj = __shfl_sync(0xffffffffu, my_s, 16 + k);
        const float fi = __shfl_sync(0xffffffffu, my_f, k);
        const float fj = __shfl_sync(0xffffffffu, my_f, 16 + k);
        const float* srci = (si >= 0 && signbit(fi)) ? M0h : Mb;
        const float* srcj = (sj >= 0 && signbit(fj)) ? M0h : Mb;
#pragma unroll
        for (int c = 0; c < QPL; ++c) {
            const int q = lane + 32 * c;
            wr[k][c] = (si >= 0 && q < Q)
                           ? __ldg(reinterpret_cast<const float4*>(srci + (size_t)si * d_v) + q)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            rd[k][c] = (sj >= 0 && q < Q)
                           ? __ldg(reinterpret_cast<const float4*>(srcj + (size_t)sj * d_v) + q)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    __syncthreads();  // every warp's slots are in shared memory

    // ---- while they land: duplicate writes, reads of written slots --------------------------
    if (tid < W) {
        const int s = s_slot[tid];
        float uw = 0.f;
        if (W <= 32) {  // the write slots are the lanes of warp 0
            const unsigned lanes = W == 32 ? 0xffffffffu : (1u << W) - 1u;
            const unsigned same = __match_any_sync(lanes, s);
            if (s >= 0 && __popc(same) > 1 && (int)(__ffs(same) - 1) == tid)
                raise_err(SDM_DEVERR_DUP_WRITE);
        } else if (s >= 0) {
            for (int i = 0; i < tid; ++i)
                if (s_slot[i] == s) raise_err(SDM_DEVERR_DUP_WRITE);
        }
        if (s >= 0)
            for (int j = 0; j < R; ++j)
                if (s_slot[W + j] == s) uw += s_w[W + j];
        s_uw[tid] = uw;
    } else if (tid < no) {
        const int s = s_slot[tid];
        int m = 0;
        if (s >= 0)
            for (int i = 0; i < W; ++i) m |= s_slot[i] == s;
        s_rm[tid - W] = m;
    }

    // ---- p = sum_i w_i seen(s_i) ------------------------------------------------------------
    {
        float4 pp[QPL];
#pragma unroll
        for (int c = 0; c < QPL; ++c) pp[c] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < RPW; ++k) {
            const int i = warp + DECODE_WARPS * k;
            if (i < W) {
                const float cw = s_w[i] * fabsf(s_f[i]);
#pragma unroll
                for (int c = 0; c < QPL; ++c) fma4(pp[c], cw, wr[k][c]);
            }
        }
#pragma unroll
        for (int c = 0; c < QPL; ++c) {
            const int q = lane + 32 * c;
            if (q < Q) reinterpret_cast<float4*>(s_pp + warp * d_v)[q] = pp[c];
        }
    }
    __syncthreads();

    // ---- d = beta (v - p); written rows, stores, partial outputs --------------------------
    {
        float4 dd[QPL], po[QPL];
#pragma unroll
        for (int c = 0; c < QPL; ++c) {
            const int q = lane + 32 * c;
            float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
            if (q < Q)
#pragma unroll
                for (int w2 = 0; w2 < DECODE_WARPS; ++w2) {
                    const float4 t = reinterpret_cast<const float4*>(s_pp + w2 * d_v)[q];
                    p.x += t.x;
                    p.y += t.y;
                    p.z += t.z;
                    p.w += t.w;
                }
            dd[c] = make_float4(bt * (vv[c].x - p.x), bt * (vv[c].y - p.y), bt * (vv[c].z - p.z),
                                bt * (vv[c].w - p.w));
            po[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < RPW; ++k) {
            const int i = warp + DECODE_WARPS * k;
            if (i < W) {
                const int s = s_slot[i];
                const float f = fabsf(s_f[i]), w = s_w[i], uw = s_uw[i];
#pragma unroll
                for (int c = 0; c < QPL; ++c) {
                    const int q = lane + 32 * c;
                    float4 r = wr[k][c];
                    r.x = fmaf(f, r.x, w * dd[c].x);
                    r.y = fmaf(f, r.y, w * dd[c].y);
                    r.z = fmaf(f, r.z, w * dd[c].z);
                    r.w = fmaf(f, r.w, w * dd[c].w);
                    if (s >= 0 && q < Q) reinterpret_cast<float4*>(Mb + (size_t)s * d_v)[q] = r;
                    fma4(po[c], uw, r);
                }
            }
            const int j = i;
            if (j < R && !s_rm[j]) {
                const float cu = s_w[W + j] * fabsf(s_f[W + j]);
#pragma unroll
                for (int c = 0; c < QPL; ++c) fma4(po[c], cu, rd[k][c]);
            }
        }
#pragma unroll
        for (int c = 0; c < QPL; ++c) {
            const int q = lane + 32 * c;
            if (q < Q) reinterpret_cast<float4*>(s_po + warp * d_v)[q] = po[c];
        }
    }
    if (tid < W && s_slot[tid] >= 0) stb[s_slot[tid]] = Lnew;
    __syncthreads();

    // ---- out = sum of the partial outputs ----------------------------------------------------
    for (int q = tid; q < Q; q += DECODE_THREADS) {
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w2 = 0; w2 < DECODE_WARPS; ++w2) {
            const float4 t = reinterpret_cast<const float4*>(s_po + w2 * d_v)[q];
            o.x += t.x;
            o.y += t.y;
            o.z += t.z;
            o.w += t.w;
        }
        reinterpret_cast<float4*>(out + bh * d_v)[q] = o;
    }
    if (tid == 0) lambda[bh] = Lnew;
}

}  // namespace sdm
