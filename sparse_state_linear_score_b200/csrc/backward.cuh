// Backward of the recurrence over one call (Sparse Delta Memory summary, appendix A.3
// "Memory-Efficient Backward": the sparse updates are applied in place and undone while
// the gradients flow back, so no copy of the memory is kept per chunk).
//
// bwd_replay_kernel: from the state at the start of the call, the tokens are replayed in
// place, one CTA per (b,h), and before every write the raw rows and stamps of the token's
// W write slots go to a log (T*W rows + T*W stamps per (b,h): the O(T*W*d) record), with
// Lambda after every token.
//
// bwd_sweep_kernel: the tokens backwards.  With G = dout[t], per token (decayed rows
// Mt = alpha M_{t-1} on the write slots, as in the forward):
//   read:   du_j = <G, M_t[r_j]>,  dM[r_j] += u_j G
//   write:  e = v - sum_i w_i Mt[s_i],  de = beta sum_i w_i dM[s_i],  dv = de,
//           dbeta = sum_i w_i <dM[s_i], e>,  dw_i = beta <dM[s_i], e> - <de, Mt[s_i]>,
//           dMt[s_i] = dM[s_i] - w_i de
//   decay:  every slot decays: dalpha = <dMt, M_{t-1}> over all N slots, obtained from a
//           running X = <dM, M> (full inner product) that only the touched rows change:
//           dalpha = (X - sum_i <dM[s_i], M_t[s_i]>) / alpha + sum_i <dMt[s_i], M_{t-1}[s_i]>,
//           then X <- alpha dalpha; dM_{t-1} = alpha dMt, kept lazily as raw rows, a
//           backward log-decay prefix Gam (+= log alpha per token) and per-row stamps.
//           Touched-slots decay: dalpha = sum_i <dMt[s_i], M_{t-1}[s_i]> and only the write
//           rows take the factor alpha.
//   then the write slots' raw rows and stamps are restored from the log, and Lambda.
// On return the state is again the state at the start of the call.
//
// Layout: warp w owns write rows w, w+8, ... and read rows w, w+8, ...; lane l owns the
// float4 columns l (+32) of d_v; sums across warps go through [8][d_v] shared partials.
#pragma once

#include <math.h>

#include "common.cuh"

namespace sdm {

constexpr int BWD_THREADS = 256;
constexpr int BWD_WARPS = BWD_THREADS / 32;
constexpr int BWD_MAXO = 128;  // W + R

// Per-(b,h) records of one call (a byte layout in the workspace).
struct BwdPtrs {
    float* log_rows;     // [BH][T][W][d_v] raw rows of the write slots before the write
    double* log_stamp;   // [BH][T][W]      their stamps before the write
    double* log_lam;     // [BH][T+1]       Lambda at the start, then after every token
    float* dM;           // [BH][N][d_v]    raw memory gradient rows
    double* dstamp;      // [BH][N]         their stamps (NaN: the row is zero)
};

__host__ __device__ inline size_t bwd_smem_bytes(int d_v) {
    return (size_t)3 * BWD_WARPS * d_v * 4 + (size_t)BWD_MAXO * 16 + 64 * 8;
}

SDM_DEV float4 f4(float a) { return make_float4(a, a, a, a); }
SDM_DEV float4 f4_fma(float s, const float4& x, const float4& y) {
    return make_float4(fmaf(s, x.x, y.x), fmaf(s, x.y, y.y), fmaf(s, x.z, y.z), fmaf(s, x.w, y.w));
}
SDM_DEV float f4_dot(const float4& a, const float4& b) {
    return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}
SDM_DEV float warp_sum(float x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}
SDM_DEV float4 f4_scale(float s, const float4& a) {
    return make_float4(s * a.x, s * a.y, s * a.z, s * a.w);
}

template <typename VT>
SDM_DEV float4 bwd_load_v4(const VT* p);
template <>
SDM_DEV float4 bwd_load_v4<float>(const float* p) {
    return *reinterpret_cast<const float4*>(p);
}
template <>
SDM_DEV float4 bwd_load_v4<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                       __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}

// e^d for a log-decay difference d taken in fp64: the exponential in fp32 (the factor is
// stored and used in fp32; rounding d to fp32 first moves it by |d| * 6e-8 relative).
SDM_DEV float bwd_exp(double d) { return expf((float)d); }

// Value factor of a slot at prefix L from its stamp (every-slot decay; the sign marks a
// pristine slot, whose row is M0); touched-slots decay: 1.
SDM_DEV float bwd_factor(double st, double L, int touched) {
    if (touched) return isnan(st) ? -1.f : 1.f;
    return isnan(st) ? -bwd_exp(L) : bwd_exp(L - st);
}

// ---- replay with the log --------------------------------------------------------------
// QPL: float4 columns per lane (d_v <= 128: 1, else 2); WPW: write rows per warp.  Each
// token's loads go out in dependent rounds (its indices were fetched during the previous
// token; then the stamps; then every row), and all stores follow the loads.
template <typename VT, int QPL, int WPW>
__global__ void __launch_bounds__(BWD_THREADS) bwd_replay_kernel(
    const VT* __restrict__ v, const float* __restrict__ alpha, const float* __restrict__ beta,
    const int32_t* __restrict__ widx, const float* __restrict__ ww, float* __restrict__ M,
    double* __restrict__ stamp, double* __restrict__ lambda, const float* __restrict__ M0,
    BwdPtrs P, int H, int N, int T, int d_v, int W, int touched) {
    extern __shared__ __align__(16) unsigned char bwd_smem[];
    const size_t bh = blockIdx.x;
    const int h = (int)(bh % H);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Q = d_v / 4;
    float* s_pp = reinterpret_cast<float*>(bwd_smem);  // [8][d_v]
    float* Mb = M + bh * (size_t)N * d_v;
    const float* M0h = M0 + (size_t)h * N * d_v;
    double* stb = stamp + bh * (size_t)N;
    double L = lambda[bh];
    if (tid == 0) P.log_lam[bh * (size_t)(T + 1)] = L;
    // indices and weights of the next token
    int nsl[WPW];
    float nwi[WPW], na = 1.f, nb = 0.f;
    auto fetch = [&](int t) {
        const size_t bt = bh * (size_t)T + t;
        na = alpha[bt];
        nb = beta[bt];
#pragma unroll
        for (int k = 0; k < WPW; ++k) {
            const int i = warp + BWD_WARPS * k;
            nsl[k] = i < W ? widx[bt * W + i] : -1;
            nwi[k] = i < W ? ww[bt * W + i] : 0.f;
        }
    };
    if (T > 0) fetch(0);
    for (int t = 0; t < T; ++t) {
        const size_t bt = bh * (size_t)T + t;
        const float a = na, bta = nb;
        int sl[WPW];
        float wi[WPW];
#pragma unroll
        for (int k = 0; k < WPW; ++k) {
            sl[k] = nsl[k];
            wi[k] = nwi[k];
            if (sl[k] >= 0 && !slot_ok(sl[k], N)) {
                if (lane == 0) raise_err(SDM_DEVERR_SLOT_RANGE);
                sl[k] = -1;
            }
        }
        if (a > 0.f) L += log((double)a);
        else if (tid == 0) raise_err(SDM_DEVERR_ALPHA);
        float4 vv[QPL];
#pragma unroll
        for (int c = 0; c < QPL; ++c) {
            const int q = lane + 32 * c;
            vv[c] = q < Q ? bwd_load_v4<VT>(v + bt * d_v + 4 * q) : f4(0.f);
        }
        double st[WPW];
#pragma unroll
        for (int k = 0; k < WPW; ++k) st[k] = sl[k] >= 0 ? stb[sl[k]] : 0.0;
        float4 raw[WPW][QPL], mraw[WPW][QPL];
        float fk[WPW];
#pragma unroll
        for (int k = 0; k < WPW; ++k) {
            const int s = sl[k];
            fk[k] = bwd_factor(st[k], L, touched) * (touched ? a : 1.f);
#pragma unroll
            for (int c = 0; c < QPL; ++c) {
                const int q = lane + 32 * c;
                raw[k][c] = mraw[k][c] = f4(0.f);
                if (s >= 0 && q < Q) {
                    mraw[k][c] = reinterpret_cast<const float4*>(Mb + (size_t)s * d_v)[q];
                    raw[k][c] = signbit(fk[k])
                                    ? reinterpret_cast<const float4*>(M0h + (size_t)s * d_v)[q]
                                    : mraw[k][c];
                }
            }
        }
        if (t + 1 < T) fetch(t + 1);
        float4 pp[QPL];
#pragma unroll
        for (int c = 0; c < QPL; ++c) pp[c] = f4(0.f);
#pragma unroll
        for (int k = 0; k < WPW; ++k)
#pragma unroll
            for (int c = 0; c < QPL; ++c) {
                raw[k][c] = f4_scale(fabsf(fk[k]), raw[k][c]);  // the decayed row, "seen"
                pp[c] = f4_fma(wi[k], raw[k][c], pp[c]);
            }
#pragma unroll
        for (int c = 0; c < QPL; ++c) {
            const int q = lane + 32 * c;
            if (q < Q) reinterpret_cast<float4*>(s_pp + warp * d_v)[q] = pp[c];
        }
        __syncthreads();
        float4 dd[QPL];
#pragma unroll
        for (int c = 0; c < QPL; ++c) {
            const int q = lane + 32 * c;
            float4 p = f4(0.f);
            if (q < Q)
                for (int w2 = 0; w2 < BWD_WARPS; ++w2) {
                    const float4 x = reinterpret_cast<const float4*>(s_pp + w2 * d_v)[q];
                    p = make_float4(p.x + x.x, p.y + x.y, p.z + x.z, p.w + x.w);
                }
            dd[c] = make_float4(bta * (vv[c].x - p.x), bta * (vv[c].y - p.y), bta * (vv[c].z - p.z),
                                bta * (vv[c].w - p.w));
        }
#pragma unroll
        for (int k = 0; k < WPW; ++k) {
            const int s = sl[k];
            if (s < 0) continue;
            const int i = warp + BWD_WARPS * k;
            const size_t lr = (bt * W + i) * (size_t)d_v;
#pragma unroll
            for (int c = 0; c < QPL; ++c) {
                const int q = lane + 32 * c;
                if (q < Q) {
                    reinterpret_cast<float4*>(P.log_rows + lr)[q] = mraw[k][c];
                    reinterpret_cast<float4*>(Mb + (size_t)s * d_v)[q] =
                        f4_fma(wi[k], dd[c], raw[k][c]);
                }
            }
            if (lane == 0) {
                P.log_stamp[bt * W + i] = st[k];
                stb[s] = L;
            }
        }
        if (tid == 0) P.log_lam[bh * (size_t)(T + 1) + t + 1] = L;
        __syncthreads();  // this token's rows and stamps before the next token's gathers
    }
    if (tid == 0) lambda[bh] = L;
}

// ---- the backward sweep ---------------------------------------------------------------
// Per token: its indices, weights, dout and v rows were fetched during the previous token;
// the read rows' stamps, then their rows (M side and gradient side) go out together; the
// write rows' M side (log stamps, current stamps, then log and current rows) is issued
// before the read rows are processed, their gradient side after the barrier that publishes
// the read rows' gradient updates.
template <typename VT, int QPL, int WPW>
__global__ void __launch_bounds__(BWD_THREADS) bwd_sweep_kernel(
    const VT* __restrict__ v, const float* __restrict__ alpha, const float* __restrict__ beta,
    const int32_t* __restrict__ widx, const float* __restrict__ ww,
    const int32_t* __restrict__ ridx, const float* __restrict__ rw, float* __restrict__ M,
    double* __restrict__ stamp, double* __restrict__ lambda, const float* __restrict__ M0,
    BwdPtrs P, const float* __restrict__ dout, float* __restrict__ dv_out,
    float* __restrict__ dalpha, float* __restrict__ dbeta, float* __restrict__ dww,
    float* __restrict__ drw, int H, int N, int T, int d_v, int W, int R, int touched) {
    extern __shared__ __align__(16) unsigned char bwd_smem[];
    const size_t bh = blockIdx.x;
    const int h = (int)(bh % H);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Q = d_v / 4;
    float* s_pp = reinterpret_cast<float*>(bwd_smem);          // [8][d_v] partial p
    float* s_pd = s_pp + BWD_WARPS * d_v;                      // [8][d_v] partial sum w dM
    double* s_part = reinterpret_cast<double*>(s_pd + BWD_WARPS * d_v);  // [8][4] partial sums
    float* Mb = M + bh * (size_t)N * d_v;
    const float* M0h = M0 + (size_t)h * N * d_v;
    double* stb = stamp + bh * (size_t)N;
    float* dMb = P.dM + bh * (size_t)N * d_v;
    double* dsb = P.dstamp + bh * (size_t)N;
    const double* lamb = P.log_lam + bh * (size_t)(T + 1);
    double X = 0.0, Gam = 0.0;  // <dM, M> over every slot; backward log-decay prefix
    constexpr int RPW = WPW;
    // the next token's inputs
    int nrs[RPW], nws[WPW];
    float nu[RPW], nwi[WPW], na = 1.f, nb = 0.f;
    float4 nG[QPL], nv[QPL];
    auto fetch = [&](int t) {
        const size_t bt = bh * (size_t)T + t;
        na = alpha[bt] > 0.f ? alpha[bt] : 1.f;
        nb = beta[bt];
#pragma unroll
        for (int k = 0; k < RPW; ++k) {
            const int j = warp + BWD_WARPS * k;
            nrs[k] = j < R ? ridx[bt * R + j] : -1;
            nu[k] = j < R ? rw[bt * R + j] : 0.f;
        }
#pragma unroll
        for (int k = 0; k < WPW; ++k) {
            const int i = warp + BWD_WARPS * k;
            nws[k] = i < W ? widx[bt * W + i] : -1;
            nwi[k] = i < W ? ww[bt * W + i] : 0.f;
        }
#pragma unroll
        for (int c = 0; c < QPL; ++c) {
            const int q = lane + 32 * c;
            nG[c] = q < Q ? reinterpret_cast<const float4*>(dout + bt * d_v)[q] : f4(0.f);
            nv[c] = q < Q ? bwd_load_v4<VT>(v + bt * d_v + 4 * q) : f4(0.f);
        }
    };
    if (T > 0) fetch(T - 1);
    for (int t = T - 1; t >= 0; --t) {
        const size_t bt = bh * (size_t)T + t;
        const float a = na, bta = nb;
        const double Lt = lamb[t + 1], Lp = lamb[t];
        int rs[RPW], sl[WPW];
        float u[RPW], wi[WPW];
        float4 G[QPL], vv[QPL];
#pragma unroll
        for (int k = 0; k < RPW; ++k) {
            rs[k] = slot_ok(nrs[k], N) ? nrs[k] : -1;  // the forward reported bad slots
            u[k] = nu[k];
        }
#pragma unroll
        for (int k = 0; k < WPW; ++k) {
            sl[k] = slot_ok(nws[k], N) ? nws[k] : -1;
            wi[k] = nwi[k];
        }
#pragma unroll
        for (int c = 0; c < QPL; ++c) {
            G[c] = nG[c];
            vv[c] = nv[c];
        }
        // -- round 1: stamps of the read rows and of the write rows (M side)
        double rst[RPW], rds[RPW], wso[WPW], wsn[WPW];
#pragma unroll
        for (int k = 0; k < RPW; ++k) {
            rst[k] = rs[k] >= 0 ? stb[rs[k]] : 0.0;
            rds[k] = rs[k] >= 0 ? dsb[rs[k]] : 0.0;
        }
#pragma unroll
        for (int k = 0; k < WPW; ++k) {
            const int i = warp + BWD_WARPS * k;
            wso[k] = sl[k] >= 0 ? P.log_stamp[bt * W + i] : 0.0;
            wsn[k] = sl[k] >= 0 ? stb[sl[k]] : 0.0;
        }
        // -- round 2: the read rows (M and dM) and the write rows' M side (log and current)
        float4 rm[RPW][QPL], rg[RPW][QPL], mp[WPW][QPL], mt[WPW][QPL];
        float fo[WPW], fn[WPW];
#pragma unroll
        for (int k = 0; k < RPW; ++k) {
            const int s = rs[k];
            const float f = bwd_factor(rst[k], Lt, touched);
            const float gf = (s < 0 || isnan(rds[k])) ? 0.f : bwd_exp(Gam - rds[k]);
#pragma unroll
            for (int c = 0; c < QPL; ++c) {
                const int q = lane + 32 * c;
                rm[k][c] = rg[k][c] = f4(0.f);
                if (s >= 0 && q < Q) {
                    const float* src = (signbit(f) ? M0h : Mb) + (size_t)s * d_v;
                    rm[k][c] = f4_scale(fabsf(f), reinterpret_cast<const float4*>(src)[q]);
                    if (gf != 0.f)
                        rg[k][c] = f4_scale(gf, reinterpret_cast<const float4*>(dMb + (size_t)s * d_v)[q]);
                }
            }
        }
#pragma unroll
        for (int k = 0; k < WPW; ++k) {
            const int s = sl[k], i = warp + BWD_WARPS * k;
            fo[k] = bwd_factor(wso[k], Lp, touched);  // value factor at t-1
            fn[k] = bwd_factor(wsn[k], Lt, touched);  // at t
            const size_t lr = (bt * W + (i < W ? i : 0)) * (size_t)d_v;
#pragma unroll
            for (int c = 0; c < QPL; ++c) {
                const int q = lane + 32 * c;
                mp[k][c] = mt[k][c] = f4(0.f);
                if (s >= 0 && q < Q) {
                    const float* so_src = signbit(fo[k]) ? M0h + (size_t)s * d_v : P.log_rows + lr;
                    mp[k][c] = f4_scale(fabsf(fo[k]), reinterpret_cast<const float4*>(so_src)[q]);
                    const float* sn_src = (signbit(fn[k]) ? M0h : Mb) + (size_t)s * d_v;
                    mt[k][c] = f4_scale(fabsf(fn[k]), reinterpret_cast<const float4*>(sn_src)[q]);
                }
            }
        }
        if (t > 0) fetch(t - 1);
        // -- read rows: du_j, dM[r_j] += u_j G, X += u_j du_j
        double xr = 0.0;
#pragma unroll
        for (int k = 0; k < RPW; ++k) {
            const int j = warp + BWD_WARPS * k;
            const int s = rs[k];
            if (s < 0) continue;  // warp-uniform
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < QPL; ++c) {
                acc += f4_dot(G[c], rm[k][c]);
                rg[k][c] = f4_fma(u[k], G[c], rg[k][c]);
            }
            const float du = warp_sum(acc);
            if (lane == 0) drw[bt * R + j] = du;
            xr += (double)u[k] * du;
#pragma unroll
            for (int c = 0; c < QPL; ++c) {
                const int q = lane + 32 * c;
                if (q < Q) reinterpret_cast<float4*>(dMb + (size_t)s * d_v)[q] = rg[k][c];
            }
            __syncwarp();
            if (lane == 0) dsb[s] = Gam;
        }
        if (lane == 0) s_part[warp * 4 + 0] = xr;
        __syncthreads();  // read rows of dM (and their stamps) before the write rows use them
        if (!touched)
            for (int w2 = 0; w2 < BWD_WARPS; ++w2) X += s_part[w2 * 4 + 0];
        // -- round 3: the write rows' gradient side
        double wds[WPW];
#pragma unroll
        for (int k = 0; k < WPW; ++k) wds[k] = sl[k] >= 0 ? dsb[sl[k]] : 0.0;
        float4 dm[WPW][QPL];
        float4 pp[QPL], pd[QPL];
#pragma unroll
        for (int c = 0; c < QPL; ++c) pp[c] = pd[c] = f4(0.f);
#pragma unroll
        for (int k = 0; k < WPW; ++k) {
            const int s = sl[k];
            const float gf = (s < 0 || isnan(wds[k])) ? 0.f : bwd_exp(Gam - wds[k]);
#pragma unroll
            for (int c = 0; c < QPL; ++c) {
                const int q = lane + 32 * c;
                dm[k][c] = f4(0.f);
                if (gf != 0.f && q < Q)
                    dm[k][c] = f4_scale(gf, reinterpret_cast<const float4*>(dMb + (size_t)s * d_v)[q]);
                pp[c] = f4_fma(wi[k] * a, mp[k][c], pp[c]);
                pd[c] = f4_fma(wi[k], dm[k][c], pd[c]);
            }
        }
#pragma unroll
        for (int c = 0; c < QPL; ++c) {
            const int q = lane + 32 * c;
            if (q < Q) {
                reinterpret_cast<float4*>(s_pp + warp * d_v)[q] = pp[c];
                reinterpret_cast<float4*>(s_pd + warp * d_v)[q] = pd[c];
            }
        }
        __syncthreads();
        float4 e[QPL], de[QPL];
#pragma unroll
        for (int c = 0; c < QPL; ++c) {
            const int q = lane + 32 * c;
            float4 p = f4(0.f), d = f4(0.f);
            if (q < Q)
                for (int w2 = 0; w2 < BWD_WARPS; ++w2) {
                    const float4 x = reinterpret_cast<const float4*>(s_pp + w2 * d_v)[q];
                    const float4 y = reinterpret_cast<const float4*>(s_pd + w2 * d_v)[q];
                    p = make_float4(p.x + x.x, p.y + x.y, p.z + x.z, p.w + x.w);
                    d = make_float4(d.x + y.x, d.y + y.y, d.z + y.z, d.w + y.w);
                }
            e[c] = make_float4(vv[c].x - p.x, vv[c].y - p.y, vv[c].z - p.z, vv[c].w - p.w);
            de[c] = f4_scale(bta, d);
            if (warp == 0 && q < Q) reinterpret_cast<float4*>(dv_out + bt * d_v)[q] = de[c];
        }
        double sb = 0.0, s1 = 0.0, s2 = 0.0;  // dbeta; <dM, M_t>; <dMt, M_{t-1}> (write rows)
#pragma unroll
        for (int k = 0; k < WPW; ++k) {
            const int i = warp + BWD_WARPS * k;
            const int s = sl[k];
            if (s < 0) continue;
            float ge = 0.f, gm = 0.f, gmt = 0.f, gmp = 0.f;
            float4 nd[QPL];
#pragma unroll
            for (int c = 0; c < QPL; ++c) {
                ge += f4_dot(dm[k][c], e[c]);
                gm += f4_dot(de[c], mp[k][c]);
                gmt += f4_dot(dm[k][c], mt[k][c]);
                nd[c] = f4_fma(-wi[k], de[c], dm[k][c]);  // dMt[s_i]
                gmp += f4_dot(nd[c], mp[k][c]);
            }
            ge = warp_sum(ge);
            gm = warp_sum(gm);
            gmt = warp_sum(gmt);
            gmp = warp_sum(gmp);
            if (lane == 0) dww[bt * W + i] = bta * ge - a * gm;
            sb += (double)wi[k] * ge;
            s1 += gmt;
            s2 += gmp;
            // dM_{t-1}[s] = alpha dMt[s]: every-slot decay keeps alpha in the prefix Gam
            const float sc = touched ? a : 1.f;
            const size_t lr = (bt * W + i) * (size_t)d_v;
#pragma unroll
            for (int c = 0; c < QPL; ++c) {
                const int q = lane + 32 * c;
                if (q < Q) {
                    reinterpret_cast<float4*>(dMb + (size_t)s * d_v)[q] = f4_scale(sc, nd[c]);
                    reinterpret_cast<float4*>(Mb + (size_t)s * d_v)[q] =
                        reinterpret_cast<const float4*>(P.log_rows + lr)[q];  // restore
                }
            }
            __syncwarp();
            if (lane == 0) {
                dsb[s] = Gam;
                stb[s] = wso[k];
            }
        }
        if (lane == 0) {
            s_part[warp * 4 + 1] = sb;
            s_part[warp * 4 + 2] = s1;
            s_part[warp * 4 + 3] = s2;
        }
        __syncthreads();
        double SB = 0.0, S1 = 0.0, S2 = 0.0;
        for (int w2 = 0; w2 < BWD_WARPS; ++w2) {
            SB += s_part[w2 * 4 + 1];
            S1 += s_part[w2 * 4 + 2];
            S2 += s_part[w2 * 4 + 3];
        }
        double da;
        if (touched) {
            da = S2;
        } else {
            da = (X - S1) / (double)a + S2;
            X = (double)a * da;
            Gam += log((double)a);
        }
        if (tid == 0) {
            dalpha[bt] = (float)da;
            dbeta[bt] = (float)SB;
        }
        __syncthreads();  // s_part and s_pp are rewritten by the next token
    }
    if (tid == 0) {
        lambda[bh] = lamb[0];
        P.log_lam[bh * (size_t)(T + 1) + T] = Gam;  // the final prefix, for the dense gradient
    }
}

// Dense gradient with respect to the state at the start of the call: dM_in[s] = raw *
// e^{Gam_final - stamp} (zero for rows never reached).
__global__ void bwd_dense_kernel(const BwdPtrs P, int T, int N, int d_v, size_t n_rows,
                                 float* __restrict__ out) {
    const int Q = d_v / 4;
    const size_t total = n_rows * Q;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        const size_t row = i / Q;
        const int q = (int)(i % Q);
        const size_t bh = row / N;
        const double ds = P.dstamp[row];
        float4 val = f4(0.f);
        if (!isnan(ds)) {
            const float g = bwd_exp(P.log_lam[bh * (size_t)(T + 1) + T] - ds);
            val = f4_scale(g, reinterpret_cast<const float4*>(P.dM + row * d_v)[q]);
        }
        reinterpret_cast<float4*>(out + row * d_v)[q] = val;
    }
}

}  // namespace sdm
