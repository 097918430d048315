// Backward of the recurrence over one call (Sparse Delta Memory summary, appendix A.3
// "Memory-Efficient Backward": the sparse updates are applied in place and undone while
// the gradients flow back, so no copy of the memory is kept per chunk).
//
// Parallel over value columns.  Once the slots and gates are fixed, the chain through the
// tokens is per column: every row operation acts column by column, and only outputs (dalpha,
// dbeta, dw, du) sum over columns.  Each (b,h) is therefore split into slices of 4 columns
// (one float4), one warp per slice, and every slice walks the tokens one at a time on its
// own.  Stamps belong to slots, not columns, and the slices run at their own pace, so each
// slice keeps private copies of the slot stamps and of the gradient stamps (all copies hold
// the same values at the same point of the walk).  Column sums are written per slice and
// added in a fixed order by bwd_reduce_kernel.
//
// bwd_replay_kernel: from the state at the start of the call, the tokens are replayed in
// place, and before every write the raw rows and stamps of the token's W write slots go to a
// log (T*W rows + T*W stamps per (b,h): the O(T*W*d) record), with Lambda after every token.
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
//           backward log-decay prefix Gam (the sum of log alpha over the later tokens)
//           and per-row stamps.
//           X is linear in its terms, so each lane carries its own share of it.
//           Touched-slots decay: dalpha = sum_i <dMt[s_i], M_{t-1}[s_i]> and only the write
//           rows take the factor alpha.
//   then the write slots' raw rows and stamps are restored from the log.
// On return the state is again the state at the start of the call (its stamps and Lambda
// are never written: the slices work on their private stamp copies).
//
// Lane layout in a slice: lane l owns write rows l, l+32, ... and read rows l, l+32, ...
// (the slice's float4 of each).  A token's loads (stamps, rows, log) all go out in one
// round; a slot both read and written in the token takes the read's gradient update: which
// read shares each write row's slot does not depend on the column, so bwd_links_kernel
// finds it once per call for all slices.
#pragma once

#include <math.h>

#include "common.cuh"

namespace sdm {

constexpr int BWD_MAXO = 128;      // W + R
constexpr int BWD_SLICE_Q = 1;     // float4 columns per slice

// Per-(b,h) records of one call (a byte layout in the workspace); S = slices per (b,h).
struct BwdPtrs {
    float* log_rows;     // [BH][T][W][d_v] raw rows of the write slots before the write
    double* log_stamp;   // [BH][T][W]      their stamps before the write
    double* log_lam;     // [BH][T+1]       Lambda at the start, then after every token
    float* dM;           // [BH][N][d_v]    raw memory gradient rows
    double* pst;         // [S][BH][N]      private slot stamps
    double* pds;         // [S][BH][N]      private gradient stamps (NaN: the row is zero)
    float* p_dww;        // [S][BH*T][W]    per-slice shares of dww
    float* p_drw;        // [S][BH*T][R]    of drw
    double* p_db;        // [S][BH*T]       of dbeta
    double* p_da;        // [S][BH*T]       of dalpha
    double* gam;         // [BH]            the final backward prefix
    int8_t* rpart;       // [BH*T][W]       the read of the same token with the write's slot, or -1
    double* x0;          // [BH][S]         each slice's share of <dM_end, M_T> (every-slot decay)
};

SDM_DEV float4 f4(float a) { return make_float4(a, a, a, a); }
SDM_DEV float4 f4_fma(float s, const float4& x, const float4& y) {
    return make_float4(fmaf(s, x.x, y.x), fmaf(s, x.y, y.y), fmaf(s, x.z, y.z), fmaf(s, x.w, y.w));
}
SDM_DEV float f4_dot(const float4& a, const float4& b) {
    return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}
SDM_DEV float4 f4_scale(float s, const float4& a) {
    return make_float4(s * a.x, s * a.y, s * a.z, s * a.w);
}
SDM_DEV float4 f4_add(const float4& a, const float4& b) {
    return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}
// sum over the warp's rows
SDM_DEV float4 f4_sum_rows(float4 x) {
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        x.x += __shfl_xor_sync(0xffffffffu, x.x, m);
        x.y += __shfl_xor_sync(0xffffffffu, x.y, m);
        x.z += __shfl_xor_sync(0xffffffffu, x.z, m);
        x.w += __shfl_xor_sync(0xffffffffu, x.w, m);
    }
    return x;
}
SDM_DEV double warp_sum_d(double x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
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

// Private stamp copies for every slice; the memory gradient at the end of the call: zero
// (NaN gradient stamps) or dM_end (its rows, stamps 0 = the backward prefix at the end);
// final prefixes and the slices' <dM_end, M_T> shares 0.
__global__ void bwd_init_kernel(const double* __restrict__ stamp, BwdPtrs P, size_t bhn,
                                int S, int BH, const float* __restrict__ dM_end, int d_v) {
    const size_t total = (size_t)S * bhn;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    const size_t i0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const double ds0 = dM_end ? 0.0 : __longlong_as_double(0x7ff8000000000000ll);
    for (size_t i = i0; i < total; i += stride) {
        P.pst[i] = stamp[i % bhn];
        P.pds[i] = ds0;
    }
    if (dM_end) {
        const size_t n4 = bhn * (size_t)(d_v / 4);
        for (size_t i = i0; i < n4; i += stride)
            reinterpret_cast<float4*>(P.dM)[i] = reinterpret_cast<const float4*>(dM_end)[i];
    }
    for (size_t i = i0; i < (size_t)BH; i += stride) P.gam[i] = 0.0;
    for (size_t i = i0; i < (size_t)BH * S; i += stride) P.x0[i] = 0.0;
}

// With an end-of-call gradient and every-slot decay, the sweep's running <dM, M> starts at
// <dM_end, M_T> over the whole table (M_T = the memory the replay left, true values):
// grid (BH * S, row blocks), each block adds its rows' share of one slice (float4 column).
constexpr int BWD_X0_ROWS = 4096;
// Each slice is one float4 column (offset 4*sc) and the replay's stamps sit in slice 0's
// copy; a wider slice would need a loop over its columns here.
static_assert(BWD_SLICE_Q == 1, "bwd_x0_kernel reads one float4 column per slice");
__global__ void __launch_bounds__(256) bwd_x0_kernel(const BwdPtrs P, const float* __restrict__ M,
                                                     const float* __restrict__ M0,
                                                     const float* __restrict__ dM_end, int H,
                                                     int N, int T, int d_v, int S) {
    __shared__ double red[256];
    const int sc = (int)(blockIdx.x % S);
    const size_t bh = blockIdx.x / S;
    const int h = (int)(bh % H);
    const double LT = P.log_lam[bh * (size_t)(T + 1) + T];
    const double* stb = P.pst + bh * (size_t)N;  // slice 0's copy: the stamps after the replay
    const size_t r0 = (size_t)blockIdx.y * BWD_X0_ROWS;
    double acc = 0.0;
    for (size_t r = r0 + threadIdx.x; r < r0 + BWD_X0_ROWS && r < (size_t)N; r += blockDim.x) {
        const double st = stb[r];
        const float f = isnan(st) ? bwd_exp(LT) : bwd_exp(LT - st);
        const float* src = (isnan(st) ? M0 + (size_t)h * N * d_v : M + bh * (size_t)N * d_v) +
                           r * d_v + 4 * sc;
        const float4 m = *reinterpret_cast<const float4*>(src);
        const float4 g = *reinterpret_cast<const float4*>(dM_end + (bh * (size_t)N + r) * d_v + 4 * sc);
        acc += (double)f * (double)f4_dot(g, m);
    }
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int m = 128; m > 0; m >>= 1) {
        if ((int)threadIdx.x < m) red[threadIdx.x] += red[threadIdx.x + m];
        __syncthreads();
    }
    if (threadIdx.x == 0) atomicAdd(&P.x0[bh * (size_t)S + sc], red[0]);
}

// For every write row, the read row of the same token that has its slot (reads are
// distinct within a token), or -1.  One thread per (token, write row).
__global__ void bwd_links_kernel(const int32_t* __restrict__ widx,
                                 const int32_t* __restrict__ ridx, size_t BHT, int W, int R,
                                 int8_t* __restrict__ rpart) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < BHT * W; e += stride) {
        const size_t bt = e / W;
        const int s = widx[e];
        int j0 = -1;
        for (int j = 0; j < R; ++j)
            if (ridx[bt * R + j] == s) {
                j0 = j;
                break;
            }
        rpart[e] = (int8_t)j0;
    }
}

// ---- replay with the log --------------------------------------------------------------
// One warp per (slice, b, h); KPL: write rows per lane (ceil(W / 16)).
template <typename VT, int KPL>
__global__ void __launch_bounds__(32) bwd_replay_kernel(
    const VT* __restrict__ v, const float* __restrict__ alpha, const float* __restrict__ beta,
    const int32_t* __restrict__ widx, const float* __restrict__ ww, float* __restrict__ M,
    const double* __restrict__ lambda, const float* __restrict__ M0, BwdPtrs P, int H, int N,
    int T, int d_v, int W, int S, int touched) {
    const int sc = (int)(blockIdx.x % S);
    const size_t bh = blockIdx.x / S, BH = gridDim.x / S;
    const int h = (int)(bh % H);
    const int lane = threadIdx.x, g = lane;
    const int q = sc;  // the slice's float4 column
    const bool lead = sc == 0;  // slice 0 writes the column-free records
    float* Mb = M + bh * (size_t)N * d_v;
    const float* M0h = M0 + (size_t)h * N * d_v;
    double* stb = P.pst + ((size_t)sc * BH + bh) * N;
    double L = lambda[bh];
    if (lead && lane == 0) P.log_lam[bh * (size_t)(T + 1)] = L;
    int nsl[KPL];
    float nwi[KPL], na = 1.f, nb = 0.f;
    double nla = 0.0;  // log alpha of the next token (0 for a gate outside (0,1], reported)
    auto fetch = [&](int t) {
        const size_t bt = bh * (size_t)T + t;
        na = alpha[bt];
        nb = beta[bt];
        nla = na > 0.f ? log((double)na) : 0.0;
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            const int i = g + 32 * k;
            nsl[k] = i < W ? widx[bt * W + i] : -1;
            nwi[k] = i < W ? ww[bt * W + i] : 0.f;
        }
    };
    if (T > 0) fetch(0);
    for (int t = 0; t < T; ++t) {
        const size_t bt = bh * (size_t)T + t;
        const float a = na, bta = nb;
        const double la = nla;
        int sl[KPL];
        float wi[KPL];
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            sl[k] = nsl[k];
            wi[k] = nwi[k];
            if (sl[k] >= 0 && !slot_ok(sl[k], N)) {
                raise_err(SDM_DEVERR_SLOT_RANGE);
                sl[k] = -1;
            }
        }
        L += la;
        if (!(a > 0.f) && lane == 0) raise_err(SDM_DEVERR_ALPHA);
        const float4 vv = bwd_load_v4<VT>(v + bt * d_v + 4 * q);
        double st[KPL];
        float4 mraw[KPL], m0[KPL];
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            const int s = sl[k];
            st[k] = s >= 0 ? stb[s] : 0.0;
            mraw[k] = m0[k] = f4(0.f);
            if (s >= 0) {
                mraw[k] = reinterpret_cast<const float4*>(Mb + (size_t)s * d_v)[q];
                m0[k] = reinterpret_cast<const float4*>(M0h + (size_t)s * d_v)[q];
            }
        }
        if (t + 1 < T) fetch(t + 1);
        float4 raw[KPL], pp = f4(0.f);
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            const float fk = bwd_factor(st[k], L, touched) * (touched ? a : 1.f);
            raw[k] = f4_scale(fabsf(fk), signbit(fk) ? m0[k] : mraw[k]);  // the decayed row
            pp = f4_fma(wi[k], raw[k], pp);
        }
        const float4 p = f4_sum_rows(pp);
        const float4 dd = make_float4(bta * (vv.x - p.x), bta * (vv.y - p.y), bta * (vv.z - p.z),
                                      bta * (vv.w - p.w));
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            const int s = sl[k];
            if (s < 0) continue;
            const int i = g + 32 * k;
            reinterpret_cast<float4*>(P.log_rows + (bt * W + i) * (size_t)d_v)[q] = mraw[k];
            reinterpret_cast<float4*>(Mb + (size_t)s * d_v)[q] = f4_fma(wi[k], dd, raw[k]);
            stb[s] = L;
            if (lead) P.log_stamp[bt * W + i] = st[k];
        }
        if (lead && lane == 0) P.log_lam[bh * (size_t)(T + 1) + t + 1] = L;
        __syncwarp();  // this token's rows and stamps before the next token's loads
    }
}

// ---- the backward sweep ---------------------------------------------------------------
template <typename VT, int KPL>
__global__ void __launch_bounds__(32) bwd_sweep_kernel(
    const VT* __restrict__ v, const float* __restrict__ alpha, const float* __restrict__ beta,
    const int32_t* __restrict__ widx, const float* __restrict__ ww,
    const int32_t* __restrict__ ridx, const float* __restrict__ rw, float* __restrict__ M,
    const float* __restrict__ M0, BwdPtrs P, const float* __restrict__ dout,
    float* __restrict__ dv_out, int H, int N, int T, int d_v, int W, int R, int S, int touched) {
    const int sc = (int)(blockIdx.x % S);
    const size_t bh = blockIdx.x / S, BH = gridDim.x / S;
    const size_t BHT = BH * (size_t)T;
    const int h = (int)(bh % H);
    const int lane = threadIdx.x, g = lane;
    const int q = sc;  // the slice's float4 column
    float* Mb = M + bh * (size_t)N * d_v;
    const float* M0h = M0 + (size_t)h * N * d_v;
    double* stb = P.pst + ((size_t)sc * BH + bh) * N;
    double* dsb = P.pds + ((size_t)sc * BH + bh) * N;
    float* dMb = P.dM + bh * (size_t)N * d_v;
    const double* lamb = P.log_lam + bh * (size_t)(T + 1);
    // this lane's share of <dM, M> (lane 0 starts with the slice's share of <dM_end, M_T>);
    // the backward log-decay prefix Gam = Lambda_T - Lambda_{t+1} before token t (sums of the
    // same logs as the replay's prefix)
    double X = lane == 0 && !touched ? P.x0[bh * (size_t)S + sc] : 0.0;
    const double LT = T > 0 ? lamb[T] : 0.0;
    // the next token's inputs
    int nrs[KPL], nws[KPL], npj[KPL];
    float nu[KPL], nwi[KPL], na = 1.f, nb = 0.f;
    double nia = 1.0;  // 1 / alpha
    float4 nG = f4(0.f), nv = f4(0.f);
    auto fetch = [&](int t) {
        const size_t bt = bh * (size_t)T + t;
        na = alpha[bt] > 0.f ? alpha[bt] : 1.f;
        nia = 1.0 / (double)na;
        nb = beta[bt];
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            const int j = g + 32 * k;
            nrs[k] = j < R ? ridx[bt * R + j] : -1;
            nu[k] = j < R ? rw[bt * R + j] : 0.f;
            nws[k] = j < W ? widx[bt * W + j] : -1;
            nwi[k] = j < W ? ww[bt * W + j] : 0.f;
            npj[k] = j < W ? (int)P.rpart[bt * W + j] : -1;
        }
        nG = reinterpret_cast<const float4*>(dout + bt * d_v)[q];
        nv = bwd_load_v4<VT>(v + bt * d_v + 4 * q);
    };
    if (T > 0) fetch(T - 1);
    for (int t = T - 1; t >= 0; --t) {
        const size_t bt = bh * (size_t)T + t;
        const float a = na, bta = nb;
        const double ia = nia;
        const double Lt = lamb[t + 1], Lp = lamb[t];
        const double Gam = touched ? 0.0 : LT - Lt;
        int rs[KPL], sl[KPL], pj[KPL];
        float u[KPL], wi[KPL];
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            rs[k] = slot_ok(nrs[k], N) ? nrs[k] : -1;  // the forward reported bad slots
            u[k] = nu[k];
            sl[k] = slot_ok(nws[k], N) ? nws[k] : -1;
            wi[k] = nwi[k];
            pj[k] = npj[k];
        }
        const float4 G = nG, vv = nv;
        // -- one round of loads: read rows (stamps, M, M0, dM), write rows (log, stamps,
        //    current row, M0, dM)
        double rst[KPL], rds[KPL], wso[KPL], wsn[KPL], wds[KPL];
        float4 rM[KPL], rM0[KPL], rG[KPL], lrow[KPL], mc[KPL], m0[KPL], wdm[KPL];
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            const int s = rs[k], sw = sl[k], i = g + 32 * k;
            rst[k] = s >= 0 ? stb[s] : 0.0;
            rds[k] = s >= 0 ? dsb[s] : 0.0;
            wso[k] = sw >= 0 ? P.log_stamp[bt * W + i] : 0.0;
            wsn[k] = sw >= 0 ? stb[sw] : 0.0;
            wds[k] = sw >= 0 ? dsb[sw] : 0.0;
            rM[k] = rM0[k] = rG[k] = lrow[k] = mc[k] = m0[k] = wdm[k] = f4(0.f);
            if (s >= 0) {
                rM[k] = reinterpret_cast<const float4*>(Mb + (size_t)s * d_v)[q];
                rM0[k] = reinterpret_cast<const float4*>(M0h + (size_t)s * d_v)[q];
                rG[k] = reinterpret_cast<const float4*>(dMb + (size_t)s * d_v)[q];
            }
            if (sw >= 0) {
                lrow[k] = reinterpret_cast<const float4*>(P.log_rows + (bt * W + i) * (size_t)d_v)[q];
                mc[k] = reinterpret_cast<const float4*>(Mb + (size_t)sw * d_v)[q];
                m0[k] = reinterpret_cast<const float4*>(M0h + (size_t)sw * d_v)[q];
                wdm[k] = reinterpret_cast<const float4*>(dMb + (size_t)sw * d_v)[q];
            }
        }
        if (t > 0) fetch(t - 1);
        // -- read rows: du_j, dM[r_j] += u_j G, X += u_j du_j
        double xr = 0.0;
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            const int s = rs[k], j = g + 32 * k;
            const float f = bwd_factor(rst[k], Lt, touched);
            const float4 rm = f4_scale(fabsf(f), signbit(f) ? rM0[k] : rM[k]);
            const float gf = (s < 0 || isnan(rds[k])) ? 0.f : bwd_exp(Gam - rds[k]);
            const float du = s >= 0 ? f4_dot(G, rm) : 0.f;
            if (j < R) P.p_drw[((size_t)sc * BHT + bt) * R + j] = du;
            xr += (double)u[k] * du;
            if (s >= 0) {
                reinterpret_cast<float4*>(dMb + (size_t)s * d_v)[q] =
                    f4_fma(u[k], G, gf != 0.f ? f4_scale(gf, rG[k]) : f4(0.f));
                dsb[s] = Gam;
            }
        }
        __syncwarp();  // the read rows' gradient stores before the write rows' (same slot)
        // a write slot that is also read in this token takes that read's weight (its update of
        // the gradient row comes first); read j sits in lane j % 32, row j / 32
        float hu[KPL];
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            hu[k] = 0.f;
#pragma unroll
            for (int k2 = 0; k2 < KPL; ++k2) {
                const float u2 = __shfl_sync(0xffffffffu, u[k2], pj[k] & 31);
                if (pj[k] >= 0 && (pj[k] >> 5) == k2) hu[k] = u2;
            }
        }
        // -- write rows
        float4 mp[KPL], mt[KPL], dm[KPL], pp = f4(0.f), pd = f4(0.f);
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            const int s = sl[k];
            const float fo = bwd_factor(wso[k], Lp, touched);  // value factor at t-1
            const float fn = bwd_factor(wsn[k], Lt, touched);  // at t
            mp[k] = f4_scale(fabsf(fo), signbit(fo) ? m0[k] : lrow[k]);
            mt[k] = f4_scale(fabsf(fn), signbit(fn) ? m0[k] : mc[k]);
            const float gf = (s < 0 || isnan(wds[k])) ? 0.f : bwd_exp(Gam - wds[k]);
            // a row never reached holds stale workspace: select zero, never scale it
            dm[k] = gf != 0.f ? f4_scale(gf, wdm[k]) : f4(0.f);
            dm[k] = f4_fma(hu[k], G, dm[k]);
            if (s < 0) mp[k] = mt[k] = dm[k] = f4(0.f);
            pp = f4_fma(wi[k] * a, mp[k], pp);
            pd = f4_fma(wi[k], dm[k], pd);
        }
        pp = f4_sum_rows(pp);
        pd = f4_sum_rows(pd);
        const float4 e = make_float4(vv.x - pp.x, vv.y - pp.y, vv.z - pp.z, vv.w - pp.w);
        const float4 de = f4_scale(bta, pd);
        if (lane == 0) reinterpret_cast<float4*>(dv_out + bt * d_v)[q] = de;
        double sb = 0.0, s1 = 0.0, s2 = 0.0;  // shares of dbeta, <dM, M_t>, <dMt, M_{t-1}>
        const float scw = touched ? a : 1.f;  // every-slot decay keeps alpha in Gam
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            const int s = sl[k], i = g + 32 * k;
            const float ge = f4_dot(dm[k], e), gm = f4_dot(de, mp[k]);
            const float4 nd = f4_fma(-wi[k], de, dm[k]);  // dMt[s_i]
            const float dw = bta * ge - a * gm;
            if (i < W) P.p_dww[((size_t)sc * BHT + bt) * W + i] = s >= 0 ? dw : 0.f;
            if (s < 0) continue;
            sb += (double)wi[k] * ge;
            s1 += f4_dot(dm[k], mt[k]);
            s2 += f4_dot(nd, mp[k]);
            reinterpret_cast<float4*>(dMb + (size_t)s * d_v)[q] = f4_scale(scw, nd);
            reinterpret_cast<float4*>(Mb + (size_t)s * d_v)[q] = lrow[k];  // restore
            dsb[s] = Gam;
            stb[s] = wso[k];
        }
        double da;
        if (touched) {
            da = s2;
        } else {
            X += xr;
            da = (X - s1) * ia + s2;
            X = (double)a * da;
        }
        da = warp_sum_d(da);
        sb = warp_sum_d(sb);
        if (lane == 0) {
            P.p_da[(size_t)sc * BHT + bt] = da;
            P.p_db[(size_t)sc * BHT + bt] = sb;
        }
        __syncwarp();  // this token's stores before the next token's loads
    }
    if (sc == 0 && lane == 0) P.gam[bh] = touched || T == 0 ? 0.0 : LT - lamb[0];
}

// The per-slice shares summed in slice order: dww, drw, dbeta, dalpha.
__global__ void bwd_reduce_kernel(const BwdPtrs P, int S, size_t BHT, int W, int R,
                                  float* __restrict__ dww, float* __restrict__ drw,
                                  float* __restrict__ dbeta, float* __restrict__ dalpha) {
    const size_t nw = BHT * W, nr = BHT * R;
    const size_t total = nw + nr + 2 * BHT;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        if (i < nw) {
            float acc = 0.f;
            for (int c = 0; c < S; ++c) acc += P.p_dww[c * nw + i];
            dww[i] = acc;
        } else if (i < nw + nr) {
            const size_t k = i - nw;
            float acc = 0.f;
            for (int c = 0; c < S; ++c) acc += P.p_drw[c * nr + k];
            drw[k] = acc;
        } else {
            const bool is_b = i < nw + nr + BHT;
            const size_t k = i - nw - nr - (is_b ? 0 : BHT);
            const double* src = is_b ? P.p_db : P.p_da;
            double acc = 0.0;
            for (int c = 0; c < S; ++c) acc += src[c * BHT + k];
            (is_b ? dbeta : dalpha)[k] = (float)acc;
        }
    }
}

// Dense gradient with respect to the state at the start of the call: dM_in[s] = raw *
// e^{Gam_final - stamp} (zero for rows never reached).  The gradient stamps of slice 0
// (all slices end with the same ones).
__global__ void bwd_dense_kernel(const BwdPtrs P, int N, int d_v, size_t n_rows,
                                 float* __restrict__ out) {
    const int Q = d_v / 4;
    const size_t total = n_rows * Q;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        const size_t row = i / Q;
        const int q = (int)(i % Q);
        const size_t bh = row / N;
        const double ds = P.pds[row];
        float4 val = f4(0.f);
        if (!isnan(ds)) {
            const float g = bwd_exp(P.gam[bh] - ds);
            val = f4_scale(g, reinterpret_cast<const float4*>(P.dM + row * d_v)[q]);
        }
        reinterpret_cast<float4*>(out + row * d_v)[q] = val;
    }
}

}  // namespace sdm
