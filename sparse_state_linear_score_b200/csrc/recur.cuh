// Row pass of the prefill recurrence: one CTA per ((b,h), block of CW value columns).
//
// The recurrence is independent per value column once the slots, weights and gates are
// fixed (p, e, the updates and the output are all column-wise), so each CTA owns a
// CW-wide column slice of one sequence's memory table and walks its chunks in order.
// For chunk j (tokens t0..t0+nt-1), with the plan's decay factors fe and links:
//
//   gather   raw[o]   = row slice of the slot of occurrence o as stored at chunk start
//                       (from M, or from M0 while the slot is pristine)
//   bulk     P0_t     = sum_i w_i |fe_i| raw[t,i]          prediction without in-chunk writes
//            Q0_t     = sum_j u_j |fe_j| raw[t,j]          read without in-chunk writes
//            d_t      = beta_t (v_t - P0_t)                final for tokens without links
//   in-chunk writes are carried as accumulated deltas A[o] (value added to the slot by the
//   writes of this chunk up to occurrence o, decayed to o's token):
//            A[o]     = e^{lam_t - lam_tp} A[link(o)] + w_o d_t
//   linked tokens, level by level (the plan gives each token 1 + the largest level of the
//   earlier tokens it links to; all tokens of one level are resolved in parallel):
//            P_t      = P0_t + sum_{i linked} w_i e^{lam_t - lam_tp} A[link]
//            d_t      = beta_t (v_t - P_t)
//            o_t      = Q0_t + sum_{j linked} u_j e^{lam_t - lam_tp} A[link]   (read after write)
//   scatter  the last write of each slot stores e^{lam_end - lam_t} (|fe| raw + A_own)
//            (its stamp, the chunk-end prefix, is written by the plan).
//
// This is the dense-decay recurrence of §2 Background "Gated DeltaNet" restricted to the
// selected slots (§3 Method "Sparse memory updates", "Sparse retrieval"), evaluated chunk
// by chunk; the in-chunk correction plays the role of the intra-chunk phase of the pages'
// Appendix A.1, with interactions only through shared slots as in Appendix A.2.
#pragma once

#include "common.cuh"
#include "plan.cuh"

namespace sdm {

constexpr int RUN_THREADS = 512;
constexpr int RUN_PAD = 8;  // floats between token blocks: spreads a warp's rows over banks

// Floats per token block of gathered rows (and of A): its slots' CW-wide slices + padding.
__host__ __device__ inline int run_tok_stride(int per_tok, int CW) { return per_tok * CW + RUN_PAD; }

__host__ __device__ inline size_t run_smem_bytes(int C, int W, int R, int CW) {
    const size_t tsw = (size_t)run_tok_stride(W, CW), tsr = (size_t)run_tok_stride(R, CW);
    const size_t no = (size_t)C * (W + R);
    size_t b = 0;
    b += (size_t)C * (tsw + tsr) * 4;   // rows: write blocks, then read blocks
    b += (size_t)C * tsw * 4;           // A (accumulated in-chunk deltas of write occurrences)
    b += (size_t)4 * C * CW * 4;        // v, P, d, o
    b += (size_t)3 * C * 8;             // link masks
    b += (size_t)3 * C * 4;             // lam, beta, level
    b += no * 4 * 5;                    // slot, coef, w, fe, lk
    return b;
}

SDM_DEV void cp_async4(void* smem_dst, const void* gmem_src) {
    unsigned dst = (unsigned)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(gmem_src) : "memory");
}

template <int CW, typename VT>
__global__ void __launch_bounds__(RUN_THREADS, 1) recur_run_kernel(
    const VT* __restrict__ v, const float* __restrict__ beta, const int32_t* __restrict__ widx,
    const float* __restrict__ ww, const int32_t* __restrict__ ridx, const float* __restrict__ rw,
    const float* __restrict__ fe, const int32_t* __restrict__ lk, const float* __restrict__ lam,
    const unsigned long long* __restrict__ tmask, float* __restrict__ M,
    const float* __restrict__ M0, float* __restrict__ out, int H, int T, int N, int d_v, int W,
    int R, int C, int J) {
    constexpr int Q = CW / 4;
    extern __shared__ __align__(16) unsigned char run_smem[];
    const int ncb = d_v / CW;
    const int cb = blockIdx.x % ncb;
    const size_t bh = blockIdx.x / ncb;
    const int h = (int)(bh % H);
    const int c0 = cb * CW;
    float* Mb = M + bh * (size_t)N * d_v;
    const float* M0h = M0 + (size_t)h * N * d_v;
    const size_t occ_base = bh * (size_t)T * (W + R);
    const int tid = threadIdx.x;
    const int tsw = run_tok_stride(W, CW), tsr = run_tok_stride(R, CW);

    const int nomax = C * (W + R);
    float* s_rows = reinterpret_cast<float*>(run_smem);
    float* s_rrows = s_rows + (size_t)C * tsw;  // read blocks
    float* s_A = s_rrows + (size_t)C * tsr;
    float* s_v = s_A + (size_t)C * tsw;
    float* s_P = s_v + C * CW;
    float* s_d = s_P + C * CW;
    float* s_o = s_d + C * CW;
    unsigned long long* s_mask = reinterpret_cast<unsigned long long*>(s_o + C * CW);
    float* s_lam = reinterpret_cast<float*>(s_mask + 3 * C);
    float* s_beta = s_lam + C;
    int* s_lev = reinterpret_cast<int*>(s_beta + C);
    int* s_slot = s_lev + C;
    float* s_coef = reinterpret_cast<float*>(s_slot + nomax);
    float* s_w = s_coef + nomax;
    float* s_fe = s_w + nomax;
    int* s_lk = reinterpret_cast<int*>(s_fe + nomax);

    // position of a write occurrence's (or its A's) slice, and of a read occurrence's slice
    auto wpos = [&](int o) { return (o / W) * tsw + (o % W) * CW; };
    auto rpos = [&](int o) { return (o / R) * tsr + (o % R) * CW; };

    for (int j = 0; j < J; ++j) {
        const int t0 = j * C, nt = min(C, T - t0);
        const int nw = nt * W, no = nt * (W + R);

        // 1. chunk metadata, copied asynchronously
        for (int o = tid; o < no; o += RUN_THREADS) {
            const int32_t* si;
            const float* sw;
            size_t g;
            if (o < nw) {
                const size_t gi = (bh * T + t0) * W + o;
                si = widx + gi;
                sw = ww + gi;
                g = occ_base + (size_t)t0 * W + o;
            } else {
                const size_t gi = (bh * T + t0) * R + (o - nw);
                si = ridx + gi;
                sw = rw + gi;
                g = occ_base + (size_t)T * W + (size_t)t0 * R + (o - nw);
            }
            cp_async4(&s_slot[o], si);
            cp_async4(&s_w[o], sw);
            cp_async4(&s_fe[o], fe + g);
            cp_async4(&s_lk[o], lk + g);
        }
        cp_async_commit();
        if (tid < nt) {
            const size_t tg = bh * T + t0 + tid;
            s_lam[tid] = lam[tg];
            s_beta[tid] = beta[tg];
            s_mask[3 * tid + 0] = tmask[tg * 4 + 0];
            s_mask[3 * tid + 1] = tmask[tg * 4 + 1];
            s_mask[3 * tid + 2] = tmask[tg * 4 + 2];
            s_lev[tid] = (int)tmask[tg * 4 + 3];
        }
        for (int e = tid; e < nt * CW; e += RUN_THREADS) {
            const int t = e / CW, c = e % CW;
            s_v[e] = to_f32(v[(bh * T + t0 + t) * d_v + c0 + c]);
        }
        cp_async_wait_all();
        __syncthreads();

        // 2. gather the row slices as stored at chunk start (from M, or M0 while pristine)
        for (int o = tid; o < no; o += RUN_THREADS) {
            const float f = s_fe[o];
            s_coef[o] = s_w[o] * fabsf(f);
            const int s = s_slot[o];
            const bool ok = slot_ok(s, N);
            const float* src = (signbit(f) ? M0h : Mb) + (ok ? (size_t)s * d_v : 0) + c0;
            float* dst = o < nw ? s_rows + wpos(o) : s_rrows + rpos(o - nw);
#pragma unroll
            for (int q = 0; q < Q; ++q) cp_async16(dst + 4 * q, src + 4 * q, ok);
        }
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();

        // 3. predictions (writes) and reads from the chunk-start memory
        for (int task = tid; task < 2 * nt * CW; task += RUN_THREADS) {
            const bool rd = task >= nt * CW;
            const int e = rd ? task - nt * CW : task;
            const int t = e / CW, c = e % CW;
            float acc = 0.f;
            if (!rd) {
                const float* rr = s_rows + t * tsw + c;
                const float* cf = s_coef + t * W;
                for (int i = 0; i < W; ++i) acc = fmaf(cf[i], rr[i * CW], acc);
                s_P[e] = acc;
                s_d[e] = s_beta[t] * (s_v[e] - acc);
            } else {
                const float* rr = s_rrows + t * tsr + c;
                const float* cf = s_coef + nw + t * R;
                for (int i = 0; i < R; ++i) acc = fmaf(cf[i], rr[i * CW], acc);
                s_o[e] = acc;
            }
        }
        __syncthreads();
        // accumulated deltas of kept write occurrences of tokens without links: A = w d
        for (int o = tid; o < nw; o += RUN_THREADS) {
            const int t = o / W;
            if (!(s_lk[o] & LK_KEEP) || s_lev[t] != 0) continue;
            const float w = s_w[o];
            float* a = s_A + wpos(o);
            const float* dd = s_d + t * CW;
#pragma unroll
            for (int c = 0; c < CW; ++c) a[c] = w * dd[c];
        }

        // 4. tokens with in-chunk links, one level at a time (the barrier of each test
        //    also closes the previous phase)
        for (int lev = 1;; ++lev) {
            const bool mine = tid < nt && s_lev[tid] == lev;
            if (!__syncthreads_or(mine)) break;
            for (int e = tid; e < nt * CW; e += RUN_THREADS) {
                const int t = e / CW, c = e % CW;
                if (s_lev[t] != lev) continue;
                const float lt = s_lam[t];
                float p = s_P[e];
                for (unsigned long long m = s_mask[3 * t]; m; m &= m - 1) {
                    const int o = t * W + (__ffsll((long long)m) - 1);
                    const int L = lk_link(s_lk[o]);
                    if (L < 0) continue;
                    p = fmaf(s_w[o] * expf(lt - s_lam[L / W]), s_A[wpos(L) + c], p);
                }
                s_d[e] = s_beta[t] * (s_v[e] - p);
            }
            __syncthreads();
            for (int e = tid; e < nt * CW; e += RUN_THREADS) {
                const int t = e / CW, c = e % CW;
                if (s_lev[t] != lev) continue;
                const float lt = s_lam[t], d = s_d[e];
                for (unsigned long long m = s_mask[3 * t + 2]; m; m &= m - 1) {
                    const int o = t * W + (__ffsll((long long)m) - 1);
                    const int L = lk_link(s_lk[o]);
                    float a = s_w[o] * d;
                    if (L >= 0) a = fmaf(expf(lt - s_lam[L / W]), s_A[wpos(L) + c], a);
                    s_A[wpos(o) + c] = a;
                }
            }
            __syncthreads();
            for (int e = tid; e < nt * CW; e += RUN_THREADS) {
                const int t = e / CW, c = e % CW;
                if (s_lev[t] != lev) continue;
                const float lt = s_lam[t];
                float qv = s_o[e];
                for (unsigned long long m = s_mask[3 * t + 1]; m; m &= m - 1) {
                    const int o = nw + t * R + (__ffsll((long long)m) - 1);
                    const int L = lk_link(s_lk[o]);
                    if (L < 0) continue;
                    qv = fmaf(s_w[o] * expf(lt - s_lam[L / W]), s_A[wpos(L) + c], qv);
                }
                s_o[e] = qv;
            }
        }

        // 5. outputs
        for (int e = tid; e < nt * Q; e += RUN_THREADS) {
            const int t = e / Q, q = e % Q;
            reinterpret_cast<float4*>(out + (bh * T + t0 + t) * d_v + c0)[q] =
                reinterpret_cast<const float4*>(s_o + t * CW)[q];
        }
        // 6. store the last write of each slot, decayed to the chunk end
        const float lam_end = s_lam[nt - 1];
        for (int e = tid; e < nw * Q; e += RUN_THREADS) {
            const int o = e / Q, q = e % Q;
            const int lko = s_lk[o];
            const int s = s_slot[o];
            if (!(lko & LK_OWNER) || !slot_ok(s, N)) continue;
            const int t = o / W;
            const float4 raw = reinterpret_cast<const float4*>(s_rows + wpos(o))[q];
            float4 a;
            if (lk_link(lko) >= 0) {
                a = reinterpret_cast<const float4*>(s_A + wpos(o))[q];
            } else {
                const float4 dd = reinterpret_cast<const float4*>(s_d + t * CW)[q];
                const float w = s_w[o];
                a = make_float4(w * dd.x, w * dd.y, w * dd.z, w * dd.w);
            }
            const float f = fabsf(s_fe[o]);
            const float g = expf(lam_end - s_lam[t]);
            float4 val;
            val.x = g * fmaf(f, raw.x, a.x);
            val.y = g * fmaf(f, raw.y, a.y);
            val.z = g * fmaf(f, raw.z, a.z);
            val.w = g * fmaf(f, raw.w, a.w);
            reinterpret_cast<float4*>(Mb + (size_t)s * d_v + c0)[q] = val;
        }
        __threadfence_block();
        __syncthreads();
    }
}

}  // namespace sdm
