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
//   linked tokens, in token order (one warp, lanes = columns):
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

constexpr int RUN_THREADS = 256;

__host__ __device__ inline size_t run_smem_bytes(int C, int W, int R, int CW) {
    const size_t no = (size_t)C * (W + R), nw = (size_t)C * W;
    size_t b = 0;
    b += no * CW * 4;                   // rows
    b += nw * CW * 4;                   // A
    b += (size_t)4 * C * CW * 4;        // v, P, d, o
    b += (size_t)3 * C * 8;             // masks
    b += (size_t)2 * C * 4;             // lam, beta
    b += no * 4 * 5;                    // slot, coef, w, fe, lk
    return b;
}

template <int CW, typename VT>
__global__ void __launch_bounds__(RUN_THREADS) recur_run_kernel(
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

    const int nomax = C * (W + R), nwmax = C * W;
    float* s_rows = reinterpret_cast<float*>(run_smem);
    float* s_A = s_rows + (size_t)nomax * CW;
    float* s_v = s_A + (size_t)nwmax * CW;
    float* s_P = s_v + C * CW;
    float* s_d = s_P + C * CW;
    float* s_o = s_d + C * CW;
    unsigned long long* s_mask = reinterpret_cast<unsigned long long*>(s_o + C * CW);
    float* s_lam = reinterpret_cast<float*>(s_mask + 3 * C);
    float* s_beta = s_lam + C;
    int* s_slot = reinterpret_cast<int*>(s_beta + C);
    float* s_coef = reinterpret_cast<float*>(s_slot + nomax);
    float* s_w = s_coef + nomax;
    float* s_fe = s_w + nomax;
    int* s_lk = reinterpret_cast<int*>(s_fe + nomax);

    for (int j = 0; j < J; ++j) {
        const int t0 = j * C, nt = min(C, T - t0);
        const int nw = nt * W, no = nt * (W + R);

        // 1. chunk metadata
        for (int o = tid; o < no; o += RUN_THREADS) {
            int s;
            float w;
            size_t g;
            if (o < nw) {
                const size_t gi = (bh * T + t0) * W + o;
                s = widx[gi];
                w = ww[gi];
                g = occ_base + (size_t)t0 * W + o;
            } else {
                const size_t gi = (bh * T + t0) * R + (o - nw);
                s = ridx[gi];
                w = rw[gi];
                g = occ_base + (size_t)T * W + (size_t)t0 * R + (o - nw);
            }
            const float f = fe[g];
            s_slot[o] = s;
            s_w[o] = w;
            s_fe[o] = f;
            s_coef[o] = w * fabsf(f);
            s_lk[o] = lk[g];
        }
        for (int t = tid; t < nt; t += RUN_THREADS) {
            s_lam[t] = lam[bh * T + t0 + t];
            s_beta[t] = beta[bh * T + t0 + t];
            s_mask[3 * t + 0] = tmask[(bh * T + t0 + t) * 3 + 0];
            s_mask[3 * t + 1] = tmask[(bh * T + t0 + t) * 3 + 1];
            s_mask[3 * t + 2] = tmask[(bh * T + t0 + t) * 3 + 2];
        }
        for (int e = tid; e < nt * CW; e += RUN_THREADS) {
            const int t = e / CW, c = e % CW;
            s_v[e] = to_f32(v[(bh * T + t0 + t) * d_v + c0 + c]);
        }
        __syncthreads();

        // 2. gather the row slices as stored at chunk start
        for (int e = tid; e < no * Q; e += RUN_THREADS) {
            const int o = e / Q, q = e % Q;
            const int s = s_slot[o];
            const bool ok = slot_ok(s, N);
            const float* src = (signbit(s_fe[o]) ? M0h : Mb) + (ok ? (size_t)s * d_v : 0) + c0 + 4 * q;
            cp_async16(&s_rows[(size_t)o * CW + 4 * q], src, ok);
        }
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();

        // 3. predictions and reads from the chunk-start memory
        for (int e = tid; e < nt * CW; e += RUN_THREADS) {
            const int t = e / CW, c = e % CW;
            float p = 0.f, qv = 0.f;
            const int ow = t * W, orr = nw + t * R;
            for (int i = 0; i < W; ++i) p = fmaf(s_coef[ow + i], s_rows[(size_t)(ow + i) * CW + c], p);
            for (int i = 0; i < R; ++i) qv = fmaf(s_coef[orr + i], s_rows[(size_t)(orr + i) * CW + c], qv);
            s_P[e] = p;
            s_d[e] = s_beta[t] * (s_v[e] - p);
            s_o[e] = qv;
        }
        __syncthreads();
        // accumulated deltas of tokens without links: A = w d
        for (int e = tid; e < nw * CW; e += RUN_THREADS) {
            const int o = e / CW, c = e % CW;
            const int t = o / W;
            if ((s_lk[o] & LK_KEEP) && !(s_mask[3 * t] | s_mask[3 * t + 1]))
                s_A[e] = s_w[o] * s_d[t * CW + c];
        }
        __syncthreads();

        // 4. tokens with in-chunk links, in order
        if (tid < 32) {
            const int c = tid;
            for (int t = 0; t < nt; ++t) {
                const unsigned long long wm = s_mask[3 * t], rm = s_mask[3 * t + 1],
                                         am = s_mask[3 * t + 2];
                if (!(wm | rm)) continue;
                if (c < CW) {
                    const float lt = s_lam[t];
                    float p = s_P[t * CW + c];
                    for (unsigned long long m = wm; m; m &= m - 1) {
                        const int o = t * W + (__ffsll((long long)m) - 1);
                        const int L = lk_link(s_lk[o]);
                        if (L < 0) continue;
                        p = fmaf(s_w[o] * expf(lt - s_lam[L / W]), s_A[(size_t)L * CW + c], p);
                    }
                    const float d = s_beta[t] * (s_v[t * CW + c] - p);
                    s_d[t * CW + c] = d;
                    for (unsigned long long m = am; m; m &= m - 1) {
                        const int o = t * W + (__ffsll((long long)m) - 1);
                        const int L = lk_link(s_lk[o]);
                        float a = s_w[o] * d;
                        if (L >= 0) a = fmaf(expf(lt - s_lam[L / W]), s_A[(size_t)L * CW + c], a);
                        s_A[(size_t)o * CW + c] = a;
                    }
                    float qv = s_o[t * CW + c];
                    for (unsigned long long m = rm; m; m &= m - 1) {
                        const int o = nw + t * R + (__ffsll((long long)m) - 1);
                        const int L = lk_link(s_lk[o]);
                        if (L < 0) continue;
                        qv = fmaf(s_w[o] * expf(lt - s_lam[L / W]), s_A[(size_t)L * CW + c], qv);
                    }
                    s_o[t * CW + c] = qv;
                }
                __syncwarp();
            }
        }
        __syncthreads();

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
            const int s = s_slot[o];
            if (!(s_lk[o] & LK_OWNER) || !slot_ok(s, N)) continue;
            const int t = o / W, i = o % W;
            const bool linked = (s_mask[3 * t] >> i) & 1ull;
            const float4 raw = reinterpret_cast<const float4*>(s_rows + (size_t)o * CW)[q];
            float4 a;
            if (linked) {
                a = reinterpret_cast<const float4*>(s_A + (size_t)o * CW)[q];
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
