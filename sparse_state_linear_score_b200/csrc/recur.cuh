// Row pass of the prefill recurrence: one CTA per ((b,h), block of CW value columns).
//
// The recurrence is independent per value column once the slots, weights and gates are
// fixed (p, e, the updates and the output are all column-wise), so each CTA owns a CW-wide
// column slice of one sequence's memory table and walks its chunks in order.  For chunk j
// (tokens t0..t0+nt-1), with the plan's decay factors fe, links and matrices Minv, G:
//
//   gather   raw[o]  = slice of the row of occurrence o's slot as stored at chunk start (from
//                      M, or M0 while pristine), issued one chunk ahead; rows the previous
//                      chunk stores after their gather are taken from that chunk's stores
//   dense    P0_t    = sum_i w_i |fe_i| raw[t,i],  Q0_t = sum_j u_j |fe_j| raw[t,j]
//            d       = Minv (beta (v - P0))          (in-chunk writes seen by later predictions)
//            o_t     = Q0_t + sum_tau G[t][tau] d_tau (read after write)
//                    = Q0_t + (GM beta (v - P0))_t    (GM = G Minv from the plan)
//   store    the last write of each slot stores e^{lam_end - lam_t} |fe| raw + sum over the
//            chunk's writes of that slot up to it of w e^{lam_end - lam_tau} d_tau (both
//            coefficients from the plan; its stamp, the chunk-end prefix, too).
//
// This is the dense-decay recurrence of §2 Background "Gated DeltaNet" restricted to the
// selected slots (§3 Method "Sparse memory updates", "Sparse retrieval"), evaluated chunk by
// chunk as in the pages' Appendix A.1 (intra-chunk triangular solve, sequential chunks).
#pragma once

#include "common.cuh"
#include "plan.cuh"

namespace sdm {

constexpr int RUN_THREADS = 512;
constexpr int RUN_PAD = 8;  // floats between token blocks: spreads a warp's rows over banks

// Floats per token block of gathered rows: its slots' CW-wide slices + padding.
__host__ __device__ inline int run_tok_stride(int per_tok, int CW) { return per_tok * CW + RUN_PAD; }
// Row stride of Minv / G in shared memory (16-byte rows, 4 floats apart in banks).
__host__ __device__ inline int run_mat_stride(int C) { return C + 4; }

// x / d for 0 <= x < 2^16 and 1 <= d <= 64 as one multiply-high: with m = ceil(2^32 / d),
// m*d - 2^32 < d, so the rounding error x*(m*d - 2^32) < 2^22 never reaches 2^32.
struct FastDiv {
    unsigned m, d;
    __host__ __device__ explicit FastDiv(unsigned dd) : m((unsigned)((0x100000000ull + dd - 1) / dd)), d(dd) {}
    SDM_DEV int div(int x) const { return (int)__umulhi((unsigned)x, m); }
    SDM_DEV int mod(int x) const { return x - div(x) * (int)d; }
};

// Row stride of a token's coefficients in shared memory: W + 1 (or R + 1) keeps the four
// tokens a warp reads at once in different banks.
__host__ __device__ inline int run_coef_stride(int per_tok) { return per_tok + 1; }

__host__ __device__ inline size_t run_smem_bytes(int C, int W, int R, int CW) {
    const size_t tsw = (size_t)run_tok_stride(W, CW), tsr = (size_t)run_tok_stride(R, CW);
    const size_t no = (size_t)C * (W + R);
    size_t b = 0;
    b += (size_t)2 * C * (tsw + tsr) * 4;           // rows, two chunks: write blocks, read blocks
    b += (size_t)2 * 2 * C * run_mat_stride(C) * 4; // Minv and G, two chunks
    b += (size_t)4 * C * CW * 4;                    // v, rhs, d, Q0
    b += (size_t)C * 4;                             // beta
    b += no * 5 * 4;                                // slot, sc, a, lk, hz
    b += (size_t)C * (run_coef_stride(W) + run_coef_stride(R)) * 4;  // coef (padded rows)
    return b;
}

constexpr int RUN_OPT = PLAN_MAX_OCC / RUN_THREADS;  // occurrences per thread per chunk



// One chunk's metadata held in registers while the previous chunk computes.
struct RunPrefetch {
    int slot[RUN_OPT], lk[RUN_OPT], hz[RUN_OPT];
    float c[RUN_OPT], sc[RUN_OPT], a[RUN_OPT];
    float beta, v;
};

template <int CW, typename VT>
__global__ void __launch_bounds__(RUN_THREADS, 1) recur_run_kernel(
    const VT* __restrict__ v, const float* __restrict__ beta, const int32_t* __restrict__ rs,
    const float* __restrict__ rc, const float* __restrict__ rsc, const float* __restrict__ ra,
    const int32_t* __restrict__ lk, const int32_t* __restrict__ hz, const float* __restrict__ mats, float* __restrict__ M, const float* __restrict__ M0,
    float* __restrict__ out, int H, int T, int N, int d_v, int W, int R, int C, int J) {
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
    const int MS = run_mat_stride(C);

    const int nomax = C * (W + R);
    float* s_rowbuf = reinterpret_cast<float*>(run_smem);  // [2][C*(tsw+tsr)]
    const int rowbuf = C * (tsw + tsr);
    float* s_matbuf = s_rowbuf + 2 * (size_t)rowbuf;       // [2][2][C][MS]
    const int matbuf = 2 * C * MS;
    float* s_v = s_matbuf + 2 * (size_t)matbuf;
    float* s_rhs = s_v + C * CW;
    float* s_d = s_rhs + C * CW;
    float* s_q = s_d + C * CW;
    float* s_beta = s_q + C * CW;
    int* s_slot = reinterpret_cast<int*>(s_beta + C);
    const int csw = run_coef_stride(W), csr = run_coef_stride(R);
    float* s_coef = reinterpret_cast<float*>(s_slot + nomax);  // [C][W+1], then [C][R+1]
    float* s_sc = s_coef + C * (csw + csr);  // writes: store coefficient of the write
    float* s_a = s_sc + nomax;                // writes: store coefficient of the gathered row
    int* s_lk = reinterpret_cast<int*>(s_a + nomax);
    int* s_hz = s_lk + nomax;                 // occurrences whose row the previous chunk stores

    const FastDiv fW((unsigned)W), fR((unsigned)R);
    // position of a write occurrence's slice, and of a read occurrence's slice
    auto wpos = [&](int o) { const int t = fW.div(o); return t * tsw + (o - t * W) * CW; };
    auto rpos = [&](int o) { const int t = fR.div(o); return C * tsw + t * tsr + (o - t * R) * CW; };
    auto pos = [&](int o, int nw) { return o < nw ? wpos(o) : rpos(o - nw); };
    // padded coefficient index of occurrence o
    auto cpos = [&](int o, int nw) {
        if (o < nw) { const int t = fW.div(o); return t * csw + (o - t * W); }
        const int r = o - nw, t = fR.div(r);
        return C * csw + t * csr + (r - t * R);
    };

    // registers <- metadata of chunk jn
    auto fetch = [&](int jn, RunPrefetch& F) {
        const int t0 = jn * C, nt = min(C, T - t0), nw = nt * W, no = nt * (W + R);
#pragma unroll
        for (int k = 0; k < RUN_OPT; ++k) {
            const int o = tid + k * RUN_THREADS;
            F.slot[k] = 0x7fffffff;
            if (o < no) {
                const size_t g = o < nw ? occ_base + (size_t)t0 * W + o
                                        : occ_base + (size_t)T * W + (size_t)t0 * R + (o - nw);
                F.slot[k] = rs[g];
                F.c[k] = rc[g];
                F.lk[k] = lk[g];
                F.hz[k] = hz[occ_base + (size_t)t0 * (W + R) + o];
                if (o < nw) {
                    F.sc[k] = rsc[g];
                    F.a[k] = ra[g];
                }
            }
        }
        if (tid < nt) {
            const size_t tg = bh * T + t0 + tid;
            F.beta = beta[tg];
        }
        if (tid < nt * CW) F.v = to_f32(v[(bh * T + t0 + tid / CW) * d_v + c0 + tid % CW]);
    };
    // shared <- registers (chunk jn's metadata)
    auto publish = [&](int jn, const RunPrefetch& F) {
        const int t0 = jn * C, nt = min(C, T - t0), nw = nt * W, no = nt * (W + R);
#pragma unroll
        for (int k = 0; k < RUN_OPT; ++k) {
            const int o = tid + k * RUN_THREADS;
            if (o < no) {
                s_slot[o] = F.slot[k];
                s_coef[cpos(o, nw)] = F.c[k];
                s_lk[o] = F.lk[k];
                s_hz[o] = F.hz[k];
                if (o < nw) {
                    s_sc[o] = F.sc[k];
                    s_a[o] = F.a[k];
                }
            }
        }
        if (tid < nt) {
            s_beta[tid] = F.beta;
        }
        if (tid < nt * CW) s_v[tid] = F.v;
    };
    // chunk jn's row gathers (rows as stored now; the ones its previous chunk is about to
    // store are replaced later from that chunk's stores) and its Minv / G.  The Q 16-byte
    // pieces of one occurrence's slice are fetched by Q adjacent lanes in one instruction,
    // so each slice is a single request to the memory system.
    auto gather = [&](int jn, const RunPrefetch& F, float* rbuf, float* mbuf) {
        const int t0 = jn * C, nt = min(C, T - t0), nw = nt * W, no = nt * (W + R);
        const int lane = tid & 31, wbase = tid - lane;
        constexpr int PER = 32 / Q;  // occurrences per instruction
#pragma unroll
        for (int k = 0; k < RUN_OPT; ++k) {
#pragma unroll
            for (int r = 0; r < Q; ++r) {
                const int src_lane = r * PER + lane / Q;
                const int sw = __shfl_sync(0xffffffffu, F.slot[k], src_lane);
                const int o = wbase + k * RUN_THREADS + src_lane;
                const int q = lane % Q;
                if (o < no) {
                    const int s = sw & 0x7fffffff;
                    const bool ok = s < N;
                    const float* src = (sw < 0 ? M0h : Mb) + (ok ? (size_t)s * d_v : 0) + c0 + 4 * q;
                    cp_async16(rbuf + pos(o, nw) + 4 * q, src, ok);
                }
            }
        }
        const float* msrc = mats + ((bh * J + jn) * 2) * (size_t)(C * C);
        for (int e = tid; e < 2 * C * (C / 4); e += RUN_THREADS) {  // 16-byte pieces
            const int row = e / (C / 4), piece = e % (C / 4);
            cp_async16(mbuf + row * MS + 4 * piece, msrc + row * C + 4 * piece, true);
        }
        cp_async_commit();
    };

    RunPrefetch F1, F2;  // chunk j+1, chunk j+2
    {
        RunPrefetch F0;
        fetch(0, F0);
        gather(0, F0, s_rowbuf, s_matbuf);
        publish(0, F0);
        if (J > 1) fetch(1, F1);
    }
    for (int j = 0; j < J; ++j) {
        const int t0 = j * C, nt = min(C, T - t0);
        const int nw = nt * W, no = nt * (W + R);
        float* rows = s_rowbuf + (size_t)(j & 1) * rowbuf;
        float* prev_rows = s_rowbuf + (size_t)((j + 1) & 1) * rowbuf;
        const float* Minv = s_matbuf + (size_t)(j & 1) * matbuf;
        const float* G = Minv + C * MS;  // GM = G Minv
        cp_async_wait_all();
        __syncthreads();
        // 1. rows the previous chunk stored after they were gathered: take its stored values
        if (j > 0) {
            for (int e = tid; e < no * Q; e += RUN_THREADS) {
                const int hv = s_hz[e / Q];
                if (hv < 0) break;  // end of the chunk's list
                const int o = hv & 0xffff, pv = hv >> 16, q = e % Q;
                reinterpret_cast<float4*>(rows + pos(o, nw))[q] =
                    reinterpret_cast<const float4*>(prev_rows + wpos(pv))[q];
            }
        }
        __syncthreads();
        // 2. the next chunk's gathers and matrices (overlap with this chunk's compute)
        if (j + 1 < J)
            gather(j + 1, F1, prev_rows, s_matbuf + (size_t)((j + 1) & 1) * matbuf);
        if (j + 2 < J) fetch(j + 2, F2);

        // 3. predictions (writes) and reads from the chunk-start memory
        for (int task = tid; task < 2 * nt * CW; task += RUN_THREADS) {
            const bool rd = task >= nt * CW;
            const int e = rd ? task - nt * CW : task;
            const int t = e / CW, c = e % CW;
            // four independent partial sums per dot product (latency of the smem loads)
            const float* rr = rd ? rows + C * tsw + t * tsr + c : rows + t * tsw + c;
            const float* cf = rd ? s_coef + C * csw + t * csr : s_coef + t * csw;
            const int n_i = rd ? R : W;
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
            int i = 0;
            for (; i + 4 <= n_i; i += 4) {
                a0 = fmaf(cf[i], rr[i * CW], a0);
                a1 = fmaf(cf[i + 1], rr[(i + 1) * CW], a1);
                a2 = fmaf(cf[i + 2], rr[(i + 2) * CW], a2);
                a3 = fmaf(cf[i + 3], rr[(i + 3) * CW], a3);
            }
            for (; i < n_i; ++i) a0 = fmaf(cf[i], rr[i * CW], a0);
            const float acc = (a0 + a1) + (a2 + a3);
            if (!rd) s_rhs[e] = s_beta[t] * (s_v[e] - acc);
            else s_q[e] = acc;
        }
        __syncthreads();
        // 4. d = Minv rhs and o = Q0 + GM rhs (both lower triangular, zero beyond the chunk)
        for (int task = tid; task < 2 * nt * CW; task += RUN_THREADS) {
            const bool oo = task >= nt * CW;
            const int e = oo ? task - nt * CW : task;
            const int t = e / CW, c = e % CW;
            const float* mr = (oo ? G : Minv) + t * MS;
            float a0 = 0.f, a1 = 0.f;
            int tau = 0;
            for (; tau + 2 <= t + 1; tau += 2) {
                a0 = fmaf(mr[tau], s_rhs[tau * CW + c], a0);
                a1 = fmaf(mr[tau + 1], s_rhs[(tau + 1) * CW + c], a1);
            }
            if (tau <= t) a0 = fmaf(mr[tau], s_rhs[tau * CW + c], a0);
            if (oo) out[(bh * T + t0 + t) * d_v + c0 + c] = s_q[e] + (a0 + a1);
            else s_d[e] = a0 + a1;
        }
        __syncthreads();
        // 5. the stores of the chunk's last writes
        for (int e = tid; e < nw * Q; e += RUN_THREADS) {
            const int o = e / Q, q = e % Q;
            const int lko = s_lk[o];
            const int s = s_slot[o] & 0x7fffffff;
            if (!(lko & LK_OWNER) || s >= N) continue;
            // this write plus the chunk's earlier writes of the slot, decayed to the chunk end
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int L = o; L >= 0; L = lk_link(s_lk[L])) {
                const int tp = fW.div(L);
                const float cfa = s_sc[L];
                const float4 dd = reinterpret_cast<const float4*>(s_d + tp * CW)[q];
                a.x = fmaf(cfa, dd.x, a.x);
                a.y = fmaf(cfa, dd.y, a.y);
                a.z = fmaf(cfa, dd.z, a.z);
                a.w = fmaf(cfa, dd.w, a.w);
            }
            float4* rp = reinterpret_cast<float4*>(rows + wpos(o)) + q;
            const float4 raw = *rp;
            const float f = s_a[o];
            float4 val;
            val.x = fmaf(f, raw.x, a.x);
            val.y = fmaf(f, raw.y, a.y);
            val.z = fmaf(f, raw.z, a.z);
            val.w = fmaf(f, raw.w, a.w);
            reinterpret_cast<float4*>(Mb + (size_t)s * d_v + c0)[q] = val;
            *rp = val;  // the next chunk forwards it
        }
        __threadfence_block();
        __syncthreads();
        // 6. next chunk's metadata into shared memory; rotate the prefetch registers
        if (j + 1 < J) publish(j + 1, F1);
        F1 = F2;
    }
}

}  // namespace sdm
