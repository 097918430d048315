// Single-token step for every (b,h): the CTA that steps a sequence owns its full slot rows,
// so it reads and writes the stamps directly (no plan needed).  Two forms: decode_kernel (one
// CTA per sequence, after a separate scoring launch) and decode_fused_kernel (clusters of two
// CTAs that score four sequences' keys and queries and then step them, one launch per step).
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
#include "score_rows.cuh"

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

// Decode smem views (decode_smem_bytes): partial sums and the occurrences' slots, weights and
// decay factors (the sign bit marks a pristine row, read from M0), writes first.
struct DecSmem {
    float* pp;   // [8][d_v] partial p
    float* po;   // [8][d_v] partial out
    int* slot;   // [W+R]
    float* w;    // [W+R]
    float* f;    // [W+R]
    float* uw;   // [W] read weight that lands on write row i
    int* rm;     // [R] read j is also written
    SDM_DEV DecSmem(unsigned char* p, int W, int R, int d_v) {
        pp = reinterpret_cast<float*>(p);
        po = pp + DECODE_WARPS * d_v;
        slot = reinterpret_cast<int*>(po + DECODE_WARPS * d_v);
        w = reinterpret_cast<float*>(slot + W + R);
        f = w + W + R;
        uw = f + W + R;
        rm = reinterpret_cast<int*>(uw + W);
    }
};

// Decay factor of an occurrence's row from its slot's stamp (NaN: pristine, the sign bit set):
// e^{Lambda' - stamp}, or under touched-slots decay alpha for a write slot and 1 for a read.
SDM_DEV float decode_factor(double st, double Lnew, bool write, float a_t, int touched) {
    if (touched) {
        const float fv = write ? a_t : 1.f;
        return isnan(st) ? -fv : fv;
    }
    return isnan(st) ? -(float)exp(Lnew) : (float)exp(Lnew - st);
}

// The rows of one sequence's step, once its occurrences (slot, weight, factor) are in d's
// arrays -- each warp reads the entries of its own rows (written by itself, or by any thread
// before a block barrier): p = sum_i w_i seen(s_i), d = beta (v - p), the written rows and
// their stamps, out = sum_j u_j (r_j after the write), Lambda'.
template <typename VT, int RPW, int QPL>
SDM_DEV void decode_apply(size_t bh, const float4 (&vv)[QPL], float bt, double Lnew, const DecSmem& d,
                          float* __restrict__ M, double* __restrict__ stamp,
                          double* __restrict__ lambda, const float* __restrict__ M0,
                          float* __restrict__ out, int H, int N, int d_v, int W, int R) {
    const int h = (int)(bh % H);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int no = W + R;
    const int Q = d_v / 4;
    float* s_pp = d.pp;
    float* s_po = d.po;
    int* s_slot = d.slot;
    float* s_w = d.w;
    float* s_f = d.f;
    float* s_uw = d.uw;
    int* s_rm = d.rm;
    float* Mb = M + bh * (size_t)N * d_v;
    const float* M0h = M0 + (size_t)h * N * d_v;
    double* stb = stamp + bh * (size_t)N;
    __syncwarp();
    float4 wr[RPW][QPL], rd[RPW][QPL];
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
        const int i = warp + DECODE_WARPS * k;
        const int si = i < W ? s_slot[i] : -1, sj = i < R ? s_slot[W + i] : -1;
        const float fi = i < W ? s_f[i] : 0.f, fj = i < R ? s_f[W + i] : 0.f;
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

// The step of sequence bh by the whole CTA (DECODE_THREADS threads; dec_smem holds
// decode_smem_bytes).  wi / wv and ri / rv are the token's W write and R read slots and
// weights.  With dep_wait the CTA waits for the launch before it (programmatic dependent
// launch) after reading v, alpha and beta and before anything that launch writes.  RPW: rows
// of each role per warp (ceil(max(W, R) / 8)); QPL: float4 columns per lane.
template <typename VT, int RPW, int QPL>
SDM_DEV void decode_seq_step(size_t bh, const VT* __restrict__ v, const float* __restrict__ alpha,
                             const float* __restrict__ beta, const int32_t* wi, const float* wv,
                             const int32_t* ri, const float* rv, float* __restrict__ M,
                             double* __restrict__ stamp, double* __restrict__ lambda,
                             const float* __restrict__ M0, float* __restrict__ out, int H, int N,
                             int d_v, int W, int R, int touched, unsigned char* dec_smem,
                             bool dep_wait) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Q = d_v / 4;
    const DecSmem d(dec_smem, W, R, d_v);
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
    const float a_t = alpha[bh];
    double la = 0.0;
    if (a_t > 0.f) la = log((double)a_t);
    else if (tid == 0) raise_err(SDM_DEVERR_ALPHA);
    if (dep_wait) asm volatile("griddepcontrol.wait;" ::: "memory");
    const double Lnew = lambda[bh] + la;  // Lambda'
    // lane k fetches write row w + 8k, lane 16 + k read row w + 8k: slot, weight, and the
    // decay factor from the slot's stamp
    {
        const bool rl = lane >= 16;
        const int k = lane & 15, i = warp + DECODE_WARPS * k;
        if (k < RPW && i < (rl ? R : W)) {
            int sl = rl ? ri[i] : wi[i];
            const float w = rl ? rv[i] : wv[i];
            float f = 0.f;
            if (!slot_ok(sl, N)) {
                raise_err(SDM_DEVERR_SLOT_RANGE);
                sl = -1;
            } else {
                f = decode_factor(stb[sl], Lnew, !rl, a_t, touched);
            }
            const int o = rl ? W + i : i;
            d.slot[o] = sl;
            d.w[o] = w;
            d.f[o] = f;
        }
    }
    decode_apply<VT, RPW, QPL>(bh, vv, bt, Lnew, d, M, stamp, lambda, M0, out, H, N, d_v, W, R);
}

// One CTA per sequence, launched after the scoring launch as its programmatic dependent: the
// prologue (v, alpha, beta) overlaps the scorer's tail, the slots are read after the wait.
template <typename VT, int RPW, int QPL>
__global__ void __launch_bounds__(DECODE_THREADS) decode_kernel(
    const VT* __restrict__ v, const float* __restrict__ alpha, const float* __restrict__ beta,
    const int32_t* __restrict__ widx, const float* __restrict__ ww,
    const int32_t* __restrict__ ridx, const float* __restrict__ rw, float* __restrict__ M,
    double* __restrict__ stamp, double* __restrict__ lambda, const float* __restrict__ M0,
    float* __restrict__ out, int H, int N, int d_v, int W, int R, int touched) {
    extern __shared__ __align__(16) unsigned char dec_smem[];
    const size_t bh = blockIdx.x;
    decode_seq_step<VT, RPW, QPL>(bh, v, alpha, beta, widx + bh * W, ww + bh * W, ridx + bh * R,
                                  rw + bh * R, M, stamp, lambda, M0, out, H, N, d_v, W, R, touched,
                                  dec_smem, true);
}

// ---- the whole decode step in one launch --------------------------------------------------
//
// A cluster of two CTAs takes four sequences b0..b0+3 of one head.  CTA rank r scores the four
// rows of role r (rank 0: the keys against the write tables, rank 1: the queries against the
// read tables) with the row scorer's phases (tensor-core dot products, per-half top-k,
// staircase combine, softmax), writes the selections out, and right away fetches the stamps
// of its selected slots into decay factors.  After a cluster barrier each CTA copies, through
// distributed shared memory, the other role's selections of the two sequences it steps (rank
// r: b0 + 2r and b0 + 2r + 1), and runs their recurrence steps (decode_apply).  The
// selections never make a round trip through memory, each CTA streams one sub-key table,
// and there is one launch per step.  k_half, W, R <= 32; bf16 x with d_k = 128 and
// 64 < n <= 32 * PL.
struct DecArgs {
    const void* v;
    const float* alpha;
    const float* beta;
    float* M;
    double* stamp;
    double* lambda;
    const float* M0;
    float* out;
    int N, d_v, touched;
};

// Shared memory of the fused step: the row scorer's (tensor-core head and common area) and
// the four rows' selections (slot, weight, factor) and Lambda'.  The two steps' partial sums
// and occurrence arrays reuse the two sub-key buffers (the host checks that they fit:
// decode_fused_fits).
__host__ __device__ inline size_t decode_fused_smem_bytes(int PL) {
    return score_rows_smem_bytes(128, PL, 32, true) + (size_t)SROW_G * 32 * 12 + SROW_G * 8;
}
__host__ __device__ inline bool decode_fused_fits(int W, int R, int d_v) {
    return 2 * ((decode_smem_bytes(W, R, d_v) + 15) & ~(size_t)15) <= 2 * (size_t)SROW_TC_KBUF;
}

SDM_DEV uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Every thread of both CTAs arrives; memory before the barrier (release) is visible to the
// other CTA after it (acquire).
SDM_DEV void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}
// 32-bit word at the same shared-memory offset in CTA `rank` of the cluster
SDM_DEV uint32_t dsmem_ld(const void* local, uint32_t rank) {
    const uint32_t a = ptx::smem_u32(local);
    uint32_t ra, v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(ra) : "memory");
    return v;
}

// QPL = 2 (d_v > 128) keeps twice the rows' columns in registers: two CTAs per SM
template <int PL, typename VT, int QPL>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(SROW_THREADS, QPL == 1 ? 4 : 2)
    decode_fused_kernel(const __grid_constant__ CUtensorMap km0,
                        const __grid_constant__ CUtensorMap km1, ScoreRowsArgs a, DecArgs dk) {
    static_assert(SROW_THREADS == DECODE_THREADS, "the step runs on the scorer's CTA");
    using SM = SrowSmem<PL, 32>;
    extern __shared__ __align__(16) unsigned char srow_smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y, n = a.n, kh = a.k_half, B = a.B, H = a.H, N = dk.N, d_v = dk.d_v;
    const uint32_t rank = cluster_ctarank();  // = the role this CTA scores
    const int role = (int)rank;
    const int b0 = (blockIdx.x >> 1) * 4;
    const int W = a.top[0], R = a.top[1], top = a.top[role];
    unsigned char* base = srow_smem + ((1024 - (ptx::smem_u32(srow_smem) & 1023)) & 1023);
    const SM sm(base + SROW_TC_HEAD);
    int32_t* sel_slot = reinterpret_cast<int32_t*>(sm.ncand + 4);    // [G][32]
    float* sel_w = reinterpret_cast<float*>(sel_slot + SROW_G * 32);  // [G][32]
    float* sel_f = sel_w + SROW_G * 32;                               // [G][32]
    double* lnew = reinterpret_cast<double*>(sel_f + SROW_G * 32);    // [G] Lambda'
    if (tid < SROW_CAND) {
        sm.cand[tid] = a.cand[role][tid];
        if (tid == 0) sm.ncand[0] = a.ncand[role];
    }
    // the decay inputs of the rows this CTA selects (warp g: sequence b0 + g) and of the
    // sequences it steps: loads issued now, used after the scores (nothing waits on them
    // before the sub-key stream is under way)
    const int bg = b0 + warp;
    float ag = 1.f;
    double lam = 0.0;
    if (warp < SROW_G && bg < B) {
        const size_t bh = (size_t)bg * H + h;
        ag = dk.alpha[bh];
        lam = dk.lambda[bh];
    }
    float4 vv[2][QPL];
    float bt[2];
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        const int b = b0 + 2 * role + s;
        const size_t bh = (size_t)(b < B ? b : 0) * H + h;
        bt[s] = b < B ? dk.beta[bh] : 0.f;
#pragma unroll
        for (int c = 0; c < QPL; ++c) {
            const int q = lane + 32 * c;
            vv[s][c] = (b < B && q < d_v / 4)
                           ? load_v4<VT>(static_cast<const VT*>(dk.v) + bh * d_v + 4 * q)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    const __nv_bfloat16* xr[SROW_G];
    int rtab[SROW_G];
#pragma unroll
    for (int g = 0; g < SROW_G; ++g) {
        rtab[g] = 0;
        const int b = b0 + g;
        xr[g] = b < B ? static_cast<const __nv_bfloat16*>(a.x[role]) + ((size_t)b * H + h) * 128
                      : nullptr;
    }
    const bool ok = srow_tc_dots<32 * PL, 1>(base, sm.segs, SM::SEG, role ? &km1 : &km0, nullptr,
                                             xr, rtab, h, n);
    {
        const int g = warp >> 1, hf = warp & 1;
        srow_half_topk<PL, 32>(sm.seg(g, hf), n, kh, sm.tv + (g * 2 + hf) * 32,
                               sm.ti + (g * 2 + hf) * 32, lane);
    }
    __syncthreads();
    if (warp < SROW_G && bg < B) {
        const int g = warp;
        if (!(ag > 0.f) && lane == 0) raise_err(SDM_DEVERR_ALPHA);  // treated as alpha = 1
        const double Lg = lam + (ag > 0.f ? log((double)ag) : 0.0);  // Lambda'
        if (lane == 0) lnew[g] = Lg;
        int2* scr = reinterpret_cast<int2*>(sm.seg(g, 0) + 32 * PL * 4);
        uint32_t slot;
        float wt;
        srow_combine32(sm.tv + (g * 2) * 32, sm.ti + (g * 2) * 32, sm.tv + (g * 2 + 1) * 32,
                       sm.ti + (g * 2 + 1) * 32, sm.cand, sm.ncand[0], n, top, scr, lane, slot,
                       wt);
        const size_t bh = (size_t)bg * H + h;
        int sl = ok ? (int)slot : -1;  // a failed dot-product phase selects nothing
        if (!ok) wt = 0.f;
        float f = 0.f;
        if (lane < top) {
            a.idx[role][bh * top + lane] = sl;
            a.w[role][bh * top + lane] = wt;
            if (slot_ok(sl, N)) {
                f = decode_factor(dk.stamp[bh * (size_t)N + sl], Lg, role == 0, ag, dk.touched);
            } else {
                raise_err(SDM_DEVERR_SLOT_RANGE);
                sl = -1;
            }
        }
        sel_slot[g * 32 + lane] = sl;
        sel_w[g * 32 + lane] = wt;
        sel_f[g * 32 + lane] = f;
    }
    cluster_sync();  // both roles' selections are complete and visible in the cluster
    // the occurrences of the two sequences this CTA steps: writes from rank 0's rows, reads
    // from rank 1's, into the step's arrays (which take the sub-key buffers)
    const DecSmem d0(base, W, R, d_v), d1(base + ((decode_smem_bytes(W, R, d_v) + 15) & ~(size_t)15), W, R,
                                                   d_v);
    for (int e = tid; e < 2 * (W + R); e += SROW_THREADS) {
        const int s = e / (W + R), o = e % (W + R);
        const int g = 2 * role + s;
        const bool rd = o >= W;
        const int i = rd ? o - W : o, src = rd ? 1 : 0;
        const int off = g * 32 + i;
        const DecSmem& dd = s ? d1 : d0;
        dd.slot[o] = (int)dsmem_ld(sel_slot + off, (uint32_t)src);
        dd.w[o] = __uint_as_float(dsmem_ld(sel_w + off, (uint32_t)src));
        dd.f[o] = __uint_as_float(dsmem_ld(sel_f + off, (uint32_t)src));
    }
    cluster_sync();  // neither CTA reads the other's shared memory after this
    for (int s = 0; s < 2; ++s) {
        const int b = b0 + 2 * role + s;
        if (b >= B) break;
        if (s > 0) __syncthreads();  // the first step's partial sums have been read
        decode_apply<VT, 4, QPL>((size_t)b * H + h, vv[s], bt[s], lnew[2 * role + s], s ? d1 : d0,
                                 dk.M, dk.stamp, dk.lambda, dk.M0, dk.out, H, N, d_v, W, R);
    }
}

}  // namespace sdm
