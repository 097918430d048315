// Planning pass of the prefill recurrence (indices, weights and gates only; no rows).
//
// The recurrence (§2 Background "Gated DeltaNet", §3 Method "Sparse memory updates") is run
// chunk by chunk: C tokens gather their rows from the memory as it stood at the chunk start,
// the dependencies between tokens of one chunk that share a slot are resolved on chip, and
// every slot written in the chunk is stored once at the chunk end.  Inside a chunk, with the
// chunk-start rows gathered (decayed to each token: P0, Q0) and d_t = beta_t (v_t - p_t):
//     p_t = P0_t + sum_{tau<t} L[t][tau] d_tau,   L[t][tau] = e^{lam_t - lam_tau} sum_{s in W_t ^ W_tau} w_t,s w_tau,s
//     =>  (I + diag(beta) L) d = beta (v - P0),   d = Minv beta (v - P0)
//     o_t = Q0_t + sum_{tau<=t} G[t][tau] d_tau,  G[t][tau] = e^{lam_t - lam_tau} sum_{s in R_t ^ W_tau} u_t,s w_tau,s
// (the intra-chunk phase of the pages' Appendix A.1; tokens interact only through shared
// slots, Appendix A.2).  Minv and G depend on nothing but indices, weights and gates, so they
// are built here once per (b,h, chunk) and shared by every column block of the row pass.
//
//   plan_local (one CTA per chunk)
//     lam[t]      = sum of log(alpha_u) from the chunk start to t (inclusive), fp32
//     csum[j]     = the same sum over the whole chunk, fp64
//     lk[o]       = for occurrence o (a write or read slot of a token in the chunk):
//                   bits 0..15: 1 + the in-chunk index of the latest earlier write of that slot
//                   (token < t for a write, token <= t for a read), 0 if none;
//                   bit 16: o is the last write of its slot in the chunk (stores it);
//                   bits 18..29: 1 + the index of the previous chunk's write occurrence
//                   that stored o's slot at that chunk's end (0: not written there) — the
//                   row pass gathers a chunk ahead and takes such rows from that store
//     Minv, GM    = Minv and GM = G Minv (fp32 [C][C+4] rows, row t = token, zero beyond the
//                   chunk), into the chunk image: d = Minv beta (v - P0), o = Q0 + GM beta (v - P0)
//     st0[o]      = the state's stamp of o's slot at call entry (NaN: pristine)
//     occw[o]     = o's slot | OCC_OWNER when o stores it
//   plan_prefix (one CTA per (b,h))
//     Lstart[j]   = log-decay prefix at the start of chunk j (Lstart[0] = state Lambda);
//                   the state Lambda becomes Lstart[J]
//   plan_fe (one CTA per chunk)
//     fe[o]       = exp(Lambda_t - stamp of the row o gathers) assuming the slot was not
//                   written earlier in this call; sign bit set when the row is the pristine
//                   M0 row
//   plan_walk (one CTA per (b,h), chunks in order, packed words streamed through a ring)
//     fe[o] is rewritten for slots written by an earlier chunk of this call (the row then
//     carries the stamp of that chunk's end); the state stamps of the slots written in the
//     call are updated.
//   plan_pack (one CTA per chunk)
//     rs and the chunk image: what the row pass reads (see PlanPtrs, RunImg).
//
// In-chunk occurrence order: the nt*W write occurrences (token-major), then the nt*R
// read occurrences.  In the per-(b,h) arrays fe / lk / st0 the T*W write entries come
// first, then the T*R read entries.
#pragma once

#include <math.h>

#include "common.cuh"

namespace sdm {

constexpr int PLAN_MAX_OCC = 2048;  // C*(W+R) never exceeds this
constexpr int PLAN_MAX_C = 32;      // tokens per chunk
constexpr int PLAN_HASH = 2048;     // hash buckets (>= the write occurrences of a chunk)
constexpr int PLAN_THREADS = 256;
constexpr int WALK_THREADS = 512;
constexpr int WALK_MAXO = PLAN_MAX_OCC / WALK_THREADS;
constexpr int WALK_RING = 8;  // chunks of packed occurrence words prefetched by the walk
constexpr uint32_t OCC_OWNER = 0x80000000u;
constexpr uint32_t OCC_SLOT = 0x7fffffffu;  // slot, or OCC_SLOT when out of range

constexpr unsigned LK_OWNER = 1u << 16;
constexpr int LK_PREV_SHIFT = 18;  // bits 18..29: 1 + previous chunk's owner of the slot

SDM_DEV int lk_link(int lk) { return (lk & 0xffff) - 1; }
SDM_DEV int lk_prev(int lk) { return ((lk >> LK_PREV_SHIFT) & 0xfff) - 1; }

SDM_DEV unsigned slot_hash(int s) { return ((unsigned)s * 2654435761u) >> (32 - 11); }
static_assert(PLAN_HASH == 1 << 11, "slot_hash takes the top 11 bits");

// Dynamic shared memory of plan_local (bytes).
__host__ __device__ inline size_t plan_local_smem_bytes() {
    return (size_t)3 * PLAN_MAX_C * PLAN_MAX_C * 4 + (size_t)2 * PLAN_MAX_C * 4 +
           (size_t)PLAN_MAX_OCC * (4 + 4 + 4 + 2 + 2 + 2 + 1) + (size_t)PLAN_HASH * 4 * 2;
}

// Inclusive block-wide prefix sum of doubles held one per thread (blockDim.x <= 1024).
SDM_DEV double block_inclusive_scan(double v, double* warp_tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const double u = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += u;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        const int nwarps = blockDim.x >> 5;
        double t = lane < nwarps ? warp_tot[lane] : 0.0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const double u = __shfl_up_sync(0xffffffffu, t, off);
            if (lane >= off) t += u;
        }
        if (lane < nwarps) warp_tot[lane] = t;
    }
    __syncthreads();
    if (warp > 0) v += warp_tot[warp - 1];
    __syncthreads();
    return v;
}

struct PlanPtrs {
    float* lam;        // [BH][T]
    double* csum;      // [BH][J]
    double* Lstart;    // [BH][J+1]
    double* st0;       // [BH][T*(W+R)]
    float* fe;         // [BH][T*(W+R)]
    int32_t* lk;       // [BH][T*(W+R)]
    uint32_t* occw;    // [BH][T*(W+R)] slot | OCC_OWNER (the walk's input)
    unsigned long long* mask;  // [BH][N][MW] chunks of this call that stored each slot, or null
    short* wtab;               // [BH][N] the walk's last storing chunk of each slot (no masks)
    int MW;                    // 64-bit words per slot in mask
    // the row pass's inputs, packed by plan_pack
    int32_t* rs;          // [BH][T*(W+R)] chunk j at j*C*(W+R), in-chunk occurrence order:
                          // slot | bit 31 when the row gathered is the pristine M0 row
    unsigned char* img;   // [BH][J][img bytes]: per-chunk image (RunImg)
    // touched-slots decay only (null otherwise), per occurrence in the lk order:
    float* vfc;  // product of alpha over the slot's writes in this chunk up to the occurrence's
                 // token (the occurrence itself included when it is a write): the factor
                 // of the gathered row
    float* vsh;  // writes: product of alpha over the slot's later writes in this chunk (the
                 // owner's included): its d's factor in the stored value
};

// Per-chunk image of the row pass's column-independent inputs, written by plan_pack and
// copied as is into the row pass's shared memory (16-byte aligned sections, byte offsets):
//   coef  [C][W+1] then [C][R+1]: w |fe| of token t's i-th write (read) occurrence (the
//         padded rows keep the tokens a warp reads at once in different banks)
//   hz    [C*(W+R)]: o | prev << 16 for the occurrences whose row the previous chunk stores
//         (prev: that chunk's write occurrence), then -1
//   wslot [C*W]: slot of each write occurrence (0x7fffffff when out of range)
//   wlk   [C*W]: its link word (LK_OWNER, in-chunk link)
//   sc    [C*W]: w e^{lam_end - lam_t}: the write's share of its slot's chunk-end value
//   a     [C*W]: |fe| e^{lam_end - lam_t}: the gathered row's share (owners)
//   beta  [C]
//   minv, gm [C][C+4]: Minv and GM = G Minv (rows padded to C+4 floats: 16-byte rows whose
//         starts fall 4 banks apart)
struct RunImg {
    int coef, hz, wslot, wlk, sc, a, beta, minv, gm, bytes;
};
__host__ __device__ inline int up16i(int x) { return (x + 15) & ~15; }
__host__ __device__ inline RunImg run_img(int C, int W, int R) {
    RunImg m;
    int o = 0;
    m.coef = o;  o += up16i(C * (W + R + 2) * 4);
    m.hz = o;    o += up16i(C * (W + R) * 4);
    m.wslot = o; o += up16i(C * W * 4);
    m.wlk = o;   o += up16i(C * W * 4);
    m.sc = o;    o += up16i(C * W * 4);
    m.a = o;     o += up16i(C * W * 4);
    m.beta = o;  o += up16i(C * 4);
    m.minv = o;  o += C * (C + 4) * 4;
    m.gm = o;    o += C * (C + 4) * 4;
    m.bytes = o;
    return m;
}

// TOUCHED: touched-slots decay (PlanPtrs::vfc and vsh are set); the default decays every slot.
template <bool TOUCHED>
__global__ void __launch_bounds__(PLAN_THREADS, 3) plan_local_kernel(
    const float* __restrict__ alpha, const float* __restrict__ beta,
    const int32_t* __restrict__ widx, const float* __restrict__ ww,
    const int32_t* __restrict__ ridx, const float* __restrict__ rw,
    const double* __restrict__ stamp, int T, int N, int W, int R, int C, int J, PlanPtrs P) {
    __shared__ double s_wtot[32];
    __shared__ float s_alf[PLAN_MAX_C];  // alpha_t (touched-slots decay)
    extern __shared__ __align__(16) unsigned char plan_smem[];
    float* s_L = reinterpret_cast<float*>(plan_smem);         // [32][32] L, then Minv
    float* s_G = s_L + PLAN_MAX_C * PLAN_MAX_C;               // [32][32]
    float* s_X = s_G + PLAN_MAX_C * PLAN_MAX_C;               // [32][32] Minv (column solves)
    float* s_lamc = s_X + PLAN_MAX_C * PLAN_MAX_C;            // [32] chunk-relative prefix
    float* s_bet = s_lamc + PLAN_MAX_C;                       // [32]
    int* s_slot = reinterpret_cast<int*>(s_bet + PLAN_MAX_C); // [2048]
    int* s_slot2 = s_slot + PLAN_MAX_OCC;                     // previous chunk's write slots
    float* s_wt = reinterpret_cast<float*>(s_slot2 + PLAN_MAX_OCC);  // [2048] weights
    int* s_head = reinterpret_cast<int*>(s_wt + PLAN_MAX_OCC);       // [PLAN_HASH] (32-bit atomics)
    int* s_head2 = s_head + PLAN_HASH;                               // [PLAN_HASH]
    short* s_link = reinterpret_cast<short*>(s_head2 + PLAN_HASH);
    short* s_next = s_link + PLAN_MAX_OCC;
    short* s_next2 = s_next + PLAN_MAX_OCC;
    unsigned char* s_owner = reinterpret_cast<unsigned char*>(s_next2 + PLAN_MAX_OCC);

    const int j = blockIdx.x;
    const size_t bh = blockIdx.y;
    const int tid = threadIdx.x;
    const int t0 = j * C;
    const int nt = min(C, T - t0);
    const int nw = nt * W, no = nt * (W + R);
    const size_t occ_base = bh * (size_t)T * (W + R);
    constexpr bool touched = TOUCHED;  // alpha scales only the write slots

    // 1. chunk-relative log-decay prefix (C <= PLAN_THREADS tokens per chunk)
    double la = 0.0;
    if (tid < nt) {
        const float a = alpha[bh * T + t0 + tid];
        if (TOUCHED) s_alf[tid] = a;
        if (a > 0.f) {
            la = log((double)a);
        } else {
            raise_err(SDM_DEVERR_ALPHA);  // treated as alpha = 1
        }
        s_bet[tid] = beta[bh * T + t0 + tid];
    }
    const double pre = block_inclusive_scan(la, s_wtot);
    if (tid < nt) {
        P.lam[bh * T + t0 + tid] = (float)pre;
        s_lamc[tid] = (float)pre;
    }
    if (tid == nt - 1) P.csum[bh * J + j] = pre;

    // 2. slots and weights of the chunk (and the previous chunk's write slots), hash heads;
    //    the slots' entry stamps are fetched now (registers) and written in step 7
    constexpr int PO = PLAN_MAX_OCC / PLAN_THREADS;
    double est[PO];
#pragma unroll
    for (int k = 0; k < PO; ++k) {
        const int o = tid + k * PLAN_THREADS;
        est[k] = 0.0;
        if (o >= no) continue;
        int s;
        float w;
        if (o < nw) {
            s = widx[(bh * T + t0) * W + o];
            w = ww[(bh * T + t0) * W + o];
        } else {
            s = ridx[(bh * T + t0) * R + (o - nw)];
            w = rw[(bh * T + t0) * R + (o - nw)];
        }
        if (!slot_ok(s, N)) {
            raise_err(SDM_DEVERR_SLOT_RANGE);
            s = -1;
        } else {
            est[k] = stamp[bh * (size_t)N + s];
        }
        s_slot[o] = s;
        s_wt[o] = w;
        s_owner[o] = 0;
    }
    for (int i = tid; i < PLAN_HASH; i += PLAN_THREADS) {
        s_head[i] = -1;
        s_head2[i] = -1;
    }
    for (int i = tid; i < PLAN_MAX_C * PLAN_MAX_C; i += PLAN_THREADS) {
        s_L[i] = 0.f;
        s_G[i] = 0.f;
    }
    const int nwp = j > 0 ? C * W : 0;  // the previous chunk is always full
    for (int o = tid; o < nwp; o += PLAN_THREADS) {
        const int sp = widx[(bh * T + (size_t)(j - 1) * C) * W + o];
        s_slot2[o] = slot_ok(sp, N) ? sp : -1;
    }
    __syncthreads();

    // 3. insert the write occurrences of this and of the previous chunk into bucket lists
    for (int o = tid; o < nw; o += PLAN_THREADS) {
        const int s = s_slot[o];
        if (s >= 0) s_next[o] = (short)atomicExch(&s_head[slot_hash(s)], o);
    }
    for (int o = tid; o < nwp; o += PLAN_THREADS) {
        const int s = s_slot2[o];
        if (s >= 0) s_next2[o] = (short)atomicExch(&s_head2[slot_hash(s)], o);
    }
    __syncthreads();

    // 4. links: latest earlier write of the same slot; owner = no later write in chunk
    const FastDiv fW((unsigned)W), fR((unsigned)R);
    for (int o = tid; o < no; o += PLAN_THREADS) {
        const int s = s_slot[o];
        int link = -1;
        if (s >= 0) {
            const bool is_w = o < nw;
            const int tl = is_w ? fW.div(o) : fR.div(o - nw);
            int best_t = -1;
            bool later = false;
            for (int p = s_head[slot_hash(s)]; p >= 0; p = s_next[p]) {
                if (s_slot[p] != s) continue;
                const int tp = fW.div(p);
                if (is_w) {
                    if (tp == tl && p != o) raise_err(SDM_DEVERR_DUP_WRITE);
                    if (tp > tl) later = true;
                    if (tp < tl && tp > best_t) {
                        best_t = tp;
                        link = p;
                    }
                } else if (tp <= tl && tp > best_t) {
                    best_t = tp;
                    link = p;
                }
            }
            if (is_w && !later) s_owner[o] = 1;
        }
        s_link[o] = (short)link;
    }
    __syncthreads();

    // 5. L and G rows: one warp per (role, token) t; its lanes walk the link chains of t's
    //    occurrences (every earlier write of the slot in the chunk) in step, and the terms of
    //    one step are added to row t in lane order (deterministic sums).  A term's decay from
    //    the earlier write at tp to t is e^{lam_t - lam_tp}; with touched-slots decay it is the
    //    product of alpha over the slot's writes after tp up to t (t's own write included)
    {
        const int warp = tid >> 5, lane = tid & 31;
        for (int task = warp; task < 2 * nt; task += PLAN_THREADS / 32) {
            const bool rd = task >= nt;
            const int t = rd ? task - nt : task;
            const int n_i = rd ? R : W;
            const int o0 = rd ? nw + t * R : t * W;
            float* row = (rd ? s_G : s_L) + t * PLAN_MAX_C;
            const float lt = s_lamc[t];
            for (int base = 0; base < n_i; base += 32) {
                const int o = o0 + base + lane;
                const bool in = base + lane < n_i;
                const float wo = in ? s_wt[o] : 0.f;
                int L = in ? s_link[o] : -1;
                float chain = TOUCHED ? (rd ? 1.f : s_alf[t]) : 0.f;  // decay of the next term
                while (__any_sync(0xffffffffu, L >= 0)) {
                    int tp = 0;
                    float val = 0.f;
                    if (L >= 0) {
                        tp = fW.div(L);
                        if (touched) {
                            val = wo * s_wt[L] * chain;
                            chain *= s_alf[tp];
                        } else {
                            val = wo * s_wt[L] * expf(lt - s_lamc[tp]);
                        }
                    }
                    for (unsigned m = __ballot_sync(0xffffffffu, L >= 0); m; m &= m - 1) {
                        const int src = __ffs(m) - 1;
                        const int tps = __shfl_sync(0xffffffffu, tp, src);
                        const float vs = __shfl_sync(0xffffffffu, val, src);
                        if (lane == 0) row[tps] += vs;
                    }
                    L = L >= 0 ? s_link[L] : -1;
                }
            }
        }
    }
    __syncthreads();
    // 6. Minv = (I + diag(beta) L)^-1, one column per thread by forward substitution with the
    //    column in registers (L is zero outside the chunk, so the full 32 x 32 form is exact)
    if (tid < PLAN_MAX_C) {
        const int k = tid;
        float x[PLAN_MAX_C];
#pragma unroll
        for (int t = 0; t < PLAN_MAX_C; ++t) {
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
            for (int tau = 0; tau < t; ++tau) {
                const float l = s_L[t * PLAN_MAX_C + tau];
                if ((tau & 3) == 0) a0 = fmaf(l, x[tau], a0);
                else if ((tau & 3) == 1) a1 = fmaf(l, x[tau], a1);
                else if ((tau & 3) == 2) a2 = fmaf(l, x[tau], a2);
                else a3 = fmaf(l, x[tau], a3);
            }
            const float bt = t < nt ? s_bet[t] : 0.f;
            x[t] = (t == k) ? 1.f : (t < k ? 0.f : -bt * ((a0 + a1) + (a2 + a3)));
        }
#pragma unroll
        for (int t = 0; t < PLAN_MAX_C; ++t) s_X[t * PLAN_MAX_C + k] = x[t];
    }
    __syncthreads();
    // GM = G Minv (lower triangular), so that o = Q0 + GM beta (v - P0) needs no d; into s_L
    for (int e = tid; e < PLAN_MAX_C * PLAN_MAX_C; e += PLAN_THREADS) {
        const int t = e / PLAN_MAX_C, tau = e % PLAN_MAX_C;
        float acc = 0.f;
        for (int k = tau; k <= t; ++k) acc = fmaf(s_G[t * PLAN_MAX_C + k], s_X[k * PLAN_MAX_C + tau], acc);
        s_L[e] = acc;
    }
    __syncthreads();
    {
        const RunImg m = run_img(C, W, R);
        unsigned char* img = P.img + (bh * J + j) * (size_t)m.bytes;
        float* minv = reinterpret_cast<float*>(img + m.minv);
        float* gm = reinterpret_cast<float*>(img + m.gm);
        const int MS = C + 4;
        for (int e = tid; e < C * MS; e += PLAN_THREADS) {
            const int t = e / MS, tau = e % MS;
            const bool in = t < nt && tau < nt;
            minv[e] = in ? s_X[t * PLAN_MAX_C + tau] : 0.f;
            gm[e] = in ? s_L[t * PLAN_MAX_C + tau] : 0.f;
        }
    }

    // 7. link words and entry stamps
#pragma unroll
    for (int k = 0; k < PO; ++k) {
        const int o = tid + k * PLAN_THREADS;
        if (o >= no) continue;
        const int link = s_link[o];
        unsigned v = (unsigned)(link + 1);
        size_t g;
        if (o < nw) {
            if (s_owner[o]) v |= LK_OWNER;
            g = occ_base + (size_t)t0 * W + o;
        } else {
            g = occ_base + (size_t)T * W + (size_t)t0 * R + (o - nw);
        }
        // the previous chunk's last write of this slot (its store at that chunk's end)
        const int sl = s_slot[o];
        if (sl >= 0 && nwp > 0) {
            int best = -1;
            for (int p = s_head2[slot_hash(sl)]; p >= 0; p = s_next2[p])
                if (s_slot2[p] == sl && p > best) best = p;  // larger index = later token
            v |= (unsigned)(best + 1) << LK_PREV_SHIFT;
        }
        P.lk[g] = (int32_t)v;
        P.st0[g] = est[k];
        if (touched) {
            // the gathered row's factor: alpha of every write of the slot in this chunk up to
            // this occurrence (its own write included)
            const bool is_w = o < nw;
            float fc = is_w ? s_alf[fW.div(o)] : 1.f;
            for (int L = link; L >= 0; L = s_link[L]) fc *= s_alf[fW.div(L)];
            P.vfc[g] = fc;
            if (is_w && sl < 0) P.vsh[g] = 0.f;
            if (is_w && s_owner[o]) {
                // down the slot's chain from its last write: each write's d reaches the stored
                // value through the alpha of the slot's later writes
                float sh = 1.f;
                for (int L = o; L >= 0; L = s_link[L]) {
                    P.vsh[occ_base + (size_t)t0 * W + L] = sh;
                    sh *= s_alf[fW.div(L)];
                }
            }
        }
        if (!P.mask)  // the walk's input
            P.occw[g] = (sl >= 0 ? (uint32_t)sl : OCC_SLOT) | (o < nw && s_owner[o] ? OCC_OWNER : 0u);
        if (P.mask && o < nw && s_owner[o] && sl >= 0)  // this chunk stores the slot
            atomicOr(P.mask + (bh * (size_t)N + sl) * P.MW + (j >> 6), 1ull << (j & 63));
    }
}

// Chunk-start log-decay prefixes of one (b,h): Lstart[0] = Lambda, Lstart[j+1] = Lstart[j] +
// csum[j]; the state Lambda advances to Lstart[J].
__global__ void __launch_bounds__(1024) plan_prefix_kernel(double* __restrict__ lambda, int J,
                                                           PlanPtrs P) {
    __shared__ double s_wtot[32];
    const size_t bh = blockIdx.x;
    const int tid = threadIdx.x;
    double* Lg = P.Lstart + bh * (size_t)(J + 1);
    const double L0 = lambda[bh];
    const int per = (J + 1023) / 1024;
    const int a = tid * per, b = min(J, a + per);
    double part = 0.0;
    for (int i = a; i < b; ++i) part += P.csum[bh * J + i];
    const double incl = block_inclusive_scan(part, s_wtot);
    double run = L0 + (incl - part);
    if (tid == 0) Lg[0] = L0;
    for (int i = a; i < b; ++i) {
        run += P.csum[bh * J + i];
        Lg[i + 1] = run;
    }
    __syncthreads();
    if (tid == 0) lambda[bh] = Lg[J];
}

// Decay factor of one occurrence (slot s < N, owner bit, token prefix lam_t, entry stamp st)
// in chunk j.  With the masks it is final (and the slot's last storing chunk writes the new
// stamp); without, it is as if the slot had not been written earlier in this call.
SDM_DEV float occ_factor(double* __restrict__ stamp, const PlanPtrs& P, size_t bh, int N, int J,
                         int j, int s, bool owner, float lam_t, double st) {
    const double* Lb = P.Lstart + bh * (size_t)(J + 1);
    const double Lj = Lb[j];
    int jw = -1;
    if (P.mask) {
        const unsigned long long* m = P.mask + (bh * (size_t)N + s) * P.MW;
        for (int wi = j >> 6; wi >= 0 && jw < 0; --wi) {
            unsigned long long bits = m[wi];
            if (wi == (j >> 6)) bits &= (j & 63) ? ((1ull << (j & 63)) - 1) : 0ull;
            if (bits) jw = wi * 64 + 63 - __clzll((long long)bits);
        }
        if (owner) {  // the slot's last storing chunk sets its stamp
            int jl = -1;
            for (int wi = P.MW - 1; wi >= 0 && jl < 0; --wi) {
                const unsigned long long bits = m[wi];
                if (bits) jl = wi * 64 + 63 - __clzll((long long)bits);
            }
            if (jl == j) stamp[bh * (size_t)N + s] = Lb[j + 1];
        }
    }
    if (jw >= 0) return expf((float)(Lj - Lb[jw + 1]) + lam_t);
    const double Lt = Lj + (double)lam_t;
    return isnan(st) ? -(float)exp(Lt) : (float)exp(Lt - st);
}

// Decay factors of every occurrence.  Without a mask: as if its slot had not been written
// earlier in this call (the walk corrects the others).  With the per-slot chunk masks: the
// last earlier chunk that stored the slot is the highest set bit below this chunk, so every
// factor is final here, and the owner in the slot's last chunk writes the slot's new stamp.
__global__ void __launch_bounds__(PLAN_THREADS) plan_fe_kernel(double* __restrict__ stamp, int T,
                                                               int N, int W, int R, int C, int J,
                                                               PlanPtrs P) {
    const int j = blockIdx.x;
    const size_t bh = blockIdx.y;
    const int t0 = j * C, nt = min(C, T - t0), nw = nt * W, no = nt * (W + R);
    const size_t occ_base = bh * (size_t)T * (W + R);
    for (int o = threadIdx.x; o < no; o += PLAN_THREADS) {
        size_t g;
        int t;
        if (o < nw) {
            g = occ_base + (size_t)t0 * W + o;
            t = o / W;
        } else {
            g = occ_base + (size_t)T * W + (size_t)t0 * R + (o - nw);
            t = (o - nw) / R;
        }
        const uint32_t w = P.occw[g];
        const int s = (int)(w & OCC_SLOT);
        if (s >= N) {
            P.fe[g] = 0.f;
            continue;
        }
        P.fe[g] = occ_factor(stamp, P, bh, N, J, j, s, (w & OCC_OWNER) != 0,
                             P.lam[bh * T + t0 + t], P.st0[g]);
    }
}

// Sequential walk over the chunks of one (b,h), split over `parts` CTAs by slot (slot % parts):
// the last chunk of this call that stored each slot (-1: none) is kept in P.wtab (int16 per
// slot in global memory, 2 bytes a slot: it stays in L2), so the CTAs need only the ring that
// streams the chunks' packed occurrence words and token prefixes, filled WALK_RING chunks
// ahead by cp.async, and every walk of the call runs at once.  Two barriers per chunk: after
// the chunk's words land (the previous chunk's table writes are then visible, and the ring
// stage it used may be refilled) and between the chunk's lookups and its own writes.
__global__ void __launch_bounds__(WALK_THREADS) plan_walk_kernel(
    double* __restrict__ stamp, int T, int N, int W, int R, int C, int J, int parts,
    int lstart_smem, PlanPtrs P) {
    extern __shared__ __align__(16) unsigned char walk_smem[];
    const int part = blockIdx.x;
    const size_t bh = blockIdx.y;
    const int tid = threadIdx.x;
    const int stage = PLAN_MAX_OCC + PLAN_MAX_C;  // words per ring stage
    uint32_t* s_ring = reinterpret_cast<uint32_t*>(walk_smem);  // [WALK_RING][stage]
    double* s_L = reinterpret_cast<double*>(s_ring + WALK_RING * stage);  // [J+1] if lstart_smem
    short* tab = P.wtab + bh * (size_t)N;
    const double* Lg = P.Lstart + bh * (size_t)(J + 1);
    if (lstart_smem)
        for (int i = tid; i <= J; i += WALK_THREADS) s_L[i] = Lg[i];
    const double* Lr = lstart_smem ? s_L : Lg;
    const size_t occ_base = bh * (size_t)T * (W + R);

    // a chunk's write words and read words are two contiguous runs: with W and R multiples of
    // 4 both start on 16-byte boundaries (here and in the ring) and move in 16-byte pieces
    const bool vec = (W & 3) == 0 && (R & 3) == 0;
    auto load_stage = [&](int jn) {
        if (jn < J && vec) {
            uint32_t* dst = s_ring + (jn % WALK_RING) * stage;
            const int t0 = jn * C, nt = min(C, T - t0), nw = nt * W, nr = nt * R;
            const uint32_t* wsrc = P.occw + occ_base + (size_t)t0 * W;
            const uint32_t* rsrc = P.occw + occ_base + (size_t)T * W + (size_t)t0 * R;
            for (int p = tid; p < (nw + nr) / 4; p += WALK_THREADS) {
                const int o = 4 * p;  // nw is a multiple of 4: a piece is all writes or all reads
                cp_async16(dst + o, o < nw ? wsrc + o : rsrc + (o - nw), true);
            }
            for (int t = tid; t < nt; t += WALK_THREADS) {
                const unsigned d = (unsigned)__cvta_generic_to_shared(dst + PLAN_MAX_OCC + t);
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(d),
                             "l"(P.lam + bh * T + t0 + t)
                             : "memory");
            }
        } else if (jn < J) {
            uint32_t* dst = s_ring + (jn % WALK_RING) * stage;
            const int t0 = jn * C, nt = min(C, T - t0), nw = nt * W, no = nt * (W + R);
            for (int o = tid; o < no; o += WALK_THREADS) {
                const size_t g = o < nw ? occ_base + (size_t)t0 * W + o
                                        : occ_base + (size_t)T * W + (size_t)t0 * R + (o - nw);
                const unsigned d = (unsigned)__cvta_generic_to_shared(dst + o);
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(d), "l"(P.occw + g)
                             : "memory");
            }
            for (int t = tid; t < nt; t += WALK_THREADS) {
                const unsigned d = (unsigned)__cvta_generic_to_shared(dst + PLAN_MAX_OCC + t);
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(d),
                             "l"(P.lam + bh * T + t0 + t)
                             : "memory");
            }
        }
        cp_async_commit();  // one group per stage, empty past the end
    };

    for (int s = 0; s < WALK_RING - 1; ++s) load_stage(s);
    for (int j = 0; j < J; ++j) {
        asm volatile("cp.async.wait_group %0;\n" ::"n"(WALK_RING - 2) : "memory");
        __syncthreads();
        load_stage(j + WALK_RING - 1);  // into the stage chunk j - 1 used (finished by now)
        const uint32_t* ow = s_ring + (j % WALK_RING) * stage;
        const float* lamc = reinterpret_cast<const float*>(ow + PLAN_MAX_OCC);
        const int t0 = j * C, nt = min(C, T - t0), nw = nt * W, no = nt * (W + R);
        const double Lj = Lr[j];
        // rows of slots written by an earlier chunk carry that chunk's end stamp: the table
        // entries of this thread's occurrences are all requested before any is used
        constexpr int PO = PLAN_MAX_OCC / WALK_THREADS;
        int jw[PO];
#pragma unroll
        for (int k = 0; k < PO; ++k) {
            const int o = tid + k * WALK_THREADS;
            const int s = o < no ? (int)(ow[o] & OCC_SLOT) : N;
            jw[k] = (s < N && s % parts == part) ? (int)tab[s] : -1;
        }
#pragma unroll
        for (int k = 0; k < PO; ++k) {
            const int o = tid + k * WALK_THREADS;
            if (jw[k] < 0) continue;
            int t;
            size_t g;
            if (o < nw) {
                t = o / W;
                g = occ_base + (size_t)t0 * W + o;
            } else {
                t = (o - nw) / R;
                g = occ_base + (size_t)T * W + (size_t)t0 * R + (o - nw);
            }
            P.fe[g] = expf((float)(Lj - Lr[jw[k] + 1]) + lamc[t]);
        }
        __syncthreads();
        for (int o = tid; o < nw; o += WALK_THREADS) {
            const uint32_t w = ow[o];
            const int s = (int)(w & OCC_SLOT);
            if (!(w & OCC_OWNER) || s >= N || s % parts != part) continue;
            tab[s] = (short)j;
        }
    }
    asm volatile("cp.async.wait_all;\n" ::: "memory");

    __syncthreads();
    // final stamps of this partition's slots written in this call
    for (size_t o = tid; o < (size_t)T * W; o += WALK_THREADS) {
        const uint32_t w = P.occw[occ_base + o];
        const int s = (int)(w & OCC_SLOT);
        if (!(w & OCC_OWNER) || s >= N || s % parts != part) continue;
        const int j = (int)(o / W) / C;
        if (tab[s] == j) stamp[bh * (size_t)N + s] = Lr[j + 1];
    }
}

// The row pass's inputs from the final decay factors: the gather words (slot, pristine flag)
// and the chunk image (coefficients, store factors, links, the list of occurrences whose row
// the previous chunk stores — in any order — and beta).
template <bool TOUCHED>
__global__ void __launch_bounds__(PLAN_THREADS) plan_pack_kernel(
    double* __restrict__ stamp, const float* __restrict__ beta, const int32_t* __restrict__ widx,
    const float* __restrict__ ww, const int32_t* __restrict__ ridx,
    const float* __restrict__ rw, int T, int N, int W, int R, int C, int J, PlanPtrs P) {
    __shared__ float s_lam[PLAN_MAX_C];
    __shared__ int s_cnt;
    const int j = blockIdx.x;
    const size_t bh = blockIdx.y;
    const int tid = threadIdx.x;
    const int t0 = j * C, nt = min(C, T - t0), nw = nt * W, no = nt * (W + R);
    const size_t occ_base = bh * (size_t)T * (W + R);
    const RunImg m = run_img(C, W, R);
    unsigned char* img = P.img + (bh * J + j) * (size_t)m.bytes;
    float* coef = reinterpret_cast<float*>(img + m.coef);
    int32_t* hz = reinterpret_cast<int32_t*>(img + m.hz);
    int32_t* wslot = reinterpret_cast<int32_t*>(img + m.wslot);
    int32_t* wlk = reinterpret_cast<int32_t*>(img + m.wlk);
    float* sc = reinterpret_cast<float*>(img + m.sc);
    float* sa = reinterpret_cast<float*>(img + m.a);
    float* bt = reinterpret_cast<float*>(img + m.beta);
    int32_t* rs = P.rs + occ_base + (size_t)t0 * (W + R);
    if (tid == 0) s_cnt = 0;
    if (tid < nt) {
        s_lam[tid] = P.lam[bh * T + t0 + tid];
        bt[tid] = beta[bh * T + t0 + tid];
    }
    __syncthreads();
    const float lam_end = s_lam[nt - 1];
    for (int o = tid; o < no; o += PLAN_THREADS) {
        size_t g;
        int s, ci;
        float w;
        if (o < nw) {
            const int t = o / W;
            g = occ_base + (size_t)t0 * W + o;
            s = widx[(bh * T + t0) * W + o];
            w = ww[(bh * T + t0) * W + o];
            ci = t * (W + 1) + (o - t * W);
        } else {
            const int r = o - nw, t = r / R;
            g = occ_base + (size_t)T * W + (size_t)t0 * R + r;
            s = ridx[(bh * T + t0) * R + r];
            w = rw[(bh * T + t0) * R + r];
            ci = C * (W + 1) + t * (R + 1) + (r - t * R);
        }
        const int lk = P.lk[g];
        const bool ok = slot_ok(s, N);
        // with the masks the factors are computed here (plan_fe is not run); after the walk
        // they are read back
        float f = !ok ? 0.f
                  : P.mask ? occ_factor(stamp, P, bh, N, J, j, s, (o < nw) && (lk & LK_OWNER),
                                        s_lam[o < nw ? o / W : (o - nw) / R], P.st0[g])
                           : P.fe[g];
        // touched-slots decay: the same pristine sign, the in-chunk product as the magnitude
        if (TOUCHED && ok) f = copysignf(P.vfc[g], f);
        rs[o] = ok ? (int32_t)((uint32_t)s | (signbit(f) ? 0x80000000u : 0u)) : 0x7fffffff;
        coef[ci] = ok ? w * fabsf(f) : 0.f;
        if (o < nw) {
            // shares of the stored (chunk-end) value: the d of this write, the gathered row
            const float e = TOUCHED ? 1.f : expf(lam_end - s_lam[o / W]);
            wslot[o] = ok ? s : 0x7fffffff;
            wlk[o] = lk;
            sc[o] = w * (TOUCHED ? P.vsh[g] : e);
            sa[o] = fabsf(f) * e;
        }
        const int pv = lk_prev(lk);
        if (pv >= 0) hz[atomicAdd(&s_cnt, 1)] = o | (pv << 16);
    }
    __syncthreads();
    for (int i = s_cnt + tid; i < C * (W + R); i += PLAN_THREADS) hz[i] = -1;
}

}  // namespace sdm
