// Product-key scoring on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), bf16 inputs,
// n <= 256 sub-keys per half (§2 Background "Product Key Memory", §3 Method "Sparse
// addressing", §4 "SDM Configuration").
//
// One CTA scores a tile of 128 rows (tokens of one head and role) and holds the whole SM
// (512 TMEM columns).  TMA brings the x tile (both halves) and the role's two sub-key tables;
// one thread issues 8 tcgen05.mma (M = 128, N = n, K = 64 per half) so that TMEM holds
// D[row][j] = <x_half[row], C_half[j]> for half 0 in columns [0, n) and half 1 in [256, 256+n).
// Warps 0-3 then select half 0 and warps 4-7 half 1, one thread per (row, half):
//   1. Threshold.  The row's mean and spread over its n scores give tau = mean + z*sd, z
//      chosen on the host so that about K + margin scores reach it (the sub-key tables make
//      each row's half-scores close to Gaussian, but nothing relies on it: a row whose count
//      falls outside [K, CAP] is filtered again with z moved, by bisection).
//   2. Filter.  The scores >= tau go, with their sub-indices, to the thread's list in shared
//      memory (CAP entries).
//   3. Order.  Keys are the differences score - tau with their list position written into the
//      low mantissa bits: distinct, and ordered like the scores except among scores whose keys
//      agree above those bits.  Blocks of KP keys are sorted by min/max networks and merged
//      keeping the best KP; the largest key dropped on the way is kept.  If it agrees with the
//      K-th kept key above the position bits, the selection is ambiguous and the list is
//      ranked again exactly (value, then sub-index); otherwise the K kept entries are the exact
//      top K, and a pass of exact compare-exchanges puts equal-key neighbours in order.
//   4. Combine (warps 0-3).  The k x k pairs that can reach the top `top` are those with
//      (a+1)(b+1) <= top (any other pair is beaten by at least `top` pairs with no smaller sum
//      and no larger slot).  The rows a = 0, 1 and columns b = 0, 1 of that staircase are
//      sorted runs; they are merged with the same keyed networks (key = max sum - sum with a
//      code of the pair), the remaining pairs are kept only if they beat the current top-th,
//      and the same ambiguity test decides whether the selection is exact or is ranked again
//      exactly over the whole staircase.  Slots s = i*n + j, equal sums to the lower slot;
//      weights = softmax of the selected sums.
// A row that the threshold search cannot settle is scored again by one warp on CUDA cores
// (exact fp32 FMA scores and selection) at the end of the tile.
#pragma once

#include <math.h>

#include "common.cuh"
#include "score_simt.cuh"
#include "tc_ptx.cuh"

namespace sdm {

constexpr int PK_THREADS = 256;
constexpr int PK_NMAX = 256;     // sub-keys per half this kernel takes (one TMEM round)
constexpr int PK_ITERS = 8;      // threshold attempts before a row goes to the exact re-scoring

// Shared-memory map (bytes from a 1024-aligned base).
constexpr uint32_t PK_OFF_X = 0;        // x tile: half 0 [0,16K), half 1 [16K,32K)
constexpr uint32_t PK_OFF_SK = 32768;   // sub-key tile of half h at + h*32K; later the sorted
                                        // half lists (values [KP][128] f32, ids [KP][128] u16)
constexpr uint32_t PK_OFF_L = 98304;    // candidate lists, then the combine's and the re-scoring's

template <int KP>
struct PkCfg {
    static constexpr int CAP = KP == 16 ? 48 : 64;  // list entries per (row, half)
    static constexpr int PB = 6;                    // key bits that hold a list position
    static constexpr int CB = KP == 16 ? 7 : 8;     // key bits that hold a combine pair code
    static constexpr int LOG_KP = KP == 16 ? 4 : 5;
    static constexpr int REST = KP;                 // remaining staircase pairs (a, b >= 2): <= KP
    static constexpr uint32_t LIST_BYTES = (uint32_t)CAP * 128 * 6;
    static constexpr uint32_t OFF_CTRL = PK_OFF_L + 2 * LIST_BYTES;
    static constexpr uint32_t SMEM = OFF_CTRL + 1024 + 1024;  // + alignment slack
    static_assert(KP * 128 * 6 <= 32768, "sorted half list fits a sub-key tile");
    static_assert(CAP <= (1 << PB), "positions fit the key bits");
    static_assert(4 * KP + 2 * REST <= (1 << CB) - 1, "pair codes fit the key bits");
    static_assert((uint32_t)REST * 128 * 6 <= LIST_BYTES, "rest list fits a list area");
};

struct PkArgs {
    int B, H, T, n, k_half, d_k;
    int top[2];
    int bt, bb, n_tt;  // a tile holds bt tokens of bb sequences; t-tiles per sequence block
    float z0;          // threshold position (-inf: take every score)
    const __nv_bfloat16* x[2];
    const __nv_bfloat16* sk[2];
    int32_t* idx[2];
    float* w[2];
};

// ---- keys ------------------------------------------------------------------------------
// f with its low B bits replaced by code (f >= 0 or any sign: truncation keeps the order).
template <int B>
SDM_DEV float pk_pack(float f, int code) {
    return __int_as_float((__float_as_int(f) & ~((1 << B) - 1)) | code);
}
template <int B>
SDM_DEV int pk_code(float k) { return __float_as_int(k) & ((1 << B) - 1); }
template <int B>
SDM_DEV int pk_hi(float k) { return __float_as_int(k) & ~((1 << B) - 1); }

// Element i of a register array at a run-time index, by a chain of selects.
template <int N>
SDM_DEV float pk_pick(const float (&r)[N], int i) {
    float x = r[0];
#pragma unroll
    for (int e = 1; e < N; ++e) x = e == i ? r[e] : x;
    return x;
}

// Descending bitonic sort of distinct keys (min/max only).
template <int N>
SDM_DEV void pk_ksort(float (&k)[N]) {
#pragma unroll
    for (int s = 2; s <= N; s <<= 1) {
#pragma unroll
        for (int j = s >> 1; j > 0; j >>= 1) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const float a = k[i], b = k[l];
                    const bool desc = (i & s) == 0;
                    k[i] = desc ? fmaxf(a, b) : fminf(a, b);
                    k[l] = desc ? fminf(a, b) : fmaxf(a, b);
                }
            }
        }
    }
}

// r <- the best N of r and s (both sorted descending), sorted; returns the largest key dropped.
template <int N>
SDM_DEV float pk_kmerge(float (&r)[N], const float (&s)[N]) {
    float dropped = -INFINITY;
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const float a = r[i], b = s[N - 1 - i];
        r[i] = fmaxf(a, b);
        dropped = fmaxf(dropped, fminf(a, b));
    }
#pragma unroll
    for (int j = N >> 1; j > 0; j >>= 1) {
#pragma unroll
        for (int i = 0; i < N; ++i) {
            const int l = i ^ j;
            if (l > i) {
                const float a = r[i], b = r[l];
                r[i] = fmaxf(a, b);
                r[l] = fminf(a, b);
            }
        }
    }
    return dropped;
}

// ---- exact (value, id) networks for the rare ambiguous rows --------------------------------
template <int N>
SDM_DEV void pk_xsort(float (&v)[N], int (&ix)[N]) {
#pragma unroll
    for (int s = 2; s <= N; s <<= 1) {
#pragma unroll
        for (int j = s >> 1; j > 0; j >>= 1) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const bool desc = (i & s) == 0;
                    const bool sw = desc ? better(v[l], ix[l], v[i], ix[i])
                                         : better(v[i], ix[i], v[l], ix[l]);
                    const float tv = sw ? v[l] : v[i];
                    const int ti = sw ? ix[l] : ix[i];
                    v[l] = sw ? v[i] : v[l];
                    ix[l] = sw ? ix[i] : ix[l];
                    v[i] = tv;
                    ix[i] = ti;
                }
            }
        }
    }
}

template <int N>
SDM_DEV void pk_xmerge(float (&r)[N], int (&ri)[N], const float (&a)[N], const int (&ai)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const bool take = better(a[N - 1 - i], ai[N - 1 - i], r[i], ri[i]);
        r[i] = take ? a[N - 1 - i] : r[i];
        ri[i] = take ? ai[N - 1 - i] : ri[i];
    }
#pragma unroll
    for (int j = N >> 1; j > 0; j >>= 1) {
#pragma unroll
        for (int i = 0; i < N; ++i) {
            const int l = i ^ j;
            if (l > i) {
                const bool sw = better(r[l], ri[l], r[i], ri[i]);
                const float tv = sw ? r[l] : r[i];
                const int ti = sw ? ri[l] : ri[i];
                r[l] = sw ? r[i] : r[l];
                ri[l] = sw ? ri[i] : ri[l];
                r[i] = tv;
                ri[i] = ti;
            }
        }
    }
}

// Adjacent exact compare-exchanges over the shared-memory list v/ix[0..m) (stride 128) until
// it is sorted (value desc, id asc), on the lanes with `act`.  Used after a keyed selection,
// where only neighbours whose keys agree above the code bits can be out of order.  Rolled
// loops; called by whole warps with a warp-uniform m.
template <typename IT>
SDM_DEV void pk_fixup_smem(float* v, IT* ix, int m, bool act) {
    constexpr int S = 128;
    for (int pass = 0; pass < 2 * m + 2; ++pass) {
        bool sw_any = false;
        for (int i = pass & 1; i + 1 < m; i += 2) {
            const float a = v[i * S], b = v[(i + 1) * S];
            const int ia = (int)ix[i * S], ib = (int)ix[(i + 1) * S];
            const bool sw = act && better(b, ib, a, ia);
            if (sw) {
                v[i * S] = b;
                v[(i + 1) * S] = a;
                ix[i * S] = (IT)ib;
                ix[(i + 1) * S] = (IT)ia;
            }
            sw_any = sw_any || sw;
        }
        if (pass > 0 && !__any_sync(0xffffffffu, sw_any)) break;
    }
}

// Predicated shared-memory stores of one list entry (value and 16-bit id).
SDM_DEV void pk_store_if(bool p, uint32_t vaddr, float v, uint32_t iaddr, int id) {
    asm volatile(
        "{\n .reg .pred q;\n setp.ne.b32 q, %0, 0;\n @q st.shared.f32 [%1], %2;\n"
        " @q st.shared.u16 [%3], %4;\n}\n" ::"r"((int)p),
        "r"(vaddr), "f"(v), "r"(iaddr), "h"((unsigned short)id)
        : "memory");
}

// ---- one (row, half) -------------------------------------------------------------------
// Appends the scores >= tau of this lane's n TMEM columns to its list while `act` (stores
// stop at CAP); returns how many reach tau.  Warp-collective (TMEM loads).
template <int CAP>
SDM_DEV int pk_filter(uint32_t tcol, int n, float tau, bool act, uint32_t lv, uint32_t li) {
    int c = 0;
    for (int c0 = 0; c0 < n; c0 += 64) {
        float v[64];
        ptx::tmem_ld64(tcol + (uint32_t)c0, v);
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            const bool take = v[i] >= tau;
            pk_store_if(act && take && c < CAP, lv + (uint32_t)c * 512u, v[i],
                        li + (uint32_t)c * 256u, c0 + i);
            c += take ? 1 : 0;
        }
    }
    return c;
}

// The exact top K of the list (c entries) by (value desc, id asc), written to Ov/Oi[0..K).
template <int KP, int CAP>
__device__ __noinline__ void pk_exact_list(const float* Lv, const uint16_t* Li, int c, int K,
                                           float* Ov, uint16_t* Oi) {
    constexpr int S = 128;
    float r[KP];
    int ri[KP];
#pragma unroll
    for (int e = 0; e < KP; ++e) {
        r[e] = -INFINITY;
        ri[e] = 0x7fffffff;
    }
    for (int b0 = 0; b0 < CAP; b0 += KP) {
        if (b0 >= c) break;
        float s[KP];
        int si[KP];
#pragma unroll
        for (int e = 0; e < KP; ++e) {
            const bool ok = b0 + e < c;
            s[e] = ok ? Lv[(b0 + e) * S] : -INFINITY;
            si[e] = ok ? (int)Li[(b0 + e) * S] : 0x7fffffff;
        }
        pk_xsort<KP>(s, si);
        pk_xmerge<KP>(r, ri, s, si);
    }
#pragma unroll
    for (int e = 0; e < KP; ++e)
        if (e < K) {
            Ov[e * S] = r[e];
            Oi[e * S] = (uint16_t)ri[e];
        }
}

// Selects the K best of this lane's row-half (TMEM columns [tcol, tcol + n)) into the sorted
// list Ov/Oi (stride 128), best first.  Returns false when the threshold search failed (the
// row is then re-scored exactly).  Warp-collective.
template <int KP>
SDM_DEV bool pk_half(uint32_t tcol, int n, int K, float z0, bool valid, uint32_t lv, uint32_t li,
                     const float* Lv, const uint16_t* Li, float* Ov, uint16_t* Oi) {
    using C = PkCfg<KP>;
    constexpr int S = 128, CAP = C::CAP, PB = C::PB;
    constexpr unsigned FULL = 0xffffffffu;
    // 1. mean and spread of the row's scores
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f, q0 = 0.f, q1 = 0.f, q2 = 0.f, q3 = 0.f;
    for (int c0 = 0; c0 < n; c0 += 64) {
        float v[64];
        ptx::tmem_ld64(tcol + (uint32_t)c0, v);
#pragma unroll
        for (int i = 0; i < 64; i += 4) {
            s0 += v[i];
            s1 += v[i + 1];
            s2 += v[i + 2];
            s3 += v[i + 3];
            q0 = fmaf(v[i], v[i], q0);
            q1 = fmaf(v[i + 1], v[i + 1], q1);
            q2 = fmaf(v[i + 2], v[i + 2], q2);
            q3 = fmaf(v[i + 3], v[i + 3], q3);
        }
    }
    const float inv_n = 1.f / (float)n;
    const float mu = ((s0 + s1) + (s2 + s3)) * inv_n;
    const float sd = sqrtf(fmaxf(((q0 + q1) + (q2 + q3)) * inv_n - mu * mu, 0.f));
    // 2. filter, with the threshold moved (bisection in z) until K <= count <= CAP
    float z = z0, zlo = -INFINITY, zhi = INFINITY;
    float tau = z0 == -INFINITY ? -INFINITY : fmaf(z0, sd, mu);
    bool ok = !valid;
    int c = 0;
    for (int it = 0; it < PK_ITERS; ++it) {
        const bool act = !ok;
        const int cc = pk_filter<CAP>(tcol, n, tau, act, lv, li);
        if (act) {
            c = cc;
            if (c >= K && c <= CAP) {
                ok = true;
            } else {
                if (c < K) zhi = z; else zlo = z;
                z = (zlo > -INFINITY && zhi < INFINITY) ? 0.5f * (zlo + zhi)
                                                          : (c < K ? z - 1.f : z + 1.f);
                tau = fmaf(z, sd, mu);
            }
        }
        if (__all_sync(FULL, ok)) break;
    }
    const bool good = ok && valid;
    // 3. keyed selection of the K best
    const float off = tau == -INFINITY ? 0.f : tau;
    float R[KP];
#pragma unroll
    for (int e = 0; e < KP; ++e) R[e] = -INFINITY;
    float dropped = -INFINITY;
#pragma unroll 1
    for (int b0 = 0; b0 < CAP; b0 += KP) {
        if (!__any_sync(FULL, good && c > b0)) break;
        float s[KP];
#pragma unroll
        for (int e = 0; e < KP; ++e)
            s[e] = b0 + e < c ? pk_pack<PB>((Lv[(b0 + e) * S] - off) + 0.f, b0 + e) : -INFINITY;
        pk_ksort<KP>(s);
        dropped = fmaxf(dropped, pk_kmerge<KP>(R, s));
    }
    if (K < KP) dropped = fmaxf(dropped, pk_pick<KP>(R, K));
    const bool amb = good && pk_hi<PB>(pk_pick<KP>(R, K - 1)) == pk_hi<PB>(dropped);
    if (__any_sync(FULL, amb)) {
        if (amb) pk_exact_list<KP, CAP>(Lv, Li, c, K, Ov, Oi);
    }
    // the keys go to the output area; each is then replaced, in order, by its list entry
    if (!amb) {
#pragma unroll
        for (int q = 0; q < KP; ++q)
            if (q < K) Ov[q * S] = R[q];
    }
    bool near = false;
#pragma unroll 4
    for (int q = 0; q < K; ++q) {
        const float key = Ov[q * S];
        const float nkey = q + 1 < K ? Ov[(q + 1) * S] : 0.f;
        near = near || (q + 1 < K && pk_hi<PB>(key) == pk_hi<PB>(nkey));
        const int pos = min(pk_code<PB>(key), CAP - 1);
        const float lvv = Lv[pos * S];
        const uint16_t lii = Li[pos * S];
        if (good && !amb) {
            Ov[q * S] = lvv;
            Oi[q * S] = lii;
        }
    }
    if (__any_sync(FULL, good && near && !amb)) pk_fixup_smem<uint16_t>(Ov, Oi, K, good && !amb);
    return ok;
}

// ---- the combine -----------------------------------------------------------------------
// Key of a staircase pair: d = off - sum (smaller is better) with the pair's code in the low
// CB bits, negated so that larger keys are better and the networks stay descending.  For
// d < 0 the code is written reflected, so that along a run (d non-decreasing, codes
// increasing) the keys fall strictly whatever the sign of d.
template <int CB>
SDM_DEV float pk_ckey(float d, int code) {
    constexpr int M = (1 << CB) - 1;
    const int bits = __float_as_int(d);
    const int low = bits < 0 ? M - code : code;
    return __int_as_float(((bits & ~M) | low) ^ (int)0x80000000);
}
template <int CB>
SDM_DEV int pk_ccode(float key) {
    constexpr int M = (1 << CB) - 1;
    const int p = __float_as_int(key) ^ (int)0x80000000;
    return p < 0 ? M - (p & M) : (p & M);
}

// The exact top t of the staircase over the sorted half lists (value desc, slot asc), written
// out as slots and weights.  Only for rows whose keyed selection stays ambiguous twice (exactly
// equal sums at the boundary).
template <int KP>
__device__ __noinline__ void pk_exact_combine(const float* Av, const uint16_t* Ai,
                                              const float* Bv, const uint16_t* Bi, int K, int t,
                                              int n, int32_t* io, float* wo) {
    constexpr int S = 128;
    float r[KP];
    int ri[KP];
#pragma unroll
    for (int e = 0; e < KP; ++e) {
        r[e] = -INFINITY;
        ri[e] = 0x7fffffff;
    }
    int a = 0, b = 0;  // next pair in (a, b) order
    while (a < K && a < t) {
        float s[KP];
        int si[KP];
#pragma unroll
        for (int e = 0; e < KP; ++e) {
            const bool ok = a < K && a < t;
            s[e] = ok ? Av[a * S] + Bv[b * S] : -INFINITY;
            si[e] = ok ? (int)Ai[a * S] * n + (int)Bi[b * S] : 0x7fffffff;
            if (ok) {
                ++b;
                if (b >= K || (a + 1) * (b + 1) > t) {
                    ++a;
                    b = 0;
                }
            }
        }
        pk_xsort<KP>(s, si);
        pk_xmerge<KP>(r, ri, s, si);
    }
    float z = 0.f;
#pragma unroll
    for (int q = 0; q < KP; ++q) z += q < t ? __expf(r[q] - r[0]) : 0.f;
    const float rz = 1.f / z;
#pragma unroll
    for (int q = 0; q < KP; ++q)
        if (q < t) {
            io[q] = ri[q];
            wo[q] = __expf(r[q] - r[0]) * rz;
        }
}

// One part of the staircase merged into R (keys, best first), the largest key dropped kept in
// `dropped`.  Part 0: rows a = 0, 1 and the remaining pairs (a, b >= 2) with a even; part 1:
// columns b = 0, 1 (a >= 2) and the remaining pairs with a odd.  Remaining pairs are kept
// (listed at rk/rab, count nr) only when they beat the current top-th key.
template <int KP>
SDM_DEV void pk_combine_part(int part, const float (&A)[KP], const float (&Bl)[KP],
                             const float* Av, const float* Bv, int K, int t, float off,
                             bool valid, uint32_t rk, uint32_t rab, const float* Rk,
                             float (&R)[KP], float& dropped) {
    using C = PkCfg<KP>;
    constexpr int S = 128, CB = C::CB;
    constexpr unsigned FULL = 0xffffffffu;
    float s[KP];
#pragma unroll 1
    for (int r = 0; r < 2; ++r) {
        const float fix = part == 0 ? (r == 0 ? A[0] : A[1]) : (r == 0 ? Bl[0] : Bl[1]);
        const int len = min(K, t / (r + 1)) - (part == 0 ? 0 : 2);
        const int code0 = 1 + (2 * part + r) * KP;
#pragma unroll
        for (int e = 0; e < KP; ++e) {
            const float sum = part == 0 ? fix + Bl[e] : A[min(e + 2, KP - 1)] + fix;
            s[e] = e < len ? pk_ckey<CB>(off - sum, code0 + e) : -INFINITY;
        }
        dropped = fmaxf(dropped, pk_kmerge<KP>(R, s));
    }
    const float kt = pk_pick<KP>(R, t - 1);
    int nr = 0;
    for (int a = 2 + part; a < K && 3 * (a + 1) <= t; a += 2) {
        const float aa = Av[a * S];
        const int bend = min(K, t / (a + 1));
        for (int b = 2; b < bend; ++b) {
            const float k = pk_ckey<CB>(off - (aa + Bv[b * S]), 1 + 4 * KP + part * C::REST + nr);
            const bool take = valid && k > kt;
            pk_store_if(take, rk + (uint32_t)nr * 512u, k, rab + (uint32_t)nr * 256u, (a << 8) | b);
            nr += take ? 1 : 0;
            dropped = take ? dropped : fmaxf(dropped, k);
        }
    }
    if (__any_sync(FULL, nr > 0)) {
        if (__any_sync(FULL, nr > 8)) {
#pragma unroll
            for (int e = 0; e < KP; ++e) s[e] = e < nr ? Rk[e * S] : -INFINITY;
            pk_ksort<KP>(s);
        } else {
            float s8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) s8[e] = e < nr ? Rk[e * S] : -INFINITY;
            pk_ksort<8>(s8);
#pragma unroll
            for (int e = 0; e < KP; ++e) s[e] = e < 8 ? s8[e] : -INFINITY;
        }
        dropped = fmaxf(dropped, pk_kmerge<KP>(R, s));
    }
}

// Pair (a, b) of a combine key's code; rest pairs are read from their part's list.
template <int KP>
SDM_DEV void pk_decode(float key, int K, const uint16_t* Rab0, const uint16_t* Rab1, int& a,
                       int& b) {
    using C = PkCfg<KP>;
    constexpr int LOG = C::LOG_KP;
    const int code = pk_ccode<C::CB>(key) - 1;
    const int rp = min(max(code - 4 * KP, 0), 2 * C::REST - 1);
    const int ab = (int)(rp < C::REST ? Rab0 : Rab1)[(rp & (C::REST - 1)) * 128];
    const bool isrow = code < 2 * KP, iscol = !isrow && code < 4 * KP;
    a = isrow ? code >> LOG : (iscol ? 2 + (code & (KP - 1)) : ab >> 8);
    b = isrow ? (code & (KP - 1)) : (iscol ? (code >> LOG) - 2 : ab & 0xff);
    a = min(max(a, 0), K - 1);
    b = min(max(b, 0), K - 1);
}

// ---- the kernel ------------------------------------------------------------------------
template <int KP>
__global__ void __launch_bounds__(PK_THREADS, 1) score_pk_kernel(
    const __grid_constant__ CUtensorMap xmap0, const __grid_constant__ CUtensorMap xmap1,
    const __grid_constant__ CUtensorMap skmap0, const __grid_constant__ CUtensorMap skmap1,
    PkArgs p) {
    using C = PkCfg<KP>;
    extern __shared__ unsigned char pk_smem_raw[];
    unsigned char* sm = pk_smem_raw + ((1024 - (ptx::smem_u32(pk_smem_raw) & 1023)) & 1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = warp >> 2;                      // half this thread selects
    const int row = ((warp & 3) << 5) | lane;     // TMEM lane
    const int role = blockIdx.z, h = blockIdx.y;
    const CUtensorMap* xmap = role ? &xmap1 : &xmap0;
    const CUtensorMap* skmap = role ? &skmap1 : &skmap0;
    const int bti = blockIdx.x / p.n_tt, tti = blockIdx.x % p.n_tt;
    const int b0 = bti * p.bb, t0 = tti * p.bt;
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + C::OFF_CTRL);
    uint64_t* bar_mma = bar_tma + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_tma + 2);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
    int* nflag = abort_flag + 1;
    int* flagged = abort_flag + 4;                // [128] rows to re-score
    unsigned char* rowbad = reinterpret_cast<unsigned char*>(flagged + 128);  // [128]

    if (warp == 0) ptx::tmem_alloc(tmem_slot, 512);
    if (tid == 0) {
        ptx::mbar_init(bar_tma, 1);
        ptx::mbar_init(bar_mma, 1);
        *abort_flag = 0;
        *nflag = 0;
        ptx::fence_mbar_init();
    }
    if (tid < 128) rowbad[tid] = 0;
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t deadline = ptx::globaltimer_ns() + 2000000000ull;
    const int n = p.n, K = p.k_half, top = p.top[role];

    if (tid == 0) {
        const uint32_t xbytes = 2u * 64u * 2u * 128u;
        ptx::mbar_arrive_expect_tx(bar_tma, xbytes + 2u * 64u * 2u * (uint32_t)n);
        ptx::tma_load_4d(sm + PK_OFF_X, xmap, 0, t0, h, b0, bar_tma);
        ptx::tma_load_4d(sm + PK_OFF_X + 16384, xmap, 64, t0, h, b0, bar_tma);
        ptx::tma_load_2d(sm + PK_OFF_SK, skmap, 0, (h * 2 + 0) * n, bar_tma);
        ptx::tma_load_2d(sm + PK_OFF_SK + 32768, skmap, 0, (h * 2 + 1) * n, bar_tma);
        if (ptx::mbar_wait_bounded(bar_tma, 0, deadline)) {
            ptx::tc_fence_after();
            const uint32_t id = ptx::idesc_bf16_f32(128, n);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint64_t ad = ptx::umma_desc_kmajor_sw128(sm + PK_OFF_X + hf * 16384);
                const uint64_t bd = ptx::umma_desc_kmajor_sw128(sm + PK_OFF_SK + hf * 32768);
#pragma unroll
                for (int k = 0; k < 4; ++k)  // K = 64 in steps of 16 (32 bytes)
                    ptx::umma_bf16(tmem + 256u * hf, ad + 2 * k, bd + 2 * k, id, k > 0 ? 1u : 0u);
            }
            ptx::umma_commit(bar_mma);
        } else {
            *abort_flag = 1;
        }
    }
    if (!ptx::mbar_wait_bounded(bar_mma, 0, deadline)) *abort_flag = 1;
    ptx::tc_fence_after();
    __syncthreads();
    const bool aborted = *abort_flag != 0;

    const int bi = row / p.bt, ti = row % p.bt;
    const int b = b0 + bi, t = t0 + ti;
    const bool row_ok = !aborted && bi < p.bb && b < p.B && t < p.T;

    // per-half selection: lists in the list area, sorted output over the (consumed) sub-key tile
    const uint32_t lbase = ptx::smem_u32(sm + PK_OFF_L + g * C::LIST_BYTES);
    const uint32_t lv = lbase + (uint32_t)row * 4u;
    const uint32_t li = lbase + (uint32_t)C::CAP * 512u + (uint32_t)row * 2u;
    const float* Lv = reinterpret_cast<const float*>(sm + PK_OFF_L + g * C::LIST_BYTES) + row;
    const uint16_t* Li =
        reinterpret_cast<const uint16_t*>(sm + PK_OFF_L + g * C::LIST_BYTES + C::CAP * 512) + row;
    float* Ov = reinterpret_cast<float*>(sm + PK_OFF_SK + g * 32768) + row;
    uint16_t* Oi = reinterpret_cast<uint16_t*>(sm + PK_OFF_SK + g * 32768 + KP * 512) + row;
    if (!aborted) {
        const bool okh = pk_half<KP>(tmem + ((uint32_t)((warp & 3) * 32) << 16) + 256u * g, n, K,
                                     p.z0, row_ok, lv, li, Lv, Li, Ov, Oi);
        if (row_ok && !okh) rowbad[row] = 1;
    }
    ptx::tc_fence_before();
    __syncthreads();

    // combine: every thread merges one part of its row's staircase (warps 0-3 part 0, warps
    // 4-7 part 1); part 1 hands its keys over through the (consumed) x tile.  Rows whose
    // boundary stays ambiguous run both parts again on warps 0-3 with keys centred on the
    // boundary sum (the same code, in the same loop).
    const int top_s = top;  // staged outputs: [128 rows][top] slots and weights
    int32_t* st_idx = reinterpret_cast<int32_t*>(sm + PK_OFF_L + C::REST * 768);
    float* st_w = reinterpret_cast<float*>(sm + PK_OFF_L + C::LIST_BYTES + C::REST * 768);
    {
        constexpr int S = 128, CB = C::CB;
        constexpr unsigned FULL = 0xffffffffu;
        const float* Av = reinterpret_cast<const float*>(sm + PK_OFF_SK) + row;
        const uint16_t* Ai = reinterpret_cast<const uint16_t*>(sm + PK_OFF_SK + KP * 512) + row;
        const float* Bv = reinterpret_cast<const float*>(sm + PK_OFF_SK + 32768) + row;
        const uint16_t* Bi = reinterpret_cast<const uint16_t*>(sm + PK_OFF_SK + 32768 + KP * 512) + row;
        // each part's list of remaining pairs sits in that half's (consumed) candidate list
        uint32_t rk[2], rab[2];
        const float* Rk[2];
        const uint16_t* Rab[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            unsigned char* base = sm + PK_OFF_L + q * C::LIST_BYTES;
            rk[q] = ptx::smem_u32(base) + (uint32_t)row * 4u;
            rab[q] = ptx::smem_u32(base) + (uint32_t)C::REST * 512u + (uint32_t)row * 2u;
            Rk[q] = reinterpret_cast<const float*>(base) + row;
            Rab[q] = reinterpret_cast<const uint16_t*>(base + C::REST * 512) + row;
        }
        const bool live = row_ok && rowbad[row] == 0;
        float A[KP], Bl[KP];
#pragma unroll
        for (int e = 0; e < KP; ++e) {
            A[e] = e < K ? Av[e * S] : 0.f;
            Bl[e] = e < K ? Bv[e * S] : 0.f;
        }
        const float M0 = A[0] + Bl[0];
        float R[KP], Rsave[KP];
#pragma unroll
        for (int e = 0; e < KP; ++e) R[e] = -INFINITY;
        float dropped = -INFINITY;
        float* X = reinterpret_cast<float*>(sm + PK_OFF_X) + row;          // [KP + 1], then sums
        int* XS = reinterpret_cast<int*>(sm + PK_OFF_X + KP * 512) + row;   // slots
        bool amb = false;
        float off2 = M0;
        int it_end = 1;
#pragma unroll 1
        for (int it = 0; it < it_end; ++it) {
            const int part = it == 0 ? g : it - 1;
            if (!aborted)
                pk_combine_part<KP>(part, A, Bl, Av, Bv, K, top, it == 0 ? M0 : off2,
                                    it == 0 ? live : amb, rk[part], rab[part], Rk[part], R,
                                    dropped);
            if (it == 0) {
                if (g == 1) {
#pragma unroll
                    for (int e = 0; e < KP; ++e) X[e * S] = R[e];
                    X[KP * S] = dropped;
                }
                __syncthreads();
                if (g == 0 && !aborted) {
                    float sx[KP];
#pragma unroll
                    for (int e = 0; e < KP; ++e) sx[e] = X[e * S];
                    dropped = fmaxf(dropped, fmaxf(X[KP * S], pk_kmerge<KP>(R, sx)));
                    if (top < KP) dropped = fmaxf(dropped, pk_pick<KP>(R, top));
                    amb = live && pk_hi<CB>(pk_pick<KP>(R, top - 1)) == pk_hi<CB>(dropped);
                    if (__any_sync(FULL, amb)) {
                        int ka, kb;
                        pk_decode<KP>(pk_pick<KP>(R, top - 1), K, Rab[0], Rab[1], ka, kb);
                        off2 = Av[ka * S] + Bv[kb * S];
#pragma unroll
                        for (int e = 0; e < KP; ++e) {
                            Rsave[e] = R[e];
                            R[e] = -INFINITY;
                        }
                        dropped = -INFINITY;
                        it_end = 3;
                    }
                }
            }
        }
        if (g == 0 && !aborted) {
            if (it_end == 3) {
                if (top < KP) dropped = fmaxf(dropped, pk_pick<KP>(R, top));
                const bool amb2 = amb && pk_hi<CB>(pk_pick<KP>(R, top - 1)) == pk_hi<CB>(dropped);
#pragma unroll
                for (int e = 0; e < KP; ++e) R[e] = amb ? R[e] : Rsave[e];
                if (amb2) pk_exact_combine<KP>(Av, Ai, Bv, Bi, K, top, n, st_idx + row * top_s,
                                               st_w + row * top_s);
                amb = amb2;
            }
            // the keys, in order, become (sum, slot); then exact order among equal keys
            const bool act = live && !amb;
#pragma unroll
            for (int e = 0; e < KP; ++e)
                if (e < top) X[e * S] = R[e];
            bool near = false;
#pragma unroll 4
            for (int q = 0; q < top; ++q) {
                const float key = X[q * S];
                const float nkey = q + 1 < top ? X[(q + 1) * S] : 0.f;
                near = near || (q + 1 < top && pk_hi<CB>(key) == pk_hi<CB>(nkey));
                int a, bb;
                pk_decode<KP>(key, K, Rab[0], Rab[1], a, bb);
                X[q * S] = Av[a * S] + Bv[bb * S];
                XS[q * S] = (int)Ai[a * S] * n + (int)Bi[bb * S];
            }
            if (__any_sync(FULL, act && near)) pk_fixup_smem<int>(X, XS, top, act);
            if (act) {
                const float mx = X[0];
                float z = 0.f;
#pragma unroll 4
                for (int q = 0; q < top; ++q) {
                    const float ev = __expf(X[q * S] - mx);
                    X[q * S] = ev;
                    z += ev;
                }
                const float rz = 1.f / z;
#pragma unroll 4
                for (int q = 0; q < top; ++q) {
                    st_idx[row * top_s + q] = XS[q * S];
                    st_w[row * top_s + q] = X[q * S] * rz;
                }
            }
            if (row_ok && rowbad[row]) flagged[atomicAdd(nflag, 1)] = row;
        }
    }
    __syncthreads();
    // staged rows out, one row per warp step (the lanes over its slots): coalesced stores
    if (!aborted) {
        for (int r = warp; r < 128; r += PK_THREADS / 32) {
            const int rb = b0 + r / p.bt, rt = t0 + r % p.bt;
            if (r / p.bt >= p.bb || rb >= p.B || rt >= p.T || rowbad[r]) continue;
            const size_t ro = (((size_t)rb * p.H + h) * p.T + rt) * top_s;
            for (int q = lane; q < top_s; q += 32) {
                p.idx[role][ro + q] = st_idx[r * top_s + q];
                p.w[role][ro + q] = st_w[r * top_s + q];
            }
        }
    }

    // rows the threshold search could not settle: exact re-scoring, one warp per row
    const int nf = *nflag;
    if (nf > 0) {
        float* ws = reinterpret_cast<float*>(sm + PK_OFF_L) +
                    (size_t)warp * score_simt_warp_floats(p.d_k, n, K, top);
        for (int f = warp; f < nf; f += PK_THREADS / 32) {
            const int r = flagged[f];
            const int fb = b0 + r / p.bt, ft = t0 + r % p.bt;
            const size_t row_off = ((size_t)fb * p.H + h) * p.T + ft;
            simt_score_row<__nv_bfloat16>(p.x[role] + row_off * p.d_k,
                                          p.sk[role] + (size_t)h * 2 * n * (p.d_k / 2), p.d_k, n,
                                          K, top, ws, p.idx[role] + row_off * top,
                                          p.w[role] + row_off * top);
        }
    }
    if (aborted && tid == 0) raise_err(SDM_DEVERR_TIMEOUT);
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
    (void)lane;
}

// Threshold position z for a half of n scores of which K are kept: about K + margin of n
// Gaussian draws reach mean + z*sd (margin: 2.5 standard deviations of that count, + 2);
// -inf when that covers every score.
inline float pk_z0(int n, int K) {
    const double kk = (double)K;
    const double m = ceil(2.5 * sqrt(kk * (1.0 - kk / n))) + 2.0;
    const double q = (kk + m) / n;  // upper-tail probability
    if (q >= 1.0) return -INFINITY;
    double lo = -10.0, hi = 10.0;  // 0.5 * erfc(z / sqrt(2)) = q
    for (int i = 0; i < 100; ++i) {
        const double mid = 0.5 * (lo + hi);
        if (0.5 * erfc(mid / sqrt(2.0)) > q) lo = mid; else hi = mid;
    }
    return (float)(0.5 * (lo + hi));
}

}  // namespace sdm
