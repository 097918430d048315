// Product-key scoring on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), bf16 inputs,
// d_k = 128 (§2 Background "Product Key Memory", §3 Method "Sparse addressing", §4 "SDM
// Configuration").
//
// One CTA scores a tile of ROWS rows (tokens of one head and role) and holds the whole SM
// (512 TMEM columns).  TMA brings the x tile (both halves) and, round by round, 256 sub-keys of
// each half table; one thread issues tcgen05.mma so that TMEM holds
// D[row][j] = <x_half[row], C_half[j]> for the round's sub-keys j:
//   ROWS = 128: one MMA per half (M = 128, K = 64); half h in columns [256h, 256h + 256).
//   ROWS = 64:  one MMA with K = 128 over A = [x_half0 | 0 ; 0 | x_half1] and B = [C0 | C1],
//               so lanes 0-63 get half 0 and lanes 64-127 half 1 of the same 64 tokens in 256
//               columns; rounds alternate between two such buffers.
// One thread per (row, half) then keeps the K best sub-keys of that half exactly:
//   1. Threshold.  The row's mean and spread over its n scores give tau = mean + z*sd, z
//      chosen on the host so that about K + margin scores reach it (the sub-key tables make
//      each row's half-scores close to Gaussian, but nothing relies on it: a row whose count
//      falls outside [K, CAP] is filtered again with z moved, by bisection).
//   2. Filter.  The scores >= tau go, with their sub-indices, to the thread's list in shared
//      memory (CAP entries).  With more than 256 sub-keys per half the rounds are computed
//      again for this pass (the tensor cores are idle otherwise).
//   3. Order.  Keys are the differences score - tau with their list position written into the
//      low mantissa bits: distinct, and ordered like the scores except among scores whose keys
//      agree above those bits.  Blocks of KP keys are sorted by min/max networks and merged
//      keeping the best KP; the largest key dropped on the way is kept.  If it agrees with the
//      K-th kept key above the position bits, the selection is ambiguous and is made again by
//      exact comparisons (value, then sub-index); otherwise the K kept entries are the exact
//      top K, and exact compare-exchanges put equal-key neighbours in order.
//   4. Combine.  The k x k pairs that can reach the top `top` are those with
//      (a+1)(b+1) <= top (any other pair is beaten by at least `top` pairs with no smaller sum
//      and no larger slot).  The thread of half 0 merges the staircase rows a = 0, 1 and the
//      remaining pairs with even a, the thread of half 1 the columns b = 0, 1 and the
//      remaining pairs with odd a, with the same keyed networks (key = offset - sum with a code
//      of the pair); then the two are merged.  An ambiguous boundary is redone with keys
//      centred on the boundary sum, and if still ambiguous (exactly equal sums) by exact
//      comparisons.  Slots s = i*n + j, equal sums to the lower slot; weights = softmax.
// A row that the threshold search cannot settle is scored again by one warp on CUDA cores
// (exact fp32 FMA scores and selection) at the end of the tile.
#pragma once

#include <math.h>

#include "common.cuh"
#include "score_simt.cuh"
#include "tc_ptx.cuh"

namespace sdm {

constexpr int PK_NMAX = 1024;   // sub-keys per half this kernel takes (rounds of 256)
constexpr int PK_ITERS = 8;     // filter passes before a row goes to the exact re-scoring

// Shared-memory map (bytes from a 1024-aligned base).
constexpr uint32_t PK_OFF_X = 0;        // x tile (A operand, 32 KB); later the combine's
                                        // exchange and its (sum, slot) lists
constexpr uint32_t PK_OFF_SK = 32768;   // a round of sub-keys (B operand, 2 x 32 KB); later the
                                        // sorted half lists (values [KP][ROWS] f32, ids u16)
constexpr uint32_t PK_OFF_L = 98304;    // candidate lists, then the remaining-pair lists, the
                                        // staged outputs and the re-scoring scratch

template <int KP, int ROWS>
struct PkCfg {
    static constexpr int THREADS = 2 * ROWS;
    static constexpr int S = ROWS;                  // stride of the per-row arrays
    static constexpr int CAP = KP == 16 ? 48 : KP == 32 ? 64 : 128;  // list entries per (row, half)
    static constexpr int PB = KP == 64 ? 7 : 6;     // key bits that hold a list position
    static constexpr int CB = KP == 16 ? 7 : KP == 32 ? 8 : 9;  // key bits of a pair code
    static constexpr int LOG_KP = KP == 16 ? 4 : KP == 32 ? 5 : 6;
    static constexpr int REST = KP;                 // remaining staircase pairs of one part: <= KP
    static constexpr uint32_t LIST_BYTES = (uint32_t)CAP * ROWS * 6;
    static constexpr uint32_t OFF_REST = 0;                          // in each list area
    static constexpr uint32_t OFF_STAGE = (uint32_t)REST * ROWS * 6;  // in each list area
    static constexpr uint32_t OFF_CTRL = PK_OFF_L + 2 * LIST_BYTES;
    static constexpr uint32_t SMEM = OFF_CTRL + 1024 + 1024;  // + alignment slack
    static_assert(KP * ROWS * 6 <= 32768, "sorted half list fits a sub-key tile");
    static_assert(2 * KP * ROWS * 4 <= 32768, "combine lists fit the x tile");
    static_assert(CAP <= (1 << PB), "positions fit the key bits");
    static_assert(4 * KP + 2 * REST <= (1 << CB) - 1, "pair codes fit the key bits");
    static_assert(OFF_STAGE + (uint32_t)ROWS * (KP + 1) * 4 <= LIST_BYTES, "staging fits");
    static_assert(OFF_CTRL + 2048 <= 227 * 1024, "shared memory");
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
// f with its low B bits replaced by code (truncation keeps the order, for either sign).
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

// Exact order among neighbours: the list v/ix[0..m) in shared memory (stride S) is loaded once,
// sorted (value desc, id asc) by odd-even transposition passes in registers until a pass swaps
// nothing, and stored back, on the lanes with `act`.  Used after a keyed selection, where only
// neighbours whose keys agree above the code bits can be out of order (a few passes).  Called
// by whole warps with a warp-uniform m <= N.
template <int N, int S, typename IT>
SDM_DEV void pk_fixup(float* vs, IT* ixs, int m, bool act) {
    float v[N];
    int ix[N];
#pragma unroll
    for (int i = 0; i < N; ++i) {
        v[i] = i < m ? vs[i * S] : -INFINITY;
        ix[i] = i < m ? (int)ixs[i * S] : 0x7fffffff;
    }
    for (int pass = 0; pass < m + 2; ++pass) {
        bool sw_any = false;
#pragma unroll
        for (int i = 0; i + 1 < N; ++i) {
            if ((i & 1) != (pass & 1)) continue;
            const bool sw = act && i + 1 < m && better(v[i + 1], ix[i + 1], v[i], ix[i]);
            const float tv = sw ? v[i + 1] : v[i];
            const int ti = sw ? ix[i + 1] : ix[i];
            v[i + 1] = sw ? v[i] : v[i + 1];
            ix[i + 1] = sw ? ix[i] : ix[i + 1];
            v[i] = tv;
            ix[i] = ti;
            sw_any = sw_any || sw;
        }
        if (pass > 0 && !__any_sync(0xffffffffu, sw_any)) break;
    }
    if (act) {
#pragma unroll
        for (int i = 0; i < N; ++i)
            if (i < m) {
                vs[i * S] = v[i];
                ixs[i * S] = (IT)ix[i];
            }
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
// Sums and sums of squares of this lane's nr TMEM columns (a multiple of 64).
SDM_DEV void pk_stats(uint32_t tcol, int nr, float (&acc)[8]) {
    for (int c0 = 0; c0 < nr; c0 += 64) {
        float v[64];
        ptx::tmem_ld64(tcol + (uint32_t)c0, v);
#pragma unroll
        for (int i = 0; i < 64; i += 4) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                acc[u] += v[i + u];
                acc[4 + u] = fmaf(v[i + u], v[i + u], acc[4 + u]);
            }
        }
    }
}

// Appends the scores >= tau of this lane's nr TMEM columns (sub-indices id0 + column) to its
// list while `act`, from position c (stores stop at CAP); returns the new count.
template <int CAP, int S>
SDM_DEV int pk_filter(uint32_t tcol, int nr, int id0, float tau, bool act, int c, uint32_t lv,
                      uint32_t li) {
    for (int c0 = 0; c0 < nr; c0 += 64) {
        float v[64];
        ptx::tmem_ld64(tcol + (uint32_t)c0, v);
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            const bool take = v[i] >= tau;
            pk_store_if(act && take && c < CAP, lv + (uint32_t)c * (4u * S), v[i],
                        li + (uint32_t)c * (2u * S), id0 + c0 + i);
            c += take ? 1 : 0;
        }
    }
    return c;
}

// Exact ties at the boundary: the keyed selection centred on the boundary value vb kept (its
// keys in Ov[0..K), best first) every entry above vb; the places left go to the entries equal to vb with the lowest ids (one
// scan of the list, the TC lowest kept in a small sorted register list).  Writes the K
// entries, values above vb first (in key order), to Ov/Oi; false when more than TC tied
// entries would be needed (the row is then re-scored).
template <int S, int PB>
__device__ __noinline__ bool pk_tie_list(float vb, const float* Lv, const uint16_t* Li, int c,
                                         int K, int CAPm1, float* Ov, uint16_t* Oi) {
    constexpr int TC = 8;
    int q = 0;  // the keys sit in Ov[0..K); entry q is written after key q is read (q <= e)
    for (int e = 0; e < K; ++e) {
        const int pos = min(pk_code<PB>(Ov[e * S]), CAPm1);
        const float v = Lv[pos * S];
        if (v > vb) {
            Ov[q * S] = v;
            Oi[q * S] = Li[pos * S];
            ++q;
        }
    }
    int tie[TC];
#pragma unroll
    for (int j = 0; j < TC; ++j) tie[j] = 0x7fffffff;
    for (int e = 0; e < c; ++e) {
        if (Lv[e * S] != vb) continue;
        int x = (int)Li[e * S];
#pragma unroll
        for (int j = 0; j < TC; ++j) {  // insert x, keeping the TC lowest in order
            const int lo = min(tie[j], x);
            x = max(tie[j], x);
            tie[j] = lo;
        }
    }
    if (K - q > TC) return false;
#pragma unroll
    for (int j = 0; j < TC; ++j)
        if (q + j < K) {
            Ov[(q + j) * S] = vb;
            Oi[(q + j) * S] = (uint16_t)tie[j];
        }
    return true;
}

// After the filter: the K best of the list (count c, threshold tau) sorted into Ov/Oi.
template <int KP, int ROWS>
SDM_DEV bool pk_finish_half(int K, int c, float tau, bool good, const float* Lv,
                            const uint16_t* Li, float* Ov, uint16_t* Oi) {
    using C = PkCfg<KP, ROWS>;
    constexpr int S = C::S, CAP = C::CAP, PB = C::PB;
    constexpr unsigned FULL = 0xffffffffu;
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
    bool amb = good && pk_hi<PB>(pk_pick<KP>(R, K - 1)) == pk_hi<PB>(dropped);
    bool tie_fail = false;
    if (__any_sync(FULL, amb)) {
        // ambiguous boundary: the keys again, centred on the boundary value (finest there);
        // the rows that stay ambiguous (exactly equal values) are ranked by exact scans
        const float off2 = Lv[min(pk_code<PB>(pk_pick<KP>(R, K - 1)), CAP - 1) * S];
        float R2[KP];
#pragma unroll
        for (int e = 0; e < KP; ++e) R2[e] = -INFINITY;
        float d2 = -INFINITY;
#pragma unroll 1
        for (int b0 = 0; b0 < CAP; b0 += KP) {
            if (!__any_sync(FULL, amb && c > b0)) break;
            float s[KP];
#pragma unroll
            for (int e = 0; e < KP; ++e)
                s[e] = b0 + e < c ? pk_pack<PB>((Lv[(b0 + e) * S] - off2) + 0.f, b0 + e) : -INFINITY;
            pk_ksort<KP>(s);
            d2 = fmaxf(d2, pk_kmerge<KP>(R2, s));
        }
        if (K < KP) d2 = fmaxf(d2, pk_pick<KP>(R2, K));
        const bool amb2 = amb && pk_hi<PB>(pk_pick<KP>(R2, K - 1)) == pk_hi<PB>(d2);
#pragma unroll
        for (int e = 0; e < KP; ++e) R[e] = amb ? R2[e] : R[e];
        if (amb2) {
#pragma unroll
            for (int e = 0; e < KP; ++e)
                if (e < K) Ov[e * S] = R[e];
            tie_fail = !pk_tie_list<S, PB>(off2, Lv, Li, c, K, CAP - 1, Ov, Oi);
        }
        amb = amb2;
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
    // (rows settled by ties are in order up to equal-key neighbours above the boundary)
    if (__any_sync(FULL, good && (near || amb))) pk_fixup<KP, S, uint16_t>(Ov, Oi, K, good);
    return !tie_fail;
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

// Exact ties at the boundary of the combine: the keyed selection centred on the boundary sum
// sb kept (its keys in X[0..t), best first) every pair above sb; the places left go to the
// pairs whose sum equals sb with the lowest slots (one scan of the staircase, the TC lowest in
// a small sorted register list).  Writes the t (sum, slot) pairs, sums above sb first, to
// X/XS; false when more than TC tied pairs would be needed (the row is then re-scored).
template <int KP, int ROWS>
__device__ __noinline__ bool pk_tie_combine(float sb, const float* Av, const uint16_t* Ai,
                                            const float* Bv, const uint16_t* Bi,
                                            const uint16_t* Rab0, const uint16_t* Rab1, int K,
                                            int t, int n, float* X, int* XS);

// One part of the staircase merged into R (keys, best first), the largest key dropped kept in
// `dropped`.  Part 0: rows a = 0, 1 and the remaining pairs (a, b >= 2) with a even; part 1:
// columns b = 0, 1 (a >= 2) and the remaining pairs with a odd.  Remaining pairs are kept
// (listed at rk/rab) only when they beat the current top-th key.
template <int KP, int ROWS>
SDM_DEV void pk_combine_part(int part, const float* Av, const float* Bv, int K, int t, float off,
                             bool valid, uint32_t rk, uint32_t rab, const float* Rk,
                             float (&R)[KP], float& dropped) {
    using C = PkCfg<KP, ROWS>;
    constexpr int S = C::S, CB = C::CB;
    constexpr unsigned FULL = 0xffffffffu;
    // the run sources: rows take the other half's list, columns this half's (from a = 2)
    float src[KP];
#pragma unroll
    for (int e = 0; e < KP; ++e) {
        const int ia = min(e + 2, KP - 1);
        src[e] = part == 0 ? (e < K ? Bv[e * S] : 0.f) : (ia < K ? Av[ia * S] : 0.f);
    }
    float s[KP];
#pragma unroll 1
    for (int r = 0; r < 2; ++r) {
        const float fix = part == 0 ? Av[r * S] : Bv[r * S];
        const int len = min(K, t / (r + 1)) - (part == 0 ? 0 : 2);
        const int code0 = 1 + (2 * part + r) * KP;
#pragma unroll
        for (int e = 0; e < KP; ++e)
            s[e] = e < len ? pk_ckey<CB>(off - (fix + src[e]), code0 + e) : -INFINITY;
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
            pk_store_if(take, rk + (uint32_t)nr * (4u * S), k, rab + (uint32_t)nr * (2u * S),
                        (a << 8) | b);
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

// Pair (a, b) of a combine key's code; remaining pairs are read from their part's list.
template <int KP, int ROWS>
SDM_DEV void pk_decode(float key, int K, const uint16_t* Rab0, const uint16_t* Rab1, int& a,
                       int& b) {
    using C = PkCfg<KP, ROWS>;
    constexpr int LOG = C::LOG_KP;
    const int code = pk_ccode<C::CB>(key) - 1;
    const int rp = min(max(code - 4 * KP, 0), 2 * C::REST - 1);
    const int ab = (int)(rp < C::REST ? Rab0 : Rab1)[(rp & (C::REST - 1)) * C::S];
    const bool isrow = code < 2 * KP, iscol = !isrow && code < 4 * KP;
    a = isrow ? code >> LOG : (iscol ? 2 + (code & (KP - 1)) : ab >> 8);
    b = isrow ? (code & (KP - 1)) : (iscol ? (code >> LOG) - 2 : ab & 0xff);
    a = min(max(a, 0), K - 1);
    b = min(max(b, 0), K - 1);
}

template <int KP, int ROWS>
__device__ __noinline__ bool pk_tie_combine(float sb, const float* Av, const uint16_t* Ai,
                                            const float* Bv, const uint16_t* Bi,
                                            const uint16_t* Rab0, const uint16_t* Rab1, int K,
                                            int t, int n, float* X, int* XS) {
    constexpr int S = ROWS, TC = 8;
    int q = 0;  // entry q is written after key q is read (q <= e)
    for (int e = 0; e < t; ++e) {
        int a, b;
        pk_decode<KP, ROWS>(X[e * S], K, Rab0, Rab1, a, b);
        const float v = Av[a * S] + Bv[b * S];
        if (v > sb) {
            X[q * S] = v;
            XS[q * S] = (int)Ai[a * S] * n + (int)Bi[b * S];
            ++q;
        }
    }
    int tie[TC];
#pragma unroll
    for (int j = 0; j < TC; ++j) tie[j] = 0x7fffffff;
    for (int a = 0; a < K && a < t; ++a) {
        const float aa = Av[a * S];
        const int bend = min(K, t / (a + 1));
        for (int b = 0; b < bend; ++b) {
            if (aa + Bv[b * S] != sb) continue;
            int x = (int)Ai[a * S] * n + (int)Bi[b * S];
#pragma unroll
            for (int j = 0; j < TC; ++j) {
                const int lo = min(tie[j], x);
                x = max(tie[j], x);
                tie[j] = lo;
            }
        }
    }
    if (t - q > TC) return false;
#pragma unroll
    for (int j = 0; j < TC; ++j)
        if (q + j < t) {
            X[(q + j) * S] = sb;
            XS[(q + j) * S] = tie[j];
        }
    return true;
}

// ---- the kernel ------------------------------------------------------------------------
template <int KP, int ROWS>
__global__ void __launch_bounds__(2 * ROWS, 1) score_pk_kernel(
    const __grid_constant__ CUtensorMap xmap0, const __grid_constant__ CUtensorMap xmap1,
    const __grid_constant__ CUtensorMap skmap0, const __grid_constant__ CUtensorMap skmap1,
    PkArgs p) {
    using C = PkCfg<KP, ROWS>;
    constexpr int S = C::S, NW = C::THREADS / 32;
    constexpr unsigned FULL = 0xffffffffu;
    extern __shared__ unsigned char pk_smem_raw[];
    unsigned char* sm = pk_smem_raw + ((1024 - (ptx::smem_u32(pk_smem_raw) & 1023)) & 1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // ROWS = 128: warps 0-3 half 0, 4-7 half 1, lane quarter = warp % 4;
    // ROWS = 64:  warps 0-1 half 0 (TMEM lanes 0-63), 2-3 half 1 (lanes 64-127)
    const int g = ROWS == 128 ? warp >> 2 : warp >> 1;
    const int row = ROWS == 128 ? (((warp & 3) << 5) | lane) : (((warp & 1) << 5) | lane);
    const uint32_t tlane = (uint32_t)((ROWS == 128 ? (warp & 3) : warp) * 32) << 16;
    const int role = blockIdx.z, h = blockIdx.y;
    const CUtensorMap* xmap = role ? &xmap1 : &xmap0;
    const CUtensorMap* skmap = role ? &skmap1 : &skmap0;
    const int bti = blockIdx.x / p.n_tt, tti = blockIdx.x % p.n_tt;
    const int b0 = bti * p.bb, t0 = tti * p.bt;
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + C::OFF_CTRL);
    uint64_t* bar_mma = bar_tma + 1;  // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_tma + 3);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
    int* nflag = abort_flag + 1;
    int* flagged = abort_flag + 4;                // [ROWS] rows to re-score
    unsigned char* rowbad = reinterpret_cast<unsigned char*>(flagged + ROWS);  // [ROWS]

    if (warp == 0) ptx::tmem_alloc(tmem_slot, 512);
    if (tid == 0) {
        ptx::mbar_init(bar_tma, 1);
        ptx::mbar_init(bar_mma, 1);
        ptx::mbar_init(bar_mma + 1, 1);
        *abort_flag = 0;
        *nflag = 0;
        ptx::fence_mbar_init();
    }
    if (tid < ROWS) rowbad[tid] = 0;
    if (ROWS == 64) {
        // the zero quadrants of A = [x_half0 | 0 ; 0 | x_half1]
        uint4* zq = reinterpret_cast<uint4*>(sm + PK_OFF_X + 8192);
        for (int i = tid; i < 16384 / 16; i += C::THREADS) zq[i] = make_uint4(0, 0, 0, 0);
        ptx::fence_proxy_async_smem();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t deadline = ptx::globaltimer_ns() + 2000000000ull;
    const int n = p.n, K = p.k_half, top = p.top[role];
    const int NR = (n + 255) >> 8;

    // x tile and the first round of sub-keys
    // thread 0: both half tables' round r on bar_tma, with the one arrival of that phase (plus
    // `extra` bytes loaded on it by the caller).  A box of min(n, 256) rows always lands whole
    // (rows past the table: the next table's or the zero fill): its bytes complete the phase.
    auto load_sk = [&](int r, uint32_t extra) {
        ptx::mbar_arrive_expect_tx(bar_tma, extra + 2u * 128u * (uint32_t)min(n, 256));
        ptx::tma_load_2d(sm + PK_OFF_SK, skmap, 0, (h * 2 + 0) * n + 256 * r, bar_tma);
        ptx::tma_load_2d(sm + PK_OFF_SK + 32768, skmap, 0, (h * 2 + 1) * n + 256 * r, bar_tma);
    };
    if (tid == 0) {
        load_sk(0, 2u * 64u * 2u * (uint32_t)ROWS);
        if (ROWS == 128) {
            ptx::tma_load_4d(sm + PK_OFF_X, xmap, 0, t0, h, b0, bar_tma);
            ptx::tma_load_4d(sm + PK_OFF_X + 16384, xmap, 64, t0, h, b0, bar_tma);
        } else {
            ptx::tma_load_4d(sm + PK_OFF_X, xmap, 0, t0, h, b0, bar_tma);
            ptx::tma_load_4d(sm + PK_OFF_X + 16384 + 8192, xmap, 64, t0, h, b0, bar_tma);
        }
    }
    uint32_t ph_tma = 0, ph_mma0 = 0, ph_mma1 = 0;
    int seq = 0;        // rounds computed so far
    bool aborted = false;
    // Round r into TMEM (thread 0 issues, everyone waits); the next round's sub-keys are
    // requested as soon as the MMA has read this round's.  Returns the TMEM buffer.
    auto run_round = [&](int r) -> int {
        const int buf = ROWS == 64 ? (seq & 1) : 0;
        const int nr = min(256, n - 256 * r);
        if (tid == 0) {
            ptx::tc_fence_after();
            if (ptx::mbar_wait_bounded(bar_tma, ph_tma, deadline)) {
                ptx::tc_fence_after();
                const uint32_t id = ptx::idesc_bf16_f32(128, nr);
                if (ROWS == 128) {
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const uint64_t ad = ptx::umma_desc_kmajor_sw128(sm + PK_OFF_X + hf * 16384);
                        const uint64_t bd = ptx::umma_desc_kmajor_sw128(sm + PK_OFF_SK + hf * 32768);
#pragma unroll
                        for (int k = 0; k < 4; ++k)  // K = 64 in steps of 16 (32 bytes)
                            ptx::umma_bf16(tmem + 256u * hf, ad + 2 * k, bd + 2 * k, id, k > 0 ? 1u : 0u);
                    }
                } else {
#pragma unroll
                    for (int kb = 0; kb < 2; ++kb) {
                        const uint64_t ad = ptx::umma_desc_kmajor_sw128(sm + PK_OFF_X + kb * 16384);
                        const uint64_t bd = ptx::umma_desc_kmajor_sw128(sm + PK_OFF_SK + kb * 32768);
#pragma unroll
                        for (int k = 0; k < 4; ++k)  // K = 128 in steps of 16
                            ptx::umma_bf16(tmem + 256u * buf, ad + 2 * k, bd + 2 * k, id,
                                           (kb | k) ? 1u : 0u);
                    }
                }
                ptx::umma_commit(bar_mma + buf);
            } else {
                *abort_flag = 1;
            }
        }
        ph_tma ^= 1;
        const uint32_t ph = buf ? ph_mma1 : ph_mma0;
        if (!ptx::mbar_wait_bounded(bar_mma + buf, ph, deadline)) *abort_flag = 1;
        if (buf) ph_mma1 ^= 1; else ph_mma0 ^= 1;
        ptx::tc_fence_after();
        if (tid == 0 && NR > 1) load_sk(r + 1 < NR ? r + 1 : 0, 0u);  // (a last prefetch is drained at exit)
        ++seq;
        return buf;
    };
    // end of a round's reads: the buffer may be written again
    auto round_done = [&]() {
        ptx::tc_fence_before();
        __syncthreads();
        aborted = *abort_flag != 0;
    };

    const int bi = row / p.bt, ti = row % p.bt;
    const int b = b0 + bi, t = t0 + ti;
    const bool row_ok = bi < p.bb && b < p.B && t < p.T;

    // 1. mean and spread of each (row, half)'s n scores
    int buf = 0;
    float acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[u] = 0.f;
    for (int r = 0; r < NR && !aborted; ++r) {
        buf = run_round(r);
        pk_stats(tmem + tlane + 256u * (ROWS == 128 ? g : buf), min(256, n - 256 * r), acc);
        round_done();
    }
    const float inv_n = 1.f / (float)n;
    const float mu = ((acc[0] + acc[1]) + (acc[2] + acc[3])) * inv_n;
    const float sd = sqrtf(fmaxf(((acc[4] + acc[5]) + (acc[6] + acc[7])) * inv_n - mu * mu, 0.f));

    // 2. filter into the lists, with the threshold moved (bisection in z) until K <= count <= CAP
    const uint32_t lbase = ptx::smem_u32(sm + PK_OFF_L + g * C::LIST_BYTES);
    const uint32_t lv = lbase + (uint32_t)row * 4u;
    const uint32_t li = lbase + (uint32_t)C::CAP * (4u * S) + (uint32_t)row * 2u;
    const float* Lv = reinterpret_cast<const float*>(sm + PK_OFF_L + g * C::LIST_BYTES) + row;
    const uint16_t* Li =
        reinterpret_cast<const uint16_t*>(sm + PK_OFF_L + g * C::LIST_BYTES + C::CAP * 4 * S) + row;
    float z = p.z0, zlo = -INFINITY, zhi = INFINITY;
    float tau = p.z0 == -INFINITY ? -INFINITY : fmaf(p.z0, sd, mu);
    bool ok = !row_ok;
    int c = 0;
    for (int it = 0; it < PK_ITERS && !aborted; ++it) {
        // one round: the scores stay in TMEM, so each warp filters again on its own; several
        // rounds: the CTA computes them again together
        if (NR == 1 ? !__any_sync(FULL, !ok) : !__syncthreads_or(!ok)) break;
        const bool act = !ok;
        int cc = 0;
        for (int r = 0; r < NR && !aborted; ++r) {
            if (NR > 1) buf = run_round(r);
            cc = pk_filter<C::CAP, S>(tmem + tlane + 256u * (ROWS == 128 ? g : buf),
                                      min(256, n - 256 * r), 256 * r, tau, act, cc, lv, li);
            if (NR > 1) round_done();
        }
        if (act) {
            c = cc;
            if (c >= K && c <= C::CAP) {
                ok = true;
            } else {
                if (c < K) zhi = z; else zlo = z;
                z = (zlo > -INFINITY && zhi < INFINITY) ? 0.5f * (zlo + zhi)
                                                          : (c < K ? z - 1.f : z + 1.f);
                tau = fmaf(z, sd, mu);
            }
        }
    }
    if (!ok && row_ok) rowbad[row] = 1;  // re-scored at the end of the tile
    ptx::tc_fence_before();
    __syncthreads();
    aborted = *abort_flag != 0;

    // 3. the K best of the list, sorted, over the (consumed) sub-key tile
    float* Ov = reinterpret_cast<float*>(sm + PK_OFF_SK + g * 32768) + row;
    uint16_t* Oi = reinterpret_cast<uint16_t*>(sm + PK_OFF_SK + g * 32768 + KP * 4 * S) + row;
    if (!aborted && !pk_finish_half<KP, ROWS>(K, c, tau, ok && row_ok, Lv, Li, Ov, Oi))
        rowbad[row] = 1;
    __syncthreads();

    // 4. combine: each thread merges one part of its row's staircase; part 1 hands its keys
    //    over through the (consumed) x tile.  Rows whose boundary stays ambiguous run both
    //    parts again on the half-0 threads with keys centred on the boundary sum (the same
    //    code, in the same loop).
    const int top_s = top + 1;  // staged outputs [ROWS][top + 1]: the pad spreads the banks
    int32_t* st_idx = reinterpret_cast<int32_t*>(sm + PK_OFF_L + C::OFF_STAGE);
    float* st_w = reinterpret_cast<float*>(sm + PK_OFF_L + C::LIST_BYTES + C::OFF_STAGE);
    {
        const float* Av = reinterpret_cast<const float*>(sm + PK_OFF_SK) + row;
        const uint16_t* Ai = reinterpret_cast<const uint16_t*>(sm + PK_OFF_SK + KP * 4 * S) + row;
        const float* Bv = reinterpret_cast<const float*>(sm + PK_OFF_SK + 32768) + row;
        const uint16_t* Bi =
            reinterpret_cast<const uint16_t*>(sm + PK_OFF_SK + 32768 + KP * 4 * S) + row;
        uint32_t rk[2], rab[2];
        const float* Rk[2];
        const uint16_t* Rab[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            unsigned char* base = sm + PK_OFF_L + q * C::LIST_BYTES + C::OFF_REST;
            rk[q] = ptx::smem_u32(base) + (uint32_t)row * 4u;
            rab[q] = ptx::smem_u32(base) + (uint32_t)C::REST * (4u * S) + (uint32_t)row * 2u;
            Rk[q] = reinterpret_cast<const float*>(base) + row;
            Rab[q] = reinterpret_cast<const uint16_t*>(base + C::REST * 4 * S) + row;
        }
        const bool live = !aborted && row_ok && rowbad[row] == 0;
        const float M0 = Av[0] + Bv[0];
        float R[KP];
#pragma unroll
        for (int e = 0; e < KP; ++e) R[e] = -INFINITY;
        float dropped = -INFINITY;
        float* X = reinterpret_cast<float*>(sm + PK_OFF_X) + row;          // [KP + 1], then sums
        int* XS = reinterpret_cast<int*>(sm + PK_OFF_X + KP * 4 * S) + row;  // slots
        bool amb = false;
        float off2 = M0;
        int it_end = 1;
#pragma unroll 1
        for (int it = 0; it < it_end; ++it) {
            const int part = it == 0 ? g : it - 1;
            if (!aborted)
                pk_combine_part<KP, ROWS>(part, Av, Bv, K, top, it == 0 ? M0 : off2,
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
                    amb = live && pk_hi<C::CB>(pk_pick<KP>(R, top - 1)) == pk_hi<C::CB>(dropped);
                    if (__any_sync(FULL, amb)) {
                        int ka, kb;
                        pk_decode<KP, ROWS>(pk_pick<KP>(R, top - 1), K, Rab[0], Rab[1], ka, kb);
                        off2 = Av[ka * S] + Bv[kb * S];
                        // the first pass's keys wait in the exchange area
#pragma unroll
                        for (int e = 0; e < KP; ++e) {
                            X[e * S] = R[e];
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
                const bool amb2 =
                    amb && pk_hi<C::CB>(pk_pick<KP>(R, top - 1)) == pk_hi<C::CB>(dropped);
#pragma unroll
                for (int e = 0; e < KP; ++e) R[e] = amb ? R[e] : X[e * S];
                if (amb2) {
#pragma unroll
                    for (int e = 0; e < KP; ++e)
                        if (e < top) X[e * S] = R[e];
                    if (!pk_tie_combine<KP, ROWS>(off2, Av, Ai, Bv, Bi, Rab[0], Rab[1], K, top, n,
                                                  X, XS))
                        rowbad[row] = 1;
                }
                amb = amb2;
            }
            // the keys, in order, become (sum, slot) (rows settled by ties already are); then
            // exact order among equal keys
            bool near = amb;
            if (!amb) {
#pragma unroll
                for (int e = 0; e < KP; ++e)
                    if (e < top) X[e * S] = R[e];
            }
#pragma unroll 4
            for (int q = 0; q < top; ++q) {
                const float key = X[q * S];
                const float nkey = q + 1 < top ? X[(q + 1) * S] : 0.f;
                int a, bb;
                pk_decode<KP, ROWS>(key, K, Rab[0], Rab[1], a, bb);
                const float sv = Av[a * S] + Bv[bb * S];
                const int sl = (int)Ai[a * S] * n + (int)Bi[bb * S];
                if (!amb) {
                    near = near || (q + 1 < top && pk_hi<C::CB>(key) == pk_hi<C::CB>(nkey));
                    X[q * S] = sv;
                    XS[q * S] = sl;
                }
            }
            const bool act = live && rowbad[row] == 0;
            if (__any_sync(FULL, act && near)) pk_fixup<KP, S, int>(X, XS, top, act);
            if (act) {
                const float mx = X[0];
                float zs = 0.f;
#pragma unroll 4
                for (int q = 0; q < top; ++q) {
                    const float ev = __expf(X[q * S] - mx);
                    X[q * S] = ev;
                    zs += ev;
                }
                const float rz = 1.f / zs;
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
        for (int r = warp; r < ROWS; r += NW) {
            const int rb = b0 + r / p.bt, rt = t0 + r % p.bt;
            if (r / p.bt >= p.bb || rb >= p.B || rt >= p.T || rowbad[r]) continue;
            const size_t ro = (((size_t)rb * p.H + h) * p.T + rt) * top;
            for (int q = lane; q < top; q += 32) {
                p.idx[role][ro + q] = st_idx[r * top_s + q];
                p.w[role][ro + q] = st_w[r * top_s + q];
            }
        }
    }
    __syncthreads();

    // rows the threshold search could not settle: exact re-scoring, one warp per row
    const int nf = *nflag;
    if (nf > 0 && !aborted) {
        float* ws = reinterpret_cast<float*>(sm + PK_OFF_L) +
                    (size_t)warp * score_simt_warp_floats(p.d_k, n, K, top);
        for (int f = warp; f < nf; f += NW) {
            const int r = flagged[f];
            const int fb = b0 + r / p.bt, ft = t0 + r % p.bt;
            const size_t row_off = ((size_t)fb * p.H + h) * p.T + ft;
            simt_score_row<__nv_bfloat16>(p.x[role] + row_off * p.d_k,
                                          p.sk[role] + (size_t)h * 2 * n * (p.d_k / 2), p.d_k, n,
                                          K, top, ws, p.idx[role] + row_off * top,
                                          p.w[role] + row_off * top);
        }
    }
    // a sub-key prefetch still in flight completes before the CTA's shared memory goes
    if (tid == 0 && NR > 1 && !aborted) {
        if (!ptx::mbar_wait_bounded(bar_tma, ph_tma, deadline)) *abort_flag = 1;
    }
    __syncthreads();
    if (*abort_flag && tid == 0) raise_err(SDM_DEVERR_TIMEOUT);
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
    (void)FULL;
}

// Threshold position z for a half of n scores of which K are kept: about K + margin of n
// Gaussian draws reach mean + z*sd (margin: 2.5 standard deviations of that count + 2 for one
// round of sub-keys, 3 + 4 when rounds are recomputed for a second pass); -inf when that
// covers every score.
inline float pk_z0(int n, int K) {
    const double kk = (double)K;
    const double sdc = sqrt(kk * (1.0 - kk / n));
    const double m = n <= 256 ? ceil(2.5 * sdc) + 2.0 : ceil(3.0 * sdc) + 4.0;
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
