// Product-key scoring on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), bf16 inputs.
//
// One CTA scores a tile of 128 rows (tokens of one head, one role) against that role's two
// sub-key tables (§2 Background "Product Key Memory", §3 Method "Sparse addressing"):
//   - TMA loads the x tile (both halves, 128-byte swizzle) and, per round, up to 256 sub-keys
//     of one half; one thread issues 4 tcgen05.mma (K = 64 = 4 x 16) into 256 TMEM columns:
//     D[row][j] = <x_half[row], C[j]> in fp32.
//   - Thread r owns row r (TMEM lane r).  It keeps the k best sub-keys of each half exactly:
//     min/max pass, a 64-bin histogram (shared-memory atomics) to find the threshold bin,
//     compaction of the bins
//     above it plus the best of the threshold bin (refined with finer bins when crowded),
//     then a register bitonic sort (best first; equal scores to the lower sub-index).
//     Halves with more than 256 sub-keys merge the per-round lists.
//   - The k x k combine ranks the pairs (a, b) of the two sorted lists with
//     (a+1)(b+1) <= k (any other pair is beaten by >= k >= top pairs) with the same exact
//     selection, ids = slots s = i*n + j (equal sums: lower slot), giving the top-W (or
//     top-R) slots best first, then the softmax of the selected scores (§4 "SDM Configuration").
#pragma once

#include <math.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace sdm {

constexpr int TC_THREADS = 128;
constexpr int TC_NB = 256;      // sub-keys per round = TMEM columns
constexpr int TC_NBIN = 64;     // histogram bins
constexpr int TC_BC = 10;       // boundary candidates ranked exactly
constexpr int TC_MAXLEV = 4;    // histogram refinement levels
constexpr int TC_KMAX = 32;     // largest k_half / top this kernel takes

// Shared-memory map (bytes from a 1024-aligned base).
constexpr uint32_t TC_OFF_A = 0;         // x tile: half 0 [0,16K), half 1 [16K,32K); later list
                                         // R1 [0, K*768) and the combine's handles [24K, 32K)
constexpr uint32_t TC_OFF_B = 32768;     // sub-key round tile, then: [0,16K) round-merge list or
                                         // combine scores, [16K, 23.5K) boundary list
constexpr uint32_t TC_OFF_BND = TC_OFF_B + 16384;
constexpr uint32_t TC_OFF_HIST = 65536;  // packed u16 histogram [32 words][128]
constexpr uint32_t TC_OFF_R0 = 81920;    // list R0: f32 [K][128] + u16 [K][128]
constexpr uint32_t TC_OFF_CTRL = 81920 + 24576;
constexpr uint32_t TC_SMEM_BYTES = TC_OFF_CTRL + 64 + 1024;  // + alignment slack

struct ScoreTcArgs {
    int B, H, T, n, k_half, top;
    int nbox;          // sub-key rows per TMA box = min(n, 256)
    int bt, bb, n_tt;  // a tile holds bt tokens of bb sequences; t-tiles per sequence block
    int32_t* idx;
    float* w;
};

// Bin position (v - lo) * sc, rounded the same way wherever it is used.
SDM_DEV float tc_pos(float v, float lo, float sc) { return __fmul_rn(__fsub_rn(v, lo), sc); }

SDM_DEV int tc_bin(float v, float lo, float sc) {
    int b = __float2int_rd(tc_pos(v, lo, sc));
    return min(max(b, 0), TC_NBIN - 1);
}

// Level-0 bin: -1 (not counted) below lo.
SDM_DEV int tc_bin0(float v, float lo, float sc) {
    return v >= lo ? min(__float2int_rd(tc_pos(v, lo, sc)), TC_NBIN - 1) : -1;
}

// Smallest v with tc_pos(v, lo, sc) >= t, i.e. with bin >= t for 1 <= t < TC_NBIN (the
// position is monotone in v): the quotient, then a walk of a few ulps.
SDM_DEV float tc_edge(int t, float lo, float sc) {
    const float ft = (float)t;
    float v = lo + __fdividef(ft, sc);
    for (int it = 0; it < 64 && tc_pos(v, lo, sc) >= ft; ++it) v = nextafterf(v, -INFINITY);
    for (int it = 0; it < 64 && tc_pos(v, lo, sc) < ft; ++it) v = nextafterf(v, INFINITY);
    return v;
}

template <int KP>
SDM_DEV void bitonic_sort_desc(float (&v)[KP], int (&ix)[KP]) {
#pragma unroll
    for (int k = 2; k <= KP; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
            for (int i = 0; i < KP; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const bool desc = (i & k) == 0;
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

// Same order, cheaper: the network compares values alone (ids follow them); equal values,
// rare, are then put in id order by the full comparison.
template <int KP>
SDM_DEV void sort_desc(float (&v)[KP], int (&ix)[KP]) {
#pragma unroll
    for (int k = 2; k <= KP; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
            for (int i = 0; i < KP; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const bool sw = (i & k) == 0 ? v[l] > v[i] : v[i] > v[l];
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
    bool tie = false;
#pragma unroll
    for (int e = 0; e + 1 < KP; ++e) tie = tie || (v[e] == v[e + 1] && v[e] > -INFINITY);
    if (__any_sync(0xffffffffu, tie)) bitonic_sort_desc<KP>(v, ix);
}

// Merge a sorted (best-first) list held in r[] with sorted a[]: r <- best KP of both, sorted.
template <int KP>
SDM_DEV void bitonic_merge_keep(float (&r)[KP], int (&ri)[KP], const float (&a)[KP],
                                const int (&ai)[KP]) {
#pragma unroll
    for (int i = 0; i < KP; ++i) {
        const bool take = better(a[KP - 1 - i], ai[KP - 1 - i], r[i], ri[i]);
        r[i] = take ? a[KP - 1 - i] : r[i];
        ri[i] = take ? ai[KP - 1 - i] : ri[i];
    }
#pragma unroll
    for (int j = KP >> 1; j > 0; j >>= 1) {
#pragma unroll
        for (int i = 0; i < KP; ++i) {
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

// Bin of v in the refinement chain lo/sc/tb[0..L): -1 when v is outside the chain (rare path).
SDM_DEV int tc_chain_bin(float v, const float* lo, const float* sc, const int* tb, int L) {
    if (tc_bin0(v, lo[0], sc[0]) != tb[0]) return -1;
    for (int l = 1; l < L; ++l)
        if (tc_bin(v, lo[l], sc[l]) != tb[l]) return -1;
    return tc_bin(v, lo[L], sc[L]);
}

// Per-thread histogram of 64 bins packed as 16-bit counters in 32 shared words (one column per
// thread).  Updates are shared-memory atomics without a return value, so consecutive scores do
// not wait on each other.
SDM_DEV void hist_clear(uint32_t* h) {
#pragma unroll
    for (int w = 0; w < TC_NBIN / 2; ++w) h[w * TC_THREADS] = 0u;
}
SDM_DEV void hist_add(uint32_t* h, int bn) {
    atomicAdd(h + (bn >> 1) * TC_THREADS, 1u << ((bn & 1) * 16));
}
// The same, performed only when p is set (a predicated reduction, no branch).
SDM_DEV void hist_add_if(bool p, uint32_t h_addr, int bn) {
    const uint32_t addr = h_addr + (uint32_t)((bn >> 1) & (TC_NBIN / 2 - 1)) * (TC_THREADS * 4);
    asm volatile("{\n .reg .pred q;\n setp.ne.b32 q, %0, 0;\n @q red.shared.add.u32 [%1], %2;\n}\n" ::
                     "r"((int)p),
                 "r"(addr), "r"(1u << ((bn & 1) * 16)));
}
// Highest bin t_b whose bins above it hold fewer than `need` (count above -> cum, in it -> cnt).
SDM_DEV void hist_threshold(const uint32_t* h, int need, int& t_b, int& cum, int& cnt) {
    uint32_t w[TC_NBIN / 2];
#pragma unroll
    for (int i = 0; i < TC_NBIN / 2; ++i) w[i] = h[i * TC_THREADS];
    int c = 0, tb = 0, above = 0, in_tb = 0;
    bool found = false;
#pragma unroll
    for (int bn = TC_NBIN - 1; bn >= 0; --bn) {
        const int k = (int)((w[bn >> 1] >> ((bn & 1) * 16)) & 0xffffu);
        const bool hit = !found && c + k >= need;
        tb = hit ? bn : tb;
        above = hit ? c : above;
        in_tb = hit ? k : in_tb;
        found = found || hit;
        c += k;
    }
    t_b = tb;
    cum = above;
    cnt = in_tb;
}

// Shared-memory stores performed only by the lanes whose p is set (predicated, no branch).
SDM_DEV void st_shared_if(bool p, uint32_t addr, float v) {
    asm volatile("{\n .reg .pred q;\n setp.ne.b32 q, %0, 0;\n @q st.shared.f32 [%1], %2;\n}\n" ::"r"(
                     (int)p),
                 "r"(addr), "f"(v)
                 : "memory");
}
SDM_DEV void st_shared_if_u16(bool p, uint32_t addr, int v) {
    asm volatile("{\n .reg .pred q;\n setp.ne.b32 q, %0, 0;\n @q st.shared.u16 [%1], %2;\n}\n" ::"r"(
                     (int)p),
                 "r"(addr), "h"((unsigned short)v)
                 : "memory");
}

struct TcRefine {
    int ns, nbd, need;
    bool small;
};

// Refinement of the threshold bin by finer histograms over its interval, for the lanes that
// are not done; called by whole warps (the loop condition is warp-uniform, and lanes that are
// done still take part in src.load).  Kept out of line: it is rare, and inlined it would cost
// the common path registers.
template <bool GUARD, class Src>
__device__ __noinline__ TcRefine tc_refine(const Src src, int NV, bool done, float lo, float sc,
                                           int t_b, TcRefine io, uint32_t* hist, float* Sv,
                                           uint16_t* Sh, float* Bv, uint16_t* Bh) {
    constexpr int S = TC_THREADS;
    constexpr unsigned FULL = 0xffffffffu;
    int ns = io.ns, nbd = io.nbd, need = io.need;
    bool small = io.small;
    float lv[TC_MAXLEV], sv[TC_MAXLEV];
    int tb[TC_MAXLEV];
    lv[0] = lo;
    sv[0] = sc;
    tb[0] = t_b;
    int L = 0;
    while (__any_sync(FULL, !done)) {
        const bool act = !done;
        if (act) {
            lv[L + 1] = lv[L] + (float)tb[L] / sv[L];
            sv[L + 1] = fminf(sv[L] * (float)TC_NBIN, 1e38f);
            ++L;
        }
        // the deepest level takes the chain members in item order
        const bool last = act && L == TC_MAXLEV - 1;
        const bool refine = act && !last;
        int cum2 = 0, t2 = 0, cnt2 = 0;
        if (refine) hist_clear(hist);
        for (int c = 0; c < NV; c += 32) {
            float v[32];
            int hd[32];
            src.load(c, v, hd);
            if (refine) {
#pragma unroll 1
                for (int i = 0; i < 32; ++i) {
                    if (GUARD && c + i >= NV) break;
                    const int bn = tc_chain_bin(v[i], lv, sv, tb, L);
                    if (bn >= 0) hist_add(hist, bn);
                }
            }
        }
        if (refine) {
            hist_threshold(hist, need, t2, cum2, cnt2);
            tb[L] = t2;
        }
        const bool small2 = refine && cnt2 <= TC_BC;
        if (small2) nbd = 0;
        int take_direct = last ? need : 0;
        for (int c = 0; c < NV; c += 32) {
            float v[32];
            int hd[32];
            src.load(c, v, hd);
            if (act) {
#pragma unroll 1
                for (int i = 0; i < 32; ++i) {
                    if (GUARD && c + i >= NV) break;
                    const int bn = tc_chain_bin(v[i], lv, sv, tb, L);
                    if (bn < 0) continue;
                    if (last) {
                        if (take_direct > 0) {
                            Sv[ns * S] = v[i];
                            Sh[ns * S] = (uint16_t)hd[i];
                            ++ns;
                            --take_direct;
                        }
                    } else if (bn > t2) {
                        Sv[ns * S] = v[i];
                        Sh[ns * S] = (uint16_t)hd[i];
                        ++ns;
                    } else if (small2 && bn == t2) {
                        Bv[nbd * S] = v[i];
                        Bh[nbd * S] = (uint16_t)hd[i];
                        ++nbd;
                    }
                }
            }
        }
        if (last) {
            done = true;
        } else if (refine) {
            need -= cum2;
            if (small2) {
                done = true;
                small = true;  // pick the remaining `need` from this level's boundary list
            }
        }
    }
    return TcRefine{ns, nbd, need, small};
}

// Rows whose items at or above lo all equal the maximum: the K best are the first K items (in
// id order) equal to it.  Called by whole warps; only the lanes with `flat` set take items.
template <bool GUARD, class Src>
__device__ __noinline__ int tc_flat(const Src src, int NV, bool flat, float mx, int K,
                                    float* Sv, uint16_t* Sh) {
    constexpr int S = TC_THREADS;
    int ns = 0;
    for (int c = 0; c < NV; c += 32) {
        float v[32];
        int hd[32];
        src.load(c, v, hd);
        if (flat) {
#pragma unroll 1
            for (int i = 0; i < 32; ++i) {
                if ((GUARD && c + i >= NV) || ns >= K) break;
                if (v[i] == mx) {
                    Sv[ns * S] = v[i];
                    Sh[ns * S] = (uint16_t)hd[i];
                    ++ns;
                }
            }
        }
    }
    return ns;
}

// Exact top-K (value desc, id asc) of the items of src.  src.for_each(f) calls
// f(value, handle, valid) for every item, in any order (for the TMEM source it is
// warp-collective: whole warps call it); src.id_of(handle) gives an item's id;
// src.bounds(lo, mx, fl) gives the maximum mx, a bound lo with at least K valid items at or
// above it (so the K-th best is >= lo) and a bound fl no valid item lies below;
// src.chunked() gives the same items 32 at a time, in id order among equal values, for the
// rare paths.  K <= 32.
// The K winners are left unsorted in Sv/Sh (strided by TC_THREADS), then returned sorted in
// a[0..K) (padding beyond).
//
// A 64-bin histogram over [lo, mx] finds the bin holding the K-th best.  Items in higher bins
// are taken; the threshold bin is ranked exactly when it holds <= TC_BC items, else refined
// with finer bins.
template <int KP, class Src>
SDM_DEV void tc_select(const Src& src, int K, uint32_t* hist, float* Sv, uint16_t* Sh,
                       float* Bv, uint16_t* Bh, float (&a)[KP], int (&ai)[KP]) {
    constexpr int S = TC_THREADS;
    constexpr unsigned FULL = 0xffffffffu;
    float lo, mx, fl;
    src.bounds(lo, mx, fl);
    // all the items at or above lo equal the maximum: the K best are the first K of them
    const bool flat = !(mx > lo);
    float sc = flat ? 0.f : fminf((float)TC_NBIN / (mx - lo), 1e38f);

    // ---- level 0 histogram ----
    int t_b = 0, cum = 0, cnt_tb = 0;
    if constexpr (Src::kClampBelow) {
        // Every item counted, those below lo in bin 0 (measured faster for dense TMEM rows).
        // A lane whose threshold lands in bin 0 takes the histogram again over [fl, mx], so
        // that bins >= the threshold bin hold no item below lo.
        bool redo = false;
        for (int attempt = 0; attempt < 2; ++attempt) {
            if (attempt == 1 && !__any_sync(FULL, redo)) break;
            const bool act = !flat && (attempt == 0 || redo);
            if (act) hist_clear(hist);
            src.for_each([&](float v, int, bool valid) {
                if (act && valid) hist_add(hist, tc_bin(v, lo, sc));
            });
            if (act) {
                hist_threshold(hist, K, t_b, cum, cnt_tb);
                redo = attempt == 0 && t_b == 0 && lo > fl;
                if (redo) {
                    lo = fl;
                    sc = fminf((float)TC_NBIN / (mx - fl), 1e38f);
                }
            }
        }
    } else {
        // only the items at or above lo counted
        if (!flat) hist_clear(hist);
        const uint32_t h0 = ptx::smem_u32(hist);
        src.for_each([&](float v, int, bool valid) {
            const int bn = tc_bin0(v, lo, sc);
            hist_add_if(!flat && valid && bn >= 0, h0, bn);
        });
        asm volatile("" ::: "memory");  // the predicated shared-memory writes precede the scan
        if (!flat) hist_threshold(hist, K, t_b, cum, cnt_tb);
    }

    // ---- compaction: bins above the threshold bin (flat rows: the first K maxima), and the
    //      threshold bin itself when it is small ----
    bool small = !flat && cnt_tb <= TC_BC;
    int ns = 0, nbd = 0;
    const uint32_t sv0 = ptx::smem_u32(Sv), sh0 = ptx::smem_u32(Sh);
    const uint32_t bv0 = ptx::smem_u32(Bv), bh0 = ptx::smem_u32(Bh);
    // bins above t_b are the values >= tau_take, bin t_b the values in [tau_bnd, tau_take)
    // (items below lo, counted in bin 0 by the clamped histogram, are in bin t_b only when
    // t_b = 0, and then no item lies below lo)
    const float tau_take = flat ? INFINITY : (t_b >= TC_NBIN - 1 ? INFINITY : tc_edge(t_b + 1, lo, sc));
    const float tau_bnd = !small ? INFINITY : (t_b == 0 ? lo : tc_edge(t_b, lo, sc));
    src.for_each([&](float v, int hd, bool valid) {
        const bool take = valid && v >= tau_take;
        const uint32_t so = (uint32_t)min(ns, K - 1);  // ns < K by the histogram count
        st_shared_if(take, sv0 + so * (S * 4), v);
        st_shared_if_u16(take, sh0 + so * (S * 2), hd);
        ns += take ? 1 : 0;
        const bool bnd = valid && !take && v >= tau_bnd;
        const uint32_t bo = (uint32_t)min(nbd, TC_BC - 1);  // nbd <= TC_BC when small
        st_shared_if(bnd, bv0 + bo * (S * 4), v);
        st_shared_if_u16(bnd, bh0 + bo * (S * 2), hd);
        nbd += bnd ? 1 : 0;
    });
    asm volatile("" ::: "memory");
    int need = flat ? 0 : K - cum;
    const bool done = flat || small;
    if (__any_sync(FULL, flat)) {
        const auto ch = src.chunked();
        const int nf = tc_flat<decltype(ch)::kGuard>(ch, ch.NV, flat, mx, K, Sv, Sh);
        if (flat) ns = nf;
    }

    // ---- rare: refinement levels inside a crowded threshold bin (out of line) ----
    if (__any_sync(FULL, !done)) {
        const auto ch = src.chunked();
        const TcRefine r = tc_refine<decltype(ch)::kGuard>(ch, ch.NV, done, lo, sc, t_b,
                                                           {ns, nbd, need, small}, hist, Sv, Sh,
                                                           Bv, Bh);
        ns = r.ns;
        nbd = r.nbd;
        need = r.need;
        small = r.small;
    }
    // the `need` best of the boundary bin (nbd <= TC_BC entries), by exact rank: the entry of
    // rank q goes to slot ns + q
    if (small) {
        float bv[TC_BC];
        int bi[TC_BC], bh[TC_BC];
#pragma unroll
        for (int e = 0; e < TC_BC; ++e) {
            const bool ok = e < nbd;
            bh[e] = ok ? (int)Bh[e * S] : 0;
            bv[e] = ok ? Bv[e * S] : -INFINITY;
            bi[e] = ok ? src.id_of(bh[e]) : 0x7fffffff;
        }
#pragma unroll
        for (int e = 0; e < TC_BC; ++e) {
            int rank = 0;
#pragma unroll
            for (int f = 0; f < TC_BC; ++f) rank += better(bv[f], bi[f], bv[e], bi[e]) ? 1 : 0;
            if (e < nbd && rank < need && ns + rank < K) {
                Sv[(ns + rank) * S] = bv[e];
                Sh[(ns + rank) * S] = (uint16_t)bh[e];
            }
        }
        ns += need;
    }
#pragma unroll
    for (int e = 0; e < KP; ++e) {
        const bool ok = e < ns && e < K;
        a[e] = ok ? Sv[e * S] : -INFINITY;
        ai[e] = ok ? src.id_of(Sh[e * S]) : 0x7fffffff;
    }
    sort_desc<KP>(a, ai);
}

// Scores of this thread's row from TMEM, 32 columns at a time (warp-collective loads);
// handles are the columns inside the round.
struct TmemSource {
    static constexpr bool kGuard = false;  // NV is a multiple of 32
    static constexpr bool kClampBelow = true;
    uint32_t trow;
    int col_base, NV;
    SDM_DEV void load(int c, float (&v)[32], int (&hd)[32]) const {
        ptx::tmem_ld32(trow + c, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) hd[i] = c + i;
    }
    template <class F>
    SDM_DEV void for_each(F&& f) const {
        for (int c = 0; c < NV; c += 32) {
            float v[32];
            ptx::tmem_ld32(trow + c, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) f(v[i], c + i, true);
        }
    }
    SDM_DEV TmemSource chunked() const { return *this; }
    SDM_DEV int id_of(int hd) const { return col_base + hd; }
    // lo = the smallest of the maxima of the 32 groups {c + i} (each group is non-empty, so
    // at least 32 items are >= lo); fl = the minimum.
    SDM_DEV void bounds(float& lo, float& mx, float& fl) const {
        float gmax[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) gmax[i] = -INFINITY;
        float mn = INFINITY;
        for (int c = 0; c < NV; c += 32) {
            float v[32];
            ptx::tmem_ld32(trow + c, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                gmax[i] = fmaxf(gmax[i], v[i]);
                mn = fminf(mn, v[i]);
            }
        }
        lo = INFINITY;
        mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            lo = fminf(lo, gmax[i]);
            mx = fmaxf(mx, gmax[i]);
        }
        fl = mn;
    }
};

// For each top <= TC_KMAX: the pairs (a, b) of positions in the two sorted half lists with
// (a+1)(b+1) <= top, in (a, b) order.  Only these can reach the top `top` of the k x k sums:
// any other pair is beaten by the (a+1)(b+1) - 1 >= top pairs (a' <= a, b' <= b), whose sums
// are no smaller and whose slots are no larger on equal sums.  When all their sums are equal,
// (a, b) order is slot order (equal half scores are listed lower sub-index first).
constexpr int TC_PAIR_TOTAL = 1724;  // sum over top = 1..32 of sum_a floor(top / a)
struct PairTab {
    uint16_t ab[TC_PAIR_TOTAL];  // (a << 8) | b
    int off[TC_KMAX + 1], cnt[TC_KMAX + 1];
};
constexpr PairTab make_pair_tab() {
    PairTab t{};
    int e = 0;
    for (int top = 1; top <= TC_KMAX; ++top) {
        t.off[top] = e;
        for (int a = 0; a < top; ++a)
            for (int b = 0; (a + 1) * (b + 1) <= top; ++b) t.ab[e++] = (uint16_t)((a << 8) | b);
        t.cnt[top] = e - t.off[top];
    }
    return t;
}
static_assert(make_pair_tab().off[TC_KMAX] + make_pair_tab().cnt[TC_KMAX] == TC_PAIR_TOTAL,
              "pair table size");
__constant__ PairTab c_pair_tab = make_pair_tab();

// Candidate pairs of the two sorted half lists (per-thread, strided by TC_THREADS in shared
// memory); handles are (a << 8) | b.
struct PairSource {
    static constexpr bool kGuard = true;
    const float* R0v;
    const uint16_t* R0i;
    const float* R1v;
    const uint16_t* R1i;
    int tab0, NV, top, n;  // this top's pairs: c_pair_tab.ab[tab0 .. tab0 + NV)
    SDM_DEV void load(int c, float (&v)[32], int (&hd)[32]) const {
        constexpr int S = TC_THREADS;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int e = c + i;  // warp-uniform: constant-cache broadcast
            const int ab = e < NV ? (int)c_pair_tab.ab[tab0 + e] : 0;
            v[i] = e < NV ? R0v[(ab >> 8) * S] + R1v[(ab & 0xff) * S] : -INFINITY;
            hd[i] = ab;
        }
    }
    SDM_DEV int id_of(int hd) const {
        return (int)R0i[(hd >> 8) * TC_THREADS] * n + (int)R1i[(hd & 0xff) * TC_THREADS];
    }
    // The pairs (0, b) and (a, 0), b, a < top, are candidates: lo = the larger of their
    // smallest sums.
    SDM_DEV void bounds(float& lo, float& mx, float& fl) const {
        const int q = (top - 1) * TC_THREADS;
        const float a0 = R0v[0], b0 = R1v[0], aq = R0v[q], bq = R1v[q];
        lo = fmaxf(a0 + bq, aq + b0);
        mx = a0 + b0;
        fl = aq + bq;
    }
};

// The same candidates enumerated as segments: for x = 0, 1, ... with (x+1)^2 <= top, the
// row (x, b), x <= b < top/(x+1), and the column (a, x), x < a < top/(x+1).  Each segment is a
// fixed entry of one list plus a run of the other, read 8 at a time.
struct PairSegSource {
    PairSource sm;
    template <class F>
    SDM_DEV void for_each(F&& f) const {
        constexpr int S = TC_THREADS;
        const int top = sm.top;
        int r = 0;
        while ((r + 1) * (r + 1) <= top) ++r;
        for (int sg = 0; sg < 2 * r; ++sg) {
            const bool col = sg >= r;
            const int x = col ? sg - r : sg;
            const float fx = (col ? sm.R1v : sm.R0v)[x * S];
            const float* run = col ? sm.R0v : sm.R1v;
            const int beg = col ? x + 1 : x, end = top / (x + 1);
            for (int j0 = beg; j0 < end; j0 += 8) {
                // all 8 loads before f (whose shared-memory atomics would delay later loads)
                float v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = fx + run[(j0 + j < end ? j0 + j : x) * S];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int y = j0 + j;
                    f(v[j], col ? (y << 8) | x : (x << 8) | y, y < end);
                }
            }
        }
    }
    SDM_DEV int id_of(int hd) const { return sm.id_of(hd); }
    static constexpr bool kClampBelow = false;
    SDM_DEV void bounds(float& lo, float& mx, float& fl) const { sm.bounds(lo, mx, fl); }
    SDM_DEV PairSource chunked() const { return sm; }
};

template <int KP>
__global__ void __launch_bounds__(TC_THREADS, 2) score_tc_kernel(
    const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap skmap,
    ScoreTcArgs p) {
    constexpr int S = TC_THREADS;
    extern __shared__ unsigned char tc_smem_raw[];
    unsigned char* sm = tc_smem_raw + ((1024 - (ptx::smem_u32(tc_smem_raw) & 1023)) & 1023);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int h = blockIdx.y;
    const int bti = blockIdx.x / p.n_tt, tti = blockIdx.x % p.n_tt;
    const int b0 = bti * p.bb, t0 = tti * p.bt;
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + TC_OFF_CTRL);
    uint64_t* bar_mma = bar_tma + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_tma + 2);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

    if (warp == 0) ptx::tmem_alloc(tmem_slot, TC_NB);
    if (tid == 0) {
        ptx::mbar_init(bar_tma, 1);
        ptx::mbar_init(bar_mma, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t deadline = ptx::globaltimer_ns() + 2000000000ull;
    uint32_t ph_tma = 0, ph_mma = 0;

    const int bi = tid / p.bt, ti = tid % p.bt;
    const int b = b0 + bi, t = t0 + ti;
    const bool row_ok = bi < p.bb && b < p.B && t < p.T;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    const int K = p.k_half, n = p.n;
    const int rounds = (n + TC_NB - 1) / TC_NB;
    const uint32_t abox = 64u * 2u * (uint32_t)(p.bt * p.bb);

    uint32_t* hist = reinterpret_cast<uint32_t*>(sm + TC_OFF_HIST) + tid;
    float* Bv = reinterpret_cast<float*>(sm + TC_OFF_BND) + tid;                     // [TC_BC]
    uint16_t* Bh = reinterpret_cast<uint16_t*>(sm + TC_OFF_BND + TC_BC * S * 4) + tid;  // [TC_BC]
    float* R0v = reinterpret_cast<float*>(sm + TC_OFF_R0) + tid;
    uint16_t* R0i = reinterpret_cast<uint16_t*>(sm + TC_OFF_R0 + K * S * 4) + tid;
    float* R1v = reinterpret_cast<float*>(sm + TC_OFF_A) + tid;
    uint16_t* R1i = reinterpret_cast<uint16_t*>(sm + TC_OFF_A + K * S * 4) + tid;
    // round-merge scratch list (multi-round halves, K * 768 <= 16K bytes)
    float* Nv = reinterpret_cast<float*>(sm + TC_OFF_B) + tid;
    uint16_t* Ni = reinterpret_cast<uint16_t*>(sm + TC_OFF_B + K * S * 4) + tid;

    bool aborted = false;
    for (int hf = 0; hf < 2 && !aborted; ++hf) {
        float* Rv = hf ? R1v : R0v;
        uint16_t* Ri = hf ? R1i : R0i;
        for (int r = 0; r < rounds; ++r) {
            const int nb = min(TC_NB, n - r * TC_NB);
            if (tid == 0) {
                // generic-proxy writes to the tile area (scratch, lists) precede this load
                ptx::fence_proxy_async_smem();
                const bool first = hf == 0 && r == 0;
                ptx::mbar_arrive_expect_tx(bar_tma, (first ? 2u * abox : 0u) + 64u * 2u * (uint32_t)p.nbox);
                if (first) {
                    ptx::tma_load_4d(sm + TC_OFF_A, &xmap, 0, t0, h, b0, bar_tma);
                    ptx::tma_load_4d(sm + TC_OFF_A + 16384, &xmap, 64, t0, h, b0, bar_tma);
                }
                ptx::tma_load_2d(sm + TC_OFF_B, &skmap, 0, (h * 2 + hf) * n + r * TC_NB, bar_tma);
                if (ptx::mbar_wait_bounded(bar_tma, ph_tma, deadline)) {
                    ptx::tc_fence_after();
                    const uint64_t ad = ptx::umma_desc_kmajor_sw128(sm + TC_OFF_A + hf * 16384);
                    const uint64_t bd = ptx::umma_desc_kmajor_sw128(sm + TC_OFF_B);
                    const uint32_t id = ptx::idesc_bf16_f32(128, nb);
#pragma unroll
                    for (int k = 0; k < 4; ++k)  // K = 64 in steps of 16 (32 bytes)
                        ptx::umma_bf16(tmem, ad + 2 * k, bd + 2 * k, id, k > 0 ? 1u : 0u);
                    ptx::umma_commit(bar_mma);
                } else {
                    *abort_flag = 1;
                }
            }
            ph_tma ^= 1;
            if (!ptx::mbar_wait_bounded(bar_mma, ph_mma, deadline)) *abort_flag = 1;
            ph_mma ^= 1;
            ptx::tc_fence_after();
            __syncthreads();
            if (*abort_flag) {
                aborted = true;
                break;
            }
            float a[KP];
            int ai[KP];
            TmemSource src{trow, r * TC_NB, nb};
            // round 0 selects straight into the half's list; later rounds into scratch
            float* Sv = r == 0 ? Rv : Nv;
            uint16_t* Si = r == 0 ? Ri : Ni;
            tc_select<KP>(src, K, hist, Sv, Si, Bv, Bh, a, ai);
            if (r > 0) {
                float rv[KP];
                int ri[KP];
#pragma unroll
                for (int e = 0; e < KP; ++e) {
                    rv[e] = e < K ? Rv[e * S] : -INFINITY;
                    ri[e] = e < K ? (int)Ri[e * S] : 0x7fffffff;
                }
                bitonic_merge_keep<KP>(rv, ri, a, ai);
#pragma unroll
                for (int e = 0; e < KP; ++e) {
                    a[e] = rv[e];
                    ai[e] = ri[e];
                }
            }
#pragma unroll
            for (int e = 0; e < KP; ++e)
                if (e < K) {
                    Rv[e * S] = a[e];
                    Ri[e * S] = (uint16_t)ai[e];
                }
            ptx::fence_proxy_async_smem();  // these generic writes precede the next TMA write
            ptx::tc_fence_before();
            __syncthreads();
        }
    }

    if (!aborted) {
        // k x k combine: exact top-`top` of the candidate pairs, ids = slots (ties: lower slot)
        const int W = p.top;
        const PairSegSource src{
            PairSource{R0v, R0i, R1v, R1i, c_pair_tab.off[W], c_pair_tab.cnt[W], W, n}};
        float* Ov = reinterpret_cast<float*>(sm + TC_OFF_B) + tid;                 // [W]
        uint16_t* Oh = reinterpret_cast<uint16_t*>(sm + TC_OFF_A + 24576) + tid;   // [W]
        float a[KP];
        int ai[KP];
        tc_select<KP>(src, W, hist, Ov, Oh, Bv, Bh, a, ai);
        if (row_ok) {
            const size_t row_off = ((size_t)b * p.H + h) * p.T + t;
            const float mx = a[0];
            float z = 0.f;
#pragma unroll
            for (int q = 0; q < KP; ++q)
                if (q < W) z += expf(a[q] - mx);
#pragma unroll
            for (int q = 0; q < KP; ++q)
                if (q < W) {
                    p.idx[row_off * W + q] = ai[q];
                    p.w[row_off * W + q] = expf(a[q] - mx) / z;
                }
        }
    } else if (tid == 0) {
        raise_err(SDM_DEVERR_TIMEOUT);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, TC_NB);
    }
}

}  // namespace sdm
