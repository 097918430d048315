// Product-key scoring with the latency of one row in mind: a decode step scores a single token
// per (b,h), so a row cannot wait behind others in a thread's queue.  Each CTA takes
// SROW_G rows of one head (and one role: blockIdx.z picks write or read, so a decode step
// scores both roles in one launch).
//
// Same definition as the other scoring paths (§2 Background "Product Key Memory", §3 Method
// "Sparse addressing", §4 "SDM Configuration"):
//   s1[i] = <x[0:h], C1[i]>,  s2[j] = <x[h:2h], C2[j]>     (fp32 FMA, d ascending)
//   the k_half best of each half, best first, ties to the lower sub-index
//   the pairs (a, b) of the two lists with (a+1)(b+1) <= top ranked by s1[a] + s2[b], ties to
//   the lower slot i*n + j; weights = softmax of the `top` selected sums.
// Scores are ranked through an order-preserving u32 key (-0 joins +0, NaN ranks as -inf);
// key 0 marks padding.
//
// Phases, all in one CTA of 8 warps:
//   1. dot products: thread t takes sub-keys of one half for all SROW_G rows, so every
//      sub-key element is loaded and widened once per CTA; the loads of a block of 32 (bf16)
//      or 16 (fp32) elements are issued together (the first block before x is staged).
//   2. per-half top-k: one warp per (row, half).
//      k_half, top <= 32: the n scores form ceil(n/32) columns of 32 lanes.  A threshold
//      that at least 32 scores reach (from each lane's second-largest) prunes them to
//      about 50 candidates, which are compacted into two columns; each column is sorted by
//      a bitonic network across the lanes and the two are merged (elementwise best
//      against the reversed partner, then a bitonic merge) into the top 32 in order.
//      up to 64: lane l sorts the block [l*PL, l*PL+PL) in registers and the warp takes
//      k_half rounds of "best lane head" (redux.sync max, ballot, lowest lane among equal
//      heads, whose block holds the lower sub-indices).
//   3. combine, one warp per row.  <= 32: the staircase candidates (at most 119) form four
//      columns and go through the same pruning, sort and merge.  Up to 64: lane l owns staircase
//      columns b = l, l + 32, whose candidates are already sorted along a, and `top` rounds
//      of best-head selection take them in order (equal sums: redux.sync min over slots).
#pragma once

#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace sdm {

// 4 consecutive fp32 columns of this thread's TMEM lane (tcgen05.ld, 32 lanes x 32 bits, x4).
SDM_DEV void tmem_ld4(uint32_t taddr, float (&v)[4]) {
    uint32_t r0, r1, r2, r3;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    v[0] = __uint_as_float(r0);
    v[1] = __uint_as_float(r1);
    v[2] = __uint_as_float(r2);
    v[3] = __uint_as_float(r3);
}

constexpr int SROW_THREADS = 256;
constexpr int SROW_G = 4;  // rows per CTA: two warps per row in phase 2

constexpr int SROW_CAND = 128;  // staircase candidates when k_half, top <= 32 (at most 119)

struct ScoreRowsArgs {
    const void* x[2];
    const void* sk[2];
    int top[2];
    int32_t* idx[2];
    float* w[2];
    int B, H, T, d_k, n, k_half;
    // per role, when k_half, top <= 32: the pairs (a, b) with (a+1)(b+1) <= top, a, b < k_half,
    // as (a << 8) | b, and their count
    uint16_t cand[2][SROW_CAND];
    int ncand[2];
};

// The staircase pairs of one role (host side; the same for every row).
inline int score_rows_staircase(int k_half, int top, uint16_t* cand) {
    int m = 0;
    for (int a0 = 0; a0 < k_half; ++a0)
        for (int b0 = 0; b0 < k_half && (a0 + 1) * (b0 + 1) <= top; ++b0)
            if (m < SROW_CAND) cand[m++] = (uint16_t)((a0 << 8) | b0);
    return m;
}

// Strictly increasing map of the floats onto u32 with -0 joined to +0 and NaN ranked as -inf,
// so unsigned comparison orders scores; 0 is left free for "no candidate".
SDM_DEV uint32_t order_key(float v) {
    if (v == 0.f) v = 0.f;
    if (v != v) v = -INFINITY;
    const uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

SDM_DEV float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

// Eight consecutive sub-key elements, loaded raw and widened to fp32 at use.
template <typename XT>
struct Chunk8;
template <>
struct Chunk8<__nv_bfloat16> {
    uint4 u;
    SDM_DEV void load(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const uint4*>(p)); }
    SDM_DEV void widen(float* k) const {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            k[2 * i] = __uint_as_float(w[i] << 16);
            k[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};
template <>
struct Chunk8<float> {
    float4 a, b;
    SDM_DEV void load(const float* p) {
        a = __ldg(reinterpret_cast<const float4*>(p));
        b = __ldg(reinterpret_cast<const float4*>(p + 4));
    }
    SDM_DEV void widen(float* k) const {
        k[0] = a.x; k[1] = a.y; k[2] = a.z; k[3] = a.w;
        k[4] = b.x; k[5] = b.y; k[6] = b.z; k[7] = b.w;
    }
};

// (key a, index ia) ranks before (key b, index ib)
SDM_DEV bool kv_better(uint32_t ka, uint32_t ia, uint32_t kb, uint32_t ib) {
    return ka > kb || (ka == kb && ia < ib);
}

// Sorts each of the C columns (one register across the 32 lanes) best first: bitonic network,
// lane pairs at distance j exchange through shuffles; in a pair the lane that keeps the
// better element is the lower one in descending runs and the upper one in ascending runs.
template <int C>
SDM_DEV void column_sort(uint32_t (&k)[C], uint32_t (&id)[C], int lane) {
#pragma unroll
    for (int kk = 2; kk <= 32; kk <<= 1) {
#pragma unroll
        for (int j = kk >> 1; j > 0; j >>= 1) {
            const bool keep_better = ((lane & kk) == 0) == ((lane & j) == 0);
#pragma unroll
            for (int c = 0; c < C; ++c) {
                const uint32_t pk = __shfl_xor_sync(0xffffffffu, k[c], j);
                const uint32_t pi = __shfl_xor_sync(0xffffffffu, id[c], j);
                if (keep_better == kv_better(pk, pi, k[c], id[c])) {
                    k[c] = pk;
                    id[c] = pi;
                }
            }
        }
    }
}

// (ka, ia) <- the best 32 of two columns sorted best first, sorted best first: the
// elementwise better of a and the reversed b is a bitonic sequence holding the best 32,
// which a bitonic merge orders.
SDM_DEV void column_merge(uint32_t& ka, uint32_t& ia, uint32_t kb, uint32_t ib, int lane) {
    const uint32_t rk = __shfl_sync(0xffffffffu, kb, 31 - lane);
    const uint32_t ri = __shfl_sync(0xffffffffu, ib, 31 - lane);
    if (kv_better(rk, ri, ka, ia)) {
        ka = rk;
        ia = ri;
    }
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        const bool keep_better = (lane & j) == 0;
        const uint32_t pk = __shfl_xor_sync(0xffffffffu, ka, j);
        const uint32_t pi = __shfl_xor_sync(0xffffffffu, ia, j);
        if (keep_better == kv_better(pk, pi, ka, ia)) {
            ka = pk;
            ia = pi;
        }
    }
}

// Column 0 <- the best 32 of all C columns (C a power of two), in order.
template <int C>
SDM_DEV void top32_columns(uint32_t (&k)[C], uint32_t (&id)[C], int lane) {
    column_sort<C>(k, id, lane);
#pragma unroll
    for (int st = 1; st < C; st <<= 1)
#pragma unroll
        for (int c = 0; c < C; c += 2 * st) column_merge(k[c], id[c], k[c + st], id[c + st], lane);
}

// (k0, i0) <- the best 32 of the C columns, in order, through a pruned candidate set: tau is
// the 16th largest over the lanes of each lane's second-largest key, so at least 16 lanes
// hold two keys >= tau and at least 32 keys are >= tau -- tau is at most the 32nd key, and
// every element that can rank in the best 32 (ties included) passes.  When at most 64 pass
// (nearly always for continuous scores) they are compacted into `scratch` (64 entries) and
// sorted as two columns; otherwise all C columns are sorted.
template <int C>
SDM_DEV void top32_pruned(uint32_t (&k)[C], uint32_t (&id)[C], int2* scratch, int lane,
                          uint32_t& k0, uint32_t& i0) {
    uint32_t m1 = 0u, m2 = 0u;
#pragma unroll
    for (int c = 0; c < C; ++c) {
        m2 = max(m2, min(m1, k[c]));
        m1 = max(m1, k[c]);
    }
#pragma unroll
    for (int kk = 2; kk <= 32; kk <<= 1) {
#pragma unroll
        for (int j = kk >> 1; j > 0; j >>= 1) {
            const bool keep_larger = ((lane & kk) == 0) == ((lane & j) == 0);
            const uint32_t p = __shfl_xor_sync(0xffffffffu, m2, j);
            m2 = keep_larger ? max(m2, p) : min(m2, p);
        }
    }
    const uint32_t tau = __shfl_sync(0xffffffffu, m2, 15);
    const uint32_t below = (1u << lane) - 1u;
    int m = 0;
#pragma unroll
    for (int c = 0; c < C; ++c) {
        const bool in = k[c] >= tau;
        const uint32_t bal = __ballot_sync(0xffffffffu, in);
        const int pos = m + __popc(bal & below);
        if (in && pos < 64) scratch[pos] = make_int2((int)k[c], (int)id[c]);
        m += __popc(bal);
    }
    if (m <= 64) {
        __syncwarp();
        uint32_t kk2[2], ii2[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int e = c * 32 + lane;
            if (e < m) {
                const int2 v = scratch[e];
                kk2[c] = (uint32_t)v.x;
                ii2[c] = (uint32_t)v.y;
            } else {
                kk2[c] = 0u;
                ii2[c] = 0x7fffff00u + (uint32_t)e;  // padding, distinct from every index
            }
        }
        __syncwarp();  // scratch is free again
        top32_columns<2>(kk2, ii2, lane);
        k0 = kk2[0];
        i0 = ii2[0];
    } else {
        top32_columns<C>(k, id, lane);
        k0 = k[0];
        i0 = id[0];
    }
}

__host__ __device__ inline size_t srow_align16(size_t b) { return (b + 15) & ~(size_t)15; }

// Tensor-core dot products (bf16, d_k = 128): 128-sub-key chunks of the head's table stream
// through two TMA buffers (128-byte swizzle) and the x rows form a 16-row operand, so each
// chunk is one M=128, N=16, K=64 product into 16 TMEM columns (lane = sub-key, column = row).
constexpr uint32_t SROW_TC_KBUF = 16384;                 // one chunk: 128 rows x 128 B
constexpr uint32_t SROW_TC_XT = 2 * SROW_TC_KBUF;        // x: 2 halves x 16 rows x 128 B
constexpr uint32_t SROW_TC_CTRL = SROW_TC_XT + 4096;     // mbarriers, TMEM address, abort
constexpr uint32_t SROW_TC_HEAD = SROW_TC_CTRL + 64;     // the common area starts here

// Bytes of one (row, half) score segment: the scores, then the 64-entry scratch of the
// pruned selection (k_half, top <= 32), or the sorted lane lists (up to 64).
__host__ __device__ inline size_t score_rows_seg_bytes(int PL, int KP) {
    return KP == 32 ? (size_t)32 * PL * 4 + 512 : (size_t)32 * PL * 8;
}

// Shared memory: x rows (CUDA-core dots) or the tensor-core staging (plus 1 KB for its
// alignment), the score segments, the per-half lists, the selected pairs, the staircase
// tables of both roles.
__host__ __device__ inline size_t score_rows_smem_bytes(int d_k, int PL, int KP, bool tcd) {
    const size_t head = tcd ? SROW_TC_HEAD + 1024 : srow_align16((size_t)SROW_G * d_k * 4);
    return head + (size_t)SROW_G * 2 * score_rows_seg_bytes(PL, KP) + (size_t)SROW_G * 2 * KP * 8 +
           (size_t)SROW_G * KP * 8 + 2 * SROW_CAND * 4 + 16;
}

// The common area after the head: score segments, per-half lists, selected pairs, the
// staircase tables.
template <int PL, int KP>
struct SrowSmem {
    static constexpr size_t SEG = KP == 32 ? (size_t)32 * PL * 4 + 512 : (size_t)32 * PL * 8;
    unsigned char* segs;  // [G][2] segments of SEG bytes
    float* tv;            // [G][2][KP] per-half values
    int* ti;              // [G][2][KP] per-half sub-indices
    float* sv;            // [G][KP] selected sums (wide combine)
    uint32_t* ss;         // [G][KP] selected slots (wide combine)
    int* cand;            // [2][SROW_CAND] staircase pairs per role
    int* ncand;           // [2]
    SDM_DEV explicit SrowSmem(unsigned char* p) {
        segs = p;
        tv = reinterpret_cast<float*>(segs + (size_t)SROW_G * 2 * SEG);
        ti = reinterpret_cast<int*>(tv + SROW_G * 2 * KP);
        sv = reinterpret_cast<float*>(ti + SROW_G * 2 * KP);
        ss = reinterpret_cast<uint32_t*>(sv + SROW_G * KP);
        cand = reinterpret_cast<int*>(ss + SROW_G * KP);
        ncand = cand + 2 * SROW_CAND;
    }
    SDM_DEV unsigned char* seg(int g, int hf) const { return segs + (size_t)(g * 2 + hf) * SEG; }
};

// Phase 1 on the tensor cores for the CTA's SROW_G rows: xr[g] is row g's x (d_k = 128 bf16;
// null: a zero row), rtab[g] the sub-key table it is scored against (0: km0, 1: km1).  The
// chunks of the TABLES tables of head h (every table's half 0 then half 1, 128 sub-keys each)
// stream through the two TMA buffers at `base`; each chunk's scores go to the segments of
// the rows that use its table.  All threads of the CTA (SROW_THREADS) take part.  Returns
// false when a bounded wait gave up (the device error word says so).
template <int NP, int TABLES>
SDM_DEV bool srow_tc_dots(unsigned char* base, unsigned char* segs, size_t seg_bytes, const CUtensorMap* km0,
                          const CUtensorMap* km1, const __nv_bfloat16* const (&xr)[SROW_G],
                          const int (&rtab)[SROW_G], int h, int n) {
    constexpr uint32_t NEED = TABLES * 2 * ((NP + 127) / 128) * 16;
    constexpr uint32_t TCOLS = NEED <= 32 ? 32 : (NEED <= 64 ? 64 : (NEED <= 128 ? 128 : 256));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(base + SROW_TC_CTRL);  // [2]
    uint64_t* bar_mma = bar_tma + 2;                                       // [2]
    uint64_t* bar_done = bar_mma + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_done + 1);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
    const int cph = (n + 127) / 128, cpt = 2 * cph, nch = TABLES * cpt;  // chunks per half, table, all
    auto chunk_map = [&](int c) { return (TABLES == 2 && c >= cpt) ? km1 : km0; };
    auto chunk_row = [&](int c) {
        const int cc = c % cpt;
        return (h * 2 + cc / cph) * n + (cc % cph) * 128;
    };
    if (warp == 0) ptx::tmem_alloc(tmem_slot, TCOLS);
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(bar_tma + i, 1);
            ptx::mbar_init(bar_mma + i, 1);
        }
        ptx::mbar_init(bar_done, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        for (int c = 0; c < 2 && c < nch; ++c) {
            ptx::mbar_arrive_expect_tx(bar_tma + c, SROW_TC_KBUF);
            ptx::tma_load_2d(base + c * SROW_TC_KBUF, chunk_map(c), 0, chunk_row(c), bar_tma + c);
        }
    }
    {   // x operand: thread t writes 16 bytes of half t/128, row (t/8)%16 (zero past the
        // CTA's rows), swizzled: 16-byte chunk index XOR row % 8
        const int hx = tid >> 7, row = (tid >> 3) & 15, ch = tid & 7;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (row < SROW_G && xr[row] != nullptr)
            val = __ldg(reinterpret_cast<const uint4*>(xr[row] + hx * 64 + ch * 8));
        *reinterpret_cast<uint4*>(base + SROW_TC_XT + hx * 2048 + row * 128 +
                                  ((ch ^ (row & 7)) << 4)) = val;
    }
    ptx::fence_proxy_async_smem();  // the x operand is read by the tensor cores
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t deadline = ptx::globaltimer_ns() + 2000000000ull;
    if (tid == 0) {
        const uint32_t idesc = ptx::idesc_bf16_f32(128, 16);
        bool ok = true;
        for (int c = 0; c < nch && ok; ++c) {
            const int bf = c & 1;
            const uint32_t par = (uint32_t)(c >> 1) & 1u;
            if (!ptx::mbar_wait_bounded(bar_tma + bf, par, deadline)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const uint64_t ad = ptx::umma_desc_kmajor_sw128(base + bf * SROW_TC_KBUF);
            const uint64_t bd =
                ptx::umma_desc_kmajor_sw128(base + SROW_TC_XT + ((c % cpt) / cph) * 2048);
#pragma unroll
            for (int k = 0; k < 4; ++k)  // K = 64 in steps of 16 (32 bytes)
                ptx::umma_bf16(tmem + 16u * (uint32_t)c, ad + 2 * k, bd + 2 * k, idesc,
                               k > 0 ? 1u : 0u);
            ptx::umma_commit(bar_mma + bf);
            if (c + 2 < nch) {  // buffer bf is free once this chunk's products are done
                if (!ptx::mbar_wait_bounded(bar_mma + bf, par, deadline)) {
                    ok = false;
                    break;
                }
                ptx::mbar_arrive_expect_tx(bar_tma + bf, SROW_TC_KBUF);
                ptx::tma_load_2d(base + bf * SROW_TC_KBUF, chunk_map(c + 2), 0, chunk_row(c + 2),
                                 bar_tma + bf);
            }
        }
        if (ok) {
            ptx::umma_commit(bar_done);
        } else {
            *abort_flag = 1;
            raise_err(SDM_DEVERR_TIMEOUT);
        }
    }
    __syncthreads();  // thread 0 has issued everything (or given up)
    bool aborted = *abort_flag != 0;
    if (!aborted && !ptx::mbar_wait_bounded(bar_done, 0u, deadline)) {
        aborted = true;
        if (tid == 0) raise_err(SDM_DEVERR_TIMEOUT);
    }
    ptx::tc_fence_after();
    if (!aborted) {  // warp w reads TMEM lanes 32 (w % 4) .. + 31 of every other chunk
        const int q = warp & 3;
        for (int c = warp >> 2; c < nch; c += 2) {
            float v[4];
            tmem_ld4(tmem + ((uint32_t)(32 * q) << 16) + 16u * (uint32_t)c, v);
            const int tb = c / cpt, cc = c % cpt;
            const int hf = cc / cph, sidx = (cc % cph) * 128 + 32 * q + lane;
            if (sidx < n)
#pragma unroll
                for (int g = 0; g < SROW_G; ++g)
                    if (rtab[g] == tb)
                        reinterpret_cast<float*>(segs + (size_t)(g * 2 + hf) * seg_bytes)[sidx] = v[g];
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, TCOLS);
    }
    return !aborted;
}

// Phase 2 for one warp: the k_half best of one (row, half) score segment into tvo / tio,
// best first.  The segment's spare bytes are the warp's scratch.
template <int PL, int KP>
SDM_DEV void srow_half_topk(unsigned char* seg, int n, int kh, float* tvo, int* tio, int lane) {
    constexpr int NP = 32 * PL;
    const float* scf = reinterpret_cast<const float*>(seg);
    if constexpr (KP == 32) {
        uint32_t key[PL], id[PL];
#pragma unroll
        for (int c = 0; c < PL; ++c) {
            const int i = c * 32 + lane;
            id[c] = (uint32_t)i;
            key[c] = i < n ? order_key(scf[i]) : 0u;
        }
        uint32_t bk, bi;
        if constexpr (PL <= 2) {
            top32_columns<PL>(key, id, lane);
            bk = key[0];
            bi = id[0];
        } else {  // the segment's second half (NP * 4 >= 512 bytes) is the scratch
            int2* scr = reinterpret_cast<int2*>(seg + NP * 4);
            top32_pruned<PL>(key, id, scr, lane, bk, bi);
        }
        if (lane < kh) {
            tvo[lane] = key_value(bk);
            tio[lane] = (int)bi;
        }
    } else {
        uint32_t key[PL];
        int id[PL];
#pragma unroll
        for (int r = 0; r < PL; ++r) {
            const int i = lane * PL + r;
            id[r] = i;
            key[r] = i < n ? order_key(scf[i]) : 0u;
        }
        // bitonic sort of the lane's block, best first (key desc, sub-index asc)
#pragma unroll
        for (int k = 2; k <= PL; k <<= 1) {
#pragma unroll
            for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
                for (int i = 0; i < PL; ++i) {
                    const int l = i ^ j;
                    if (l > i) {
                        const bool l_better =
                            key[l] > key[i] || (key[l] == key[i] && id[l] < id[i]);
                        if (((i & k) == 0) == l_better) {
                            const uint32_t tk = key[i];
                            key[i] = key[l];
                            key[l] = tk;
                            const int tix = id[i];
                            id[i] = id[l];
                            id[l] = tix;
                        }
                    }
                }
            }
        }
        __syncwarp();  // every lane has read its scores: the segment now holds the lists
        int2* lst = reinterpret_cast<int2*>(seg);  // [32][PL]
#pragma unroll
        for (int r = 2; r < PL; ++r) lst[lane * PL + r] = make_int2((int)key[r], id[r]);
        __syncwarp();
        uint32_t hk = key[0];
        int hi = id[0];
        uint32_t nk = PL > 1 ? key[PL > 1 ? 1 : 0] : 0u;
        int ni = PL > 1 ? id[PL > 1 ? 1 : 0] : 0;
        int p = 1;  // position of (nk, ni) in the lane's list
        for (int q = 0; q < kh; ++q) {
            const uint32_t mx = __reduce_max_sync(0xffffffffu, hk);
            const uint32_t bal = __ballot_sync(0xffffffffu, hk == mx);
            if (lane == __ffs(bal) - 1) {
                tvo[q] = key_value(hk);
                tio[q] = hi;
                hk = nk;
                hi = ni;
                ++p;
                if (p < PL) {
                    const int2 e = lst[lane * PL + p];
                    nk = (uint32_t)e.x;
                    ni = e.y;
                } else {
                    nk = 0u;
                    ni = 0;
                }
            }
        }
    }
}

// Phase 3 for one warp, k_half and top <= 32: the `top` best staircase pairs (cand, nc) of
// the row's two half lists, ranked by their sums; lane q < top gets the q-th slot and its
// softmax weight.  scr: 64 entries of scratch.
SDM_DEV void srow_combine32(const float* t1, const int* i1, const float* t2, const int* i2,
                            const int* cand, int nc, int n, int top, int2* scr, int lane,
                            uint32_t& slot, float& weight) {
    constexpr int C = SROW_CAND / 32;
    uint32_t key[C], id[C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
        const int e = c * 32 + lane;
        if (e < nc) {
            const int pr = cand[e], pa = pr >> 8, pb = pr & 255;
            key[c] = order_key(t1[pa] + t2[pb]);
            id[c] = (uint32_t)i1[pa] * (uint32_t)n + (uint32_t)i2[pb];
        } else {
            key[c] = 0u;
            id[c] = 0x40000000u + (uint32_t)e;  // padding, distinct from every slot
        }
    }
    uint32_t bk, bi;
    if (nc <= 64) {
        uint32_t k2[2] = {key[0], key[1]}, i2c[2] = {id[0], id[1]};
        top32_columns<2>(k2, i2c, lane);
        bk = k2[0];
        bi = i2c[0];
    } else {
        top32_pruned<C>(key, id, scr, lane, bk, bi);
    }
    const float v = key_value(bk);
    const float mx = __shfl_sync(0xffffffffu, v, 0);
    const float ex = lane < top ? expf(v - mx) : 0.f;
    float z = ex;
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) z += __shfl_xor_sync(0xffffffffu, z, m);
    slot = bi;
    weight = ex / z;
}

// Phase 3 for one warp, k_half or top up to 64: lane l owns staircase columns b = l, l + 32,
// whose candidates are already sorted along a, and `top` rounds of best-head selection take
// them in order (equal sums: redux.sync min over slots); svo / sso receive the selection.
template <int KP>
SDM_DEV void srow_combine_wide(const float* t1, const int* i1, const float* t2, const int* i2,
                               int kh, int n, int top, float* svo, uint32_t* sso, int lane,
                               int32_t* idx_row, float* w_row) {
    constexpr int CPL = KP / 32;
    int ca[CPL], lim[CPL];
    float v2[CPL], cv[CPL];
    uint32_t j2[CPL], ck[CPL], cs[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const int bcol = lane + 32 * c;
        ca[c] = 0;
        lim[c] = bcol < kh ? min(kh, top / (bcol + 1)) : 0;
        v2[c] = bcol < kh ? t2[bcol] : 0.f;
        j2[c] = bcol < kh ? (uint32_t)i2[bcol] : 0u;
    }
    auto head = [&](int c) {
        if (ca[c] < lim[c]) {
            cv[c] = t1[ca[c]] + v2[c];
            ck[c] = order_key(cv[c]);
            cs[c] = (uint32_t)i1[ca[c]] * (uint32_t)n + j2[c];
        } else {
            cv[c] = 0.f;
            ck[c] = 0u;
            cs[c] = 0xffffffffu;
        }
    };
#pragma unroll
    for (int c = 0; c < CPL; ++c) head(c);
    for (int q = 0; q < top; ++q) {
        uint32_t bk = ck[0], bs = cs[0];
        float bv = cv[0];
        int bc = 0;
#pragma unroll
        for (int c = 1; c < CPL; ++c)
            if (ck[c] > bk || (ck[c] == bk && cs[c] < bs)) {
                bk = ck[c];
                bs = cs[c];
                bv = cv[c];
                bc = c;
            }
        const uint32_t mx = __reduce_max_sync(0xffffffffu, bk);
        const bool eq = bk == mx;
        uint32_t bal = __ballot_sync(0xffffffffu, eq);
        if (__popc(bal) > 1) {  // equal sums: the lower slot first
            const uint32_t ms = __reduce_min_sync(0xffffffffu, eq ? bs : 0xffffffffu);
            bal = __ballot_sync(0xffffffffu, eq && bs == ms);
        }
        if (lane == __ffs(bal) - 1) {
            svo[q] = bv;
            sso[q] = bs;
#pragma unroll
            for (int c = 0; c < CPL; ++c)
                if (c == bc) {
                    ++ca[c];
                    head(c);
                }
        }
    }
    __syncwarp();
    const float mx = svo[0];
    float ex[CPL], z = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const int q = lane + 32 * c;
        ex[c] = q < top ? expf(svo[q] - mx) : 0.f;
        z += ex[c];
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) z += __shfl_xor_sync(0xffffffffu, z, m);
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const int q = lane + 32 * c;
        if (q < top) {
            idx_row[q] = (int32_t)sso[q];
            w_row[q] = ex[c] / z;
        }
    }
}

template <typename XT, int PL, int KP, bool TCD>
__global__ void __launch_bounds__(SROW_THREADS, 4) score_rows_kernel(
    const __grid_constant__ CUtensorMap km0, const __grid_constant__ CUtensorMap km1,
    ScoreRowsArgs a) {
    constexpr int NB = 2;  // 8-element chunks per load block
    using SM = SrowSmem<PL, KP>;
    extern __shared__ __align__(16) unsigned char srow_smem[];
    const int role = blockIdx.z;
    const XT* __restrict__ x = static_cast<const XT*>(role ? a.x[1] : a.x[0]);
    const XT* __restrict__ sk = static_cast<const XT*>(role ? a.sk[1] : a.sk[0]);
    const int top = role ? a.top[1] : a.top[0];
    int32_t* __restrict__ idx_out = role ? a.idx[1] : a.idx[0];
    float* __restrict__ w_out = role ? a.w[1] : a.w[0];
    // a launch that reads this one's outputs may start now and wait for them itself
    asm volatile("griddepcontrol.launch_dependents;");
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y, d_k = a.d_k, hd = d_k >> 1, n = a.n, kh = a.k_half;
    const long long rows = (long long)a.B * a.T;
    const long long r0 = (long long)blockIdx.x * SROW_G;

    unsigned char* base = srow_smem;
    if constexpr (TCD) base += (1024 - (ptx::smem_u32(srow_smem) & 1023)) & 1023;
    float* xs = reinterpret_cast<float*>(base);  // [G][d_k] (CUDA-core dots)
    const SM sm(base + (TCD ? (size_t)SROW_TC_HEAD : srow_align16((size_t)SROW_G * d_k * 4)));
    // element offset of row r = b*T + t in the [B,H,T,.] tensors: (b*H + h)*T + t
    auto row_off = [&](long long r) -> size_t {
        const long long b = a.T == 1 ? r : r / a.T;
        return ((size_t)b * a.H + h) * a.T + (size_t)(r - b * a.T);
    };
    if (KP == 32 && tid < SROW_CAND) {
        sm.cand[tid] = role ? a.cand[1][tid] : a.cand[0][tid];
        if (tid == 0) sm.ncand[0] = role ? a.ncand[1] : a.ncand[0];
    }

    if constexpr (TCD) {
        // ---- 1. tensor-core dot products ----------------------------------------------------
        const __nv_bfloat16* xr[SROW_G];
        int rtab[SROW_G];
#pragma unroll
        for (int g = 0; g < SROW_G; ++g) {
            xr[g] = r0 + g < rows
                        ? reinterpret_cast<const __nv_bfloat16*>(x) + row_off(r0 + g) * 128
                        : nullptr;
            rtab[g] = 0;
        }
        srow_tc_dots<32 * PL, 1>(base, sm.segs, SM::SEG, role ? &km1 : &km0, nullptr, xr, rtab,
                                 h, n);
    } else {
        // ---- 1a. first sub-key block in flight while x is staged -----------------------------
        const int hf1 = tid >> 7, j1 = tid & 127;  // threads 0..127 half 0, 128..255 half 1
        const XT* tab = sk + (size_t)(h * 2 + hf1) * n * hd;
        Chunk8<XT> r0c[NB], r1c[NB];
        auto load_block = [&](int s0, int d0) {
            const int s1 = s0 + 128 < n ? s0 + 128 : s0;
    #pragma unroll
            for (int c = 0; c < NB; ++c)
                if (d0 + 8 * c < hd) {
                    r0c[c].load(tab + (size_t)s0 * hd + d0 + 8 * c);
                    r1c[c].load(tab + (size_t)s1 * hd + d0 + 8 * c);
                }
        };
        if (j1 < n) load_block(j1, 0);

        // ---- 0. x rows (zeros past the last row) --------------------------------------------
    #pragma unroll
        for (int g = 0; g < SROW_G; ++g) {
            const bool live = r0 + g < rows;
            for (int c = tid; c < d_k; c += SROW_THREADS)
                xs[g * d_k + c] = live ? to_f32(x[row_off(r0 + g) * d_k + c]) : 0.f;
        }
        __syncthreads();

        // ---- 1b. dot products: sub-keys j, j + 128 (then + 256, + 384) of this thread's half --
        {
            const float* xh = xs + hf1 * hd;
            for (int s0 = j1; s0 < n; s0 += 256) {
                const int s1 = s0 + 128;
                float acc0[SROW_G], acc1[SROW_G];
    #pragma unroll
                for (int g = 0; g < SROW_G; ++g) acc0[g] = acc1[g] = 0.f;
                for (int d0 = 0; d0 < hd; d0 += 8 * NB) {
                    if (d0 > 0) load_block(s0, d0);
    #pragma unroll
                    for (int c = 0; c < NB; ++c) {
                        if (d0 + 8 * c >= hd) break;
                        float k0[8], k1[8];
                        r0c[c].widen(k0);
                        r1c[c].widen(k1);
                        const int d = d0 + 8 * c;
    #pragma unroll
                        for (int g = 0; g < SROW_G; ++g) {
                            const float4 xa = *reinterpret_cast<const float4*>(xh + g * d_k + d);
                            const float4 xb = *reinterpret_cast<const float4*>(xh + g * d_k + d + 4);
                            const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
    #pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                acc0[g] = fmaf(xv[e], k0[e], acc0[g]);
                                acc1[g] = fmaf(xv[e], k1[e], acc1[g]);
                            }
                        }
                    }
                }
                if (s0 + 256 < n) load_block(s0 + 256, 0);
    #pragma unroll
                for (int g = 0; g < SROW_G; ++g) {
                    float* scf = reinterpret_cast<float*>(sm.seg(g, hf1));
                    scf[s0] = acc0[g];
                    if (s1 < n) scf[s1] = acc1[g];
                }
            }
        }
        __syncthreads();
    }

    // ---- 2. per-half top-k: warp (g, hf) ---------------------------------------------------
    {
        const int g = warp >> 1, hf = warp & 1;
        srow_half_topk<PL, KP>(sm.seg(g, hf), n, kh, sm.tv + (g * 2 + hf) * KP,
                               sm.ti + (g * 2 + hf) * KP, lane);
    }
    __syncthreads();

    // ---- 3. combine and softmax: warp g --------------------------------------------------
    if (warp >= SROW_G || r0 + warp >= rows) return;
    const int g = warp;
    const float* t1 = sm.tv + (g * 2) * KP;
    const int* i1 = sm.ti + (g * 2) * KP;
    const float* t2 = sm.tv + (g * 2 + 1) * KP;
    const int* i2 = sm.ti + (g * 2 + 1) * KP;
    const size_t ro = row_off(r0 + g);
    if constexpr (KP == 32) {
        // scratch: the second half of the row's first score segment (free by now)
        int2* scr = reinterpret_cast<int2*>(sm.seg(g, 0) + 32 * PL * 4);
        uint32_t slot;
        float wt;
        srow_combine32(t1, i1, t2, i2, sm.cand, sm.ncand[0], n, top, scr, lane, slot, wt);
        if (lane < top) {
            idx_out[ro * top + lane] = (int32_t)slot;
            w_out[ro * top + lane] = wt;
        }
    } else {
        srow_combine_wide<KP>(t1, i1, t2, i2, kh, n, top, sm.sv + g * KP, sm.ss + g * KP, lane,
                              idx_out + ro * top, w_out + ro * top);
    }
}

}  // namespace sdm
