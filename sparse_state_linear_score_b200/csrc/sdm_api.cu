// C ABI of the SDM hot path (declared in include/sdm.h): host-side validation,
// workspace layout and kernel launches.  One translation unit holds every kernel.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "backward.cuh"
#include "decode.cuh"
#include "plan.cuh"
#include "recur.cuh"
#include "score_bwd.cuh"
#include "score_pk.cuh"
#include "score_rows.cuh"
#include "score_simt.cuh"
#include "score_tc.cuh"
#include "state.cuh"
#include "stats.cuh"
#include "gemm_tc.cuh"
#include "layer.cuh"

using namespace sdm;

namespace {

constexpr int kMaxTop = 64;
constexpr size_t kSmemBudget = 220 * 1024;  // dynamic shared memory per CTA we plan for
constexpr size_t kMaskBudget = size_t(512) << 20;  // workspace bytes for per-slot chunk masks
                                                     // (or a quarter of the state, if larger)

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

sdm_status check_dims(const sdm_dims* d) {
    if (!d) return SDM_ERR_ARG;
    if (d->x_dtype != SDM_F32 && d->x_dtype != SDM_BF16) return SDM_ERR_DTYPE;
    if (d->v_dtype != SDM_F32 && d->v_dtype != SDM_BF16) return SDM_ERR_DTYPE;
    if (d->decay != SDM_DECAY_ALL && d->decay != SDM_DECAY_TOUCHED) return SDM_ERR_ARG;
    if (d->B < 1 || d->H < 1 || d->T < 0) return SDM_ERR_SHAPE;
    if ((long long)d->B * d->H > 65535) return SDM_ERR_SHAPE;
    if (d->d_k < 16 || d->d_k > 256 || (d->d_k / 2) % 8 != 0 || d->d_k % 2 != 0) return SDM_ERR_SHAPE;
    if (d->n_sub < 1 || d->n_sub > 4096) return SDM_ERR_SHAPE;
    if (d->d_v < 4 || d->d_v > 256 || d->d_v % 4 != 0) return SDM_ERR_SHAPE;
    if (d->k_half < 1 || d->k_half > 64 || d->k_half > d->n_sub) return SDM_ERR_SHAPE;
    if (d->W < 1 || d->W > kMaxTop || d->R < 1 || d->R > kMaxTop) return SDM_ERR_SHAPE;
    if (d->W > d->k_half * d->k_half || d->R > d->k_half * d->k_half) return SDM_ERR_SHAPE;
    return SDM_OK;
}

inline long long N_of(const sdm_dims* d) { return (long long)d->n_sub * d->n_sub; }
inline long long BH_of(const sdm_dims* d) { return (long long)d->B * d->H; }
// Tokens per chunk of the prefill recurrence with CW-column slices: as many as fit the plan's
// occurrence budget, the run kernel's shared memory and the 256-token scan of plan_local.
int chunk_tokens_cw(const sdm_dims* d, int CW) {
    int C = PLAN_MAX_OCC / (d->W + d->R);
    if (C > PLAN_MAX_C) C = PLAN_MAX_C;
    C &= ~3;  // matrices move in 16-byte rows
    while (C > 4 && run_smem_bytes(C, d->W, d->R, CW, 4) > kSmemBudget) C -= 4;
    return C < 4 ? 4 : C;
}

int device_sms() {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0, n = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
            sms = n;
        else
            return 148;
    }
    return sms;
}

// Value columns per row-pass CTA.  The row pass is bound by the SM's rate of scattered row
// requests, not by their bytes (4-column slices take as long per chunk as 8-column ones), so
// wider slices move more bytes per request.  16 columns when the row is a multiple of 16, the
// chunk size stays what 8 columns allow, and the CTAs still fill the SMs (B*H*d_v/16 of
// them); else 8, else 4.
int col_width(const sdm_dims* d) {
    if (d->d_v % 16 == 0 && chunk_tokens_cw(d, 16) == chunk_tokens_cw(d, 8) &&
        BH_of(d) * (d->d_v / 16) >= device_sms())
        return 16;
    return d->d_v % 8 == 0 ? 8 : 4;
}

int chunk_tokens(const sdm_dims* d) { return chunk_tokens_cw(d, col_width(d)); }

struct WsLayout {
    int C, J;
    int walk_parts;
    bool lstart_smem;
    size_t walk_smem;
    size_t off_lam, off_csum, off_Lstart, off_st0, off_fe, off_lk, off_occw, off_mask, off_wtab,
        off_cnt;
    size_t off_rs, off_img, off_vfc, off_vsh, total;
    int MW;  // mask words per slot, 0 when the walk is used
};

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

WsLayout ws_layout(const sdm_dims* d) {
    WsLayout L{};
    const size_t BH = (size_t)BH_of(d), T = (size_t)d->T, N = (size_t)N_of(d);
    const size_t occ = T * (size_t)(d->W + d->R);
    L.C = chunk_tokens(d);
    L.J = (int)((T + L.C - 1) / L.C);
    // the walk: one CTA per (b,h) and slot partition, the chunk-start prefixes in shared memory
    // when they fit; as many partitions as keep every walk of the call in one wave
    const size_t ring = (size_t)WALK_RING * (PLAN_MAX_OCC + PLAN_MAX_C) * 4;
    L.lstart_smem = ring + (size_t)(L.J + 1) * 8 <= kSmemBudget;
    L.walk_smem = ring + (L.lstart_smem ? (size_t)(L.J + 1) * 8 : 0);
    const size_t per_sm = (size_t)(228 * 1024) / (L.walk_smem + 1024);
    L.walk_parts = (int)(148 * (per_sm < 1 ? 1 : (per_sm > 4 ? 4 : per_sm)) / BH);
    L.walk_parts = L.walk_parts < 1 ? 1 : (L.walk_parts > 16 ? 16 : L.walk_parts);
    size_t o = 0;
    L.off_lam = o;    o = up256(o + BH * T * 4);
    L.off_csum = o;   o = up256(o + BH * L.J * 8);
    L.off_Lstart = o; o = up256(o + BH * (L.J + 1) * 8);
    L.off_st0 = o;    o = up256(o + BH * occ * 8);
    L.off_fe = o;     o = up256(o + BH * occ * 4);
    L.off_lk = o;     o = up256(o + BH * occ * 4);
    L.off_occw = o;   o = up256(o + BH * occ * 4);
    // per-slot chunk masks replace the sequential walk when they stay small: within a fixed
    // budget, or within a quarter of the state's own rows (whose gathers dwarf their traffic)
    const size_t mw = (size_t)(L.J + 63) / 64;
    const size_t state_rows = BH * N * (size_t)d->d_v * 4;
    const size_t budget = kMaskBudget > state_rows / 4 ? kMaskBudget : state_rows / 4;
    L.MW = (L.J <= 512 && BH * N * mw * 8 <= budget) ? (int)mw : 0;
    L.off_mask = o;   o = up256(o + BH * N * (size_t)L.MW * 8);
    L.off_wtab = o;   o = up256(o + (L.MW ? 0 : BH * N * 2));
    L.off_cnt = o;    o = up256(o + BH * (size_t)L.J * 4);
    L.off_rs = o;     o = up256(o + BH * occ * 4);
    L.off_img = o;    o = up256(o + BH * (size_t)L.J * run_img(L.C, d->W, d->R).bytes);
    // touched-slots decay: in-chunk decay products of each occurrence (see PlanPtrs)
    const size_t vt = d->decay == SDM_DECAY_TOUCHED ? BH * occ * 4 : 0;
    L.off_vfc = o;    o = up256(o + vt);
    L.off_vsh = o;    o = up256(o + vt);
    L.total = o;
    return L;
}

PlanPtrs plan_ptrs(const WsLayout& L, void* ws) {
    unsigned char* b = static_cast<unsigned char*>(ws);
    PlanPtrs P;
    P.lam = reinterpret_cast<float*>(b + L.off_lam);
    P.csum = reinterpret_cast<double*>(b + L.off_csum);
    P.Lstart = reinterpret_cast<double*>(b + L.off_Lstart);
    P.st0 = reinterpret_cast<double*>(b + L.off_st0);
    P.fe = reinterpret_cast<float*>(b + L.off_fe);
    P.lk = reinterpret_cast<int32_t*>(b + L.off_lk);
    P.occw = reinterpret_cast<uint32_t*>(b + L.off_occw);
    P.mask = L.MW ? reinterpret_cast<unsigned long long*>(b + L.off_mask) : nullptr;
    P.MW = L.MW;
    P.wtab = L.MW ? nullptr : reinterpret_cast<short*>(b + L.off_wtab);
    P.rs = reinterpret_cast<int32_t*>(b + L.off_rs);
    P.img = b + L.off_img;
    const bool touched = L.off_vsh != L.off_vfc;
    P.vfc = touched ? reinterpret_cast<float*>(b + L.off_vfc) : nullptr;
    P.vsh = touched ? reinterpret_cast<float*>(b + L.off_vsh) : nullptr;
    return P;
}

sdm_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? SDM_OK : SDM_ERR_CUDA;
}

template <typename K>
bool set_smem(K kernel, size_t bytes) {
    if (bytes <= 48 * 1024) return true;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) ==
           cudaSuccess;
}

sdm_status check_state(const sdm_state* st) {
    if (!st || !st->M || !st->stamp || !st->Lambda || !st->M0) return SDM_ERR_ARG;
    if (!aligned16(st->M) || !aligned16(st->stamp) || !aligned16(st->M0)) return SDM_ERR_ALIGN;
    if (((uintptr_t)st->Lambda & 7u) != 0) return SDM_ERR_ALIGN;
    return SDM_OK;
}

// ---- tensor-core scoring: TMA descriptors and dispatch ------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// Shapes the tensor-core kernel takes: bf16, 64-wide halves, sub-key count a multiple of 64,
// at most 32 kept per half and selected, and enough tokens per sequence for full tiles
// (single-token decode stays on the CUDA-core kernel, which spreads rows over all SMs).
bool score_tc_eligible(const sdm_dims* d, int top) {
    if (d->x_dtype != SDM_BF16 || d->d_k != 128) return false;
    if (d->n_sub % 64 != 0 || d->n_sub > 4096) return false;
    if (d->k_half > TC_KMAX || top > TC_KMAX) return false;
    if (d->n_sub > TC_NB && d->k_half * TC_THREADS * 6 > 16384) return false;  // R1 beside x half 1
    if (top > d->k_half) return false;  // the pair staircase covers top <= k_half
    return d->T >= 64;
}

template <int KP>
sdm_status launch_score_tc_t(const sdm_dims* d, const CUtensorMap& xm, const CUtensorMap& km,
                             const ScoreTcArgs& a, dim3 grid, cudaStream_t s) {
    auto kern = score_tc_kernel<KP>;
    if (!set_smem(kern, TC_SMEM_BYTES)) return SDM_ERR_CUDA;
    kern<<<grid, TC_THREADS, TC_SMEM_BYTES, s>>>(xm, km, a);
    return launch_status();
}

sdm_status launch_score_tc(const sdm_dims* d, const void* x, const void* sk, int top,
                           int32_t* idx, float* w, cudaStream_t s) {
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return SDM_ERR_CUDA;
    ScoreTcArgs a{};
    a.B = d->B; a.H = d->H; a.T = d->T; a.n = d->n_sub; a.k_half = d->k_half; a.top = top;
    a.nbox = d->n_sub < TC_NB ? d->n_sub : TC_NB;
    // A tile is always 128 rows that the TMA fills: 128 tokens of one sequence, or 64 tokens
    // of two when T = 64.  Rows past T or B are the load's zero fill, so the tensor cores
    // never read rows that no load wrote.
    a.bt = d->T == 64 ? 64 : 128;
    a.bb = 128 / a.bt;
    a.n_tt = (d->T + a.bt - 1) / a.bt;
    a.idx = idx;
    a.w = w;
    const int n_bt = (d->B + a.bb - 1) / a.bb;
    CUtensorMap xm, km;
    {
        const cuuint64_t dims[4] = {(cuuint64_t)d->d_k, (cuuint64_t)d->T, (cuuint64_t)d->H,
                                    (cuuint64_t)d->B};
        const cuuint64_t strides[3] = {(cuuint64_t)d->d_k * 2, (cuuint64_t)d->T * d->d_k * 2,
                                       (cuuint64_t)d->H * d->T * d->d_k * 2};
        const cuuint32_t box[4] = {64, (cuuint32_t)a.bt, 1, (cuuint32_t)a.bb};
        const cuuint32_t es[4] = {1, 1, 1, 1};
        if (enc(&xm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(x), dims, strides, box,
                es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return SDM_ERR_CUDA;
    }
    {
        const cuuint64_t dims[2] = {64, (cuuint64_t)d->H * 2 * d->n_sub};
        const cuuint64_t strides[1] = {64 * 2};
        const cuuint32_t box[2] = {64, (cuuint32_t)a.nbox};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&km, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(sk), dims, strides, box,
                es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return SDM_ERR_CUDA;
    }
    const dim3 grid((unsigned)(a.n_tt * n_bt), (unsigned)d->H);
    const int k = d->k_half;
    if (k <= 8) return launch_score_tc_t<8>(d, xm, km, a, grid, s);
    if (k <= 16) return launch_score_tc_t<16>(d, xm, km, a, grid, s);
    return launch_score_tc_t<32>(d, xm, km, a, grid, s);
}

// Shapes the tensor-core scorer takes: bf16, 64-wide halves, at most 1024 sub-keys per half (a
// multiple of 64), at most 64 kept per half, top <= k_half (the staircase), and calls of at
// least 64 tokens (shorter ones go to the row scorer, which spreads rows over all SMs).
bool score_pk_eligible(const sdm_dims* d, int top) {
    if (d->x_dtype != SDM_BF16 || d->d_k != 128) return false;
    if (d->n_sub % 64 != 0 || d->n_sub > PK_NMAX) return false;
    if (d->k_half > 64 || top > d->k_half) return false;
    return d->T >= 64;
}

bool encode_x_map(EncodeTiledFn enc, CUtensorMap* m, const sdm_dims* d, const void* x, int bt,
                  int bb) {
    const cuuint64_t dims[4] = {(cuuint64_t)d->d_k, (cuuint64_t)d->T, (cuuint64_t)d->H,
                                (cuuint64_t)d->B};
    const cuuint64_t strides[3] = {(cuuint64_t)d->d_k * 2, (cuuint64_t)d->T * d->d_k * 2,
                                   (cuuint64_t)d->H * d->T * d->d_k * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)bt, 1, (cuuint32_t)bb};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(x), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_sk_map(EncodeTiledFn enc, CUtensorMap* m, const sdm_dims* d, const void* sk, int rows) {
    const cuuint64_t dims[2] = {64, (cuuint64_t)d->H * 2 * d->n_sub};
    const cuuint64_t strides[1] = {64 * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)rows};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(sk), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KP, int ROWS>
sdm_status launch_score_pk_t(const CUtensorMap (&xm)[2], const CUtensorMap (&km)[2],
                             const PkArgs& a, dim3 grid, cudaStream_t s) {
    auto kern = score_pk_kernel<KP, ROWS>;
    constexpr size_t smem = PkCfg<KP, ROWS>::SMEM;
    if (!set_smem(kern, smem)) return SDM_ERR_CUDA;
    kern<<<grid, 2 * ROWS, smem, s>>>(xm[0], xm[1], km[0], km[1], a);
    return launch_status();
}

// `roles` (1 or 2) scorings of the same shape in one launch (grid.z = role): role r scores
// x[r] against sk[r] into idx[r], w[r] with top[r] slots.  Lists of up to 32 per half take
// tiles of 128 rows, longer ones tiles of 64 (their candidate lists fill the shared memory).
sdm_status launch_score_pk(const sdm_dims* d, int roles, const void* const* x,
                           const void* const* sk, const int* top, int32_t* const* idx,
                           float* const* w, cudaStream_t s) {
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return SDM_ERR_CUDA;
    const int rows = d->k_half <= 32 ? 128 : 64;
    PkArgs a{};
    a.B = d->B; a.H = d->H; a.T = d->T; a.n = d->n_sub; a.k_half = d->k_half; a.d_k = d->d_k;
    // a tile is always `rows` rows that the TMA fills: tokens of one sequence, or 64 tokens of
    // two when T = 64 and rows = 128; rows past T or B are the load's zero fill, not selected
    a.bt = (rows == 128 && d->T == 64) ? 64 : rows;
    a.bb = rows / a.bt;
    a.n_tt = (d->T + a.bt - 1) / a.bt;
    a.z0 = pk_z0(d->n_sub, d->k_half);
    CUtensorMap xm[2], km[2];
    for (int r = 0; r < 2; ++r) {
        const int q = r < roles ? r : 0;
        a.top[r] = top[q];
        a.x[r] = static_cast<const __nv_bfloat16*>(x[q]);
        a.sk[r] = static_cast<const __nv_bfloat16*>(sk[q]);
        a.idx[r] = idx[q];
        a.w[r] = w[q];
        if (!encode_x_map(enc, &xm[r], d, x[q], a.bt, a.bb)) return SDM_ERR_CUDA;
        if (!encode_sk_map(enc, &km[r], d, sk[q], d->n_sub < 256 ? d->n_sub : 256)) return SDM_ERR_CUDA;
    }
    const int n_bt = (d->B + a.bb - 1) / a.bb;
    const dim3 grid((unsigned)(a.n_tt * n_bt), (unsigned)d->H, (unsigned)roles);
    if (d->k_half <= 16) return launch_score_pk_t<16, 128>(xm, km, a, grid, s);
    if (d->k_half <= 32) return launch_score_pk_t<32, 128>(xm, km, a, grid, s);
    return launch_score_pk_t<64, 64>(xm, km, a, grid, s);
}

// The row scorer keeps a lane's block of n/32 half-scores in registers (at most 16) and the
// selected lists in shared memory; check_dims already bounds k_half and top by 64 and makes
// the half width a multiple of 8.
bool score_rows_eligible(const sdm_dims* d) { return d->n_sub <= 32 * 16; }

struct RowMaps {
    CUtensorMap km[2];
};

// Tensor maps of two sub-key tables for the row scorer's tensor-core dots: [H*2*n rows][64]
// bf16, boxes of 128 rows, 128-byte swizzle.
bool encode_row_maps(const sdm_dims* d, const void* sk0, const void* sk1, RowMaps* m) {
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return false;
    const void* sk[2] = {sk0, sk1};
    for (int r = 0; r < 2; ++r) {
        const cuuint64_t dims[2] = {64, (cuuint64_t)d->H * 2 * d->n_sub};
        const cuuint64_t strides[1] = {64 * 2};
        const cuuint32_t box[2] = {64, 128};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&m->km[r], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(sk[r]), dims,
                strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    return true;
}

template <typename XT, int PL, bool TCD>
sdm_status launch_score_rows_t(const RowMaps& m, const ScoreRowsArgs& a, int kp, dim3 grid,
                               cudaStream_t s) {
    if (kp <= 32) {
        auto kern = score_rows_kernel<XT, PL, 32, TCD>;
        const size_t smem = score_rows_smem_bytes(a.d_k, PL, 32, TCD);
        if (!set_smem(kern, smem)) return SDM_ERR_CUDA;
        kern<<<grid, SROW_THREADS, smem, s>>>(m.km[0], m.km[1], a);
    } else {
        auto kern = score_rows_kernel<XT, PL, 64, TCD>;
        const size_t smem = score_rows_smem_bytes(a.d_k, PL, 64, TCD);
        if (!set_smem(kern, smem)) return SDM_ERR_CUDA;
        kern<<<grid, SROW_THREADS, smem, s>>>(m.km[0], m.km[1], a);
    }
    return launch_status();
}

// Dot products on the tensor cores for bf16 rows of d_k = 128 and n > 64 (the sub-key
// tables then have 128-byte rows, one 128-byte swizzle span), on CUDA cores otherwise.
template <typename XT>
sdm_status launch_score_rows_x(const RowMaps& m, bool tcd, const ScoreRowsArgs& a, int kp,
                               dim3 grid, cudaStream_t s) {
    const int pl = (a.n + 31) / 32;
    if constexpr (sizeof(XT) == 2) {
        if (tcd) {
            if (pl <= 4) return launch_score_rows_t<XT, 4, true>(m, a, kp, grid, s);
            if (pl <= 8) return launch_score_rows_t<XT, 8, true>(m, a, kp, grid, s);
            return launch_score_rows_t<XT, 16, true>(m, a, kp, grid, s);
        }
    }
    if (pl <= 1) return launch_score_rows_t<XT, 1, false>(m, a, kp, grid, s);
    if (pl <= 2) return launch_score_rows_t<XT, 2, false>(m, a, kp, grid, s);
    if (pl <= 4) return launch_score_rows_t<XT, 4, false>(m, a, kp, grid, s);
    if (pl <= 8) return launch_score_rows_t<XT, 8, false>(m, a, kp, grid, s);
    return launch_score_rows_t<XT, 16, false>(m, a, kp, grid, s);
}

// One launch for `roles` (1 or 2) scorings of the same shape: role r scores x[r] against
// sk[r] into idx[r], w[r] with top[r] slots.
sdm_status launch_score_rows(const sdm_dims* d, int roles, const void* const* x,
                             const void* const* sk, const int* top, int32_t* const* idx,
                             float* const* w, cudaStream_t s) {
    ScoreRowsArgs a{};
    int kp = d->k_half;
    for (int r = 0; r < 2; ++r) {
        const int q = r < roles ? r : 0;
        a.x[r] = x[q];
        a.sk[r] = sk[q];
        a.top[r] = top[q];
        a.idx[r] = idx[q];
        a.w[r] = w[q];
        a.ncand[r] = score_rows_staircase(d->k_half, top[q], a.cand[r]);
        if (top[q] > kp) kp = top[q];
    }
    a.B = d->B; a.H = d->H; a.T = d->T; a.d_k = d->d_k; a.n = d->n_sub; a.k_half = d->k_half;
    const long long rows = (long long)d->B * d->T;
    const dim3 grid((unsigned)((rows + SROW_G - 1) / SROW_G), (unsigned)d->H, (unsigned)roles);
    RowMaps m;
    memset(&m, 0, sizeof(m));
    const bool tcd = d->x_dtype == SDM_BF16 && d->d_k == 128 && d->n_sub > 64;
    if (tcd && !encode_row_maps(d, a.sk[0], a.sk[1], &m)) return SDM_ERR_CUDA;
    if (d->x_dtype == SDM_F32) return launch_score_rows_x<float>(m, false, a, kp, grid, s);
    return launch_score_rows_x<__nv_bfloat16>(m, tcd, a, kp, grid, s);
}

// The one-launch decode step (decode_fused_kernel): bf16 keys and queries of d_k = 128, 64 < n
// <= 512 (the row scorer's tensor-core dot products), k_half, W, R <= 32, d_v <= 256.
bool decode_fused_eligible(const sdm_dims* d) {
    return d->x_dtype == SDM_BF16 && d->d_k == 128 && d->n_sub > 64 && d->n_sub <= 512 &&
           d->k_half <= 32 && d->W <= 32 && d->R <= 32 && d->d_v <= 256 &&
           decode_fused_fits(d->W, d->R, d->d_v);
}

template <int PL, typename VT, int QPL>
sdm_status launch_decode_fused_t(const RowMaps& m, const ScoreRowsArgs& a, const DecArgs& dk,
                                 dim3 grid, cudaStream_t s) {
    auto kern = decode_fused_kernel<PL, VT, QPL>;
    const size_t smem = decode_fused_smem_bytes(PL);
    if (!set_smem(kern, smem)) return SDM_ERR_CUDA;
    kern<<<grid, SROW_THREADS, smem, s>>>(m.km[0], m.km[1], a, dk);
    return launch_status();
}

template <typename VT>
sdm_status launch_decode_fused_v(int pl, int qpl, const RowMaps& m, const ScoreRowsArgs& a,
                                 const DecArgs& dk, dim3 grid, cudaStream_t s) {
    if (qpl <= 1) {
        if (pl <= 4) return launch_decode_fused_t<4, VT, 1>(m, a, dk, grid, s);
        if (pl <= 8) return launch_decode_fused_t<8, VT, 1>(m, a, dk, grid, s);
        return launch_decode_fused_t<16, VT, 1>(m, a, dk, grid, s);
    }
    if (pl <= 4) return launch_decode_fused_t<4, VT, 2>(m, a, dk, grid, s);
    if (pl <= 8) return launch_decode_fused_t<8, VT, 2>(m, a, dk, grid, s);
    return launch_decode_fused_t<16, VT, 2>(m, a, dk, grid, s);
}

sdm_status launch_decode_fused(const sdm_dims* d, const void* q, const void* k, const void* v,
                               const float* alpha, const float* beta, const void* skw,
                               const void* skr, const sdm_state* st, int32_t* widx, float* ww,
                               int32_t* ridx, float* rw, float* out, cudaStream_t s) {
    ScoreRowsArgs a{};
    const void* xs[2] = {k, q};
    const void* sks[2] = {skw, skr};
    const int tops[2] = {d->W, d->R};
    int32_t* idxs[2] = {widx, ridx};
    float* wts[2] = {ww, rw};
    for (int r = 0; r < 2; ++r) {
        a.x[r] = xs[r];
        a.sk[r] = sks[r];
        a.top[r] = tops[r];
        a.idx[r] = idxs[r];
        a.w[r] = wts[r];
        a.ncand[r] = score_rows_staircase(d->k_half, tops[r], a.cand[r]);
    }
    a.B = d->B; a.H = d->H; a.T = 1; a.d_k = d->d_k; a.n = d->n_sub; a.k_half = d->k_half;
    DecArgs dk{};
    dk.v = v;
    dk.alpha = alpha;
    dk.beta = beta;
    dk.M = st->M;
    dk.stamp = st->stamp;
    dk.lambda = st->Lambda;
    dk.M0 = st->M0;
    dk.out = out;
    dk.N = (int)N_of(d);
    dk.d_v = d->d_v;
    dk.touched = d->decay == SDM_DECAY_TOUCHED;
    RowMaps m;
    memset(&m, 0, sizeof(m));
    if (!encode_row_maps(d, skw, skr, &m)) return SDM_ERR_CUDA;
    const dim3 grid((unsigned)(2 * ((d->B + 3) / 4)), (unsigned)d->H);  // clusters of 2 CTAs
    const int pl = (d->n_sub + 31) / 32, qpl = (d->d_v / 4 + 31) / 32;
    if (d->v_dtype == SDM_BF16)
        return launch_decode_fused_v<__nv_bfloat16>(pl, qpl, m, a, dk, grid, s);
    return launch_decode_fused_v<float>(pl, qpl, m, a, dk, grid, s);
}

sdm_status launch_score(const sdm_dims* d, const void* x, const void* sk, int top, int32_t* idx,
                        float* w, cudaStream_t s);

// Both roles of one call (keys against the write tables, queries against the read tables):
// two tensor-core launches when the shape takes them, else one row-scorer launch for both
// roles (grid.z = role), else the generic path per role.  Arguments as sdm_score_topk.
sdm_status score_both_roles(const sdm_dims* d, const void* q, const void* k, const void* skw,
                            const void* skr, int32_t* widx, float* ww, int32_t* ridx, float* rw,
                            cudaStream_t s) {
    if (!q || !k || !skw || !skr || !widx || !ww || !ridx || !rw) return SDM_ERR_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(skw) || !aligned16(skr) ||
        !aligned16(widx) || !aligned16(ww) || !aligned16(ridx) || !aligned16(rw))
        return SDM_ERR_ALIGN;
    if ((long long)d->B * d->T == 0) return SDM_OK;
    if (score_pk_eligible(d, d->W) && score_pk_eligible(d, d->R)) {
        const void* xs[2] = {k, q};
        const void* sks[2] = {skw, skr};
        const int tops[2] = {d->W, d->R};
        int32_t* idxs[2] = {widx, ridx};
        float* wts[2] = {ww, rw};
        return launch_score_pk(d, 2, xs, sks, tops, idxs, wts, s);
    }
    if (!(score_tc_eligible(d, d->W) && score_tc_eligible(d, d->R)) && score_rows_eligible(d)) {
        const void* xs[2] = {k, q};
        const void* sks[2] = {skw, skr};
        const int tops[2] = {d->W, d->R};
        int32_t* idxs[2] = {widx, ridx};
        float* wts[2] = {ww, rw};
        return launch_score_rows(d, 2, xs, sks, tops, idxs, wts, s);
    }
    sdm_status e = launch_score(d, k, skw, d->W, widx, ww, s);
    if (e) return e;
    return launch_score(d, q, skr, d->R, ridx, rw, s);
}

// column slices per (b,h) in the backward (4 columns each)
int bwd_slices(const sdm_dims* d) { return (d->d_v / 4 + BWD_SLICE_Q - 1) / BWD_SLICE_Q; }

struct BwdLayout {
    size_t off_rows, off_lstamp, off_lam, off_dM, off_pst, off_pds, off_pdww, off_pdrw, off_pdb,
        off_pda, off_gam, off_rpart, off_x0, total;
};

BwdLayout bwd_layout(const sdm_dims* d) {
    BwdLayout L{};
    const size_t BH = (size_t)BH_of(d), T = (size_t)d->T, N = (size_t)N_of(d);
    const size_t S = (size_t)bwd_slices(d);
    size_t o = 0;
    L.off_rows = o;   o = up256(o + BH * T * (size_t)d->W * d->d_v * 4);
    L.off_lstamp = o; o = up256(o + BH * T * (size_t)d->W * 8);
    L.off_lam = o;    o = up256(o + BH * (T + 1) * 8);
    L.off_dM = o;     o = up256(o + BH * N * (size_t)d->d_v * 4);
    L.off_pst = o;    o = up256(o + S * BH * N * 8);
    L.off_pds = o;    o = up256(o + S * BH * N * 8);
    L.off_pdww = o;   o = up256(o + S * BH * T * (size_t)d->W * 4);
    L.off_pdrw = o;   o = up256(o + S * BH * T * (size_t)d->R * 4);
    L.off_pdb = o;    o = up256(o + S * BH * T * 8);
    L.off_pda = o;    o = up256(o + S * BH * T * 8);
    L.off_gam = o;    o = up256(o + BH * 8);
    L.off_rpart = o;  o = up256(o + BH * T * (size_t)d->W);
    L.off_x0 = o;     o = up256(o + BH * S * 8);
    L.total = o;
    return L;
}

template <typename VT, int KPL>
sdm_status launch_backward_t(const sdm_dims* d, const BwdPtrs& P, const void* v,
                             const float* alpha, const float* beta, const int32_t* widx,
                             const float* ww, const int32_t* ridx, const float* rw,
                             const sdm_state* st, const float* dout, const float* dM_end,
                             float* dv, cudaStream_t s) {
    const int touched = d->decay == SDM_DECAY_TOUCHED;
    const int S = bwd_slices(d);
    const unsigned grid = (unsigned)((size_t)BH_of(d) * S);
    bwd_replay_kernel<VT, KPL><<<grid, 32, 0, s>>>((const VT*)v, alpha, beta, widx, ww, st->M,
                                                   st->Lambda, st->M0, P, d->H, (int)N_of(d),
                                                   d->T, d->d_v, d->W, S, touched);
    if (dM_end && !touched) {
        const dim3 xg(grid, (unsigned)((N_of(d) + BWD_X0_ROWS - 1) / BWD_X0_ROWS));
        bwd_x0_kernel<<<xg, 256, 0, s>>>(P, st->M, st->M0, dM_end, d->H, (int)N_of(d), d->T,
                                         d->d_v, S);
    }
    bwd_sweep_kernel<VT, KPL><<<grid, 32, 0, s>>>((const VT*)v, alpha, beta, widx, ww, ridx, rw,
                                                  st->M, st->M0, P, dout, dv, d->H, (int)N_of(d),
                                                  d->T, d->d_v, d->W, d->R, S, touched);
    return launch_status();
}

template <typename XT, int HPL, int TPL>
sdm_status launch_score_bwd_t(const sdm_dims* d, const void* x, const void* sk, int top,
                              const int32_t* idx, const float* w, const float* dw, float* dx,
                              float* dsk, cudaStream_t s) {
    const long long rows = (long long)d->B * d->T;
    const dim3 grid((unsigned)((rows + SBWD_ROWS - 1) / SBWD_ROWS), (unsigned)d->H);
    score_backward_kernel<XT, HPL, TPL><<<grid, SBWD_THREADS, 0, s>>>(
        (const XT*)x, (const XT*)sk, idx, w, dw, d->B, d->H, d->T, d->d_k, d->n_sub, top, dx, dsk);
    return launch_status();
}

template <typename XT>
sdm_status launch_score_bwd_x(const sdm_dims* d, const void* x, const void* sk, int top,
                              const int32_t* idx, const float* w, const float* dw, float* dx,
                              float* dsk, cudaStream_t s) {
    const int hpl = (d->d_k / 2 + 31) / 32;  // d_k <= 256: at most 4
    const bool t2 = top > 32;
#define SDM_SB(H, TP) launch_score_bwd_t<XT, H, TP>(d, x, sk, top, idx, w, dw, dx, dsk, s)
    if (hpl <= 1) return t2 ? SDM_SB(1, 2) : SDM_SB(1, 1);
    if (hpl <= 2) return t2 ? SDM_SB(2, 2) : SDM_SB(2, 1);
    return t2 ? SDM_SB(4, 2) : SDM_SB(4, 1);
#undef SDM_SB
}

template <typename VT, int RPW, int QPL>
sdm_status launch_decode(const sdm_dims* d, const void* v, const float* alpha, const float* beta,
                         const sdm_state* st, const int32_t* widx, const float* ww,
                         const int32_t* ridx, const float* rw, float* out, sdm_stream_t stream) {
    auto kern = decode_kernel<VT, RPW, QPL>;
    const size_t smem = decode_smem_bytes(d->W, d->R, d->d_v);
    if (!set_smem(kern, smem)) return SDM_ERR_CUDA;
    // programmatic dependent launch: the kernel may start while the scoring launch before it
    // finishes; it reads that launch's outputs only after griddepcontrol.wait
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)BH_of(d));
    cfg.blockDim = dim3(DECODE_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = (cudaStream_t)stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, (const VT*)v, alpha, beta, widx, ww, ridx, rw, st->M,
                           st->stamp, st->Lambda, (const float*)st->M0, out, d->H, (int)N_of(d),
                           d->d_v, d->W, d->R, (int)(d->decay == SDM_DECAY_TOUCHED)) != cudaSuccess)
        return SDM_ERR_CUDA;
    return launch_status();
}

sdm_status launch_score(const sdm_dims* d, const void* x, const void* sk, int top, int32_t* idx,
                        float* w, cudaStream_t s) {
    const long long rows = (long long)d->B * d->T;
    if (rows == 0) return SDM_OK;
    if (score_pk_eligible(d, top)) return launch_score_pk(d, 1, &x, &sk, &top, &idx, &w, s);
    if (score_tc_eligible(d, top)) return launch_score_tc(d, x, sk, top, idx, w, s);
    if (score_rows_eligible(d)) return launch_score_rows(d, 1, &x, &sk, &top, &idx, &w, s);
    const int threads = 128, warps = threads / 32;
    const size_t smem =
        (size_t)warps * score_simt_warp_floats(d->d_k, d->n_sub, d->k_half, top) * sizeof(float);
    long long gx = (rows + warps * 4 - 1) / (warps * 4);
    if (gx > 65535LL * 16) gx = 65535LL * 16;
    dim3 grid((unsigned)gx, (unsigned)d->H);
    if (d->x_dtype == SDM_F32) {
        if (!set_smem(score_simt_kernel<float>, smem)) return SDM_ERR_CUDA;
        score_simt_kernel<float><<<grid, threads, smem, s>>>(
            (const float*)x, (const float*)sk, d->B, d->H, d->T, d->d_k, d->n_sub, d->k_half, top,
            idx, w);
    } else {
        if (!set_smem(score_simt_kernel<__nv_bfloat16>, smem)) return SDM_ERR_CUDA;
        score_simt_kernel<__nv_bfloat16><<<grid, threads, smem, s>>>(
            (const __nv_bfloat16*)x, (const __nv_bfloat16*)sk, d->B, d->H, d->T, d->d_k, d->n_sub,
            d->k_half, top, idx, w);
    }
    return launch_status();
}

template <int CW, typename VT>
sdm_status launch_run_t(const sdm_dims* d, const WsLayout& L, const PlanPtrs& P, const void* v,
                        const float* beta, const int32_t* widx, const float* ww,
                        const int32_t* ridx, const float* rw, const sdm_state* st, float* out,
                        const RunEpi& ep, cudaStream_t s) {
    const size_t smem = run_smem_bytes(L.C, d->W, d->R, CW, (int)sizeof(VT));
    auto kern = ep.g ? recur_run_kernel<CW, VT, true> : recur_run_kernel<CW, VT, false>;
    if (!set_smem(kern, smem)) return SDM_ERR_CUDA;
    const long long grid = BH_of(d) * (d->d_v / CW);
    kern<<<(unsigned)grid, RUN_THREADS, smem, s>>>(
        (const VT*)v, P.rs, P.img, st->M, st->M0, out, d->H, d->T, (int)N_of(d), d->d_v,
        d->W, d->R, L.C, L.J, ep);
    return launch_status();
}

// ---- workspace of sdm_forward_noalloc: a fixed array in device memory -------------------
// Every GPU that loads the library holds this array until the process exits.
constexpr size_t kNoAllocWorkspaceBytes = size_t(64) << 20;  // 64 MiB
constexpr int kNoAllocMaxDevices = 64;

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_ws[kNoAllocWorkspaceBytes];

namespace {

std::mutex g_noalloc_mu;
struct NoAllocSlot {
    CUcontext ctx;  // the context the address belongs to
    void* ptr;
};
NoAllocSlot g_noalloc_slot[kNoAllocMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The driver's cuCtxGetCurrent, reached through the runtime (the library links no driver
// library); null when the driver does not offer it.
CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(f);
    });
    return fn;
}

CUcontext current_ctx() {
    CUcontext c = nullptr;
    const CtxGetCurrentFn fn = ctx_get_current();
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

// Device address of g_noalloc_ws in the current context.  In host code the array's name is
// only a host-side stand-in, so the address is looked up with the device current and cached
// per device together with the context it belongs to.  A device reset (or any teardown of the
// primary context) gives the device a new context, in which the library's module is loaded
// again and the array may sit elsewhere: the changed context makes the next call look the
// address up again instead of launching on the old one.
sdm_status noalloc_workspace(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return SDM_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return SDM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoAllocSlot& slot = g_noalloc_slot[dev];
    const CUcontext ctx = current_ctx();
    if (!slot.ptr || ctx == nullptr || ctx != slot.ctx) {
        void* p = nullptr;
        // also makes the device's primary context current if no call has yet
        if (cudaGetSymbolAddress(&p, g_noalloc_ws) != cudaSuccess || p == nullptr)
            return SDM_ERR_CUDA;
        slot.ptr = p;
        slot.ctx = current_ctx();
    }
    *out = slot.ptr;
    return SDM_OK;
}

}  // namespace

extern "C" {

const char* sdm_status_str(int32_t status) {
    switch (status) {
        case SDM_OK: return "SDM_OK";
        case SDM_ERR_ARG: return "SDM_ERR_ARG: null pointer or invalid argument";
        case SDM_ERR_SHAPE: return "SDM_ERR_SHAPE: dimensions outside the supported ranges";
        case SDM_ERR_DTYPE: return "SDM_ERR_DTYPE: unknown dtype";
        case SDM_ERR_ALIGN: return "SDM_ERR_ALIGN: pointer not 16-byte aligned";
        case SDM_ERR_CUDA: return "SDM_ERR_CUDA: CUDA runtime call failed";
        case SDM_ERR_BAD_INDEX: return "SDM_ERR_BAD_INDEX: device error word is set";
        case SDM_ERR_WORKSPACE: return "SDM_ERR_WORKSPACE: workspace missing or too small";
        case SDM_ERR_UNSUPPORTED: return "SDM_ERR_UNSUPPORTED: not implemented for these arguments";
        default: return "SDM_ERR_UNKNOWN";
    }
}

int32_t sdm_abi_version(void) { return 4; }

sdm_status sdm_state_bytes(const sdm_dims* dims, size_t* M_bytes, size_t* stamp_bytes,
                           size_t* lambda_bytes) {
    if (!M_bytes || !stamp_bytes || !lambda_bytes) return SDM_ERR_ARG;
    const sdm_status e = check_dims(dims);
    if (e) return e;
    const size_t BH = (size_t)BH_of(dims), N = (size_t)N_of(dims);
    *M_bytes = BH * N * dims->d_v * sizeof(float);
    *stamp_bytes = BH * N * sizeof(double);
    *lambda_bytes = BH * sizeof(double);
    return SDM_OK;
}

sdm_status sdm_state_reset(const sdm_dims* dims, const sdm_state* st, sdm_stream_t stream) {
    sdm_status e = check_dims(dims);
    if (e) return e;
    if ((e = check_state(st))) return e;
    const size_t n = (size_t)BH_of(dims) * N_of(dims);
    const int threads = 256;
    size_t blocks = (n / 2 + threads - 1) / threads;
    if (blocks > 148 * 32) blocks = 148 * 32;
    if (blocks < 1) blocks = 1;
    state_reset_kernel<<<(unsigned)blocks, threads, 0, stream>>>(st->stamp, n, st->Lambda,
                                                                 (int)BH_of(dims));
    return launch_status();
}

sdm_status sdm_state_materialize(const sdm_dims* dims, const sdm_state* st, float* M_out,
                                 sdm_stream_t stream) {
    sdm_status e = check_dims(dims);
    if (e) return e;
    if ((e = check_state(st))) return e;
    if (!M_out) return SDM_ERR_ARG;
    if (!aligned16(M_out)) return SDM_ERR_ALIGN;
    if (M_out == st->M) return SDM_ERR_ARG;
    const size_t rows = (size_t)BH_of(dims) * N_of(dims);
    const size_t total = rows * (dims->d_v / 4);
    const int threads = 256;
    size_t blocks = (total + threads - 1) / threads;
    if (blocks > 148 * 64) blocks = 148 * 64;
    state_materialize_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
        st->M, st->stamp, st->Lambda, st->M0, dims->H, (int)N_of(dims), dims->d_v, rows,
        (int)(dims->decay == SDM_DECAY_TOUCHED), M_out);
    return launch_status();
}

// Byte offsets of the call log's sections (rows, stamps, Lambda), 16-byte aligned.
struct CallLog {
    size_t rows, stamps, lam, total;
};
CallLog call_log_layout(const sdm_dims* d) {
    CallLog L{};
    const size_t occ = (size_t)BH_of(d) * (size_t)d->T * (size_t)d->W;
    L.rows = 0;
    L.stamps = up256(occ * (size_t)d->d_v * 4);
    L.lam = up256(L.stamps + occ * 8);
    L.total = up256(L.lam + (size_t)BH_of(d) * 8);
    return L;
}

size_t sdm_call_log_bytes(const sdm_dims* dims) {
    if (check_dims(dims) != SDM_OK) return 0;
    return call_log_layout(dims).total;
}

static sdm_status call_log(const sdm_dims* dims, const int32_t* widx, const sdm_state* st,
                           void* log, size_t log_bytes, bool save, sdm_stream_t stream) {
    sdm_status e = check_dims(dims);
    if (e) return e;
    if ((e = check_state(st))) return e;
    if (!widx || !log) return SDM_ERR_ARG;
    if (!aligned16(widx) || !aligned16(log)) return SDM_ERR_ALIGN;
    const CallLog L = call_log_layout(dims);
    if (log_bytes < L.total) return SDM_ERR_WORKSPACE;
    unsigned char* b = static_cast<unsigned char*>(log);
    const size_t occ = (size_t)BH_of(dims) * (size_t)dims->T * (size_t)dims->W;
    const size_t total = occ * (size_t)(dims->d_v / 4);
    const int threads = 256;
    size_t blocks = (total + threads - 1) / threads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks == 0) blocks = 1;
    auto kern = save ? call_log_kernel<true> : call_log_kernel<false>;
    kern<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(
        widx, st->M, st->stamp, st->Lambda, reinterpret_cast<float*>(b + L.rows),
        reinterpret_cast<double*>(b + L.stamps), reinterpret_cast<double*>(b + L.lam), occ,
        dims->T * dims->W, (int)N_of(dims), dims->d_v, (int)BH_of(dims));
    return launch_status();
}

sdm_status sdm_call_log_save(const sdm_dims* dims, const int32_t* widx, const sdm_state* st,
                             void* log, size_t log_bytes, sdm_stream_t stream) {
    return call_log(dims, widx, st, log, log_bytes, true, stream);
}

sdm_status sdm_call_log_restore(const sdm_dims* dims, const int32_t* widx, const void* log,
                                size_t log_bytes, const sdm_state* st, sdm_stream_t stream) {
    return call_log(dims, widx, st, const_cast<void*>(log), log_bytes, false, stream);
}

sdm_status sdm_score_topk(const sdm_dims* dims, const void* x, const void* subkeys, int32_t top,
                          int32_t* idx, float* w, sdm_stream_t stream) {
    const sdm_status e = check_dims(dims);
    if (e) return e;
    if (!x || !subkeys || !idx || !w) return SDM_ERR_ARG;
    if (top < 1 || top > kMaxTop || top > dims->k_half * dims->k_half) return SDM_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(subkeys) || !aligned16(idx) || !aligned16(w)) return SDM_ERR_ALIGN;
    return launch_score(dims, x, subkeys, top, idx, w, stream);
}

int32_t sdm_score_path(const sdm_dims* dims, int32_t top) {
    const sdm_status e = check_dims(dims);
    if (e) return -(int32_t)e;
    if (score_pk_eligible(dims, top)) return SDM_SCORE_TC;
    if (score_tc_eligible(dims, top)) return SDM_SCORE_TC;
    if (score_rows_eligible(dims)) return SDM_SCORE_ROWS;
    return SDM_SCORE_WARP;
}

int32_t sdm_decode_path(const sdm_dims* dims) {
    const sdm_status e = check_dims(dims);
    if (e) return -(int32_t)e;
    return decode_fused_eligible(dims) ? SDM_DECODE_FUSED : SDM_DECODE_TWO;
}

sdm_status sdm_score_qk(const sdm_dims* dims, const void* q, const void* k, const void* skw,
                        const void* skr, int32_t* widx, float* ww, int32_t* ridx, float* rw,
                        sdm_stream_t stream) {
    const sdm_status e = check_dims(dims);
    if (e) return e;
    return score_both_roles(dims, q, k, skw, skr, widx, ww, ridx, rw, (cudaStream_t)stream);
}

size_t sdm_forward_workspace_bytes(const sdm_dims* dims) {
    if (check_dims(dims) != SDM_OK) return 0;
    return ws_layout(dims).total;
}

sdm_status sdm_forward_plan(const sdm_dims* dims, const float* alpha, const float* beta,
                            const int32_t* widx, const float* ww, const int32_t* ridx,
                            const float* rw, const sdm_state* st, void* ws, size_t ws_bytes,
                            sdm_stream_t stream) {
    sdm_status e = check_dims(dims);
    if (e) return e;
    if ((e = check_state(st))) return e;
    if (dims->T == 0) return SDM_OK;
    if (!alpha || !beta || !widx || !ww || !ridx || !rw) return SDM_ERR_ARG;
    if (!aligned16(alpha) || !aligned16(beta) || !aligned16(widx) || !aligned16(ww) ||
        !aligned16(ridx) || !aligned16(rw))
        return SDM_ERR_ALIGN;
    const WsLayout L = ws_layout(dims);
    if (L.J > 32767) return SDM_ERR_SHAPE;  // chunk indices are 16-bit in the walk's table
    if (!ws || ws_bytes < L.total) return SDM_ERR_WORKSPACE;
    if (!aligned16(ws)) return SDM_ERR_ALIGN;
    const PlanPtrs P = plan_ptrs(L, ws);
    const int N = (int)N_of(dims);
    const size_t BH = (size_t)BH_of(dims);
    if (P.mask &&
        cudaMemsetAsync(P.mask, 0, BH * (size_t)N * L.MW * 8, stream) != cudaSuccess)
        return SDM_ERR_CUDA;
    const bool touched = dims->decay == SDM_DECAY_TOUCHED;
    auto local = touched ? plan_local_kernel<true> : plan_local_kernel<false>;
    if (!set_smem(local, plan_local_smem_bytes())) return SDM_ERR_CUDA;
    local<<<dim3((unsigned)L.J, (unsigned)BH), PLAN_THREADS, plan_local_smem_bytes(), stream>>>(
        alpha, beta, widx, ww, ridx, rw, st->stamp, dims->T, N, dims->W, dims->R, L.C, L.J, P);
    if ((e = launch_status())) return e;
    plan_prefix_kernel<<<(unsigned)BH, 1024, 0, stream>>>(st->Lambda, L.J, P);
    if ((e = launch_status())) return e;
    if (!P.mask) {  // factors as if unwritten in this call; the walk finishes them and the stamps
        plan_fe_kernel<<<dim3((unsigned)L.J, (unsigned)BH), PLAN_THREADS, 0, stream>>>(
            st->stamp, dims->T, N, dims->W, dims->R, L.C, L.J, P);
        if ((e = launch_status())) return e;
        if (cudaMemsetAsync(P.wtab, 0xff, BH * (size_t)N * 2, stream) != cudaSuccess)
            return SDM_ERR_CUDA;
        if (!set_smem(plan_walk_kernel, L.walk_smem)) return SDM_ERR_CUDA;
        plan_walk_kernel<<<dim3((unsigned)L.walk_parts, (unsigned)BH), WALK_THREADS, L.walk_smem,
                           stream>>>(st->stamp, dims->T, N, dims->W, dims->R, L.C, L.J,
                                     L.walk_parts, L.lstart_smem ? 1 : 0, P);
        if ((e = launch_status())) return e;
    }
    // with the masks, plan_pack computes the final factors and stamps itself
    auto pack = touched ? plan_pack_kernel<true> : plan_pack_kernel<false>;
    pack<<<dim3((unsigned)L.J, (unsigned)BH), PLAN_THREADS, 0, stream>>>(
        st->stamp, beta, widx, ww, ridx, rw, dims->T, N, dims->W, dims->R, L.C, L.J, P);
    return launch_status();
}

}  // extern "C"

namespace {

// The row pass, with the layer epilogue when ep.g is set.
sdm_status forward_run_impl(const sdm_dims* dims, const void* v, const float* beta,
                            const int32_t* widx, const float* ww, const int32_t* ridx,
                            const float* rw, const sdm_state* st, float* out, RunEpi ep, void* ws,
                            size_t ws_bytes, cudaStream_t stream) {
    sdm_status e = check_dims(dims);
    if (e) return e;
    if ((e = check_state(st))) return e;
    if (dims->T == 0) return SDM_OK;
    if (!v || !beta || !widx || !ww || !ridx || !rw || !out) return SDM_ERR_ARG;
    if (!aligned16(v) || !aligned16(beta) || !aligned16(widx) || !aligned16(ww) ||
        !aligned16(ridx) || !aligned16(rw) || !aligned16(out))
        return SDM_ERR_ALIGN;
    const WsLayout L = ws_layout(dims);
    if (!ws || ws_bytes < L.total) return SDM_ERR_WORKSPACE;
    if (!aligned16(ws)) return SDM_ERR_ALIGN;
    const PlanPtrs P = plan_ptrs(L, ws);
    if (ep.g) {
        ep.cnt = reinterpret_cast<int*>(static_cast<unsigned char*>(ws) + L.off_cnt);
        if (cudaMemsetAsync(ep.cnt, 0, (size_t)BH_of(dims) * L.J * 4, stream) != cudaSuccess)
            return SDM_ERR_CUDA;
    }
    const int CW = col_width(dims);
    if (CW == 16) {
        if (dims->v_dtype == SDM_BF16)
            return launch_run_t<16, __nv_bfloat16>(dims, L, P, v, beta, widx, ww, ridx, rw, st, out, ep, stream);
        return launch_run_t<16, float>(dims, L, P, v, beta, widx, ww, ridx, rw, st, out, ep, stream);
    }
    if (CW == 8) {
        if (dims->v_dtype == SDM_BF16)
            return launch_run_t<8, __nv_bfloat16>(dims, L, P, v, beta, widx, ww, ridx, rw, st, out, ep, stream);
        return launch_run_t<8, float>(dims, L, P, v, beta, widx, ww, ridx, rw, st, out, ep, stream);
    }
    if (dims->v_dtype == SDM_BF16)
        return launch_run_t<4, __nv_bfloat16>(dims, L, P, v, beta, widx, ww, ridx, rw, st, out, ep, stream);
    return launch_run_t<4, float>(dims, L, P, v, beta, widx, ww, ridx, rw, st, out, ep, stream);
}

}  // namespace

extern "C" {

sdm_status sdm_forward_run(const sdm_dims* dims, const void* v, const float* beta,
                           const int32_t* widx, const float* ww, const int32_t* ridx,
                           const float* rw, const sdm_state* st, float* out, void* ws,
                           size_t ws_bytes, sdm_stream_t stream) {
    return forward_run_impl(dims, v, beta, widx, ww, ridx, rw, st, out, RunEpi{}, ws, ws_bytes,
                            (cudaStream_t)stream);
}

sdm_status sdm_forward_run_gated(const sdm_dims* dims, const void* v, const float* beta,
                                 const int32_t* widx, const float* ww, const int32_t* ridx,
                                 const float* rw, const sdm_state* st, float* out, const void* g,
                                 const float* wn, float eps, void* a, void* ws, size_t ws_bytes,
                                 sdm_stream_t stream) {
    if (!g || !wn || !a) return SDM_ERR_ARG;
    if (!(eps >= 0.f)) return SDM_ERR_ARG;
    if (!aligned16(g) || !aligned16(wn) || !aligned16(a)) return SDM_ERR_ALIGN;
    RunEpi ep{};
    ep.g = static_cast<const __nv_bfloat16*>(g);
    ep.wn = wn;
    ep.eps = eps;
    ep.a = static_cast<__nv_bfloat16*>(a);
    return forward_run_impl(dims, v, beta, widx, ww, ridx, rw, st, out, ep, ws, ws_bytes,
                            (cudaStream_t)stream);
}

sdm_status sdm_forward(const sdm_dims* dims, const void* v, const float* alpha, const float* beta,
                       const int32_t* widx, const float* ww, const int32_t* ridx, const float* rw,
                       const sdm_state* st, float* out, void* ws, size_t ws_bytes,
                       sdm_stream_t stream) {
    sdm_status e = check_dims(dims);
    if (e) return e;
    if ((e = check_state(st))) return e;
    if (dims->T == 0) return SDM_OK;
    if (!v || !alpha || !beta || !widx || !ww || !ridx || !rw || !out) return SDM_ERR_ARG;
    const WsLayout L = ws_layout(dims);
    if (!ws || ws_bytes < L.total) return SDM_ERR_WORKSPACE;
    if ((e = sdm_forward_plan(dims, alpha, beta, widx, ww, ridx, rw, st, ws, ws_bytes, stream)))
        return e;
    return sdm_forward_run(dims, v, beta, widx, ww, ridx, rw, st, out, ws, ws_bytes, stream);
}

sdm_status sdm_prefill(const sdm_dims* dims, const void* q, const void* k, const void* v,
                       const float* alpha, const float* beta, const void* skw, const void* skr,
                       const sdm_state* st, int32_t* widx, float* ww, int32_t* ridx, float* rw,
                       float* out, void* ws, size_t ws_bytes, sdm_stream_t stream) {
    sdm_status e = check_dims(dims);
    if (e) return e;
    if ((e = check_state(st))) return e;
    if (dims->T == 0) return SDM_OK;
    if (!q || !k || !v || !alpha || !beta || !skw || !skr || !widx || !ww || !ridx || !rw || !out)
        return SDM_ERR_ARG;
    const WsLayout L = ws_layout(dims);
    if (!ws || ws_bytes < L.total) return SDM_ERR_WORKSPACE;
    if ((e = score_both_roles(dims, q, k, skw, skr, widx, ww, ridx, rw, stream))) return e;
    return sdm_forward(dims, v, alpha, beta, widx, ww, ridx, rw, st, out, ws, ws_bytes, stream);
}

sdm_status sdm_decode_step(const sdm_dims* dims, const void* q, const void* k, const void* v,
                           const float* alpha, const float* beta, const void* skw,
                           const void* skr, const sdm_state* st, int32_t* widx, float* ww,
                           int32_t* ridx, float* rw, float* out, sdm_stream_t stream) {
    sdm_status e = check_dims(dims);
    if (e) return e;
    if (dims->T != 1) return SDM_ERR_SHAPE;
    if ((e = check_state(st))) return e;
    if (!q || !k || !v || !alpha || !beta || !skw || !skr || !widx || !ww || !ridx || !rw || !out)
        return SDM_ERR_ARG;
    if (!aligned16(v) || !aligned16(alpha) || !aligned16(beta) || !aligned16(out))
        return SDM_ERR_ALIGN;
    if (decode_fused_eligible(dims)) {
        if (!aligned16(q) || !aligned16(k) || !aligned16(skw) || !aligned16(skr) ||
            !aligned16(widx) || !aligned16(ww) || !aligned16(ridx) || !aligned16(rw))
            return SDM_ERR_ALIGN;
        if (dims->B == 0) return SDM_OK;
        return launch_decode_fused(dims, q, k, v, alpha, beta, skw, skr, st, widx, ww, ridx, rw,
                                   out, (cudaStream_t)stream);
    }
    if ((e = score_both_roles(dims, q, k, skw, skr, widx, ww, ridx, rw, stream))) return e;
    const int rpw = ((dims->W > dims->R ? dims->W : dims->R) + DECODE_WARPS - 1) / DECODE_WARPS;
    const int qpl = (dims->d_v / 4 + 31) / 32;
    if (dims->v_dtype == SDM_BF16) {
        if (rpw <= 4) e = qpl <= 1 ? launch_decode<__nv_bfloat16, 4, 1>(dims, v, alpha, beta, st, widx, ww, ridx, rw, out, stream)
                                   : launch_decode<__nv_bfloat16, 4, 2>(dims, v, alpha, beta, st, widx, ww, ridx, rw, out, stream);
        else e = qpl <= 1 ? launch_decode<__nv_bfloat16, 8, 1>(dims, v, alpha, beta, st, widx, ww, ridx, rw, out, stream)
                          : launch_decode<__nv_bfloat16, 8, 2>(dims, v, alpha, beta, st, widx, ww, ridx, rw, out, stream);
    } else {
        if (rpw <= 4) e = qpl <= 1 ? launch_decode<float, 4, 1>(dims, v, alpha, beta, st, widx, ww, ridx, rw, out, stream)
                                   : launch_decode<float, 4, 2>(dims, v, alpha, beta, st, widx, ww, ridx, rw, out, stream);
        else e = qpl <= 1 ? launch_decode<float, 8, 1>(dims, v, alpha, beta, st, widx, ww, ridx, rw, out, stream)
                          : launch_decode<float, 8, 2>(dims, v, alpha, beta, st, widx, ww, ridx, rw, out, stream);
    }
    return e;
}

sdm_status sdm_score_backward(const sdm_dims* dims, const void* x, const void* subkeys,
                              int32_t top, const int32_t* idx, const float* w, const float* dw,
                              float* dx, float* dsubkeys, sdm_stream_t stream) {
    const sdm_status e = check_dims(dims);
    if (e) return e;
    if (!x || !subkeys || !idx || !w || !dw || !dx || !dsubkeys) return SDM_ERR_ARG;
    if (top < 1 || top > kMaxTop || top > dims->k_half * dims->k_half) return SDM_ERR_SHAPE;
    if ((long long)dims->B * dims->T == 0) return SDM_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if (dims->x_dtype == SDM_F32)
        return launch_score_bwd_x<float>(dims, x, subkeys, top, idx, w, dw, dx, dsubkeys, s);
    return launch_score_bwd_x<__nv_bfloat16>(dims, x, subkeys, top, idx, w, dw, dx, dsubkeys, s);
}

size_t sdm_backward_workspace_bytes(const sdm_dims* dims) {
    if (check_dims(dims) != SDM_OK) return 0;
    return bwd_layout(dims).total;
}

sdm_status sdm_backward(const sdm_dims* dims, const void* v, const float* alpha, const float* beta,
                        const int32_t* widx, const float* ww, const int32_t* ridx, const float* rw,
                        const sdm_state* st, const float* dout, const float* dM_end, float* dv,
                        float* dalpha, float* dbeta, float* dww, float* drw, float* dM_in,
                        void* ws, size_t ws_bytes, sdm_stream_t stream) {
    sdm_status e = check_dims(dims);
    if (e) return e;
    if ((e = check_state(st))) return e;
    if (!v || !alpha || !beta || !widx || !ww || !ridx || !rw || !dout || !dv || !dalpha ||
        !dbeta || !dww || !drw || !dM_in)
        return SDM_ERR_ARG;
    if (!aligned16(v) || !aligned16(dout) || !aligned16(dv) || !aligned16(dM_in) ||
        (dM_end && !aligned16(dM_end)))
        return SDM_ERR_ALIGN;
    if (dims->W + dims->R > BWD_MAXO) return SDM_ERR_SHAPE;
    const BwdLayout L = bwd_layout(dims);
    if (!ws || ws_bytes < L.total) return SDM_ERR_WORKSPACE;
    if (!aligned16(ws)) return SDM_ERR_ALIGN;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t rows = (size_t)BH_of(dims) * (size_t)N_of(dims);
    const int S = bwd_slices(dims);
    if ((size_t)BH_of(dims) * S > 0x7fffffffull) return SDM_ERR_SHAPE;
    unsigned char* b = static_cast<unsigned char*>(ws);
    BwdPtrs P;
    P.log_rows = reinterpret_cast<float*>(b + L.off_rows);
    P.log_stamp = reinterpret_cast<double*>(b + L.off_lstamp);
    P.log_lam = reinterpret_cast<double*>(b + L.off_lam);
    P.dM = reinterpret_cast<float*>(b + L.off_dM);
    P.pst = reinterpret_cast<double*>(b + L.off_pst);
    P.pds = reinterpret_cast<double*>(b + L.off_pds);
    P.p_dww = reinterpret_cast<float*>(b + L.off_pdww);
    P.p_drw = reinterpret_cast<float*>(b + L.off_pdrw);
    P.p_db = reinterpret_cast<double*>(b + L.off_pdb);
    P.p_da = reinterpret_cast<double*>(b + L.off_pda);
    P.gam = reinterpret_cast<double*>(b + L.off_gam);
    P.rpart = reinterpret_cast<int8_t*>(b + L.off_rpart);
    P.x0 = reinterpret_cast<double*>(b + L.off_x0);
    const int threads = 256;
    auto grid_for = [](size_t n) {
        size_t blocks = (n + 255) / 256;
        if (blocks > 148 * 64) blocks = 148 * 64;
        return (unsigned)(blocks == 0 ? 1 : blocks);
    };
    // private stamp copies per slice, every memory-gradient row at zero (NaN stamp)
    bwd_init_kernel<<<grid_for((size_t)S * rows), threads, 0, s>>>(st->stamp, P, rows, S,
                                                                   (int)BH_of(dims), dM_end,
                                                                   dims->d_v);
    if (dims->T > 0) {
        const size_t BHT = (size_t)BH_of(dims) * dims->T;
        bwd_links_kernel<<<grid_for(BHT * dims->W), threads, 0, s>>>(widx, ridx, BHT, dims->W,
                                                                     dims->R, P.rpart);
        const int m = dims->W > dims->R ? dims->W : dims->R;
#define SDM_BWD(VT, K) launch_backward_t<VT, K>(dims, P, v, alpha, beta, widx, ww, ridx, rw, st, dout, dM_end, dv, s)
        if (dims->v_dtype == SDM_BF16) {
            e = m <= 32 ? SDM_BWD(__nv_bfloat16, 1) : m <= 64 ? SDM_BWD(__nv_bfloat16, 2)
                                                    : SDM_BWD(__nv_bfloat16, 4);
        } else {
            e = m <= 32 ? SDM_BWD(float, 1) : m <= 64 ? SDM_BWD(float, 2) : SDM_BWD(float, 4);
        }
#undef SDM_BWD
        if (e) return e;
        bwd_reduce_kernel<<<grid_for(BHT * (dims->W + dims->R + 2)), threads, 0, s>>>(
            P, S, BHT, dims->W, dims->R, dww, drw, dbeta, dalpha);
    }
    bwd_dense_kernel<<<grid_for(rows * (dims->d_v / 4)), threads, 0, s>>>(P, (int)N_of(dims),
                                                                          dims->d_v, rows, dM_in);
    return launch_status();
}

sdm_status sdm_forward_noalloc(const sdm_dims* dims, const void* v, const float* alpha,
                               const float* beta, const int32_t* widx, const float* ww,
                               const int32_t* ridx, const float* rw, const sdm_state* st,
                               float* out, sdm_stream_t stream) {
    sdm_status e = check_dims(dims);
    if (e) return e;
    if ((e = check_state(st))) return e;
    if (dims->T == 0) return SDM_OK;
    if (!v || !alpha || !beta || !widx || !ww || !ridx || !rw || !out) return SDM_ERR_ARG;
    const WsLayout L = ws_layout(dims);
    if (L.total > kNoAllocWorkspaceBytes) return SDM_ERR_WORKSPACE;
    void* ws = nullptr;
    if ((e = noalloc_workspace(&ws))) return e;
    return sdm_forward(dims, v, alpha, beta, widx, ww, ridx, rw, st, out, ws,
                       kNoAllocWorkspaceBytes, stream);
}

sdm_status sdm_gemm_bf16(int32_t M, int32_t N, int32_t K, const void* A, const void* Bt, float* C,
                         sdm_stream_t stream) {
    if (M < 1 || N < 1 || K < 8 || K % 8 != 0) return SDM_ERR_SHAPE;
    if (!A || !Bt || !C) return SDM_ERR_ARG;
    if (!aligned16(A) || !aligned16(Bt) || !aligned16(C)) return SDM_ERR_ALIGN;
    if ((long long)((M + GEMM_BM - 1) / GEMM_BM) * ((N + GEMM_BN - 1) / GEMM_BN) > 0x7fffffffLL)
        return SDM_ERR_SHAPE;
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return SDM_ERR_CUDA;
    CUtensorMap am, bm;
    const cuuint32_t es[2] = {1, 1};
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {GEMM_BK, GEMM_BM};
        if (enc(&am, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(A), dims, strides, box,
                es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return SDM_ERR_CUDA;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {GEMM_BK, GEMM_BN};
        if (enc(&bm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(Bt), dims, strides, box,
                es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return SDM_ERR_CUDA;
    }
    // C by TMA stores when its rows are 16-byte multiples
    CUtensorMap cm;
    memset(&cm, 0, sizeof(cm));
    int cm_ok = 0;
    if (N % 4 == 0) {
        const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
        const cuuint64_t strides[1] = {(cuuint64_t)N * 4};
        const cuuint32_t box[2] = {32, 32};  // one epilogue warp's 32 rows x 32 columns
        cm_ok = enc(&cm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, C, dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    auto kern = gemm_bf16_tc_kernel;
    const uint32_t smem = GEMM_SMEM_BYTES;
    if (!set_smem(kern, smem)) return SDM_ERR_CUDA;
    // persistent: one CTA per SM (or per tile, when there are fewer tiles)
    const long long tiles = (long long)((M + GEMM_BM - 1) / GEMM_BM) * ((N + GEMM_BN - 1) / GEMM_BN);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return SDM_ERR_CUDA;
    const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
    kern<<<grid, GEMM_THREADS, smem, stream>>>(am, bm, cm, cm_ok, C, M, N, K);
    return launch_status();
}

size_t sdm_layer_in_workspace_bytes(const sdm_dims* dims) {
    if (check_dims(dims) != SDM_OK) return 0;
    const size_t hs = (size_t)(2 * dims->d_k + 2 * dims->d_v + 2);
    return (size_t)dims->B * dims->T * dims->H * hs * 4;
}

sdm_status sdm_layer_in(const sdm_dims* dims, const void* x, const void* Win_t,
                        const float* A_log, const float* dt_bias, int32_t d_model, void* q,
                        void* k, void* v, void* g, float* alpha, float* beta, void* ws,
                        size_t ws_bytes, sdm_stream_t stream) {
    sdm_status e = check_dims(dims);
    if (e) return e;
    if (dims->T == 0) return SDM_OK;
    if (dims->x_dtype != SDM_BF16) return SDM_ERR_DTYPE;  // q, k are written as bf16
    if (!x || !Win_t || !A_log || !dt_bias || !q || !k || !v || !g || !alpha || !beta)
        return SDM_ERR_ARG;
    if (d_model < 8 || d_model % 8 != 0) return SDM_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(Win_t) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
        !aligned16(g) || !aligned16(alpha) || !aligned16(beta))
        return SDM_ERR_ALIGN;
    const size_t need = sdm_layer_in_workspace_bytes(dims);
    if (!ws || ws_bytes < need) return SDM_ERR_WORKSPACE;
    if (!aligned16(ws)) return SDM_ERR_ALIGN;
    const long long rows = (long long)dims->B * dims->T;
    const int Nin = dims->H * (2 * dims->d_k + 2 * dims->d_v + 2);
    if (rows > 0x7fffffffLL) return SDM_ERR_SHAPE;
    float* P = static_cast<float*>(ws);
    if ((e = sdm_gemm_bf16((int32_t)rows, Nin, d_model, x, Win_t, P, stream))) return e;
    const long long total = rows * Nin;
    long long blocks = (total + LAYER_THREADS - 1) / LAYER_THREADS;
    if (blocks > 148LL * 64) blocks = 148LL * 64;
    if (dims->v_dtype == SDM_BF16)
        layer_in_split_kernel<__nv_bfloat16><<<(unsigned)blocks, LAYER_THREADS, 0, stream>>>(
            P, A_log, dt_bias, dims->B, dims->H, dims->T, dims->d_k, dims->d_v,
            static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k),
            static_cast<__nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(g), alpha, beta);
    else
        layer_in_split_kernel<float><<<(unsigned)blocks, LAYER_THREADS, 0, stream>>>(
            P, A_log, dt_bias, dims->B, dims->H, dims->T, dims->d_k, dims->d_v,
            static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k),
            static_cast<float*>(v), static_cast<__nv_bfloat16*>(g), alpha, beta);
    return launch_status();
}

size_t sdm_layer_out_workspace_bytes(const sdm_dims* dims) {
    if (check_dims(dims) != SDM_OK) return 0;
    return (size_t)dims->B * dims->T * dims->H * dims->d_v * 2;
}

sdm_status sdm_layer_out(const sdm_dims* dims, const float* o, const void* g, const float* wn,
                         float eps, const void* Wo_t, int32_t d_model, float* y, void* ws,
                         size_t ws_bytes, sdm_stream_t stream) {
    sdm_status e = check_dims(dims);
    if (e) return e;
    if (dims->T == 0) return SDM_OK;
    if (!o || !g || !wn || !Wo_t || !y) return SDM_ERR_ARG;
    if (!(eps >= 0.f) || d_model < 1) return SDM_ERR_ARG;
    const int K = dims->H * dims->d_v;
    if (K % 8 != 0) return SDM_ERR_SHAPE;
    if (!aligned16(o) || !aligned16(g) || !aligned16(wn) || !aligned16(Wo_t) || !aligned16(y))
        return SDM_ERR_ALIGN;
    const size_t need = sdm_layer_out_workspace_bytes(dims);
    if (!ws || ws_bytes < need) return SDM_ERR_WORKSPACE;
    if (!aligned16(ws)) return SDM_ERR_ALIGN;
    const long long rows = (long long)dims->B * dims->T;
    if (rows > 0x7fffffffLL) return SDM_ERR_SHAPE;
    __nv_bfloat16* a = static_cast<__nv_bfloat16*>(ws);
    const long long warps = rows * dims->H;
    const long long blocks = (warps * 32 + LAYER_THREADS - 1) / LAYER_THREADS;
    const int per = (dims->d_v + 31) / 32;
    const __nv_bfloat16* gb = static_cast<const __nv_bfloat16*>(g);
    if (per <= 1)
        layer_prologue_kernel<1><<<(unsigned)blocks, LAYER_THREADS, 0, stream>>>(
            o, gb, wn, eps, dims->B, dims->H, dims->T, dims->d_v, a);
    else if (per <= 2)
        layer_prologue_kernel<2><<<(unsigned)blocks, LAYER_THREADS, 0, stream>>>(
            o, gb, wn, eps, dims->B, dims->H, dims->T, dims->d_v, a);
    else if (per <= 4)
        layer_prologue_kernel<4><<<(unsigned)blocks, LAYER_THREADS, 0, stream>>>(
            o, gb, wn, eps, dims->B, dims->H, dims->T, dims->d_v, a);
    else
        layer_prologue_kernel<8><<<(unsigned)blocks, LAYER_THREADS, 0, stream>>>(
            o, gb, wn, eps, dims->B, dims->H, dims->T, dims->d_v, a);
    if ((e = launch_status())) return e;
    return sdm_gemm_bf16((int32_t)rows, d_model, K, a, Wo_t, y, stream);
}

size_t sdm_weight_stats_workspace_bytes(int64_t rows, int32_t K) {
    if (rows < 1 || K < 1 || K > STATS_MAXK) return 0;
    const size_t blocks = (size_t)((rows + STATS_THREADS - 1) / STATS_THREADS);
    return blocks * (size_t)(K + 1) * sizeof(float);
}

sdm_status sdm_weight_stats(int64_t rows, int32_t K, const float* w, float* cum, float* eff,
                            float* mean, int32_t nprobs, const double* probs, float* quant,
                            void* ws, size_t ws_bytes, sdm_stream_t stream) {
    if (rows < 1 || K < 1 || K > STATS_MAXK) return SDM_ERR_SHAPE;
    if (nprobs < 0 || nprobs > STATS_MAXP) return SDM_ERR_ARG;
    if (!w || !eff || !mean || (nprobs > 0 && (!probs || !quant))) return SDM_ERR_ARG;
    const uintptr_t a = (uintptr_t)w | (uintptr_t)eff | (uintptr_t)mean | (uintptr_t)cum |
                        (uintptr_t)quant | (uintptr_t)ws;
    if (a & 3u) return SDM_ERR_ALIGN;
    StatsProbs P{};
    for (int q = 0; q < nprobs; ++q) {
        if (!(probs[q] >= 0.0 && probs[q] <= 1.0)) return SDM_ERR_ARG;
        P.p[q] = probs[q];
    }
    const size_t need = sdm_weight_stats_workspace_bytes(rows, K);
    if (!ws || ws_bytes < need) return SDM_ERR_WORKSPACE;
    const long long blocks = (rows + STATS_THREADS - 1) / STATS_THREADS;
    if (blocks > 0x7fffffffLL) return SDM_ERR_SHAPE;
    float* part = static_cast<float*>(ws);
    weight_stats_rows_kernel<<<(unsigned)blocks, STATS_THREADS, 0, stream>>>(w, rows, K, cum,
                                                                            eff, part);
    sdm_status e = launch_status();
    if (e) return e;
    weight_stats_summary_kernel<<<1, 1024, 0, stream>>>(part, (int)blocks, rows, K, eff, mean,
                                                        nprobs, P, quant);
    return launch_status();
}

sdm_status sdm_device_error(uint32_t* bits, int32_t clear, sdm_stream_t stream) {
    if (!bits) return SDM_ERR_ARG;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_err, sizeof(v), 0, cudaMemcpyDeviceToHost, stream) !=
        cudaSuccess)
        return SDM_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return SDM_ERR_CUDA;
    if (clear) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbolAsync(g_err, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice,
                                    stream) != cudaSuccess)
            return SDM_ERR_CUDA;
        if (cudaStreamSynchronize(stream) != cudaSuccess) return SDM_ERR_CUDA;
    }
    *bits = v;
    return v ? SDM_ERR_BAD_INDEX : SDM_OK;
}

}  // extern "C"
