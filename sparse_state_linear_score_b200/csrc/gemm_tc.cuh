// Dense bf16 GEMM on the 5th-generation tensor cores: C[M][N] (fp32) = A[M][K] x B[N][K]^T,
// A and B bf16 and K-contiguous, accumulation in fp32 in TMEM.
//
// Persistent and warp-specialised: one CTA per SM walks the 128 x 256 output tiles
// blockIdx.x, blockIdx.x + gridDim.x, ... (n fastest, so the CTAs running together take every
// column block of a few row blocks: each A block is read from memory about once while the B
// blocks stay in L2).  Its six warps take three roles:
//   warp 0      (one lane) TMA producer: the A and B K-blocks (64 wide, 128-byte swizzle) of
//               every tile into a GEMM_STAGES-deep ring; full[s] completes on the bytes,
//               empty[s] is the MMA's release of the stage.
//   warp 1      (one lane) MMA issuer: four tcgen05.mma (K = 16 each) per K-block into one of
//               two 256-column TMEM accumulators; a commit frees each stage, a commit per
//               tile signals tfull[acc]; before a tile it waits tempty[acc], the epilogue's
//               release of that accumulator's previous tile.
//   warps 2..5  epilogue, each warp on its own: TMEM lanes 32 (w % 4) .. + 31 are its 32
//               tile rows; 32 columns at a time into its 32 x 32 fp32 staging tile (the
//               128-byte swizzle: 16-byte chunk index XOR row % 8, conflict-free writes),
//               stored by one TMA store (GEMM_WBUF staging tiles per warp in flight); then an
//               arrival on tempty[acc] (four per tile).
// So a tile's epilogue overlaps the next tile's MMAs, and the loads run ahead of both.
// Without a C tensor map (N not a multiple of 4) the epilogue threads store their rows
// directly.  Every wait is bounded; on timeout the device error word gets
// SDM_DEVERR_TIMEOUT and the CTA stops issuing work.
//
// Loads past M, N or K read zeros (TMA bounds), stores are clipped or guarded, so M and N are
// free; K must be a multiple of 8 (16-byte rows).
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace sdm {

constexpr int GEMM_THREADS = 192;
constexpr int GEMM_BM = 128;
constexpr int GEMM_BN = 256;
constexpr int GEMM_BK = 64;
constexpr uint32_t GEMM_A_BYTES = GEMM_BM * GEMM_BK * 2;  // 16 KB
constexpr uint32_t GEMM_B_BYTES = GEMM_BN * GEMM_BK * 2;  // 32 KB
constexpr uint32_t GEMM_STAGE_BYTES = GEMM_A_BYTES + GEMM_B_BYTES;
constexpr uint32_t GEMM_WSTG_BYTES = 32 * 32 * 4;  // one warp's 32 x 32 fp32 staging tile

constexpr int GEMM_STAGES = 4;  // operand ring (more stores in flight instead measured slower)
constexpr int GEMM_WBUF = 2;    // staging tiles per epilogue warp
constexpr uint32_t GEMM_OFF_STG = GEMM_STAGES * GEMM_STAGE_BYTES;
constexpr uint32_t GEMM_OFF_CTRL = GEMM_OFF_STG + 4 * GEMM_WBUF * GEMM_WSTG_BYTES;
constexpr uint32_t GEMM_SMEM_BYTES = GEMM_OFF_CTRL + 128 + 1024;
static_assert(GEMM_SMEM_BYTES <= 232448, "one CTA per SM");

SDM_DEV void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(ptx::smem_u32(bar)) : "memory");
}

__global__ void __launch_bounds__(GEMM_THREADS, 1) gemm_bf16_tc_kernel(
    const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
    const __grid_constant__ CUtensorMap cmap, int cmap_ok, float* __restrict__ C, int M, int N,
    int K) {
    extern __shared__ unsigned char gemm_smem_raw[];
    unsigned char* sm =
        gemm_smem_raw + ((1024 - (ptx::smem_u32(gemm_smem_raw) & 1023)) & 1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + GEMM_OFF_CTRL);
    uint64_t* empty = full + GEMM_STAGES;
    uint64_t* tfull = empty + GEMM_STAGES;  // [2]
    uint64_t* tempty = tfull + 2;           // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int num_m = (M + GEMM_BM - 1) / GEMM_BM, num_n = (N + GEMM_BN - 1) / GEMM_BN;
    const int tiles = num_m * num_n;
    const int nk = (K + GEMM_BK - 1) / GEMM_BK;

    if (warp == 1) ptx::tmem_alloc(tmem_slot, 2 * GEMM_BN);
    if (tid == 0) {
        for (int s = 0; s < GEMM_STAGES; ++s) {
            ptx::mbar_init(full + s, 1);
            ptx::mbar_init(empty + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(tfull + a, 1);
            ptx::mbar_init(tempty + a, 4);  // one arrival per epilogue warp
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t deadline = ptx::globaltimer_ns() + 4000000000ull;
    auto fail = [&]() {
        *abort_flag = 1;
        raise_err(SDM_DEVERR_TIMEOUT);
    };

    if (warp == 0 && lane == 0) {
        // ---- producer ----
        uint32_t it = 0;
        for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
            const int m0 = (t / num_n) * GEMM_BM, n0 = (t % num_n) * GEMM_BN;
            for (int kb = 0; kb < nk; ++kb, ++it) {
                const uint32_t s = it % GEMM_STAGES, use = it / GEMM_STAGES;
                if (use > 0 && !ptx::mbar_wait_bounded(empty + s, (use - 1) & 1u, deadline)) {
                    fail();
                    break;
                }
                unsigned char* st = sm + s * GEMM_STAGE_BYTES;
                ptx::mbar_arrive_expect_tx(full + s, GEMM_STAGE_BYTES);
                ptx::tma_load_2d(st, &amap, kb * GEMM_BK, m0, full + s);
                ptx::tma_load_2d(st + GEMM_A_BYTES, &bmap, kb * GEMM_BK, n0, full + s);
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer ----
        const uint32_t idesc = ptx::idesc_bf16_f32(GEMM_BM, GEMM_BN);
        uint32_t it = 0, lt = 0;
        for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x, ++lt) {
            const uint32_t acc = lt & 1u, use = lt >> 1;
            if (use > 0 && !ptx::mbar_wait_bounded(tempty + acc, (use - 1) & 1u, deadline)) {
                fail();
                break;
            }
            ptx::tc_fence_after();
            const uint32_t d = tmem + acc * GEMM_BN;
            bool ok = true;
            for (int kb = 0; kb < nk; ++kb, ++it) {
                const uint32_t s = it % GEMM_STAGES;
                if (!ptx::mbar_wait_bounded(full + s, (it / GEMM_STAGES) & 1u, deadline)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                unsigned char* st = sm + s * GEMM_STAGE_BYTES;
                const uint64_t ad = ptx::umma_desc_kmajor_sw128(st);
                const uint64_t bd = ptx::umma_desc_kmajor_sw128(st + GEMM_A_BYTES);
#pragma unroll
                for (int k = 0; k < GEMM_BK / 16; ++k)  // 16 bf16 = 32 bytes per step
                    ptx::umma_bf16(d, ad + 2 * k, bd + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
                ptx::umma_commit(empty + s);
            }
            if (!ok) {
                fail();
                break;
            }
            ptx::umma_commit(tfull + acc);
        }
    } else if (warp >= 2) {
        // ---- epilogue: each warp on its own (its 32 rows, its staging tiles and stores) ----
        const int q = warp & 3;  // TMEM lane quadrant of this warp = its rows of the tile
        unsigned char* wst = sm + GEMM_OFF_STG + (warp - 2) * GEMM_WBUF * GEMM_WSTG_BYTES;
        uint32_t lt = 0, gc = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
            const uint32_t acc = lt & 1u, use = lt >> 1;
            int go = 0;
            if (lane == 0) go = !*abort_flag && ptx::mbar_wait_bounded(tfull + acc, use & 1u, deadline);
            go = __shfl_sync(0xffffffffu, go, 0);
            if (!go) {
                if (lane == 0 && !*abort_flag) fail();
                break;
            }
            ptx::tc_fence_after();
            const int m0 = (t / num_n) * GEMM_BM, n0 = (t % num_n) * GEMM_BN;
            const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + acc * GEMM_BN;
            for (int c = 0; c < GEMM_BN; c += 32, ++gc) {
                float v[32];
                if (cmap_ok) {
                    unsigned char* tile = wst + (gc % GEMM_WBUF) * GEMM_WSTG_BYTES;
                    if (lane == 0 && gc >= GEMM_WBUF) ptx::bulk_wait_group_read<GEMM_WBUF - 1>();
                    __syncwarp();
                    ptx::tmem_ld32(trow + c, v);
                    unsigned char* rowp = tile + lane * 128;
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<float4*>(rowp + ((j ^ (lane & 7)) << 4)) =
                            make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        ptx::tma_store_2d(&cmap, n0 + c, m0 + q * 32, tile);
                        ptx::bulk_commit_group();
                    }
                } else {
                    ptx::tmem_ld32(trow + c, v);
                    const int row = m0 + q * 32 + lane;
                    if (row < M) {
                        float* dst = C + (size_t)row * N + n0 + c;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (n0 + c + i < N) dst[i] = v[i];
                    }
                }
            }
            // every TMEM read of this accumulator has completed (tmem_ld32 waits): release it
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty + acc);
        }
        if (lane == 0) ptx::bulk_wait_group_read<0>();  // staging read before the CTA exits
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 2 * GEMM_BN);
    }
}

}  // namespace sdm
