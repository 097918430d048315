// Dense bf16 GEMM on the 5th-generation tensor cores: C[M][N] (fp32) = A[M][K] x B[N][K]^T,
// A and B bf16 and K-contiguous, accumulation in fp32 in TMEM.
//
// One CTA computes a 128 x GEMM_BN tile.  Thread 0 runs a GEMM_STAGES-deep pipeline: TMA
// loads of the A and B K-blocks (64 wide, 128-byte swizzle) complete on full[s]; four
// tcgen05.mma (K = 16 each) per K-block accumulate into GEMM_BN TMEM columns and commit to
// empty[s], which frees the stage for the load GEMM_STAGES blocks later; a last commit
// signals the epilogue.  All four warps then read their 32 TMEM lanes (rows) 32 columns at
// a time into a 128 x 32 fp32 staging tile in the (now free) stage memory, laid out with the
// 128-byte swizzle (16-byte chunk index XOR row % 8: conflict-free writes), and thread 0
// stores each tile with one TMA store (two tiles in flight).  Without a C tensor map (N not
// a multiple of 4) the threads store their rows directly.  Two CTAs fit an SM (TMEM 2 x 256
// columns, 2 x 97 KB smem), so one CTA's epilogue overlaps the other's MMAs.  Every mbarrier wait is bounded; on timeout
// the device error word gets SDM_DEVERR_TIMEOUT and the CTA skips its stores.
//
// Loads past M, N or K read zeros (TMA bounds), stores are guarded, so M and N are free;
// K must be a multiple of 8 (16-byte rows).
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace sdm {

constexpr int GEMM_THREADS = 128;
constexpr int GEMM_BM = 128;
constexpr int GEMM_BN = 256;
constexpr int GEMM_BK = 64;
constexpr int GEMM_STAGES = 2;
constexpr uint32_t GEMM_A_BYTES = GEMM_BM * GEMM_BK * 2;  // 16 KB
constexpr uint32_t GEMM_B_BYTES = GEMM_BN * GEMM_BK * 2;  // 32 KB
constexpr uint32_t GEMM_STAGE_BYTES = GEMM_A_BYTES + GEMM_B_BYTES;
constexpr uint32_t GEMM_SMEM_BYTES = GEMM_STAGES * GEMM_STAGE_BYTES + 64 + 1024;

__global__ void __launch_bounds__(GEMM_THREADS, 2) gemm_bf16_tc_kernel(
    const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
    const __grid_constant__ CUtensorMap cmap, int cmap_ok, float* __restrict__ C, int M, int N,
    int K) {
    extern __shared__ unsigned char gemm_smem_raw[];
    unsigned char* sm =
        gemm_smem_raw + ((1024 - (ptx::smem_u32(gemm_smem_raw) & 1023)) & 1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + GEMM_STAGES * GEMM_STAGE_BYTES);
    uint64_t* empty = full + GEMM_STAGES;
    uint64_t* done = empty + GEMM_STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int m0 = blockIdx.y * GEMM_BM, n0 = blockIdx.x * GEMM_BN;
    const int nk = (K + GEMM_BK - 1) / GEMM_BK;

    if (warp == 0) ptx::tmem_alloc(tmem_slot, GEMM_BN);
    if (tid == 0) {
        for (int s = 0; s < GEMM_STAGES; ++s) {
            ptx::mbar_init(full + s, 1);
            ptx::mbar_init(empty + s, 1);
        }
        ptx::mbar_init(done, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t deadline = ptx::globaltimer_ns() + 2000000000ull;

    if (tid == 0) {
        const uint32_t idesc = ptx::idesc_bf16_f32(GEMM_BM, GEMM_BN);
        bool ok = true;
        auto load = [&](int kb) {
            const int s = kb % GEMM_STAGES;
            unsigned char* st = sm + s * GEMM_STAGE_BYTES;
            ptx::mbar_arrive_expect_tx(full + s, GEMM_STAGE_BYTES);
            ptx::tma_load_2d(st, &amap, kb * GEMM_BK, m0, full + s);
            ptx::tma_load_2d(st + GEMM_A_BYTES, &bmap, kb * GEMM_BK, n0, full + s);
        };
        auto mma = [&](int kb) {
            const int s = kb % GEMM_STAGES;
            unsigned char* st = sm + s * GEMM_STAGE_BYTES;
            if (!ptx::mbar_wait_bounded(full + s, (uint32_t)((kb / GEMM_STAGES) & 1), deadline)) {
                ok = false;
                return;
            }
            ptx::tc_fence_after();
            const uint64_t ad = ptx::umma_desc_kmajor_sw128(st);
            const uint64_t bd = ptx::umma_desc_kmajor_sw128(st + GEMM_A_BYTES);
#pragma unroll
            for (int k = 0; k < GEMM_BK / 16; ++k)  // 16 bf16 = 32 bytes per step
                ptx::umma_bf16(tmem, ad + 2 * k, bd + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
            ptx::umma_commit(empty + s);
        };
        for (int kb = 0; kb < nk && ok; ++kb) {
            if (kb >= GEMM_STAGES) {  // stage reuse: the MMAs of block kb - STAGES are done
                const int s = kb % GEMM_STAGES;
                if (!ptx::mbar_wait_bounded(empty + s, (uint32_t)(((kb / GEMM_STAGES) - 1) & 1),
                                            deadline)) {
                    ok = false;
                    break;
                }
            }
            load(kb);
            if (kb >= GEMM_STAGES - 1) mma(kb - (GEMM_STAGES - 1));
        }
        for (int kb = nk - (GEMM_STAGES - 1); ok && kb < nk; ++kb)
            if (kb >= 0) mma(kb);
        if (ok) {
            ptx::umma_commit(done);
        } else {
            *abort_flag = 1;
            raise_err(SDM_DEVERR_TIMEOUT);
        }
    }
    __syncthreads();  // thread 0 has issued everything (or given up)
    if (!*abort_flag && !ptx::mbar_wait_bounded(done, 0u, deadline)) {
        if (tid == 0) raise_err(SDM_DEVERR_TIMEOUT);
        *abort_flag = 1;
    }
    ptx::tc_fence_after();
    __syncthreads();
    if (!*abort_flag && cmap_ok) {
        // epilogue through swizzled staging tiles and TMA stores; the stage memory was last
        // touched by the async proxy (loads, MMA reads)
        ptx::fence_proxy_async_smem();
        const int r = warp * 32 + (tid & 31);  // row inside the tile = TMEM lane
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        for (int c = 0; c < GEMM_BN; c += 32) {
            const int buf = (c / 32) & 1;
            unsigned char* tile = sm + buf * (GEMM_BM * 32 * 4);  // 16 KB, 1024-aligned
            if (c >= 64 && tid == 0) ptx::bulk_wait_group_read<1>();  // tile buf is free
            __syncthreads();
            float v[32];
            ptx::tmem_ld32(trow + c, v);
            unsigned char* rowp = tile + r * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<float4*>(rowp + ((j ^ (r & 7)) << 4)) =
                    make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            ptx::fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0) {
                ptx::tma_store_2d(&cmap, n0 + c, m0, tile);
                ptx::bulk_commit_group();
            }
        }
        if (tid == 0) ptx::bulk_wait_group_read<0>();  // staging read before the CTA exits
    } else if (!*abort_flag) {
        // epilogue: warp w holds rows m0 + 32 w .. + 31 (TMEM lanes), 32 columns per load
        const int row = m0 + warp * 32 + (tid & 31);
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        for (int c = 0; c < GEMM_BN; c += 32) {
            float v[32];
            ptx::tmem_ld32(trow + c, v);
            if (row < M) {
                float* dst = C + (size_t)row * N + n0 + c;
                if (n0 + c + 32 <= N && (N & 3) == 0) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (n0 + c + i < N) dst[i] = v[i];
                }
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, GEMM_BN);
    }
}

}  // namespace sdm
