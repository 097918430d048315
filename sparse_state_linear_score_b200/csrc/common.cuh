// Shared device helpers for the SDM kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sdm.h"

#define SDM_DEV __device__ __forceinline__

namespace sdm {

// Device error word (SDM_DEVERR_* bits).  One per device; read by sdm_device_error.
__device__ unsigned int g_err;

SDM_DEV void raise_err(unsigned bits) { atomicOr(&g_err, bits); }

SDM_DEV float to_f32(float x) { return x; }
SDM_DEV float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Ordered comparison used by every top-k: larger score first, equal scores to the
// lower index.
SDM_DEV bool better(float sa, int ia, float sb, int ib) {
    return sa > sb || (sa == sb && ia < ib);
}

// Is this slot index inside [0, N)?
SDM_DEV bool slot_ok(int s, int N) { return (unsigned)s < (unsigned)N; }

// 16-byte global -> shared asynchronous copy (L2 only), with zero-fill when !pred.
SDM_DEV void cp_async16(void* smem_dst, const void* gmem_src, bool pred) {
    unsigned dst = (unsigned)__cvta_generic_to_shared(smem_dst);
    int n = pred ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(gmem_src),
                 "r"(n)
                 : "memory");
}
// 8-byte copy (through L1; the 16-byte form bypasses it).
SDM_DEV void cp_async8(void* smem_dst, const void* gmem_src) {
    unsigned dst = (unsigned)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(dst), "l"(gmem_src) : "memory");
}
SDM_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
SDM_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

// x / d for 0 <= x < 2^16 and 1 <= d <= 64 as one multiply-high: with m = ceil(2^32 / d),
// m*d - 2^32 < d, so the rounding error x*(m*d - 2^32) < 2^22 never reaches 2^32.
struct FastDiv {
    unsigned m, d;
    __host__ __device__ explicit FastDiv(unsigned dd) : m((unsigned)((0x100000000ull + dd - 1) / dd)), d(dd) {}
    SDM_DEV int div(int x) const { return (int)__umulhi((unsigned)x, m); }
    SDM_DEV int mod(int x) const { return x - div(x) * (int)d; }
};

}  // namespace sdm
