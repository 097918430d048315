// Row pass of the prefill recurrence: one CTA per ((b,h), block of CW value columns).
//
// The recurrence is independent per value column once the slots, weights and gates are
// fixed (p, e, the updates and the output are all column-wise), so each CTA owns a CW-wide
// column slice of one sequence's memory table and walks its chunks in order.  For chunk j
// (tokens t0..t0+nt-1), with the plan's chunk image (coefficients, links, store factors) and
// matrices Minv, GM = G Minv:
//
//   gather   raw[o]  = slice of the row of occurrence o's slot as stored at chunk start (from
//                      M, or M0 while pristine), issued one chunk ahead; rows the previous
//                      chunk stores after their gather are taken from that chunk's stores
//   dense    P0_t    = sum_i w_i |fe_i| raw[t,i],  Q0_t = sum_j u_j |fe_j| raw[t,j]
//            rhs     = beta (v - P0)
//            d       = Minv rhs                      (in-chunk writes seen by later predictions)
//            o_t     = Q0_t + sum_tau G[t][tau] d_tau = Q0_t + (GM rhs)_t   (read after write)
//   store    the last write of each slot stores e^{lam_end - lam_t} |fe| raw + sum over the
//            chunk's writes of that slot up to it of w e^{lam_end - lam_tau} d_tau (both
//            coefficients from the plan; its stamp, the chunk-end prefix, too).
//
// This is the dense-decay recurrence of §2 Background "Gated DeltaNet" restricted to the
// selected slots (§3 Method "Sparse memory updates", "Sparse retrieval"), evaluated chunk by
// chunk as in the pages' Appendix A.1 (intra-chunk triangular solve, sequential chunks).
//
// Warp roles.  Warps 0..7 (producers) only move data: while the consumers compute chunk j
// they gather chunk j+1's rows into the other row buffer (cp.async, 16-byte pieces, the Q
// pieces of a slice fetched by adjacent lanes of one instruction), copy its image (one bulk
// copy on an mbarrier) and values into the other halves of the double buffers, and load
// chunk j+2's gather words into registers.  Warps 8..15 (consumers) compute.  Named barriers
// hand the buffers over:
//   BAR_READY  producers arrive when chunk j+1's inputs have landed; consumers wait on it
//   BAR_FIXED  consumers arrive when chunk j's forwarded rows are taken from the other row
//              buffer; producers wait on it before gathering into that buffer
//   BAR_CONS   consumers among themselves, between compute phases
// Every thread of both roles takes part in every instance of BAR_READY and BAR_FIXED (J of
// each), so the hand-over cannot wait for a thread that has left.
#pragma once

#include "common.cuh"
#include "plan.cuh"
#include "tc_ptx.cuh"

namespace sdm {

constexpr int RUN_THREADS = 512;
constexpr int RUN_PRODUCERS = 256;  // warps 0..7
constexpr int RUN_CONSUMERS = RUN_THREADS - RUN_PRODUCERS;
constexpr int RUN_PAD = 8;  // floats between token blocks: spreads a warp's rows over banks
constexpr int RUN_GW = PLAN_MAX_OCC / RUN_PRODUCERS;  // gather words per producer thread
constexpr int BAR_READY = 1, BAR_FIXED = 2, BAR_CONS = 3;

SDM_DEV void named_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
SDM_DEV void named_arrive(int id, int count) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Floats per token block of gathered rows: its slots' CW-wide slices + padding.
__host__ __device__ inline int run_tok_stride(int per_tok, int CW) { return per_tok * CW + RUN_PAD; }
// Row stride of Minv / GM in the chunk image (16-byte rows, 4 floats apart in banks).
__host__ __device__ inline int run_mat_stride(int C) { return C + 4; }

// Shared memory of the row pass (bytes), in this order: rows [2][C*(tsw+tsr)] floats,
// images [2][img bytes], values [2][C*CW] of VT (16-byte padded), rhs, d, Q0 [C*CW] floats
// each, the image copies' mbarrier.
__host__ __device__ inline int run_vst_bytes(int C, int CW, int vbytes) {
    return up16i(C * CW * vbytes);
}
__host__ __device__ inline size_t run_smem_bytes(int C, int W, int R, int CW, int vbytes) {
    const size_t tsw = (size_t)run_tok_stride(W, CW), tsr = (size_t)run_tok_stride(R, CW);
    size_t b = 0;
    b += (size_t)2 * C * (tsw + tsr) * 4;            // rows, two chunks
    b += (size_t)2 * run_img(C, W, R).bytes;         // chunk images, two chunks
    b += (size_t)2 * run_vst_bytes(C, CW, vbytes);   // values, two chunks
    b += (size_t)3 * C * CW * 4;                     // rhs, d, Q0
    b += 16;                                         // mbarrier
    b += 16;                                         // the epilogue's flag
    return b;
}

// Optional epilogue of the row pass: the layer output side's RMS-norm and swish gate (§3
// Method "Sparse retrieval"; the same arithmetic as layer_prologue_kernel)
//   a[b,t][h*d_v + c] = o_c / sqrt(mean_c o_c^2 + eps) * wn[c] * swish(g[b,t][h*d_v + c])
// needs a token's whole row, which d_v / CW column slices produce.  Each slice counts itself
// finished with a chunk (an acquire-release atomic after its outputs); the slice that completes
// the count reads the chunk's rows back (from L2) and writes a.  No slice waits for another.
struct RunEpi {
    const __nv_bfloat16* g;  // [B][T][H*d_v] gate pre-activation; null: no epilogue
    const float* wn;         // [d_v] RMS-norm weight
    float eps;
    __nv_bfloat16* a;        // [B][T][H*d_v] out (bf16: the output projection's operand)
    int* cnt;                // [B*H][J] slices finished with each chunk, zero at launch
};

// Atomic add with acquire-release semantics at GPU scope (returns the old value).
SDM_DEV int atom_add_acq_rel(int* p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
                 : "memory");
    return old;
}

// The epilogue of tokens t0..t0+nt-1 (nt <= 32) of sequence bh by the consumer warps: warp cw
// takes tokens cw, cw+8, cw+16, cw+24, and every load of its four tokens (the rows from L2, the
// gates) is issued before any is used.
SDM_DEV void run_epilogue(const RunEpi& ep, const float* out, size_t bh, int H, int T, int d_v,
                          int t0, int nt, int cw, int lane) {
    constexpr int TPW = PLAN_MAX_C / (RUN_CONSUMERS / 32);  // tokens per consumer warp
    const int b = (int)(bh / H), h = (int)(bh % H);
    float4 x[TPW][2];
    uint2 gr[TPW][2];
#pragma unroll
    for (int u = 0; u < TPW; ++u) {
        const int t = cw + u * (RUN_CONSUMERS / 32);
        const float4* orow = reinterpret_cast<const float4*>(out + (bh * T + t0 + t) * d_v);
        const size_t grow = (((size_t)b * T + t0 + t) * H + h) * d_v;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int c4 = lane + 32 * k;
            const bool in = t < nt && 4 * c4 < d_v;
            x[u][k] = in ? __ldcg(orow + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
            gr[u][k] = in ? *reinterpret_cast<const uint2*>(ep.g + grow + 4 * c4) : make_uint2(0, 0);
        }
    }
#pragma unroll
    for (int u = 0; u < TPW; ++u) {
        const int t = cw + u * (RUN_CONSUMERS / 32);
        float ss = 0.f;
#pragma unroll
        for (int k = 0; k < 2; ++k)
            ss = fmaf(x[u][k].x, x[u][k].x, fmaf(x[u][k].y, x[u][k].y,
                 fmaf(x[u][k].z, x[u][k].z, fmaf(x[u][k].w, x[u][k].w, ss))));
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
        if (t >= nt) continue;
        const float r = rsqrtf(ss / (float)d_v + ep.eps);
        const size_t grow = (((size_t)b * T + t0 + t) * H + h) * d_v;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int c = 4 * (lane + 32 * k);
            if (c >= d_v) continue;
            const float4 w4 = *reinterpret_cast<const float4*>(ep.wn + c);
            const float xs[4] = {x[u][k].x, x[u][k].y, x[u][k].z, x[u][k].w};
            const float ws[4] = {w4.x, w4.y, w4.z, w4.w};
            const unsigned gw[2] = {gr[u][k].x, gr[u][k].y};
            unsigned short ab[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float z = __bfloat162float(
                    __ushort_as_bfloat16((unsigned short)(gw[e >> 1] >> ((e & 1) * 16))));
                const float sw = z / (1.f + expf(-z));
                ab[e] = __bfloat16_as_ushort(__float2bfloat16_rn(xs[e] * r * ws[e] * sw));
            }
            *reinterpret_cast<uint2*>(ep.a + grow + c) =
                make_uint2((unsigned)ab[0] | ((unsigned)ab[1] << 16),
                           (unsigned)ab[2] | ((unsigned)ab[3] << 16));
        }
    }
}

template <int CW, typename VT, bool EPI>
__global__ void __launch_bounds__(RUN_THREADS, 1) recur_run_kernel(
    const VT* __restrict__ v, const int32_t* __restrict__ rs,
    const unsigned char* __restrict__ imgs, float* __restrict__ M, const float* __restrict__ M0,
    float* __restrict__ out, int H, int T, int N, int d_v, int W, int R, int C, int J,
    RunEpi ep) {
    constexpr int Q = CW / 4;
    extern __shared__ __align__(16) unsigned char run_smem[];
    const int ncb = d_v / CW;
    const int cb = blockIdx.x % ncb;
    const size_t bh = blockIdx.x / ncb;
    const int h = (int)(bh % H);
    const int c0 = cb * CW;
    float* Mb = M + bh * (size_t)N * d_v;
    const float* M0h = M0 + (size_t)h * N * d_v;
    const size_t occ_base = bh * (size_t)T * (W + R);
    const int tid = threadIdx.x;
    const int tsw = run_tok_stride(W, CW), tsr = run_tok_stride(R, CW);
    const int MS = run_mat_stride(C);
    const RunImg im = run_img(C, W, R);

    float* s_rowbuf = reinterpret_cast<float*>(run_smem);  // [2][C*(tsw+tsr)]
    const int rowbuf = C * (tsw + tsr);
    unsigned char* s_imgbuf = reinterpret_cast<unsigned char*>(s_rowbuf + 2 * (size_t)rowbuf);
    unsigned char* s_vbuf = s_imgbuf + 2 * (size_t)im.bytes;
    const int vst = run_vst_bytes(C, CW, (int)sizeof(VT));
    float* s_rhs = reinterpret_cast<float*>(s_vbuf + 2 * (size_t)vst);
    float* s_d = s_rhs + C * CW;
    float* s_q = s_d + C * CW;
    uint64_t* bar_img = reinterpret_cast<uint64_t*>(s_q + C * CW);
    int* s_last = reinterpret_cast<int*>(bar_img + 1);  // this slice finished a chunk last

    if (tid == 0) {
        ptx::mbar_init(bar_img, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();

    const FastDiv fW((unsigned)W), fR((unsigned)R);
    // position of a write occurrence's slice, and of a read occurrence's slice
    auto wpos = [&](int o) { const int t = fW.div(o); return t * tsw + (o - t * W) * CW; };
    auto rpos = [&](int o) { const int t = fR.div(o); return C * tsw + t * tsr + (o - t * R) * CW; };
    auto pos = [&](int o, int nw) { return o < nw ? wpos(o) : rpos(o - nw); };

    if (tid < RUN_PRODUCERS) {
        // ------------------------------------ producers ------------------------------------
        const int lane = tid & 31, wbase = tid - lane;
        constexpr int PER = 32 / Q;  // occurrences per cp.async instruction
        int gw[RUN_GW];              // gather words of the next chunk to gather
        auto load_words = [&](int jn) {
            const int no = min(C, T - jn * C) * (W + R);
            const int32_t* src = rs + occ_base + (size_t)jn * C * (W + R);
#pragma unroll
            for (int k = 0; k < RUN_GW; ++k) {
                const int o = tid + k * RUN_PRODUCERS;
                gw[k] = o < no ? src[o] : 0x7fffffff;
            }
        };
        // chunk jn's rows (as stored now; those its previous chunk stores afterwards are
        // replaced from that chunk's stores), image, matrices and values
        auto stage = [&](int jn) {
            const int t0 = jn * C, nt = min(C, T - t0), nw = nt * W, no = nt * (W + R);
            float* rbuf = s_rowbuf + (size_t)(jn & 1) * rowbuf;
#pragma unroll
            for (int k = 0; k < RUN_GW; ++k) {
#pragma unroll
                for (int r = 0; r < Q; ++r) {
                    const int src_lane = r * PER + lane / Q;
                    const int sw = __shfl_sync(0xffffffffu, gw[k], src_lane);
                    const int o = wbase + k * RUN_PRODUCERS + src_lane;
                    const int q = lane % Q;
                    if (o < no) {
                        const int s = sw & 0x7fffffff;
                        const bool ok = s < N;
                        const float* src =
                            (sw < 0 ? M0h : Mb) + (ok ? (size_t)s * d_v : 0) + c0 + 4 * q;
                        cp_async16(rbuf + pos(o, nw) + 4 * q, src, ok);
                    }
                }
            }
            // image (with Minv and GM): one bulk copy.  The consumers' reads of this buffer
            // (chunk jn-2) precede it through BAR_FIXED.
            if (tid == 0) {
                ptx::fence_proxy_async_smem();
                ptx::mbar_arrive_expect_tx(bar_img, (uint32_t)im.bytes);
                ptx::bulk_load(s_imgbuf + (size_t)(jn & 1) * im.bytes,
                               imgs + (bh * J + jn) * (size_t)im.bytes, (uint32_t)im.bytes, bar_img);
            }
            // values: nt rows of CW elements, in 16-byte (or, for 8-byte rows, 8-byte) pieces
            constexpr int VROW = CW * (int)sizeof(VT);
            constexpr int VB = VROW >= 16 ? 16 : VROW;
            constexpr int VP = VROW / VB;
            unsigned char* vdst = s_vbuf + (size_t)(jn & 1) * vst;
            for (int e = tid; e < nt * VP; e += RUN_PRODUCERS) {
                const int t = e / VP, piece = e % VP;
                const unsigned char* vsrc =
                    reinterpret_cast<const unsigned char*>(v + (bh * T + t0 + t) * d_v + c0) +
                    piece * VB;
                if constexpr (VB == 16) cp_async16(vdst + t * VROW + piece * VB, vsrc, true);
                else cp_async8(vdst + t * VROW + piece * VB, vsrc);
            }
            cp_async_commit();
        };

        // chunk jn's copies have landed (the image's wait is bounded: past the deadline the
        // device error word records it and the pass goes on, so no barrier is left waiting)
        auto landed = [&](int jn) {
            cp_async_wait_all();
            const uint64_t deadline = ptx::globaltimer_ns() + 2000000000ull;
            if (!ptx::mbar_wait_bounded(bar_img, (uint32_t)(jn & 1), deadline) && tid == 0)
                raise_err(SDM_DEVERR_TIMEOUT);
        };
        load_words(0);
        stage(0);
        if (J > 1) load_words(1);
        landed(0);
        named_arrive(BAR_READY, RUN_THREADS);
        for (int j = 0; j < J; ++j) {
            // the consumers have taken chunk j's forwarded rows: the other buffers are free
            named_sync(BAR_FIXED, RUN_THREADS);
            if (j + 1 < J) {
                stage(j + 1);
                if (j + 2 < J) load_words(j + 2);
                landed(j + 1);
                named_arrive(BAR_READY, RUN_THREADS);
            }
        }
        return;
    }

    // ------------------------------------- consumers ---------------------------------------
    const int ctid = tid - RUN_PRODUCERS;
    const int csw = W + 1, csr = R + 1;
    for (int j = 0; j < J; ++j) {
        const int t0 = j * C, nt = min(C, T - t0);
        const int nw = nt * W, no = nt * (W + R);
        float* rows = s_rowbuf + (size_t)(j & 1) * rowbuf;
        const float* prev_rows = s_rowbuf + (size_t)((j + 1) & 1) * rowbuf;
        const unsigned char* img = s_imgbuf + (size_t)(j & 1) * im.bytes;
        const float* Minv = reinterpret_cast<const float*>(img + im.minv);
        const float* GM = reinterpret_cast<const float*>(img + im.gm);
        const float* s_coef = reinterpret_cast<const float*>(img + im.coef);
        const int* s_hz = reinterpret_cast<const int*>(img + im.hz);
        const int* s_wslot = reinterpret_cast<const int*>(img + im.wslot);
        const int* s_wlk = reinterpret_cast<const int*>(img + im.wlk);
        const float* s_sc = reinterpret_cast<const float*>(img + im.sc);
        const float* s_a = reinterpret_cast<const float*>(img + im.a);
        const float* s_beta = reinterpret_cast<const float*>(img + im.beta);
        const VT* s_v = reinterpret_cast<const VT*>(s_vbuf + (size_t)(j & 1) * vst);

        named_sync(BAR_READY, RUN_THREADS);
        // 1. rows the previous chunk stored after they were gathered: take its stored values
        if (j > 0) {
            for (int e = ctid; e < no * Q; e += RUN_CONSUMERS) {
                const int hv = s_hz[e / Q];
                if (hv < 0) break;  // end of the chunk's list
                const int o = hv & 0xffff, pv = hv >> 16, q = e % Q;
                reinterpret_cast<float4*>(rows + pos(o, nw))[q] =
                    reinterpret_cast<const float4*>(prev_rows + wpos(pv))[q];
            }
        }
        named_arrive(BAR_FIXED, RUN_THREADS);
        named_sync(BAR_CONS, RUN_CONSUMERS);

        // 2. predictions (writes) and reads from the chunk-start memory; a task is two
        //    adjacent columns of one token
        constexpr int CP = CW / 2;
        for (int task = ctid; task < 2 * nt * CP; task += RUN_CONSUMERS) {
            const bool rd = task >= nt * CP;
            const int e = rd ? task - nt * CP : task;
            const int t = e / CP, c = 2 * (e % CP);
            // four independent partial sums per column (latency of the smem loads)
            const float* rr = rd ? rows + C * tsw + t * tsr + c : rows + t * tsw + c;
            const float* cf = rd ? s_coef + C * csw + t * csr : s_coef + t * csw;
            const int n_i = rd ? R : W;
            float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
            int i = 0;
            for (; i + 4 <= n_i; i += 4) {
                const float2 r0 = *reinterpret_cast<const float2*>(rr + i * CW);
                const float2 r1 = *reinterpret_cast<const float2*>(rr + (i + 1) * CW);
                const float2 r2 = *reinterpret_cast<const float2*>(rr + (i + 2) * CW);
                const float2 r3 = *reinterpret_cast<const float2*>(rr + (i + 3) * CW);
                a0.x = fmaf(cf[i], r0.x, a0.x);
                a0.y = fmaf(cf[i], r0.y, a0.y);
                a1.x = fmaf(cf[i + 1], r1.x, a1.x);
                a1.y = fmaf(cf[i + 1], r1.y, a1.y);
                a2.x = fmaf(cf[i + 2], r2.x, a2.x);
                a2.y = fmaf(cf[i + 2], r2.y, a2.y);
                a3.x = fmaf(cf[i + 3], r3.x, a3.x);
                a3.y = fmaf(cf[i + 3], r3.y, a3.y);
            }
            for (; i < n_i; ++i) {
                const float2 r0 = *reinterpret_cast<const float2*>(rr + i * CW);
                a0.x = fmaf(cf[i], r0.x, a0.x);
                a0.y = fmaf(cf[i], r0.y, a0.y);
            }
            const float accx = (a0.x + a1.x) + (a2.x + a3.x);
            const float accy = (a0.y + a1.y) + (a2.y + a3.y);
            const int ev = t * CW + c;
            if (!rd) {
                const float b = s_beta[t];
                s_rhs[ev] = b * (to_f32(s_v[ev]) - accx);
                s_rhs[ev + 1] = b * (to_f32(s_v[ev + 1]) - accy);
            } else {
                *reinterpret_cast<float2*>(s_q + ev) = make_float2(accx, accy);
            }
        }
        named_sync(BAR_CONS, RUN_CONSUMERS);
        // 3. d = Minv rhs and o = Q0 + GM rhs (both lower triangular, zero beyond the chunk);
        //    a task is two adjacent columns of one token
        for (int task = ctid; task < 2 * nt * CP; task += RUN_CONSUMERS) {
            const bool oo = task >= nt * CP;
            const int e = oo ? task - nt * CP : task;
            const int t = e / CP, c = 2 * (e % CP);
            const float* mr = (oo ? GM : Minv) + t * MS;
            float2 a0 = make_float2(0.f, 0.f), a1 = a0;
            int tau = 0;
            for (; tau + 2 <= t + 1; tau += 2) {
                const float2 r0 = *reinterpret_cast<const float2*>(s_rhs + tau * CW + c);
                const float2 r1 = *reinterpret_cast<const float2*>(s_rhs + (tau + 1) * CW + c);
                a0.x = fmaf(mr[tau], r0.x, a0.x);
                a0.y = fmaf(mr[tau], r0.y, a0.y);
                a1.x = fmaf(mr[tau + 1], r1.x, a1.x);
                a1.y = fmaf(mr[tau + 1], r1.y, a1.y);
            }
            if (tau <= t) {
                const float2 r0 = *reinterpret_cast<const float2*>(s_rhs + tau * CW + c);
                a0.x = fmaf(mr[tau], r0.x, a0.x);
                a0.y = fmaf(mr[tau], r0.y, a0.y);
            }
            const int ev = t * CW + c;
            const float2 r = make_float2(a0.x + a1.x, a0.y + a1.y);
            if (oo) {
                const float2 q = *reinterpret_cast<const float2*>(s_q + ev);
                *reinterpret_cast<float2*>(out + (bh * T + t0 + t) * d_v + c0 + c) =
                    make_float2(q.x + r.x, q.y + r.y);
            } else {
                *reinterpret_cast<float2*>(s_d + ev) = r;
            }
        }
        named_sync(BAR_CONS, RUN_CONSUMERS);
        if (EPI) {
            // one acquire-release count per slice and chunk, after the barrier that orders every
            // consumer's output stores before it: it publishes them and, for the last slice,
            // makes the other slices' stores visible to the consumers after the next barrier
            // (the epilogue itself follows the chunk's memory stores, below)
            if (ctid == 0) *s_last = atom_add_acq_rel(ep.cnt + bh * J + j, 1) == ncb - 1;
        }
        // 4. the stores of the chunk's last writes (also written back to the rows, from where
        //    the next chunk takes the ones it gathered before they were stored)
        //    The Q 16-byte pieces of a slice are handled by adjacent lanes, so that one store
        //    instruction writes whole 32-byte sectors.
        //    Two tasks per step, their loads issued together (most chains are the write
        //    itself; the links to earlier writes of the slot, rare, are followed after).
        for (int e0 = ctid; e0 < nw * Q; e0 += 2 * RUN_CONSUMERS) {
            int o[2], q[2], lk[2], sl[2];
            bool own[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int e = e0 + u * RUN_CONSUMERS;
                const bool in = e < nw * Q;
                o[u] = in ? e / Q : 0;
                q[u] = e % Q;
                lk[u] = s_wlk[o[u]];
                sl[u] = s_wslot[o[u]];
                own[u] = in && (lk[u] & LK_OWNER) && sl[u] < N;
            }
            float4 a[2], raw[2];
            float f[2];
            float4* rp[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const float cf = s_sc[o[u]];
                const float4 dd = reinterpret_cast<const float4*>(s_d + fW.div(o[u]) * CW)[q[u]];
                a[u] = make_float4(cf * dd.x, cf * dd.y, cf * dd.z, cf * dd.w);
                rp[u] = reinterpret_cast<float4*>(rows + wpos(o[u])) + q[u];
                raw[u] = *rp[u];
                f[u] = s_a[o[u]];
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                if (!own[u]) continue;
                // the chunk's earlier writes of the slot, decayed to the chunk end
                for (int L = lk_link(lk[u]); L >= 0; L = lk_link(s_wlk[L])) {
                    const float cfa = s_sc[L];
                    const float4 dd = reinterpret_cast<const float4*>(s_d + fW.div(L) * CW)[q[u]];
                    a[u].x = fmaf(cfa, dd.x, a[u].x);
                    a[u].y = fmaf(cfa, dd.y, a[u].y);
                    a[u].z = fmaf(cfa, dd.z, a[u].z);
                    a[u].w = fmaf(cfa, dd.w, a[u].w);
                }
                float4 val;
                val.x = fmaf(f[u], raw[u].x, a[u].x);
                val.y = fmaf(f[u], raw[u].y, a[u].y);
                val.z = fmaf(f[u], raw[u].z, a[u].z);
                val.w = fmaf(f[u], raw[u].w, a[u].w);
                reinterpret_cast<float4*>(Mb + (size_t)sl[u] * d_v + c0)[q[u]] = val;
                *rp[u] = val;  // the next chunk forwards it
            }
        }
        // the stores precede the gathers that follow the next BAR_FIXED arrival
        __threadfence_block();
        if (EPI) {
            named_sync(BAR_CONS, RUN_CONSUMERS);
            if (*s_last) run_epilogue(ep, out, bh, H, T, d_v, t0, nt, ctid >> 5, tid & 31);
        }
    }
}

}  // namespace sdm
