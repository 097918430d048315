/*
 * sdm.h — C ABI of the Sparse Delta Memory (SDM) hot path on NVIDIA B200 (sm_100a).
 *
 * Sparse Delta Memory ("Sparse Delta Memory: Scaling the State of Linear RNNs
 * through Sparsity", arXiv 2607.07386) replaces the dense Gated DeltaNet state
 * with an N-slot memory table per head.  Each token selects W write slots from
 * its key and R read slots from its query by product-key top-k scoring, applies
 * a gated delta update to the W write slots and reads a weighted sum of the R
 * read slots.  The library computes that path on the GPU:
 *
 *   sdm_score_topk   product-key scoring, per-half top-k, k x k combine,
 *                    top-W (or top-R) slot indices and softmax weights
 *   sdm_score_qk     both roles of one call (keys: writes, queries: reads)
 *   sdm_forward      the sparse gated-delta recurrence over T tokens (prefill)
 *   sdm_decode_step  one token per sequence (scoring + recurrence)
 *
 * Notation: B sequences, H heads, T tokens, key width d_k (two halves of
 * h = d_k/2), n sub-keys per half (N = n*n slots, slot s = i*n + j where i is
 * the rank source of the first half), value width d_v, per-half top-k k_half,
 * W write / R read slots per token, decay gate alpha in (0,1], input gate beta.
 *
 * Conventions shared by every entry point
 *   - Every pointer is caller-owned device memory (except where a comment says
 *     host), contiguous, row-major, 16-byte aligned.  The library never allocates
 *     device memory on a compute call; scratch comes from the caller through a
 *     workspace whose size a *_workspace_bytes query returns.
 *   - All GPU work is enqueued asynchronously on `stream` (a cudaStream_t; NULL
 *     is the legacy default stream).  Arguments are validated on the host before
 *     anything is enqueued; a failed validation enqueues nothing.
 *   - Nothing aborts, traps or prints.  Problems found on the device (an
 *     out-of-range slot index, a repeated write slot within one token, alpha <= 0)
 *     set bits of a device error word, skip the offending access and let the
 *     kernel finish; read the word with sdm_device_error.
 *   - Dimensions supported: 1 <= W, R <= 64; 1 <= k_half <= min(n, 64);
 *     top <= k_half^2; d_v a multiple of 4 with d_v <= 256; d_k even with
 *     d_k/2 a multiple of 8 and d_k <= 256; 1 <= n <= 4096.
 */
#ifndef SDM_H
#define SDM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* sdm_stream_t;

typedef enum {
    SDM_OK = 0,
    SDM_ERR_ARG = 1,        /* null pointer, negative size, unsupported option */
    SDM_ERR_SHAPE = 2,      /* dimensions outside the supported ranges */
    SDM_ERR_DTYPE = 3,      /* unknown dtype tag */
    SDM_ERR_ALIGN = 4,      /* pointer not 16-byte aligned */
    SDM_ERR_CUDA = 5,       /* a CUDA runtime call failed (launch, memset, ...) */
    SDM_ERR_BAD_INDEX = 6,  /* returned by sdm_device_error when an index bit is set */
    SDM_ERR_WORKSPACE = 7,  /* workspace missing or smaller than the query returned */
    SDM_ERR_UNSUPPORTED = 8 /* valid request this build does not implement */
} sdm_status;

typedef enum { SDM_F32 = 0, SDM_BF16 = 1 } sdm_dtype;

/*
 * Which slots the decay gate alpha_t scales at token t.  The pages (Sparse Delta Memory
 * summary, §3 Method "Sparse memory updates") say the gated delta updates act only on the
 * W selected slots and (§3 "Connection to GDN") that selecting every slot gives Gated
 * DeltaNet; they leave open whether the decay reaches the other slots.
 *   SDM_DECAY_ALL     every slot, every token (the dense Gated DeltaNet rule, applied
 *                     lazily through Lambda and the stamps)            -- the default
 *   SDM_DECAY_TOUCHED only the token's write slots, at the write; a slot that is not
 *                     written keeps its value, and one never written stays M0
 * With alpha = 1, or with every slot written at every token, the two agree.
 */
typedef enum { SDM_DECAY_ALL = 0, SDM_DECAY_TOUCHED = 1 } sdm_decay;

/* Bits of the device error word (sdm_device_error). */
#define SDM_DEVERR_SLOT_RANGE 1u   /* a slot index outside [0, N) */
#define SDM_DEVERR_DUP_WRITE 2u    /* a write slot repeated within one token */
#define SDM_DEVERR_ALPHA 4u        /* alpha <= 0 (its log is undefined) */
#define SDM_DEVERR_TIMEOUT 8u      /* a bounded on-chip wait gave up (the call's results are invalid) */

typedef struct {
    int32_t B, H, T;   /* sequences, heads, tokens in this call (T = 1 for decode) */
    int32_t d_k;       /* key / query width: two halves of d_k/2 */
    int32_t n_sub;     /* sub-keys per half; N = n_sub^2 slots per head */
    int32_t d_v;       /* value width = slot row width */
    int32_t k_half;    /* per-half top-k */
    int32_t W, R;      /* write and read slots per token */
    int32_t x_dtype;   /* sdm_dtype of q, k and the sub-key tables */
    int32_t v_dtype;   /* sdm_dtype of v */
    int32_t decay;     /* sdm_decay: which slots alpha scales (0 = every slot) */
} sdm_dims;

/*
 * Memory state of B*H sequences, all caller-owned device memory.  It is kept in
 * lazy-decay form so that no call ever sweeps the whole table:
 *   M      [B][H][N][d_v] fp32  raw slot rows
 *   stamp  [B][H][N]      fp64  log-decay prefix at the slot's last write;
 *                               NaN marks a pristine slot whose value is M0
 *   Lambda [B][H]         fp64  running log-decay prefix sum_t log(alpha_t)
 *   M0     [H][N][d_v]    fp32  initial memory, shared by the batch (read only)
 * The true value of slot s is  M[s] * exp(Lambda - stamp[s]),  or
 * M0[h][s] * exp(Lambda) while the slot is pristine.  (The pages give the decay
 * as a per-token multiplication of every slot; this form is equal to it.)  Under
 * SDM_DECAY_TOUCHED the value is M[s] itself (M0[h][s] while pristine): the stamps
 * then only mark pristine slots, and Lambda is kept but not used.
 */
typedef struct {
    float* M;
    double* stamp;
    double* Lambda;
    const float* M0;
} sdm_state;

/* Human-readable name of a status code (static string, never NULL). */
const char* sdm_status_str(int32_t status);

/* ABI version of this library; bumped whenever a signature or layout changes. */
int32_t sdm_abi_version(void);

/*
 * Bytes of each state array for `dims` (M, stamp, Lambda).  Host only.
 * Returns SDM_ERR_ARG on NULL outputs, SDM_ERR_SHAPE on unsupported dims.
 */
sdm_status sdm_state_bytes(const sdm_dims* dims, size_t* M_bytes, size_t* stamp_bytes,
                           size_t* lambda_bytes);

/*
 * Start B*H fresh sequences: every slot becomes pristine (its value is M0) and
 * Lambda = 0.  Writes stamp and Lambda only — O(B*H*N) stamps, no row traffic.
 * Source: §3 Method, "Learned initial state" (the memory starts from M0).
 */
sdm_status sdm_state_reset(const sdm_dims* dims, const sdm_state* st, sdm_stream_t stream);

/*
 * Dense memory of every sequence: M_out[b][h][s] = true value of slot s
 * ([B][H][N][d_v] fp32, caller-owned device buffer, may not alias st->M).
 * Sweeps the whole table; meant for checks, not for the hot path.
 */
sdm_status sdm_state_materialize(const sdm_dims* dims, const sdm_state* st, float* M_out,
                                 sdm_stream_t stream);

/*
 * Product-key top-k scoring for one role (write: x = k, read: x = q).
 * Source: §2 Background "Product Key Memory" and §3 Method "Sparse addressing";
 * softmax weights per §4 "SDM Configuration".
 *   x       [B][H][T][d_k]      dims->x_dtype
 *   subkeys [H][2][n_sub][d_k/2] dims->x_dtype   (half 1 table, then half 2)
 *   top     W for the write role, R for the read role (1 <= top <= 64)
 *   idx     [B][H][T][top] int32 out: slot indices, best first
 *   w       [B][H][T][top] fp32  out: softmax over the selected scores
 * Score of slot s = i*n + j is <x[0:h], C1[i]> + <x[h:2h], C2[j]> (fp32
 * accumulation of the stored inputs); larger first, equal scores to the lower
 * slot.  The k_half best sub-keys per half are kept and their k_half^2 sums
 * ranked; this equals ranking all N slots whenever k_half >= top.
 */
sdm_status sdm_score_topk(const sdm_dims* dims, const void* x, const void* subkeys, int32_t top,
                          int32_t* idx, float* w, sdm_stream_t stream);

/*
 * Which scoring kernel sdm_score_topk / sdm_score_qk launch for `dims` and `top` (host-side
 * query, no GPU work): SDM_SCORE_TC = the tensor-core kernel (TMA-fed tcgen05.mma into TMEM,
 * exact per-row selection; bf16, d_k = 128, n_sub a multiple of 64 up to 1024, top <= k_half
 * <= 64, T >= 64), SDM_SCORE_ROWS = the row scorer (short calls such as decode; n_sub <= 512),
 * SDM_SCORE_WARP = one warp per row on CUDA cores (every other shape); negative: a status
 * code (bad dims).
 */
enum { SDM_SCORE_TC = 1, SDM_SCORE_ROWS = 2, SDM_SCORE_WARP = 3 };
int32_t sdm_score_path(const sdm_dims* dims, int32_t top);

/*
 * Both scorings of one call: the keys against the write-role tables and the queries against
 * the read-role tables (§3 Method "Sparse addressing": keys choose the slots written,
 * queries the slots read), with the results of two sdm_score_topk calls but in one launch
 * where the shape allows it.
 *   q, k       [B][H][T][d_k]        dims->x_dtype
 *   skw, skr   [H][2][n_sub][d_k/2]  dims->x_dtype (the same pointer twice shares one table)
 *   widx, ww   [B][H][T][W]          int32 / fp32 out (write role, best first)
 *   ridx, rw   [B][H][T][R]          int32 / fp32 out (read role, best first)
 * Errors as sdm_score_topk.
 */
sdm_status sdm_score_qk(const sdm_dims* dims, const void* q, const void* k, const void* skw,
                        const void* skr, int32_t* widx, float* ww, int32_t* ridx, float* rw,
                        sdm_stream_t stream);

/* Workspace bytes sdm_forward / sdm_prefill need for `dims` (0 on bad dims). */
size_t sdm_forward_workspace_bytes(const sdm_dims* dims);

/*
 * Sparse gated-delta recurrence over T tokens (prefill), state updated in place.
 * Source: §2 Background "Gated DeltaNet"; §3 Method "Sparse memory updates",
 * "Sparse retrieval", "Connection to GDN".  Per token t, in order:
 *   every slot decays by alpha_t; p = sum_i w_i M[s_i]; e = v_t - p;
 *   M[s_i] += beta_t w_i e for the W (distinct) write slots;
 *   out_t = sum_j u_j M[r_j]   (read after the write).
 *   v      [B][H][T][d_v]  dims->v_dtype
 *   alpha, beta [B][H][T]  fp32
 *   widx, ww [B][H][T][W]  int32 / fp32   write slots and weights
 *   ridx, rw [B][H][T][R]  int32 / fp32   read slots and weights
 *   out    [B][H][T][d_v]  fp32 out
 *   ws     workspace of at least sdm_forward_workspace_bytes(dims) bytes
 * T = 0 is a valid no-op.
 */
sdm_status sdm_forward(const sdm_dims* dims, const void* v, const float* alpha, const float* beta,
                       const int32_t* widx, const float* ww, const int32_t* ridx, const float* rw,
                       const sdm_state* st, float* out, void* ws, size_t ws_bytes,
                       sdm_stream_t stream);

/*
 * The two stages of sdm_forward, callable separately (same arguments):
 *   sdm_forward_plan  pass over indices, weights and gates only (no rows): decay factors
 *                     of the rows each token gathers (from the slot stamps), links between
 *                     occurrences of the same slot inside each chunk, and per chunk the
 *                     C x C matrices that resolve them (a triangular solve, the intra-chunk
 *                     phase of the pages' Appendix A.1), packed with every other
 *                     column-independent input of the row pass into ws; writes ws,
 *                     st->stamp and st->Lambda.
 *   sdm_forward_run   the row pass: gathers, delta updates, stores, outputs (reads v and ws
 *                     -- the plan's packed copy of indices, weights and beta -- updates
 *                     st->M, writes out).  widx/ww/ridx/rw are validated, not re-read.
 * A run must follow the plan of the same call, on the same stream, with the same index,
 * weight and gate arrays and unchanged ws.
 */
sdm_status sdm_forward_plan(const sdm_dims* dims, const float* alpha, const float* beta,
                            const int32_t* widx, const float* ww, const int32_t* ridx,
                            const float* rw, const sdm_state* st, void* ws, size_t ws_bytes,
                            sdm_stream_t stream);
sdm_status sdm_forward_run(const sdm_dims* dims, const void* v, const float* beta,
                           const int32_t* widx, const float* ww, const int32_t* ridx,
                           const float* rw, const sdm_state* st, float* out, void* ws,
                           size_t ws_bytes, sdm_stream_t stream);

/*
 * Prefill = sdm_score_topk(k, skw, W) + sdm_score_topk(q, skr, R) + sdm_forward.
 *   q, k [B][H][T][d_k] (x_dtype); skw, skr [H][2][n_sub][d_k/2] (x_dtype)
 *   widx/ww, ridx/rw: caller buffers that receive the selections (as above)
 */
sdm_status sdm_prefill(const sdm_dims* dims, const void* q, const void* k, const void* v,
                       const float* alpha, const float* beta, const void* skw, const void* skr,
                       const sdm_state* st, int32_t* widx, float* ww, int32_t* ridx, float* rw,
                       float* out, void* ws, size_t ws_bytes, sdm_stream_t stream);

/*
 * One token for each of the B*H sequences (dims->T must be 1): scoring of k and
 * q, then the same recurrence step as sdm_forward.  Layouts drop the T axis:
 *   q, k [B][H][d_k]; v [B][H][d_v]; alpha, beta [B][H]; out [B][H][d_v];
 *   widx/ww [B][H][W], ridx/rw [B][H][R] receive the selections.
 * No workspace.  Equal to sdm_forward with T = 1 up to rounding order.
 * Where sdm_decode_path says SDM_DECODE_FUSED (bf16 q and k with d_k = 128,
 * 64 < n_sub <= 512, k_half, W, R <= 32, d_v <= 256) the step is one launch: each CTA
 * scores the keys and queries of two sequences of one head and runs their recurrence
 * steps from the selections it holds on chip; the selections are still written to
 * widx/ww/ridx/rw.  Otherwise it is a scoring launch followed by the recurrence launch.
 */
sdm_status sdm_decode_step(const sdm_dims* dims, const void* q, const void* k, const void* v,
                           const float* alpha, const float* beta, const void* skw,
                           const void* skr, const sdm_state* st, int32_t* widx, float* ww,
                           int32_t* ridx, float* rw, float* out, sdm_stream_t stream);

/*
 * Call log: what one call overwrites in the state, so that the state at the call's start can
 * be put back after it (Sparse Delta Memory summary, appendix A.3 "Memory-Efficient
 * Backward": the sparse updates are undone in place instead of keeping a copy of the
 * memory; here across calls).  A sequence run as calls 1..C is differentiated from the last
 * call back: restore call c's log, then sdm_backward over call c from that state, its dM_in
 * the dM_end of call c-1.  A call (sdm_forward, sdm_prefill, sdm_decode_step) writes only
 * the rows and stamps of its write slots and Lambda, so the log holds, for each write
 * occurrence, the raw row and stamp of its slot before the call, and Lambda:
 *   rows [B][H][T][W][d_v] fp32, stamps [B][H][T][W] fp64, Lambda [B][H] fp64
 * (sdm_call_log_bytes: the size, sections 256-byte aligned; O(T*W*d_v) per call).
 *   sdm_call_log_save     before the call, on its stream: copies from st into log.
 *                         widx [B][H][T][W] int32 are the call's write slots (for a
 *                         prefill, sdm_score_topk of the keys gives them before the call).
 *   sdm_call_log_restore  after the call (and after every later call has been restored):
 *                         copies log back into st, which then equals, bit for bit, the
 *                         state before the call.
 * log is caller-owned device memory of at least sdm_call_log_bytes(dims) bytes, 16-byte
 * aligned (SDM_ERR_WORKSPACE if smaller).  Slots outside [0, N) are skipped and set
 * SDM_DEVERR_SLOT_RANGE.
 */
size_t sdm_call_log_bytes(const sdm_dims* dims);
sdm_status sdm_call_log_save(const sdm_dims* dims, const int32_t* widx, const sdm_state* st,
                             void* log, size_t log_bytes, sdm_stream_t stream);
sdm_status sdm_call_log_restore(const sdm_dims* dims, const int32_t* widx, const void* log,
                                size_t log_bytes, const sdm_state* st, sdm_stream_t stream);

/*
 * The launches sdm_decode_step makes for these dims: SDM_DECODE_FUSED (one launch: scoring
 * and recurrence step in the same CTAs) or SDM_DECODE_TWO (a scoring launch, then the
 * recurrence launch); a negative sdm_status code for bad dims (dims->T is not looked at).
 */
enum { SDM_DECODE_FUSED = 1, SDM_DECODE_TWO = 2 };
int32_t sdm_decode_path(const sdm_dims* dims);

/*
 * Backward of the recurrence over one call of T tokens (Sparse Delta Memory summary,
 * appendix A.3 "Memory-Efficient Backward"): gradients with respect to v, alpha, beta and
 * the write and read weights, and with respect to the memory at the start of the call, for
 * an output gradient dout; the slot selections are fixed (not differentiated), under the
 * dims' decay rule.
 *   st    the state at the START of the call (as it was passed to the sdm_forward that
 *         produced the outputs).  The call replays the T tokens in place, logging the raw
 *         rows and stamps of each token's write slots before the write (the T*W*d_v record
 *         of the workspace), then walks the tokens backwards, restoring each token's write
 *         slots from the log: on return the state is again the start state (the memory is
 *         never copied; peak memory O(N*d_v + T*W*d_v) per sequence).
 *   dout  [B][H][T][d_v] fp32 gradient of the loss with respect to out
 *   dM_end [B][H][N][d_v] fp32 gradient of the loss with respect to the true slot values
 *         after the last token (a loss that also reads the final memory, e.g. the next
 *         call's dM_in when a sequence is processed in several calls), or NULL for zero
 *   outputs, fp32, caller-allocated, every element written:
 *         dv [B][H][T][d_v], dalpha [B][H][T], dbeta [B][H][T], dww [B][H][T][W],
 *         drw [B][H][T][R], dM_in [B][H][N][d_v] (with respect to the true slot values at
 *         the start; for a fresh state, summing it over b gives the gradient of M0)
 *   ws    device workspace of at least sdm_backward_workspace_bytes(dims) bytes, 16-byte
 *         aligned.
 * Each sequence's tokens are walked one at a time, split over 4-column slices of d_v (one warp
 * per slice); the workspace holds the write log, private stamp copies per slice and
 * per-slice shares of the column sums.
 * Errors: as sdm_forward; W + R <= 128; the slots must be in range and distinct within a
 * token.
 */
/*
 * Gradient through the scoring of one role with the selected slots held fixed (the top-k
 * choice is piecewise constant and has no gradient): with w the selection weights that
 * sdm_score_topk returned for x (softmax of the selected scores) and dw their gradient,
 *   dscore_q = w_q (dw_q - sum_r w_r dw_r); dx and the sub-key tables' gradient follow
 *   through the two half-score dot products (slot = i*n + j: C1[i], C2[j]).
 *   x, subkeys, top, idx, w   as given to / returned by sdm_score_topk
 *   dw    [B][H][T][top] fp32 (e.g. dww or drw of sdm_backward)
 *   dx    [B][H][T][d_k] fp32, written
 *   dsubkeys [H][2][n][d_k/2] fp32, ADDED TO (zero it first; calls accumulate)
 * One launch; the table gradient uses atomic adds, so its summation order is not fixed.
 */
sdm_status sdm_score_backward(const sdm_dims* dims, const void* x, const void* subkeys,
                              int32_t top, const int32_t* idx, const float* w, const float* dw,
                              float* dx, float* dsubkeys, sdm_stream_t stream);

size_t sdm_backward_workspace_bytes(const sdm_dims* dims);
sdm_status sdm_backward(const sdm_dims* dims, const void* v, const float* alpha, const float* beta,
                        const int32_t* widx, const float* ww, const int32_t* ridx, const float* rw,
                        const sdm_state* st, const float* dout, const float* dM_end, float* dv,
                        float* dalpha, float* dbeta, float* dww, float* drw, float* dM_in,
                        void* ws, size_t ws_bytes, sdm_stream_t stream);

/*
 * sdm_forward without a caller workspace and without any allocation: for callers that
 * cannot call cudaMalloc or hand out scratch memory themselves — for example a custom
 * operator inside a host framework that owns the device allocator and forbids side
 * allocations, or a loop whose memory budget is fixed when the process starts.  The paper
 * has no counterpart of this call; it only changes where the scratch lives.
 *   Arguments, layouts and results are those of sdm_forward.
 *   Scratch: one fixed 64 MiB array in device memory, defined in the library and held by
 *     every GPU that loads it until the process exits.  Calls whose workspace would
 *     exceed it (sdm_forward_workspace_bytes(dims) > 64 MiB) return SDM_ERR_WORKSPACE and
 *     enqueue nothing.  Each call writes every part of the array it later reads, so no
 *     contents carry over from the previous call.
 *   All calls on a device share the array: calls that can overlap on the GPU (different
 *     streams, or several host threads) race on it and must be serialised by the caller.
 *   The first call on a device looks up the array's device address (once per device, with
 *     the stream's device current); make that first call before any stream capture.  After
 *     a device reset the device has a new context, and the next call looks the address up
 *     again.
 *   Never calls cudaMalloc, cudaFree or any allocating routine.
 */
sdm_status sdm_forward_noalloc(const sdm_dims* dims, const void* v, const float* alpha,
                               const float* beta, const int32_t* widx, const float* ww,
                               const int32_t* ridx, const float* rw, const sdm_state* st,
                               float* out, sdm_stream_t stream);

/*
 * sdm_forward_run with the first step of the layer's output side fused into the read (§3
 * Method "Sparse retrieval": the read result is RMS-normalised and elementwise gated, then
 * mixed across heads by the output projection).  Besides out, it writes the projection's
 * operand
 *   a[b,t][h*d_v + c] = o_c / sqrt(mean_c o_c^2 + eps) * wn[c] * swish(g[b,t][h*d_v + c])
 *                       with o = out[b][h][t][:], swish(z) = z * sigmoid(z)
 * so that y = a @ Wo is one sdm_gemm_bf16(B*T, d_model, H*d_v, a, Wo_t, y).  The column
 * slices of a sequence finish each chunk in any order; the last to finish a chunk normalises
 * its tokens (no slice waits for another).
 *   g  [B][T][H*d_v] bf16 (the gate's pre-activation); wn [d_v] fp32; eps >= 0
 *   a  [B][T][H*d_v] bf16 out
 * Other arguments, workspace and errors as sdm_forward_run.
 */
sdm_status sdm_forward_run_gated(const sdm_dims* dims, const void* v, const float* beta,
                                 const int32_t* widx, const float* ww, const int32_t* ridx,
                                 const float* rw, const sdm_state* st, float* out, const void* g,
                                 const float* wn, float eps, void* a, void* ws, size_t ws_bytes,
                                 sdm_stream_t stream);

/*
 * Dense GEMM on the tensor cores (tcgen05, bf16 operands, fp32 accumulation):
 *   C[M][N] fp32 = A[M][K] x Bt[N][K]^T,  A and Bt bf16 row-major (K contiguous)
 * K a multiple of 8; M, N free.  Pointers 16-byte aligned.  One launch.
 */
sdm_status sdm_gemm_bf16(int32_t M, int32_t N, int32_t K, const void* A, const void* Bt, float* C,
                         sdm_stream_t stream);

/*
 * Input side of an SDM layer: the projections of the layer input into the per-head query,
 * key, value, output-gate pre-activation and the two gates (§2 Background "Gated DeltaNet":
 * decay gate alpha in (0,1), input gate beta in [0,1]; §4 "SDM Configuration": gates as in
 * GDN/FLA):
 *   P = x @ Win  (tensor cores), per head the columns [q (d_k) | k (d_k) | v (d_v) | g (d_v) | a | b]
 *   alpha = exp(-exp(A_log[h]) * softplus(a + dt_bias[h])),  beta = sigmoid(b)
 *   x     [B][T][d_model] bf16 (d_model a multiple of 8)
 *   Win_t [H*(2 d_k + 2 d_v + 2)][d_model] bf16 (Win transposed); A_log, dt_bias [H] fp32
 *   q, k  [B][H][T][d_k] bf16 (dims->x_dtype must be bf16); v [B][H][T][d_v] (v_dtype)
 *   g     [B][T][H*d_v] bf16 (for sdm_layer_out); alpha, beta [B][H][T] fp32
 *   ws    at least sdm_layer_in_workspace_bytes(dims) bytes (P, fp32)
 * No short convolution and no q/k normalisation.  Two launches.
 */
size_t sdm_layer_in_workspace_bytes(const sdm_dims* dims);
sdm_status sdm_layer_in(const sdm_dims* dims, const void* x, const void* Win_t,
                        const float* A_log, const float* dt_bias, int32_t d_model, void* q,
                        void* k, void* v, void* g, float* alpha, float* beta, void* ws,
                        size_t ws_bytes, sdm_stream_t stream);

/*
 * Output side of an SDM layer (§3 Method "Sparse retrieval": the read result is
 * RMS-normalised, elementwise gated and mixed across heads by the output projection):
 *   a[b,t][h*d_v + c] = x_c / sqrt(mean_c x_c^2 + eps) * wn[c] * swish(g[b,t][h*d_v + c])
 *                       with x = o[b][h][t][:], swish(z) = z * sigmoid(z)
 *   y[b,t][:] = a[b,t][:] @ Wo
 *   o    [B][H][T][d_v] fp32 (the recurrence output)
 *   g    [B][T][H*d_v] bf16 (the gate's pre-activation)
 *   wn   [d_v] fp32 (the RMS-norm weight, shared by the heads); eps >= 0
 *   Wo_t [d_model][H*d_v] bf16 (Wo transposed)
 *   y    [B][T][d_model] fp32
 *   ws   at least sdm_layer_out_workspace_bytes(dims) bytes (a, bf16)
 * Requires H*d_v a multiple of 8.  Two launches: the prologue, then sdm_gemm_bf16.
 */
size_t sdm_layer_out_workspace_bytes(const sdm_dims* dims);
sdm_status sdm_layer_out(const sdm_dims* dims, const float* o, const void* g, const float* wn,
                         float eps, const void* Wo_t, int32_t d_model, float* y, void* ws,
                         size_t ws_bytes, sdm_stream_t stream);

/*
 * Memory-utilisation diagnostics of post-softmax selected-slot weights (the pages'
 * Appendix D.1 "Memory Utilization and Access": cumulative top-k mass and an entropy-based
 * effective-key measure, summarised by the mean and token-level quantiles over batch, head
 * and time).  Rows are given best first, as sdm_score_topk writes them.
 *   w     [rows][K] fp32 (e.g. the ww or rw of a prefill: rows = B*H*T, K = W or R)
 *   cum   [rows][K] fp32, or NULL: cum[r][k] = w[r][0] + ... + w[r][k]
 *   eff   [rows] fp32: exp(H_r) / K with H_r = -sum_k w[r][k] ln w[r][k] (0 ln 0 = 0):
 *         1 for uniform weights, 1/K for one-hot
 *   mean  [K+1] fp32: the means over rows of cum[.][k] for k < K, then of eff
 *   probs HOST array of nprobs (0..16) values in [0, 1]
 *   quant [nprobs] fp32: the order statistic of eff at index floor(probs[q] * (rows-1))
 *         of its ascending sort (exact, ties included)
 *   ws    device workspace of at least sdm_weight_stats_workspace_bytes(rows, K) bytes
 * Requires rows >= 1, 1 <= K <= 64; device pointers 4-byte aligned.  Means are summed in a
 * fixed order (run to run identical).  Three kernel launches.
 */
size_t sdm_weight_stats_workspace_bytes(int64_t rows, int32_t K);
sdm_status sdm_weight_stats(int64_t rows, int32_t K, const float* w, float* cum, float* eff,
                            float* mean, int32_t nprobs, const double* probs, float* quant,
                            void* ws, size_t ws_bytes, sdm_stream_t stream);

/*
 * Read the device error word into *bits (host pointer; SDM_DEVERR_* bits), then
 * clear it when `clear` is non-zero.  Synchronises `stream`.  Returns SDM_OK when
 * no bit is set, SDM_ERR_BAD_INDEX when any is, SDM_ERR_CUDA if the copy fails.
 * The word is per device and shared by every call on that device.
 */
sdm_status sdm_device_error(uint32_t* bits, int32_t clear, sdm_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SDM_H */
