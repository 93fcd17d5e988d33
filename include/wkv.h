/*
 * wkv.h -- C ABI of the B200 (sm_100a) WKV kernel library libwkv_b200.so.
 *
 * The library evaluates RWKV's WKV time-mixing recurrence on one GPU:
 *   - RWKV-4 WKV forward and backward (the operator RWKV_TimeMix.forward calls
 *     as RUN_CUDA(B, T, C, time_decay, time_first, k, v); RWKV-LM v4 code
 *     walkthrough page "代码连连看——RWKV", section RWKV_TimeMix),
 *   - the same RWKV-4 recurrence as a state-carrying step over batched,
 *     variable-length inference slots (web-rwkv crate page, section
 *     "批量推理" / batched inference: slots, token_chunk_size, empty slots
 *     skipped, state persisting across run() calls),
 *   - the RWKV-6 head-state recurrence forward (rwkv-ops package page,
 *     section "rwkv6op 使用方法": RWKV6_OP call and argument tables).
 *
 * RWKV-4 definition, per lane (b, c), with decay rate w_c > 0 (the model's
 * exp(time_decay_c)) and bonus u_c (time_first_c):
 *
 *   y_t = ( sum_{i<t} e^{-(t-1-i) w + k_i} v_i + e^{u + k_t} v_t )
 *       / ( sum_{i<t} e^{-(t-1-i) w + k_i}     + e^{u + k_t} )
 *
 * evaluated with the overflow-safe running-max state: the past sums are
 * a = aa * 2^(P + ref) and b = bb * 2^(P + ref) with P = base - n * w * log2(e).
 * ref = fl(k_first * log2(e)) is a per-lane reference fixed by the first key
 * the lane absorbs (k_first = k[b][0][c] for wkv4_forward), so exponents have
 * the size of the key range, not of the keys; n counts the decay steps since
 * the exponent was last set, so the decay never accumulates rounding error.
 *
 * RWKV-6 definition, per (batch b, head h), key index i, value index j:
 *
 *   o_t[j]    = sum_i r_t[i] * ( S_{t-1}[i][j] + u[i] k_t[i] v_t[j] )
 *   S_t[i][j] = w_t[i] * S_{t-1}[i][j] + k_t[i] v_t[j]
 *
 * Conventions shared by every entry point
 *   Memory      All pointers are DEVICE pointers unless stated otherwise. The
 *               caller owns every buffer; the library allocates nothing on
 *               these paths and keeps no per-call state.
 *   Layout      Activations are dense row-major [B][T][C] (C fastest), with no
 *               padding. Per-channel parameters are dense [C] float32.
 *   Alignment   Every device pointer must be 16-byte aligned.
 *   Sizes       64-bit. A zero B, T or C (S, N) is a valid no-op (WKV_OK).
 *   dtype       WKV_F32 or WKV_BF16 selects the storage type of the
 *               activations (k, v, y, gy, gk, gv, r, w, o); arithmetic and
 *               recurrent state are float32 in both cases. bf16 outputs are
 *               rounded to nearest even.
 *   C granularity  C must be a multiple of 4 for WKV_F32 and of 8 for
 *               WKV_BF16 (rows must be whole 16-byte units).
 *   Streams     `stream` is a cudaStream_t (NULL = legacy default stream).
 *               Every call is asynchronous on that stream and never
 *               synchronises the device.
 *   Errors      Argument errors are detected on the host, before anything is
 *               launched, and returned as WKV_ERR_INVALID_ARG or
 *               WKV_ERR_UNSUPPORTED; a launch failure returns WKV_ERR_CUDA.
 *               wkv_last_error() gives a one-line message for the calling
 *               thread's most recent failure. No C++ exception crosses this
 *               interface. Kernels never trap: a bounded wait that gives up
 *               records a code that wkv_device_error() returns.
 *   Threads     The library is thread-safe; calls on different streams may
 *               run concurrently.
 */
#ifndef WKV_B200_H
#define WKV_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define WKV_ABI_VERSION 1

/* Steps between two RWKV-4 forward state checkpoints (see wkv4_forward). */
#define WKV4_CKPT_LEN 16

typedef enum {
    WKV_OK = 0,
    WKV_ERR_INVALID_ARG = 1, /* null/misaligned pointer, negative size, bad dtype */
    WKV_ERR_UNSUPPORTED = 2, /* well-formed request outside what the kernels cover */
    WKV_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed       */
    WKV_ERR_DEVICE = 4       /* a kernel recorded a device-side error code        */
} wkv_status;

typedef enum { WKV_F32 = 0, WKV_BF16 = 1 } wkv_dtype;

/* Device-side error codes reported by wkv_device_error (bit flags). */
#define WKV_DEVERR_WAIT_TIMEOUT 0x1u /* a bounded wait on a copy gave up      */
#define WKV_DEVERR_BAD_SLOT     0x2u /* a slot's token range was out of bounds */
#define WKV_DEVERR_BAD_STATE    0x4u /* a state_map entry was out of range    */

/* ABI version of the loaded library (WKV_ABI_VERSION). */
int wkv_abi_version(void);

/* Static, human-readable name of a wkv_status value. */
const char *wkv_status_string(int status);

/* Message of the calling thread's last failing call ("" if none). */
const char *wkv_last_error(void);

/*
 * Read (and, if reset != 0, clear) the device-side error word of the current
 * device. SYNCHRONOUS: waits for all work on the current device. *code gets
 * an OR of WKV_DEVERR_* bits (0 = no error).
 */
wkv_status wkv_device_error(uint32_t *code, int reset);

/* ------------------------------------------------------------------------ */
/* RWKV-4                                                                    */
/* ------------------------------------------------------------------------ */

/* Number of floats of the checkpoint buffer: B * ceil(T / WKV4_CKPT_LEN) * 3 * C. */
size_t wkv4_ckpt_floats(int64_t B, int64_t T, int64_t C);

/*
 * RWKV-4 WKV forward.
 *   w, u   [C] float32. w is the per-step decay RATE (> 0): the state is
 *          multiplied by e^{-w} per token. u is the current-token bonus.
 *   k, v   [B][T][C] of `dtype`.
 *   y      [B][T][C] of `dtype`, written. May be NULL to only produce ckpt.
 *   ckpt   NULL, or [B][ceil(T/WKV4_CKPT_LEN)][3][C] float32, written: entry
 *          [b][m] holds (aa, bb, P) of every channel *before* token
 *          m * WKV4_CKPT_LEN of sample b (P relative to the lane's ref).
 *          wkv4_backward reads it.
 * The state starts from the empty past (aa = bb = 0, exponent -1e38).
 */
wkv_status wkv4_forward(int64_t B, int64_t T, int64_t C, int dtype,
                        const float *w, const float *u,
                        const void *k, const void *v, void *y,
                        float *ckpt, void *stream);

/* Bytes of device workspace wkv4_backward needs (has_ckpt: ckpt != NULL). */
size_t wkv4_backward_workspace_bytes(int64_t B, int64_t T, int64_t C, int has_ckpt);

/*
 * RWKV-4 WKV backward: gradients of L = sum(gy * y) for y = wkv4_forward(...).
 *   gy          [B][T][C] of `dtype`.
 *   ckpt        the checkpoints wkv4_forward wrote for the same inputs, or
 *               NULL (then they are regenerated inside `workspace`).
 *   gk, gv      [B][T][C] of `dtype`, written (not accumulated).
 *   gw, gu      [C] float32, written: dL/dw and dL/du summed over batch and
 *               time. (dL/dtime_decay = gw * w.) The batch sum is taken in a
 *               fixed order, so results are run-to-run deterministic.
 *   workspace   device scratch of at least
 *               wkv4_backward_workspace_bytes(B, T, C, ckpt != NULL) bytes,
 *               16-byte aligned; its contents on entry are ignored.
 */
wkv_status wkv4_backward(int64_t B, int64_t T, int64_t C, int dtype,
                         const float *w, const float *u,
                         const void *k, const void *v, const void *gy,
                         const float *ckpt,
                         void *gk, void *gv, float *gw, float *gu,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * RWKV-4 WKV forward with the time-mix gate fused into its output: the
 * receptance gate of RWKV_TimeMix ("代码连连看——RWKV", section
 * RWKV_TimeMix: the block output is sigmoid(r) * WKV before the output
 * projection), y = sigmoid(r) * wkv4_forward(...), in one pass over HBM.
 *   r           [B][T][C] of `dtype`: the gate input (receptance before the
 *               sigmoid), read-only.
 *   y           [B][T][C] of `dtype`, required (the gated output).
 *   ckpt        as for wkv4_forward (optional): the checkpoints do not
 *               depend on r.
 * Other arguments, errors and limits are those of wkv4_forward. r and y
 * must not overlap.
 */
wkv_status wkv4_forward_gated(int64_t B, int64_t T, int64_t C, int dtype,
                              const float *w, const float *u,
                              const void *k, const void *v, const void *r,
                              void *y, float *ckpt, void *stream);

/*
 * Gradients of L = sum(gy * y) for y = wkv4_forward_gated(...): with
 * s = sigmoid(r) and wkv the ungated output, the WKV sees the output
 * gradient gy * s, and dL/dr = gy * wkv * s * (1 - s).
 *   r           [B][T][C] of `dtype`, the gate input of the forward.
 *   gy          [B][T][C] of `dtype`, gradient of the gated output.
 *   gr          [B][T][C] of `dtype`, written: dL/dr.
 *   ckpt, gk, gv, gw, gu, workspace: as for wkv4_backward (the workspace
 *               size is wkv4_backward_workspace_bytes for the same shape).
 */
wkv_status wkv4_backward_gated(int64_t B, int64_t T, int64_t C, int dtype,
                               const float *w, const float *u,
                               const void *k, const void *v, const void *r,
                               const void *gy, const float *ckpt,
                               void *gk, void *gv, void *gr, float *gw, float *gu,
                               void *workspace, size_t workspace_bytes, void *stream);

/*
 * Time-shift mix, the prologue of RWKV_TimeMix ("代码连连看——RWKV", section
 * RWKV_TimeMix, jit_func): time_shift moves the input one token along T
 * (a zero row padded before t = 0, the last row dropped), and each of the
 * k, v, r inputs of the projections blends the token with the shifted one
 * per channel:
 *
 *     out[m][b][t][c] = x[b][t][c] * mix[m][c] + xx[b][t][c] * (1 - mix[m][c])
 *     xx[b][t] = x[b][t-1] for t > 0,  xx[b][0] = x_prev[b] (zeros if NULL)
 *
 *   n_mix       number of blends, 1..3 (3 for time_mix_k, _v, _r).
 *   x           [B][T][C] of `dtype`.
 *   mix         [n_mix][C] float32.
 *   x_prev      [B][C] of `dtype` or NULL: the token before x (the last
 *               token of the previous piece when a sequence is fed in pieces).
 *   out         [n_mix][B][T][C] of `dtype`, written; must not overlap x.
 * Alignment and C rules as for wkv4_forward; n_mix outside 1..3 is
 * WKV_ERR_INVALID_ARG; empty problems are no-ops.
 */
wkv_status wkv4_time_shift_mix(int64_t B, int64_t T, int64_t C, int dtype, int64_t n_mix,
                               const void *x, const float *mix, const void *x_prev,
                               void *out, void *stream);

/* Bytes of device workspace wkv4_time_shift_mix_backward needs. */
size_t wkv4_time_shift_mix_backward_workspace_bytes(int64_t B, int64_t T, int64_t C,
                                                    int dtype, int64_t n_mix);

/*
 * Gradients of L = sum(g * out) for out = wkv4_time_shift_mix(...):
 *   g           [n_mix][B][T][C] of `dtype`.
 *   gx          [B][T][C] of `dtype`, written:
 *               sum_m g[m][t] mix[m] + sum_m g[m][t+1] (1 - mix[m]).
 *   gmix        [n_mix][C] float32, written: sum over b, t of
 *               g[m][b][t] (x[b][t] - xx[b][t]), added in a fixed order
 *               (run-to-run deterministic).
 *   gx_prev     [B][C] of `dtype` or NULL; if given, written:
 *               sum_m g[m][b][0] (1 - mix[m]).
 *   workspace   device scratch of at least
 *               wkv4_time_shift_mix_backward_workspace_bytes(B, T, C, dtype, n_mix)
 *               bytes, 16-byte aligned; contents on entry are ignored.
 */
wkv_status wkv4_time_shift_mix_backward(int64_t B, int64_t T, int64_t C, int dtype, int64_t n_mix,
                                        const void *x, const float *mix, const void *x_prev,
                                        const void *g, void *gx, float *gmix, void *gx_prev,
                                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * Set S slot states [S][5][C] float32 to the empty past:
 * aa = bb = 0, base = -1e38, n = 0, ref = 0 (ref is set by the first token).
 */
wkv_status wkv4_state_init(int64_t S, int64_t C, float *state, void *stream);

/*
 * One batched inference call over S slots (web-rwkv's batched inference).
 *   k, v, y     [n_tokens][C] of `dtype`: the tokens of all slots packed back
 *               to back, slot 0 first; y is written for every consumed token.
 *   cu_tokens   DEVICE int32 [S+1], cu_tokens[0] = 0, nondecreasing: slot s
 *               consumes tokens cu_tokens[s] .. cu_tokens[s+1]-1 in order. A
 *               slot with no tokens is skipped and its state left untouched.
 *               A slot whose range is decreasing or exceeds n_tokens is
 *               skipped too and WKV_DEVERR_BAD_SLOT is recorded.
 *   state       [S][5][C] float32 (aa, bb, base, n, ref per channel), read
 *               and written in place: it carries each slot across calls. A
 *               slot whose base is still -1e38 (empty) takes ref from the
 *               first token it absorbs.
 * Feeding a sequence in several calls gives bit-identical y and state to
 * feeding it in one call, and bit-identical y to wkv4_forward on the same
 * tokens (all three run the same float32 step in the same order).
 */
wkv_status wkv4_chunk_step(int64_t S, int64_t C, int dtype,
                           const float *w, const float *u,
                           const void *k, const void *v, void *y, int64_t n_tokens,
                           const int32_t *cu_tokens, float *state, void *stream);

/*
 * The T = 1 fast path of wkv4_chunk_step (batched decode): every one of the S
 * slots takes exactly one token.
 *   k, v        [S][C] of `dtype`: slot s's token is row s.
 *   y           [S][C] of `dtype`, written.
 *   state       [S][5][C] float32, read and written, as for wkv4_chunk_step.
 * y and the new state are bit-identical to wkv4_chunk_step with
 * cu_tokens = {0, 1, ..., S} on the same inputs (the same float32 step in
 * the same order); a slot whose state is the empty past takes its reference
 * exponent from this token. Pointers are required (16-byte aligned); size
 * rules as for wkv4_chunk_step; S = 0 or C = 0 is a no-op. Launches one
 * kernel; no device error codes (there are no offsets to check).
 */
wkv_status wkv4_decode_step(int64_t S, int64_t C, int dtype,
                            const float *w, const float *u,
                            const void *k, const void *v, void *y,
                            float *state, void *stream);

/*
 * wkv4_backward without a workspace argument, for callers that cannot
 * allocate device memory per call (code behind a plain C interface that only
 * receives the tensors it reads and writes, or latency-critical loops that
 * must not call cudaMalloc/cudaFree). The method's source pages have no
 * counterpart: this is a deployment convenience of the library, not part
 * of the method.
 *   Arguments and results are those of wkv4_backward; the workspace is a
 *   file-scope device array of 4 MiB that every GPU loading the library
 *   keeps until the process exits.
 *   Problems whose workspace, wkv4_backward_workspace_bytes(B, T, C,
 *   ckpt != NULL), exceeds 4 MiB return WKV_ERR_UNSUPPORTED (the partial sums
 *   take 2*B*NSEG*C floats, NSEG the sequence segments of short batches, at
 *   most 8; a NULL ckpt adds the regenerated checkpoints): pass ckpt, or call
 *   wkv4_backward.
 *   The array used is the one of the current device, which must be the
 *   device of the tensors and of the stream. The first call on a device
 *   looks up the array's device address (with that device current); make
 *   that first call before any stream capture.
 *   All calls share the array: calls whose kernels overlap on the GPU race on
 *   it and must be serialised by the caller. Nothing in it needs clearing:
 *   every scratch element a call reads was written earlier in that call
 *   (after a copy wait that gave up, reported as WKV_DEVERR_WAIT_TIMEOUT, the
 *   call's results are undefined, as for wkv4_backward).
 *   Allocates nothing (no cudaMalloc, cudaFree or allocating library call).
 */
wkv_status wkv4_backward_noalloc(int64_t B, int64_t T, int64_t C, int dtype,
                                 const float *w, const float *u,
                                 const void *k, const void *v, const void *gy,
                                 const float *ckpt,
                                 void *gk, void *gv, float *gw, float *gu, void *stream);

/*
 * The failure path of the bounded waits, on demand: launches one warp that
 * waits on a barrier nothing will complete, giving up after limit_ns
 * nanoseconds (1000 .. 10^10). It records WKV_DEVERR_WAIT_TIMEOUT in the
 * device error word -- what every kernel does if a copy it waits on never
 * lands -- and returns; the context stays usable. For tests of the error
 * reporting (read it with wkv_device_error). Returns WKV_ERR_INVALID_ARG for
 * a limit outside the range.
 */
wkv_status wkv_wait_selfcheck(int64_t limit_ns, void *stream);

/* ------------------------------------------------------------------------ */
/* RWKV-6                                                                    */
/* ------------------------------------------------------------------------ */

/*
 * RWKV-6 head-state WKV forward (RWKV6_OP(head_size=K)(r, k, v, w, u,
 * with_state, init_state, state_map) on the rwkv-ops package page).
 *   K            head size; 64 is the supported value (else UNSUPPORTED).
 *   dtype        WKV_BF16 (else UNSUPPORTED).
 *   r, k, v, w   [B][T][H*K] bf16; w is the per-step decay, in (0, 1].
 *   u            [H*K] float32 (the (num_heads, head_size) bonus, flattened).
 *   init_state   NULL (every sample starts from S = 0) or
 *                [n_state][H][K][K] float32, indexed [.][h][i][j] with i the
 *                key index and j the value index.
 *   state_map    NULL or DEVICE int32 [B]: sample b starts from
 *                init_state[state_map[b]]. Without it, n_state must be 1
 *                (shared) or B (one per sample). An out-of-range entry makes
 *                that sample start from zero and records WKV_DEVERR_BAD_STATE.
 *   final_state  NULL or [B][H][K][K] float32, written: S after the last token.
 *   o            [B][T][H*K] bf16, written.
 */
wkv_status wkv6_forward(int64_t B, int64_t T, int64_t H, int64_t K, int dtype,
                        const void *r, const void *k, const void *v, const void *w,
                        const float *u,
                        const float *init_state, const int32_t *state_map, int64_t n_state,
                        float *final_state, void *o, void *stream);

/* Bytes of workspace wkv6_backward needs for K = 64 (0 for another K), with
 * nch = ceil(T / 64) chunks, each piece rounded up to a multiple of 256 bytes:
 *   2 x 4*B*H*nch*64*64   the state entering every chunk, forward (S) and
 *                         backward (G = dL/dS)
 *   4*B*H*nch*64          per-chunk partial sums of gu. */
size_t wkv6_backward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t K);

/*
 * RWKV-6 head-state WKV backward: the gradients of
 *   L = sum(dout * o) + sum(g_final * S_final)
 * for wkv6_forward with the same arguments (RWKV6_OP on the rwkv-ops package
 * page is a trained operator; its table lists the PyTorch CUDA version).
 *   K, dtype, r, k, v, w, u, init_state, state_map, n_state
 *                as wkv6_forward (K = 64, bf16 only).
 *   dout         [B][T][H*K] bf16: dL/do.
 *   g_final      NULL (zero) or [B][H][K][K] float32: dL/dS after the last token.
 *   gr, gk, gv   [B][T][H*K] bf16, written.
 *   glogw        [B][T][H*K] bf16, written: w * dL/dw, the gradient with
 *                respect to log w (w = exp(-exp(d)) gives dL/dd = -exp(d) glogw).
 *                It is formed without dividing by w, so it stays accurate
 *                where w is tiny; dL/dw itself is glogw / w.
 *   gu           [H*K] float32, written: summed over samples and tokens in a
 *                fixed order (deterministic).
 *   g_init       NULL or [B][H][K][K] float32, written: dL/dS_{-1} of each
 *                sample (adding rows that share an init_state entry is the
 *                caller's).
 *   workspace    device memory of workspace_bytes >= wkv6_backward_workspace_bytes,
 *                16-byte aligned; overwritten, nothing in it needs clearing.
 * Every device pointer must be 16-byte aligned. The forward kernel runs twice
 * (on the inputs, recording the state entering every 64-token chunk, and as
 * the time-reversed recurrence of k, r, dout, w from g_final, which gives gv,
 * g_init and dL/dS at every chunk boundary); then one tensor-core CTA per
 * chunk forms gr, gk, glogw and gu partials, and a last kernel sums gu.
 * Returns WKV_ERR_INVALID_ARG for a missing pointer or a short workspace,
 * WKV_ERR_UNSUPPORTED for K != 64 or a dtype other than WKV_BF16.
 */
wkv_status wkv6_backward(int64_t B, int64_t T, int64_t H, int64_t K, int dtype,
                         const void *r, const void *k, const void *v, const void *w,
                         const float *u,
                         const float *init_state, const int32_t *state_map, int64_t n_state,
                         const void *dout, const float *g_final,
                         void *gr, void *gk, void *gv, void *glogw, float *gu, float *g_init,
                         void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* RWKV-7                                                                    */
/* ------------------------------------------------------------------------ */

/*
 * RWKV-7 generalized delta rule forward (generalized_delta_rule / rwkv7_op on
 * the rwkv-ops package page: r, w, k, v, a, b with w the decay in log space,
 * initial and final state [N, H, K, V]). Per head, with the key index j and
 * the value index i of the state S[j][i]:
 *   S_t = (diag(e^{w_t}) + b_t a_t^T) S_{t-1} + k_t^T v_t,    o_t = r_t S_t
 * (the page gives the interface; this diagonal-plus-rank-one transition is
 * the recurrence taken for it).
 *   K            head size (= value size); 64 is the supported value.
 *   dtype        WKV_BF16 (else UNSUPPORTED).
 *   r, w, k, v, a, b  [B][T][H*K] bf16.
 *   init_state   NULL (every sample starts from S = 0) or [B][H][K][K]
 *                float32 indexed [b][h][j][i] (one sequence per sample).
 *   final_state  NULL or [B][H][K][K] float32, written: S after the last token.
 *   o            [B][T][H*K] bf16, written.
 * One CTA of 128 threads walks each head's sequence in order (fp32 state).
 * T = 1 is the decode step of rwkv7_op_rnn.
 */
wkv_status wkv7_forward(int64_t B, int64_t T, int64_t H, int64_t K, int dtype,
                        const void *r, const void *w, const void *k, const void *v,
                        const void *a, const void *b,
                        const float *init_state, float *final_state, void *o, void *stream);

/* Bytes of device workspace wkv7_backward needs (0 for an unsupported shape). */
size_t wkv7_backward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t K);

/*
 * Gradients of L = sum(dout * o) + sum(g_final * S_final) for
 * o, S_final = wkv7_forward(...) on the same inputs (generalized_delta_rule
 * of the rwkv-ops package page carries gradients). With G = dL/dS_t walked
 * down from the last token (j key, i value, d = e^{w_t}, sa = a_t S_{t-1}):
 *   G += r_t^T dout_t;  dr_t = S_t dout_t;  dk_t = G v_t;  db_t = G sa;
 *   dw_t = d o rowsum(G o S_{t-1});  dsa = b_t G;  dv_t = k_t G;
 *   da_t = S_{t-1} dsa;  G <- diag(d) G + a_t^T dsa;  d_init = G at the end.
 *   r, w, k, v, a, b, dout  [B][T][H*K] bf16 (w the log decay, as for
 *               wkv7_forward); dw is the gradient with respect to w.
 *   init_state  [B][H][K][K] float32 or NULL (zeros), as for the forward.
 *   g_final     [B][H][K][K] float32 or NULL (no final-state term).
 *   dr, dw, dk, dv, da, db  [B][T][H*K] bf16, written.
 *   d_init      [B][H][K][K] float32, written (dL/dS_init).
 *   workspace   device scratch of at least wkv7_backward_workspace_bytes
 *               bytes: the state before every 4th token, written by a
 *               checkpoint sweep of the forward kernel, read back per group.
 * bf16 and K = 64 only (WKV_ERR_UNSUPPORTED otherwise). T = 0 gives
 * d_init = g_final (or 0). Launches two kernels on `stream`.
 */
wkv_status wkv7_backward(int64_t B, int64_t T, int64_t H, int64_t K, int dtype,
                         const void *r, const void *w, const void *k, const void *v,
                         const void *a, const void *b, const float *init_state,
                         const void *dout, const float *g_final,
                         void *dr, void *dw, void *dk, void *dv, void *da, void *db,
                         float *d_init, void *workspace, size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* WKV_B200_H */
