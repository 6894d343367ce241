/*
 * wkv7.h -- C ABI of the B200 (sm_100a) WKV-7 library.
 *
 * The WKV-7 operator is the time-mixing recurrence of RWKV-7 "Goose". Per batch
 * element b and head h it carries an N x N fp32 state S (row i = value channel,
 * column j = key channel) through the tokens t = 0..T-1:
 *
 *     S_t = S_{t-1} diag(w_t) - (S_{t-1} kk_t)(kk_t * a_t)^T + v_t k_t^T
 *     y_t = S_t r_t
 *
 * (RWKV-7 rebuttal page, numpy time_mixing listing: the update and readout lines;
 * ARWKV verdict page, key_machinery: the same update in row-vector form.)
 * The optional epilogue (same listing: group_norm lambda and the bonus line)
 * replaces y_t, per head, by
 *
 *     (y_t - mean) / sqrt(var + gn_eps) * ln_w[h] + ln_b[h]
 *       + (sum_j r_t[j] k_t[j] r_k[h][j]) * v_t
 *
 * with the population variance over the N channels of the head.
 *
 * Conventions for every entry point:
 *   - N is 64 on every path, or 128 (the larger head size the pages name as the next
 *     one) on the sequential scan, its epilogue, the decode step and the backward pass.
 *     The chunked algorithms take N = 64 only: WKV7_ALGO_CHUNK / SPLIT with N = 128
 *     return WKV7_ERR_UNSUPPORTED, and WKV7_ALGO_AUTO runs N = 128 on the scan.
 *   - Token tensors r, w, k, v, kk, a are [B][T][H][N] row-major (decode: [B][H][N]),
 *     all of the dtype given by `dt`. States are [B][H][N][N] fp32 row-major.
 *     y is fp32 with the layout of the token tensors.
 *   - Every pointer is a device pointer (cudaMalloc / caching allocator / managed)
 *     on the current device, 16-byte aligned. Host pointers are rejected before
 *     any launch (WKV7_ERR_ARG), as are pointers whose allocation is too small
 *     for the stated sizes (when the driver can report the allocation's range).
 *   - The caller owns every buffer. The library never allocates device memory and
 *     never synchronises; work is enqueued on `stream` (a cudaStream_t, NULL for
 *     the legacy default stream). Asynchronous faults appear at the caller's next
 *     synchronisation, as for any CUDA kernel.
 *   - Input contract (not validated on the hot path): kk is already L2-normalised
 *     per head, k is the replacement key, w is the decay multiplier in (0, 1],
 *     a is the in-context learning rate (any finite value is accepted).
 *   - Errors are returned as wkv7_status; nothing is thrown across the ABI.
 *     wkv7_last_error() gives a human-readable detail for the calling thread.
 */
#ifndef WKV7_H
#define WKV7_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define WKV7_API __attribute__((visibility("default")))
#else
#define WKV7_API
#endif

#define WKV7_ABI_VERSION 6
#define WKV7_HEAD_SIZE 64
#define WKV7_MAX_SEGMENTS 8   /* CTAs per (b, h) of WKV7_ALGO_SPLIT (one thread-block cluster) */

typedef enum wkv7_status {
    WKV7_OK = 0,
    WKV7_ERR_ARG = 1,          /* null / host / too-small pointer, bad size or option   */
    WKV7_ERR_UNSUPPORTED = 2,  /* valid request the library does not implement (N not 64 or 128,
                                  or 128 on a path that takes 64 only) */
    WKV7_ERR_ALIGN = 3,        /* a pointer is not 16-byte aligned                       */
    WKV7_ERR_CUDA = 4,         /* a CUDA call or kernel launch failed                    */
    WKV7_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up (see poll below)    */
    WKV7_ERR_WORKSPACE = 6     /* workspace missing or smaller than wkv7_workspace_bytes */
} wkv7_status;

typedef enum wkv7_dtype {
    WKV7_F32 = 0,
    WKV7_BF16 = 1
} wkv7_dtype;

typedef enum wkv7_algo {
    WKV7_ALGO_AUTO = 0,   /* pick from dtype, T and B*H                                  */
    WKV7_ALGO_SEQ = 1,    /* token-by-token scan, fp32 FMA; any T, any dtype             */
    WKV7_ALGO_CHUNK = 2,  /* chunked prefill on tcgen05 tensor cores, fp32 chunk carry;  */
                          /* bf16 inputs, chunk 64, w >= exp(-e^-1/2) as on the pages      */
    WKV7_ALGO_SPLIT = 3   /* chunked prefill with the chunks of one (b, h) spread over   */
                          /* `segments` CTAs of a thread-block cluster: CTA r takes      */
                          /* chunks r, r + segments, ... and passes the fp32 state to    */
                          /* CTA r + 1 through distributed shared memory (chunk carry    */
                          /* S_{c+1} = S_c P_c + Q_c, the chain being the only serial    */
                          /* part); same inputs and limits as CHUNK                      */
} wkv7_algo;

/* Options of wkv7_forward. Obtain defaults with wkv7_opts_default(). */
typedef struct wkv7_opts {
    int algo;             /* wkv7_algo                                                   */
    int chunk;            /* 0 (default) or 64: the chunked kernel's chunk; 16 and 32 are */
                          /* accepted and run on the scan under AUTO (CHUNK/SPLIT refuse) */
    int snap_every;       /* 0 = no snapshots; else store S after every snap_every tokens */
    float *snapshots;     /* [B][T / snap_every][H][N][N] fp32, required if snap_every>0 */
    const float *ln_w;    /* epilogue: all three NULL (off) or all three [H][N] fp32     */
    const float *ln_b;
    const float *r_k;
    float gn_eps;         /* epilogue epsilon added to the variance (default 64e-5)      */
    int segments;         /* WKV7_ALGO_SPLIT: CTAs per (b, h), 1..WKV7_MAX_SEGMENTS, or  */
                          /* 0 = automatic (AUTO always chooses; CHUNK uses one)         */
    unsigned int handoff_wait_us;   /* limit of each wait for a state (or for its receipt)    */
                          /* between the CTAs of one head in split mode, in microseconds; */
                          /* 0 = the default 2 s. Every other device-side wait keeps 2 s. */
    int withhold_handoff; /* failure-path test only: 1 = in split mode the first CTA of   */
                          /* each head withholds its first state hand-off, so the waiting */
                          /* CTA's bounded wait runs out, the kernel records the error    */
                          /* and returns (wkv7_poll_device_error then gives               */
                          /* WKV7_ERR_TIMEOUT; y and S_T are incomplete). Accepted only   */
                          /* with WKV7_ALGO_SPLIT and segments >= 2; 0 = normal.          */
} wkv7_opts;

/* Fills *opts with the defaults: AUTO, default chunk, no snapshots, no epilogue,
 * gn_eps = 64e-5, automatic segments, default hand-off wait limit, no withheld hand-off. */
WKV7_API void wkv7_opts_default(wkv7_opts *opts);

/*
 * Prefill / full-sequence forward.
 *
 * Inputs  r, w, k, v, kk, a : [B][T][H][N] of dtype dt.
 *         S0                : [B][H][N][N] fp32, or NULL for a zero initial state.
 * Outputs y                 : [B][T][H][N] fp32 (epilogue applied when enabled).
 *         S_T               : [B][H][N][N] fp32 final state, or NULL. May equal S0
 *                             (in-place hand-off); must not otherwise overlap inputs.
 *         opts->snapshots   : states after tokens snap_every * m, m = 1..T/snap_every.
 * Workspace: device memory of at least wkv7_workspace_bytes(...) bytes for the same
 *         arguments (0 bytes for most configurations; NULL is then allowed).
 * B, H >= 1; T >= 0 (T = 0 copies S0 to S_T, or zeros when S0 is NULL).
 * (RWKV-7 paper summary, section 8: chunked pre-fill with a user-chosen chunk,
 * forward inference with and without state storage.)
 */
WKV7_API wkv7_status wkv7_forward(int B, int T, int H, int N, wkv7_dtype dt,
                         const void *r, const void *w, const void *k, const void *v,
                         const void *kk, const void *a,
                         const float *S0, float *y, float *S_T,
                         const wkv7_opts *opts,
                         void *workspace, size_t workspace_bytes,
                         void *stream);

/*
 * Prefill / full-sequence forward from the raw time-mixing values: the pre-processing the
 * pages place before the update (rebuttal page, the numpy time_mixing listing: the decay, the
 * in-context learning rate, the removal key and its normalisation, the key update) is
 * done on the device in the load stage of whichever kernel runs (chunked or scan, and in the
 * separate epilogue kernel for the bonus), then the same recurrence and epilogue as
 * wkv7_forward:
 *     w  = exp(-sigmoid(w_logit) / sqrt(e))          a  = sigmoid(a_logit)
 *     kk = (k * k_k) / max(||k * k_k||_2, 1e-12)     (per head, over its N channels)
 *     k~ = k + k * (a - 1) * k_a                     (kk uses k, the update and bonus use k~)
 *
 * Inputs  r, w_logit, k, v, a_logit : [B][T][H][N] of dtype dt (k is the key before its
 *                                     update).
 *         k_k                       : [H][N] fp32, required.   k_a : [H][N] fp32 or NULL (= 0).
 * Everything else (S0, y, S_T, opts, workspace, errors) as wkv7_forward; the prepared values
 * are never written to memory. WKV7_ERR_ARG also when k_k is NULL (T > 0).
 */
WKV7_API wkv7_status wkv7_forward_raw(int B, int T, int H, int N, wkv7_dtype dt,
                             const void *r, const void *w_logit, const void *k, const void *v,
                             const void *a_logit, const float *k_k, const float *k_a,
                             const float *S0, float *y, float *S_T,
                             const wkv7_opts *opts,
                             void *workspace, size_t workspace_bytes,
                             void *stream);

/*
 * wkv7_forward on HOST buffers: the end-to-end path for a caller whose inputs and results live
 * in host memory. Every pointer argument (r, w, k, v, kk, a, S0, y, S_T, opts->snapshots and the
 * epilogue parameters opts->ln_w, ln_b, r_k) is a host pointer with the layout of wkv7_forward;
 * page-locked (pinned) memory lets the copies run asynchronously and overlap. The batch is cut
 * into slices of whole sequences (up to 8, at least 24 MB of input each); each slice's
 * host-to-device copies run on a copy stream of the library, its forward on `stream`, its
 * device-to-host copies on a second copy stream, so copies in both directions overlap the
 * kernels of the other slices. The device copies live in `workspace` (device memory of at least
 * wkv7_forward_host_workspace_bytes(...) bytes, 256-byte aligned): nothing is allocated. The
 * library makes its two copy streams and their events once per device (first call on a device:
 * make it before any stream capture).
 * Returns once everything is enqueued; the host outputs are complete when `stream` is
 * (cudaStreamSynchronize). Calls on one device are serialised while they enqueue; a call's
 * copies start after all work already on `stream`, so the workspace may be reused by the next
 * call on the same stream. Host output buffers must not overlap the inputs.
 * Errors as wkv7_forward, plus WKV7_ERR_ARG for device or managed pointers (use wkv7_forward),
 * WKV7_ERR_WORKSPACE, WKV7_ERR_ALIGN for a workspace not 256-byte aligned.
 * (RWKV-7 paper summary, section 8: the forward over a sequence; the host path itself has no
 * counterpart on the pages.)
 */
WKV7_API wkv7_status wkv7_forward_host(int B, int T, int H, int N, wkv7_dtype dt,
                              const void *r, const void *w, const void *k, const void *v,
                              const void *kk, const void *a, const float *S0, float *y, float *S_T,
                              const wkv7_opts *opts, void *workspace, size_t workspace_bytes,
                              void *stream);

/* Device workspace bytes of wkv7_forward_host: device copies of every input and output of the
 * whole batch (S0 and S_T always counted) plus wkv7_workspace_bytes. 0 for invalid sizes. */
WKV7_API size_t wkv7_forward_host_workspace_bytes(int B, int T, int H, int N, wkv7_dtype dt,
                                                  const wkv7_opts *opts);

/*
 * Backward pass of wkv7_forward (no epilogue): the gradients of every input for the scalar
 * L = <dy, y> + <dS_T, S_T>, in fp32. The pages time a backward pass and state the precision
 * of an fp32 one (RWKV-7 rebuttal page, the answer on numerical precision; paper summary,
 * the speed figures for the forward that keeps its states and for the backward); the
 * operation is the chain rule through the update and readout of the rebuttal page's numpy
 * time_mixing listing, token by token in reverse:
 *     dS += dy_t r_t^T, dr_t = S_t^T dy_t, dv_t = dS k_t, dk_t = dS^T v_t,
 *     dw_t = column sums of S_{t-1} (.) dS, db = -dS^T (S_{t-1} kk_t), ds = -dS (kk_t a_t),
 *     dkk_t = S_{t-1}^T ds + db (.) a_t, da_t = db (.) kk_t, dS_{t-1} = dS diag(w_t) + ds kk_t^T.
 * The states S_{t-1} are recomputed on the device, starting from S0 and from the forward's
 * snapshots when given: pass the snapshots a wkv7_forward call wrote with
 * the same snap_every (the states after tokens snap_every, 2 snap_every, ...) to bound the
 * recomputation and the workspace; snap_every = 0 recomputes from S0 alone.
 *
 * Inputs  r, w, k, v, kk, a : [B][T][H][N] of dtype dt, the forward's inputs.
 *         S0                : [B][H][N][N] fp32 or NULL (zeros).
 *         snapshots         : [B][T/snap_every][H][N][N] fp32; required when snap_every > 0
 *                             and T >= snap_every, else ignored.
 *         dy                : [B][T][H][N] fp32 gradient of y (required when T > 0).
 *         dS_T              : [B][H][N][N] fp32 or NULL (zero gradient on the final state).
 * Outputs dr, dw, dk, dv, dkk, da : [B][T][H][N] fp32 (required when T > 0).
 *         dS0               : [B][H][N][N] fp32 or NULL; may equal dS_T exactly (in place).
 * Workspace: at least wkv7_backward_workspace_bytes(B, T, H, N, snap_every) bytes of device
 * memory (the recomputation's checkpoints, one state per 4 tokens of a segment at N = 64, per 2
 * tokens at N = 128); it must not overlap any other argument and its contents need no
 * initialisation.
 * Errors as wkv7_forward: WKV7_ERR_ARG for sizes, NULL required pointers, snap_every < 0,
 * missing snapshots, overlapping outputs, host or too-small buffers; WKV7_ERR_ALIGN;
 * WKV7_ERR_UNSUPPORTED for N other than 64 and 128; WKV7_ERR_WORKSPACE. T = 0 copies dS_T (or
 * zeros) to dS0.
 */
WKV7_API wkv7_status wkv7_backward(int B, int T, int H, int N, wkv7_dtype dt,
                          const void *r, const void *w, const void *k, const void *v,
                          const void *kk, const void *a, const float *S0,
                          const float *snapshots, int snap_every,
                          const float *dy, const float *dS_T,
                          float *dr, float *dw, float *dk, float *dv, float *dkk, float *da,
                          float *dS0, void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of workspace wkv7_backward needs: B * H * ceil(K / 4) * N * N * 4 at N = 64 and
 * B * H * ceil(K / 2) * N * N * 4 at N = 128, with K the snapshot interval (or T when snap_every
 * is 0 or >= T); 0 when T = 0 or an argument is invalid. Host only. */
WKV7_API size_t wkv7_backward_workspace_bytes(int B, int T, int H, int N, int snap_every);

/*
 * wkv7_backward without a workspace argument and without any allocation: the checkpoints go
 * to a scratch array of 32 MiB (33,554,432 bytes) that the library's device code holds at
 * module scope; its address is looked up once per device. This entry has no counterpart on
 * the pages; it serves callers that cannot provide device memory.
 * Limit: wkv7_backward_workspace_bytes(B, T, H, N, snap_every) must be at most 32 MiB
 * (2048 checkpoints: B * H * ceil(K / 4) <= 2048, K the snapshot interval, or T without
 * snapshots); larger requests return WKV7_ERR_WORKSPACE before anything is enqueued.
 * Nothing in the scratch needs to start at zero (every checkpoint is written before it is read).
 * The scratch is shared by every call on a device: calls that may overlap in time (different
 * streams, or host threads without ordering between them) race on it and corrupt each other's
 * results; order such calls on one stream. The first call on a device looks up the scratch's
 * device address (make it before any stream capture); the address is kept for later calls
 * and belongs to that device's context, so it is not valid after cudaDeviceReset. Arguments,
 * outputs and errors otherwise as wkv7_backward.
 */
WKV7_API wkv7_status wkv7_backward_static(int B, int T, int H, int N, wkv7_dtype dt,
                          const void *r, const void *w, const void *k, const void *v,
                          const void *kk, const void *a, const float *S0,
                          const float *snapshots, int snap_every,
                          const float *dy, const float *dS_T,
                          float *dr, float *dw, float *dk, float *dv, float *dkk, float *da,
                          float *dS0, void *stream);

/*
 * One RWKV-7 time-mixing layer over a sequence (RWKV-7 rebuttal page, the numpy time_mixing
 * listing, applied token after token with state, previous token and the first layer's values
 * carried along). With C = H * N channels, M = B * T token rows, x_p the previous token
 * (last_x for t = 0) and every vector below per token:
 *     x_m = x + m (x_p - x) for the six mixes m in {mr, mw, mk, mv, ma, mg}
 *     r = Wr x_r, k = Wk x_k, v = Wv x_v
 *     w_logit = tanh(x_w Ww1) Ww2 + w_bias, a_logit = x_a Wa1 Wa2 + a_bias
 *     v <- v + (v0 - v) sigmoid(x_v Wv1 Wv2 + v_bias)          (only when v0 is given)
 *     g = sigmoid(x_g Wg1) Wg2
 *     y = wkv7_forward_raw(r, w_logit, k, v, a_logit, k_k, k_a) with the epilogue (ln_w, ln_b, r_k)
 *     out = Wo (y * g)
 * Every projection is this library's GEMM: tcgen05 tensor cores with bf16 operands and fp32
 * accumulation for WKV7_BF16, the fp32 FMA pipe for WKV7_F32. The seven products of the mixed x
 * (r, k, v and the four low-rank first factors) run as one launch and the four second factors as
 * another; the token-shift mixes are formed in the operand load (fp32 arithmetic, rounded once to
 * dt) and tanh, sigmoid, the biases and the value residual in the store. r, k, v, the two logits
 * and the low-rank hidden values are stored in dt, g and y in fp32; y * g is formed in one
 * element-wise pass, rounded to dt, before the output projection. Each call also copies the
 * low-rank factors, transposed and zero-padded to multiples of 64, into the workspace.
 *
 * dims:   H, N (64, or 128 on the scan), low-rank widths d_w, d_a, d_v, d_g (>= 1).
 * params: fp32 mixes and biases [C]; fp32 r_k, k_k, k_a, ln_w, ln_b [H][N] (k_a may be NULL);
 *         Wr, Wk, Wv, Wo [C][C] of dt applied as W x (row = output channel);
 *         Ww1, Wa1, Wv1, Wg1 [C][d] and Ww2, Wa2, Wv2, Wg2 [d][C] of dt applied as x W
 *         (Wv1, Wv2, v_bias unused when v0 is NULL).
 * x       [B][T][C] dt.     last_x [B][C] dt or NULL (zeros).
 * v0      [B][T][C] dt: the first layer's values; NULL means this is the first layer.
 * S       [B][H][N][N] fp32, read and updated in place (NULL: zero state, not returned).
 * out     [B][T][C] fp32.   v0_out [B][T][C] dt or NULL: receives v when v0 is NULL.
 * last_x_out [B][C] dt or NULL: receives x[:, T-1]; may be last_x itself (in place).
 * opts: algorithm, chunk, segments and snapshots of the recurrence (its epilogue fields are
 *       replaced by params'); NULL = defaults.
 * Workspace: wkv7_layer_workspace_bytes(B, T, dt, dims) bytes, not overlapping any argument.
 * Errors: WKV7_ERR_ARG (sizes, NULL dims / params / required pointers, overlapping outputs,
 * host or too-small buffers, v0 without Wv1 / Wv2 / v_bias), WKV7_ERR_ALIGN (every
 * pointer 16-byte aligned), WKV7_ERR_UNSUPPORTED (N), WKV7_ERR_WORKSPACE, WKV7_ERR_CUDA (a launch
 * failed; the message names the step). T = 0 only copies last_x.
 */
typedef struct {
    int H, N;
    int d_w, d_a, d_v, d_g;
} wkv7_layer_dims;

typedef struct {
    const float *mr, *mw, *mk, *mv, *ma, *mg;
    const float *w_bias, *a_bias, *v_bias;
    const float *r_k, *k_k, *k_a, *ln_w, *ln_b;
    const void *Wr, *Wk, *Wv, *Wo;
    const void *Ww1, *Ww2, *Wa1, *Wa2, *Wv1, *Wv2, *Wg1, *Wg2;
} wkv7_layer_params;

WKV7_API wkv7_status wkv7_layer_forward(int B, int T, wkv7_dtype dt, const wkv7_layer_dims *dims,
                          const wkv7_layer_params *params, const void *x, const void *last_x,
                          const void *v0, float *S, float *out, void *v0_out, void *last_x_out,
                          const wkv7_opts *opts, void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes of wkv7_layer_forward (0 when T = 0 or the arguments are invalid). Host only. */
WKV7_API size_t wkv7_layer_workspace_bytes(int B, int T, wkv7_dtype dt, const wkv7_layer_dims *dims);

/*
 * The epilogue on its own, out of place (RWKV-7 rebuttal page, numpy time_mixing listing: the
 * group_norm lambda and the bonus line after the readout): per (b, t, h) row of N channels
 *     out = (y - mean(y)) / sqrt(var(y) + gn_eps) * ln_w + ln_b + (sum_j r_j k_j r_k[j]) v
 * with the population variance: the operation wkv7_forward applies when opts carries ln_w, ln_b
 * and r_k. A training step runs wkv7_forward without the epilogue, keeps its readout y for the
 * backward, and applies this.
 * y, out  [B][T][H][N] fp32 (out may be y: in place; otherwise they must not overlap).
 * r, k, v [B][T][H][N] of dt (prepared inputs: k is the replacement key).
 * ln_w, ln_b, r_k [H][N] fp32; gn_eps > 0 (64e-5 in the pages). N 64 or 128.
 * Errors: WKV7_ERR_ARG, WKV7_ERR_ALIGN (every pointer 16-byte aligned), WKV7_ERR_UNSUPPORTED (N),
 * WKV7_ERR_CUDA. T = 0 does nothing.
 */
WKV7_API wkv7_status wkv7_epilogue(int B, int T, int H, int N, wkv7_dtype dt, const float *y, const void *r,
                                   const void *k, const void *v, const float *ln_w, const float *ln_b,
                                   const float *r_k, float gn_eps, float *out, void *stream);

/*
 * Backward of wkv7_epilogue for L = <dout, out>. The pages print the forward only; this is its
 * chain rule. With yn the normalised row, inv its inverse standard deviation and
 * beta = sum_j r_j k_j r_k[j], per row:
 *     dv = beta dout,  dbeta = sum_i dout_i v_i,  dr = dbeta k r_k,  dk = dbeta r r_k,
 *     dy = inv (g - mean(g) - yn mean(g yn))  with g = dout ln_w,
 * and over all rows dr_k = sum dbeta r k, dln_w = sum dout yn, dln_b = sum dout.
 * Inputs as wkv7_epilogue (y: the readout before the epilogue) plus dout [B][T][H][N] fp32.
 * Outputs (fp32, overwritten, no overlap with each other or the inputs): dy (the gradient that
 * wkv7_backward takes as its dy), the bonus's share of dr, dk, dv [B][T][H][N] (add them to
 * wkv7_backward's), dln_w, dln_b, dr_k [H][N]. The parameter sums run in a fixed order, so
 * repeated calls give identical results.
 * Workspace: wkv7_epilogue_backward_workspace_bytes(B, T, H, N) bytes. Errors as wkv7_epilogue,
 * plus WKV7_ERR_WORKSPACE. T = 0 writes zero parameter gradients.
 */
WKV7_API size_t wkv7_epilogue_backward_workspace_bytes(int B, int T, int H, int N);
WKV7_API wkv7_status wkv7_epilogue_backward(int B, int T, int H, int N, wkv7_dtype dt, const float *y,
                                            const void *r, const void *k, const void *v, const float *ln_w,
                                            const float *ln_b, const float *r_k, float gn_eps, const float *dout,
                                            float *dy, float *dr, float *dk, float *dv, float *dln_w,
                                            float *dln_b, float *dr_k, void *workspace, size_t workspace_bytes,
                                            void *stream);

/*
 * One decode step for every (b, h): the recurrence for a single token, with the
 * state read and written in place.
 *
 * Inputs  r, w, k, v, kk, a : [B][H][N] of dtype dt.
 * In/out  S                 : [B][H][N][N] fp32, updated in place.
 * Output  y                 : [B][H][N] fp32 readout of the updated state.
 * (RWKV-7 paper summary, section 8: single-token inference at constant memory.)
 */
WKV7_API wkv7_status wkv7_decode_step(int B, int H, int N, wkv7_dtype dt,
                             const void *r, const void *w, const void *k, const void *v,
                             const void *kk, const void *a,
                             float *S, float *y, void *stream);

/*
 * wkv7_decode_step with the fused group_norm + bonus epilogue of wkv7_forward: the head's N
 * readouts are normalised over the head (population variance plus gn_eps), scaled by ln_w and
 * shifted by ln_b, and (sum_j r_j k_j r_k[j]) v is added; y receives the result. ln_w, ln_b,
 * r_k: [H][N] fp32, all three or none (none = wkv7_decode_step); gn_eps > 0 when they are given
 * (64e-5 in the pages). Other arguments and errors as wkv7_decode_step; the parameters must be
 * 16-byte aligned device memory. (Rebuttal page, the numpy time_mixing listing, output lines.)
 */
WKV7_API wkv7_status wkv7_decode_step_ex(int B, int H, int N, wkv7_dtype dt,
                                         const void *r, const void *w, const void *k, const void *v,
                                         const void *kk, const void *a, float *S, float *y,
                                         const float *ln_w, const float *ln_b, const float *r_k,
                                         float gn_eps, void *stream);

/*
 * One decode step from the raw time-mixing values, the pre-processing of wkv7_forward_raw done in
 * the step's load (w = exp(-sigmoid(w_logit) / sqrt(e)), a = sigmoid(a_logit),
 * kk = (k * k_k) / max(||k * k_k||_2, 1e-12) over the head's channels, k~ = k + k (a - 1) k_a;
 * kk uses k, the update and the bonus use k~), with the optional epilogue of
 * wkv7_decode_step_ex. Inputs r, w_logit, k, v, a_logit: [B][H][N] of dtype dt; k_k [H][N] fp32
 * required, k_a [H][N] fp32 or NULL (= 0). S, y, the epilogue arguments and the errors as
 * wkv7_decode_step_ex; WKV7_ERR_ARG also when k_k is NULL.
 */
WKV7_API wkv7_status wkv7_decode_step_raw(int B, int H, int N, wkv7_dtype dt,
                                          const void *r, const void *w_logit, const void *k, const void *v,
                                          const void *a_logit, const float *k_k, const float *k_a,
                                          float *S, float *y, const float *ln_w, const float *ln_b,
                                          const float *r_k, float gn_eps, void *stream);

/*
 * Synchronises `stream`, then reports whether a kernel of this library gave up one
 * of its bounded device-side waits since the last call (WKV7_ERR_TIMEOUT; the
 * affected outputs are then incomplete) and clears the flag. Kernels never trap or
 * spin forever: a wait that exceeds its limit (2 s) records the error and returns.
 */
WKV7_API wkv7_status wkv7_poll_device_error(void *stream);

/*
 * The path wkv7_forward takes for these arguments on the current device, without running
 * anything: *algo = WKV7_ALGO_SEQ or WKV7_ALGO_CHUNK, and *segments = CTAs per (b, h) of the
 * chunked path (1: one CTA per head; 2..WKV7_MAX_SEGMENTS: the chunks of a head spread over a
 * thread-block cluster) or 0 for the scan; *launches = kernel launches of the call (1 or 2;
 * 0 for T = 0 without a state copy). When the heads fill whole waves of the GPU and part of
 * another, AUTO may run the whole waves with one CTA per head and the rest in a second launch
 * with more; *segments then reports the second launch. Reads the current device's SM count and cluster
 * occupancy (WKV7_ERR_CUDA without a usable device); argument errors as in wkv7_forward.
 * T = 0 (state copy only) and the scan report SEQ and 0 without touching the device.
 * This query has no counterpart on the pages; it reports the dispatch of this library.
 */
WKV7_API wkv7_status wkv7_plan(int B, int T, int H, int N, wkv7_dtype dt, const wkv7_opts *opts,
                               int *algo, int *segments, int *launches);

/* Bytes of device workspace wkv7_forward needs for these arguments (opts may be NULL). */
WKV7_API size_t wkv7_workspace_bytes(int B, int T, int H, int N, wkv7_dtype dt, const wkv7_opts *opts);

/* Static string naming a status. */
WKV7_API const char *wkv7_status_string(wkv7_status status);

/* Detail of the last error returned on the calling thread ("" if none). */
WKV7_API const char *wkv7_last_error(void);

/*
 * Peak-rate probes (no counterpart on the pages): kernels that keep one pipe busy and nothing
 * else, for measuring the roofline denominators on the device at hand. Each enqueues one launch
 * on `stream` and stores in *flops the floating-point operations it performs; time the launch
 * with CUDA events on that stream and divide.
 *   wkv7_probe_fp32_fma: `blocks` CTAs of 256 threads, each thread `iters` x 128 fused
 *     multiply-adds on 8 independent chains (2 flops each). blocks, iters >= 1.
 *   wkv7_probe_tf32_mma: one CTA per SM issuing `iters` x 4 tcgen05.mma kind::tf32 of
 *     M = 128, N = n (64, 128 or 256), K = 8 back to back into tensor memory. iters >= 1.
 * WKV7_ERR_ARG for other values, WKV7_ERR_CUDA for a failed launch; a bounded wait that gives
 * up is reported by wkv7_poll_device_error. Host pointers only for `flops`.
 */
WKV7_API wkv7_status wkv7_probe_fp32_fma(int blocks, int iters, void *stream, double *flops);
WKV7_API wkv7_status wkv7_probe_tf32_mma(int n, int iters, void *stream, double *flops);

/* WKV7_ABI_VERSION of the loaded library. */
WKV7_API int wkv7_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* WKV7_H */
