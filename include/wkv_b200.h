/*
 * wkv_b200.h -- C ABI of the B200 (sm_100a) RWKV-4 WKV forward and
 * per-channel diagonal linear scan library (libwkv_b200.so).
 *
 * Operations
 * ----------
 * wkv_forward / wkv_forward_bf16
 *   The RWKV-4 time-mixing WKV operator, eq. (14) of "RWKV：基于RNN的LLM"
 *   (section 二.1, Time-mixing block), written 0-based: for every batch row
 *   b, channel c and step t,
 *
 *     y[b,t,c] = ( sum_{i<t} e^{-(t-1-i) w[c] + k[b,i,c]} v[b,i,c] + e^{u[c] + k[b,t,c]} v[b,t,c] )
 *              / ( sum_{i<t} e^{-(t-1-i) w[c] + k[b,i,c]}          + e^{u[c] + k[b,t,c]} )
 *
 *   w is the per-channel decay, non-negative per eq. (10) of the same page
 *   (section 一.2); u is the bonus of the current token.  y[b,0,c] = v[b,0,c].
 *
 * diag_scan
 *   The per-channel diagonal linear recurrence the LRU and minGRU pages reduce
 *   their RNNs to ("Were RNNs All We Needed?", model-architecture section:
 *   v_t = a_t (.) v_{t-1} + b_t; review of "Resurrecting Recurrent Neural
 *   Networks for Long Sequences", linear-RNN section):
 *
 *     h[b,t,d] = a[b,t,d] * h[b,t-1,d] + b[b,t,d],    h[b,-1,d] = h0[b,d] (or 0).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout    k, v, y, a, b, h are dense row-major [B, T, C] (or [B, T, D])
 *           tensors with the channel index fastest; w, u are [C]; h0 is [B, D].
 * Memory    every pointer is a DEVICE pointer on the current CUDA device,
 *           owned by the caller.  Outputs must not overlap inputs.
 * Streams   calls are asynchronous on `stream` (NULL = legacy default stream):
 *           a return of WKV_OK means the work was queued.
 * Types     fp32 entry points read and write IEEE float.  wkv_forward_bf16
 *           reads k, v and writes y as bfloat16 bit patterns (wkv_bf16_t),
 *           computes in fp32 and rounds y to nearest even; w, u stay fp32.
 * Sizes     B, T, C (D) >= 0; an empty tensor (any size 0) is a no-op.
 *           B*T*C must be < 2^62.
 * Scratch   inputs with T longer than one tile carry state between thread
 *           blocks through a small library-owned device workspace, one per
 *           (device, stream), allocated with cudaMalloc on first use and
 *           grown when a larger problem needs it.  The tile length is chosen
 *           per call (wkv_tile_steps_for() below returns it; unless
 *           wkv_set_tile_steps() fixed it): 128 steps, or 256 for sequences
 *           longer than 4096 steps with fewer than 64 tiles per time
 *           segment.  Make one call of each size before capturing a stream
 *           into a CUDA graph.  Calls on different streams use different
 *           workspaces and may run concurrently.
 * Rounding  results match the operator to fp32 rounding.  They are bitwise
 *           reproducible from run to run when T spans at most two tiles
 *           (256 steps at the 128-step default, 512 where the call takes
 *           256-step tiles).  Beyond that the carry between tiles may fold
 *           a different, equivalent set of partial results, which can move
 *           the last bits.
 * Errors    argument errors are detected on the host before anything is
 *           launched and return a non-zero wkv_status; wkv_last_error()
 *           then describes the problem (thread-local, valid until the next
 *           call on that thread).  Value preconditions (w >= 0, finite
 *           inputs) are documented, not checked: NaN propagates.
 *           A device-side wait that gives up (see wkv_device_status) writes
 *           NaN outputs for the affected tile and raises WKV_ERR_TIMEOUT
 *           instead of hanging.
 */
#ifndef WKV_B200_H
#define WKV_B200_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define WKV_API __attribute__((visibility("default")))
#else
#define WKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WKV_OK = 0,
    WKV_ERR_INVALID_ARG = 1,  /* bad size, NULL pointer, overlapping output  */
    WKV_ERR_ALIGNMENT = 2,    /* pointer not aligned to its element size     */
    WKV_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed           */
    WKV_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up          */
    WKV_ERR_OOM = 5           /* workspace allocation failed                 */
} wkv_status;

/* bfloat16 storage: the upper 16 bits of the IEEE float32 pattern */
typedef uint16_t wkv_bf16_t;

/* WKV forward, fp32 I/O.  k, v, y: [B, T, C] float; w, u: [C] float.
 * Pointers must be 4-byte aligned.  (16-byte aligned pointers with C a
 * multiple of 4 take the TMA tile path; anything else takes the same kernel
 * with element-wise tile loads.) */
WKV_API wkv_status wkv_forward(int64_t B, int64_t T, int64_t C,
                       const float *w, const float *u,
                       const float *k, const float *v, float *y,
                       cudaStream_t stream);

/* WKV forward, bfloat16 k/v/y with fp32 state.  w, u: [C] float.
 * Pointers must be 2-byte aligned (TMA path: 16-byte and C % 8 == 0). */
WKV_API wkv_status wkv_forward_bf16(int64_t B, int64_t T, int64_t C,
                            const float *w, const float *u,
                            const wkv_bf16_t *k, const wkv_bf16_t *v, wkv_bf16_t *y,
                            cudaStream_t stream);

/* WKV forward from a given state, with the state after the last step
 * returned: streaming a sequence over several calls, and RNN-mode decoding
 * one token per call (T = 1).  The RNN-mode reading of eq. (14) (RWKV
 * evolution article, section RWKV-V4; "RWKV：基于RNN的LLM" section 三,
 * sequential decoding): the state before step t is the pair of past sums
 *
 *     num_t = sum_{i<t} e^{-(t-1-i) w + k_i} v_i,   den_t = the same without v_i,
 *
 * and each step decays it by e^{-w} and adds e^{k_t} (v_t, 1), so a state
 * handed in as the sums before step 0 enters step t weighted by e^{-t w}:
 *
 *     y_t = (e^{-t w} num_in + sum_{0<=i<t} ... + e^{u+k_t} v_t)
 *         / (e^{-t w} den_in + sum_{0<=i<t} ... + e^{u+k_t}).
 *
 * State layout: s_in, s_out are [B, 3, C] float -- for batch row b the planes
 * a, b, p of C floats each, standing for (num, den) = (a, b) * e^p (p in
 * natural-log units; any scaling of one state is the same state).  s_in NULL,
 * or a = b = 0, or p = -inf, is the empty past (then this is wkv_forward).
 * A valid non-empty state has b > 0 and finite fields.  s_out NULL: no state
 * out.  The library writes s_out with b > 0 and p the scale it computed in.
 * Passing the s_out of one call as the s_in of the next continues the
 * sequence (the outputs equal those of one call over all steps, within
 * rounding).  s_out may be the same buffer as s_in (update in place); any
 * other overlap between s_in, s_out and k, v, y, w, u is WKV_ERR_INVALID_ARG.
 * Other arguments, checks and layout as wkv_forward / wkv_forward_bf16;
 * s_in / s_out need 4-byte alignment.  Sequences of at most 16 steps (and
 * wkv_forward's too) run on a kernel that keeps each channel's state in one
 * thread's registers and needs no workspace. */
WKV_API wkv_status wkv_forward_state(int64_t B, int64_t T, int64_t C,
                                     const float *w, const float *u,
                                     const float *k, const float *v, float *y,
                                     const float *s_in, float *s_out,
                                     cudaStream_t stream);

/* wkv_forward_state with bfloat16 k/v/y (fp32 w, u and fp32 state). */
WKV_API wkv_status wkv_forward_bf16_state(int64_t B, int64_t T, int64_t C,
                                          const float *w, const float *u,
                                          const wkv_bf16_t *k, const wkv_bf16_t *v,
                                          wkv_bf16_t *y, const float *s_in, float *s_out,
                                          cudaStream_t stream);

/* WKV forward with the receptance gate fused into its output: eq. (15) of
 * "RWKV：基于RNN的LLM" (section 二.1) applies sigma(r_t) (.) wkv_t before the
 * output projection (the same gate closes the RWKV form in the review of
 * "Resurrecting Recurrent Neural Networks for Long Sequences"), so
 *
 *     y[b,t,c] = wkv[b,t,c] / (1 + e^{-r[b,t,c]})
 *
 * with wkv as in wkv_forward_state.  r: [B, T, C] of the I/O type, read in the
 * same pass as k and v, so the gate costs one extra input stream and no extra
 * output round trip.  s_in / s_out: as wkv_forward_state (either may be NULL).
 * r must not overlap y or s_out; other arguments, checks and layout as
 * wkv_forward_state. */
WKV_API wkv_status wkv_forward_gated(int64_t B, int64_t T, int64_t C,
                                     const float *w, const float *u,
                                     const float *k, const float *v, const float *r, float *y,
                                     const float *s_in, float *s_out, cudaStream_t stream);

/* wkv_forward_gated with bfloat16 k/v/r/y (fp32 w, u and fp32 state). */
WKV_API wkv_status wkv_forward_bf16_gated(int64_t B, int64_t T, int64_t C,
                                          const float *w, const float *u,
                                          const wkv_bf16_t *k, const wkv_bf16_t *v,
                                          const wkv_bf16_t *r, wkv_bf16_t *y,
                                          const float *s_in, float *s_out, cudaStream_t stream);

/* Token shift, the prologue of the time-mixing block: eqs. (11)-(13) of
 * "RWKV：基于RNN的LLM" (section 二.1) feed each projection the interpolation
 *
 *     out[m, b, t, c] = mu[m, c] * x[b, t, c] + (1 - mu[m, c]) * x[b, t-1, c]
 *
 * of every token with the one before it, one mixing vector per projection
 * (the pages also print eqs. (16)-(17) with a minus sign; the plus of eqs.
 * (11)-(13) is the reading taken).  All n_mix (1..4) interpolations come from
 * one read of x.  x[b, -1] is x_prev[b] (the last token of the previous call,
 * the layer's saved "last_x" in the HarmonyOS RWKV article's time-mixing
 * code), or 0 when x_prev is NULL; x_last (if not NULL) receives x[b, T-1].
 * Layout: x [B, T, C]; mu [n_mix, C] float; out [n_mix, B, T, C] (one dense
 * [B, T, C] tensor per mixing vector); x_prev, x_last [B, C].  x_last may be
 * the same buffer as x_prev (update in place); out must not overlap any
 * input, nor x_last.  mu = 1 reproduces x and mu = 0 the shifted x exactly. */
WKV_API wkv_status wkv_token_shift(int64_t B, int64_t T, int64_t C, int64_t n_mix,
                                   const float *x, const float *x_prev, const float *mu,
                                   float *out, float *x_last, cudaStream_t stream);

/* wkv_token_shift on bfloat16 x / x_prev / out / x_last (fp32 mu; computed in
 * fp32, rounded to nearest even). */
WKV_API wkv_status wkv_token_shift_bf16(int64_t B, int64_t T, int64_t C, int64_t n_mix,
                                        const wkv_bf16_t *x, const wkv_bf16_t *x_prev,
                                        const float *mu, wkv_bf16_t *out, wkv_bf16_t *x_last,
                                        cudaStream_t stream);

/* Diagonal linear scan, fp32.  a, b, h: [B, T, D] float; h0: [B, D] float or
 * NULL (zero initial state).  Pointers must be 4-byte aligned. */
WKV_API wkv_status diag_scan(int64_t B, int64_t T, int64_t D,
                     const float *a, const float *b, const float *h0, float *h,
                     cudaStream_t stream);

/* Gradients of the fp32 WKV forward (no state in): given gy = dL/dy [B, T, C],
 * writes gk, gv [B, T, C] and gw, gu [C] (summed over batch rows and steps).
 * The pages give no gradient formulas; eq. (14) of "RWKV：基于RNN的LLM" is a
 * softmax-weighted mean of v_0..v_t with logits l_{t,j} = -(t-1-j) w + k_j
 * (j < t) and l_{t,t} = u + k_t, weights beta_{t,j}, so
 *     gv_j = sum_{t>=j} gy_t beta_{t,j},   gk_j = sum_{t>=j} gy_t beta_{t,j} (v_j - y_t),
 *     gu   = sum_t gy_t beta_{t,t} (v_t - y_t),
 *     gw   = -sum_t sum_{j<t} (t-1-j) gy_t beta_{t,j} (v_j - y_t).
 * Time-parallel over segments of steps, recomputing the forward outputs per
 * segment and running the sums over later outputs backwards in time,
 * max-stabilised (every exponent <= 0 for finite inputs).  When every
 * pointer is 16-byte aligned and C is a multiple of 4 (rows a tensor map
 * can describe): 32-step segments in four launches (forward states and
 * reverse segment summaries, with the forward state carried between
 * 128-step tiles by the decoupled look-back of the forward kernel; reverse
 * carries; gradients; the gw/gu reduction), k, v, gy read twice.  Otherwise
 * 16-step segments in six launches (forward segment summaries, forward
 * carries, reverse segment summaries, reverse carries, gradients, the
 * reduction), k, v read three times.  gw and gu are reduced over rows and
 * segments in a fixed order.  Results are bitwise reproducible on the
 * six-launch path and, on the four-launch path, up to two 128-step tiles;
 * beyond that reproducible to rounding (the look-back may fold the forward
 * carry from different predecessors from run to run).  Scratch (40 bytes per row, segment and channel, plus 64 bytes
 * per channel and a counter per 32 channels) is library-owned per-stream
 * memory, allocated on first use like the look-back workspace (make one call
 * of each size before stream capture).
 * No output may overlap an input or another output.  Pointers 4-byte
 * aligned.  B or T = 0 with C > 0 sets gw, gu to 0. */
WKV_API wkv_status wkv_backward(int64_t B, int64_t T, int64_t C, const float *w, const float *u,
                                const float *k, const float *v, const float *gy, float *gk,
                                float *gv, float *gw, float *gu, cudaStream_t stream);

/* The LRU's complex diagonal recurrence (review of "Resurrecting Recurrent
 * Neural Networks for Long Sequences", linear-RNN section), per complex
 * channel d:
 *
 *     x[b,t,d] = lambda_d x[b,t-1,d] + gamma_d u[b,t,d],
 *     lambda_d = e^{-nu_d + i theta_d},  nu_d = e^{nu_log[d]},  theta_d = e^{theta_log[d]}
 *
 * (the page's parameterisation: |lambda| = e^{-nu} <= 1 for any nu_log), with
 * x[b,-1,d] = x0[b,d] or 0.  u, x: [B, T, D] complex64, i.e. interleaved
 * (re, im) float pairs, [B, T, D, 2] floats; x0: [B, D] complex64 or NULL;
 * nu_log, theta_log, gamma: [D] float, gamma NULL = 1 (the page initialises
 * it to sqrt(1 - |lambda|^2)).  Pointers to complex data must be 8-byte
 * aligned (TMA path: 16-byte and D even).  lambda^n across chunk boundaries
 * is evaluated in double precision, so phases n theta of any size stay
 * exact; inside a chunk the state steps with single-precision lambda.  x must
 * not overlap an input.  Errors, streams and scratch as diag_scan. */
WKV_API wkv_status lru_scan(int64_t B, int64_t T, int64_t D, const float *nu_log,
                            const float *theta_log, const float *gamma, const float *u,
                            const float *x0, float *x, cudaStream_t stream);

/* Diagonal linear scan with bfloat16 a, b, h (fp32 h0 [B, D] or NULL; the
 * state is carried in fp32 and each h is rounded to nearest even).  Pointers
 * must be 2-byte aligned (TMA path: 16-byte and D % 8 == 0). */
WKV_API wkv_status diag_scan_bf16(int64_t B, int64_t T, int64_t D,
                                  const wkv_bf16_t *a, const wkv_bf16_t *b, const float *h0,
                                  wkv_bf16_t *h, cudaStream_t stream);

/* WKV forward, fp32, without allocating any device memory.  The pages this
 * library follows have no counterpart of this entry point: it exists for
 * callers that cannot call cudaMalloc -- code running inside an engine that
 * has already reserved the GPU's memory for its own pool, plugin interfaces
 * that hand an operator nothing but its input and output buffers, and
 * latency-critical paths that must not pay for an allocation or for the
 * device-wide synchronisation cudaMalloc / cudaFree can cause.
 *
 * Same operation, arguments, layout and host-side checks as wkv_forward.
 * Instead of a workspace, the state passed between thread blocks lives in one
 * fixed 16 MiB device array; every GPU that uses this entry point holds it
 * from its first call until the process exits.  A problem whose scratch would
 * not fit -- more than 32,767 tiles, i.e. B * ceil(C/32) * ceil(T/128) >
 * 32,767 (sequences of at most 128 steps need no scratch) -- is rejected with
 * WKV_ERR_INVALID_ARG before anything runs; use wkv_forward for it.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and sets kernel
 * attributes; make that first call before any stream capture.
 * Every call on a device shares the one array and first clears (cudaMemsetAsync
 * on `stream`) the counters and records that must start at zero, so calls whose
 * work overlaps on the GPU -- on different streams, or from several host
 * threads -- race and give wrong results: serialise them.  A device-side wait
 * that gives up leaves NaN in the affected outputs; wkv_device_status does not
 * report it for this entry point. */
WKV_API wkv_status wkv_forward_noalloc(int64_t B, int64_t T, int64_t C,
                                       const float *w, const float *u,
                                       const float *k, const float *v, float *y,
                                       cudaStream_t stream);

/* The same three operations on HOST buffers (every pointer, w/u/h0 included,
 * is host memory; NULL h0 = zeros).  The call copies the inputs to the
 * device, runs the kernel and copies the outputs back, and returns when they
 * are in the output buffer (synchronous; no stream argument).  The work is cut
 * into up to 8 independent chunks of at least 16 MB of input -- batch rows, or
 * 64-channel-aligned channel slices when B is 1 -- pipelined over three
 * internal streams so the uploads of one chunk overlap the compute and
 * download of another.  Page-locked host
 * memory (cudaHostAlloc / cudaHostRegister) gives full overlap; pageable memory
 * works but its copies are staged by the driver.  The library allocates device
 * staging (three chunks of inputs, outputs and parameters) on first use and
 * grows it on demand.  Calls are serialised across host threads.  Returns
 * WKV_ERR_TIMEOUT if a device-side wait gave up during the call. */
WKV_API wkv_status wkv_forward_host(int64_t B, int64_t T, int64_t C,
                                    const float *w, const float *u,
                                    const float *k, const float *v, float *y);
WKV_API wkv_status wkv_forward_bf16_host(int64_t B, int64_t T, int64_t C,
                                         const float *w, const float *u,
                                         const wkv_bf16_t *k, const wkv_bf16_t *v,
                                         wkv_bf16_t *y);
WKV_API wkv_status diag_scan_host(int64_t B, int64_t T, int64_t D,
                                  const float *a, const float *b, const float *h0, float *h);

/* Synchronise `stream`, then return and clear the device status word of that
 * stream's workspace: WKV_OK, or WKV_ERR_TIMEOUT if a device-side wait gave up
 * since the last query.  WKV_ERR_CUDA if the synchronisation itself failed. */
WKV_API wkv_status wkv_device_status(cudaStream_t stream);

/* Message for the last non-OK return on the calling thread ("" if none). */
WKV_API const char *wkv_last_error(void);

/* Free every workspace the library holds on the current device (synchronises
 * the device first).  Later calls allocate again on demand. */
WKV_API wkv_status wkv_release_workspaces(void);

/* Tuning knob, process-wide: the number of steps one thread block stages per
 * tile (8, 32, 64, 128 or 256), or 0 (the default) to let each call choose:
 * 128, or 256 for sequences longer than 4096 steps whose rows and channels
 * make fewer than 64 tiles per tile-length of time.  Results do not depend on
 * it beyond rounding: it only moves the boundaries where chunk summaries are
 * combined.  WKV_ERR_INVALID_ARG for any other value. */
WKV_API wkv_status wkv_set_tile_steps(int steps);
WKV_API int wkv_get_tile_steps(void);
/* The tile length a WKV or scan call of this shape uses now (elem_bytes: 4
 * for fp32 I/O, 2 for bf16); 0 for an invalid shape. */
WKV_API int wkv_tile_steps_for(int64_t B, int64_t T, int64_t C, int elem_bytes);

/* Test hook for failure detection, process-wide, for later launches of the
 * allocating entry points.  skip_tile >= 0: that tile (in the launch's
 * ticket numbering) never publishes its state, so the bounded look-back waits
 * of the tiles after it in time run out; spin_limit > 0 replaces the number
 * of polls a wait makes before giving up (0 restores the default, about a
 * second).  The outcome is WKV_ERR_TIMEOUT from wkv_device_status and NaN in
 * the affected outputs; the context stays usable.  (-1, 0) turns it off.
 * WKV_ERR_INVALID_ARG for skip_tile < -1 or spin_limit < 0. */
WKV_API wkv_status wkv_set_fault_injection(int skip_tile, long long spin_limit);

#ifdef __cplusplus
}
#endif

#endif /* WKV_B200_H */
