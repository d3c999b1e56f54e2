/*
 * rib.h -- C ABI of librib.so: RIB windowed attention on NVIDIA B200 (sm_100a).
 *
 * RIB (Rank-factorized Implicit Neural Bias) is windowed multi-head
 * self-attention over image feature maps whose positional bias is the
 * low-rank product Qp Kp^T.  Qp and Kp come from a Fourier-feature MLP on
 * window coordinates and are concatenated channel-wise with the content
 * tokens, so the score [Qc,Qp][Kc,Kp]^T = Qc Kc^T + Qp Kp^T is one dot
 * product and attention runs flash-style without an N x N score or bias
 * matrix.  Sources: "Rank-Factorized Implicit Neural Bias: Scaling
 * Super-Resolution Transformer with FlashAttention" (arXiv 2603.06738) --
 * its abstract, and the gist.science summaries (English: Technical Summary
 * §2.A "Rank-Factorized Implicit Neural Bias (RIB)", steps 1-4 and the score
 * equation; German: Methodik §A; Chinese: 核心方法论 §A).
 *
 * Conventions for every entry point
 *   - Pointers are caller-owned.  Tensor arguments are DEVICE pointers on the
 *     current CUDA device unless stated otherwise; the library allocates no
 *     device memory: scratch comes from the caller's workspace.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is asynchronous: a return of RIB_OK means "validated and
 *     launched".  Faults seen inside kernels (a bounded wait that ran out)
 *     are recorded in a per-device status word read by rib_last_status().
 *   - Arguments are validated before anything is launched; on error nothing
 *     is enqueued and a negative RIB_ERR_* code is returned.  No C++
 *     exception crosses this boundary.
 *   - Layouts are row-major, innermost index last.  bf16 = IEEE bfloat16
 *     stored as 16-bit words; conversion is round-to-nearest-even.
 *   - Device buffers must be 16-byte aligned (TMA); violations return
 *     RIB_ERR_ALIGN.  The attention outputs (out, out_gated, dqkv) are
 *     written in whole 32-byte sectors when they are also 32-byte aligned
 *     (faster; the values are the same either way).
 *   - The work entry points make no synchronous CUDA call and allocate
 *     nothing, so a sequence of them may be captured into a CUDA graph on
 *     `stream` and replayed (the kernel parameters, tensor maps included,
 *     are fixed at capture: replays read and write the same buffers).  Only
 *     the status and debug queries (rib_last_status, rib_debug_guard_info)
 *     synchronise the device; rib_pos_tokens_bwd_noalloc's first call on a
 *     device must precede any capture.
 *
 * Notation: B batch, H x W feature map, M window side, N = M*M tokens per
 * window, nW = (H/M)(W/M) windows, h heads, d = 32 content head dim,
 * r = 16 (or 0) rank, F Fourier frequencies, s cyclic shift.  A "unit" is
 * one (batch, window, head) attention problem.
 *
 * Window partition with cyclic shift (no region mask): token (i, j) of
 * window (wy, wx) is map pixel ((wy*M + i + s) mod H, (wx*M + j + s) mod W),
 * i.e. a roll of the map by -s followed by a partition; outputs are written
 * back to the same pixels (the inverse roll).
 */
#ifndef RIB_H_
#define RIB_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RIB_OK               0
#define RIB_ERR_ARG         -1  /* null pointer, negative size, bad scalar */
#define RIB_ERR_SHAPE       -2  /* H % M != 0, W % M != 0, shift outside [0, M) */
#define RIB_ERR_UNSUPPORTED -3  /* valid but not built: d != 32, r not in {0,16},
                                   M % 16 != 0, s % 8 != 0, ... */
#define RIB_ERR_WORKSPACE   -4  /* workspace missing or smaller than required */
#define RIB_ERR_CUDA        -5  /* a CUDA runtime/driver call failed */
#define RIB_ERR_TIMEOUT     -6  /* a kernel's bounded wait ran out (status word) */
#define RIB_ERR_ALIGN       -7  /* a device pointer is not 16-byte aligned */
#define RIB_ERR_BOUNDS      -8  /* debug build: a guarded access fell outside its buffer */

/* Position-MLP weights (device, fp32, PyTorch Linear layout weight[out][in]).
 * d_in = 4*n_freq (features [sin(w x), cos(w x), sin(w y), cos(w y)]),
 * hidden = d_hidden, d_out = heads*rank (output column o = head*rank + r).
 * Two MLPs of the same shape: q_* gives Qp, k_* gives Kp; passing the same
 * pointers for both ties them.  freqs[n_freq] are angular frequencies. */
typedef struct {
    int n_freq;
    const float* freqs;
    int d_hidden;
    int heads;
    int rank;
    const float *q_w1, *q_b1, *q_w2, *q_b2;   /* [hid][4F], [hid], [h*r][hid], [h*r] */
    const float *k_w1, *k_b1, *k_w2, *k_b2;
} rib_mlp_t;

/* Gradients of the position MLPs (device, fp32, same shapes as rib_mlp_t). */
typedef struct {
    float *q_dw1, *q_db1, *q_dw2, *q_db2;
    float *k_dw1, *k_db1, *k_dw2, *k_db2;
} rib_mlp_grad_t;

/* ------------------------------------------------------------------------
 * rib_pos_tokens -- positional tokens for one window geometry.
 *
 * English summary §2.A steps 1-2 (German §A step 1: normalised 2D coordinate
 * in [-1, 1]; Fourier feature map; lightweight MLP -> low-rank Qp, Kp).
 * Coordinates are local to the window with endpoints included:
 * y_i = -1 + 2i/(M-1), x_j = -1 + 2j/(M-1) (M = 1 gives 0).  Hidden layer:
 * GELU (erf form).  Qp/Kp depend only on the geometry (Chinese summary §A:
 * precomputed and cached), so one call serves every window, batch entry and
 * layer with this M and these weights.
 *
 *   mlp      : host pointer to the weight struct (device weight pointers)
 *   window   : M, 1 <= M <= 256
 *   qp, kp   : out, fp32 [heads][M][M][rank]
 *   qp_bf16, kp_bf16 : out, bf16 copies of the same shape (may be NULL)
 * Computes in fp32 (coordinate Fourier features in fp64, rounded to fp32).
 * ------------------------------------------------------------------------ */
int rib_pos_tokens(const rib_mlp_t* mlp, int window, float* qp, float* kp,
                   void* qp_bf16, void* kp_bf16, void* stream);

/* ------------------------------------------------------------------------
 * rib_pos_tokens_bwd -- backward of rib_pos_tokens: gradients of the two
 * position MLPs given dL/dQp and dL/dKp (the chain rule through Linear ->
 * GELU(erf) -> Linear, with the Fourier features recomputed).  Sums over the
 * M*M tokens run in a fixed order (per-chunk partials, then a chunk sum), so
 * the result is deterministic.
 *
 *   dqp, dkp : fp32 [heads][M][M][rank]
 *   dmlp     : host pointer to device gradient buffers (fp32, weight shapes)
 *   workspace: device scratch of rib_pos_tokens_bwd_workspace() bytes,
 *              256-byte aligned
 * ------------------------------------------------------------------------ */
size_t rib_pos_tokens_bwd_workspace(const rib_mlp_t* mlp, int window);
int rib_pos_tokens_bwd(const rib_mlp_t* mlp, int window, const float* dqp,
                       const float* dkp, const rib_mlp_grad_t* dmlp,
                       void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * rib_pos_tokens_bwd_noalloc -- rib_pos_tokens_bwd without a workspace.
 *
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory when they need the gradients: code that
 * runs while a CUDA graph is being captured (cudaMalloc is not allowed
 * there), hosts and plugins whose allocator owns every device byte, and
 * latency-bound loops that cannot afford the device-wide synchronisation a
 * cudaMalloc/cudaFree pair implies.  It computes exactly what
 * rib_pos_tokens_bwd computes, using a scratch area that is part of the
 * library itself: a statically allocated device array of
 * RIB_NOALLOC_SCRATCH_BYTES (24 MiB), which every GPU that loads the library
 * keeps until the process exits.  Sizes whose scratch need
 * (rib_pos_tokens_bwd_workspace) exceeds that return RIB_ERR_WORKSPACE.
 *
 *   The first call on each device looks up the device address of the array
 *   (a host-side step, done once per device with that device current); make
 *   that first call before any stream capture begins.
 *   All calls share the one array: calls whose kernels may overlap on the
 *   GPU (different streams without ordering between them) race on it and
 *   give undefined results.  Every scratch byte a call reads is written by
 *   the same call first, so no clearing is needed between calls.
 *   Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 * ------------------------------------------------------------------------ */
#define RIB_NOALLOC_SCRATCH_BYTES (24u * 1024u * 1024u)
int rib_pos_tokens_bwd_noalloc(const rib_mlp_t* mlp, int window, const float* dqp,
                               const float* dkp, const rib_mlp_grad_t* dmlp,
                               void* stream);

/* ------------------------------------------------------------------------
 * rib_window_attn_fwd -- RIB window attention forward.
 *
 * English summary §2.A steps 3-4 and the score equation; the paper's
 * abstract (channel-wise concatenation turns the bias addition into a dot
 * product so FlashAttention-style kernels apply).  Per unit:
 *   S = scale * [Qc,Qp][Kc,Kp]^T,  P = softmax_rows(S),  O = P V,
 *   lse = ln sum_k exp(S[:,k]),
 * computed flash-style (online softmax on tcgen05/TMEM), never forming S.
 *
 *   qkv      : bf16 [B][H][W][3][heads][head_dim]  (Qc, Kc, V)
 *   qp_bf16, kp_bf16 : bf16 [heads][M][M][rank] from rib_pos_tokens
 *                      (ignored when rank == 0)
 *   rank     : 0 or 16
 *   scale    : softmax scale; <= 0 selects 1/sqrt(head_dim + rank)
 *   out      : bf16 [B][H][W][heads][head_dim]
 *   lse      : fp32 [B][heads][H][W] (natural log), needed by the backward
 * Supported: head_dim == 32, M % 16 == 0, 16 <= M <= 256, s % 8 == 0.
 * B == 0 (an empty batch) is valid: nothing is read, written or launched,
 * and the pointers are not looked at.
 * ------------------------------------------------------------------------ */
int rib_window_attn_fwd(const void* qkv, int B, int H, int W, int heads,
                        int head_dim, int window, int shift,
                        const void* qp_bf16, const void* kp_bf16, int rank,
                        float scale, void* out, float* lse, void* stream);

/* ------------------------------------------------------------------------
 * rib_cla_gate -- gating map of the convolutional local attention (CLA).
 *
 * English summary, Technical Summary §2.B (a lightweight path of a
 * depth-wise convolution, a point-wise convolution and a sigmoid produces a
 * gating map); Chinese summary §2.B (3x3 depth-wise, 1x1 point-wise):
 *   y[b,i,j,c] = b_dw[c] + sum_{u,v<3} w_dw[c][u][v] x[b,i+u-1,j+v-1,c]
 *                (zero padding of one pixel; cross-correlation)
 *   z[b,i,j,o] = b_pw[o] + sum_c w_pw[o][c] y[b,i,j,c]
 *   G = 1 / (1 + exp(-z))
 *
 *   x      : bf16 [B][H][W][C], the layer's input feature map (device)
 *   w_dw   : fp32 [C][3][3]; b_dw : fp32 [C]            (device)
 *   w_pw   : fp32 [C][C] ([out][in]); b_pw : fp32 [C]    (device)
 *   gate   : out, bf16 [B][H][W][C]                      (device)
 * The point-wise convolution runs on the tensor cores with y and w_pw
 * rounded to bf16 (fp32 accumulation).  Requires C % 32 == 0, C <= 192,
 * H % 8 == 0, W % 16 == 0 (else RIB_ERR_UNSUPPORTED / RIB_ERR_SHAPE); B == 0
 * is a valid no-op (pointers not looked at); x and
 * gate 16-byte aligned, w_pw 8-byte aligned (RIB_ERR_ALIGN).  Asynchronous
 * on `stream`; allocates nothing.
 * ------------------------------------------------------------------------ */
int rib_cla_gate(const void* x, int B, int H, int W, int C, const float* w_dw,
                 const float* b_dw, const float* w_pw, const float* b_pw,
                 void* gate, void* stream);

/* ------------------------------------------------------------------------
 * rib_window_attn_fwd_tf32 -- RIB window attention forward for fp32 inputs.
 *
 * The same computation as rib_window_attn_fwd (English summary §2.A steps
 * 3-4 and the score equation: S = scale * [Qc,Qp][Kc,Kp]^T, P =
 * softmax_rows(S), O = P V, lse = ln sum_k exp(S[:,k])), for features and
 * position tokens kept in fp32: nothing is rounded to bf16.  The tcgen05
 * tensor cores read the fp32 operands as tf32 (10 explicit mantissa bits)
 * and accumulate in fp32; P is rounded to tf32 (to nearest) before the PV
 * product and the softmax denominator is summed from the rounded P.
 *
 *   qkv      : fp32 [B][H][W][3][heads][head_dim]  (Qc, Kc, V)
 *   qp, kp   : fp32 [heads][M][M][rank], e.g. the fp32 outputs of
 *              rib_pos_tokens (ignored when rank == 0)
 *   rank     : 0 or 16
 *   scale    : softmax scale; <= 0 selects 1/sqrt(head_dim + rank)
 *   out      : out, fp32 [B][H][W][heads][head_dim]
 *   lse      : out, fp32 [B][heads][H][W] (natural log)
 * Same shape support, errors and B == 0 behaviour as rib_window_attn_fwd;
 * every pointer 16-byte aligned (RIB_ERR_ALIGN).  Device pointers, caller
 * owned; asynchronous on `stream`.  No shift mask, no CLA gate.
 * ------------------------------------------------------------------------ */
int rib_window_attn_fwd_tf32(const float* qkv, int B, int H, int W, int heads,
                             int head_dim, int window, int shift, const float* qp,
                             const float* kp, int rank, float scale, float* out,
                             float* lse, void* stream);

/* ------------------------------------------------------------------------
 * rib_window_attn_fwd_cla -- rib_window_attn_fwd with the CLA gate applied
 * in the same kernel's epilogue (German summary, Methodik §B: O' = O * G).
 *
 *   gate      : bf16 [B][H][W][heads*head_dim] from rib_cla_gate (channel
 *               head*head_dim + e gates output channel e of that head)
 *   out       : out, bf16 O [B][H][W][heads][head_dim] (kept: the backward
 *               needs the ungated output)
 *   out_gated : out, bf16 O * G, same layout
 * Every other argument, requirement and error is as for
 * rib_window_attn_fwd; gate and out_gated must be 16-byte aligned.
 * ------------------------------------------------------------------------ */
int rib_window_attn_fwd_cla(const void* qkv, int B, int H, int W, int heads,
                            int head_dim, int window, int shift,
                            const void* qp_bf16, const void* kp_bf16, int rank,
                            float scale, const void* gate, void* out,
                            void* out_gated, float* lse, void* stream);

/* ------------------------------------------------------------------------
 * rib_cla_bwd -- backward of the CLA gate (the gradients of O' = O * G for
 * the gate of rib_cla_gate; English summary §2.B, German summary §B).
 * With dO' the gradient of the gated output:
 *   dO = dO' * G,   dz = dO' * O * G * (1 - G),
 *   db_pw = sum_pixels dz,   dW_pw = sum_pixels dz^T y   (y recomputed),
 *   dy = dz W_pw,   db_dw = sum_pixels dy,
 *   dW_dw[c][u][v] = sum_pixels dy[p][c] x[p + (u-1, v-1)][c],
 *   dx[p][c] = sum_{u,v} W_dw[c][u][v] dy[p - (u-1, v-1)][c]  (zero outside).
 *
 *   x, w_dw, b_dw, w_pw : as given to rib_cla_gate (device)
 *   gate       : bf16 [B][H][W][C], G from rib_cla_gate
 *   out        : bf16 [B][H][W][C], the ungated attention output O
 *   dout_gated : bf16 [B][H][W][C], dO'
 *   dout       : out, bf16 dO (pass it to rib_window_attn_bwd as its dout)
 *   dx         : out, bf16 [B][H][W][C], the CLA path's share of dL/dx
 *   dw_dw, db_dw, dw_pw, db_pw : out, fp32, shapes of the weights
 *   workspace  : device, >= rib_cla_bwd_workspace() bytes, 256-byte aligned
 * The point-wise GEMMs run on the tensor cores with bf16 operands (dz, y,
 * W_pw rounded) and fp32 accumulation; sums over pixels go through per-CTA
 * partials added in a fixed order, so results are deterministic.  Same
 * shape requirements and errors as rib_cla_gate; RIB_ERR_WORKSPACE for a
 * missing or short workspace.  B == 0 zeroes the four weight gradients and
 * touches nothing else.  Asynchronous on `stream`.
 * ------------------------------------------------------------------------ */
size_t rib_cla_bwd_workspace(int B, int H, int W, int C);
int rib_cla_bwd(const void* x, int B, int H, int W, int C, const float* w_dw,
                const float* b_dw, const float* w_pw, const void* gate,
                const void* out, const void* dout_gated, void* dout, void* dx,
                float* dw_dw, float* db_dw, float* dw_pw, float* db_pw,
                void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace rib_window_attn_bwd needs for these sizes;
 * `mlp` (host pointer, may be NULL) adds the MLP-gradient scratch. */
size_t rib_window_attn_bwd_workspace(int B, int H, int W, int heads,
                                     int head_dim, int window, int rank,
                                     const rib_mlp_t* mlp);

/* ------------------------------------------------------------------------
 * rib_window_attn_bwd -- RIB window attention backward (+ MLP gradients).
 *
 * Gradients of sum(out * dout) for the forward above (training, per the
 * abstract's training-time claim).  With D = rowsum(dO * O):
 *   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),
 *   d[Qc,Qp] = scale dS [Kc,Kp],  d[Kc,Kp] = scale dS^T [Qc,Qp].
 * dqp/dkp are summed over batch entries and windows (the tokens are shared
 * by every window).  If mlp and dmlp are both non-NULL the position-MLP
 * weight gradients are computed from dqp/dkp as well (sums over tokens in a
 * fixed order).
 *
 * Reproducibility: dKc, dV, dkp and the key MLP's gradients are bit-identical
 * from call to call (each key tile's sums run in query-tile order inside one
 * CTA; dkp and the MLP sums are fixed-order reductions).  dQc, dqp and the
 * query MLP's gradients are NOT: every key tile of a unit adds its dQ_aug
 * partial to one fp32 accumulator per query tile with a bulk reduce-add, and
 * the order of those adds depends on how the CTAs are scheduled.  Repeated
 * calls agree to fp32 rounding of the accumulator (within the stated
 * tolerance), not bit for bit.
 *
 *   qkv, out, lse : as produced for / by rib_window_attn_fwd
 *   dout     : bf16 [B][H][W][heads][head_dim]
 *   dqkv     : out, bf16 [B][H][W][3][heads][head_dim]
 *   dqp, dkp : out, fp32 [heads][M][M][rank] (may be NULL when rank == 0)
 *   mlp      : host pointer (may be NULL), must match heads/rank
 *   dmlp     : host pointer to device gradient buffers (may be NULL)
 *   workspace: device scratch of at least rib_window_attn_bwd_workspace()
 *              bytes, 256-byte aligned; contents need not be initialised
 * B == 0 is valid: dqp, dkp and the MLP gradients (when requested) are
 * zeroed, being sums over no windows, and nothing else is touched.
 * dQ partials of the key tiles are summed with fp32 reduce-adds in no fixed
 * order, so dqkv's query part and dqp may differ in the last bits between
 * runs.
 * ------------------------------------------------------------------------ */
int rib_window_attn_bwd(const void* qkv, const void* out, const void* dout,
                        const float* lse, int B, int H, int W, int heads,
                        int head_dim, int window, int shift,
                        const void* qp_bf16, const void* kp_bf16, int rank,
                        float scale, void* dqkv, float* dqp, float* dkp,
                        const rib_mlp_t* mlp, const rib_mlp_grad_t* dmlp,
                        void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * rib_window_attn_fwd_masked / rib_window_attn_bwd_masked -- the same
 * forward and backward with the shifted-window region mask, an optional
 * variant the pages do not describe (they use a pure cyclic roll).  On the
 * map rolled by -shift, rows fall into the bands [0, H-M), [H-M, H-shift),
 * [H-shift, H) and columns likewise; a query attends only to keys of its own
 * (row band, column band).  Only windows in the last window row or column
 * hold more than one region; elsewhere, and with shift == 0, the results
 * equal the unmasked calls.  Masked pairs get P = 0 exactly (their dS is 0
 * too).  Arguments, layouts, limits and errors are those of
 * rib_window_attn_fwd / rib_window_attn_bwd; pass lse from the masked
 * forward to the masked backward.
 * ------------------------------------------------------------------------ */
int rib_window_attn_fwd_masked(const void* qkv, int B, int H, int W, int heads,
                               int head_dim, int window, int shift,
                               const void* qp_bf16, const void* kp_bf16, int rank,
                               float scale, void* out, float* lse, void* stream);
int rib_window_attn_bwd_masked(const void* qkv, const void* out, const void* dout,
                               const float* lse, int B, int H, int W, int heads,
                               int head_dim, int window, int shift,
                               const void* qp_bf16, const void* kp_bf16, int rank,
                               float scale, void* dqkv, float* dqp, float* dkp,
                               const rib_mlp_t* mlp, const rib_mlp_grad_t* dmlp,
                               void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * rib_window_gather / rib_window_scatter -- the window partition with cyclic
 * shift as a standalone copy (the same rolled TMA tile addressing the
 * attention kernels use), for bit-exact checks and for callers that want
 * window-contiguous tensors.
 *
 *   x   : [B][H][W][C] elements of elem_bytes (1, 2 or 4) each
 *   xw  : [B][nW][M*M][C], window index wy*(W/M)+wx, token index i*M+j
 * gather: xw[b][w][i*M+j] = x[b][(wy*M+i+s) % H][(wx*M+j+s) % W];
 * scatter writes the inverse.  Requires C*elem_bytes % 16 == 0,
 * M % 8 == 0, s % 8 == 0.  Pure copies: bit-exact.
 * ------------------------------------------------------------------------ */
int rib_window_gather(const void* x, int B, int H, int W, int C,
                      int elem_bytes, int window, int shift, void* xw,
                      void* stream);
int rib_window_scatter(const void* xw, int B, int H, int W, int C,
                       int elem_bytes, int window, int shift, void* x,
                       void* stream);

/* ------------------------------------------------------------------------
 * Status and failure detection.
 * Every wait inside the kernels (mbarrier phases of the TMA / tensor-core
 * pipelines) is bounded by a time limit; when it runs out the kernel records
 * RIB_ERR_TIMEOUT in a per-device status word, drains its in-flight copies
 * and tensor-core work, frees its tensor memory and returns.
 * ------------------------------------------------------------------------ */

/* Human-readable name of a status code (static string). */
const char* rib_status_string(int status);

/* Synchronises the current device, returns the first error recorded by a
 * kernel since the previous call (RIB_OK if none) and clears it.  If `site`
 * is non-NULL it receives a code naming the wait that gave up. */
int rib_last_status(int* site);

/* Form of the attention backward kernel (rib_window_attn_bwd and
 * rib_window_attn_bwd_masked).  Both compute the same gradients (the same
 * arithmetic in the same order per key tile):
 *   RIB_BWD_PER_ITEM    one CTA per (unit, key tile);
 *   RIB_BWD_PERSISTENT  one CTA per SM walking the (unit, key tile) items,
 *                       the next item's loads and MMAs overlapping the end
 *                       of the current one;
 *   RIB_BWD_AUTO        (default) the persistent form for windows up to
 *                       64 x 64, where per-CTA set-up weighs on few query
 *                       tiles, and the per-item form above.
 * rib_set_bwd_kernel sets it process-wide (RIB_ERR_ARG for another value);
 * rib_bwd_kernel_for returns the form a call with this window would use. */
#define RIB_BWD_AUTO         0
#define RIB_BWD_PER_ITEM     1
#define RIB_BWD_PERSISTENT   2
int rib_set_bwd_kernel(int which);
int rib_bwd_kernel_for(int window);

/* Time limit, in nanoseconds, of every bounded wait in kernels launched
 * after this call (process-wide; default 1e9 = 1 s; 0 restores it). */
int rib_set_wait_limit_ns(unsigned long long limit_ns);

/* ------------------------------------------------------------------------
 * Debug build.  librib_debug.so is this library compiled with RIB_DEBUG: every
 * global-memory access of its kernels that does not go through a TMA tensor
 * map first tests its element index against the extent of its buffer, as
 * the call's shapes define it.  A refused access is skipped (nothing out of
 * range is read or written); the first one records RIB_ERR_BOUNDS, reported
 * by rib_last_status with the code of the guarded site, and its index and
 * extent, reported by rib_debug_guard_info.  Results are otherwise those of
 * the release library, at lower speed.  It stands in for a memory checker.
 *
 * rib_debug_build         1 in the debug build, 0 in the release build.
 * rib_debug_guard_info    synchronises, writes {index, extent} of the first
 *                         refused access since the last call (zeros if none,
 *                         and always zeros in the release build), clears it.
 * rib_debug_guard_selftest  launches one CTA that writes element `index` of
 *                         a 32-float shared array whose first `extent`
 *                         elements are in bounds, through a guard; index >=
 *                         extent must be refused and recorded.  Release
 *                         build: RIB_ERR_UNSUPPORTED, nothing launched.
 * ------------------------------------------------------------------------ */
int rib_debug_build(void);
int rib_debug_guard_info(unsigned long long* index_extent);
int rib_debug_guard_selftest(int index, int extent, void* stream);

/* Test hook for the failure path: launches one CTA that waits on an
 * mbarrier nothing will arrive on, with the given limit, using the same
 * bounded-wait routine as the attention kernels.  The wait runs out and the
 * kernel records RIB_ERR_TIMEOUT; nothing faults and the context stays
 * usable. */
int rib_debug_wait_timeout(unsigned long long limit_ns, void* stream);

/* ------------------------------------------------------------------------
 * Tracing: per-kernel device time measured with CUDA events recorded on
 * the launch stream around every kernel the library launches.
 * ------------------------------------------------------------------------ */
typedef struct {
    const char* kernel;   /* static name */
    int launches;
    double total_ms;
} rib_trace_entry_t;

/* Turns tracing on (1) or off (0) for later launches (process-wide).
 * Turning it on discards records not yet collected. */
int rib_trace_enable(int on);

/* Waits for the traced launches, aggregates them per kernel into
 * entries[0 .. *n_entries) (at most max_entries) and clears the records. */
int rib_trace_collect(rib_trace_entry_t* entries, int max_entries, int* n_entries);

/* Test hook for the FMA-pipe exponential of the attention kernels:
 * y[i] = 2^x[i] computed as the forward kernel computes it (Cody-Waite
 * reduction + degree-3 minimax polynomial, inputs clamped at -125), for
 * device arrays of n fp32 values (n even). */
int rib_debug_exp2(const float* x, float* y, int n, void* stream);

/* Library version, e.g. "rib-b200 0.1 sm_100a". */
const char* rib_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RIB_H_ */
