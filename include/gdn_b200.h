/*
 * gdn_b200.h -- C ABI of the B200 (sm_100a) frame-recurrence library.
 *
 * Two recurrences that replace softmax attention in linear video diffusion
 * transformers, both block-causal over latent frames:
 *
 *  1. Frame-wise Gated DeltaNet ("SANA-WM, an open-source 2.6B world model for
 *     1-minute 720p video", GeekNews vi.news.hada.io/topic?id=29572, section
 *     "Core design and generation pipeline": a hybrid linear diffusion
 *     transformer with frame-wise Gated DeltaNet; dothoosh.com, "How NVIDIA
 *     SANA-WM generates 60-second 720p video on one GPU": most attention
 *     blocks are Gated DeltaNet with a fixed-size recurrent state).
 *  2. Block-causal ReLU linear attention with a constant-memory block KV cache
 *     ("SANA-Video: Efficient Video Generation with Block Linear Diffusion
 *     Transformer", ICLR 2026 oral talk transcript, block KV cache passage:
 *     the state is a fixed D x D matrix; block i adds its KV contribution to
 *     the cached state of block i-1, and each block reads that state).
 *
 * The pages give no equations; the update rules stated per entry point are
 * this library's definition (the plainest reading consistent with them).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller, except in
 *    gdn_frame_fwd_host(), whose tensor pointers are HOST pointers.
 *  - Layouts are row-major and contiguous.  N = F * L tokens per head.
 *      q, k : [B, H, N, dk]   (element type opts->in_dtype)
 *      v    : [B, H, N, dv]   (element type opts->in_dtype)
 *      o    : [B, H, N, dv]   float32
 *      state: [B, H, dk, dv]  float32, S[i][j] with i over d_k, j over d_v
 *  - Every pointer must be 16-byte aligned.
 *  - Calls are asynchronous on opts->stream (stream-ordered) and return after
 *    launch; errors found on the host are returned at once, errors found on
 *    the device (a bounded wait that ran out) are written to *opts->status.
 *  - The library allocates no memory.  Kernels that need scratch take it
 *    from opts->workspace (size from gdn_workspace_bytes()).  Two calls that
 *    share a workspace must be ordered on the GPU (same stream).
 *  - Thread-safe, with one exception: the only global mutable state is a
 *    per-device cache of the SM count, of the driver's tensor-map encoder
 *    entry point and of the no-allocation scratch address, and the device
 *    scratch array of gdn_frame_fwd_noalloc(), which all of that entry
 *    point's calls share (see there).
 */
#ifndef GDN_B200_H_
#define GDN_B200_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#define GDN_ABI_VERSION 7

/* return / status codes */
#define GDN_OK 0
#define GDN_ERR_INVALID_ARG 1   /* null pointer, bad size, misaligned pointer, bad workspace */
#define GDN_ERR_UNSUPPORTED 2   /* valid arguments this build does not handle (e.g. dk > 128) */
#define GDN_ERR_CUDA 3          /* a CUDA runtime/driver call failed */
#define GDN_ERR_TIMEOUT 4       /* device: a bounded in-kernel wait expired (outputs invalid) */
#define GDN_ERR_NO_DEVICE 5     /* no usable sm_100 device for this call */
#define GDN_ERR_RANGE 6         /* device: a value met the fp16 range of the tensor-core operands
                                   (|q|, |v| or |S| >= 65504, or NaN); outputs invalid */

/* element types of q, k, v */
#define GDN_DTYPE_F32 0
#define GDN_DTYPE_BF16 1

/* kernel selection (GDN_IMPL_AUTO picks the fastest valid one) */
#define GDN_IMPL_AUTO 0
#define GDN_IMPL_SEQ 1          /* per-token SIMT recurrence, one CTA per head (reference-simple) */
#define GDN_IMPL_FRAME_SIMT 2   /* frame maps + ticketed frame chain, CUDA cores, fp32 arithmetic */
#define GDN_IMPL_TC 3           /* frame maps + chain on tcgen05/TMEM tensor cores (bf16 inputs),
                                   residual form (any d_k, d_v multiple of 16 up to 128; splits frames
                                   into chunk segments when frames are few) */
#define GDN_IMPL_TC_PFORM 4     /* tcgen05 kernel with the chunk map in product form, one CTA per
                                   frame (sizes where its shared-memory and TMEM maps fit; see
                                   gdn_pform_supported in the library); GDN_ERR_UNSUPPORTED otherwise */

/* operation ids for gdn_workspace_bytes() */
#define GDN_OP_GDN 0
#define GDN_OP_RELU_LA 1
#define GDN_OP_GDN_BWD 2

typedef struct gdn_opts {
  int in_dtype;           /* GDN_DTYPE_F32 or GDN_DTYPE_BF16: element type of q, k, v */
  int gates_are_logits;   /* gdn only. 1: alpha[] holds logits a, alpha_f = exp(-softplus(a));
                             beta[] holds logits b, beta_t = sigmoid(b).  0: the gate values */
  int impl;               /* GDN_IMPL_* */
  void *stream;           /* cudaStream_t; NULL = legacy default stream */
  void *workspace;        /* device scratch of >= gdn_workspace_bytes() bytes, 256-byte aligned */
  size_t workspace_bytes;
  int *status;            /* optional device int; kernels write a GDN_ERR_* code on a device-side
                             failure and never clear it (caller zeroes it) */
  int max_ctas;           /* 0 = one persistent CTA per SM; else an upper bound (testing) */
  int spin_limit_us;      /* bound on any in-kernel wait; 0 = 2,000,000 us */
  int test_withhold_unit; /* testing only.  0: off.  u + 1: unit u (u = (f*P + s)*B*H + b*H + h,
                             P segments, P = 1 unless segments are in use) never publishes its
                             state, so the wait of the unit after it in its chain expires and the
                             kernel reports GDN_ERR_TIMEOUT through *status */
  int segments;           /* gdn on GDN_IMPL_TC.  0 = automatic; P >= 1: split every frame into P
                             runs of whole 64-token chunks handled by P CTAs (see gdn_frame_fwd);
                             P is lowered to the chunk count and to what fits one resident grid */
  int rope_grid_w;        /* gdn only (gdn_frame_fwd and gdn_frame_bwd).  0: no position
                             embedding.  > 0: the 3D rotary position embedding on q and k (k before
                             its normalisation): a frame's L tokens are a grid of L / rope_grid_w
                             rows of rope_grid_w tokens (L must be a multiple); see gdn_frame_fwd.
                             Not taken by GDN_IMPL_TC_PFORM */
  int rope_frame_offset;  /* time coordinate of the call's first frame (a streaming call: its
                             frame index in the video) */
  float rope_base;        /* frequency base; 0 = 10000 */
} gdn_opts_t;

/*
 * gdn_frame_fwd -- frame-wise Gated DeltaNet forward.
 *
 * Per head (b, h), with S starting at state_in (zero if state_in == NULL):
 *   for each frame f = 0..F-1:
 *     S <- alpha_f * S                       (decay once, at the frame start)
 *     for each token t of frame f, in increasing t:
 *       khat = k_t / max(||k_t||_2, 1e-6)
 *       S    <- S - beta_t * khat (S^T khat - v_t)^T        (delta rule)
 *     for each token t of frame f:  o_t = S^T q_t            (end-of-frame state)
 *   state_out <- S                           (skipped if state_out == NULL)
 *
 * alpha: [B, H, F] float32; beta: [B, H, N] float32 (logits or values, see
 * opts->gates_are_logits).  state_in may equal state_out (in-place carry).
 * q, k, v, o must not overlap each other or the states.
 *
 * Sizes: B, H, F, L >= 1; 1 <= dk, dv <= 128; dk and dv multiples of 16 for
 * GDN_IMPL_TC (others: any size up to 128).  Streaming decode is this call with
 * F = 1, state_in = the cached state and state_out = NULL until the step that
 * commits the frame.
 *
 * Segments (GDN_IMPL_TC): when the B*H*F frames are few (streaming calls), a
 * frame is split into P segments of consecutive 64-token chunks, one CTA each.
 * Segment s builds its own map (A_s, B_s) over its tokens, so that the frame
 * state is S = A_{P-1}(...(A_0 (alpha_f S_{f-1}) + B_0)...) + B_{P-1}, the
 * chain running through the segments in order; every segment then reads out
 * its tokens against the state after the frame's last segment.  Segments are
 * used only when all B*H*F*P CTAs fit on the device at once (one cooperative
 * launch), so no CTA waits for work that has not started.  The automatic
 * choice takes P > 1 only when at most half the SMs would otherwise be busy.
 *
 * 3D position embedding (opts->rope_grid_w > 0; SANA-Video's "3D RoPE for
 * the linear attention", which the talk names without a formula; this is the
 * library's reading): q_t and k_t are rotated before use, k_t before its
 * normalisation.  With d = d_k, a time part of dt = d - 4 floor(d/6)
 * dimensions comes first, then a height and a width part of 2 floor(d/6)
 * each; in each part the pair (2i, 2i+1) turns by pos * base^(-2i/part_length)
 * with pos the token's frame (f + rope_frame_offset), row (t / rope_grid_w)
 * or column (t % rope_grid_w), t its index in the frame.  The workspace then
 * also holds a table of the angles' cosines and sines (gdn_workspace_bytes
 * counts it); d_k must be even and L a multiple of rope_grid_w.
 *
 * Precision: fp32 inputs use fp32 arithmetic throughout (GDN_IMPL_SEQ /
 * FRAME_SIMT).  bf16 inputs on GDN_IMPL_TC multiply on tensor cores with
 * fp16 operands (11-bit significands) and fp32 accumulation; state and
 * outputs are fp32.  The frame state passes from frame to frame as fp16 (each
 * frame's map contracts, so the rounding does not accumulate); state_in is
 * taken as fp16 high and low parts (about 22 significant bits).  The fp16
 * operands need |q|, |v| and |S| below 65504: the kernels report
 * GDN_ERR_RANGE otherwise.
 *
 * Returns GDN_OK or GDN_ERR_*.
 */
GDN_API int gdn_frame_fwd(const void *q, const void *k, const void *v, const float *alpha, const float *beta,
                  const float *state_in, float *state_out, float *o, int B, int H, int F, int L,
                  int dk, int dv, const gdn_opts_t *opts);

/*
 * gdn_frame_bwd -- backward of gdn_frame_fwd, with or without the 3D position
 * embedding.
 *
 * The model is trained (SANA-WM GeekNews summary, "Core design and generation
 * pipeline": 64 H100 GPUs over 15 days), so the recurrence needs its
 * gradient.  For a loss L, given d_o = dL/do [B, H, N, dv] and d_state_out =
 * dL/dstate_out [B, H, dk, dv] (zero if NULL), this writes
 *   d_q, d_k  [B, H, N, dk]  dL/dq, dL/dk
 *   d_v       [B, H, N, dv]  dL/dv
 *   d_alpha   [B, H, F]      dL/d(alpha input): with respect to the logit a when
 *                            opts->gates_are_logits (alpha = exp(-softplus(a))),
 *                            else to the gate value
 *   d_beta    [B, H, N]      the same for beta (beta = sigmoid(b) with logits)
 *   d_state_in [B, H, dk, dv]  dL/dstate_in (skipped if NULL; with state_in ==
 *                            NULL, the gradient at the zero start state)
 * all float32.  The inputs q, k, v, alpha, beta, state_in are those of the
 * forward call (the forward is recomputed; nothing is kept between calls).
 * The outputs may overlap neither one another nor the inputs.
 *
 * Method: with G_f = dL/dS_f, the gradient at frame f's end state,
 *   G_{F-1} = dS_out + Q_{F-1}^T dO_{F-1},  G_{f-1} = Q_{f-1}^T dO_{f-1} + alpha_f A_f^T G_f,
 * A_f being the frame's transition (ordered product of I - beta khat khat^T),
 * and d_alpha_f = <A_f^T G_f, S_{f-1}>, d_state_in = alpha_0 A_0^T G_0.  Inside a
 * frame the token gradients come from two sweeps over chunks of 48 tokens in
 * the UT form: forward from alpha_f S_{f-1}, then in reverse from G_f.  Four
 * launches on opts->stream: the forward recompute keeping every frame's A_f
 * and S_f (GDN_IMPL_TC for bf16 inputs where it applies, else FRAME_SIMT in
 * fp32; opts->impl may force either), Q_f^T dO_f for every frame, the chain
 * over frames, and one CTA per frame for the token gradients.
 *
 * Sizes: as gdn_frame_fwd, with dk, dv <= 112.  Workspace:
 * gdn_workspace_bytes(GDN_OP_GDN_BWD, ...) (four fp32 d x d matrices per frame,
 * with bf16 inputs a 48 x 48 matrix per 48-token chunk and, when dv > dk, a
 * row per token, plus the recompute's scratch, plus the RoPE table).
 *
 * 3D RoPE (opts->rope_grid_w > 0, the forward call's rope_grid_w,
 * rope_frame_offset and rope_base; the same checks): every kernel rotates q
 * and k where it loads them, and d_q, d_k are turned back through the
 * transpose rotation, so they are gradients with respect to the unrotated
 * inputs, as the forward receives them (one more launch, and one first for
 * the angle table).
 *
 * Precision: with bf16 inputs the recomputed A_f and S_f carry the tensor-core
 * forward's rounding (see gdn_frame_fwd), and the products of Q_f^T dO_f and of
 * the token gradients take tf32 operands (10-bit significands) with fp32
 * accumulation; with fp32 inputs everything is fp32 (Q_f^T dO_f with tf32
 * high/low operand splits, about fp32).  Returns GDN_OK or GDN_ERR_*.
 */
GDN_API int gdn_frame_bwd(const void *q, const void *k, const void *v, const float *alpha, const float *beta,
                  const float *state_in, const float *d_o, const float *d_state_out, float *d_q, float *d_k,
                  float *d_v, float *d_alpha, float *d_beta, float *d_state_in, int B, int H, int F, int L,
                  int dk, int dv, const gdn_opts_t *opts);

/*
 * relu_la_block_fwd -- block-causal ReLU linear attention forward.
 *
 * Per head (b, h), with S = kv_in (zero if NULL) [dk x dv] and z = z_in (zero
 * if NULL) [dk]:
 *   for each frame f:
 *     S <- S + sum_{t in f} relu(k_t) v_t^T;   z <- z + sum_{t in f} relu(k_t)
 *     for each token t of f:  o_t = relu(q_t)^T S / (relu(q_t)^T z + eps)
 *   kv_out <- S, z_out <- z                  (each skipped if NULL)
 *
 * kv_in/kv_out: [B, H, dk, dv] float32; z_in/z_out: [B, H, dk] float32.
 * In-place carry (kv_in == kv_out, z_in == z_out) is allowed.
 */
GDN_API int relu_la_block_fwd(const void *q, const void *k, const void *v, const float *kv_in, const float *z_in,
                      float *kv_out, float *z_out, float *o, int B, int H, int F, int L, int dk, int dv,
                      float eps, const gdn_opts_t *opts);

/*
 * temporal_conv_fwd -- causal temporal convolution of one block of latent
 * frames with the block-boundary cache.
 *
 * SANA-Video's causal feed-forward network convolves along time (talk
 * transcript, causal FFN passage): in training a zero token separates two
 * blocks, so the first block cannot see the second, and the second block is
 * prefixed with the first block's last frame; both inserted tokens are
 * dropped after the convolution.  Generated block by block, the same result
 * comes from carrying the last frame of each block in a cache.  The talk gives
 * no kernel size; this library's reading is a depthwise convolution of kernel
 * 3, centred on the frame (one zero token is exactly the separation a kernel
 * of 3 needs).  For every batch b, latent position n < HW and channel c < C:
 *
 *   y[b,f,n,c] = w[c][0] x[b,f-1,n,c] + w[c][1] x[b,f,n,c] + w[c][2] x[b,f+1,n,c] + bias[c]
 *
 * with x[b,-1,n,c] = cache_in[b,n,c] (zero if cache_in == NULL: the first
 * block) and x[b,F,n,c] = 0 (a block never sees the next one); then
 * cache_out[b,n,c] <- x[b,F-1,n,c] (skipped if cache_out == NULL).  Calling
 * this once per block with cache_in = the previous call's cache_out gives the
 * training construction's result over the whole video.
 *
 * x, y: [B, F, HW, C], element type opts->in_dtype; cache_in, cache_out:
 * [B, HW, C], the same type (a copy of a frame, exact); w: [C, 3] float32;
 * bias: [C] float32 or NULL.  The arithmetic is fp32 and y is rounded once
 * to the element type (nearest even for bf16).  cache_in may equal cache_out
 * (in-place carry); no other two of x, y and the caches may overlap
 * (GDN_ERR_INVALID_ARG).  Sizes: B, F, HW, C >= 1.  Options used: in_dtype,
 * stream, max_ctas; no workspace.  Returns GDN_OK or GDN_ERR_*.
 */
GDN_API int temporal_conv_fwd(const void *x, const float *w, const float *bias, const void *cache_in,
                              void *cache_out, void *y, int B, int F, int HW, int C, const gdn_opts_t *opts);

/*
 * softmax_window_fwd -- windowed block-causal softmax attention.
 *
 * SANA-WM's hybrid transformer interleaves the frame-wise Gated DeltaNet with
 * softmax attention layers ("SANA-WM, an open-source 2.6B world model for
 * 1-minute 720p video", GeekNews, "Core design and generation pipeline":
 * periodic softmax; the Vietnamese post on SANA-WM: softmax windows between
 * the Gated DeltaNet layers keep long rollouts coherent; the SANA-Video talk:
 * minute-long video needs softmax kept inside a sliding window).  The pages
 * give no window shape; this library's reading, per head (b, h): token t of
 * frame f attends to every token of frames max(0, f-W+1) .. f (its own frame
 * in full, block-causal like the linear modes),
 *
 *   o_t = sum_s softmax_s(scale * q_t . k_s) v_s,   scale = 1/sqrt(dk) if 0.
 *
 * q, k: [B, H, F*L, dk]; v: [B, H, F*L, dv] (element type opts->in_dtype);
 * o: [B, H, F*L, dv] float32, not overlapping the inputs.  dk, dv <= 128;
 * W >= 1 (W >= F: all earlier frames).  Kernels (opts->impl): GDN_IMPL_TC
 * (bf16 inputs, dk and dv multiples of 16) forms the scores on tensor cores
 * with fp32 accumulation and feeds the probabilities and v to the second
 * product as fp16 (11-bit significands; |v| < 65504, else GDN_ERR_RANGE), o
 * accumulated in fp32; GDN_IMPL_FRAME_SIMT runs in fp32 on CUDA cores (any
 * shape, fp32 or bf16 inputs); GDN_IMPL_AUTO takes the tensor cores when they
 * apply.  Options used: in_dtype, impl, stream, status, spin_limit_us; no
 * workspace.  Returns GDN_OK or GDN_ERR_*.
 */
GDN_API int softmax_window_fwd(const void *q, const void *k, const void *v, float *o, int B, int H, int F, int L,
                               int dk, int dv, int W, float scale, const gdn_opts_t *opts);

/*
 * gdn_frame_fwd_host -- gdn_frame_fwd with HOST tensors.
 *
 * Same semantics and layouts as gdn_frame_fwd, but q, k, v, alpha, beta,
 * state_in (inputs) and o, state_out (outputs) are host pointers (pinned
 * memory gives full PCIe bandwidth).  The call streams the sequence through
 * the caller's device workspace in groups of frames: the inputs of the next
 * group are copied in and the output of the previous group is copied out
 * while a group runs, on two streams the call creates and destroys, ordered
 * after the work already queued on opts->stream.  The state passes from group
 * to group through state_out / state_in in fp32 (the tensor-core kernel takes
 * it as fp16 high and low parts, a little finer than its fp16 frame hand-off
 * inside one call), so the result agrees with gdn_frame_fwd over the whole
 * sequence to that rounding.  The call synchronises opts->stream before
 * returning.
 * opts->workspace must hold gdn_workspace_bytes_host() bytes (two groups'
 * inputs and outputs, four states and one group's kernel workspace).
 */
GDN_API int gdn_frame_fwd_host(const void *q, const void *k, const void *v, const float *alpha, const float *beta,
                       const float *state_in, float *state_out, float *o, int B, int H, int F, int L,
                       int dk, int dv, const gdn_opts_t *opts);

/*
 * gdn_frame_fwd_noalloc -- gdn_frame_fwd without a caller-provided workspace.
 *
 * The pages describe no counterpart of this call; it exists for callers that
 * cannot allocate device memory at all (for example a plugin inside a host
 * program that owns every device allocation and passes the plugin only its
 * input and output buffers, or a runtime with a fixed memory plan that allows
 * no allocation after start-up).  Arguments, semantics and layouts are those of
 * gdn_frame_fwd; opts->workspace and opts->workspace_bytes are ignored.
 *
 * The frame-chain scratch comes from a fixed array inside the library, of
 * GDN_NOALLOC_SCRATCH_BYTES on every GPU that loads the library, kept until
 * the process exits.  Calls whose gdn_workspace_bytes(GDN_OP_GDN, ...) exceeds
 * that size return GDN_ERR_UNSUPPORTED without launching anything.  The first
 * call on a device looks up the array's device address; make that first call
 * before any stream capture.  Later calls made outside stream capture look it
 * up again, so the address stays right after a device reset.  All calls share
 * the array: calls that may run at the same time on the GPU (other streams,
 * unordered host threads) race on it and must be serialised by the caller.
 * Each call clears the part of the array that must start at zero before its
 * kernel runs.  The call allocates no memory.
 */
#define GDN_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
GDN_API int gdn_frame_fwd_noalloc(const void *q, const void *k, const void *v, const float *alpha,
                                  const float *beta, const float *state_in, float *state_out, float *o, int B,
                                  int H, int F, int L, int dk, int dv, const gdn_opts_t *opts);

/* Device scratch bytes that op (GDN_OP_*) needs for these sizes and options. */
GDN_API size_t gdn_workspace_bytes(int op, int B, int H, int F, int L, int dk, int dv, const gdn_opts_t *opts);

/* Device scratch bytes that gdn_frame_fwd_host() needs (staging + workspace). */
GDN_API size_t gdn_workspace_bytes_host(int B, int H, int F, int L, int dk, int dv, const gdn_opts_t *opts);

/* Static description of a status code (never NULL).  gdn_status_str is the
 * same function under a shorter name. */
GDN_API const char *gdn_status_string(int status);
GDN_API const char *gdn_status_str(int status);

/* GDN_ABI_VERSION of the loaded library. */
GDN_API int gdn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_B200_H_ */
