/*
 * vdn.h - C ABI of the B200 (sm_100a) frame-wise delta-rule memory (VDA).
 *
 * The operations follow the paper "Video DeltaNet: A Video-Native Hybrid
 * Attention for Livestream Video Generation" (summary page). Notation, per
 * (batch b, head h): frames t = 0..T-1, tokens u = 0..U-1, keys/queries of
 * width d_k, values of width d_v, state S of shape [d_v, d_k] (S maps a key to
 * a value; a query reads S q). Chunks hold `chunk` (= 5) consecutive frames,
 * C = ceil(T / chunk), the last one possibly partial.
 *
 * Conventions shared by every call
 * --------------------------------
 * Layout     : dense row-major, innermost index fastest. Q, K, V are
 *              [B, H, T, U, d]; text keys/values are [B, H, n_text, d];
 *              per-frame matrices are [B, H, T, d, d]; chunk maps are
 *              [B, H, C, d, d]; boundary states are [B, H, C+1, d_v, d_k].
 * Types      : Q/K/V/Kx/Vx are float32 or bfloat16 (shape.in_dtype); O is
 *              float32 or bfloat16 (shape.out_dtype); beta, alpha, every
 *              matrix and every state are float32.
 * Memory     : every pointer is a DEVICE pointer, 16-byte aligned, owned by
 *              the caller. The library never allocates, frees or keeps a
 *              pointer after the call; the fused call takes a caller
 *              workspace.
 * Streams    : each call validates its arguments on the host, enqueues its
 *              kernels on `stream` (NULL = the legacy default stream) and
 *              returns without synchronising. There is no global mutable
 *              state but one: the fixed scratch array of
 *              vdn_text_state_noalloc (see there), which calls of that entry
 *              point share. Calls of every other entry point on different
 *              streams may run concurrently if their outputs do not overlap.
 * Errors     : argument problems are reported synchronously (VDN_ERR_INVALID
 *              or VDN_ERR_UNSUPPORTED) before anything is enqueued; a launch
 *              failure returns VDN_ERR_CUDA. vdn_last_error() gives a one-line
 *              message for the calling thread. A numeric failure on the device
 *              (a non-positive or non-finite pivot when factoring I + A_t) is
 *              written to the device word *info: 0 = success, otherwise
 *              1 + the smallest failing linear frame index (b*H + h)*T + t.
 *              No kernel traps, asserts or waits without a time limit; a
 *              pipeline wait that exceeds its limit sets *info to
 *              VDN_INFO_TIMEOUT instead.
 * Sizes      : B, H, T, U, n_text >= 0 (zero sizes are valid and do no work);
 *              d_k == d_v in {16, 32, 64, 128}; 1 <= chunk <= 16.
 */
#ifndef VDN_H
#define VDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL selects the legacy default stream. */
typedef struct CUstream_st *vdn_stream_t;

typedef enum {
  VDN_OK = 0,
  VDN_ERR_INVALID = 1,     /* null/misaligned pointer, bad size or enum */
  VDN_ERR_UNSUPPORTED = 2, /* valid request this build has no kernel for */
  VDN_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  VDN_ERR_NUMERIC = 4      /* reserved for host-side numeric checks */
} vdn_status;

typedef enum { VDN_F32 = 0, VDN_BF16 = 1 } vdn_dtype;

/* *info value written when a device-side wait ran out of time. */
#define VDN_INFO_TIMEOUT (-1)

typedef struct {
  int32_t B, H, T, U; /* batch, heads, latent frames, tokens per frame */
  int32_t dk, dv;     /* key and value width (equal in this build) */
  int32_t n_text;     /* text tokens per (b, h) */
  int32_t chunk;      /* frames per chunk (5 in the paper) */
  int32_t anchors;    /* 1: frames 0 and T-1 are anchors (no write, no read) */
  int32_t in_dtype;   /* vdn_dtype of Q, K, V, Kx, Vx */
  int32_t out_dtype;  /* vdn_dtype of O */
  int32_t beta_per_token; /* 0: one write gate per frame, beta [B,H,T] and
                             beta_x [B,H]; 1: one per token ("Core method":
                             beta_{t,u}), beta [B,H,T,U] and beta_x
                             [B,H,n_text] */
  int32_t decay_bridge;   /* 0: frame t of chunk c reads R_c = F[max(c-1,0)]
                             + G[min(c+2,C)]; 1: the readout goes through the
                             decay bridge ("Method steps" step (5)):
                               R_t = F[max(c-1,0)] Diag(pf_t)
                                   + G[min(c+2,C)] Diag(pb_t),
                             pf_t = prod_{r=f0..t} alpha_r, pb_t =
                             prod_{r=t..f1} alpha_r over the window's frames
                             (f0 = chunk*max(c-1,0), f1 = min(chunk*(c+2),T)-1;
                             an anchor frame's alpha counts as 1): the states
                             outside the window carried to frame t through
                             the decay of the window's frames, whose writes
                             the softmax branch holds */
} vdn_shape;

/*
 * Frame statistics. Paper: "Method steps", step (3):
 *   A_t = K_t^T Diag(beta_t) K_t   [d_k, d_k]   (symmetric)
 *   B_t = V_t^T Diag(beta_t) K_t   [d_v, d_k]
 * with one scalar write gate beta_t per (b, h, t), or (shape.beta_per_token)
 * one gate beta_{t,u} per token.
 * In : K [B,H,T,U,dk], V [B,H,T,U,dv] (in_dtype); beta [B,H,T] or
 *      [B,H,T,U] float32.
 * Precision of the tensor-core path (bf16, d = 128) with per-token gates:
 * beta_{t,u} k_{t,u} is rounded to bf16 before the product (2^-9 relative per
 * term); with one gate per frame the products are exact and beta_t scales the
 * fp32 sums.
 * Out: A [B,H,T,dk,dk], Bm [B,H,T,dv,dk] float32 (fully overwritten).
 * Every frame, anchors included, is computed (the factor step skips anchors).
 * info: optional device int32 (may be NULL) that receives VDN_INFO_TIMEOUT if
 *       a pipeline wait runs out of time; it is not reset by this call.
 */
vdn_status vdn_frame_grams(const vdn_shape *s, const void *K, const void *V,
                           const float *beta, float *A, float *Bm,
                           int32_t *info, vdn_stream_t stream);

/*
 * Per-frame factor/solve. Paper: "Core method" (closed form
 * S_t = (S_{t-1} Diag(alpha_t) + B_t)(I + A_t)^{-1}) and "Method steps",
 * step (3) ("factor I + A_t in batch to get the transition M_t and the
 * injection J_t"):
 *   M_t = Diag(alpha_t) (I + A_t)^{-1},   J_t = B_t (I + A_t)^{-1},
 * so that S_t = S_{t-1} M_t + J_t. Anchor frames (shape.anchors) get M = I,
 * J = 0. The frames do not depend on the state and are factored in parallel.
 * In : A [B,H,T,dk,dk], Bm [B,H,T,dv,dk], alpha [B,H,T,dk] float32.
 * Out: M [B,H,T,dk,dk], J [B,H,T,dv,dk] float32; *info (device int32) is
 *      reset to 0 and then set as described in the file header.
 */
vdn_status vdn_frame_factor(const vdn_shape *s, const float *A, const float *Bm,
                            const float *alpha, float *M, float *J,
                            int32_t *info, vdn_stream_t stream);

/*
 * Per-frame inverse, the factor step as the fused path runs it:
 *   W_t = (I + A_t)^{-1}      (symmetric; anchors are not special-cased here)
 * so that M_t = Diag(alpha_t) W_t and J_t = B_t W_t. Paper: "Core method"
 * (closed form) and "Method steps" step (3); "Technical novelty" (the inverse
 * is produced directly, without a separate solve pipeline).
 * In : A [B,H,T,dk,dk] float32.  Out: W [B,H,T,dk,dk] float32.
 * *info is reset to 0 and then set as for vdn_frame_factor.
 * Shapes of the fused tensor-core pass (bf16 in/out, d = 128) use the blocked
 * symmetric sweep with the matrix in tensor memory, its rank-32 updates on
 * the tensor cores in split fp16 (about fp32 accuracy, relative error ~1e-6);
 * other shapes use the fp32 symmetric sweep on the CUDA cores. (The fused
 * passes themselves form the frames' inverses as a 2 x 2 block inverse whose
 * first half runs inside the Gram kernel.)
 */
vdn_status vdn_frame_invert(const vdn_shape *s, const float *A, float *W,
                            int32_t *info, vdn_stream_t stream);

/*
 * Chunk-level composition. Paper: "Technical novelty" (frame-level affine
 * transitions are composed into chunk-level transitions before the scan,
 * cutting the scan depth to about 1/5) and "Method steps", step (4)
 * (S_out = S_in M_chunk + J_chunk). For chunk c with frames f0 < ... < fn:
 *   forward : S -> S Mf_c + Jf_c applies frames f0, f1, ..., fn in order;
 *   backward: S -> S Mb_c + Jb_c applies frames fn, ..., f1, f0.
 * In : M [B,H,T,dk,dk], J [B,H,T,dv,dk] (from vdn_frame_factor).
 * Out: Mf, Mb [B,H,C,dk,dk]; Jf, Jb [B,H,C,dv,dk] float32.
 */
vdn_status vdn_chunk_compose(const vdn_shape *s, const float *M, const float *J,
                             float *Mf, float *Jf, float *Mb, float *Jb,
                             vdn_stream_t stream);

/*
 * Forward scan over chunk boundaries. Paper: "Core method" (the forward scan
 * summarises the context before the window; the text state initialises both
 * scans) and step (4) (half-and-half initialisation):
 *   F_0 = S_T / 2,   F_{c+1} = F_c Mf_c + Jf_c,   c = 0..C-1.
 * In : Mf [B,H,C,dk,dk], Jf [B,H,C,dv,dk], S_T [B,H,dv,dk].
 * Out: F [B,H,C+1,dv,dk] float32.
 */
vdn_status vdn_scan_fwd(const vdn_shape *s, const float *Mf, const float *Jf,
                        const float *S_T, float *F, vdn_stream_t stream);

/*
 * Backward scan, the mirror of vdn_scan_fwd:
 *   G_C = S_T / 2,   G_c = G_{c+1} Mb_c + Jb_c,   c = C-1..0.
 * Out: G [B,H,C+1,dv,dk] float32.
 */
vdn_status vdn_scan_bwd(const vdn_shape *s, const float *Mb, const float *Jb,
                        const float *S_T, float *G, vdn_stream_t stream);

/* Both scans in one launch, on separate thread blocks. */
vdn_status vdn_scan_bidir(const vdn_shape *s, const float *Mf, const float *Jf,
                          const float *Mb, const float *Jb, const float *S_T,
                          float *F, float *G, vdn_stream_t stream);

/*
 * Chunk readout. Paper: "Core method" (each query chunk keeps exact softmax
 * attention inside a chunk-aligned bidirectional 15-frame window; the linear
 * memory carries everything outside it; the forward and backward readouts are
 * summed, so nothing is counted twice) and step (2) (the linear branch drops
 * the anchor rows). For frame t of chunk c = t / chunk:
 *   R_c = F_{max(c-1,0)} + G_{min(c+2,C)},   o_{t,u} = R_c q_{t,u},
 * and o = 0 on anchor frames.
 * In : Q [B,H,T,U,dk] (in_dtype); F, G [B,H,C+1,dv,dk] float32.
 * Out: O [B,H,T,U,dv] (out_dtype, rounded to nearest even), fully written.
 * info: optional, as for vdn_frame_grams.
 */
vdn_status vdn_chunk_readout(const vdn_shape *s, const void *Q, const float *F,
                             const float *G, void *O, int32_t *info,
                             vdn_stream_t stream);
/* (vdn_chunk_readout and vdn_chunk_readout_gated take no alpha: with
 * shape.decay_bridge = 1 they return VDN_ERR_INVALID; use
 * vdn_chunk_readout_bridged.) */

/*
 * Readout epilogue. Paper: "Method steps", step (5) ("after the readout,
 * RMSNorm and a sigmoid gate") and "Core method" (the linear branch is gated
 * with an RMSNorm first). Every token's readout o (d_v channels) becomes
 *   y_i = o_i / sqrt(mean_j o_j^2 + eps) * norm_weight[h][i] * sigmoid(gate_i),
 * and anchor rows stay 0.
 */
typedef struct {
  const void *gate;         /* [B,H,T,U,dv] in_dtype: gate logits per token and channel */
  const float *norm_weight; /* [H, dv] float32: RMSNorm weight of each head */
  float eps;                /* > 0, finite */
} vdn_out_gate;

/*
 * vdn_chunk_readout followed by the epilogue above, in the same kernel (the
 * ungated O is never written). og must not be NULL; gate and norm_weight are
 * device pointers, 16-byte aligned. Same errors as vdn_chunk_readout, plus
 * VDN_ERR_INVALID for a bad og.
 */
vdn_status vdn_chunk_readout_gated(const vdn_shape *s, const void *Q, const float *F,
                                   const float *G, const vdn_out_gate *og, void *O,
                                   int32_t *info, vdn_stream_t stream);

/*
 * Chunk readout through the decay bridge (shape.decay_bridge = 1; see the
 * field's comment for R_t). Paper: "Method steps" step (5) (the states at the
 * window boundary continue through the decay bridge prod alpha_r before the
 * readout) and "Core method" (the frame recurrence Sbar_t = S_{t-1}
 * Diag(alpha_t)). In : Q, F, G as for vdn_chunk_readout; alpha [B,H,T,dk]
 * float32 (the decay gates of the scans). og: NULL, or the readout epilogue
 * as for vdn_chunk_readout_gated. Out: O [B,H,T,U,dv] (out_dtype), anchor
 * rows 0. Errors as for vdn_chunk_readout_gated, plus VDN_ERR_INVALID when
 * shape.decay_bridge is 0 or alpha is NULL/misaligned.
 */
vdn_status vdn_chunk_readout_bridged(const vdn_shape *s, const void *Q, const float *F,
                                     const float *G, const float *alpha,
                                     const vdn_out_gate *og, void *O, int32_t *info,
                                     vdn_stream_t stream);

/*
 * Text state. Paper: "Core method" (the text prompt is summarised into a text
 * state S^T that initialises both scans). Reading: one VDA update from the
 * zero state over the n_text text tokens, with gate beta_x and no decay:
 *   S_T = beta_x V_x^T K_x (I + beta_x K_x^T K_x)^{-1}.
 * In : Kx [B,H,n_text,dk], Vx [B,H,n_text,dv] (in_dtype); beta_x [B,H]
 *      float32, or [B,H,n_text] with shape.beta_per_token (then beta_x is a
 *      per-token vector in the formula above: K_x^T Diag(beta_x) K_x).
 * Out: S_T [B,H,dv,dk] float32; *info as for vdn_frame_factor.
 * workspace: device scratch of at least vdn_text_state_workspace_bytes(s)
 * bytes, 256-byte aligned, not read before it is written.
 */
size_t vdn_text_state_workspace_bytes(const vdn_shape *s);
vdn_status vdn_text_state(const vdn_shape *s, const void *Kx, const void *Vx,
                          const float *beta_x, float *S_T, void *workspace,
                          size_t workspace_bytes, int32_t *info,
                          vdn_stream_t stream);

/*
 * Text state without a caller workspace (the paper has no counterpart: this
 * is a deployment addition). Same result as vdn_text_state, for callers that
 * cannot allocate device memory, such as a serving engine that reserves all
 * of its memory at start-up or a real-time loop that must not call cudaMalloc.
 * The two Gram matrices per (b, h) go to a fixed 4 MiB scratch array that the
 * library keeps in device memory on every GPU that loads it, until exit; so
 * 2 * B * H * dk * dk * 4 bytes must not exceed 4 MiB (B*H <= 32 at d = 128),
 * else VDN_ERR_UNSUPPORTED is returned before anything is enqueued.
 * The first call on a device looks up the array's device address (once per
 * device and context, with that device current); make it before any stream
 * capture. A call after the device's context was destroyed and recreated
 * (cudaDeviceReset) looks the address up again.
 * Shapes are validated as for vdn_text_state, then against the scratch size.
 * Every call shares the array and it keeps the last call's contents (nothing
 * in it needs to start at zero); calls that overlap on the GPU race on it.
 * In/Out/info as for vdn_text_state. Allocates nothing.
 */
vdn_status vdn_text_state_noalloc(const vdn_shape *s, const void *Kx,
                                  const void *Vx, const float *beta_x,
                                  float *S_T, int32_t *info,
                                  vdn_stream_t stream);

/*
 * The whole linear branch in one call: text state, frame statistics,
 * factor, chunk composition, both scans and the chunk readout.
 * In : Q, K, V [B,H,T,U,d] and Kx, Vx [B,H,n_text,d] (in_dtype);
 *      beta [B,H,T], alpha [B,H,T,dk], beta_x [B,H] float32 (beta
 *      [B,H,T,U] and beta_x [B,H,n_text] with shape.beta_per_token).
 * Out: O [B,H,T,U,dv] (out_dtype). If F and G are not NULL they receive the
 *      boundary states [B,H,C+1,dv,dk]; *info as for vdn_frame_factor.
 * workspace: at least vdn_forward_workspace_bytes(s) bytes, 256-byte aligned.
 * stage_events: NULL, or 7 cudaEvent_t (entries may be NULL) recorded on
 *      `stream` before the text state and after the text state, the frame
 *      statistics, the factor, the composition, the scans and the readout.
 * With bf16 inputs and output and d = 128 the factor, composition and scans
 * run on the tensor-core path (per-frame inverses W_t, then
 * X <- (X Diag(alpha_t) + B_t) W_t chains, which equal X M_t + J_t); other
 * shapes use the CUDA-core kernels of the stage calls above.
 * og: NULL for O as read out, or the readout epilogue of
 *      vdn_chunk_readout_gated (O then holds y).
 * With shape.decay_bridge the readout goes through the decay bridge, as
 * vdn_chunk_readout_bridged with this call's alpha.
 */
size_t vdn_forward_workspace_bytes(const vdn_shape *s);
vdn_status vdn_forward(const vdn_shape *s, const void *Q, const void *K,
                       const void *V, const float *beta, const float *alpha,
                       const void *Kx, const void *Vx, const float *beta_x,
                       void *O, float *F, float *G, void *workspace,
                       size_t workspace_bytes, int32_t *info,
                       const void *const *stage_events, const vdn_out_gate *og,
                       vdn_stream_t stream);

/*
 * The fused pass of vdn_forward (bf16 inputs and output, d = 128 only) with
 * the text state on a second stream, `aux`, beside the frame Grams on
 * `stream`; the Grams may be split into `groups` launches over contiguous
 * head groups. The block inverse, the composition, the scans and the readout
 * then run over all pairs on `stream`. Same inputs, outputs, workspace and
 * *info as vdn_forward, bit for bit (a failing frame is reported by its
 * index over all B*H*T frames). The library records and waits on the
 * caller's events and creates or allocates nothing.
 * events: 8 + groups cudaEvent_t, none NULL: [0] start (stream); [1] / [2]
 *   before / after the text state (aux); [3 + g] after the Grams of group g
 *   (stream); at 3 + groups: +0 after `stream` waited for `aux`, +1 / +2 /
 *   +3 / +4 after the block inverse, the composition, the scans and the
 *   readout.
 *   On return `stream` has waited for all work on `aux`.
 */
vdn_status vdn_forward_pipelined(const vdn_shape *s, const void *Q, const void *K,
                                 const void *V, const float *beta,
                                 const float *alpha, const void *Kx,
                                 const void *Vx, const float *beta_x, void *O,
                                 float *F, float *G, void *workspace,
                                 size_t workspace_bytes, int32_t *info,
                                 int32_t groups, vdn_stream_t aux,
                                 const void *const *events, const vdn_out_gate *og,
                                 vdn_stream_t stream);

/*
 * Causal streaming variant: one segment of a live stream, read through the
 * forward memory only. Paper: "Video DeltaNet: A Video-Native Hybrid
 * Attention for Livestream Video Generation" (summary page) — the method
 * targets livestream generation ("Future directions": continuous generation
 * with streaming systems). In a stream the frames after the current segment
 * do not exist yet, so the backward scan cannot run; this call keeps the
 * forward scan, carried from segment to segment, and each chunk c of the
 * stream reads R_c = F_{max(c-1,0)} (the forward state before the chunk
 * ahead of it), with no backward term.
 * The segment holds frames frame0 .. frame0 + T - 1 of the stream (shape.T =
 * T; frame0 a multiple of shape.chunk; every segment but the stream's last
 * holds whole chunks). shape.n_text is not used: the text state enters
 * through the carried states. With shape.anchors the stream's first frame
 * (frame0 = 0 only) is an anchor; a stream has no last-frame anchor.
 * In : Q, K, V [B,H,T,U,d] (in_dtype); beta [B,H,T] (or [B,H,T,U] with
 *      beta_per_token), alpha [B,H,T,dk] float32;
 *      S_prev, S_in [B,H,dv,dk] float32: the stream's forward states before
 *      chunks c0 - 1 and c0 (c0 = frame0 / chunk); for the first segment
 *      both are the text state S^T (vdn_text_state), which a forward-only
 *      stream counts once.
 * Out: O [B,H,T,U,dv] (out_dtype); F [B,H,C+1,dv,dk] float32: F[0] = S_in
 *      and F[c+1] the state after the segment's chunk c (C = ceil(T /
 *      chunk)). The next segment continues from S_prev = F[C - 1] and
 *      S_in = F[C]. *info as for vdn_frame_factor.
 * workspace: at least vdn_stream_workspace_bytes(s) bytes, 256-byte aligned.
 * Errors: VDN_ERR_INVALID for a frame0 that is negative or not a multiple of
 * the chunk, and as for vdn_forward; VDN_ERR_UNSUPPORTED with
 * shape.decay_bridge (the bridge of a segment's first chunk needs the
 * previous segment's decay product: vdn_stream_segment_bridged takes it).
 * Same kernels as vdn_forward (the tensor-core path for bf16 d = 128), run in
 * one direction.
 */
size_t vdn_stream_workspace_bytes(const vdn_shape *s);
vdn_status vdn_stream_segment(const vdn_shape *s, const void *Q, const void *K,
                              const void *V, const float *beta, const float *alpha,
                              long long frame0, const float *S_prev, const float *S_in,
                              void *O, float *F, void *workspace,
                              size_t workspace_bytes, int32_t *info,
                              vdn_stream_t stream);

/*
 * A stream segment read through the decay bridge ("Method steps" step (5):
 * the state read at a window boundary is carried on through prod alpha_r),
 * forward half: frame t of chunk c reads
 *   R_t = F_{c-1} Diag(prod_{r=f0..t} alpha_r),
 * f0 the first frame of chunk c - 1, an anchor frame's alpha counting as 1.
 * The window of the segment's chunk 0 starts in the previous segment's last
 * chunk, so that chunk's decay product enters its factor:
 *   R_t = S_prev Diag(alpha_prev * prod_{r=0..t} alpha_r).
 * Needs shape.decay_bridge = 1. Arguments as for vdn_stream_segment, plus:
 * In : alpha_prev [B,H,dk] float32: the previous segment's alpha_tail; NULL
 *      (all ones) for the stream's first segment.
 * Out: alpha_tail [B,H,dk] float32 (may be NULL): prod alpha_r over this
 *      segment's last chunk, to pass as the next segment's alpha_prev.
 * Errors: as for vdn_stream_segment; VDN_ERR_INVALID without
 * shape.decay_bridge.
 */
vdn_status vdn_stream_segment_bridged(const vdn_shape *s, const void *Q,
                                      const void *K, const void *V,
                                      const float *beta, const float *alpha,
                                      long long frame0, const float *S_prev,
                                      const float *S_in, const float *alpha_prev,
                                      void *O, float *F, float *alpha_tail,
                                      void *workspace, size_t workspace_bytes,
                                      int32_t *info, vdn_stream_t stream);

/*
 * Self-test of the bounded pipeline waits that every tensor-core kernel uses:
 * launches one CTA whose threads wait, through the same bounded wait, on a
 * barrier that nothing arrives at. The wait gives up after its limit (1.5 s
 * of device time), the kernel writes VDN_INFO_TIMEOUT to *info and returns;
 * nothing traps or hangs, and the CUDA context stays usable. info: a device
 * int32 (overwritten). VDN_ERR_INVALID for a NULL info.
 */
vdn_status vdn_selftest_wait(int32_t *info, vdn_stream_t stream);

/* Name of a status code (static string). */
const char *vdn_status_string(vdn_status st);
/* Message of the last failing call on this thread ("" if none). */
const char *vdn_last_error(void);
/* Library version, major * 10000 + minor * 100 + patch. */
int32_t vdn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* VDN_H */
