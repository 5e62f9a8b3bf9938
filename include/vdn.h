/*
 * vdn.h — C ABI of libvdn, the sm_100a (B200) implementation of the VDN-H3 hybrid
 * attention layer, forward pass.
 *
 * Method sources (page titles, with the passages each entry point follows):
 *   [ART]  "VDN-MiniMax-H3 开源：全新混合注意力加速视频生成，8步生成，近乎无损画质"
 *          (ModelScope community article), section 技术解读:
 *          "局部精确计算，远程线性记忆" paragraphs 1-4 and "独立门控，融合两条注意力分支".
 *   [BLOG] "MiniMax H3 加速五件套" (H3, accelerated), section III "VDN: Splitting
 *          Attention by Distance" (delta-rule linear attention).
 *   [CARD] "Video DeltaNet: Hybrid Attention to Speed Up Video Models with Near-Lossless
 *          Quality" (vdn-minimax-h3 model card), "Set up" (window softmax) and "Inference
 *          with Diffusers" (fp8 e4m3 inference).
 *
 * Notation: F latent frames, T tokens per frame, C frames per chunk, L text tokens,
 * H heads, D head dimension (32, 64 or 128), N_v = F*T video tokens, HD = H*D.
 *
 * Conventions shared by every entry point:
 *   - Tensors are caller-owned, contiguous, row-major, in the layout stated.  Video
 *     q/k/v are [N_v][H][D] frame-major (token t of frame f is row f*T + t); text kt/vt
 *     are [L][H][D].  Device pointers unless stated otherwise.
 *   - Element types follow vdn_dtype: VDN_F32 float, VDN_BF16 bfloat16 (raw 16-bit),
 *     VDN_E4M3 fp8 e4m3 bytes with per-head float scales.
 *   - The library never allocates or frees device memory and never synchronises
 *     implicitly (except vdn_check_device_status).  Work goes onto `stream` (a
 *     cudaStream_t; NULL = legacy default stream) of the current device.
 *   - `ws` is a caller-owned device workspace of at least the size the matching
 *     *_workspace_size function returns; its first 256 bytes hold the device status
 *     word, which kernels set when a bounded device wait gives up or a check fails.
 *     Calls that share one workspace must not overlap on the GPU.
 *   - All arguments are checked before anything is launched.  Errors are returned as
 *     a vdn_status; the library never aborts, throws or traps.  vdn_last_error() gives
 *     a message for the last failing call on the calling thread.
 */
#ifndef VDN_H_
#define VDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define VDN_API __attribute__((visibility("default")))
#else
#define VDN_API
#endif

typedef int vdn_status;
#define VDN_OK 0
#define VDN_ERR_INVALID_ARG 1   /* null pointer, bad shape, inconsistent sizes */
#define VDN_ERR_UNSUPPORTED 2   /* D not in {32,64,128}, dtype not supported here, no sm_100 */
#define VDN_ERR_WORKSPACE 3     /* workspace missing, misaligned or too small */
#define VDN_ERR_CUDA 4          /* a CUDA runtime call or launch failed */
#define VDN_ERR_TIMEOUT 5       /* a device wait hit its bound (vdn_check_device_status) */
#define VDN_ERR_DEVICE 6        /* a device-side check failed (vdn_check_device_status) */

/* VDN_E4M3: bf16 tensors, softmax branch in e4m3.  VDN_E4M3_PROJ: the same, and the
 * output projections in e4m3 too (whole layer and vdn_out_proj_e4m3 only). */
typedef enum { VDN_F32 = 0, VDN_BF16 = 1, VDN_E4M3 = 2, VDN_E4M3_PROJ = 3 } vdn_dtype;

/* Linear branch kind.  ELU1: phi = elu+1 linear attention with a normaliser ([ART]
 * 局部精确计算 para. 1-3).  DELTA: delta-rule state over frame-mean keys/values
 * ([BLOG] III). */
typedef enum { VDN_LIN_ELU1 = 0, VDN_LIN_DELTA = 1 } vdn_lin_kind;

typedef struct {
  int32_t frames;            /* F >= 1 */
  int32_t tokens_per_frame;  /* T >= 1 */
  int32_t chunk_frames;      /* C >= 1 (5 in the deployed model) */
  int32_t text_tokens;       /* L >= 0 */
  int32_t heads;             /* H >= 1 */
  int32_t head_dim;          /* D in {32, 64, 128} */
} vdn_shape;

typedef void *vdn_stream; /* cudaStream_t */

/* Library version (major*10000 + minor*100 + patch). */
VDN_API int vdn_version(void);

/* Message describing the last error on the calling thread ("" if none). */
VDN_API const char *vdn_last_error(void);

/* ------------------------------------------------------------------ layout
 * vdn_mask_layout_build — host only, synchronous, integer only, bit-exact.
 * [ART] 局部精确计算 para. 1 (chunks of C frames; a chunk sees itself and both
 * neighbour chunks; frames 0 and F-1 are anchors read by all and reading all; the
 * forward/backward memories hold the frames before/after the window, without window
 * and anchor frames), para. 2 (frame-7 illustration), para. 3 (text in the softmax set).
 * Chunks start at frame 0; the last chunk may be short.
 *
 * frame_tab: int32[F][8] per query frame: group, win_lo, win_hi, is_anchor, fwd_lo,
 *   fwd_hi, bwd_lo, bwd_hi.  win = [max(0,(c-1)C), min(F,(c+2)C)) for c = f/C, or
 *   [0, F) for an anchor; memory ranges are half-open frame ranges, empty = (0, 0).
 * group_tab: int32[cap][16] per group (maximal run of consecutive query frames with the
 *   same softmax set and memories): frame_lo, frame_hi, n_seg, 0, four (lo, hi) softmax
 *   key segments in the concatenated [text | video] key index space (text token j is
 *   j, video token n is L + n; segments sorted and merged; unused (0, 0)), fwd_lo,
 *   fwd_hi, bwd_lo, bwd_hi.
 * n_groups: receives G.  group_tab_cap: rows available; vdn_max_groups() rows always
 *   suffice.  Returns VDN_ERR_INVALID_ARG if cap < G (nothing written past cap). */
VDN_API vdn_status vdn_mask_layout_build(const vdn_shape *shape, int32_t *frame_tab, int32_t *group_tab,
                                 int32_t *n_groups, size_t group_tab_cap);

/* Upper bound on the group count: ceil(F/C) + 2. */
VDN_API int32_t vdn_max_groups(const vdn_shape *shape);

/* ------------------------------------------------------------------ workspaces
 * Bytes of workspace for vdn_hybrid_attn_fwd (all intermediates of the layer). */
VDN_API size_t vdn_hybrid_attn_workspace_size(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype);
/* Bytes of workspace for the step entry points below (tables, tile list, status). */
VDN_API size_t vdn_step_workspace_size(const vdn_shape *shape);
/* Clears the device status word of a workspace (enqueued on stream).  Call once after
 * allocating a workspace; vdn_check_device_status clears it again after each read. */
VDN_API vdn_status vdn_workspace_init(void *ws, size_t ws_bytes, vdn_stream stream);

/* ------------------------------------------------------------------ softmax branch
 * vdn_softmax_branch_fwd — local block-sparse softmax attention.  [ART] 局部精确计算
 * para. 1 and 3; [CARD] "Set up" (window softmax).  For each video query token and
 * head: O_s = softmax(q K^T * sm_scale) V over the text tokens plus every token of the
 * frames of the query's softmax set (window chunks and both anchors; anchors: all
 * frames).  sm_scale <= 0 selects 1/sqrt(D).
 *   dtype VDN_F32:  q,k,v,kt,vt float; o_s float.
 *   dtype VDN_BF16: q,k,v,kt,vt bf16;  o_s bf16 (fp32 accumulation, fp32 softmax).
 *   dtype VDN_E4M3: q,k,v,kt,vt e4m3 with scales = float[3][H] (q, k, v dequantisation
 *                   scales per head; text shares the video k/v scales), as written by
 *                   vdn_fp8_quant_per_head; P is rounded to e4m3 at unit scale for P.V;
 *                   o_s bf16; head_dim 128 only.
 *   lse: optional float[N_v][H], natural-log sum of exp of the scaled scores.
 * scales must be NULL unless dtype is VDN_E4M3. */
VDN_API vdn_status vdn_softmax_branch_fwd(const vdn_shape *shape, vdn_dtype dtype, const void *q, const void *k,
                                  const void *v, const void *kt, const void *vt, const float *scales,
                                  float sm_scale, void *o_s, float *lse, void *ws, size_t ws_bytes,
                                  vdn_stream stream);

/* vdn_softmax_branch_fwd_noalloc — the same softmax branch without a workspace.  The
 * pages have no counterpart: this is a library convenience for callers that cannot
 * allocate device memory, for example plug-ins that only receive tensors from a host
 * framework that owns all device memory, or code that must not allocate once running.
 * Such a caller cannot size and pass a workspace, so this call keeps its scratch
 * (status word, layout tables, query-tile list) in a fixed 256 KiB array that the
 * library holds in device memory on every GPU that loads it, until the process exits.
 * Nothing is allocated or freed: no cudaMalloc, no cudaFree, no allocating library call.
 *   - Arguments, checks and results as vdn_softmax_branch_fwd, for dtype VDN_F32 or
 *     VDN_BF16 (both entry points run the same argument checks).
 *   - Capacity: the array holds the layout tables (about 80 bytes per frame) and the
 *     query-tile list (32 bytes per tile of at most 256 query rows).  At 1008 tokens per
 *     frame in 5-frame chunks that is up to 1343 frames (about 1.35M video tokens); at 256
 *     tokens per frame, 2604 frames.  Larger shapes are rejected with VDN_ERR_WORKSPACE
 *     before any device work.
 *   - Every call looks up the array's device address in the context current at that
 *     moment (cudaGetSymbolAddress, a host-side lookup).  The first call on a device, or
 *     in a new context, also loads the library's device code there: make that first
 *     call before any stream capture.
 *   - Every call shares the one array, which keeps the last call's contents; each call
 *     clears the status word and rewrites the tables before its kernels run.  Calls
 *     that overlap on the GPU (other streams, other host threads) race on the array and
 *     must be serialised by the caller.
 *   - Device-side errors (a wait timeout, or a layout-table error that makes the softmax
 *     kernel skip its work and leave o_s and lse unwritten) are recorded in the array's
 *     status word but not reported: the call never synchronises.  Launch errors are
 *     returned. */
VDN_API vdn_status vdn_softmax_branch_fwd_noalloc(const vdn_shape *shape, vdn_dtype dtype, const void *q,
                                                  const void *k, const void *v, const void *kt, const void *vt,
                                                  float sm_scale, void *o_s, float *lse, vdn_stream stream);

/* vdn_fp8_quant_per_head — per-head e4m3 quantisation of the softmax branch's inputs
 * ([CARD] "Inference with Diffusers": fp8 e4m3).  For each head h and tensor X in
 * (q; k with kt; v with vt): s_X[h] = amax / 448 over the video rows and, for k and v,
 * the text rows too (text shares the video scale); X8 = e4m3(X / s_X[h]), round to
 * nearest even, saturating.  Inputs bf16 [N_v][H][D] and [L][H][D]; outputs e4m3 bytes
 * in the same layouts; scales float[3][H] (q, k, v), the dequantisation factors that
 * vdn_softmax_branch_fwd takes with VDN_E4M3.  An all-zero head gets scale 1.
 * Requires H*D <= 16384.  ws: vdn_step_workspace_size bytes. */
VDN_API vdn_status vdn_fp8_quant_per_head(const vdn_shape *shape, const void *q, const void *k, const void *v,
                                          const void *kt, const void *vt, void *q8, void *k8, void *v8, void *kt8,
                                          void *vt8, float *scales, void *ws, size_t ws_bytes, vdn_stream stream);

/* ------------------------------------------------------------------ linear branch
 * vdn_linear_state_build — per-frame states.  [ART] 局部精确计算 para. 1 (frame-wise
 * linear branch) and para. 3 (text written into the memories).
 *   ELU1:  S[F][H][D][D] = sum_{t in f} phi(k_t)^T v_t, z[F][H][D] = sum phi(k_t),
 *          S_txt[H][D][D], z_txt[H][D] the same over the L text tokens (not halved).
 *          phi = elu + 1.  S[f][h][i][j]: i indexes the key feature, j the value dim.
 *   DELTA: S <- kbar[F][H][D] (L2-normalised mean key of each frame), z <- vbar[F][H][D]
 *          (mean value), S_txt[H][D][D] = sum_text khat vt^T with per-token
 *          L2-normalised text keys (not halved); z_txt unused (may be NULL).
 * dtype VDN_F32 or VDN_BF16 (inputs); outputs float. */
VDN_API vdn_status vdn_linear_state_build(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype, const void *k,
                                  const void *v, const void *kt, const void *vt, float *S, float *z, float *S_txt,
                                  float *z_txt, void *ws, size_t ws_bytes, vdn_stream stream);

/* vdn_linear_state_scan — per-group memories, offset by the window.  [ART] 局部精确计算
 * para. 1-3.  G = groups of vdn_mask_layout_build; outputs [G][H][D][D] and [G][H][D].
 *   ELU1:  S_fwd[g] = S_txt/2 + sum_{f in [fwd_lo, fwd_hi)} S[f], S_bwd[g] likewise over
 *          [bwd_lo, bwd_hi); z the same.  Exclusive prefix/suffix over frames; frames 0
 *          and F-1 never enter.  beta unused.
 *   DELTA: S_fwd[g] = state after applying S <- (I - beta kbar kbar^T) S + beta kbar vbar^T
 *          for frames fwd_lo..fwd_hi-1 ascending from S_txt/2; S_bwd[g] the same for
 *          frames bwd_hi-1..bwd_lo descending.  beta float[F][H]; z/z_txt/z_fwd/z_bwd
 *          unused (may be NULL).  [BLOG] III. */
VDN_API vdn_status vdn_linear_state_scan(const vdn_shape *shape, vdn_lin_kind kind, const float *S, const float *z,
                                 const float *S_txt, const float *z_txt, const float *beta, float *S_fwd,
                                 float *S_bwd, float *z_fwd, float *z_bwd, void *ws, size_t ws_bytes,
                                 vdn_stream stream);

/* vdn_linear_read — read both memories at the query position.  [ART] 局部精确计算
 * para. 2-3.
 *   ELU1:  o = phi(q)(S_fwd+S_bwd) / (phi(q).(z_fwd+z_bwd)), 0 if the normaliser is 0.
 *   DELTA: o = (S_fwd+S_bwd)^T q/||q||.
 * q [N_v][H][D] and o_l [N_v][H][D] in dtype (VDN_F32 or VDN_BF16). */
VDN_API vdn_status vdn_linear_read(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype, const void *q,
                           const float *S_fwd, const float *S_bwd, const float *z_fwd, const float *z_bwd,
                           void *o_l, void *ws, size_t ws_bytes, vdn_stream stream);

/* vdn_linear_branch_bwd — backward of the elu+1 linear branch (gradients of
 * sum(o_l * do_l) over every video query row), for training the linear branch ([CARD]
 * "Training"; [ART] 分阶段适配 A1/A2 train it, with the softmax branch frozen).  Recomputes
 * the per-frame states and the groups' memories from k, v, kt, vt, then for every query row
 * dq = (Num dnum + Den dden) * phi'(q) with dnum = do / den, dden = -(do . o) / den (0 where
 * the normaliser is 0), and for every key row, with dS_f the sum of the groups' dNum =
 * sum phi(q)^T dnum over the groups whose memory holds frame f (all groups for the text):
 * dk = (dS_f v + dz_f) * phi'(k), dv = dS_f^T phi(k).  CUDA cores, fp32; every sum in a
 * fixed order, so a call repeats bit for bit.
 *   kind VDN_LIN_ELU1 and dtype VDN_BF16 only (VDN_ERR_UNSUPPORTED otherwise).
 *   q, k, v [N_v][H][D] and kt, vt [L][H][D] bf16; do_l float [N_v][H][D];
 *   dq, dk, dv float [N_v][H][D]; dkt, dvt float [L][H][D] (NULL allowed when L = 0).
 *   All pointers device memory, 16-byte aligned, owned by the caller.
 *   Layouts with more groups than the key kernel's shared memory can flag (29184 at
 *   D = 128; only one-frame chunks over tens of thousands of frames get there) give
 *   VDN_ERR_UNSUPPORTED before any device work.
 * ws: vdn_linear_branch_bwd_workspace_size(shape) bytes (tables, the states and memories,
 * and per-row and per-group scratch). */
VDN_API size_t vdn_linear_branch_bwd_workspace_size(const vdn_shape *shape);
VDN_API vdn_status vdn_linear_branch_bwd(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype, const void *q,
                                         const void *k, const void *v, const void *kt, const void *vt,
                                         const float *do_l, float *dq, float *dk, float *dv, float *dkt, float *dvt,
                                         void *ws, size_t ws_bytes, vdn_stream stream);

/* ------------------------------------------------------------------ fuse
 * vdn_hybrid_fuse — per-branch gates and RMSNorm.  [ART] 独立门控，融合两条注意力分支.
 *   g_s = sigmoid(q_h . w_gate_s[h]);  g_l = sigmoid(q_h W_l[h]) (G_l = D: element-wise,
 *   G_l = 1: scalar);  A[n] = [ g_s * O_s | g_l * gamma * O_l / sqrt(mean_D(O_l^2) + eps) ].
 * q, o_s, o_l [N_v][H][D] and a [N_v][2*H*D] (softmax half first, head-major) in dtype
 * (VDN_F32 or VDN_BF16); w_gate_s float[H][D]; w_gate_l float[H][D][G_l];
 * gamma float[H][D]. */
VDN_API vdn_status vdn_hybrid_fuse(const vdn_shape *shape, vdn_dtype dtype, const void *q, const void *o_s,
                           const void *o_l, const float *w_gate_s, const float *w_gate_l, int32_t G_l,
                           const float *gamma, float eps, void *a, vdn_stream stream);

/* vdn_out_proj — separate output projections of the two branches, summed.  [ART]
 * 独立门控 para. 1.  y[N_v][HD] = A[:, :HD] W_os^T + A[:, HD:] W_ol^T, with W_os, W_ol
 * [HD (out)][HD (in)] row-major; no bias (the residual add is the caller's).  dtype
 * VDN_F32 or VDN_BF16 for a, w and y (fp32 accumulation).  ws: vdn_step_workspace_size
 * bytes (its status word receives bounded-wait timeouts of the tensor-core kernel). */
VDN_API vdn_status vdn_out_proj(const vdn_shape *shape, vdn_dtype dtype, const void *a, const void *w_os,
                                const void *w_ol, void *y, void *ws, size_t ws_bytes, vdn_stream stream);

/* vdn_out_proj_e4m3 — the same projections with e4m3 operands on the tensor cores ([CARD]
 * "Inference with Diffusers": every wide Linear in fp8 e4m3).
 *   a8 [N_v][2*H*D] e4m3 codes; column c's value is a8 * a_scales[c / D], so a_scales
 *   float[2][H] holds one dequantisation scale per (branch half, head): softmax half
 *   first.  w_os, w_ol bf16 [HD][HD]; y bf16 [N_v][HD].
 *   Each call folds a_scales into an e4m3 copy of [W_os | W_ol] quantised with one scale
 *   per output column (its amax / 448, round to nearest, saturating), then runs one GEMM
 *   with K = 2HD, fp32 accumulation, the column scale applied to y.  Needs H*D a multiple
 *   of 256 (VDN_ERR_UNSUPPORTED otherwise).
 * ws: vdn_out_proj_e4m3_workspace_size(shape) bytes (status word and the weight copy). */
VDN_API size_t vdn_out_proj_e4m3_workspace_size(const vdn_shape *shape);
VDN_API vdn_status vdn_out_proj_e4m3(const vdn_shape *shape, const void *a8, const float *a_scales,
                                     const void *w_os, const void *w_ol, void *y, void *ws, size_t ws_bytes,
                                     vdn_stream stream);

/* ------------------------------------------------------------------ whole layer
 * vdn_hybrid_attn_fwd — the layer: both branches, fuse and projections, in one call.
 *   dtype VDN_F32:  every tensor float.
 *   dtype VDN_BF16: q,k,v,kt,vt,w_os,w_ol,y bf16.
 *   dtype VDN_E4M3: inputs as for VDN_BF16; the softmax branch quantises Q/K/V to e4m3
 *                   with per-head scales amax/448 ([CARD] "Inference with Diffusers").
 *   dtype VDN_E4M3_PROJ: as VDN_E4M3, and the output projections run in e4m3 as in
 *                   vdn_out_proj_e4m3: the branch epilogues write A as e4m3 codes with
 *                   per-head scales from static bounds (softmax half: the V scale, since
 *                   g_s O_s is a gated convex combination of V rows; linear half:
 *                   max|gamma_h| sqrt(D) / 448, since g_l gamma O_l / rms(O_l) is bounded
 *                   by it).  head_dim 128 and H*D a multiple of 256.
 *   kind selects the linear branch; beta float[F][H] for DELTA, else NULL.
 *   w_gate_s, w_gate_l (G_l columns), gamma as for vdn_hybrid_fuse; eps of RMSNorm.
 * ws: vdn_hybrid_attn_workspace_size(shape, kind, dtype) bytes. */
VDN_API vdn_status vdn_hybrid_attn_fwd(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype, const void *q,
                               const void *k, const void *v, const void *kt, const void *vt, const float *beta,
                               const float *w_gate_s, const float *w_gate_l, int32_t G_l, const float *gamma,
                               float eps, const void *w_os, const void *w_ol, void *y, void *ws,
                               size_t ws_bytes, vdn_stream stream);

/* vdn_hybrid_attn_fwd_partial — one rank's share of the layer split by heads across
 * GPUs ([CARD] "Set up" and "Inference with SGLang" run the model on 8 GPUs; heads are
 * independent through both branches and the fuse, so the split needs one exchange, a sum
 * of the projections' partial outputs).
 *   shape.heads is this rank's head count H_r; q, k, v, kt, vt, w_gate_s, w_gate_l,
 *   gamma are those heads' slices (layouts as for vdn_hybrid_attn_fwd with H = H_r);
 *   beta float[F][H_r] for DELTA.  w_os, w_ol are bf16 [out_features][H_r*D]: the
 *   columns of the full projections that multiply these heads' A columns.
 *   y_partial float [N_v][out_features] = A_r[:, :H_r D] w_os^T + A_r[:, H_r D:] w_ol^T.
 *   Summed over the ranks (for example an all-reduce or reduce-scatter), the partials
 *   give the layer's y in float.
 *   dtype VDN_BF16 or VDN_E4M3, head_dim 128, out_features a multiple of 32
 *   (VDN_ERR_UNSUPPORTED / VDN_ERR_INVALID_ARG otherwise).
 * ws: vdn_hybrid_attn_workspace_size(shape, kind, dtype) bytes with shape.heads = H_r. */
VDN_API vdn_status vdn_hybrid_attn_fwd_partial(const vdn_shape *shape, int32_t out_features, vdn_lin_kind kind,
                                               vdn_dtype dtype, const void *q, const void *k, const void *v,
                                               const void *kt, const void *vt, const float *beta,
                                               const float *w_gate_s, const float *w_gate_l, int32_t G_l,
                                               const float *gamma, float eps, const void *w_os, const void *w_ol,
                                               float *y_partial, void *ws, size_t ws_bytes, vdn_stream stream);

/* vdn_hybrid_attn_fwd_host — the layer with its per-call tensors in HOST memory.  No
 * counterpart in the pages: it is the streaming form of vdn_hybrid_attn_fwd.
 *   q, k, v, kt, vt (and beta for DELTA) are read from host memory and y is written to
 *   host memory; weights (w_gate_s, w_gate_l, gamma, w_os, w_ol) stay device pointers.
 *   Everything is enqueued on `stream`: one cudaMemcpyAsync per input into the staging
 *   area at the end of ws, the layer, and one copy of y back.  y_host is complete when
 *   the stream is.  Host buffers should be page-locked, or the copies do not overlap
 *   other work.  Calls on two streams with two workspaces overlap the copies of one
 *   call with the kernels of the other.
 * ws: vdn_hybrid_attn_host_workspace_size(shape, kind, dtype) bytes. */
VDN_API size_t vdn_hybrid_attn_host_workspace_size(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype);
VDN_API vdn_status vdn_hybrid_attn_fwd_host(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype,
                                            const void *q_host, const void *k_host, const void *v_host,
                                            const void *kt_host, const void *vt_host, const float *beta_host,
                                            const float *w_gate_s, const float *w_gate_l, int32_t G_l,
                                            const float *gamma, float eps, const void *w_os, const void *w_ol,
                                            void *y_host, void *ws, size_t ws_bytes, vdn_stream stream);

/* Device pointers (inside ws) of the layer's intermediates after vdn_hybrid_attn_fwd:
 * which = 0: O_s [N_v][H][D] (bf16, or float for VDN_F32); 1: O_l (same type);
 * 2: A [N_v][2HD]; 3: per-group S_fwd; 4: S_bwd (both NULL on the fused ELU1 path,
 * whose scan stores only the bf16 sum S_fwd + S_bwd); 5: frame table int32[F][8];
 * 6: group table int32[G][16]; 7: query-tile list int32[n][8] (group, row_lo, row_hi,
 * keys, first tile of the group, tiles of the group, 0, 0) of 256-row tiles, groups with
 * the longest key set first; 8: meta int32[2] (G, n); 9: scan plan int32
 * {nseg, G, 0, 0, bnd[F + 1], ie[max_groups], ib[max_groups]}: the frames [1, F-1) cut
 * at every memory boundary into nseg segments starting at bnd[j] (bnd[nseg] = F - 1);
 * group g's forward memory sums segments [0, ie[g]), its backward memory segments
 * [ib[g], nseg).  Entries 5-9 are also
 * written by the step entry points that take a workspace.  NULL if not materialised.
 * Valid until the next call that uses ws. */
VDN_API void *vdn_hybrid_attn_intermediate(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype, void *ws,
                                   int which);

/* ------------------------------------------------------------------ status
 * Synchronises `stream`, reads and clears the device status word in ws.  Returns
 * VDN_OK, VDN_ERR_TIMEOUT (a bounded device wait gave up) or VDN_ERR_DEVICE (another
 * device-side check failed); vdn_last_error() then names the kernel and block. */
VDN_API vdn_status vdn_check_device_status(void *ws, size_t ws_bytes, vdn_stream stream);

/* Test hook for the bounded device wait: launches one block that waits on a flag in ws
 * that nothing sets, giving up after `max_polls` polls (1 <= max_polls <= 10^6, about
 * 64 ms at most; other values give VDN_ERR_INVALID_ARG) and recording VDN_ERR_TIMEOUT in
 * the status word.  Read the outcome with vdn_check_device_status. */
VDN_API vdn_status vdn_debug_unset_flag_wait(void *ws, size_t ws_bytes, uint32_t max_polls, vdn_stream stream);

/* ------------------------------------------------------------------ kernel timing
 * Per-kernel device timing of the entry points (the layer, its steps and the linear
 * branch's backward) with CUDA events recorded on the launching stream around each kernel.  vdn_profile_begin enables recording (host state
 * of the calling process, up to max_launches launches); vdn_profile_end waits for the
 * recorded events, writes per kernel id k < n the summed milliseconds ms[k] and launch
 * count launches[k], and disables recording.  Kernel ids: 1 tables, 2 softmax (CUDA
 * cores), 3 softmax (tensor cores), 4 state build, 5 scan, 6 read, 7 fuse, 8 projection
 * (CUDA cores), 9 projection (tensor cores), 10 fp8 quantisation, 11 delta statistics,
 * 13 state build (tensor cores), 14 read staging, 15 read (tensor cores), and the linear
 * branch's backward: 16 per query row (dq), 17 per-frame gradient sums, 18 per key row
 * (dk, dv), 19 per-group gradient sums (its state rebuild and scan count as 4 and 5). */
#define VDN_PROF_KERNELS 20
VDN_API vdn_status vdn_profile_begin(int32_t max_launches);
VDN_API vdn_status vdn_profile_end(float *ms, int32_t *launches, int32_t n);

#ifdef __cplusplus
}
#endif
#endif /* VDN_H_ */
