/*
 * mta.h -- C ABI of libmta: Multi-Token Attention (MTA) forward on NVIDIA B200
 * (sm_100a).
 *
 * What is computed (sources are the pages' titles and sections):
 *   "Multi-Token Attention | Summary" (greeksharifa),
 *     section 2  : per-head logits A_hat = Q K^T / sqrt(d), causal -inf mask,
 *                  softmax over keys, A V, concatenation, output projection;
 *     section 3.1: A = Softmax(Mask_-inf(Conv2d_theta(Mask_0(A_hat)))), one
 *                  c_q x c_k kernel per head over (previous queries, neighbouring
 *                  keys);
 *     section 3.2: head mixing inside groups of c_h heads, before or after the
 *                  softmax (A1_new = w11 A1 + w12 A2, ...);
 *     section 3.3: group normalisation of each head's output with a scale;
 *   "Multi-Token Attention" (bycloud), mechanism item 3: group normalisation
 *     with depth scaling.
 *
 * Index conventions (the readings this library implements):
 *   theta[h][a][t] multiplies Mask_0(A_hat)[i-a][j-(t-c_k/2)], a = 0..c_q-1
 *   (current and previous queries), t = 0..c_k-1 (keys centred on j); entries
 *   outside [0,L) and future keys of the shifted query count as 0.  The
 *   identity kernel is theta[h][0][c_k/2] = 1.
 *   w_head[g][r][s] weighs source head g*c_h+s in destination head g*c_h+r.
 *   Post-softmax mixing is not renormalised; the mixed map of head r
 *   multiplies head r's own values.  Pre-softmax mixing follows the
 *   key-query convolution.  The post-softmax kernel theta_post[h][a][t]
 *   multiplies A[i-a][j-(t-c_k/2)] of the softmax weights in the same way;
 *   post-softmax mixing follows it.
 *
 * Ownership and threading: every pointer is a DEVICE pointer owned by the
 * caller (theta, w_head, gamma and beta included).  The library allocates no
 * memory and keeps no state between calls; scratch space comes from
 * cfg->workspace.  Calls are asynchronous on cfg->stream and re-entrant;
 * calls that share a workspace must be ordered on one stream.
 *
 * Errors: every argument is checked before anything is enqueued; a bad
 * argument returns MTA_ERR_INVALID / MTA_ERR_UNSUPPORTED / MTA_ERR_WORKSPACE
 * and enqueues nothing.  A failed launch returns MTA_ERR_CUDA.  Kernels never
 * wait without a bound: a wait that runs out sets a flag in the workspace and
 * the kernel returns; mta_sync_status() reports it as MTA_ERR_TIMEOUT.
 * Outputs must not alias inputs: an output whose bytes overlap an input's
 * (q, k, v or dout of the attention; x, Wqkv or Wo of the layer), or another
 * output's, is refused with MTA_ERR_INVALID.
 */
#ifndef MTA_H
#define MTA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MTA_ABI_VERSION 3

typedef enum {
  MTA_OK = 0,
  MTA_ERR_INVALID = 1,      /* null pointer, bad shape or inconsistent configuration */
  MTA_ERR_UNSUPPORTED = 2,  /* a valid configuration the library has no kernel for */
  MTA_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or smaller than required */
  MTA_ERR_CUDA = 4,         /* a CUDA runtime call or a kernel launch failed */
  MTA_ERR_TIMEOUT = 5       /* a kernel's bounded wait ran out (see mta_sync_status) */
} mta_status;

typedef enum { MTA_F32 = 0, MTA_BF16 = 1 } mta_dtype;

/* Where a mixing step sits relative to the softmax.  kq_place: OFF, PRE
 * (pre-softmax key-query convolution of Mask_0(A_hat), section 3.1) or
 * PRE_EXACT (the same convolution with the exact causal indicator: a tap at
 * output (i, j) reads A_hat[i-a][j-b] whenever its key j-b is not after the
 * output query i; section 3.1 contrasts it with the Mask_0 form).  head_place:
 * OFF, PRE or POST (section 3.2). */
typedef enum { MTA_OFF = 0, MTA_PRE = 1, MTA_POST = 2, MTA_PRE_EXACT = 3 } mta_place;

typedef struct mta_cfg {
  int B;                 /* batch size, >= 1                                     */
  int H;                 /* heads, >= 1, multiple of c_h                         */
  int L;                 /* sequence length, >= 1                                */
  int d;                 /* head dimension: 16..128, multiple of 8               */
  int c_q;               /* query taps of the key-query kernel, 1..8             */
  int c_k;               /* key taps, odd, 1..15                                 */
  int c_h;               /* heads per mixing group, 1..16 (1 = no mixing)        */
  int kq_place;          /* MTA_OFF, MTA_PRE or MTA_PRE_EXACT                    */
  int head_place;        /* MTA_OFF, MTA_PRE or MTA_POST (OFF when c_h == 1)     */
  int kq_post;           /* 1: a second key-query convolution acts on the softmax
                            weights (section 3.1: the kernel may act before or
                            after the softmax; section 4 uses both), then Mask_0
                            zeroes the future keys again: A' = Mask_0(Conv2d(A)),
                            not renormalised, before any post-softmax head mix;
                            its kernels follow the pre-softmax ones in theta_kq.
                            Served by the contraction kernel (bf16, c_q x c_k =
                            6 x 11, a pre-softmax convolution on) and by the
                            CUDA-core kernel; 0: none                            */
  int dtype;             /* mta_dtype of q, k, v and out (x, W and out in a layer) */
  int path;              /* attention kernel: 0 = choose (the contraction kernel
                            where it applies and the workspace holds its operands,
                            else the direct tensor-core kernel where it applies,
                            else the CUDA-core kernel); 1 = CUDA-core kernel;
                            2 = tensor-core kernel with the convolution on CUDA
                            cores; 3 = tensor-core kernel with the convolution as
                            a contraction of length c_q*d (MTA_ERR_UNSUPPORTED
                            where the forced kernel does not apply)             */
  float scale;           /* logit scale; 0 selects 1/sqrt(d)                     */
  long long qkv_row_stride; /* elements between consecutive tokens of q, k and v;
                              0 selects H*d (dense [B][L][H][d]); ignored by
                              mta_layer_fwd                                       */
  void *stream;          /* cudaStream_t to enqueue on; NULL = legacy default    */
  void *workspace;       /* device scratch, 256-byte aligned                      */
  size_t workspace_bytes;
  void *const *events;   /* optional timing events (cudaEvent_t handles created by
                            the caller, 0 .. 64 of them; NULL when n_events = 0):
                            a call records events[0] on cfg->stream just before
                            its first kernel and events[k] just after its k-th
                            kernel, while k < n_events, so that the time of each
                            kernel of the call can be read with
                            cudaEventElapsedTime.  The kernels of a call, in
                            order: mta_attn_fwd, the contraction path: the key
                            prepass, (with kq_post) the value prepass, the
                            attention kernel; other paths: the attention kernel.
                            mta_layer_fwd: the QKV GEMM, the attention kernels
                            as above (with the norm fused), or, on the CUDA-core
                            path, the attention kernel and then the stand-alone
                            group norm; the output GEMM.  mta_attn_bwd: the
                            whole backward (one mark after its last kernel).
                            mta_layer_bwd: see there.                            */
  int n_events;          /* number of handles in events, 0 .. 64                 */
} mta_cfg;

/* Scaled group normalisation of head outputs (section 3.3; bycloud item 3):
 * y = m_h * ((o - mean_d) / sqrt(var_d + eps) * gamma + beta) per (token, head h),
 * biased variance over the d channels of one head.  The multiplier m_h is the
 * depth scale lambda, or, with a gate, the sigmoid scalar gate of section 3.3:
 * m_h = 1 / (1 + exp(-gate[h])). */
typedef struct mta_gn {
  const float *gamma;    /* [H*d] device, fp32                                   */
  const float *beta;     /* [H*d] device, fp32                                   */
  float eps;             /* <= 0 selects 1e-5                                    */
  int layer;             /* layer index for the default depth scale             */
  float depth_scale;     /* lambda; < 0 selects 1 - 0.8*exp(-0.3*layer)         */
  const float *gate;     /* [H] device, fp32 gate logits; NULL = depth scale     */
} mta_gn;

/* Bytes of workspace mta_attn_fwd needs for cfg (0 if cfg is invalid): 256
 * bytes, plus, where the contraction kernel applies, its per-call operands
 * (the convolved keys, c_q*B*H*L*d fp16, their B*H*L fp32 scales,
 * B*H*L*(c_q-1+2*(c_k/2)) fp32 dot products, with post-softmax mixing an
 * exchange buffer of at most 160*4*d*128 fp32 for the kernel's persistent CTAs,
 * and with kq_post the values convolved by the post-softmax kernels,
 * n_v*c_q*B*H*L*d bf16, n_v = 2 with post-softmax mixing, else 1).
 * With a smaller workspace path 0 uses another kernel. */
size_t mta_attn_workspace_bytes(const mta_cfg *cfg);

/* MTA attention core, sections 2, 3.1, 3.2 (steps: logits, Mask_0, key-query
 * convolution, pre-softmax head mix, Mask_-inf, softmax, post-softmax head mix,
 * A V).  Never materialises an L x L map.
 *   q, k, v  : [B][L][H][d] with token stride cfg->qkv_row_stride, cfg->dtype
 *   theta_kq : [n][H][c_q][c_k] fp32, n = (kq_place != MTA_OFF) + kq_post: the
 *              pre-softmax kernels first, then the post-softmax kernels (NULL
 *              allowed when n == 0)
 *   w_head   : [H/c_h][c_h][c_h] fp32 (ignored when head_place == MTA_OFF)
 *   out      : [B][L][H][d] dense, cfg->dtype
 * Pointers to bf16 data must be 16-byte aligned and the row stride a multiple
 * of 8 elements for the tensor-core path; other layouts use the CUDA-core path. */
mta_status mta_attn_fwd(const void *q, const void *k, const void *v,
                        const float *theta_kq, const float *w_head,
                        const mta_cfg *cfg, void *out);

/* The attention kernel mta_attn_fwd would run for cfg, decided on the host
 * without enqueuing anything or calling CUDA: 1 = the CUDA-core kernel, 2 = the
 * direct tensor-core kernel, 3 = the contraction kernel (after its prepasses).
 * cfg->workspace_bytes counts as for mta_attn_fwd (the contraction kernel needs
 * its operands there); cfg->workspace is not read, and the tensors are taken to
 * be 16-byte aligned.  Returns -s for the status s the call would return
 * instead of launching (-MTA_ERR_INVALID, -MTA_ERR_UNSUPPORTED or
 * -MTA_ERR_WORKSPACE). */
int mta_attn_kernel(const mta_cfg *cfg);

/* Bytes of workspace mta_layer_fwd uses for cfg (0 if cfg is invalid): the
 * error word, QKV, the attention output and the normalised output (all bf16),
 * plus the contraction kernel's operands where it applies (as for
 * mta_attn_workspace_bytes).  The layer runs with less as long as the first
 * four fit; path 0 then takes another attention kernel. */
size_t mta_layer_workspace_bytes(const mta_cfg *cfg);

/* Full MTA attention layer (bf16 only):
 *   QKV = x Wqkv^T (section 2), attention as mta_attn_fwd, depth-scaled group
 *   norm (section 3.3), out = Y Wo^T (section 2).
 *   x    : [B][L][D] bf16, D = H*d
 *   Wqkv : [3D][D] bf16, rows [Q | K | V], each head-major (row h*d+e)
 *   Wo   : [D][D] bf16 (out x in)
 *   out  : [B][L][D] bf16
 * QKV and Y are kept in the workspace (bf16); no L x L map is stored. */
mta_status mta_layer_fwd(const void *x, const void *Wqkv, const float *theta,
                         const float *w_head, const mta_gn *gn, const void *Wo,
                         const mta_cfg *cfg, void *out);

/* mta_layer_fwd without a caller-supplied workspace.  The paper has no
 * counterpart to this entry point; it exists for callers that cannot allocate
 * device memory (for example a runtime that is handed device pointers to its
 * inputs and outputs by another component and has no allocator of its own, or
 * a loop that must not call cudaMalloc because allocation can synchronise the
 * device).  The layer's scratch lives in a static device buffer of
 * MTA_STATIC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits.  cfg->workspace and
 * cfg->workspace_bytes are ignored; everything else is as for mta_layer_fwd.
 * Returns MTA_ERR_WORKSPACE, enqueuing nothing, when the layer's fixed scratch
 * (mta_layer_workspace_bytes(cfg) less the contraction kernel's operands)
 * exceeds MTA_STATIC_SCRATCH_BYTES; the contraction kernel runs where the
 * whole of mta_layer_workspace_bytes(cfg) fits.  The first call on a device looks up the
 * buffer's address on that device (make it before any stream capture) and keeps
 * it for the life of the process; after cudaDeviceReset on a device that address
 * is stale, so do not call this entry point on a device after resetting it.  All
 * calls on a device share the buffer: calls that overlap on the GPU race, so
 * order them on one stream.  A bounded wait that runs out is recorded in the
 * static buffer and is not reported; use mta_layer_fwd with a workspace and
 * mta_sync_status to observe it.  Allocates no memory. */
#define MTA_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)
mta_status mta_layer_fwd_static(const void *x, const void *Wqkv, const float *theta,
                                const float *w_head, const mta_gn *gn, const void *Wo,
                                const mta_cfg *cfg, void *out);

/* Building blocks of mta_layer_fwd, exposed for testing and timing. */

/* C[M][N] = A[M][K] * Bm[N][K]^T, bf16 in, fp32 accumulate, bf16 out.
 * M, N, K >= 1; K a multiple of 8 and all pointers 16-byte aligned.
 * Enqueued on `stream`. */
mta_status mta_gemm_bf16_nt(const void *A, const void *Bm, void *C, int M, int N, int K,
                            void *stream);

/* y = depth-scaled group norm of o, both [tokens][H][d] bf16, dense. */
mta_status mta_group_norm_scale(const void *o, const mta_gn *gn, int tokens, int H, int d,
                                void *y, void *stream);

/* C[M][N] = A B^T, bf16 in, fp32 accumulate, as the layer's GEMMs run it.
 * A is [M][K] (a_mn = 0) or stored transposed as [K][M] (a_mn = 1); B is [N][K]
 * (b_mn = 0) or [K][N] (b_mn = 1); C is bf16 (f32_out = 0) or fp32 (1), dense.
 * All pointers 16-byte aligned; the contiguous extent of each operand (K for a
 * [rows][K] operand, M or N for a transposed one) a multiple of 8.  Enqueued on
 * `stream`. */
mta_status mta_gemm_bf16(const void *A, const void *Bm, void *C, int M, int N, int K, int a_mn, int b_mn,
                         int f32_out, void *stream);

/* Backward of mta_group_norm_scale as mta_layer_bwd runs it: for o [tokens][H][d]
 * bf16 and dy [tokens][H][d] fp32 writes y (the forward output, bf16) and
 * dout = dL/do (bf16), and overwrites dgamma, dbeta [H*d] and, with gn->gate,
 * dgate [H] (fp32, summed with atomic additions).  d in {32, 64, 96, 128}. */
mta_status mta_group_norm_scale_bwd(const void *o, const float *dy, const mta_gn *gn, int tokens, int H, int d,
                                    void *y, void *dout, float *dgamma, float *dbeta, float *dgate,
                                    void *stream);

/* Backward pass of mta_attn_fwd (the pages train with this forward; section 4).
 * Given dout = dL/dout, writes the gradients of q, k, v, of the key-query kernels
 * and of the head-mixing weights, each forward step taken in reverse order (see
 * attn_bwd_simt.cu for the chain of adjoints):
 *   q, k, v      : as for mta_attn_fwd (cfg->dtype, token stride cfg->qkv_row_stride)
 *   theta_kq     : [n][H][c_q][c_k] fp32 as for mta_attn_fwd (the pre-softmax
 *                  kernels when kq_place is on, then the post-softmax ones when
 *                  kq_post = 1)
 *   w_head       : [H/c_h][c_h][c_h] fp32 (ignored when head_place == MTA_OFF)
 *   dout         : [B][L][H][d] dense, cfg->dtype
 *   dq, dk, dv   : [B][L][H][d] dense fp32, overwritten
 *   dtheta       : [n][H][c_q][c_k] fp32, laid out as theta_kq, overwritten (may be
 *                  NULL; n = 0 leaves it unused)
 *   dw           : [H/c_h][c_h][c_h] fp32, overwritten (may be NULL; ignored when
 *                  head_place == MTA_OFF)
 * Two implementations (cfg->path):
 *   3: the contractions on the tensor cores (attn_bwd_tc.cu): bf16, d = 64, 96 or
 *      128, c_q = 6, c_k = 11, kq_place = MTA_PRE (with or without the
 *      post-softmax convolution, kq_post), c_h = 2 with head mixing; query
 *      blocks of R - 10 rows (R - 15 with kq_post; R = 384 up to L = 3072, else
 *      512), every head at once, their maps in strips of the workspace (S = s Q K^T, dA'' = dO V^T, dQ, dK, dV as batched
 *      tcgen05 GEMMs; the convolutions, their adjoints and the softmax on the
 *      CUDA cores).  MTA_ERR_UNSUPPORTED for other configurations,
 *      MTA_ERR_WORKSPACE when the strips do not fit.
 *   1: the CUDA cores in fp32 arithmetic, every forward configuration
 *      (attn_bwd_simt.cu; attn_bwd_post_simt.cu with the post-softmax
 *      convolution).
 *   0: 3 where it applies and the workspace holds its strips, else 1.
 *   2 returns MTA_ERR_UNSUPPORTED.
 * Both agree with fp64 to a relative error of about 1e-5: path 3 feeds its
 * computed MMA operands (dS, A'') as two bf16 halves.  dtheta and dw (both
 * paths) and dk, dv (path 1) are summed with atomic additions, so their last
 * bits may differ between runs.  The workspace (mta_attn_bwd_workspace_bytes)
 * holds the error word and, where path 3 applies, its strips: for one query
 * block of every head, an R-row S strip and two (three with pre-softmax mixing)
 * fp32 strips of R - 5 rows over the keys, and two bf16 strips of 2R rows
 * (B*H*pitch*(R*4 + 2*(R-5)*4 + 2*2R*2) bytes, pitch = L rounded up to 64, each
 * strip rounded up to 256 bytes; c_q = 6); with kq_post three more fp32 strips
 * (R - 5, R - 10 and R - 15 rows).  No L x L map is stored. */
size_t mta_attn_bwd_workspace_bytes(const mta_cfg *cfg);
mta_status mta_attn_bwd(const void *q, const void *k, const void *v, const float *theta_kq,
                        const float *w_head, const void *dout, const mta_cfg *cfg, float *dq,
                        float *dk, float *dv, float *dtheta, float *dw);

/* Backward pass of mta_layer_fwd: the gradients of the layer's every input and
 * parameter for dout = dL/dout, so that a training step of the layer runs through
 * the library (the pages train with this layer, section 4 and appendix F).  Each
 * forward step is taken in reverse ("Multi-Token Attention | Summary"
 * (greeksharifa), section 2 projections, sections 3.1-3.2 attention, section 3.3
 * group norm):
 *   1. QKV = x Wqkv^T and the attention output O are recomputed (as in
 *      mta_layer_fwd, cfg->path choosing the attention kernel);
 *   2. dY = dout Wo;
 *   3. the group norm's backward: Y, dO, dgamma, dbeta (and dgate);
 *   4. dWo = dout^T Y;
 *   5. the attention core's backward (as mta_attn_bwd, on the CUDA cores):
 *      dq, dk, dv, dtheta, dw;
 *   6. dx = dQKV Wqkv and dWqkv = dQKV^T x, dQKV = (dq | dk | dv) in bf16.
 * The GEMMs run on the tensor cores with bf16 operands and fp32 accumulation,
 * reading transposed operands in place (no transpose pass).
 *   x, Wqkv, theta, w_head, gn, Wo : as for mta_layer_fwd (bf16 only; gn->depth_scale
 *              has no gradient)
 *   dout     : [B][L][D] bf16
 *   dx       : [B][L][D] fp32, overwritten
 *   dWqkv    : [3D][D] fp32, dWo: [D][D] fp32, overwritten
 *   dtheta   : as for mta_attn_bwd (may be NULL); dw: as for mta_attn_bwd (may be NULL)
 *   dgamma, dbeta : [H*d] fp32, overwritten
 *   dgate    : [H] fp32, overwritten; required when gn->gate is set, else unused
 * d must be 32, 64, 96 or 128; x, Wqkv, Wo, dout, dx, dWqkv and dWo 16-byte aligned.
 * Outputs must not share memory with the inputs or with one another
 * (MTA_ERR_INVALID).  dk, dv, dtheta, dw, dgamma, dbeta and dgate are summed with
 * atomic additions, so the last bits of every gradient may differ between runs.
 * The workspace (mta_layer_bwd_workspace_bytes) holds, in this order, each at a
 * 256-byte boundary: 256 bytes of status; QKV [T][3D] bf16 (T = B*L); O [T][D]
 * bf16 (the attention output); Y [T][D] bf16; dY [T][D] fp32; dO [T][D] bf16; dq,
 * dk, dv [T][D] fp32 each; dQKV [T][3D] bf16; then the contraction kernel's
 * operands where they apply.  Each keeps its value after the call, for
 * inspection.  The call runs with the fixed part alone, the forward recompute
 * then taking another attention kernel under path 0.  Timing events
 * (cfg->events), in order: the QKV GEMM, the attention kernels as for
 * mta_attn_fwd, the dY GEMM, the group-norm backward, the dWo GEMM, the
 * attention backward, the dQKV pack, the dx GEMM, the dWqkv GEMM.  No L x L map
 * is stored. */
size_t mta_layer_bwd_workspace_bytes(const mta_cfg *cfg);
mta_status mta_layer_bwd(const void *x, const void *Wqkv, const float *theta, const float *w_head,
                         const mta_gn *gn, const void *Wo, const void *dout, const mta_cfg *cfg, float *dx,
                         float *dWqkv, float *dWo, float *dtheta, float *dw, float *dgamma, float *dbeta,
                         float *dgate);

/* Waits for cfg->stream and reports whether a kernel of the last call that used
 * cfg->workspace gave up a bounded wait (MTA_ERR_TIMEOUT), else MTA_OK or
 * MTA_ERR_CUDA.  Blocking; for tests and diagnostics. */
mta_status mta_sync_status(const mta_cfg *cfg);

/* Diagnostic of the library's failure reporting (the pages have no counterpart
 * to it): enqueues on cfg->stream one small kernel whose
 * mbarrier waits can never complete, with every wait bounded by limit_us
 * microseconds (1 .. 2,000,000) instead of the library's 2 s.  The kernel gives
 * up through the same path as the attention kernels: the first wait to run out
 * sets the error word at the start of cfg->workspace (which the call clears
 * first) and an abort flag, the other threads' waits then return at once, and
 * the kernel ends.  mta_sync_status(cfg) then returns MTA_ERR_TIMEOUT, and the
 * next call on the same workspace starts from a clear error word.  The two
 * unsigned words after the error word count the threads (128) whose first and
 * second wait gave up.  Nothing faults and no wait is unbounded.  Returns
 * MTA_ERR_INVALID for a null cfg or a limit out of range, MTA_ERR_WORKSPACE
 * without a 256-byte aligned workspace of at least 256 bytes (only
 * cfg->workspace, cfg->workspace_bytes and cfg->stream are read). */
mta_status mta_selftest_wait_timeout(const mta_cfg *cfg, unsigned limit_us);

/* Static description of a status code. */
const char *mta_status_string(mta_status s);

/* MTA_ABI_VERSION of the loaded library. */
int mta_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MTA_H */
