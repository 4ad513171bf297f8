// internal.h -- host-side launchers shared by the C-ABI layer (mta_api.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace mta {

// Bits of the error word kept at the start of the caller's workspace.
enum : unsigned { ERRBIT_TIMEOUT = 1u };

// Optional timing events of one call (mta_cfg.events): next() records events[i]
// on the call's stream, i = 0 just before the call's first kernel and i = k just
// after its k-th kernel, while i < n.
struct Marks {
  void *const *ev = nullptr;
  int n = 0, i = 0;
  cudaStream_t st = nullptr;
  cudaError_t next() {
    if (!ev || i >= n) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(ev[i++]), st);
  }
};

// Arguments of one attention call, already validated by the C-ABI layer.
struct AttnArgs {
  const void *q, *k, *v;  // [B][L][H][d], token stride rs elements
  long long rs;
  const float *theta;     // [H][c_q][c_k] pre-softmax kernels
  const float *theta_post;  // [H][c_q][c_k] post-softmax kernels (kqp == 1)
  const float *w;         // [H/c_h][c_h][c_h]
  void *out;              // [B][L][H][d] dense
  int B, H, L, d, cq, ck, ch, kq, hp, dtype;
  int kqp;                // 1: key-query convolution after the softmax as well
  float scale;
  unsigned *err;          // error word in the workspace
  cudaStream_t stream;
  Marks *marks;           // timing events of the call, or null
};
inline cudaError_t mark(const AttnArgs &a) { return a.marks ? a.marks->next() : cudaSuccess; }

// Depth-scaled group norm fused into an attention epilogue (optional).
struct GnArgs {
  const float *gamma, *beta;  // [H*d]
  float eps, lam;
  const float *gate;          // [H] sigmoid gate logits, replacing lam; may be null
};

// Generic CUDA-core kernel: every supported configuration, fp32 arithmetic.
size_t attn_simt_smem_bytes(const AttnArgs &a, int BR, int BC);
int attn_simt_pick_rows(const AttnArgs &a, int BC);  // 0 if nothing fits
cudaError_t launch_attn_simt(const AttnArgs &a);

// Backward pass of the attention (CUDA cores, fp32 arithmetic).
struct BwdArgs {
  const void *q, *k, *v;  // [B][L][H][d], token stride rs
  long long rs;
  const void *dout;       // [B][L][H][d] dense, gradient of the output
  const float *theta;     // [H][c_q][c_k]
  const float *w;         // [H/c_h][c_h][c_h]
  float *dq, *dk, *dv;    // [B][L][H][d] dense fp32
  float *dtheta;          // [H][c_q][c_k] or null
  float *dw;              // [H/c_h][c_h][c_h] or null
  const float *theta_post;  // [H][c_q][c_k] post-softmax kernels (kq_post)
  float *dtheta_post;       // their gradient (kq_post) or null
  int B, H, L, d, cq, ck, ch, kq, hp, dtype;
  int kqp;                // 1: the convolution also acts after the softmax
  float scale;
  cudaStream_t stream;
  unsigned *err;          // status word (bounded waits of the tensor-core path)
};
int attn_bwd_simt_pick_rows(const BwdArgs &a);  // 0 if nothing fits
// The backward with its contractions on the tensor cores (attn_bwd_tc.cu): the
// configurations it serves, its workspace (strips of every head for one query
// block), and the launch.
bool attn_bwd_tc_supported(const BwdArgs &a);
size_t attn_bwd_tc_workspace_bytes(int B, int H, int L, int cq, int hp, int kqp);
cudaError_t launch_attn_bwd_tc(const BwdArgs &a, void *ws);
cudaError_t launch_attn_bwd_simt(const BwdArgs &a);
// With the post-softmax convolution (kqp == 1).
int attn_bwd_post_pick_rows(const BwdArgs &a);
cudaError_t launch_attn_bwd_post(const BwdArgs &a);

// tcgen05 kernel (bf16, fused); attn_tc_supported() says whether it applies.
bool attn_tc_supported(const AttnArgs &a);
cudaError_t launch_attn_tc(const AttnArgs &a, const GnArgs *gn);

// Contraction form of the key-query convolution (tensor cores): a prepass
// builds the per-row-convolved keys Kt and the near-diagonal dot products U,
// then the attention kernel contracts shifted queries against Kt.
struct KqPrepArgs {
  const void *q, *k;      // [B][L][H][d] bf16, token stride rs
  long long rs;
  const float *theta;     // [H][c_q][c_k]
  void *kt;               // [B][H][c_q*d/64][L][64] fp16, key j's contraction operand by 64-element chunks, times 2^e_j
  float *fac;             // [B][H][lpad] scale_log2 * 2^-e_j (0 for j >= L)
  float *vp;              // [B][H][L][M] past dot products q[i] . k[i-m], m < M
  float scale_log2;       // logit scale times log2(e)
  int B, H, L, d, cq, ck, M, n_tiles, lpad;
  int exact;              // exact causal indicator: Vp[i][m] = q[i] . k[i-m+(cq-1)]
  unsigned *zero;         // n_zero words the prepass sets to 0 (counters of the attention kernel), or null
  int n_zero;
};
cudaError_t launch_kq_prep(const KqPrepArgs &a, cudaStream_t stream);
// Values convolved by the post-softmax kernels along the keys (bf16):
//   Vt[b][s][hd][a][j] = sum_t theta_post[s][a][t] v_{head(s,hd)}[j + t - c_k/2]
// for the source head s and, with post-softmax mixing (nvh = 2), both heads hd of
// its group, else (nvh = 1) head s itself; zero outside [0, L).
struct VtPrepArgs {
  const void *v;            // [B][L][H][d] bf16, token stride rs
  long long rs;
  const float *theta_post;  // [H][c_q][c_k]
  void *vt;                 // [B][H][nvh][c_q][L][d] bf16
  int B, H, L, d, cq, ck, nvh, n_tiles;
};
cudaError_t launch_vt_prep(const VtPrepArgs &a, cudaStream_t stream);
// Workspace bytes of the contraction path (beyond the error word) and whether it applies.
bool attn_kq_supported(const AttnArgs &a);
size_t attn_kq_workspace_bytes(int B, int H, int L, int d, int cq, int ck, int hp, int kqp);
// ws: workspace area for Kt / fac / Vp (attn_kq_workspace_bytes bytes, 256-byte aligned).
cudaError_t launch_attn_kq(const AttnArgs &a, const GnArgs *gn, void *ws);
// The contraction kernel on CTA pairs (attn_kq_pair.cu): the shapes it serves, the
// scratch it needs after the prepass's operands, and its launch.
bool attn_kq_pair_applies(int d, int kq, int hp, int kqp, int L);
size_t attn_kq_pair_scratch_bytes(int B, int H, int L, int d, int hp);
cudaError_t launch_attn_kq_pair(const AttnArgs &a, const GnArgs *gn, const KqPrepArgs &pa, void *scratch);

// tcgen05 GEMM: C[M][N] = A[M][K] * B[N][K]^T (bf16 -> fp32 -> bf16).
// Batched GEMM of the attention backward (gemm_batched.cu).  An operand tensor is
// a bf16 array seen through a four-dimensional TMA map: dims[0] contiguous, then
// three more with byte strides; one of positions 1 and 2 holds the row index and
// the other the head, position 3 the batch.
struct BgTensor {
  const void *base;
  unsigned long long dims[4];
  unsigned long long strides[3];  // bytes, of dims 1..3
  int pos_row;                    // 1 or 2
};
struct BgOperand {
  int mn;      // 1: MN-major (contiguous index = M or N, row index = K); 0: K-major
  int pos_row; // as the tensor's
  int off_mn;  // added to the M (or N) index
  int off_k;   // added to the K index
  // K index k reads the operand at k mod k_period (a multiple of 64; 0 = no
  // period), its M (N) index shifted by (k / k_period) * period_shift: two halves
  // of one operand summed in one GEMM against the same other operand
  int k_period;
  int period_shift;
};
struct BgArgs {
  int Z, H;         // batches z = b * H + h
  int M, N, K;
  float alpha;
  int accumulate;   // C += alpha A B^T instead of C = alpha A B^T
  float *C;         // element (b, h, m, n) at C + b*sb + h*sh + m*sm + n
  long long sb, sh, sm;
  BgOperand a, b;
  unsigned *err;
  int split_ok;     // accumulating into a zeroed C: the launcher may split K in two
  int c_pos_row;    // set by the launcher: position of m in the output map (1, or 2 when sh < sm)
  int ksplit;       // set by the launcher: K ranges per output tile (1 or 2)
};
// C is written through a TMA map: its base and the strides sm, sh, sb (in elements)
// must be multiples of 16 bytes; cudaErrorInvalidValue otherwise.
cudaError_t launch_gemm_batched(const BgTensor &A, const BgTensor &B, const BgArgs &args, cudaStream_t stream);

// C[M][N] = A B^T with A [M][K] (a_mn: stored [K][M]) and B [N][K] (b_mn: stored
// [K][N]), bf16 in, fp32 accumulate, bf16 or (f32_out) fp32 out.
cudaError_t launch_gemm(const void *A, const void *B, void *C, int M, int N, int K, bool a_mn, bool b_mn,
                        bool f32_out, unsigned *err, cudaStream_t stream);
cudaError_t launch_gemm_bf16_nt(const void *A, const void *B, void *C, int M, int N, int K,
                                unsigned *err, cudaStream_t stream);

// Depth-scaled group norm over [tokens][H][d] bf16.
cudaError_t launch_group_norm(const void *o, const GnArgs &gn, int tokens, int H, int d, void *y,
                              cudaStream_t stream);
// Backward of the group norm (d in {32, 64, 96, 128}): o, y, dout bf16 and dy fp32,
// all [tokens][H][d]; adds into dgamma, dbeta [H*d] and (with a gate) dgate [H].
cudaError_t launch_group_norm_bwd(const void *o, const float *dy, const GnArgs &gn, int tokens, int H, int d,
                                  void *y, void *dout, float *dgamma, float *dbeta, float *dgate,
                                  cudaStream_t stream);
// [tokens][3 H d] bf16 = (dq | dk | dv), each fp32 [tokens][H d]
cudaError_t launch_pack_qkv_grad(const float *dq, const float *dk, const float *dv, long long tokens, int hd,
                                 void *dqkv, cudaStream_t stream);

// Diagnostic: one CTA whose bounded waits cannot complete (selftest.cu); err is the
// workspace's error word, out[2] counters of the waits that gave up.
cudaError_t launch_wait_timeout_selftest(unsigned long long limit_ns, unsigned *err, unsigned *out,
                                         cudaStream_t stream);

// cuTensorMapEncodeTiled through the runtime's driver entry point.
// dims/strides innermost first; strides in bytes for dims 1..rank-1.
bool encode_tmap_bf16(void *map_out, const void *base, int rank, const unsigned long long *dims,
                      const unsigned long long *strides_bytes, const unsigned *box,
                      bool swizzle128);
// The same for fp32 elements.
bool encode_tmap_f32(void *map_out, const void *base, int rank, const unsigned long long *dims,
                     const unsigned long long *strides_bytes, const unsigned *box, bool swizzle128);

}  // namespace mta
