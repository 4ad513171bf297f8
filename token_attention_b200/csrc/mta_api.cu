// mta_api.cu -- the C ABI declared in include/mta.h: argument checks, workspace
// layout, kernel selection.  Every check runs before anything is enqueued, and
// nothing here calls CUDA before the arguments have passed.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>

#include "internal.h"
#include "mta.h"

namespace mta {
namespace {

constexpr size_t kAlign = 256;
constexpr size_t kStatusBytes = 256;  // error word + padding at the workspace start

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shape and option checks shared by the attention and the layer.
mta_status check_cfg(const mta_cfg *c) {
  if (!c) return MTA_ERR_INVALID;
  if (c->B < 1 || c->H < 1 || c->L < 1) return MTA_ERR_INVALID;
  if (c->B > 65535) return MTA_ERR_UNSUPPORTED;
  if (c->d < 16 || c->d > 128 || c->d % 8 != 0) return MTA_ERR_UNSUPPORTED;
  if (c->c_q < 1 || c->c_q > 8) return MTA_ERR_INVALID;
  if (c->c_k < 1 || c->c_k > 15 || c->c_k % 2 == 0) return MTA_ERR_INVALID;
  if (c->c_h < 1 || c->c_h > 16 || c->H % c->c_h != 0) return MTA_ERR_INVALID;
  if (c->kq_place != MTA_OFF && c->kq_place != MTA_PRE && c->kq_place != MTA_PRE_EXACT)
    return MTA_ERR_INVALID;
  if (c->head_place != MTA_OFF && c->head_place != MTA_PRE && c->head_place != MTA_POST)
    return MTA_ERR_INVALID;
  if (c->kq_post != 0 && c->kq_post != 1) return MTA_ERR_INVALID;
  if (c->dtype != MTA_F32 && c->dtype != MTA_BF16) return MTA_ERR_INVALID;
  if (c->path < 0 || c->path > 3) return MTA_ERR_INVALID;
  if (!isfinite(c->scale) || c->scale < 0.f) return MTA_ERR_INVALID;
  if (c->n_events < 0 || c->n_events > 64 || (c->n_events > 0 && !c->events)) return MTA_ERR_INVALID;
  const long long hd = static_cast<long long>(c->H) * c->d;
  if (c->qkv_row_stride != 0 && c->qkv_row_stride < hd) return MTA_ERR_INVALID;
  return MTA_OK;
}

AttnArgs make_args(const void *q, const void *k, const void *v, const float *theta,
                   const float *w, const mta_cfg *c, void *out) {
  AttnArgs a;
  a.q = q; a.k = k; a.v = v; a.theta = theta; a.w = w; a.out = out;
  // theta holds the pre-softmax kernels (when kq_place is on), then the post-softmax ones
  a.kqp = c->kq_post;
  a.theta_post = (c->kq_post && theta)
                     ? theta + (c->kq_place != MTA_OFF ? static_cast<size_t>(c->H) * c->c_q * c->c_k : 0)
                     : nullptr;
  a.rs = c->qkv_row_stride ? c->qkv_row_stride : static_cast<long long>(c->H) * c->d;
  a.B = c->B; a.H = c->H; a.L = c->L; a.d = c->d;
  a.cq = c->c_q; a.ck = c->c_k; a.ch = c->c_h;
  a.kq = c->kq_place; a.hp = c->head_place; a.dtype = c->dtype;
  a.scale = c->scale > 0.f ? c->scale : 1.0f / sqrtf(static_cast<float>(c->d));
  a.err = static_cast<unsigned *>(c->workspace);
  a.stream = static_cast<cudaStream_t>(c->stream);
  a.marks = nullptr;
  return a;
}

Marks make_marks(const mta_cfg *c) {
  Marks m;
  m.ev = c->events;
  m.n = c->n_events;
  m.st = static_cast<cudaStream_t>(c->stream);
  return m;
}

enum Kernel { K_SIMT = 1, K_TC = 2, K_KQ = 3 };

// Shape-level test for the contraction kernel (pointer alignment aside): used
// to size the workspace.
bool kq_shape_ok(const mta_cfg *c) {
  return c->dtype == MTA_BF16 && (c->d == 64 || c->d == 96 || c->d == 128) &&
         (c->kq_place == MTA_PRE || c->kq_place == MTA_PRE_EXACT) &&
         c->c_q == 6 && c->c_k == 11 &&
         (c->head_place == MTA_OFF || ((c->head_place == MTA_PRE || c->head_place == MTA_POST) && c->c_h == 2));
}

size_t kq_bytes(const mta_cfg *c) {
  return kq_shape_ok(c) ? attn_kq_workspace_bytes(c->B, c->H, c->L, c->d, c->c_q, c->c_k, c->head_place,
                                                  c->kq_post)
                        : 0;
}

// Which attention kernel serves `a` under cfg->path: 0 chooses the contraction
// kernel where it applies and `kq_room` bytes of workspace hold its operands,
// else the direct tensor-core kernel where it applies, else the CUDA-core
// kernel; 1, 2, 3 force the CUDA-core, direct tensor-core, contraction kernel.
mta_status select_kernel(const AttnArgs &a, int path, size_t kq_room, Kernel *k) {
  const bool kq_ok = attn_kq_supported(a) &&
                     kq_room >= attn_kq_workspace_bytes(a.B, a.H, a.L, a.d, a.cq, a.ck, a.hp, a.kqp);
  const bool tc_ok = attn_tc_supported(a);
  const bool simt_ok = attn_simt_pick_rows(a, 32) != 0;
  if (path == 3) {
    if (!attn_kq_supported(a)) return MTA_ERR_UNSUPPORTED;
    if (!kq_ok) return MTA_ERR_WORKSPACE;
    *k = K_KQ;
  } else if (path == 2) {
    if (!tc_ok) return MTA_ERR_UNSUPPORTED;
    *k = K_TC;
  } else if (path == 1) {
    if (!simt_ok) return MTA_ERR_UNSUPPORTED;
    *k = K_SIMT;
  } else {
    *k = kq_ok ? K_KQ : tc_ok ? K_TC : K_SIMT;
    if (*k == K_SIMT && !simt_ok) return MTA_ERR_UNSUPPORTED;
  }
  return MTA_OK;
}

// Launches the attention kernel(s) of `k`, recording a timing mark after each.
cudaError_t launch_kernel(Kernel k, const AttnArgs &a, const GnArgs *gn, void *kq_ws) {
  if (k == K_KQ) return launch_attn_kq(a, gn, kq_ws);
  const cudaError_t e = k == K_TC ? launch_attn_tc(a, gn) : launch_attn_simt(a);
  return e != cudaSuccess ? e : mark(a);
}

// Whether the byte ranges [a, a + na) and [b, b + nb) share a byte.
bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

// Bytes spanned by q, k or v of cfg ([B][L][H][d] with token stride qkv_row_stride).
size_t qkv_span(const mta_cfg *c, size_t es) {
  const size_t rs = c->qkv_row_stride ? static_cast<size_t>(c->qkv_row_stride) : static_cast<size_t>(c->H) * c->d;
  return ((static_cast<size_t>(c->B) * c->L - 1) * rs + static_cast<size_t>(c->H) * c->d) * es;
}

// A dense [B][L][H][d] output of element size oes must not share memory with q, k or v.
bool output_aliases_qkv(const void *q, const void *k, const void *v, const mta_cfg *c, const void *out,
                        size_t oes) {
  const size_t es = c->dtype == MTA_F32 ? 4 : 2, n = qkv_span(c, es);
  const size_t no = static_cast<size_t>(c->B) * c->L * c->H * c->d * oes;
  return overlaps(out, no, q, n) || overlaps(out, no, k, n) || overlaps(out, no, v, n);
}

mta_status check_attn_pointers(const void *q, const void *k, const void *v, const float *theta,
                               const float *w, const mta_cfg *c, const void *out) {
  if (!q || !k || !v || !out) return MTA_ERR_INVALID;
  if ((c->kq_place != MTA_OFF || c->kq_post) && !theta) return MTA_ERR_INVALID;
  if (c->head_place != MTA_OFF && !w) return MTA_ERR_INVALID;
  const size_t es = c->dtype == MTA_F32 ? 4 : 2;
  if (!aligned(q, es) || !aligned(k, es) || !aligned(v, es) || !aligned(out, es))
    return MTA_ERR_INVALID;
  if ((theta && !aligned(theta, 4)) || (w && !aligned(w, 4))) return MTA_ERR_INVALID;
  return MTA_OK;
}

mta_status check_workspace(const mta_cfg *c, size_t need) {
  if (!c->workspace || c->workspace_bytes < need || !aligned(c->workspace, kAlign))
    return MTA_ERR_WORKSPACE;
  return MTA_OK;
}

// Clears the first 16 bytes of the status area: the error word (0), the
// self-test's counters (1, 2) and the attention kernel's work-queue counter (3).
mta_status clear_status(const mta_cfg *c) {
  return cudaMemsetAsync(c->workspace, 0, 4 * sizeof(unsigned), static_cast<cudaStream_t>(c->stream)) ==
                 cudaSuccess
             ? MTA_OK
             : MTA_ERR_CUDA;
}

size_t layer_tokens(const mta_cfg *c) { return static_cast<size_t>(c->B) * c->L; }

GnArgs make_gn(const mta_gn *gn) {
  GnArgs g;
  g.gamma = gn->gamma;
  g.beta = gn->beta;
  g.eps = gn->eps > 0.f ? gn->eps : 1e-5f;
  g.lam = gn->depth_scale >= 0.f ? gn->depth_scale
                                 : static_cast<float>(1.0 - 0.8 * exp(-0.3 * gn->layer));
  g.gate = gn->gate;
  return g;
}

// The attention backward's arguments (see mta_attn_bwd).
BwdArgs make_bwd_args(const void *q, const void *k, const void *v, const float *theta_kq, const float *w_head,
                      const void *dout, const mta_cfg *cfg, float *dq, float *dk, float *dv, float *dtheta,
                      float *dw) {
  BwdArgs a;
  a.q = q; a.k = k; a.v = v; a.dout = dout;
  a.rs = cfg->qkv_row_stride ? cfg->qkv_row_stride : static_cast<long long>(cfg->H) * cfg->d;
  a.theta = theta_kq; a.w = w_head;
  a.dq = dq; a.dk = dk; a.dv = dv;
  // theta_kq (and dtheta) hold the pre-softmax kernels when on, then the post-softmax ones
  const size_t nth = static_cast<size_t>(cfg->H) * cfg->c_q * cfg->c_k;
  a.dtheta = cfg->kq_place != MTA_OFF ? dtheta : nullptr;
  a.kqp = cfg->kq_post;
  a.theta_post = cfg->kq_post ? theta_kq + (cfg->kq_place != MTA_OFF ? nth : 0) : nullptr;
  a.dtheta_post = (cfg->kq_post && dtheta) ? dtheta + (cfg->kq_place != MTA_OFF ? nth : 0) : nullptr;
  a.dw = cfg->head_place != MTA_OFF ? dw : nullptr;
  a.B = cfg->B; a.H = cfg->H; a.L = cfg->L; a.d = cfg->d;
  a.cq = cfg->c_q; a.ck = cfg->c_k; a.ch = cfg->c_h;
  a.kq = cfg->kq_place; a.hp = cfg->head_place; a.dtype = cfg->dtype;
  a.scale = cfg->scale > 0.f ? cfg->scale : 1.0f / sqrtf(static_cast<float>(cfg->d));
  a.stream = static_cast<cudaStream_t>(cfg->stream);
  a.err = static_cast<unsigned *>(cfg->workspace);
  return a;
}

bool bwd_supported(const BwdArgs &a) {
  return (a.kqp ? attn_bwd_post_pick_rows(a) : attn_bwd_simt_pick_rows(a)) != 0;
}

// The tensor-core backward's strips for cfg, or 0 where its shape does not apply
// (pointer alignment aside).
size_t bwd_tc_bytes(const mta_cfg *c) {
  const bool shape = c->dtype == MTA_BF16 && (c->d == 64 || c->d == 96 || c->d == 128) && c->c_q == 6 && c->c_k == 11 &&
                     c->kq_place == MTA_PRE && (c->head_place == MTA_OFF || c->c_h == 2);
  return shape ? attn_bwd_tc_workspace_bytes(c->B, c->H, c->L, c->c_q, c->head_place, c->kq_post) : 0;
}

// Which backward serves `a`: path 0 the tensor-core one where it applies and
// `room` bytes hold its strips, else the CUDA-core one; 1 the CUDA-core one; 3
// the tensor-core one.  Returns the status of the choice; *tc says which.
mta_status select_bwd(const BwdArgs &a, const mta_cfg *cfg, int path, size_t room, bool *tc) {
  const bool tc_shape = attn_bwd_tc_supported(a);
  const size_t need = bwd_tc_bytes(cfg);
  if (path == 3) {
    if (!tc_shape || need == 0) return MTA_ERR_UNSUPPORTED;
    if (room < need) return MTA_ERR_WORKSPACE;
    *tc = true;
    return MTA_OK;
  }
  if (path == 2) return MTA_ERR_UNSUPPORTED;
  *tc = path == 0 && tc_shape && need != 0 && room >= need;
  if (!*tc && !bwd_supported(a)) return MTA_ERR_UNSUPPORTED;
  return MTA_OK;
}

// The layer backward's fixed scratch, in this order (each 256-byte aligned): the
// error word; QKV, O, Y (bf16); dY (fp32); dO (bf16); the attention core's fp32
// gradients dq, dk, dv; dQKV (bf16).  All of them hold their values after the call.
size_t layer_bwd_fixed_bytes(const mta_cfg *cfg) {
  if (check_cfg(cfg) != MTA_OK) return 0;
  const size_t T = static_cast<size_t>(cfg->B) * cfg->L, D = static_cast<size_t>(cfg->H) * cfg->d;
  return kStatusBytes + 2 * align_up(T * 3 * D * 2) + 3 * align_up(T * D * 2) + 4 * align_up(T * D * 4);
}

}  // namespace

namespace {
bool encode_tmap(CUtensorMapDataType dtype, void *map_out, const void *base, int rank,
                 const unsigned long long *dims, const unsigned long long *strides_bytes, const unsigned *box,
                 bool swizzle128) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  if (!fn) return false;
  cuuint64_t gdim[5], gstr[4];
  cuuint32_t bdim[5], estr[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estr[i] = 1;
    if (i > 0) gstr[i - 1] = strides_bytes[i - 1];
  }
  CUresult r = fn(static_cast<CUtensorMap *>(map_out), dtype,
                  static_cast<cuuint32_t>(rank), const_cast<void *>(base), gdim, gstr, bdim, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
}  // namespace

bool encode_tmap_bf16(void *map_out, const void *base, int rank, const unsigned long long *dims,
                      const unsigned long long *strides_bytes, const unsigned *box, bool swizzle128) {
  return encode_tmap(CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, map_out, base, rank, dims, strides_bytes, box, swizzle128);
}

bool encode_tmap_f32(void *map_out, const void *base, int rank, const unsigned long long *dims,
                     const unsigned long long *strides_bytes, const unsigned *box, bool swizzle128) {
  return encode_tmap(CU_TENSOR_MAP_DATA_TYPE_FLOAT32, map_out, base, rank, dims, strides_bytes, box, swizzle128);
}

// The layer's fixed scratch: error word, QKV, attention output O, normalised Y
// (the contraction kernel's operands come on top where they fit).
size_t layer_base_workspace_bytes(const mta_cfg *cfg) {
  if (check_cfg(cfg) != MTA_OK) return 0;
  const size_t T = layer_tokens(cfg), D = static_cast<size_t>(cfg->H) * cfg->d;
  return kStatusBytes + align_up(T * 3 * D * 2) + 2 * align_up(T * D * 2);
}

}  // namespace mta

using namespace mta;

extern "C" {

int mta_abi_version(void) { return MTA_ABI_VERSION; }

const char *mta_status_string(mta_status s) {
  switch (s) {
    case MTA_OK: return "ok";
    case MTA_ERR_INVALID: return "invalid argument";
    case MTA_ERR_UNSUPPORTED: return "unsupported configuration";
    case MTA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MTA_ERR_CUDA: return "CUDA error";
    case MTA_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
  }
  return "unknown status";
}

size_t mta_attn_workspace_bytes(const mta_cfg *cfg) {
  if (check_cfg(cfg) != MTA_OK) return 0;
  return kStatusBytes + kq_bytes(cfg);
}

mta_status mta_attn_fwd(const void *q, const void *k, const void *v, const float *theta_kq,
                        const float *w_head, const mta_cfg *cfg, void *out) {
  mta_status s = check_cfg(cfg);
  if (s != MTA_OK) return s;
  if ((s = check_attn_pointers(q, k, v, theta_kq, w_head, cfg, out)) != MTA_OK) return s;
  if (output_aliases_qkv(q, k, v, cfg, out, cfg->dtype == MTA_F32 ? 4 : 2)) return MTA_ERR_INVALID;
  if ((s = check_workspace(cfg, kStatusBytes)) != MTA_OK) return s;
  AttnArgs a = make_args(q, k, v, theta_kq, w_head, cfg, out);
  Kernel kern = K_SIMT;
  if ((s = select_kernel(a, cfg->path, cfg->workspace_bytes - kStatusBytes, &kern)) != MTA_OK) return s;
  if ((s = clear_status(cfg)) != MTA_OK) return s;
  Marks m = make_marks(cfg);
  a.marks = &m;
  if (m.next() != cudaSuccess) return MTA_ERR_CUDA;
  const cudaError_t e = launch_kernel(kern, a, nullptr, static_cast<char *>(cfg->workspace) + kStatusBytes);
  return e == cudaSuccess ? MTA_OK : MTA_ERR_CUDA;
}

int mta_attn_kernel(const mta_cfg *cfg) {
  mta_status s = check_cfg(cfg);
  if (s != MTA_OK) return -static_cast<int>(s);
  if (cfg->workspace_bytes < kStatusBytes) return -static_cast<int>(MTA_ERR_WORKSPACE);
  // no tensor is read: null pointers stand for 16-byte aligned ones
  const AttnArgs a = make_args(nullptr, nullptr, nullptr, nullptr, nullptr, cfg, nullptr);
  Kernel kern = K_SIMT;
  if ((s = select_kernel(a, cfg->path, cfg->workspace_bytes - kStatusBytes, &kern)) != MTA_OK)
    return -static_cast<int>(s);
  return static_cast<int>(kern);
}

size_t mta_layer_workspace_bytes(const mta_cfg *cfg) {
  const size_t base = layer_base_workspace_bytes(cfg);
  return base ? base + kq_bytes(cfg) : 0;
}

mta_status mta_layer_fwd(const void *x, const void *Wqkv, const float *theta, const float *w_head,
                         const mta_gn *gn, const void *Wo, const mta_cfg *cfg, void *out) {
  mta_status s = check_cfg(cfg);
  if (s != MTA_OK) return s;
  if (cfg->dtype != MTA_BF16) return MTA_ERR_UNSUPPORTED;
  if (!x || !Wqkv || !Wo || !out || !gn || !gn->gamma || !gn->beta) return MTA_ERR_INVALID;
  if ((cfg->kq_place != MTA_OFF || cfg->kq_post) && !theta) return MTA_ERR_INVALID;
  if (cfg->head_place != MTA_OFF && !w_head) return MTA_ERR_INVALID;
  if (theta && !aligned(theta, 4)) return MTA_ERR_INVALID;
  if (!aligned(x, 16) || !aligned(Wqkv, 16) || !aligned(Wo, 16) || !aligned(out, 16) ||
      !aligned(gn->gamma, 4) || !aligned(gn->beta, 4))
    return MTA_ERR_INVALID;
  const size_t T = layer_tokens(cfg), D = static_cast<size_t>(cfg->H) * cfg->d;
  if (T > static_cast<size_t>(65535) * 128 || 3 * D > static_cast<size_t>(1) << 30)
    return MTA_ERR_UNSUPPORTED;
  if (overlaps(out, T * D * 2, x, T * D * 2) || overlaps(out, T * D * 2, Wqkv, 3 * D * D * 2) ||
      overlaps(out, T * D * 2, Wo, D * D * 2))
    return MTA_ERR_INVALID;
  if ((s = check_workspace(cfg, layer_base_workspace_bytes(cfg))) != MTA_OK) return s;

  char *ws = static_cast<char *>(cfg->workspace);
  void *qkv = ws + kStatusBytes;
  void *obuf = ws + kStatusBytes + align_up(T * 3 * D * 2);
  void *ybuf = static_cast<char *>(obuf) + align_up(T * D * 2);
  const uint16_t *qkvb = static_cast<const uint16_t *>(qkv);  // bf16 elements

  mta_cfg acfg = *cfg;
  acfg.qkv_row_stride = static_cast<long long>(3 * D);
  AttnArgs a = make_args(qkvb, qkvb + D, qkvb + 2 * D, theta, w_head, &acfg, obuf);
  void *kq_ws = static_cast<char *>(ybuf) + align_up(T * D * 2);
  const size_t kq_room = cfg->workspace_bytes - (static_cast<char *>(kq_ws) - ws);
  Kernel kern = K_SIMT;
  if ((s = select_kernel(a, cfg->path, kq_room, &kern)) != MTA_OK) return s;

  const GnArgs g = make_gn(gn);
  cudaStream_t st = static_cast<cudaStream_t>(cfg->stream);
  unsigned *err = static_cast<unsigned *>(cfg->workspace);
  if ((s = clear_status(cfg)) != MTA_OK) return s;
  Marks m = make_marks(cfg);
  a.marks = &m;
  if (m.next() != cudaSuccess) return MTA_ERR_CUDA;
  // QKV = x Wqkv^T
  if (launch_gemm_bf16_nt(x, Wqkv, qkv, static_cast<int>(T), static_cast<int>(3 * D),
                          static_cast<int>(D), err, st) != cudaSuccess || m.next() != cudaSuccess)
    return MTA_ERR_CUDA;
  if (kern != K_SIMT) {
    // attention with the group norm and depth scale fused into its epilogue: Y
    a.out = ybuf;
    if (launch_kernel(kern, a, &g, kq_ws) != cudaSuccess) return MTA_ERR_CUDA;
  } else {
    // attention output O, then the stand-alone group norm O -> Y
    a.out = obuf;
    if (launch_kernel(kern, a, nullptr, kq_ws) != cudaSuccess) return MTA_ERR_CUDA;
    if (launch_group_norm(obuf, g, static_cast<int>(T), cfg->H, cfg->d, ybuf, st) != cudaSuccess ||
        m.next() != cudaSuccess)
      return MTA_ERR_CUDA;
  }
  // out = Y Wo^T
  if (launch_gemm_bf16_nt(ybuf, Wo, out, static_cast<int>(T), static_cast<int>(D),
                          static_cast<int>(D), err, st) != cudaSuccess || m.next() != cudaSuccess)
    return MTA_ERR_CUDA;
  return MTA_OK;
}

size_t mta_attn_bwd_workspace_bytes(const mta_cfg *cfg) {
  return check_cfg(cfg) == MTA_OK ? kStatusBytes + bwd_tc_bytes(cfg) : 0;
}

mta_status mta_attn_bwd(const void *q, const void *k, const void *v, const float *theta_kq,
                        const float *w_head, const void *dout, const mta_cfg *cfg, float *dq,
                        float *dk, float *dv, float *dtheta, float *dw) {
  mta_status s = check_cfg(cfg);
  if (s != MTA_OK) return s;
  if (cfg->path == 2) return MTA_ERR_UNSUPPORTED;
  if ((s = check_attn_pointers(q, k, v, theta_kq, w_head, cfg, dout)) != MTA_OK) return s;
  if (!dq || !dk || !dv || !aligned(dq, 4) || !aligned(dk, 4) || !aligned(dv, 4)) return MTA_ERR_INVALID;
  {
    const size_t es = cfg->dtype == MTA_F32 ? 4 : 2;
    const size_t ng = static_cast<size_t>(cfg->B) * cfg->L * cfg->H * cfg->d * 4;
    for (const float *g : {dq, dk, dv})
      if (output_aliases_qkv(q, k, v, cfg, g, 4) || overlaps(g, ng, dout, ng / 4 * es)) return MTA_ERR_INVALID;
    if (overlaps(dq, ng, dk, ng) || overlaps(dq, ng, dv, ng) || overlaps(dk, ng, dv, ng)) return MTA_ERR_INVALID;
  }
  if ((dtheta && !aligned(dtheta, 4)) || (dw && !aligned(dw, 4))) return MTA_ERR_INVALID;
  if ((s = check_workspace(cfg, kStatusBytes)) != MTA_OK) return s;
  BwdArgs a = make_bwd_args(q, k, v, theta_kq, w_head, dout, cfg, dq, dk, dv, dtheta, dw);
  bool tc = false;
  if ((s = select_bwd(a, cfg, cfg->path, cfg->workspace_bytes - kStatusBytes, &tc)) != MTA_OK) return s;
  if ((s = clear_status(cfg)) != MTA_OK) return s;
  Marks m = make_marks(cfg);
  if (m.next() != cudaSuccess) return MTA_ERR_CUDA;
  const cudaError_t e = tc ? launch_attn_bwd_tc(a, static_cast<char *>(cfg->workspace) + kStatusBytes)
                           : (a.kqp ? launch_attn_bwd_post(a) : launch_attn_bwd_simt(a));
  if (e != cudaSuccess) return MTA_ERR_CUDA;
  return m.next() == cudaSuccess ? MTA_OK : MTA_ERR_CUDA;
}

size_t mta_layer_bwd_workspace_bytes(const mta_cfg *cfg) {
  const size_t fixed = layer_bwd_fixed_bytes(cfg);
  // the forward recompute's contraction operands and the backward's strips are
  // live at different times and share the space after the fixed part
  return fixed ? fixed + std::max(kq_bytes(cfg), bwd_tc_bytes(cfg)) : 0;
}

mta_status mta_layer_bwd(const void *x, const void *Wqkv, const float *theta, const float *w_head,
                         const mta_gn *gn, const void *Wo, const void *dout, const mta_cfg *cfg, float *dx,
                         float *dWqkv, float *dWo, float *dtheta, float *dw, float *dgamma, float *dbeta,
                         float *dgate) {
  mta_status s = check_cfg(cfg);
  if (s != MTA_OK) return s;
  if (cfg->dtype != MTA_BF16) return MTA_ERR_UNSUPPORTED;
  if (!x || !Wqkv || !Wo || !dout || !gn || !gn->gamma || !gn->beta) return MTA_ERR_INVALID;
  if (!dx || !dWqkv || !dWo || !dgamma || !dbeta || (gn->gate && !dgate)) return MTA_ERR_INVALID;
  if ((cfg->kq_place != MTA_OFF || cfg->kq_post) && !theta) return MTA_ERR_INVALID;
  if (cfg->head_place != MTA_OFF && !w_head) return MTA_ERR_INVALID;
  if (!aligned(x, 16) || !aligned(Wqkv, 16) || !aligned(Wo, 16) || !aligned(dout, 16)) return MTA_ERR_INVALID;
  if (!aligned(dx, 16) || !aligned(dWqkv, 16) || !aligned(dWo, 16) || !aligned(dgamma, 4) ||
      !aligned(dbeta, 4) || (dgate && !aligned(dgate, 4)) || (dtheta && !aligned(dtheta, 4)) ||
      (dw && !aligned(dw, 4)) || (theta && !aligned(theta, 4)) || !aligned(gn->gamma, 4) || !aligned(gn->beta, 4))
    return MTA_ERR_INVALID;
  const size_t T = layer_tokens(cfg), D = static_cast<size_t>(cfg->H) * cfg->d;
  if (T > static_cast<size_t>(65535) * 64 || 3 * D > static_cast<size_t>(1) << 30) return MTA_ERR_UNSUPPORTED;
  if (cfg->d != 32 && cfg->d != 64 && cfg->d != 96 && cfg->d != 128) return MTA_ERR_UNSUPPORTED;
  {
    // no output may share memory with an input or with another output
    const void *in[4] = {x, Wqkv, Wo, dout};
    const size_t nin[4] = {T * D * 2, 3 * D * D * 2, D * D * 2, T * D * 2};
    const void *outp[3] = {dx, dWqkv, dWo};
    const size_t nout[3] = {T * D * 4, 3 * D * D * 4, D * D * 4};
    for (int i = 0; i < 3; ++i) {
      for (int j = 0; j < 4; ++j)
        if (overlaps(outp[i], nout[i], in[j], nin[j])) return MTA_ERR_INVALID;
      for (int j = 0; j < i; ++j)
        if (overlaps(outp[i], nout[i], outp[j], nout[j])) return MTA_ERR_INVALID;
    }
  }
  if ((s = check_workspace(cfg, layer_bwd_fixed_bytes(cfg))) != MTA_OK) return s;

  char *ws = static_cast<char *>(cfg->workspace);
  char *qkv = ws + kStatusBytes;
  char *obuf = qkv + align_up(T * 3 * D * 2);
  char *ybuf = obuf + align_up(T * D * 2);
  char *dybuf = ybuf + align_up(T * D * 2);
  char *dobuf = dybuf + align_up(T * D * 4);
  float *dq = reinterpret_cast<float *>(dobuf + align_up(T * D * 2));
  float *dk = reinterpret_cast<float *>(reinterpret_cast<char *>(dq) + align_up(T * D * 4));
  float *dv = reinterpret_cast<float *>(reinterpret_cast<char *>(dk) + align_up(T * D * 4));
  char *dqkv = reinterpret_cast<char *>(dv) + align_up(T * D * 4);
  char *kq_ws = dqkv + align_up(T * 3 * D * 2);
  const size_t kq_room = cfg->workspace_bytes - (kq_ws - ws);
  const uint16_t *qkvb = reinterpret_cast<const uint16_t *>(qkv);

  // the forward's attention (recomputed) and the attention backward, both on QKV
  mta_cfg acfg = *cfg;
  acfg.qkv_row_stride = static_cast<long long>(3 * D);
  AttnArgs a = make_args(qkvb, qkvb + D, qkvb + 2 * D, theta, w_head, &acfg, obuf);
  Kernel kern = K_SIMT;
  if ((s = select_kernel(a, cfg->path, kq_room, &kern)) != MTA_OK) return s;
  mta_cfg bcfg = acfg;
  bcfg.path = 0;
  BwdArgs ba = make_bwd_args(qkvb, qkvb + D, qkvb + 2 * D, theta, w_head, dobuf, &bcfg, dq, dk, dv, dtheta, dw);
  bool bwd_tc = false;
  if ((s = select_bwd(ba, &bcfg, 0, kq_room, &bwd_tc)) != MTA_OK) return s;

  const GnArgs g = make_gn(gn);
  cudaStream_t st = static_cast<cudaStream_t>(cfg->stream);
  unsigned *err = static_cast<unsigned *>(cfg->workspace);
  if ((s = clear_status(cfg)) != MTA_OK) return s;
  if (cudaMemsetAsync(dgamma, 0, D * 4, st) != cudaSuccess || cudaMemsetAsync(dbeta, 0, D * 4, st) != cudaSuccess ||
      (gn->gate && cudaMemsetAsync(dgate, 0, cfg->H * 4, st) != cudaSuccess))
    return MTA_ERR_CUDA;
  Marks m = make_marks(cfg);
  a.marks = &m;
  const int iT = static_cast<int>(T), iD = static_cast<int>(D), i3D = static_cast<int>(3 * D);
  if (m.next() != cudaSuccess) return MTA_ERR_CUDA;
  // forward: QKV = x Wqkv^T, O = attention(QKV)
  if (launch_gemm(x, Wqkv, qkv, iT, i3D, iD, false, false, false, err, st) != cudaSuccess || m.next() != cudaSuccess)
    return MTA_ERR_CUDA;
  if (launch_kernel(kern, a, nullptr, kq_ws) != cudaSuccess) return MTA_ERR_CUDA;
  // dY = dOut Wo (Wo read as the MN-major operand)
  if (launch_gemm(dout, Wo, dybuf, iT, iD, iD, false, true, true, err, st) != cudaSuccess || m.next() != cudaSuccess)
    return MTA_ERR_CUDA;
  // group norm: Y, dO, dgamma, dbeta, dgate
  if (launch_group_norm_bwd(obuf, reinterpret_cast<const float *>(dybuf), g, iT, cfg->H, cfg->d, ybuf, dobuf, dgamma,
                            dbeta, dgate, st) != cudaSuccess ||
      m.next() != cudaSuccess)
    return MTA_ERR_CUDA;
  // dWo = dOut^T Y (both operands MN-major, K = tokens)
  if (launch_gemm(dout, ybuf, dWo, iD, iD, iT, true, true, true, err, st) != cudaSuccess || m.next() != cudaSuccess)
    return MTA_ERR_CUDA;
  // attention core: dq, dk, dv (fp32), dtheta, dw
  if ((bwd_tc ? launch_attn_bwd_tc(ba, kq_ws) : ba.kqp ? launch_attn_bwd_post(ba) : launch_attn_bwd_simt(ba)) !=
          cudaSuccess ||
      m.next() != cudaSuccess)
    return MTA_ERR_CUDA;
  if (launch_pack_qkv_grad(dq, dk, dv, static_cast<long long>(T), iD, dqkv, st) != cudaSuccess ||
      m.next() != cudaSuccess)
    return MTA_ERR_CUDA;
  // dx = dQKV Wqkv, dWqkv = dQKV^T x
  if (launch_gemm(dqkv, Wqkv, dx, iT, iD, i3D, false, true, true, err, st) != cudaSuccess || m.next() != cudaSuccess)
    return MTA_ERR_CUDA;
  if (launch_gemm(dqkv, x, dWqkv, i3D, iD, iT, true, true, true, err, st) != cudaSuccess || m.next() != cudaSuccess)
    return MTA_ERR_CUDA;
  return MTA_OK;
}

mta_status mta_gemm_bf16_nt(const void *A, const void *Bm, void *C, int M, int N, int K, void *stream) {
  if (!A || !Bm || !C || M < 1 || N < 1 || K < 1) return MTA_ERR_INVALID;
  if (K % 8 != 0 || !aligned(A, 16) || !aligned(Bm, 16) || !aligned(C, 16)) return MTA_ERR_INVALID;
  if (M > 65535 * 128) return MTA_ERR_UNSUPPORTED;
  return launch_gemm_bf16_nt(A, Bm, C, M, N, K, nullptr, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MTA_OK
             : MTA_ERR_CUDA;
}

mta_status mta_group_norm_scale(const void *o, const mta_gn *gn, int tokens, int H, int d, void *y,
                                void *stream) {
  if (!o || !gn || !gn->gamma || !gn->beta || !y || tokens < 0 || H < 1 || d < 1 || d > 128)
    return MTA_ERR_INVALID;
  if (!aligned(o, 2) || !aligned(y, 2) || !aligned(gn->gamma, 4) || !aligned(gn->beta, 4))
    return MTA_ERR_INVALID;
  return launch_group_norm(o, make_gn(gn), tokens, H, d, y, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MTA_OK
             : MTA_ERR_CUDA;
}

mta_status mta_gemm_bf16(const void *A, const void *Bm, void *C, int M, int N, int K, int a_mn, int b_mn,
                         int f32_out, void *stream) {
  if (!A || !Bm || !C || M < 1 || N < 1 || K < 1) return MTA_ERR_INVALID;
  if ((a_mn != 0 && a_mn != 1) || (b_mn != 0 && b_mn != 1) || (f32_out != 0 && f32_out != 1))
    return MTA_ERR_INVALID;
  if ((a_mn ? M : K) % 8 != 0 || (b_mn ? N : K) % 8 != 0) return MTA_ERR_INVALID;
  if (!aligned(A, 16) || !aligned(Bm, 16) || !aligned(C, 16)) return MTA_ERR_INVALID;
  const size_t es = f32_out ? 4 : 2;
  if (overlaps(C, static_cast<size_t>(M) * N * es, A, static_cast<size_t>(M) * K * 2) ||
      overlaps(C, static_cast<size_t>(M) * N * es, Bm, static_cast<size_t>(N) * K * 2))
    return MTA_ERR_INVALID;
  return launch_gemm(A, Bm, C, M, N, K, a_mn != 0, b_mn != 0, f32_out != 0, nullptr,
                     static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MTA_OK
             : MTA_ERR_CUDA;
}

mta_status mta_group_norm_scale_bwd(const void *o, const float *dy, const mta_gn *gn, int tokens, int H, int d,
                                    void *y, void *dout, float *dgamma, float *dbeta, float *dgate,
                                    void *stream) {
  if (!o || !dy || !gn || !gn->gamma || !gn->beta || !y || !dout || !dgamma || !dbeta || tokens < 0 || H < 1)
    return MTA_ERR_INVALID;
  if (gn->gate && !dgate) return MTA_ERR_INVALID;
  if (d != 32 && d != 64 && d != 96 && d != 128) return MTA_ERR_UNSUPPORTED;
  if (tokens > 65535 * 64) return MTA_ERR_UNSUPPORTED;
  if (!aligned(o, 2) || !aligned(y, 2) || !aligned(dout, 2) || !aligned(dy, 4) || !aligned(dgamma, 4) ||
      !aligned(dbeta, 4) || (dgate && !aligned(dgate, 4)) || !aligned(gn->gamma, 4) || !aligned(gn->beta, 4))
    return MTA_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t hd = static_cast<size_t>(H) * d;
  if (cudaMemsetAsync(dgamma, 0, hd * 4, st) != cudaSuccess || cudaMemsetAsync(dbeta, 0, hd * 4, st) != cudaSuccess ||
      (gn->gate && cudaMemsetAsync(dgate, 0, static_cast<size_t>(H) * 4, st) != cudaSuccess))
    return MTA_ERR_CUDA;
  return launch_group_norm_bwd(o, dy, make_gn(gn), tokens, H, d, y, dout, dgamma, dbeta, dgate, st) == cudaSuccess
             ? MTA_OK
             : MTA_ERR_CUDA;
}

mta_status mta_selftest_wait_timeout(const mta_cfg *cfg, unsigned limit_us) {
  if (!cfg) return MTA_ERR_INVALID;
  if (limit_us < 1 || limit_us > 2000000) return MTA_ERR_INVALID;
  mta_status s = check_workspace(cfg, kStatusBytes);
  if (s != MTA_OK) return s;
  if ((s = clear_status(cfg)) != MTA_OK) return s;  // also zeroes the counters
  // counters of the waits that gave up, after the error word
  unsigned *word = static_cast<unsigned *>(cfg->workspace);
  cudaStream_t st = static_cast<cudaStream_t>(cfg->stream);
  return launch_wait_timeout_selftest(1000ull * limit_us, word, word + 1, st) == cudaSuccess ? MTA_OK
                                                                                              : MTA_ERR_CUDA;
}

mta_status mta_sync_status(const mta_cfg *cfg) {
  if (!cfg || !cfg->workspace) return MTA_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(cfg->stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MTA_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpy(&word, cfg->workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MTA_ERR_CUDA;
  return (word & ERRBIT_TIMEOUT) ? MTA_ERR_TIMEOUT : MTA_OK;
}

}  // extern "C"
