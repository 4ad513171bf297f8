// attn_simt.cu -- MTA attention on CUDA cores, fp32 arithmetic, any supported
// configuration (the fp32 path, and the path for shapes the tensor-core kernel
// does not take).
//
// Steps per "Multi-Token Attention | Summary" (greeksharifa): logits Q K^T/sqrt(d)
// (section 2), Mask_0, key-query convolution over (previous queries, neighbouring
// keys) (section 3.1), pre-softmax head mix (section 3.2), Mask_-inf and softmax
// (section 2), post-softmax head mix (section 3.2), A V (section 2).
//
// One CTA owns one (batch, head group, tile of BR queries).  Two sweeps over the
// key tiles: the first gathers the exact row maxima and sums of the softmax, the
// second recomputes the logits, normalises, mixes and multiplies by V.  The
// L x L maps only ever exist as BR x BC tiles in shared memory.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"

namespace mta {
namespace {

constexpr int kThreads = 256;
constexpr int kBC = 32;          // keys per tile
constexpr int kSmemCap = 200 * 1024;

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Offsets (in floats) of the shared-memory arrays.
struct SimtLayout {
  int Qs, Ks, Sh, Ct, Pm, m, l, acc, th, wg, total;
};

__host__ __device__ inline SimtLayout simt_layout(int BR, int BC, int d, int cq, int ck, int ch) {
  const int c = ck / 2, HR = BR + cq - 1, HC = BC + 2 * c, dp = d + 1;
  SimtLayout s;
  int o = 0;
  s.Qs = o;  o += HR * dp;        // query rows i0-(cq-1) .. i0+BR-1 of one head
  s.Ks = o;  o += HC * dp;        // key rows j0-c .. j0+BC+c-1 of one head
  s.Sh = o;  o += HR * HC;        // Mask_0(A_hat) on the halo tile
  s.Ct = o;  o += ch * BR * BC;   // convolved (then mixed) logits / probabilities
  s.Pm = o;  o += ch * BR * BC;   // mixing scratch
  s.m = o;   o += ch * BR;        // row max
  s.l = o;   o += ch * BR;        // row sum
  s.acc = o; o += ch * BR * d;    // output accumulators
  s.th = o;  o += ch * cq * ck;   // key-query kernels of the group
  s.wg = o;  o += ch * ch;        // head-mixing weights of the group
  s.total = o;
  return s;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) attn_simt_kernel(AttnArgs a, int BR) {
  extern __shared__ float sm[];
  const int BC = kBC;
  const int d = a.d, cq = a.cq, ck = a.ck, ch = a.ch, c = ck / 2, L = a.L, H = a.H;
  const int HR = BR + cq - 1, HC = BC + 2 * c, dp = d + 1;
  const SimtLayout S = simt_layout(BR, BC, d, cq, ck, ch);
  float *Qs = sm + S.Qs, *Ks = sm + S.Ks, *Sh = sm + S.Sh, *Ct = sm + S.Ct, *Pm = sm + S.Pm;
  float *rm = sm + S.m, *rl = sm + S.l, *acc = sm + S.acc, *th = sm + S.th, *wg = sm + S.wg;
  const int i0 = blockIdx.x * BR, g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const T *q = static_cast<const T *>(a.q);
  const T *k = static_cast<const T *>(a.k);
  const T *v = static_cast<const T *>(a.v);
  T *out = static_cast<T *>(a.out);
  const float NEG_INF = -INFINITY;
  const bool kq = (a.kq != 0);
  const bool exact = (a.kq == 3);  // exact causal indicator instead of Mask_0

  for (int i = tid; i < ch * cq * ck; i += kThreads) th[i] = kq ? a.theta[g * ch * cq * ck + i] : 0.f;
  for (int i = tid; i < ch * ch; i += kThreads)
    wg[i] = (a.hp != 0) ? a.w[g * ch * ch + i] : (i / ch == i % ch ? 1.f : 0.f);
  for (int i = tid; i < ch * BR; i += kThreads) { rm[i] = NEG_INF; rl[i] = 0.f; }
  for (int i = tid; i < ch * BR * d; i += kThreads) acc[i] = 0.f;
  __syncthreads();

  const int q_end = min(L, i0 + BR);  // queries of this tile are i0 .. q_end-1
  const int tile = BR * BC;
  for (int pass = 0; pass < 2; ++pass) {
    for (int j0 = 0; j0 < q_end; j0 += BC) {
      for (int hl = 0; hl < ch; ++hl) {
        const int h = g * ch + hl;
        for (int i = tid; i < HR * d; i += kThreads) {
          const int r = i / d, e = i % d, iq = i0 - (cq - 1) + r;
          Qs[r * dp + e] = (iq >= 0 && iq < L) ? to_f(q[((long long)b * L + iq) * a.rs + h * d + e]) : 0.f;
        }
        for (int i = tid; i < HC * d; i += kThreads) {
          const int s = i / d, e = i % d, jk = j0 - c + s;
          Ks[s * dp + e] = (jk >= 0 && jk < L) ? to_f(k[((long long)b * L + jk) * a.rs + h * d + e]) : 0.f;
        }
        __syncthreads();
        // Mask_0(A_hat) on the halo tile: future keys of each (shifted) query are 0
        // (with the exact indicator the logits stay unmasked here; see below)
        for (int i = tid; i < HR * HC; i += kThreads) {
          const int r = i / HC, s = i % HC, iq = i0 - (cq - 1) + r, jk = j0 - c + s;
          float val = 0.f;
          if (iq >= 0 && iq < L && jk >= 0 && jk < L && (!kq || exact || jk <= iq)) {
            const float *qr = Qs + r * dp, *kr = Ks + s * dp;
            for (int e = 0; e < d; ++e) val = fmaf(qr[e], kr[e], val);
            val *= a.scale;
          }
          Sh[i] = val;
        }
        __syncthreads();
        // key-query convolution: C[i][j] = sum_a sum_t theta[a][t] M0[i-a][j-(t-c)];
        // with the exact indicator a tap counts when its key j-(t-c) <= i
        for (int i = tid; i < tile; i += kThreads) {
          const int r = i / BC, j = i % BC;
          float val;
          if (kq) {
            val = 0.f;
            const float *tk = th + hl * cq * ck;
            const int t0 = exact ? max(0, (j0 + j) + c - (i0 + r)) : 0;
            for (int aa = 0; aa < cq; ++aa) {
              const float *srow = Sh + (r + cq - 1 - aa) * HC + j + 2 * c;
              for (int t = t0; t < ck; ++t) val = fmaf(tk[aa * ck + t], srow[-t], val);
            }
          } else {
            val = Sh[(r + cq - 1) * HC + j + c];
          }
          Ct[hl * tile + i] = val;
        }
        __syncthreads();
      }
      if (a.hp == 1) {  // pre-softmax head mix
        for (int i = tid; i < ch * tile; i += kThreads) {
          const int hl = i / tile, rem = i % tile;
          float val = 0.f;
          for (int s = 0; s < ch; ++s) val = fmaf(wg[hl * ch + s], Ct[s * tile + rem], val);
          Pm[i] = val;
        }
        __syncthreads();
        for (int i = tid; i < ch * tile; i += kThreads) Ct[i] = Pm[i];
        __syncthreads();
      }
      // Mask_-inf: keys after the query (and past the sequence) get -inf
      for (int i = tid; i < ch * tile; i += kThreads) {
        const int rem = i % tile, r = rem / BC, j = rem % BC;
        if (j0 + j > i0 + r || j0 + j >= L) Ct[i] = NEG_INF;
      }
      __syncthreads();
      if (pass == 0) {
        for (int i = tid; i < ch * BR; i += kThreads) {
          const float *row = Ct + i * BC;
          float mx = NEG_INF;
          for (int j = 0; j < BC; ++j) mx = fmaxf(mx, row[j]);
          const float mn = fmaxf(rm[i], mx);
          if (mn == NEG_INF) continue;
          float s = rl[i] * expf(rm[i] - mn);
          for (int j = 0; j < BC; ++j) s += expf(row[j] - mn);
          rm[i] = mn;
          rl[i] = s;
        }
        __syncthreads();
      } else {
        for (int i = tid; i < ch * tile; i += kThreads) {
          const int hr = i / BC;
          Pm[i] = expf(Ct[i] - rm[hr]) / rl[hr];
        }
        __syncthreads();
        for (int i = tid; i < ch * tile; i += kThreads) {  // post-softmax head mix
          const int hl = i / tile, rem = i % tile;
          float val;
          if (a.hp == 2) {
            val = 0.f;
            for (int s = 0; s < ch; ++s) val = fmaf(wg[hl * ch + s], Pm[s * tile + rem], val);
          } else {
            val = Pm[i];
          }
          Ct[i] = val;
        }
        __syncthreads();
        for (int i = tid; i < ch * BR * d; i += kThreads) {  // acc += A V (head's own V)
          const int hl = i / (BR * d), rem = i % (BR * d), r = rem / d, e = rem % d;
          const int h = g * ch + hl;
          const float *prow = Ct + (hl * BR + r) * BC;
          float s = acc[i];
          const int jn = min(BC, L - j0);
          for (int j = 0; j < jn; ++j)
            s = fmaf(prow[j], to_f(v[((long long)b * L + j0 + j) * a.rs + h * d + e]), s);
          acc[i] = s;
        }
        __syncthreads();
      }
    }
  }
  for (int i = tid; i < ch * BR * d; i += kThreads) {
    const int hl = i / (BR * d), rem = i % (BR * d), r = rem / d, e = rem % d;
    const int iq = i0 + r;
    if (iq < L) out[(((long long)b * L + iq) * H + g * ch + hl) * d + e] = from_f<T>(acc[i]);
  }
}

}  // namespace

size_t attn_simt_smem_bytes(const AttnArgs &a, int BR, int BC) {
  return static_cast<size_t>(simt_layout(BR, BC, a.d, a.cq, a.ck, a.ch).total) * sizeof(float);
}

int attn_simt_pick_rows(const AttnArgs &a, int BC) {
  for (int BR = 16; BR >= 1; BR /= 2)
    if (attn_simt_smem_bytes(a, BR, BC) <= static_cast<size_t>(kSmemCap)) return BR;
  return 0;
}

cudaError_t launch_attn_simt(const AttnArgs &a) {
  const int BR = attn_simt_pick_rows(a, kBC);
  if (BR == 0) return cudaErrorInvalidConfiguration;
  const size_t smem = attn_simt_smem_bytes(a, BR, kBC);
  dim3 grid((a.L + BR - 1) / BR, a.H / a.ch, a.B);
  cudaError_t e;
  if (a.dtype == 0) {
    e = cudaFuncSetAttribute(attn_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attn_simt_kernel<float><<<grid, kThreads, smem, a.stream>>>(a, BR);
  } else {
    e = cudaFuncSetAttribute(attn_simt_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attn_simt_kernel<__nv_bfloat16><<<grid, kThreads, smem, a.stream>>>(a, BR);
  }
  return cudaGetLastError();
}

}  // namespace mta
