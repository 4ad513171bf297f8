// attn_simt.cu -- MTA attention on CUDA cores, fp32 arithmetic, any supported
// configuration (the fp32 path, and the path for shapes the tensor-core kernel
// does not take).
//
// Steps per "Multi-Token Attention | Summary" (greeksharifa): logits Q K^T/sqrt(d)
// (section 2), Mask_0, key-query convolution over (previous queries, neighbouring
// keys) (section 3.1), pre-softmax head mix (section 3.2), Mask_-inf and softmax
// (section 2), the key-query convolution of the softmax weights followed by
// Mask_0 (section 3.1, after the softmax), post-softmax head mix (section 3.2),
// A V (section 2).
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
  int Qs, Ks, Sh, Ct, Pm, m, l, acc, th, thp, wg, total;
};

// With the post-softmax convolution the tile's weights are needed on a wider
// region: pr = c_q-1 more query rows above and pc = c_k/2 more keys on each side.
__host__ __device__ inline SimtLayout simt_layout(int BR, int BC, int d, int cq, int ck, int ch,
                                                  int kqp) {
  const int c = ck / 2, pr = kqp ? cq - 1 : 0, pc = kqp ? c : 0;
  const int CR = BR + pr, CC = BC + 2 * pc;           // region of C and A
  const int HR = CR + cq - 1, HC = CC + 2 * c, dp = d + 1;
  SimtLayout s;
  int o = 0;
  s.Qs = o;  o += HR * dp;        // query rows i0-pr-(cq-1) .. i0+BR-1 of one head
  s.Ks = o;  o += HC * dp;        // key rows j0-pc-c .. j0+BC+pc+c-1 of one head
  s.Sh = o;  o += HR * HC;        // Mask_0(A_hat) on the halo tile
  s.Ct = o;  o += ch * CR * CC;   // convolved (then mixed) logits / probabilities
  s.Pm = o;  o += ch * CR * CC;   // softmax weights / mixing scratch
  s.m = o;   o += ch * CR;        // row max
  s.l = o;   o += ch * CR;        // row sum
  s.acc = o; o += ch * BR * d;    // output accumulators
  s.th = o;  o += ch * cq * ck;   // pre-softmax key-query kernels of the group
  s.thp = o; o += ch * cq * ck;   // post-softmax key-query kernels of the group
  s.wg = o;  o += ch * ch;        // head-mixing weights of the group
  s.total = o;
  return s;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) attn_simt_kernel(AttnArgs a, int BR) {
  extern __shared__ float sm[];
  const int BC = kBC;
  const int d = a.d, cq = a.cq, ck = a.ck, ch = a.ch, c = ck / 2, L = a.L, H = a.H;
  const int kqp = a.kqp, pr = kqp ? cq - 1 : 0, pc = kqp ? c : 0;
  const int CR = BR + pr, CC = BC + 2 * pc;
  const int HR = CR + cq - 1, HC = CC + 2 * c, dp = d + 1;
  const SimtLayout S = simt_layout(BR, BC, d, cq, ck, ch, kqp);
  float *Qs = sm + S.Qs, *Ks = sm + S.Ks, *Sh = sm + S.Sh, *Ct = sm + S.Ct, *Pm = sm + S.Pm;
  float *rm = sm + S.m, *rl = sm + S.l, *acc = sm + S.acc, *th = sm + S.th, *thp = sm + S.thp;
  float *wg = sm + S.wg;
  const int i0 = blockIdx.x * BR, g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const T *q = static_cast<const T *>(a.q);
  const T *k = static_cast<const T *>(a.k);
  const T *v = static_cast<const T *>(a.v);
  T *out = static_cast<T *>(a.out);
  const float NEG_INF = -INFINITY;
  const bool kq = (a.kq != 0);
  const bool exact = (a.kq == 3);  // exact causal indicator instead of Mask_0

  for (int i = tid; i < ch * cq * ck; i += kThreads) {
    th[i] = kq ? a.theta[g * ch * cq * ck + i] : 0.f;
    thp[i] = kqp ? a.theta_post[g * ch * cq * ck + i] : 0.f;
  }
  for (int i = tid; i < ch * ch; i += kThreads)
    wg[i] = (a.hp != 0) ? a.w[g * ch * ch + i] : (i / ch == i % ch ? 1.f : 0.f);
  for (int i = tid; i < ch * CR; i += kThreads) { rm[i] = NEG_INF; rl[i] = 0.f; }
  for (int i = tid; i < ch * BR * d; i += kThreads) acc[i] = 0.f;
  __syncthreads();

  const int q_end = min(L, i0 + BR);  // queries of this tile are i0 .. q_end-1
  const int region = CR * CC, tile = BR * BC;
  const int rq0 = i0 - pr, rk0_ofs = -pc;  // region row r is query rq0 + r, column s key j0 - pc + s
  for (int pass = 0; pass < 2; ++pass) {
    for (int j0 = 0; j0 < q_end; j0 += BC) {
      const int rk0 = j0 + rk0_ofs;
      for (int hl = 0; hl < ch; ++hl) {
        const int h = g * ch + hl;
        for (int i = tid; i < HR * d; i += kThreads) {
          const int r = i / d, e = i % d, iq = rq0 - (cq - 1) + r;
          Qs[r * dp + e] = (iq >= 0 && iq < L) ? to_f(q[((long long)b * L + iq) * a.rs + h * d + e]) : 0.f;
        }
        for (int i = tid; i < HC * d; i += kThreads) {
          const int s = i / d, e = i % d, jk = rk0 - c + s;
          Ks[s * dp + e] = (jk >= 0 && jk < L) ? to_f(k[((long long)b * L + jk) * a.rs + h * d + e]) : 0.f;
        }
        __syncthreads();
        // Mask_0(A_hat) on the halo tile: future keys of each (shifted) query are 0
        // (with the exact indicator the logits stay unmasked here; see below)
        for (int i = tid; i < HR * HC; i += kThreads) {
          const int r = i / HC, s = i % HC, iq = rq0 - (cq - 1) + r, jk = rk0 - c + s;
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
        for (int i = tid; i < region; i += kThreads) {
          const int r = i / CC, s = i % CC;
          float val;
          if (kq) {
            val = 0.f;
            const float *tk = th + hl * cq * ck;
            const int t0 = exact ? max(0, (rk0 + s) + c - (rq0 + r)) : 0;
            for (int aa = 0; aa < cq; ++aa) {
              const float *srow = Sh + (r + cq - 1 - aa) * HC + s + 2 * c;
              for (int t = t0; t < ck; ++t) val = fmaf(tk[aa * ck + t], srow[-t], val);
            }
          } else {
            val = Sh[(r + cq - 1) * HC + s + c];
          }
          Ct[hl * region + i] = val;
        }
        __syncthreads();
      }
      if (a.hp == 1) {  // pre-softmax head mix
        for (int i = tid; i < ch * region; i += kThreads) {
          const int hl = i / region, rem = i % region;
          float val = 0.f;
          for (int s = 0; s < ch; ++s) val = fmaf(wg[hl * ch + s], Ct[s * region + rem], val);
          Pm[i] = val;
        }
        __syncthreads();
        for (int i = tid; i < ch * region; i += kThreads) Ct[i] = Pm[i];
        __syncthreads();
      }
      // Mask_-inf: keys after the query, outside the sequence, and rows before it get -inf
      for (int i = tid; i < ch * region; i += kThreads) {
        const int rem = i % region, iq = rq0 + rem / CC, jk = rk0 + rem % CC;
        if (jk > iq || jk >= L || jk < 0 || iq < 0) Ct[i] = NEG_INF;
      }
      __syncthreads();
      if (pass == 0) {  // statistics over this tile's own keys (columns pc .. pc+BC-1)
        for (int i = tid; i < ch * CR; i += kThreads) {
          const float *row = Ct + i * CC + pc;
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
        // softmax weights A on the region (0 at masked entries and empty rows)
        for (int i = tid; i < ch * region; i += kThreads) {
          const int hr = i / CC;
          Pm[i] = (Ct[i] == NEG_INF || rm[hr] == NEG_INF) ? 0.f : expf(Ct[i] - rm[hr]) / rl[hr];
        }
        __syncthreads();
        // post-softmax convolution, then Mask_0: A'[i][j] = [j <= i] sum theta_post[a][t] A[i-a][j-(t-c)]
        for (int i = tid; i < ch * tile; i += kThreads) {
          const int hl = i / tile, rem = i % tile, r = rem / BC, j = rem % BC;
          float val;
          if (kqp) {
            val = 0.f;
            if (j0 + j <= i0 + r) {
              const float *tk = thp + hl * cq * ck;
              for (int aa = 0; aa < cq; ++aa) {
                const float *prow = Pm + hl * region + (r + pr - aa) * CC + j + pc + c;
                for (int t = 0; t < ck; ++t) val = fmaf(tk[aa * ck + t], prow[-t], val);
              }
            }
          } else {
            val = Pm[hl * region + r * CC + j];
          }
          Ct[i] = val;
        }
        __syncthreads();
        for (int i = tid; i < ch * tile; i += kThreads) {  // post-softmax head mix
          const int hl = i / tile, rem = i % tile;
          float val;
          if (a.hp == 2) {
            val = 0.f;
            for (int s = 0; s < ch; ++s) val = fmaf(wg[hl * ch + s], Ct[s * tile + rem], val);
          } else {
            val = Ct[i];
          }
          Pm[i] = val;
        }
        __syncthreads();
        for (int i = tid; i < ch * BR * d; i += kThreads) {  // acc += A V (head's own V)
          const int hl = i / (BR * d), rem = i % (BR * d), r = rem / d, e = rem % d;
          const int h = g * ch + hl;
          const float *prow = Pm + (hl * BR + r) * BC;
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
  return static_cast<size_t>(simt_layout(BR, BC, a.d, a.cq, a.ck, a.ch, a.kqp).total) * sizeof(float);
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
