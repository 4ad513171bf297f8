// attn_bwd_simt.cu -- backward pass of MTA attention on CUDA cores, fp32 arithmetic.
//
// The forward of "Multi-Token Attention | Summary" (greeksharifa): logits
// A_hat = s Q K^T (section 2), C = Conv2d_theta(Mask_0(A_hat)) (section 3.1; or the
// exact causal indicator), pre-softmax head mix C' = sum_s w[h][s] C_s (section
// 3.2), A = Softmax(Mask_-inf(C')), post-softmax mix A'' = sum_s w[h][s] A_s, and
// O_h = A''_h V_h.  Its gradients, each step taken in reverse:
//   dV_h = A''_h^T dO_h;   dA''_h = dO_h V_h^T;   dA_s = sum_h w[h][s] dA''_h
//   dw[h][s] = sum_ij dA''_h A_s  (post) or sum_ij dC'_h C_s  (pre)
//   dC'_h = A_h * (dA_h - D_h),   D_h[i] = sum_j dA_h[i][j] A_h[i][j]
//   dC_s = sum_h w[h][s] dC'_h  (pre)
//   dtheta_s[a][t] = sum_ij dC_s[i][j] Mask_0(A_hat_s)[i-a][j-(t-c)]
//   dA_hat_s[i][j] = [j <= i] sum_a sum_t theta_s[a][t] dC_s[i+a][j+(t-c)]
//   dQ = s dA_hat K,  dK = s dA_hat^T Q.
//
// One CTA owns one (batch, head group, tile of BR queries).  It recomputes the
// forward maps on a region widened by c_q-1 rows below the tile and c_k/2 keys on
// each side (the adjoint of the convolution reads dC there), with a further halo
// for the convolution itself.  Two sweeps over the key tiles: the first gathers
// the exact row statistics of the softmax and the row sums D, the second forms
// the gradients.  dQ rows are owned by the CTA; dK, dV, dtheta and dw are summed
// over CTAs with atomic adds (the caller's buffers are zeroed first).  The L x L
// maps only ever exist as tiles in shared memory.
#include <cuda_bf16.h>
#include <math.h>

#include "bwd_common.cuh"
#include "internal.h"

namespace mta {
namespace {

constexpr int kThreads = 256;
constexpr int kBC = 32;
constexpr int kSmemCap = 200 * 1024;
constexpr int kTwoPerSm = 112 * 1024;  // two CTAs per SM (228 KB of shared memory)

template <typename T>
__device__ __forceinline__ float ld(const T *p);
template <>
__device__ __forceinline__ float ld<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

struct BwdLayout {
  int Qs, Ks, DO, Sh, Cp, P, Gd, Dc, Tmp, A3, m, l, Ds, dqa, th, wg, dth, dwa, total;
};

__host__ __device__ inline BwdLayout bwd_layout(int BR, int BC, int d, int cq, int ck, int ch, bool kq) {
  const int c = ck / 2, PR = kq ? cq - 1 : 0, PC = kq ? c : 0;
  const int CR = BR + PR, CC = BC + 2 * PC, HR = CR + cq - 1, HC = CC + 2 * c, dp = d + 1;
  BwdLayout s;
  int o = 0;
  s.Qs = o;  o += HR * dp;            // query rows i0-(cq-1) .. i0+CR-1 of one head
  s.Ks = o;  o += HC * dp;            // key rows j0-PC-c .. (then value rows j0-PC ..)
  s.DO = o;  o += ch * CR * dp;       // output-gradient rows i0 .. i0+CR-1, every head
  s.Sh = o;  o += ch * HR * HC;       // Mask_0(A_hat) (unmasked with the exact indicator), every head
  s.Cp = o;  o += ch * CR * CC;       // convolved logits C_s on the region
  s.P = o;   o += ch * CR * CC;       // mixed logits, then softmax weights A
  s.Gd = o;  o += ch * CR * CC;       // dO_h . v_h
  s.Dc = o;  o += ch * CR * CC;       // dA, then dC' and dC
  s.Tmp = o; o += BR * BC;            // dA_hat of the tile, one head
  s.A3 = o;  o += ch * BR * BC;       // post-softmax-mixed weights A'' of the tile
  s.m = o;   o += ch * CR;
  s.l = o;   o += ch * CR;
  s.Ds = o;  o += ch * CR;            // D (row sums), accumulated then normalised
  s.dqa = o; o += ch * BR * d;        // dQ accumulators
  s.th = o;  o += ch * cq * ck;
  s.wg = o;  o += ch * ch;
  s.dth = o; o += ch * cq * ck;       // dtheta partial sums of the CTA
  s.dwa = o; o += ch * ch;            // dw partial sums of the CTA
  s.total = o;
  return s;
}

// The shape parameters DT, CQT, CKT, CHT, BRT are compile-time constants when
// nonzero (the index arithmetic of every loop then folds), else read at run time.
template <typename T, int DT, int CQT, int CKT, int CHT, int BRT>
__global__ void __launch_bounds__(kThreads) attn_bwd_simt_kernel(BwdArgs a, int BR_) {
  const int BR = BRT ? BRT : BR_;
  extern __shared__ float sm[];
  const int BC = kBC;
  const int d = DT ? DT : a.d, cq = CQT ? CQT : a.cq, ck = CKT ? CKT : a.ck, ch = CHT ? CHT : a.ch, c = ck / 2, L = a.L, H = a.H;
  const bool kq = a.kq != 0, exact = a.kq == 3;
  const int PR = kq ? cq - 1 : 0, PC = kq ? c : 0;
  const int CR = BR + PR, CC = BC + 2 * PC, HR = CR + cq - 1, HC = CC + 2 * c, dp = d + 1;
  const int region = CR * CC;
  const BwdLayout S = bwd_layout(BR, BC, d, cq, ck, ch, kq);
  float *Qs = sm + S.Qs, *Ks = sm + S.Ks, *DO = sm + S.DO, *Sh = sm + S.Sh, *Cp = sm + S.Cp;
  float *P = sm + S.P, *Gd = sm + S.Gd, *Dc = sm + S.Dc, *Tmp = sm + S.Tmp, *A3 = sm + S.A3;
  float *rm = sm + S.m, *rl = sm + S.l, *Ds = sm + S.Ds, *dqa = sm + S.dqa;
  float *th = sm + S.th, *wg = sm + S.wg, *dth = sm + S.dth, *dwa = sm + S.dwa;
  const int i0 = blockIdx.x * BR, g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const T *q = static_cast<const T *>(a.q);
  const T *k = static_cast<const T *>(a.k);
  const T *v = static_cast<const T *>(a.v);
  const T *dout = static_cast<const T *>(a.dout);
  const float NEG_INF = -INFINITY;
  auto gidx = [&](int tok, int h) { return (static_cast<long long>(b) * L + tok) * a.rs + static_cast<long long>(h) * d; };
  auto oidx = [&](int tok, int h) { return ((static_cast<long long>(b) * L + tok) * H + h) * d; };

  for (int i = tid; i < ch * cq * ck; i += kThreads) {
    th[i] = kq ? a.theta[g * ch * cq * ck + i] : 0.f;
    dth[i] = 0.f;
  }
  for (int i = tid; i < ch * ch; i += kThreads) {
    wg[i] = (a.hp != 0) ? a.w[g * ch * ch + i] : (i / ch == i % ch ? 1.f : 0.f);
    dwa[i] = 0.f;
  }
  for (int i = tid; i < ch * CR; i += kThreads) { rm[i] = NEG_INF; rl[i] = 0.f; Ds[i] = 0.f; }
  for (int i = tid; i < ch * BR * d; i += kThreads) dqa[i] = 0.f;
  // output-gradient rows of the region, every head (fixed for the CTA)
  for (int i = tid; i < ch * CR * d; i += kThreads) {
    const int hl = i / (CR * d), rem = i % (CR * d), r = rem / d, e = rem % d, iq = i0 + r;
    DO[(hl * CR + r) * dp + e] = iq < L ? ld(dout + oidx(iq, g * ch + hl) + e) : 0.f;
  }
  __syncthreads();

  const int r_end = min(L, i0 + CR);  // region rows are queries i0 .. r_end-1
  for (int pass = 0; pass < 2; ++pass) {
    for (int j0 = 0; j0 < r_end; j0 += BC) {
      // ---- forward maps of the region, every head: Sh, C_s, and G_h = dO_h . v_h
      for (int hl = 0; hl < ch; ++hl) {
        const int h = g * ch + hl;
        for (int i = tid; i < HR * d; i += kThreads) {
          const int r = i / d, e = i % d, iq = i0 - (cq - 1) + r;
          Qs[r * dp + e] = (iq >= 0 && iq < L) ? ld(q + gidx(iq, h) + e) : 0.f;
        }
        for (int i = tid; i < HC * d; i += kThreads) {
          const int s = i / d, e = i % d, jk = j0 - PC - c + s;
          Ks[s * dp + e] = (jk >= 0 && jk < L) ? ld(k + gidx(jk, h) + e) : 0.f;
        }
        __syncthreads();
        float *sh = Sh + hl * HR * HC;
        dot_rows4<kThreads>(Qs, Ks, HR, HC, d, dp, [&](int r, int s, float v) {
          const int iq = i0 - (cq - 1) + r, jk = j0 - PC - c + s;
          const bool ok = iq >= 0 && iq < L && jk >= 0 && jk < L && (!kq || exact || jk <= iq);
          sh[r * HC + s] = ok ? v * a.scale : 0.f;
        });
        __syncthreads();
        for (int i = tid; i < region; i += kThreads) {
          const int r = i / CC, s = i % CC;
          float val;
          if (kq) {
            val = 0.f;
            const float *tk = th + hl * cq * ck;
            const int t0 = exact ? max(0, (j0 - PC + s) + c - (i0 + r)) : 0;
            for (int aa = 0; aa < cq; ++aa) {
              const float *srow = sh + (r + cq - 1 - aa) * HC + s + 2 * c;
              for (int t = t0; t < ck; ++t) val = fmaf(tk[aa * ck + t], srow[-t], val);
            }
          } else {
            val = sh[(r + cq - 1) * HC + s + c];
          }
          Cp[hl * region + i] = val;
        }
        // value rows of the region's keys into Ks (the key rows are no longer needed)
        __syncthreads();
        for (int i = tid; i < CC * d; i += kThreads) {
          const int s = i / d, e = i % d, jk = j0 - PC + s;
          Ks[s * dp + e] = (jk >= 0 && jk < L) ? ld(v + gidx(jk, h) + e) : 0.f;
        }
        __syncthreads();
        dot_rows4<kThreads>(DO + hl * CR * dp, Ks, CR, CC, d, dp,
                            [&](int r, int s, float v) { Gd[hl * region + r * CC + s] = v; });
        __syncthreads();
      }
      // ---- mixed logits (pre-softmax mix), Mask_-inf; dA (post-softmax mix adjoint)
      for (int i = tid; i < ch * region; i += kThreads) {
        const int hl = i / region, rem = i % region, r = rem / CC, s = rem % CC;
        const int iq = i0 + r, jk = j0 - PC + s;
        float cv;
        if (a.hp == 1) {
          cv = 0.f;
          for (int s2 = 0; s2 < ch; ++s2) cv = fmaf(wg[hl * ch + s2], Cp[s2 * region + rem], cv);
        } else {
          cv = Cp[i];
        }
        P[i] = (iq < L && jk >= 0 && jk <= iq) ? cv : NEG_INF;
        float da;
        if (a.hp == 2) {  // dA_s = sum_h w[h][s] dO_h . v_h
          da = 0.f;
          for (int h2 = 0; h2 < ch; ++h2) da = fmaf(wg[h2 * ch + hl], Gd[h2 * region + rem], da);
        } else {
          da = Gd[i];
        }
        Dc[i] = da;
      }
      __syncthreads();
      if (pass == 0) {
        // exact statistics over this tile's own keys (columns PC .. PC+BC-1):
        // max, sum and D = sum_j exp(C' - max) dA, rescaled as the max grows
        for (int i = tid; i < ch * CR; i += kThreads) {
          const float *row = P + i * CC + PC, *dar = Dc + i * CC + PC;
          float mx = NEG_INF;
          for (int j = 0; j < BC; ++j) mx = fmaxf(mx, row[j]);
          const float mn = fmaxf(rm[i], mx);
          if (mn == NEG_INF) continue;
          const float sc = expf(rm[i] - mn);
          float s = rl[i] * sc, dsum = Ds[i] * sc;
          for (int j = 0; j < BC; ++j) {
            const float e = expf(row[j] - mn);
            s += e;
            dsum = fmaf(e, dar[j], dsum);
          }
          rm[i] = mn;
          rl[i] = s;
          Ds[i] = dsum;
        }
        __syncthreads();
        continue;
      }
      // ---- pass 2: softmax weights, dC' = A (dA - D)
      for (int i = tid; i < ch * region; i += kThreads) {
        const int hr = i / CC;  // (head, region row)
        const float pv = (P[i] == NEG_INF || rm[hr] == NEG_INF) ? 0.f : expf(P[i] - rm[hr]) / rl[hr];
        P[i] = pv;
        Dc[i] = pv * (Dc[i] - Ds[hr]);
      }
      __syncthreads();
      // dw over the tile's own (row, key) positions
      if (a.hp != 0) {
        for (int pr = 0; pr < ch * ch; ++pr) {
          const int hl = pr / ch, sl = pr % ch;
          // post: sum dO_h.v_h x A_s; pre: sum dC'_h x C_s
          const float *x = a.hp == 2 ? Gd + hl * region : Dc + hl * region;
          const float *y = a.hp == 2 ? P + sl * region : Cp + sl * region;
          float part = 0.f;
          for (int i = tid; i < BR * BC; i += kThreads) {
            const int r = i / BC, s = i % BC + PC, jk = j0 + i % BC;
            if (i0 + r < L && jk < L) part = fmaf(x[r * CC + s], y[r * CC + s], part);
          }
          for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
          if ((tid & 31) == 0) atomicAdd(dwa + pr, part);
        }
      }
      __syncthreads();
      // dC_s = sum_h w[h][s] dC'_h (pre-softmax mixing), into Gd
      const float *dcs = Dc;
      if (a.hp == 1) {
        for (int i = tid; i < ch * region; i += kThreads) {
          const int sl = i / region, rem = i % region;
          float val = 0.f;
          for (int h2 = 0; h2 < ch; ++h2) val = fmaf(wg[h2 * ch + sl], Dc[h2 * region + rem], val);
          Gd[i] = val;
        }
        __syncthreads();
        dcs = Gd;
      }
      // A'' = post-softmax mix of A on the tile (rows past L are 0), then
      // dV_h[j] += sum over the tile's rows of A''_h[i][j] dO_h[i]
      for (int i = tid; i < ch * BR * BC; i += kThreads) {
        const int hl = i / (BR * BC), rem = i % (BR * BC), r = rem / BC, s = rem % BC;
        float pa = 0.f;
        if (i0 + r < L) {
          if (a.hp == 2) {
            for (int s2 = 0; s2 < ch; ++s2) pa = fmaf(wg[hl * ch + s2], P[(s2 * CR + r) * CC + s + PC], pa);
          } else {
            pa = P[(hl * CR + r) * CC + s + PC];
          }
        }
        A3[i] = pa;
      }
      __syncthreads();
      for (int i = tid; i < ch * BC * d; i += kThreads) {
        const int hl = i / (BC * d), rem = i % (BC * d), s = rem / d, e = rem % d, jk = j0 + s;
        if (jk >= L) continue;
        float acc = 0.f;
        for (int r = 0; r < BR; ++r) acc = fmaf(A3[(hl * BR + r) * BC + s], DO[(hl * CR + r) * dp + e], acc);
        atomicAdd(a.dv + oidx(jk, g * ch + hl) + e, acc);
      }
      // per source head: dtheta, dA_hat of the tile, dQ, dK
      for (int sl = 0; sl < ch; ++sl) {
        const int h = g * ch + sl;
        const float *dcr = dcs + sl * region, *sh = Sh + sl * HR * HC;
        if (kq) {  // dtheta[a][t] = sum over the tile's positions of dC[i][j] x shifted logits
          for (int pr = tid; pr < cq * ck * 8; pr += kThreads) {
            const int at = pr / 8, part8 = pr % 8, aa = at / ck, t = at % ck;
            float acc = 0.f;
            for (int i = part8; i < BR * BC; i += 8) {
              const int r = i / BC, s = i % BC + PC, iq = i0 + r, jk = j0 + i % BC;
              if (iq >= L || jk > iq) continue;
              const int keyv = jk - (t - c);  // key read by the tap
              if (exact && keyv > iq) continue;
              acc = fmaf(dcr[r * CC + s], sh[(r + cq - 1 - aa) * HC + s + 2 * c - t], acc);
            }
            atomicAdd(dth + sl * cq * ck + at, acc);
          }
        }
        // dA_hat[i][j] for the tile's rows and keys: the convolution's adjoint of dC, then
        // Mask_0 (or the exact indicator's per-tap condition)
        for (int i = tid; i < BR * BC; i += kThreads) {
          const int r = i / BC, s = i % BC, iq = i0 + r, jk = j0 + s;
          float val = 0.f;
          if (iq < L && jk < L) {
            if (kq) {
              const float *tk = th + sl * cq * ck;
              for (int aa = 0; aa < cq; ++aa) {
                if (i0 + r + aa >= L) break;
                if (!exact && jk > iq) break;
                if (exact && jk > iq + aa) continue;
                const float *drow = dcr + (r + aa) * CC + s + PC - c;
                for (int t = 0; t < ck; ++t) val = fmaf(tk[aa * ck + t], drow[t], val);
              }
            } else {
              val = dcr[r * CC + s];
            }
          }
          Tmp[i] = val * a.scale;
        }
        __syncthreads();
        // restage q (the tile's rows) into Qs and k (the tile's keys) into Ks of head h
        for (int i = tid; i < BR * d; i += kThreads) {
          const int r = i / d, e = i % d, iq = i0 + r;
          Qs[r * dp + e] = iq < L ? ld(q + gidx(iq, h) + e) : 0.f;
        }
        for (int i = tid; i < BC * d; i += kThreads) {
          const int s = i / d, e = i % d, jk = j0 + s;
          Ks[s * dp + e] = jk < L ? ld(k + gidx(jk, h) + e) : 0.f;
        }
        __syncthreads();
        // dQ += dA_hat K and dK += dA_hat^T Q, four rows (columns) per thread sharing
        // each K (Q) load
        for (int i = tid; i < (BR + 3) / 4 * d; i += kThreads) {
          const int r0 = 4 * (i / d), e = i % d;
          float acc[4];
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) acc[k2] = r0 + k2 < BR ? dqa[(sl * BR + r0 + k2) * d + e] : 0.f;
          for (int s = 0; s < BC; ++s) {
            const float x = Ks[s * dp + e];
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) acc[k2] = fmaf(Tmp[min(r0 + k2, BR - 1) * BC + s], x, acc[k2]);
          }
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2)
            if (r0 + k2 < BR) dqa[(sl * BR + r0 + k2) * d + e] = acc[k2];
        }
        for (int i = tid; i < BC / 4 * d; i += kThreads) {
          const int s0 = 4 * (i / d), e = i % d;
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          for (int r = 0; r < BR; ++r) {
            const float x = Qs[r * dp + e];
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) acc[k2] = fmaf(Tmp[r * BC + s0 + k2], x, acc[k2]);
          }
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2)
            if (j0 + s0 + k2 < L) atomicAdd(a.dk + oidx(j0 + s0 + k2, h) + e, acc[k2]);
        }
        __syncthreads();
      }
    }
    if (pass == 0) {  // D = sum_j A dA: normalise by the row sum
      for (int i = tid; i < ch * CR; i += kThreads) Ds[i] = rl[i] > 0.f ? Ds[i] / rl[i] : 0.f;
      __syncthreads();
    }
  }
  for (int i = tid; i < ch * BR * d; i += kThreads) {
    const int hl = i / (BR * d), rem = i % (BR * d), r = rem / d, e = rem % d, iq = i0 + r;
    if (iq < L) a.dq[oidx(iq, g * ch + hl) + e] = dqa[i];
  }
  __syncthreads();
  if (kq && a.dtheta)
    for (int i = tid; i < ch * cq * ck; i += kThreads) atomicAdd(a.dtheta + g * ch * cq * ck + i, dth[i]);
  if (a.hp != 0 && a.dw)
    for (int i = tid; i < ch * ch; i += kThreads) atomicAdd(a.dw + g * ch * ch + i, dwa[i]);
}

}  // namespace

// Rows per CTA: the largest BR whose tile lets two CTAs share an SM (the kernel is
// latency-bound at one), else the largest that fits at all.
int attn_bwd_simt_pick_rows(const BwdArgs &a) {
  auto bytes = [&](int BR) {
    return static_cast<size_t>(bwd_layout(BR, kBC, a.d, a.cq, a.ck, a.ch, a.kq != 0).total) * sizeof(float);
  };
  for (int BR = 16; BR >= 4; BR /= 2)
    if (bytes(BR) <= static_cast<size_t>(kTwoPerSm)) return BR;
  for (int BR = 16; BR >= 1; BR /= 2)
    if (bytes(BR) <= static_cast<size_t>(kSmemCap)) return BR;
  return 0;
}

cudaError_t launch_attn_bwd_simt(const BwdArgs &a) {
  const int BR = attn_bwd_simt_pick_rows(a);
  if (BR == 0) return cudaErrorInvalidConfiguration;
  const size_t smem = static_cast<size_t>(bwd_layout(BR, kBC, a.d, a.cq, a.ck, a.ch, a.kq != 0).total) * sizeof(float);
  const size_t n = static_cast<size_t>(a.B) * a.L * a.H * a.d;
  cudaError_t e;
  if ((e = cudaMemsetAsync(a.dk, 0, n * sizeof(float), a.stream)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(a.dv, 0, n * sizeof(float), a.stream)) != cudaSuccess) return e;
  if (a.kq && a.dtheta &&
      (e = cudaMemsetAsync(a.dtheta, 0, static_cast<size_t>(a.H) * a.cq * a.ck * sizeof(float), a.stream)) != cudaSuccess)
    return e;
  if (a.hp && a.dw &&
      (e = cudaMemsetAsync(a.dw, 0, static_cast<size_t>(a.H) * a.ch * sizeof(float), a.stream)) != cudaSuccess)
    return e;
  dim3 grid((a.L + BR - 1) / BR, a.H / a.ch, a.B);
  auto run = [&](auto kern) -> cudaError_t {
    cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e2 != cudaSuccess) return e2;
    kern<<<grid, kThreads, smem, a.stream>>>(a, BR);
    return cudaGetLastError();
  };
  // specialisations of the pretraining recipe (bf16, c_q = 6, c_k = 11, groups of 2)
  if (a.dtype == 1 && a.cq == 6 && a.ck == 11 && a.ch == 2) {
    if (a.d == 128 && BR == 8) return run(attn_bwd_simt_kernel<__nv_bfloat16, 128, 6, 11, 2, 8>);
    if (a.d == 64 && BR == 8) return run(attn_bwd_simt_kernel<__nv_bfloat16, 64, 6, 11, 2, 8>);
    if (a.d == 64 && BR == 16) return run(attn_bwd_simt_kernel<__nv_bfloat16, 64, 6, 11, 2, 16>);
  }
  if (a.dtype == 0) return run(attn_bwd_simt_kernel<float, 0, 0, 0, 0, 0>);
  return run(attn_bwd_simt_kernel<__nv_bfloat16, 0, 0, 0, 0, 0>);
}

}  // namespace mta
