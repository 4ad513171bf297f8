// attn_bwd_post_simt.cu -- backward pass of MTA attention with the key-query
// convolution also after the softmax, on CUDA cores, fp32 arithmetic.
//
// Forward ("Multi-Token Attention | Summary" (greeksharifa), sections 2, 3.1, 3.2):
//   C = Conv2d_theta(Mask_0(s Q K^T)) (or the exact indicator, or no convolution),
//   C' = pre-softmax mix of C,  A = Softmax(Mask_-inf(C')),
//   A2 = Mask_0(Conv2d_theta_post(A)),  A3 = post-softmax mix of A2,  O = A3 V.
// Backward, each step in reverse:
//   dV_h = A3_h^T dO_h;  G_h = dO_h V_h^T;  dA2_s = sum_h w[h][s] G_h (post mix)
//   dw[h][s] = sum G_h * A2_s (post) or sum dC'_h * C_s (pre)
//   g_s = Mask_0(dA2_s);  dA_s[i][j] = sum_a sum_t theta_post[a][t] g_s[i+a][j+(t-c)]
//   dtheta_post_s[a][t] = sum_ij g_s[i][j] A_s[i-a][j-(t-c)]
//   dC'_s = A_s * (dA_s - D_s),  D_s[i] = sum_j dA_s[i][j] A_s[i][j]
//   then, as without the post-softmax convolution, the pre-softmax mix, the
//   convolution's adjoint and kernel gradient, dQ and dK.
//
// One CTA owns one (batch, head group, tile of BR queries) and sweeps the key
// tiles twice (row statistics and D first, gradients second).  Its maps live on
// regions around the tile (P1 = c_q-1, c = c_k/2):
//   A  : queries i0-P1 .. i0+BR+P1-1, keys j0-c .. j0+BC+c-1 (A2 of the tile reads
//        rows above it, dC' rows below it);
//   g  : queries i0 .. i0+BR+2 P1-1, keys j0-2c .. j0+BC+2c-1 (dA reads rows below);
//   Mask_0(A_hat) for the convolution of the A region: P1 more rows above, c more
//        keys on each side.
// dQ rows are owned by the CTA; dK, dV and the parameter gradients are summed with
// atomic adds.
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
__device__ __forceinline__ float ldv(const T *p);
template <>
__device__ __forceinline__ float ldv<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ldv<__nv_bfloat16>(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

struct PostGeo {
  int P1, c, NRA, NKA, NRM, NKM, NRG, NKG, dp;
};
__host__ __device__ inline PostGeo post_geo(int BR, int BC, int d, int cq, int ck) {
  PostGeo g;
  g.P1 = cq - 1;
  g.c = ck / 2;
  g.NRA = BR + 2 * g.P1;
  g.NKA = BC + 2 * g.c;
  g.NRM = g.NRA + g.P1;
  g.NKM = g.NKA + 2 * g.c;
  g.NRG = BR + 2 * g.P1;
  g.NKG = BC + 4 * g.c;
  g.dp = d + 1;
  return g;
}

struct PostLayout {
  int Qs, Ks, DO, Sh, Cp, P, dA, G, gg, A2, Tmp, m, l, Ds, dqa, th, thp, wg, dth, dthp, dwa, total;
};
__host__ __device__ inline PostLayout post_layout(int BR, int BC, int d, int cq, int ck, int ch) {
  const PostGeo q = post_geo(BR, BC, d, cq, ck);
  const int RA = q.NRA * q.NKA, RG = q.NRG * q.NKG;
  PostLayout s;
  int o = 0;
  s.Qs = o;  o += q.NRM * q.dp;         // query rows i0-2P1 .. of one head
  s.Ks = o;  o += q.NKM * q.dp;         // key rows j0-2c .. (then value rows)
  s.DO = o;  o += ch * q.NRG * q.dp;    // output-gradient rows i0 .. i0+NRG-1, every head
  s.Sh = o;  o += ch * q.NRM * q.NKM;   // Mask_0(A_hat) on the halo, every head
  s.Cp = o;  o += ch * RA;              // C_s on the A region
  s.P = o;   o += ch * RA;              // masked C', then A
  s.dA = o;  o += ch * RA;              // dA, then dC', then dC
  s.G = o;   o += ch * RG;              // dO_h . v_h on the g region
  s.gg = o;  o += ch * RG;              // g_s
  s.A2 = o;  o += ch * BR * BC;         // A2 of the tile, then A3 (scratch)
  s.Tmp = o; o += BR * BC;              // dA_hat of the tile, one head
  s.m = o;   o += ch * q.NRA;
  s.l = o;   o += ch * q.NRA;
  s.Ds = o;  o += ch * q.NRA;
  s.dqa = o; o += ch * BR * d;
  s.th = o;  o += ch * cq * ck;
  s.thp = o; o += ch * cq * ck;
  s.wg = o;  o += ch * ch;
  s.dth = o; o += ch * cq * ck;
  s.dthp = o; o += ch * cq * ck;
  s.dwa = o; o += ch * ch;
  s.total = o;
  return s;
}

// The shape parameters DT, CQT, CKT, CHT, BRT are compile-time constants when
// nonzero (the index arithmetic of every loop then folds), else read at run time.
template <typename T, int DT, int CQT, int CKT, int CHT, int BRT>
__global__ void __launch_bounds__(kThreads) attn_bwd_post_kernel(BwdArgs a, int BR_) {
  const int BR = BRT ? BRT : BR_;
  extern __shared__ float sm[];
  const int BC = kBC;
  const int d = DT ? DT : a.d, cq = CQT ? CQT : a.cq, ck = CKT ? CKT : a.ck, ch = CHT ? CHT : a.ch, L = a.L, H = a.H;
  const bool kq = a.kq != 0, exact = a.kq == 3;
  const PostGeo q = post_geo(BR, BC, d, cq, ck);
  const int P1 = q.P1, c = q.c, NRA = q.NRA, NKA = q.NKA, NRM = q.NRM, NKM = q.NKM;
  const int NRG = q.NRG, NKG = q.NKG, dp = q.dp;
  const int RA = NRA * NKA, RG = NRG * NKG, TILE = BR * BC;
  const PostLayout S = post_layout(BR, BC, d, cq, ck, ch);
  float *Qs = sm + S.Qs, *Ks = sm + S.Ks, *DO = sm + S.DO, *Sh = sm + S.Sh, *Cp = sm + S.Cp;
  float *P = sm + S.P, *dA = sm + S.dA, *Gd = sm + S.G, *gg = sm + S.gg, *A2 = sm + S.A2;
  float *Tmp = sm + S.Tmp, *rm = sm + S.m, *rl = sm + S.l, *Ds = sm + S.Ds, *dqa = sm + S.dqa;
  float *th = sm + S.th, *thp = sm + S.thp, *wg = sm + S.wg, *dth = sm + S.dth, *dthp = sm + S.dthp;
  float *dwa = sm + S.dwa;
  const int i0 = blockIdx.x * BR, g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const T *qp = static_cast<const T *>(a.q);
  const T *kp = static_cast<const T *>(a.k);
  const T *vp = static_cast<const T *>(a.v);
  const T *dout = static_cast<const T *>(a.dout);
  const float NEG_INF = -INFINITY;
  auto gidx = [&](int tok, int h) { return (static_cast<long long>(b) * L + tok) * a.rs + static_cast<long long>(h) * d; };
  auto oidx = [&](int tok, int h) { return ((static_cast<long long>(b) * L + tok) * H + h) * d; };

  for (int i = tid; i < ch * cq * ck; i += kThreads) {
    th[i] = kq ? a.theta[g * ch * cq * ck + i] : 0.f;
    thp[i] = a.theta_post[g * ch * cq * ck + i];
    dth[i] = 0.f;
    dthp[i] = 0.f;
  }
  for (int i = tid; i < ch * ch; i += kThreads) {
    wg[i] = (a.hp != 0) ? a.w[g * ch * ch + i] : (i / ch == i % ch ? 1.f : 0.f);
    dwa[i] = 0.f;
  }
  for (int i = tid; i < ch * NRA; i += kThreads) { rm[i] = NEG_INF; rl[i] = 0.f; Ds[i] = 0.f; }
  for (int i = tid; i < ch * BR * d; i += kThreads) dqa[i] = 0.f;
  for (int i = tid; i < ch * NRG * d; i += kThreads) {
    const int hl = i / (NRG * d), rem = i % (NRG * d), r = rem / d, e = rem % d, iq = i0 + r;
    DO[(hl * NRG + r) * dp + e] = iq < L ? ldv(dout + oidx(iq, g * ch + hl) + e) : 0.f;
  }
  __syncthreads();

  const int r_end = min(L, i0 + BR + 2 * P1);  // the last query any map here reads
  for (int pass = 0; pass < 2; ++pass) {
    for (int j0 = 0; j0 < r_end; j0 += BC) {
      // ---- per head: Mask_0(A_hat) on the halo, C on the A region, G on the g region
      for (int hl = 0; hl < ch; ++hl) {
        const int h = g * ch + hl;
        for (int i = tid; i < NRM * d; i += kThreads) {
          const int r = i / d, e = i % d, iq = i0 - 2 * P1 + r;
          Qs[r * dp + e] = (iq >= 0 && iq < L) ? ldv(qp + gidx(iq, h) + e) : 0.f;
        }
        for (int i = tid; i < NKM * d; i += kThreads) {
          const int s = i / d, e = i % d, jk = j0 - 2 * c + s;
          Ks[s * dp + e] = (jk >= 0 && jk < L) ? ldv(kp + gidx(jk, h) + e) : 0.f;
        }
        __syncthreads();
        float *sh = Sh + hl * NRM * NKM;
        dot_rows4<kThreads>(Qs, Ks, NRM, NKM, d, dp, [&](int r, int s, float v) {
          const int iq = i0 - 2 * P1 + r, jk = j0 - 2 * c + s;
          const bool ok = iq >= 0 && iq < L && jk >= 0 && jk < L && (!kq || exact || jk <= iq);
          sh[r * NKM + s] = ok ? v * a.scale : 0.f;
        });
        __syncthreads();
        for (int i = tid; i < RA; i += kThreads) {  // C on the A region
          const int ra = i / NKA, ka = i % NKA;
          float val;
          if (kq) {
            val = 0.f;
            const float *tk = th + hl * cq * ck;
            const int iq = i0 - P1 + ra, jk = j0 - c + ka;
            const int t0 = exact ? max(0, jk + c - iq) : 0;
            for (int aa = 0; aa < cq; ++aa) {
              const float *srow = sh + (ra + P1 - aa) * NKM + ka + 2 * c;
              for (int t = t0; t < ck; ++t) val = fmaf(tk[aa * ck + t], srow[-t], val);
            }
          } else {
            val = sh[(ra + P1) * NKM + ka + c];
          }
          Cp[hl * RA + i] = val;
        }
        __syncthreads();
        for (int i = tid; i < NKG * d; i += kThreads) {  // value rows of the g region's keys
          const int s = i / d, e = i % d, jk = j0 - 2 * c + s;
          Ks[s * dp + e] = (jk >= 0 && jk < L) ? ldv(vp + gidx(jk, h) + e) : 0.f;
        }
        __syncthreads();
        dot_rows4<kThreads>(DO + hl * NRG * dp, Ks, NRG, NKG, d, dp,
                            [&](int r, int s, float v) { Gd[hl * RG + r * NKG + s] = v; });
        __syncthreads();
      }
      // ---- mixed logits with Mask_-inf (A region); g = Mask_0(post-mix adjoint of G)
      for (int i = tid; i < ch * RA; i += kThreads) {
        const int hl = i / RA, rem = i % RA, ra = rem / NKA, ka = rem % NKA;
        const int iq = i0 - P1 + ra, jk = j0 - c + ka;
        float cv;
        if (a.hp == 1) {
          cv = 0.f;
          for (int s2 = 0; s2 < ch; ++s2) cv = fmaf(wg[hl * ch + s2], Cp[s2 * RA + rem], cv);
        } else {
          cv = Cp[i];
        }
        P[i] = (iq >= 0 && iq < L && jk >= 0 && jk <= iq) ? cv : NEG_INF;
      }
      for (int i = tid; i < ch * RG; i += kThreads) {
        const int sl = i / RG, rem = i % RG, rg = rem / NKG, kg = rem % NKG;
        const int iq = i0 + rg, jk = j0 - 2 * c + kg;
        float val = 0.f;
        if (iq < L && jk >= 0 && jk <= iq) {
          if (a.hp == 2) {
            for (int h2 = 0; h2 < ch; ++h2) val = fmaf(wg[h2 * ch + sl], Gd[h2 * RG + rem], val);
          } else {
            val = Gd[i];
          }
        }
        gg[i] = val;
      }
      __syncthreads();
      // ---- dA on the rows at and below the tile (ra >= P1): the post convolution's adjoint
      for (int i = tid; i < ch * RA; i += kThreads) {
        const int sl = i / RA, rem = i % RA, ra = rem / NKA, ka = rem % NKA;
        float val = 0.f;
        if (ra >= P1) {
          const float *tk = thp + sl * cq * ck;
          for (int aa = 0; aa < cq; ++aa) {
            const float *grow = gg + sl * RG + (ra - P1 + aa) * NKG + ka;
            for (int t = 0; t < ck; ++t) val = fmaf(tk[aa * ck + t], grow[t], val);
          }
        }
        dA[i] = val;
      }
      __syncthreads();
      if (pass == 0) {
        // exact statistics over the tile's own keys (ka = c .. c+BC-1): max, sum and
        // D = sum_j exp(C' - max) dA (rows at and below the tile)
        for (int i = tid; i < ch * NRA; i += kThreads) {
          const float *row = P + i * NKA + c, *dar = dA + i * NKA + c;
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
      // ---- pass 2: A with the final statistics; dC' = A (dA - D) below the top rows
      for (int i = tid; i < ch * RA; i += kThreads) {
        const int hr = i / NKA, ra = (i % RA) / NKA;
        const float pv = (P[i] == NEG_INF || rm[hr] == NEG_INF) ? 0.f : expf(P[i] - rm[hr]) / rl[hr];
        P[i] = pv;
        dA[i] = ra >= P1 ? pv * (dA[i] - Ds[hr]) : 0.f;
      }
      __syncthreads();
      // A2 of the tile: Mask_0(post convolution of A)
      for (int i = tid; i < ch * TILE; i += kThreads) {
        const int sl = i / TILE, rem = i % TILE, r = rem / BC, s = rem % BC;
        const int iq = i0 + r, jk = j0 + s;
        float val = 0.f;
        if (iq < L && jk <= iq) {
          const float *tk = thp + sl * cq * ck;
          for (int aa = 0; aa < cq; ++aa) {
            const float *prow = P + sl * RA + (P1 + r - aa) * NKA + s + 2 * c;
            for (int t = 0; t < ck; ++t) val = fmaf(tk[aa * ck + t], prow[-t], val);
          }
        }
        A2[i] = val;
      }
      __syncthreads();
      // parameter gradients over the tile's positions: dw (post: G_h x A2_s; pre: dC'_h x C_s),
      // dtheta_post (g x shifted A)
      if (a.hp != 0) {
        for (int pr = 0; pr < ch * ch; ++pr) {
          const int hl = pr / ch, sl = pr % ch;
          float part = 0.f;
          for (int i = tid; i < TILE; i += kThreads) {
            const int r = i / BC, s = i % BC;
            if (i0 + r >= L || j0 + s >= L) continue;
            if (a.hp == 2) part = fmaf(Gd[hl * RG + r * NKG + s + 2 * c], A2[sl * TILE + i], part);
            else part = fmaf(dA[hl * RA + (P1 + r) * NKA + s + c], Cp[sl * RA + (P1 + r) * NKA + s + c], part);
          }
          for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
          if ((tid & 31) == 0) atomicAdd(dwa + pr, part);
        }
      }
      for (int pr = tid; pr < ch * cq * ck * 4; pr += kThreads) {
        const int at = pr / 4, part4 = pr % 4, sl = at / (cq * ck), aa = (at / ck) % cq, t = at % ck;
        float acc = 0.f;
        for (int i = part4; i < TILE; i += 4) {
          const int r = i / BC, s = i % BC;
          if (i0 + r >= L || j0 + s > i0 + r) continue;
          acc = fmaf(gg[sl * RG + r * NKG + s + 2 * c], P[sl * RA + (P1 + r - aa) * NKA + s + 2 * c - t], acc);
        }
        atomicAdd(dthp + at, acc);
      }
      __syncthreads();
      // A3 = post mix of A2, in place (the parameter gradients above are done with A2),
      // then dV_h[j] += sum over the tile's rows of A3_h[i][j] dO_h[i]
      if (a.hp == 2) {
        for (int i = tid; i < TILE; i += kThreads) {
          float x[16];
          for (int s2 = 0; s2 < ch; ++s2) x[s2] = A2[s2 * TILE + i];
          for (int hl = 0; hl < ch; ++hl) {
            float pa = 0.f;
            for (int s2 = 0; s2 < ch; ++s2) pa = fmaf(wg[hl * ch + s2], x[s2], pa);
            A2[hl * TILE + i] = pa;
          }
        }
        __syncthreads();
      }
      for (int i = tid; i < ch * BC * d; i += kThreads) {
        const int hl = i / (BC * d), rem = i % (BC * d), s = rem / d, e = rem % d, jk = j0 + s;
        if (jk >= L) continue;
        float acc = 0.f;
        for (int r = 0; r < BR; ++r) acc = fmaf(A2[hl * TILE + r * BC + s], DO[(hl * NRG + r) * dp + e], acc);
        atomicAdd(a.dv + oidx(jk, g * ch + hl) + e, acc);
      }
      // dC_s = sum_h w[h][s] dC'_h (pre-softmax mixing), written over C_s (no longer needed
      // once dw is taken)
      __syncthreads();
      const float *dcs = dA;
      if (a.hp == 1) {
        for (int i = tid; i < ch * RA; i += kThreads) {
          const int sl = i / RA, rem = i % RA;
          float val = 0.f;
          for (int h2 = 0; h2 < ch; ++h2) val = fmaf(wg[h2 * ch + sl], dA[h2 * RA + rem], val);
          Cp[i] = val;
        }
        __syncthreads();
        dcs = Cp;
      }
      for (int sl = 0; sl < ch; ++sl) {
        const int h = g * ch + sl;
        const float *dcr = dcs + sl * RA, *sh = Sh + sl * NRM * NKM;
        if (kq) {  // dtheta over the tile's positions: dC x shifted Mask_0(A_hat)
          for (int pr = tid; pr < cq * ck * 8; pr += kThreads) {
            const int at = pr / 8, part8 = pr % 8, aa = at / ck, t = at % ck;
            float acc = 0.f;
            for (int i = part8; i < TILE; i += 8) {
              const int r = i / BC, s = i % BC, iq = i0 + r, jk = j0 + s;
              if (iq >= L || jk > iq) continue;
              if (exact && jk - (t - c) > iq) continue;
              acc = fmaf(dcr[(P1 + r) * NKA + s + c], sh[(r + 2 * P1 - aa) * NKM + s + 3 * c - t], acc);
            }
            atomicAdd(dth + sl * cq * ck + at, acc);
          }
        }
        // dA_hat of the tile: the pre convolution's adjoint of dC, then Mask_0 / the indicator
        for (int i = tid; i < TILE; i += kThreads) {
          const int r = i / BC, s = i % BC, iq = i0 + r, jk = j0 + s;
          float val = 0.f;
          if (iq < L && jk < L) {
            if (kq) {
              const float *tk = th + sl * cq * ck;
              for (int aa = 0; aa < cq; ++aa) {
                if (iq + aa >= L) break;
                if (!exact && jk > iq) break;
                if (exact && jk > iq + aa) continue;
                const float *drow = dcr + (P1 + r + aa) * NKA + s;
                for (int t = 0; t < ck; ++t) val = fmaf(tk[aa * ck + t], drow[t], val);
              }
            } else {
              val = dcr[(P1 + r) * NKA + s + c];
            }
          }
          Tmp[i] = val * a.scale;
        }
        __syncthreads();
        for (int i = tid; i < BR * d; i += kThreads) {
          const int r = i / d, e = i % d, iq = i0 + r;
          Qs[r * dp + e] = iq < L ? ldv(qp + gidx(iq, h) + e) : 0.f;
        }
        for (int i = tid; i < BC * d; i += kThreads) {
          const int s = i / d, e = i % d, jk = j0 + s;
          Ks[s * dp + e] = jk < L ? ldv(kp + gidx(jk, h) + e) : 0.f;
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
    if (pass == 0) {
      for (int i = tid; i < ch * NRA; i += kThreads) Ds[i] = rl[i] > 0.f ? Ds[i] / rl[i] : 0.f;
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
  if (a.dtheta_post)
    for (int i = tid; i < ch * cq * ck; i += kThreads) atomicAdd(a.dtheta_post + g * ch * cq * ck + i, dthp[i]);
  if (a.hp != 0 && a.dw)
    for (int i = tid; i < ch * ch; i += kThreads) atomicAdd(a.dw + g * ch * ch + i, dwa[i]);
}

}  // namespace

// Rows per CTA: the largest BR whose tile lets two CTAs share an SM, else the
// largest that fits at all.
int attn_bwd_post_pick_rows(const BwdArgs &a) {
  auto bytes = [&](int BR) {
    return static_cast<size_t>(post_layout(BR, kBC, a.d, a.cq, a.ck, a.ch).total) * sizeof(float);
  };
  for (int BR = 16; BR >= 4; BR /= 2)
    if (bytes(BR) <= static_cast<size_t>(kTwoPerSm)) return BR;
  for (int BR = 16; BR >= 1; BR /= 2)
    if (bytes(BR) <= static_cast<size_t>(kSmemCap)) return BR;
  return 0;
}

cudaError_t launch_attn_bwd_post(const BwdArgs &a) {
  const int BR = attn_bwd_post_pick_rows(a);
  if (BR == 0) return cudaErrorInvalidConfiguration;
  const size_t smem = static_cast<size_t>(post_layout(BR, kBC, a.d, a.cq, a.ck, a.ch).total) * sizeof(float);
  const size_t n = static_cast<size_t>(a.B) * a.L * a.H * a.d;
  const size_t nth = static_cast<size_t>(a.H) * a.cq * a.ck * sizeof(float);
  cudaError_t e;
  if ((e = cudaMemsetAsync(a.dk, 0, n * sizeof(float), a.stream)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(a.dv, 0, n * sizeof(float), a.stream)) != cudaSuccess) return e;
  if (a.kq && a.dtheta && (e = cudaMemsetAsync(a.dtheta, 0, nth, a.stream)) != cudaSuccess) return e;
  if (a.dtheta_post && (e = cudaMemsetAsync(a.dtheta_post, 0, nth, a.stream)) != cudaSuccess) return e;
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
    if (a.d == 128 && BR == 8) return run(attn_bwd_post_kernel<__nv_bfloat16, 128, 6, 11, 2, 8>);
    if (a.d == 64 && BR == 8) return run(attn_bwd_post_kernel<__nv_bfloat16, 64, 6, 11, 2, 8>);
    if (a.d == 64 && BR == 16) return run(attn_bwd_post_kernel<__nv_bfloat16, 64, 6, 11, 2, 16>);
  }
  if (a.dtype == 0) return run(attn_bwd_post_kernel<float, 0, 0, 0, 0, 0>);
  return run(attn_bwd_post_kernel<__nv_bfloat16, 0, 0, 0, 0, 0>);
}

}  // namespace mta
