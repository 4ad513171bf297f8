// attn_bwd_tc.cu -- the MTA attention backward with its contractions on the
// tensor cores ("Multi-Token Attention | Summary" (greeksharifa), sections 2,
// 3.1 and 3.2, each forward step taken in reverse; the pages train with this
// forward, section 4 and appendix F).
//
// The forward per head group: logits S = s Q K^T, Mask_0, the key-query
// convolution C = Conv2d_theta(Mask_0 S), optional pre-softmax mixing
// C'_h = sum_s w[h][s] C_s, Mask_-inf and the softmax A, optional post-softmax
// mixing A''_h = sum_s w[h][s] A_s, O_h = A''_h V_h.  Its adjoints:
//   dA''_h = dO_h V_h^T                      (tensor cores)
//   dV_h   = A''_h^T dO_h                    (tensor cores)
//   dA_s   = sum_h w[h][s] dA''_h, dw[h][s] = sum dA''_h . A_s   (post mixing)
//   dC_s   = A_s (dA_s - D_s), D_s = rowsum(dA_s . A_s)          (softmax)
//   dC_s   = sum_h w[h][s] dC'_h, dw[h][s] = sum dC'_h . C_s     (pre mixing)
//   dS[i][j] = [j <= i] sum_{a,t} theta[a][t] dC[i+a][j+t-c]     (the convolution's adjoint)
//   dtheta[a][t] = sum dC[i][j] Mask_0 S[i-a][j-(t-c)]
//   dQ = s dS K, dK = s dS^T Q               (tensor cores)
//
// Query blocks of NO = R - 2 (c_q - 1) rows (R = 384 or 512, block_rows below) are
// processed one after another, all heads at once.  For block rows r0 .. r0+NO-1
// the maps are held in strips of the workspace that span every key up to the
// block's last row: S for rows r0-(c_q-1) .. r0+NO+c_q-2 (R rows: the convolution
// reads c_q-1 earlier query
// rows, its adjoint c_q-1 later ones), A, dA'' then dC for rows r0 .. r0+NO+c_q-2,
// dS and A'' for the block's own rows.  A strip holds whole rows, so the softmax
// statistics and D come from the strip itself (no statistics pass).  The strips
// are O(B H R L): never an L x L map.  Per block:
//   1. S strip      = s Q K^T                      batched GEMM (fp32 out)
//   2. dA'' strip   = dO V^T                       batched GEMM
//   3. C, softmax, then dC, D, dw, A''             bwd_scores_kernel (CUDA cores)
//   4. dS, dtheta                                  bwd_adjoint_kernel
//   5. dQ rows (=), dK, dV (+=)                    batched GEMMs
// With the convolution after the softmax, A' = Mask_0(Conv2d_theta_post A) sits
// between the softmax and the post-softmax mixing; its adjoint reads G = dL/dA'
// c_q-1 rows below each row and A' reads A c_q-1 rows above, so a block carries a
// second halo: NO = R - 3 (c_q - 1), S from row r0 - 2 (c_q - 1), the weights A
// from r0 - (c_q - 1).  Step 3 then writes the normalised weights only, and four
// kernels follow it: G (bwd_post_grad_kernel), dA = its adjoint with dtheta_post
// and A' of the own rows (bwd_adjoint_kernel, mode 1), A'' and the post-mixing dw
// (bwd_post_mix_kernel), dC and D (bwd_post_softmax_kernel).
// dS and A'' enter the GEMMs of step 5 as two bf16 halves, hi = bf16(x) and
// lo = bf16(x - hi), summed by two GEMMs into the same fp32 output: the operands
// then carry about 16 significant bits and the gradients stay within fp32
// tolerance of the CUDA-core backward.  The other GEMM operands (q, k, v, dO) are
// the bf16 inputs themselves.
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace mta {
namespace {

// Rows of a query block's S strip (and of each half of its dS / A'' strips): 384 up
// to L = 3072, else 512.  Measured on one B200 (d = 128, groups of 2): at L = 2048,
// 4.61 ms with 384 rows against 4.74 with 256 and 4.87 with 512 (four full blocks and
// a 40-row one); at L = 4096, 9.68 ms with 512 against 9.92 with 384 and 9.97 with 256.
int block_rows(int L) { return L <= 3072 ? 384 : 512; }
constexpr int kKeyTile = 128;
constexpr int kThreadsB = 256;

struct Geo {
  int halo, c, no, rc, pitch;  // c_q - 1, c_k / 2, own rows, C rows, strip pitch (elements)
  int rt;                      // rows of the S strip and of each dS / A'' half (block_rows)
};

struct StripArgs {
  int B, H, L, ch, hp;        // hp: 0 off, 1 pre, 2 post
  int r0, W, Wp;              // block's first row, keys 0 .. W-1 (Wp = W rounded up to 64)
  Geo g;
  const float *theta;         // [H][c_q][c_k]
  const float *w;             // [H/c_h][c_h][c_h]
  float *S;                   // [B][H][R][pitch]
  float *Cpre;                // [B][H][rc][pitch] pre-mixing C (pre mixing only)
  float *A;                   // [B][H][rc][pitch]
  float *D;                   // [B][H][rc][pitch]: dA'' from the GEMM, then dC
  __nv_bfloat16 *dS;          // [B][H][2R][pitch]: hi rows 0..R-1, lo rows R..2R-1
  __nv_bfloat16 *Ap;          // [B][H][2R][pitch]: A'' hi / lo
  float *dtheta, *dw;
  int post;                   // the convolution after the softmax: the scores kernel
                              // only writes the normalised weights A
};

__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16 &hi, __nv_bfloat16 &lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// Step 3: C = Conv2d_theta(Mask_0 S) for the block's C rows (and pre mixing),
// Mask_-inf, the softmax statistics of each row (its logits kept in the A strip)
// and, in the same pass, D = sum_j dA A and the post-mixing dw online (rescaled
// with the running maximum as the sum is); then the softmax's backward on the
// same rows: dA (post mixing: mixed back to the sources), dC = A (dA - D) (pre
// mixing: then mixed back) into the dA'' strip, the pre-mixing dw, and A'' (hi /
// lo) of the block's own rows.  CTA: one head group, 16 rows; thread (row, seg):
// 8 consecutive keys 8 seg .. 8 seg + 7 of every 128-key tile.  For each tap row
// a the thread loads the 24 staged values around its keys (keys jb - 8 .. jb + 15,
// 8 + 2c of them used) once and forms its 8 outputs x c_k taps from registers.
// Key tiles past the CTA's last row are skipped (their weights are zero and
// nothing reads them).
constexpr int kRows = 16;               // rows of a CTA in the convolution kernels
constexpr int kSeg = 8;                 // consecutive keys of a thread
// Staged rows are 164 floats (128 + 2c keys, padded): 656 bytes, 16 modulo 128, so
// that the 16-byte window loads of a quarter warp -- four threads of one row and
// four of the next, 32 bytes apart along a row -- fall on eight different bank
// groups.
constexpr int kTilePitch = 164;
constexpr int kTileCols = kKeyTile + 16;  // columns staged: keys j0 - 8 .. j0 + 135
constexpr int kStagedRows = kRows + 5;     // rows staged for c_q = 6 (dynamic shared memory)
// thread -> (row, seg): a warp holds rows 2 warp, 2 warp + 1; lane bit 2 picks
// the row, the other bits the 8-key segment
__device__ __forceinline__ int tile_row(int tid) { return 2 * (tid >> 5) + ((tid >> 2) & 1); }
__device__ __forceinline__ int tile_seg(int tid) { return (tid & 3) | (((tid & 31) >> 3) << 2); }

// Starts staging TR rows of a strip into tile[TR][kTilePitch]: tile row r gets
// strip row row0 + r (its query q0 + r; zeros once the strip row reaches nrows or
// the query reaches L), tile column cc key j0 - 8 + cc, zero for a key below 0 or
// past the row's query (Mask_0 and the causal mask of the gradients).  A warp per
// row, one 16-byte copy per four keys (aligned: the strip pitch is a multiple of
// 64); the copy of a group that straddles the row's query takes only its valid
// leading keys and zero-fills the rest.
template <int TR>
__device__ __forceinline__ void stage_rows(float (*tile)[kTilePitch], const float *strip0, int P, int row0,
                                           int nrows, int q0, int L, int j0) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NV = kTileCols / 4;
  for (int r = warp; r < TR; r += kThreadsB / 32) {
    const int sr = row0 + r, q = q0 + r;
    const bool rv = sr < nrows && q >= 0 && q < L;
    const float *src = strip0 + static_cast<long long>(rv ? sr : 0) * P;
    for (int v = lane; v < NV; v += 32) {
      const int k0 = j0 - 8 + 4 * v;
      const int n = (rv && k0 >= 0) ? min(4, max(0, q - k0 + 1)) : 0;
      cp_async16(&tile[r][4 * v], n ? src + k0 : strip0, 4 * n);
    }
  }
}

template <int CQ, int CK, int CH>
__global__ void __launch_bounds__(kThreadsB) bwd_scores_kernel(StripArgs p) {
  constexpr int HALO = CQ - 1, C = CK / 2, TR = kRows + HALO, WIN = kSeg + 16;
  static_assert(C <= 8 && kKeyTile + 16 <= kTileCols && kTileCols <= kTilePitch, "tile columns");
  static_assert(TR == kStagedRows, "dynamic shared memory sized for c_q = 6");
  extern __shared__ __align__(16) float dyn[];
  float(*tile)[CH][TR][kTilePitch] = reinterpret_cast<float(*)[CH][TR][kTilePitch]>(dyn);  // [2 stages]
  __shared__ float th[CH][CQ * CK], wm[CH * CH];
  const int G = p.H / CH, bg = blockIdx.y, b = bg / G, g = bg % G;
  const int u0 = blockIdx.x * kRows, row = tile_row(threadIdx.x), seg = tile_seg(threadIdx.x);
  const int u = u0 + row, i = p.r0 + u;
  const bool valid = u < p.g.rc && i < p.L;
  const int P = p.g.pitch;
  for (int x = threadIdx.x; x < CH * CQ * CK; x += kThreadsB)
    th[x / (CQ * CK)][x % (CQ * CK)] = p.theta[(g * CH + x / (CQ * CK)) * CQ * CK + x % (CQ * CK)];
  for (int x = threadIdx.x; x < CH * CH; x += kThreadsB) wm[x] = p.w ? p.w[g * CH * CH + x] : (x % (CH + 1) == 0);
  auto strip = [&](float *base, int hl, int rows) {
    return base + ((static_cast<long long>(b) * p.H + g * CH + hl) * rows) * P;
  };
  // online statistics of each softmax head s: max m, sum l = sum_j e_j, and, with
  // e_j = exp(C_s[j] - m), Dt = sum_j dA_s[j] e_j (D_s = Dt / l) and, with post
  // mixing on the own rows, Wt[h][s] = sum_j dA''_h[j] e_j (dw[h][s] += Wt / l)
  float m[CH], l[CH], Dt[CH], Wt[CH * CH];
#pragma unroll
  for (int h = 0; h < CH; ++h) { m[h] = -INFINITY; l[h] = 0.f; Dt[h] = 0.f; }
#pragma unroll
  for (int x = 0; x < CH * CH; ++x) Wt[x] = 0.f;
  const bool own = valid && u < p.g.no;
  const int i_last = min(p.L - 1, p.r0 + u0 + kRows - 1);  // the CTA's last query
  const int ntiles = i_last / kKeyTile + 1;
  // Mask_0 S: strip rows u0 .. u0+TR-1 (queries r0 - HALO + su), keys j0 - 8 ..
  auto stage = [&](int tt) {
#pragma unroll
    for (int hl = 0; hl < CH; ++hl)
      stage_rows<TR>(tile[tt & 1][hl], strip(p.S, hl, p.g.rt), P, u0, p.g.rt, p.r0 - HALO + u0, p.L, tt * kKeyTile);
  };
  stage(0);
  cp_async_commit();
  for (int tt = 0; tt < ntiles; ++tt) {
    const int j0 = tt * kKeyTile;
    if (tt + 1 < ntiles) stage(tt + 1);  // the next tile's copies run under this tile's arithmetic
    cp_async_commit();
    cp_async_wait_prev();
    __syncthreads();
    const int jb = j0 + kSeg * seg;  // first key of the thread
    if (valid && jb <= i) {
    if (!p.post) {  // dA'' of the thread's keys, read after the convolution: fetch it now
#pragma unroll
      for (int h = 0; h < CH; ++h) prefetch_l1(strip(p.D, h, p.g.rc) + u * P + jb);
    }
    float cv[CH][kSeg];
#pragma unroll
    for (int h = 0; h < CH; ++h) {
#pragma unroll
      for (int x = 0; x < kSeg; ++x) cv[h][x] = 0.f;
#pragma unroll
      for (int a = 0; a < CQ; ++a) {
        // keys jb - 8 .. jb + 15 of query i - a: tile columns 8 seg .. 8 seg + 23
        float w[WIN];
        const float4 *src = reinterpret_cast<const float4 *>(&tile[tt & 1][h][row + HALO - a][kSeg * seg]);
#pragma unroll
        for (int v4 = 0; v4 < WIN / 4; ++v4) {
          const float4 q4 = src[v4];
          w[4 * v4 + 0] = q4.x; w[4 * v4 + 1] = q4.y; w[4 * v4 + 2] = q4.z; w[4 * v4 + 3] = q4.w;
        }
        // C[i][j] += theta[a][t] S[i-a][j-(t-c)]: key jb + x - t + c = window x + 8 + c - t
#pragma unroll
        for (int t = 0; t < CK; ++t)
#pragma unroll
          for (int x = 0; x < kSeg; ++x) cv[h][x] = fmaf(th[h][a * CK + t], w[x + 8 + C - t], cv[h][x]);
      }
    }
    if (p.hp == 1 && p.Cpre) {
#pragma unroll
      for (int h = 0; h < CH; ++h) {
        float *dst = strip(p.Cpre, h, p.g.rc) + u * P + jb;
#pragma unroll
        for (int x = 0; x < kSeg; x += 4)
          *reinterpret_cast<float4 *>(dst + x) = make_float4(cv[h][x], cv[h][x + 1], cv[h][x + 2], cv[h][x + 3]);
      }
    }
    // dA'' of every head of the group at the thread's keys (the GEMM ran before;
    // with the convolution after the softmax the D strip holds other rows: unused)
    float da2[CH][kSeg];
#pragma unroll
    for (int h = 0; h < CH; ++h) {
      const float *src = strip(p.D, h, p.g.rc) + u * P + jb;
#pragma unroll
      for (int x = 0; x < kSeg; x += 4) {
        const float4 v = p.post ? make_float4(0.f, 0.f, 0.f, 0.f) : *reinterpret_cast<const float4 *>(src + x);
        da2[h][x] = v.x; da2[h][x + 1] = v.y; da2[h][x + 2] = v.z; da2[h][x + 3] = v.w;
      }
    }
#pragma unroll
    for (int h = 0; h < CH; ++h) {
      float lg[kSeg];
#pragma unroll
      for (int x = 0; x < kSeg; ++x) {
        float z = cv[h][x];
        if (p.hp == 1) {
          z = 0.f;
#pragma unroll
          for (int s2 = 0; s2 < CH; ++s2) z = fmaf(wm[h * CH + s2], cv[s2][x], z);
        }
        z = jb + x <= i ? z : -INFINITY;  // Mask_-inf
        lg[x] = z;
        if (z == -INFINITY) continue;
        // dA of softmax head h: post mixing mixes dA'' back to the source
        float d = da2[h][x];
        if (p.hp == 2) {
          d = 0.f;
#pragma unroll
          for (int h2 = 0; h2 < CH; ++h2) d = fmaf(wm[h2 * CH + h], da2[h2][x], d);
        }
        float e = 1.f;
        if (z > m[h]) {
          const float sc = __expf(m[h] - z);
          l[h] *= sc;
          Dt[h] *= sc;
          if (p.hp == 2) {
#pragma unroll
            for (int h2 = 0; h2 < CH; ++h2) Wt[h2 * CH + h] *= sc;
          }
          m[h] = z;
        } else {
          e = __expf(z - m[h]);
        }
        l[h] += e;
        Dt[h] = fmaf(d, e, Dt[h]);
        if (p.hp == 2 && own) {
#pragma unroll
          for (int h2 = 0; h2 < CH; ++h2) Wt[h2 * CH + h] = fmaf(da2[h2][x], e, Wt[h2 * CH + h]);
        }
      }
      float *dst = strip(p.A, h, p.g.rc) + u * P + jb;  // logits for now
#pragma unroll
      for (int x = 0; x < kSeg; x += 4)
        *reinterpret_cast<float4 *>(dst + x) = make_float4(lg[x], lg[x + 1], lg[x + 2], lg[x + 3]);
    }
    }
    __syncthreads();  // the buffer is restaged two tiles on
  }
  // row statistics over the 16 threads of the row (the lanes with the same bit 2)
  float mr[CH], lr[CH], Dr[CH], dwp[CH * CH];
#pragma unroll
  for (int x = 0; x < CH * CH; ++x) dwp[x] = 0.f;
#pragma unroll
  for (int h = 0; h < CH; ++h) {
    float mx = m[h];
#pragma unroll
    for (int o : {1, 2, 8, 16}) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float sc = m[h] == -INFINITY ? 0.f : __expf(m[h] - mx);
    float part = l[h] * sc, dpart = Dt[h] * sc;
#pragma unroll
    for (int o : {1, 2, 8, 16}) {
      part += __shfl_xor_sync(0xffffffffu, part, o);
      dpart += __shfl_xor_sync(0xffffffffu, dpart, o);
    }
    mr[h] = mx;
    lr[h] = part;
    Dr[h] = part > 0.f ? dpart / part : 0.f;
    if (p.hp == 2) {
      // dw[h2][h] over this row: Wt / l, summed over the row's 16 threads (each
      // thread's share taken once, by the block reduction below)
#pragma unroll
      for (int h2 = 0; h2 < CH; ++h2) dwp[h2 * CH + h] = part > 0.f ? Wt[h2 * CH + h] * sc / part : 0.f;
    }
  }
  float inv[CH];
#pragma unroll
  for (int h = 0; h < CH; ++h) inv[h] = 1.f / lr[h];
  if (p.post) {
    // the convolution after the softmax comes between the weights and their
    // gradient: store the normalised weights A (zero past the diagonal) and stop
    if (!valid) return;
    for (int jb = kSeg * seg; jb <= i; jb += kKeyTile) {
#pragma unroll
      for (int h = 0; h < CH; ++h) {
        float *a = strip(p.A, h, p.g.rc) + u * P + jb;
#pragma unroll
        for (int x = 0; x < kSeg; x += 4) {
          float4 v = *reinterpret_cast<float4 *>(a + x);
          v.x = jb + x + 0 <= i ? __expf(v.x - mr[h]) * inv[h] : 0.f;
          v.y = jb + x + 1 <= i ? __expf(v.y - mr[h]) * inv[h] : 0.f;
          v.z = jb + x + 2 <= i ? __expf(v.z - mr[h]) * inv[h] : 0.f;
          v.w = jb + x + 3 <= i ? __expf(v.w - mr[h]) * inv[h] : 0.f;
          *reinterpret_cast<float4 *>(a + x) = v;
        }
      }
    }
    return;
  }
  // ---- the softmax's backward on the same rows: the weights A_s = exp(C - m) / l
  // are recomputed from the logits wherever they are needed, never stored
  auto weights = [&](int jb, int h, float (&a)[kSeg]) {
    const float *lg = strip(p.A, h, p.g.rc) + u * P + jb;
#pragma unroll
    for (int x = 0; x < kSeg; x += 4) {
      const float4 v = *reinterpret_cast<const float4 *>(lg + x);
      a[x + 0] = jb + x + 0 <= i ? __expf(v.x - mr[h]) * inv[h] : 0.f;
      a[x + 1] = jb + x + 1 <= i ? __expf(v.y - mr[h]) * inv[h] : 0.f;
      a[x + 2] = jb + x + 2 <= i ? __expf(v.z - mr[h]) * inv[h] : 0.f;
      a[x + 3] = jb + x + 3 <= i ? __expf(v.w - mr[h]) * inv[h] : 0.f;
    }
  };
  auto grads = [&](int jb, int h, float (&da)[kSeg]) {  // dA'' from the GEMM
    const float *src = strip(p.D, h, p.g.rc) + u * P + jb;
#pragma unroll
    for (int x = 0; x < kSeg; x += 4) {
      const float4 v = *reinterpret_cast<const float4 *>(src + x);
      da[x + 0] = jb + x + 0 <= i ? v.x : 0.f;
      da[x + 1] = jb + x + 1 <= i ? v.y : 0.f;
      da[x + 2] = jb + x + 2 <= i ? v.z : 0.f;
      da[x + 3] = jb + x + 3 <= i ? v.w : 0.f;
    }
  };
  // pass 2: dC = A (dA - D) into the dA'' strip (pre mixing: dC'_h, then mixed
  // back, with dw = sum dC'_h C_s); A'' (hi / lo) of the own rows
  if (valid) {
    for (int jb = kSeg * seg; jb <= i; jb += kKeyTile) {
      if (jb + kKeyTile <= i) {  // the next chunk's logits and dA'', while this one is computed
#pragma unroll
        for (int h = 0; h < CH; ++h) {
          prefetch_l1(strip(p.A, h, p.g.rc) + u * P + jb + kKeyTile);
          prefetch_l1(strip(p.D, h, p.g.rc) + u * P + jb + kKeyTile);
        }
      }
      float a[CH][kSeg], da[CH][kSeg], dc[CH][kSeg];
#pragma unroll
      for (int h = 0; h < CH; ++h) { weights(jb, h, a[h]); grads(jb, h, da[h]); }
      if (p.hp == 1) {
#pragma unroll
        for (int x = 0; x < kSeg; ++x) {
          float dcp[CH];
#pragma unroll
          for (int h = 0; h < CH; ++h) dcp[h] = a[h][x] * (da[h][x] - Dr[h]);
#pragma unroll
          for (int s2 = 0; s2 < CH; ++s2) {
            float v = 0.f;
#pragma unroll
            for (int h = 0; h < CH; ++h) v = fmaf(wm[h * CH + s2], dcp[h], v);
            dc[s2][x] = v;
          }
          if (own && jb + x <= i) {
#pragma unroll
            for (int s2 = 0; s2 < CH; ++s2) {
              const float cs = strip(p.Cpre, s2, p.g.rc)[u * P + jb + x];
#pragma unroll
              for (int h = 0; h < CH; ++h) dwp[h * CH + s2] = fmaf(dcp[h], cs, dwp[h * CH + s2]);
            }
          }
        }
      } else {
#pragma unroll
        for (int s2 = 0; s2 < CH; ++s2)
#pragma unroll
          for (int x = 0; x < kSeg; ++x) {
            float d = da[s2][x];
            if (p.hp == 2) {
              d = 0.f;
#pragma unroll
              for (int h = 0; h < CH; ++h) d = fmaf(wm[h * CH + s2], da[h][x], d);
            }
            dc[s2][x] = a[s2][x] * (d - Dr[s2]);
          }
      }
#pragma unroll
      for (int s2 = 0; s2 < CH; ++s2) {
        float *dst = strip(p.D, s2, p.g.rc) + u * P + jb;
#pragma unroll
        for (int x = 0; x < kSeg; x += 4)
          *reinterpret_cast<float4 *>(dst + x) = make_float4(dc[s2][x], dc[s2][x + 1], dc[s2][x + 2], dc[s2][x + 3]);
      }
      if (own) {
        // A''_h = sum_s w[h][s] A_s (post mixing), else A_h
#pragma unroll
        for (int h = 0; h < CH; ++h) {
          uint32_t hi[kSeg / 2], lo[kSeg / 2];
#pragma unroll
          for (int x = 0; x < kSeg; x += 2) {
            float y[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              float v = a[h][x + e];
              if (p.hp == 2) {
                v = 0.f;
#pragma unroll
                for (int s2 = 0; s2 < CH; ++s2) v = fmaf(wm[h * CH + s2], a[s2][x + e], v);
              }
              y[e] = v;
            }
            __nv_bfloat16 h0, l0, h1, l1;
            split_bf16(y[0], h0, l0);
            split_bf16(y[1], h1, l1);
            hi[x / 2] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
            lo[x / 2] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
          }
          __nv_bfloat16 *ap = reinterpret_cast<__nv_bfloat16 *>(
              p.Ap + ((static_cast<long long>(b) * p.H + g * CH + h) * 2 * p.g.rt) * P);
          *reinterpret_cast<uint4 *>(ap + static_cast<long long>(u) * P + jb) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4 *>(ap + static_cast<long long>(p.g.rt + u) * P + jb) =
              make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
    }
  }
  if (p.hp != 0 && p.dw) {
    __shared__ float dwr[CH * CH];
    if (threadIdx.x < CH * CH) dwr[threadIdx.x] = 0.f;
    __syncthreads();
#pragma unroll
    for (int x = 0; x < CH * CH; ++x) {
      float v = dwp[x];
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if ((threadIdx.x & 31) == 0) atomicAdd(&dwr[x], v);
    }
    __syncthreads();
    if (threadIdx.x < CH * CH) atomicAdd(p.dw + g * CH * CH + threadIdx.x, dwr[threadIdx.x]);
  }
}

// The adjoint of one key-query convolution, for the rows of one head:
//   out[i][j] = [j <= i] sum_{a,t} theta[a][t] G[i+a][j+t-c]
//   dtheta[a][t] += sum over the own rows of G[i][j] X[i-a][j-(t-c)]
// where G is the gradient at the convolution's output (zero past the diagonal)
// and X its input.  MODE 0, the convolution before the softmax: G = dC, X =
// Mask_0 S, out = dS written as hi / lo bf16 halves for the own rows (zeros for
// the others).  MODE 1, the convolution after the softmax: G = Mask_0 dA', X = A,
// out = dA in fp32 for every row below out_rows; the kernel also forms the
// convolution itself on the own rows, A' = Mask_0(Conv2d(A)), into a strip.
struct AdjArgs {
  const float *G;       // [B][H][g_rows][pitch], row u <-> query r0 + u
  int g_rows;
  const float *X;       // [B][H][x_rows][pitch], row u <-> query x_base + u
  int x_rows, x_base;
  const float *theta;   // [H][c_q][c_k]
  float *dtheta;        // [H][c_q][c_k] (or null)
  int out_rows;         // MODE 1: rows of dA
  __nv_bfloat16 *dS;    // MODE 0: [B][H][2R][pitch]
  float *dA;            // MODE 1: [B][H][out_rows][pitch]
  float *Ac;            // MODE 1: A' of the own rows, [B][H][no][pitch]
};

// Step 4: CTA = one head and 16 rows u = 0 .. R-1; thread (row, seg): 8
// consecutive keys, register windows of the staged rows as in the scores kernel.
// Key tiles past the CTA's last row only write zeros (MODE 0).
template <int CQ, int CK, int MODE>
__global__ void __launch_bounds__(kThreadsB) bwd_adjoint_kernel(StripArgs p, AdjArgs q) {
  constexpr int HALO = CQ - 1, C = CK / 2, TR = kRows + HALO, NT = CQ * CK, WIN = kSeg + 16;
  static_assert(C <= 8 && TR == kStagedRows, "window; dynamic shared memory sized for c_q = 6");
  extern __shared__ __align__(16) float dyn[];
  // [2 stages]: G rows and X rows, tile column cc = key j0 - 8 + cc
  float(*dct)[TR][kTilePitch] = reinterpret_cast<float(*)[TR][kTilePitch]>(dyn);
  float(*st)[TR][kTilePitch] = reinterpret_cast<float(*)[TR][kTilePitch]>(dyn + 2 * TR * kTilePitch);
  __shared__ float th[NT];
  const int z = blockIdx.y, h = z % p.H;
  const int u0 = blockIdx.x * kRows, row = tile_row(threadIdx.x), seg = tile_seg(threadIdx.x);
  const int u = u0 + row, i = p.r0 + u;
  const bool own = u < p.g.no && i < p.L;
  // rows whose convolution adjoint is written
  const int n_out = MODE == 0 ? p.g.no : q.out_rows;
  const bool outr = u < n_out && i < p.L;
  const int P = p.g.pitch;
  const float *Gz = q.G + static_cast<long long>(z) * q.g_rows * P;
  const float *Xz = q.X + static_cast<long long>(z) * q.x_rows * P;
  // X row of query i - a for tile row row + HALO - a: X rows start at u0 + xoff
  const int xoff = p.r0 - q.x_base - HALO;
  for (int x = threadIdx.x; x < NT; x += kThreadsB) th[x] = q.theta[h * NT + x];
  float dth[NT];
#pragma unroll
  for (int x = 0; x < NT; ++x) dth[x] = 0.f;
  const int i_last = min(p.L - 1, p.r0 + min(u0 + kRows - 1, n_out - 1));  // last written query of the CTA
  // key tiles with work (uniform over the CTA); the later ones only write zeros
  const int nwork = u0 < n_out ? i_last / kKeyTile + 1 : 0;
  auto stage = [&](int tt) {
    // G rows u0 .. u0+TR-1 (queries r0 + u'), zero past its rows, the sequence and the diagonal
    stage_rows<TR>(dct[tt & 1], Gz, P, u0, q.g_rows, p.r0 + u0, p.L, tt * kKeyTile);
    // X rows of queries r0 + u0 - HALO .. (Mask_0 S, or A: zero past the diagonal)
    stage_rows<TR>(st[tt & 1], Xz, P, u0 + xoff, q.x_rows, q.x_base + u0 + xoff, p.L, tt * kKeyTile);
  };
  if (nwork) stage(0);
  cp_async_commit();
  const int jend = MODE == 0 ? p.Wp : (nwork ? nwork * kKeyTile : 0);
  for (int j0 = 0, tt = 0; j0 < jend; j0 += kKeyTile, ++tt) {
    const int jb = j0 + kSeg * seg;
    const bool work = tt < nwork;
    if (work) {
      if (tt + 1 < nwork) stage(tt + 1);
      cp_async_commit();
      cp_async_wait_prev();
      __syncthreads();
    }
    float ds[kSeg], ac[kSeg];
#pragma unroll
    for (int x = 0; x < kSeg; ++x) { ds[x] = 0.f; ac[x] = 0.f; }
    if (work && outr && jb <= i && jb < p.Wp) {
      // G[i][j] of the thread's keys (zero past the diagonal) for dtheta, own rows only
      const int bf = tt & 1;
      float gk[kSeg];
#pragma unroll
      for (int x = 0; x < kSeg; ++x) gk[x] = own ? dct[bf][row][kSeg * seg + 8 + x] : 0.f;
#pragma unroll
      for (int a = 0; a < CQ; ++a) {
        // tile columns 8 seg .. 8 seg + 23: keys jb - 8 .. jb + 15
        float w[WIN], v[WIN];
        const float4 *sd = reinterpret_cast<const float4 *>(&dct[bf][row + a][kSeg * seg]);
        const float4 *ss = reinterpret_cast<const float4 *>(&st[bf][row + HALO - a][kSeg * seg]);
#pragma unroll
        for (int v4 = 0; v4 < WIN / 4; ++v4) {
          const float4 q4 = sd[v4], s4 = ss[v4];
          w[4 * v4 + 0] = q4.x; w[4 * v4 + 1] = q4.y; w[4 * v4 + 2] = q4.z; w[4 * v4 + 3] = q4.w;
          v[4 * v4 + 0] = s4.x; v[4 * v4 + 1] = s4.y; v[4 * v4 + 2] = s4.z; v[4 * v4 + 3] = s4.w;
        }
#pragma unroll
        for (int t = 0; t < CK; ++t) {
          const float th_at = th[a * CK + t];
          float acc = dth[a * CK + t];
#pragma unroll
          for (int x = 0; x < kSeg; ++x) {
            // out[i][j] += theta[a][t] G[i+a][j+t-c]: key jb + x + t - c = window x + 8 + t - c
            ds[x] = fmaf(th_at, w[x + 8 + t - C], ds[x]);
            // dtheta[a][t] += G[i][j] X[i-a][j-(t-c)]: window x + 8 + c - t
            acc = fmaf(gk[x], v[x + 8 + C - t], acc);
            // MODE 1: A'[i][j] += theta[a][t] A[i-a][j-(t-c)] (the convolution itself)
            if (MODE == 1) ac[x] = fmaf(th_at, v[x + 8 + C - t], ac[x]);
          }
          dth[a * CK + t] = acc;
        }
      }
#pragma unroll
      for (int x = 0; x < kSeg; ++x) {
        ds[x] = jb + x <= i ? ds[x] : 0.f;
        ac[x] = jb + x <= i ? ac[x] : 0.f;
      }
    }
    if (MODE == 0 && jb < p.Wp) {
      __nv_bfloat16 *dSz = q.dS + static_cast<long long>(z) * 2 * p.g.rt * P;
      uint32_t hi[kSeg / 2], lo[kSeg / 2];
#pragma unroll
      for (int x = 0; x < kSeg; x += 2) {
        __nv_bfloat16 h0, l0, h1, l1;
        split_bf16(ds[x], h0, l0);
        split_bf16(ds[x + 1], h1, l1);
        hi[x / 2] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
        lo[x / 2] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
      }
      *reinterpret_cast<uint4 *>(dSz + static_cast<long long>(u) * P + jb) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4 *>(dSz + static_cast<long long>(p.g.rt + u) * P + jb) =
          make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    if (MODE == 1 && work && outr && jb <= i && jb < p.Wp) {
      float *dst = q.dA + (static_cast<long long>(z) * q.out_rows + u) * P + jb;
      reinterpret_cast<float4 *>(dst)[0] = make_float4(ds[0], ds[1], ds[2], ds[3]);
      reinterpret_cast<float4 *>(dst)[1] = make_float4(ds[4], ds[5], ds[6], ds[7]);
      if (own) {
        float *ad = q.Ac + (static_cast<long long>(z) * p.g.no + u) * P + jb;
        reinterpret_cast<float4 *>(ad)[0] = make_float4(ac[0], ac[1], ac[2], ac[3]);
        reinterpret_cast<float4 *>(ad)[1] = make_float4(ac[4], ac[5], ac[6], ac[7]);
      }
    }
    if (work) __syncthreads();  // the buffer is restaged two tiles on
  }
  if (q.dtheta) {
#pragma unroll
    for (int x = 0; x < NT; ++x) {
      float v = dth[x];
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if ((threadIdx.x & 31) == 0 && v != 0.f) atomicAdd(q.dtheta + h * NT + x, v);
    }
  }
}

// The convolution after the softmax: per head group, the gradient at its output
// G_s = Mask_0(sum_h w[h][s] dA''_h) (post mixing; dA''_s otherwise), rows u <->
// query r0 + u, keys up to each row's query (the rest is never read).
template <int CH>
__global__ void __launch_bounds__(kThreadsB) bwd_post_grad_kernel(StripArgs p, float *G) {
  const int G_ = p.H / CH, bg = blockIdx.y, b = bg / G_, g = bg % G_;
  const int u = blockIdx.x * kRows + tile_row(threadIdx.x), seg = tile_seg(threadIdx.x);
  const int i = p.r0 + u, P = p.g.pitch;
  if (u >= p.g.rc || i >= p.L) return;
  float wm[CH * CH];
#pragma unroll
  for (int x = 0; x < CH * CH; ++x) wm[x] = (p.hp == 2 && p.w) ? p.w[g * CH * CH + x] : (x % (CH + 1) == 0);
  const long long z0 = static_cast<long long>(b) * p.H + g * CH;
  for (int jb = kSeg * seg; jb <= i; jb += kKeyTile) {
    float da[CH][kSeg];
#pragma unroll
    for (int h = 0; h < CH; ++h) {
      const float *src = p.D + ((z0 + h) * p.g.rc + u) * P + jb;
      const float4 a = reinterpret_cast<const float4 *>(src)[0], c = reinterpret_cast<const float4 *>(src)[1];
      da[h][0] = a.x; da[h][1] = a.y; da[h][2] = a.z; da[h][3] = a.w;
      da[h][4] = c.x; da[h][5] = c.y; da[h][6] = c.z; da[h][7] = c.w;
    }
#pragma unroll
    for (int s2 = 0; s2 < CH; ++s2) {
      float o[kSeg];
#pragma unroll
      for (int x = 0; x < kSeg; ++x) {
        float v = 0.f;
#pragma unroll
        for (int h = 0; h < CH; ++h) v = fmaf(wm[h * CH + s2], da[h][x], v);
        o[x] = jb + x <= i ? v : 0.f;
      }
      float *dst = G + ((z0 + s2) * p.g.rc + u) * P + jb;
      reinterpret_cast<float4 *>(dst)[0] = make_float4(o[0], o[1], o[2], o[3]);
      reinterpret_cast<float4 *>(dst)[1] = make_float4(o[4], o[5], o[6], o[7]);
    }
  }
}

// The convolution after the softmax, own rows: A''_h = sum_s w[h][s] A'_s (post
// mixing; A'_h otherwise) as hi / lo halves for dV, and the post-mixing dw[h][s] +=
// sum dA''_h A'_s.
template <int CH>
__global__ void __launch_bounds__(kThreadsB) bwd_post_mix_kernel(StripArgs p, const float *Ac) {
  __shared__ float dwr[CH * CH];
  const int G_ = p.H / CH, bg = blockIdx.y, b = bg / G_, g = bg % G_;
  const int u = blockIdx.x * kRows + tile_row(threadIdx.x), seg = tile_seg(threadIdx.x);
  const int i = p.r0 + u, P = p.g.pitch;
  const bool own = u < p.g.no && i < p.L;
  if (threadIdx.x < CH * CH) dwr[threadIdx.x] = 0.f;
  __syncthreads();
  float wm[CH * CH], dwp[CH * CH];
#pragma unroll
  for (int x = 0; x < CH * CH; ++x) {
    wm[x] = (p.hp == 2 && p.w) ? p.w[g * CH * CH + x] : (x % (CH + 1) == 0);
    dwp[x] = 0.f;
  }
  const long long z0 = static_cast<long long>(b) * p.H + g * CH;
  if (own) {
    for (int jb = kSeg * seg; jb <= i; jb += kKeyTile) {
      float ac[CH][kSeg], da[CH][kSeg];
#pragma unroll
      for (int h = 0; h < CH; ++h) {
        const float *sa = Ac + ((z0 + h) * p.g.no + u) * P + jb;
        const float *sd = p.D + ((z0 + h) * p.g.rc + u) * P + jb;
#pragma unroll
        for (int x = 0; x < kSeg; x += 4) {
          const float4 a = *reinterpret_cast<const float4 *>(sa + x), d = *reinterpret_cast<const float4 *>(sd + x);
          ac[h][x] = a.x; ac[h][x + 1] = a.y; ac[h][x + 2] = a.z; ac[h][x + 3] = a.w;
          da[h][x] = d.x; da[h][x + 1] = d.y; da[h][x + 2] = d.z; da[h][x + 3] = d.w;
        }
      }
#pragma unroll
      for (int h = 0; h < CH; ++h) {
        uint32_t hi[kSeg / 2], lo[kSeg / 2];
#pragma unroll
        for (int x = 0; x < kSeg; x += 2) {
          float y[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            float v = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < CH; ++s2) v = fmaf(wm[h * CH + s2], ac[s2][x + e], v);
            y[e] = jb + x + e <= i ? v : 0.f;
          }
          __nv_bfloat16 h0, l0, h1, l1;
          split_bf16(y[0], h0, l0);
          split_bf16(y[1], h1, l1);
          hi[x / 2] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
          lo[x / 2] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
        }
        __nv_bfloat16 *ap = p.Ap + ((z0 + h) * 2 * p.g.rt) * P;
        *reinterpret_cast<uint4 *>(ap + static_cast<long long>(u) * P + jb) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4 *>(ap + static_cast<long long>(p.g.rt + u) * P + jb) =
            make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      if (p.hp == 2) {
#pragma unroll
        for (int h = 0; h < CH; ++h)
#pragma unroll
          for (int s2 = 0; s2 < CH; ++s2)
#pragma unroll
            for (int x = 0; x < kSeg; ++x)
              if (jb + x <= i) dwp[h * CH + s2] = fmaf(da[h][x], ac[s2][x], dwp[h * CH + s2]);
      }
    }
  }
  if (p.hp == 2 && p.dw) {
#pragma unroll
    for (int x = 0; x < CH * CH; ++x) {
      float v = dwp[x];
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if ((threadIdx.x & 31) == 0) atomicAdd(&dwr[x], v);
    }
    __syncthreads();
    if (threadIdx.x < CH * CH) atomicAdd(p.dw + g * CH * CH + threadIdx.x, dwr[threadIdx.x]);
  }
}

// The softmax's backward with the convolution after the softmax: dA from the
// adjoint kernel (rows u <-> query r0 + u), A from the A strip (row u + a_off),
// D = sum_j dA A, dC = A (dA - D) in place of dA (pre mixing: dC'_h = A_h (dA_h -
// D_h) mixed back to the sources, and dw[h][s] += sum dC'_h C_s over the own rows).
template <int CH>
__global__ void __launch_bounds__(kThreadsB) bwd_post_softmax_kernel(StripArgs p, float *dA, int da_rows, int a_off) {
  __shared__ float dwr[CH * CH];
  const int G_ = p.H / CH, bg = blockIdx.y, b = bg / G_, g = bg % G_;
  const int u = blockIdx.x * kRows + tile_row(threadIdx.x), seg = tile_seg(threadIdx.x);
  const int i = p.r0 + u, P = p.g.pitch;
  const bool valid = u < da_rows && i < p.L, own = valid && u < p.g.no;
  if (threadIdx.x < CH * CH) dwr[threadIdx.x] = 0.f;
  __syncthreads();
  float wm[CH * CH], dwp[CH * CH], Dp[CH];
#pragma unroll
  for (int x = 0; x < CH * CH; ++x) {
    wm[x] = (p.hp == 1 && p.w) ? p.w[g * CH * CH + x] : (x % (CH + 1) == 0);
    dwp[x] = 0.f;
  }
#pragma unroll
  for (int h = 0; h < CH; ++h) Dp[h] = 0.f;
  const long long z0 = static_cast<long long>(b) * p.H + g * CH;
  auto load8 = [&](const float *src, float (&o)[kSeg]) {
    const float4 a = reinterpret_cast<const float4 *>(src)[0], c = reinterpret_cast<const float4 *>(src)[1];
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = c.x; o[5] = c.y; o[6] = c.z; o[7] = c.w;
  };
  if (valid) {
    for (int jb = kSeg * seg; jb <= i; jb += kKeyTile) {
#pragma unroll
      for (int h = 0; h < CH; ++h) {
        float a[kSeg], d[kSeg];
        load8(p.A + ((z0 + h) * p.g.rc + u + a_off) * P + jb, a);
        load8(dA + ((z0 + h) * da_rows + u) * P + jb, d);
#pragma unroll
        for (int x = 0; x < kSeg; ++x)
          if (jb + x <= i) Dp[h] = fmaf(d[x], a[x], Dp[h]);
      }
    }
  }
  float Dr[CH];
#pragma unroll
  for (int h = 0; h < CH; ++h) {
    float v = Dp[h];
#pragma unroll
    for (int o : {1, 2, 8, 16}) v += __shfl_xor_sync(0xffffffffu, v, o);
    Dr[h] = v;
  }
  if (valid) {
    for (int jb = kSeg * seg; jb <= i; jb += kKeyTile) {
      float a[CH][kSeg], d[CH][kSeg], dc[CH][kSeg];
#pragma unroll
      for (int h = 0; h < CH; ++h) {
        load8(p.A + ((z0 + h) * p.g.rc + u + a_off) * P + jb, a[h]);
        load8(dA + ((z0 + h) * da_rows + u) * P + jb, d[h]);
      }
      if (p.hp == 1) {
#pragma unroll
        for (int x = 0; x < kSeg; ++x) {
          float dcp[CH];
#pragma unroll
          for (int h = 0; h < CH; ++h) dcp[h] = a[h][x] * (d[h][x] - Dr[h]);
#pragma unroll
          for (int s2 = 0; s2 < CH; ++s2) {
            float v = 0.f;
#pragma unroll
            for (int h = 0; h < CH; ++h) v = fmaf(wm[h * CH + s2], dcp[h], v);
            dc[s2][x] = jb + x <= i ? v : 0.f;
          }
          if (own && jb + x <= i) {
#pragma unroll
            for (int s2 = 0; s2 < CH; ++s2) {
              const float cs = p.Cpre[((z0 + s2) * p.g.rc + u + a_off) * P + jb + x];
#pragma unroll
              for (int h = 0; h < CH; ++h) dwp[h * CH + s2] = fmaf(dcp[h], cs, dwp[h * CH + s2]);
            }
          }
        }
      } else {
#pragma unroll
        for (int h = 0; h < CH; ++h)
#pragma unroll
          for (int x = 0; x < kSeg; ++x) dc[h][x] = jb + x <= i ? a[h][x] * (d[h][x] - Dr[h]) : 0.f;
      }
#pragma unroll
      for (int h = 0; h < CH; ++h) {
        float *dst = dA + ((z0 + h) * da_rows + u) * P + jb;
        reinterpret_cast<float4 *>(dst)[0] = make_float4(dc[h][0], dc[h][1], dc[h][2], dc[h][3]);
        reinterpret_cast<float4 *>(dst)[1] = make_float4(dc[h][4], dc[h][5], dc[h][6], dc[h][7]);
      }
    }
  }
  if (p.hp == 1 && p.dw) {
#pragma unroll
    for (int x = 0; x < CH * CH; ++x) {
      float v = dwp[x];
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if ((threadIdx.x & 31) == 0) atomicAdd(&dwr[x], v);
    }
    __syncthreads();
    if (threadIdx.x < CH * CH) atomicAdd(p.dw + g * CH * CH + threadIdx.x, dwr[threadIdx.x]);
  }
}

int scores_smem(int ch) { return 2 * ch * kStagedRows * kTilePitch * 4; }
int adjoint_smem() { return 2 * 2 * kStagedRows * kTilePitch * 4; }

// Rows of a block (R = block_rows(L)).  Without the convolution after the softmax:
// own rows NO = R - 2 (c_q - 1), C / dC rows NO + c_q - 1.  With it, one more halo
// of c_q - 1 rows on each side: own rows R - 3 (c_q - 1), A rows (and dA'' rows)
// NO + 2 (c_q - 1).
Geo geometry(const BwdArgs &a) {
  Geo g;
  g.halo = a.cq - 1;
  g.c = a.ck / 2;
  g.rt = block_rows(a.L);
  g.no = g.rt - (a.kqp ? 3 : 2) * g.halo;
  g.rc = g.no + (a.kqp ? 2 : 1) * g.halo;
  g.pitch = (a.L + 63) / 64 * 64;
  return g;
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// [B][L][H][d] bf16 with token stride rs: dims (d, H, L, B), the row index at position 2
BgTensor qkv_tensor(const void *base, const BwdArgs &a, long long rs) {
  BgTensor t;
  t.base = base;
  t.dims[0] = a.d; t.dims[1] = a.H; t.dims[2] = a.L; t.dims[3] = a.B;
  t.strides[0] = static_cast<unsigned long long>(a.d) * 2;
  t.strides[1] = static_cast<unsigned long long>(rs) * 2;
  t.strides[2] = static_cast<unsigned long long>(rs) * a.L * 2;
  t.pos_row = 2;
  return t;
}
// a bf16 strip [B][H][rows][pitch]: dims (pitch, rows, H, B), the row index at position 1
BgTensor strip_tensor(const void *base, const BwdArgs &a, int rows, int pitch) {
  BgTensor t;
  t.base = base;
  t.dims[0] = pitch; t.dims[1] = rows; t.dims[2] = a.H; t.dims[3] = a.B;
  t.strides[0] = static_cast<unsigned long long>(pitch) * 2;
  t.strides[1] = static_cast<unsigned long long>(pitch) * rows * 2;
  t.strides[2] = static_cast<unsigned long long>(pitch) * rows * a.H * 2;
  t.pos_row = 1;
  return t;
}

}  // namespace

bool attn_bwd_tc_supported(const BwdArgs &a) {
  return a.dtype == 1 && (a.d == 64 || a.d == 96 || a.d == 128) && a.cq == 6 && a.ck == 11 && a.kq == 1 &&
         (!a.kqp || a.theta_post) && (a.hp == 0 || a.ch == 2) && a.rs % 8 == 0 &&
         (reinterpret_cast<uintptr_t>(a.q) | reinterpret_cast<uintptr_t>(a.k) | reinterpret_cast<uintptr_t>(a.v) |
          reinterpret_cast<uintptr_t>(a.dout)) % 16 == 0 &&
         (reinterpret_cast<uintptr_t>(a.dq) | reinterpret_cast<uintptr_t>(a.dk) | reinterpret_cast<uintptr_t>(a.dv)) %
                 16 == 0;
}

size_t attn_bwd_tc_workspace_bytes(int B, int H, int L, int cq, int hp, int kqp) {
  const size_t Z = static_cast<size_t>(B) * H, P = (static_cast<size_t>(L) + 63) / 64 * 64;
  const size_t halo = static_cast<size_t>(cq - 1), RT = static_cast<size_t>(block_rows(L));
  const size_t no = RT - (kqp ? 3 : 2) * halo, rc = no + (kqp ? 2 : 1) * halo;
  size_t b = up256(Z * RT * P * 4) + 2 * up256(Z * rc * P * 4) + (hp == 1 ? up256(Z * rc * P * 4) : 0) +
             2 * up256(Z * 2 * RT * P * 2);
  // with the convolution after the softmax: its output gradient G, dA (then dC) and A'
  if (kqp) b += up256(Z * rc * P * 4) + up256(Z * (no + halo) * P * 4) + up256(Z * no * P * 4);
  return b;
}

cudaError_t launch_attn_bwd_tc(const BwdArgs &a, void *ws) {
  const Geo g = geometry(a);
  const size_t Z = static_cast<size_t>(a.B) * a.H, P = g.pitch;
  const int post = a.kqp ? 1 : 0, ndc = g.no + g.halo;  // rows of dA / dC with post
  char *w = static_cast<char *>(ws);
  float *S = reinterpret_cast<float *>(w);
  w += up256(Z * g.rt * P * 4);
  float *A = reinterpret_cast<float *>(w);
  w += up256(Z * g.rc * P * 4);
  float *D = reinterpret_cast<float *>(w);
  w += up256(Z * g.rc * P * 4);
  float *Cpre = nullptr;
  if (a.hp == 1) {
    Cpre = reinterpret_cast<float *>(w);
    w += up256(Z * g.rc * P * 4);
  }
  __nv_bfloat16 *dS = reinterpret_cast<__nv_bfloat16 *>(w);
  w += up256(Z * 2 * g.rt * P * 2);
  __nv_bfloat16 *Ap = reinterpret_cast<__nv_bfloat16 *>(w);
  w += up256(Z * 2 * g.rt * P * 2);
  float *Gp = nullptr, *dAp = nullptr, *Ac = nullptr;
  if (post) {
    Gp = reinterpret_cast<float *>(w);
    w += up256(Z * g.rc * P * 4);
    dAp = reinterpret_cast<float *>(w);
    w += up256(Z * ndc * P * 4);
    Ac = reinterpret_cast<float *>(w);
  }

  cudaStream_t st = a.stream;
  const size_t n = static_cast<size_t>(a.B) * a.L * a.H * a.d;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(bwd_scores_kernel<6, 11, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                scores_smem(2))) != cudaSuccess ||
      (e = cudaFuncSetAttribute(bwd_scores_kernel<6, 11, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                scores_smem(1))) != cudaSuccess ||
      (e = cudaFuncSetAttribute(bwd_adjoint_kernel<6, 11, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                adjoint_smem())) != cudaSuccess ||
      (e = cudaFuncSetAttribute(bwd_adjoint_kernel<6, 11, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                adjoint_smem())) != cudaSuccess)
    return e;
  if ((e = cudaMemsetAsync(a.dq, 0, n * 4, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(a.dk, 0, n * 4, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(a.dv, 0, n * 4, st)) != cudaSuccess) return e;
  const size_t nth = static_cast<size_t>(a.H) * a.cq * a.ck * 4;
  if (a.dtheta && (e = cudaMemsetAsync(a.dtheta, 0, nth, st)) != cudaSuccess) return e;
  if (post && a.dtheta_post && (e = cudaMemsetAsync(a.dtheta_post, 0, nth, st)) != cudaSuccess) return e;
  if (a.hp && a.dw && (e = cudaMemsetAsync(a.dw, 0, static_cast<size_t>(a.H) * a.ch * 4, st)) != cudaSuccess)
    return e;
  // A'' is written for the own rows up to each row's query only: the rest stays zero
  if ((e = cudaMemsetAsync(Ap, 0, Z * 2 * g.rt * P * 2, st)) != cudaSuccess) return e;

  const BgTensor tq = qkv_tensor(a.q, a, a.rs), tk = qkv_tensor(a.k, a, a.rs), tv = qkv_tensor(a.v, a, a.rs);
  const BgTensor tdo = qkv_tensor(a.dout, a, static_cast<long long>(a.H) * a.d);
  const BgTensor tdS = strip_tensor(dS, a, 2 * g.rt, g.pitch), tAp = strip_tensor(Ap, a, 2 * g.rt, g.pitch);
  const long long HD = static_cast<long long>(a.H) * a.d, LHD = HD * a.L;
  const int ch = a.hp ? a.ch : 1, G = a.H / ch;
  unsigned *err = a.err;

  StripArgs sp;
  sp.B = a.B; sp.H = a.H; sp.L = a.L; sp.ch = ch; sp.hp = a.hp;
  sp.g = g;
  sp.theta = a.theta; sp.w = a.hp ? a.w : nullptr;
  sp.S = S; sp.Cpre = Cpre; sp.A = A; sp.D = D; sp.dS = dS; sp.Ap = Ap;
  sp.dtheta = a.dtheta; sp.dw = a.hp ? a.dw : nullptr;
  sp.post = post;

  auto K_major = [](int pos_row, int off_mn, int off_k) { return BgOperand{0, pos_row, off_mn, off_k, 0, 0}; };
  auto MN_major = [](int pos_row, int off_mn, int off_k) { return BgOperand{1, pos_row, off_mn, off_k, 0, 0}; };
  auto periodic = [](BgOperand o, int period, int shift) {
    o.k_period = period;
    o.period_shift = shift;
    return o;
  };
  auto check = [&]() { return cudaGetLastError(); };
  const int s_lead = (post ? 2 : 1) * g.halo;  // S strip row 0 is query r0 - s_lead
  for (int r0 = 0; r0 < a.L; r0 += g.no) {
    // keys 0 .. W-1: up to the last row of the block's maps
    const int W = std::min(a.L, r0 + g.rc), Wp = (W + 63) / 64 * 64;
    sp.r0 = r0; sp.W = W; sp.Wp = Wp;
    // 1. S strip = s Q K^T: rows r0 - s_lead .. r0 - s_lead + R - 1, keys 0 .. W-1
    BgArgs ga = {};
    ga.Z = static_cast<int>(Z); ga.H = a.H; ga.err = err;
    ga.M = g.rt; ga.N = W; ga.K = a.d; ga.alpha = a.scale; ga.accumulate = 0;
    ga.C = S; ga.sm = g.pitch; ga.sh = static_cast<long long>(g.rt) * g.pitch; ga.sb = ga.sh * a.H;
    ga.a = K_major(2, r0 - s_lead, 0); ga.b = K_major(2, 0, 0);
    if ((e = launch_gemm_batched(tq, tk, ga, st)) != cudaSuccess) return e;
    // 2. dA'' strip = dO V^T: rows r0 .. r0 + rc - 1
    ga.M = g.rc; ga.alpha = 1.f;
    ga.C = D; ga.sh = static_cast<long long>(g.rc) * g.pitch; ga.sb = ga.sh * a.H;
    ga.a = K_major(2, r0, 0); ga.b = K_major(2, 0, 0);
    if ((e = launch_gemm_batched(tdo, tv, ga, st)) != cudaSuccess) return e;
    // 3. convolution, mixing, softmax (rows r0 .. without the convolution after the
    //    softmax, with its backward fused; with it, rows r0 - halo .., the weights only)
    const dim3 grid_g((g.rc + kRows - 1) / kRows, a.B * G);
    StripArgs s3 = sp;
    if (post) s3.r0 = r0 - g.halo;
    if (ch == 2)
      bwd_scores_kernel<6, 11, 2><<<grid_g, kThreadsB, scores_smem(2), st>>>(s3);
    else
      bwd_scores_kernel<6, 11, 1><<<grid_g, kThreadsB, scores_smem(1), st>>>(s3);
    if ((e = check()) != cudaSuccess) return e;
    const dim3 grid_h(g.rt / kRows, static_cast<unsigned>(Z));
    if (post) {
      // 3a. the gradient at the post-softmax convolution's output, G = Mask_0(mix back dA'')
      if (ch == 2)
        bwd_post_grad_kernel<2><<<grid_g, kThreadsB, 0, st>>>(sp, Gp);
      else
        bwd_post_grad_kernel<1><<<grid_g, kThreadsB, 0, st>>>(sp, Gp);
      if ((e = check()) != cudaSuccess) return e;
      // 3b. its adjoint dA (rows r0 .. r0 + no + halo - 1), dtheta_post, and A' of the own rows
      AdjArgs q1 = {};
      q1.G = Gp; q1.g_rows = g.rc;
      q1.X = A; q1.x_rows = g.rc; q1.x_base = r0 - g.halo;
      q1.theta = a.theta_post; q1.dtheta = a.dtheta_post;
      q1.out_rows = ndc; q1.dA = dAp; q1.Ac = Ac;
      bwd_adjoint_kernel<6, 11, 1><<<grid_h, kThreadsB, adjoint_smem(), st>>>(sp, q1);
      if ((e = check()) != cudaSuccess) return e;
      // 3c. A'' = mix(A') for dV, and the post-mixing dw
      if (ch == 2)
        bwd_post_mix_kernel<2><<<grid_g, kThreadsB, 0, st>>>(sp, Ac);
      else
        bwd_post_mix_kernel<1><<<grid_g, kThreadsB, 0, st>>>(sp, Ac);
      if ((e = check()) != cudaSuccess) return e;
      // 3d. the softmax's backward: dC in place of dA (pre mixing: mixed back, dw)
      if (ch == 2)
        bwd_post_softmax_kernel<2><<<grid_g, kThreadsB, 0, st>>>(sp, dAp, ndc, g.halo);
      else
        bwd_post_softmax_kernel<1><<<grid_g, kThreadsB, 0, st>>>(sp, dAp, ndc, g.halo);
      if ((e = check()) != cudaSuccess) return e;
    }
    // 4. dS (hi / lo), dtheta: the adjoint of the convolution before the softmax
    AdjArgs q0 = {};
    q0.G = post ? dAp : D; q0.g_rows = post ? ndc : g.rc;
    q0.X = S; q0.x_rows = g.rt; q0.x_base = r0 - s_lead;
    q0.theta = a.theta; q0.dtheta = a.dtheta; q0.dS = dS;
    bwd_adjoint_kernel<6, 11, 0><<<grid_h, kThreadsB, adjoint_smem(), st>>>(sp, q0);
    if ((e = check()) != cudaSuccess) return e;
    // 5. dQ rows r0 .. r0 + no - 1 = s dS K: K runs over the keys twice, the hi
    //    rows of dS against K, then its lo rows (R further) against K again
    const int own = std::min(g.no, a.L - r0);
    BgArgs gq = {};
    gq.Z = static_cast<int>(Z); gq.H = a.H; gq.err = err;
    // (added into the zeroed dq: the GEMM may split K in two)
    gq.M = own; gq.N = a.d; gq.K = 2 * Wp; gq.alpha = a.scale; gq.accumulate = 1; gq.split_ok = 1;
    gq.C = a.dq + static_cast<long long>(r0) * HD; gq.sm = HD; gq.sh = a.d; gq.sb = LHD;
    gq.a = periodic(K_major(1, 0, 0), Wp, g.rt);
    gq.b = periodic(MN_major(2, 0, 0), Wp, 0);
    if ((e = launch_gemm_batched(tdS, tk, gq, st)) != cudaSuccess) return e;
    //    dK += s dS^T Q and dV += A''^T dO over the block's rows (keys 0 .. W-1): K runs
    //    over the rows of the hi and lo halves, the block's query rows twice
    BgArgs gk = {};
    gk.Z = static_cast<int>(Z); gk.H = a.H; gk.err = err;
    gk.M = W; gk.N = a.d; gk.K = 2 * g.rt; gk.accumulate = 1;
    gk.sm = HD; gk.sh = a.d; gk.sb = LHD;
    gk.a = MN_major(1, 0, 0);
    gk.b = periodic(MN_major(2, 0, r0), g.rt, 0);
    gk.alpha = a.scale; gk.C = a.dk;
    if ((e = launch_gemm_batched(tdS, tq, gk, st)) != cudaSuccess) return e;
    gk.alpha = 1.f; gk.C = a.dv;
    if ((e = launch_gemm_batched(tAp, tdo, gk, st)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace mta
