// kq_prep.cu -- prepass of the contraction form of the key-query convolution.
//
// "Multi-Token Attention | Summary" (greeksharifa), section 3.1: the pre-softmax
// key-query convolution C = Conv2d_theta(Mask_0(Q K^T / sqrt(d))).  Away from the
// diagonal (i - j >= W = (c_q-1) + c, c = c_k/2) no tap reads a masked logit and
// the convolution is a contraction:
//   C[i][j] = s * sum_a q[i-a] . Kt_a[j],   Kt_a[j] = sum_t theta[a][t] k[j-(t-c)],
// the c_q shifted query rows against c_q per-row-convolved key rows (contraction
// length c_q*d).  In the band 0 <= i - j < W the attention kernel evaluates the
// convolution tap by tap from the past dot products
//   Vp[i][m] = q[i] . k[i-m],   m = 0 .. M-1,   M = (c_q-1) + 2c,
// which covers every unmasked tap of the band (m = i-a - key >= 0).
//
// This kernel writes, per (batch, head, tile of 128 keys):
//   Kt  [B][H][c_q][L][d] fp16: Kt_a[j] * 2^e_j, e_j a power-of-2 exponent per key
//       row chosen from max|k| over the rows j-c .. j+c that Kt_a[j] reads (so no
//       value exceeds 2^14 and small keys keep fp16's relative precision);
//   fac [B][H][L] fp32: 2^-e_j;
//   Vp  [B][H][L][M] fp32: raw past dot products (no scale).
// Every value written for key or query j depends on inputs at positions <= j + c
// only, and Kt_a[j] is used only for queries i >= j + W > j + c: the path stays
// exactly causal.  One CTA per (key tile, head, batch); the key rows with their
// halo are staged in shared memory as fp32.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"

namespace mta {
namespace {

constexpr int kPrepThreads = 256;
constexpr int kTile = 128;
constexpr int kRun = 16;  // consecutive keys one thread convolves from a register window

template <int D, int CQ, int CK>
struct PrepGeo {
  static constexpr int C = CK / 2;
  static constexpr int M = (CQ - 1) + 2 * C;          // past dot products per query
  static constexpr int LO = M - 1;                    // staged rows before the tile
  static constexpr int ROWS = kTile + LO + C;         // keys j0-LO .. j0+kTile-1+C
  static constexpr int SMEM = ROWS * D * 4;
};

__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }  // |e| <= 126

template <int D, int CQ, int CK>
__global__ void __launch_bounds__(kPrepThreads) kq_prep_kernel(KqPrepArgs p) {
  using G = PrepGeo<D, CQ, CK>;
  extern __shared__ float ks[];  // [ROWS][D] fp32, row r = key j0 - LO + r
  __shared__ float rmax[G::ROWS];
  __shared__ int es[kTile];
  __shared__ float th[CQ * CK];
  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int L = p.L, j0 = tile * kTile;
  const long long bh = static_cast<long long>(b) * p.H + h;
  const __nv_bfloat16 *kb = static_cast<const __nv_bfloat16 *>(p.k);
  const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(p.q);

  for (int i = tid; i < CQ * CK; i += kPrepThreads) th[i] = p.theta[static_cast<long long>(h) * CQ * CK + i];
  for (int i = tid; i < G::ROWS; i += kPrepThreads) rmax[i] = 0.f;
  __syncthreads();
  // stage key rows (zero outside [0, L)) and their max |k|
  for (int i = tid; i < G::ROWS * (D / 8); i += kPrepThreads) {
    const int r = i / (D / 8), e8 = (i % (D / 8)) * 8, key = j0 - G::LO + r;
    float v[8];
    if (key >= 0 && key < L) {
      const uint4 raw = *reinterpret_cast<const uint4 *>(kb + (static_cast<long long>(b) * L + key) * p.rs +
                                                         static_cast<long long>(h) * D + e8);
      const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
      for (int u = 0; u < 4; ++u) { v[2 * u] = __low2float(p2[u]); v[2 * u + 1] = __high2float(p2[u]); }
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = 0.f;
    }
    float m = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      ks[r * D + e8 + u] = v[u];
      m = fmaxf(m, fabsf(v[u]));
    }
    atomicMax(reinterpret_cast<int *>(rmax + r), __float_as_int(m));  // non-negative floats order as ints
  }
  __syncthreads();
  // per-key exponent: bound on |Kt_a[j]| = max_a sum_t |theta[a][t]| * max |k| over rows j-c .. j+c
  if (tid < kTile) {
    float t1 = 0.f;
#pragma unroll
    for (int a = 0; a < CQ; ++a) {
      float s = 0.f;
#pragma unroll
      for (int t = 0; t < CK; ++t) s += fabsf(th[a * CK + t]);
      t1 = fmaxf(t1, s);
    }
    float wm = 0.f;
#pragma unroll
    for (int t = -G::C; t <= G::C; ++t) wm = fmaxf(wm, rmax[tid + G::LO + t]);
    const float bound = wm * t1;
    int e = 0;
    if (bound > 0.f) e = max(-60, min(60, static_cast<int>(floorf(log2f(16384.f / bound)))));
    es[tid] = e;
    if (j0 + tid < L) p.fac[bh * L + j0 + tid] = pow2i(-e);
  }
  __syncthreads();

  // Kt_a[j] = sum_t theta[a][t] k[j - (t - c)]: each work item is one pair of
  // channels x kRun consecutive keys, convolved from a register window of rows.
  __half *kt = static_cast<__half *>(p.kt);
  constexpr int NPAIR = D / 2, NRUN = kTile / kRun;
  for (int item = tid; item < NPAIR * NRUN; item += kPrepThreads) {
    const int e2 = (item % NPAIR) * 2, jr = (item / NPAIR) * kRun;
    float2 win[kRun + 2 * G::C];  // keys j0+jr-c .. j0+jr+kRun-1+c
#pragma unroll
    for (int w = 0; w < kRun + 2 * G::C; ++w)
      win[w] = *reinterpret_cast<const float2 *>(ks + (jr + w + G::LO - G::C) * D + e2);
#pragma unroll
    for (int a = 0; a < CQ; ++a) {
      float ta[CK];
#pragma unroll
      for (int t = 0; t < CK; ++t) ta[t] = th[a * CK + t];
#pragma unroll
      for (int u = 0; u < kRun; ++u) {
        const int key = j0 + jr + u;
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int t = 0; t < CK; ++t) {  // key j - (t - c) is window entry u + 2c - t
          s0 = fmaf(ta[t], win[u + 2 * G::C - t].x, s0);
          s1 = fmaf(ta[t], win[u + 2 * G::C - t].y, s1);
        }
        if (key < L) {
          const float sc = pow2i(es[jr + u]);
          const long long o = ((bh * CQ + a) * L + key) * D + e2;
          *reinterpret_cast<__half2 *>(kt + o) = __floats2half2_rn(s0 * sc, s1 * sc);
        }
      }
    }
  }

  // Vp[i][m] = q[i] . k[i-m]: one warp per query row, channels spread over lanes
  constexpr int PER_LANE = D / 32;
  const int warp = tid >> 5, lane = tid & 31;
  for (int r = warp; r < kTile; r += kPrepThreads / 32) {
    const int qi = j0 + r;
    if (qi >= L) break;
    const __nv_bfloat16 *qr = qb + (static_cast<long long>(b) * L + qi) * p.rs + static_cast<long long>(h) * D;
    float qv[PER_LANE];
#pragma unroll
    for (int u = 0; u < PER_LANE; ++u) qv[u] = __bfloat162float(qr[lane * PER_LANE + u]);
    float mine = 0.f;
#pragma unroll
    for (int m = 0; m < G::M; ++m) {
      const float *kr = ks + (r + G::LO - m) * D + lane * PER_LANE;
      float s = 0.f;
#pragma unroll
      for (int u = 0; u < PER_LANE; ++u) s = fmaf(qv[u], kr[u], s);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == m) mine = s;
    }
    if (lane < G::M) p.vp[(bh * L + qi) * G::M + lane] = mine;
  }
}

template <int D, int CQ, int CK>
cudaError_t launch_prep_one(const KqPrepArgs &p, cudaStream_t stream) {
  using G = PrepGeo<D, CQ, CK>;
  auto kern = kq_prep_kernel<D, CQ, CK>;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<dim3(p.n_tiles, p.H, p.B), kPrepThreads, G::SMEM, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_kq_prep(const KqPrepArgs &p, cudaStream_t stream) {
  if (p.cq != 6 || p.ck != 11 || p.M != PrepGeo<128, 6, 11>::M) return cudaErrorInvalidValue;
  return p.d == 128 ? launch_prep_one<128, 6, 11>(p, stream) : launch_prep_one<64, 6, 11>(p, stream);
}

}  // namespace mta
