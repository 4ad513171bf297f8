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
//   Kt  fp16, every value Kt_a[j] * 2^e_j, e_j a power-of-2 exponent per key row
//       chosen from max|k| over the rows j-c .. j+c that Kt_a[j] reads (so no value
//       exceeds 2^14 and small keys keep fp16's relative precision); laid out as
//       [B][H][c_q][L][d] when d is a multiple of 64, else as [B][H][c_q*d/64][L][64]:
//       element kappa = a*d + e of key j's contraction operand in chunk kappa/64 at
//       column kappa%64, so that a 64-element box of 128 keys is contiguous;
//   fac [B][H][Lpad] fp32: s * log2(e) * 2^-e_j (the attention kernel's column
//       factor; 0 for the padding keys L <= j < Lpad, Lpad = L rounded up to 128);
//   Vp  [B][H][L][M] fp32: raw past dot products (no scale); with the exact causal
//       indicator shifted by c_q-1: Vp[i][m] = q[i] . k[i-m+(c_q-1)], so that the
//       band can also read keys up to c_q-1 after a shifted query.
// Every value written for key or query j depends on inputs at positions <= j + c
// only, and Kt_a[j] is used only for queries i >= j + W > j + c: the path stays
// exactly causal.  One CTA per (key tile, head, batch); the key rows with their
// halo are staged in shared memory as bf16, and the convolution runs in packed
// fp32 FMAs on channel pairs.  Four CTAs per SM (64 registers a thread): 78.9
// against 83.8 us with three at B = 4, H = 16, L = 2048, d = 128.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

#include <type_traits>

#include "internal.h"
#include "ptx.cuh"

namespace mta {
namespace {

constexpr int kPrepThreads = 256;
constexpr int kTile = 128;
constexpr int kRun = 8;   // consecutive keys one thread convolves from a register window

template <int D, int CQ, int CK, bool EXACT>
struct PrepGeo {
  static constexpr int C = CK / 2;
  static constexpr int M = (CQ - 1) + 2 * C;          // dot products per query
  static constexpr int OFF = EXACT ? CQ - 1 : 0;      // Vp[i][m] = q[i] . k[i-m+OFF]
  static constexpr int LO = M - 1;                    // staged rows before the tile
  // keys j0-LO .. : the Kt window reaches kTile-1+C past j0, a warp's 32-key tile of
  // dot products 16*7+31+OFF-LO
  static constexpr int ROWS = (kTile + LO + C) > (16 * 7 + 32 + OFF) ? (kTile + LO + C) : (16 * 7 + 32 + OFF);
  static constexpr int KSTR = D + 8;                  // staged row stride (bf16): conflict-free fragments
  static constexpr int SMEM = ROWS * KSTR * 2;
  static_assert(M - 1 + 16 <= 32, "past dot products of a 16-row block span 32 keys");
};

// D[16x8] += A[16x16] * B[16x8], bf16 inputs, fp32 accumulate (warp-wide).
__device__ __forceinline__ void mma_m16n8k16_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                                  uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// two bf16 values (low half = first) as floats
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t v) {
  return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }  // |e| <= 126

// c + a * b on a pair of floats with one packed instruction (each lane rounds as fmaf)
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 r;
  asm("{\n\t.reg .b64 pa, pb, pc, pd;\n\t"
      "mov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\tmov.b64 pc, {%6, %7};\n\t"
      "fma.rn.f32x2 pd, pa, pb, pc;\n\tmov.b64 {%0, %1}, pd;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}

template <int D, int CQ, int CK, bool EXACT>
__global__ void __launch_bounds__(kPrepThreads, 4) kq_prep_kernel(KqPrepArgs p) {
  using G = PrepGeo<D, CQ, CK, EXACT>;
  extern __shared__ uint32_t ks[];  // [ROWS][KSTR/2] bf16 pairs, row r = key j0 - LO + r
  __shared__ float rmax[G::ROWS];
  __shared__ int es[kTile];
  __shared__ float th[CQ * CK];
  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int L = p.L, j0 = tile * kTile;
  const long long bh = static_cast<long long>(b) * p.H + h;
  const __nv_bfloat16 *kb = static_cast<const __nv_bfloat16 *>(p.k);
  // the attention kernel (launched as this grid's programmatic dependent) may start
  // its prologue once every CTA of this grid is running; it waits for this grid's
  // completion before it reads anything written here
  pdl_launch_dependents();
  const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(p.q);

  if (p.zero && tile == 0 && h == 0 && b == 0)  // counters the attention kernel starts from 0
    for (int i = tid; i < p.n_zero; i += kPrepThreads) p.zero[i] = 0u;
  for (int i = tid; i < CQ * CK; i += kPrepThreads) th[i] = p.theta[static_cast<long long>(h) * CQ * CK + i];
  for (int i = tid; i < G::ROWS; i += kPrepThreads) rmax[i] = 0.f;
  __syncthreads();
  // stage key rows as bf16 (zero outside [0, L)) and their max |k|
  for (int i = tid; i < G::ROWS * (D / 8); i += kPrepThreads) {
    const int r = i / (D / 8), e8 = (i % (D / 8)) * 8, key = j0 - G::LO + r;
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    if (key >= 0 && key < L)
      raw = *reinterpret_cast<const uint4 *>(kb + (static_cast<long long>(b) * L + key) * p.rs +
                                             static_cast<long long>(h) * D + e8);
    *reinterpret_cast<uint4 *>(ks + (r * G::KSTR + e8) / 2) = raw;
    const uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
    float m = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = bf16x2_to_float2(wds[u]);
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
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
    p.fac[bh * p.lpad + j0 + tid] = j0 + tid < L ? pow2i(-e) * p.scale_log2 : 0.f;
  }
  __syncthreads();

  // Kt_a[j] = sum_t theta[a][t] k[j - (t - c)]: each work item is one pair of
  // channels x kRun consecutive keys, convolved from a register window of rows.
  __half *kt = static_cast<__half *>(p.kt);
  constexpr int NCHK = CQ * D / 64;  // 64-element chunks of a key's contraction operand
  constexpr int NPAIR = D / 2, NRUN = kTile / kRun;
  // d a multiple of 64: rows [c_q][L][d] (a 64-element chunk = 64 channels of one tap
  // row); else chunk-major [c_q*d/64][L][64]
  constexpr bool ROWS = D % 64 == 0;
  constexpr int KSTEP = ROWS ? D : 64;  // elements between consecutive keys
  const long long LD = static_cast<long long>(L) * D;  // elements between the Kt_a of one head (rows)
  for (int item = tid; item < NPAIR * NRUN; item += kPrepThreads) {
    const int e2 = (item % NPAIR) * 2, jr = (item / NPAIR) * kRun;
    if (j0 + jr >= L) continue;
    const int nkeys = min(kRun, L - (j0 + jr));
    float2 win[kRun + 2 * G::C];  // keys j0+jr-c .. j0+jr+kRun-1+c
#pragma unroll
    for (int w = 0; w < kRun + 2 * G::C; ++w)
      win[w] = bf16x2_to_float2(ks[((jr + w + G::LO - G::C) * G::KSTR + e2) / 2]);
    float scu[kRun];
#pragma unroll
    for (int u = 0; u < kRun; ++u) scu[u] = pow2i(es[jr + u]);
    __half *o0 = ROWS ? kt + (bh * CQ * L + j0 + jr) * D + e2 : kt + (bh * NCHK * L + j0 + jr) * 64;
#pragma unroll
    for (int a = 0; a < CQ; ++a) {
      // kRun x 2 independent accumulators; taps in the outer loop (no dependent chains)
      float2 acc[kRun];
#pragma unroll
      for (int u = 0; u < kRun; ++u) acc[u] = make_float2(0.f, 0.f);
#pragma unroll
      for (int t = 0; t < CK; ++t) {
        const float2 ta = make_float2(th[a * CK + t], th[a * CK + t]);
#pragma unroll
        for (int u = 0; u < kRun; ++u)  // key j - (t - c) is window entry u + 2c - t
          acc[u] = fma2(ta, win[u + 2 * G::C - t], acc[u]);
      }
      __half *oa;
      if constexpr (ROWS) {
        oa = o0 + a * LD;
      } else {
        const int kap = a * D + e2;  // contraction element of channel pair e2 in tap row a
        oa = o0 + static_cast<long long>(kap / 64) * L * 64 + kap % 64;
      }
#pragma unroll
      for (int u = 0; u < kRun; ++u)
        if (nkeys == kRun || u < nkeys)
          *reinterpret_cast<__half2 *>(oa + u * KSTEP) = __floats2half2_rn(acc[u].x * scu[u], acc[u].y * scu[u]);
    }
  }

  // Vp[i][m] = q[i] . k[i-m+OFF]: per warp a block of 16 query rows i0 .. i0+15
  // against the 32 keys i0-(M-1)+OFF .. i0+32-M+OFF (a 16x32 tile of Q K^T on the
  // tensor cores, exact products of bf16 values, fp32 sums), of which m < M is kept.
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, tq = lane & 3;
  const int i0 = 16 * warp;                 // local query row of the block
  const int krow0 = i0 + G::OFF;            // staged row of key j0+i0-(M-1)+OFF (LO = M-1)
  float acc[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[nt][u] = 0.f;
  const uint32_t *q32[2];
  bool qok[2];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int qi = j0 + i0 + g + 8 * hh;
    qok[hh] = qi < L;
    q32[hh] = reinterpret_cast<const uint32_t *>(qb + (static_cast<long long>(b) * L + (qok[hh] ? qi : 0)) * p.rs +
                                                 static_cast<long long>(h) * D);
  }
#pragma unroll
  for (int kc = 0; kc < D / 16; ++kc) {
    const int c0 = kc * 16 + 2 * tq;
    uint32_t a[4];
    a[0] = qok[0] ? q32[0][c0 / 2] : 0u;
    a[1] = qok[1] ? q32[1][c0 / 2] : 0u;
    a[2] = qok[0] ? q32[0][c0 / 2 + 4] : 0u;
    a[3] = qok[1] ? q32[1][c0 / 2 + 4] : 0u;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const uint32_t *kr = ks + ((krow0 + 8 * nt + g) * G::KSTR + c0) / 2;
      mma_m16n8k16_bf16(acc[nt], a, kr[0], kr[4]);
    }
  }
  // acc[nt][u]: row i0 + g + 8*(u/2), key column kk = 8*nt + 2*tq + (u&1); m = row - key
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int il = g + 8 * (u >> 1), kk = 8 * nt + 2 * tq + (u & 1);
      const int m = il + (G::M - 1) - kk, qi = j0 + i0 + il;
      if (m >= 0 && m < G::M && qi < L) p.vp[(bh * L + qi) * G::M + m] = acc[nt][u];
    }
}

template <int D, int CQ, int CK, bool EXACT>
cudaError_t launch_prep_one(const KqPrepArgs &p, cudaStream_t stream) {
  using G = PrepGeo<D, CQ, CK, EXACT>;
  auto kern = kq_prep_kernel<D, CQ, CK, EXACT>;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<dim3(p.n_tiles, p.H, p.B), kPrepThreads, G::SMEM, stream>>>(p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Values convolved by the post-softmax kernels.  Section 3.1's convolution after
// the softmax, A'[i][j] = sum_a sum_t theta_post[a][t] A[i-a][j-(t-c)], moves onto
// the values away from the diagonal:
//   sum_j A'[i][j] v[j] = sum_a sum_j' A[i-a][j'] Vt_a[j'],  Vt_a[j'] = sum_t theta_post[a][t] v[j'+t-c],
// so the attention kernel multiplies row-shifted weights by Vt_a on the tensor
// cores.  One CTA per (key tile, source head, batch); the value rows with their
// +-c halo are staged as bf16, and each thread convolves a channel pair over
// kRun consecutive keys from a register window.
template <int D, int CQ, int CK, int NVH>
__global__ void __launch_bounds__(kPrepThreads, 3) vt_prep_kernel(VtPrepArgs p) {
  constexpr int C = CK / 2, ROWS = kTile + 2 * C, VSTR = D + 8;
  extern __shared__ uint32_t vs[];  // [ROWS][VSTR/2] bf16 pairs, row r = key j0 - C + r
  __shared__ float th[CQ * CK];
  const int tile = blockIdx.x, s = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int L = p.L, j0 = tile * kTile;
  pdl_launch_dependents();  // as in kq_prep_kernel
  const __nv_bfloat16 *vb = static_cast<const __nv_bfloat16 *>(p.v);
  __nv_bfloat16 *vt = static_cast<__nv_bfloat16 *>(p.vt);
  for (int i = tid; i < CQ * CK; i += kPrepThreads) th[i] = p.theta_post[static_cast<long long>(s) * CQ * CK + i];
  constexpr int NPAIR = D / 2, NRUN = kTile / kRun;
#pragma unroll 1
  for (int hd = 0; hd < NVH; ++hd) {
    const int hv = NVH == 2 ? (s & ~1) + hd : s;
    __syncthreads();  // the previous head's window is consumed (and th is loaded)
    for (int i = tid; i < ROWS * (D / 8); i += kPrepThreads) {
      const int r = i / (D / 8), e8 = (i % (D / 8)) * 8, key = j0 - C + r;
      uint4 raw = make_uint4(0u, 0u, 0u, 0u);
      if (key >= 0 && key < L)
        raw = *reinterpret_cast<const uint4 *>(vb + (static_cast<long long>(b) * L + key) * p.rs +
                                               static_cast<long long>(hv) * D + e8);
      *reinterpret_cast<uint4 *>(vs + (r * VSTR + e8) / 2) = raw;
    }
    __syncthreads();
    const long long z0 = ((static_cast<long long>(b) * p.H + s) * NVH + hd) * CQ;
    for (int item = tid; item < NPAIR * NRUN; item += kPrepThreads) {
      const int e2 = (item % NPAIR) * 2, jr = (item / NPAIR) * kRun;
      if (j0 + jr >= L) continue;
      const int nkeys = min(kRun, L - (j0 + jr));
      float2 win[kRun + 2 * C];  // keys j0+jr-c .. j0+jr+kRun-1+c
#pragma unroll
      for (int w = 0; w < kRun + 2 * C; ++w) win[w] = bf16x2_to_float2(vs[((jr + w) * VSTR + e2) / 2]);
#pragma unroll
      for (int a = 0; a < CQ; ++a) {
        float2 acc[kRun];
#pragma unroll
        for (int u = 0; u < kRun; ++u) acc[u] = make_float2(0.f, 0.f);
#pragma unroll
        for (int t = 0; t < CK; ++t) {
          const float2 ta = make_float2(th[a * CK + t], th[a * CK + t]);
#pragma unroll
          for (int u = 0; u < kRun; ++u)  // value j + (t - c) is window entry u + t
            acc[u] = fma2(ta, win[u + t], acc[u]);
        }
        __nv_bfloat16 *oa = vt + ((z0 + a) * L + j0 + jr) * D + e2;
#pragma unroll
        for (int u = 0; u < kRun; ++u)
          if (nkeys == kRun || u < nkeys)
            *reinterpret_cast<__nv_bfloat162 *>(oa + u * D) = __floats2bfloat162_rn(acc[u].x, acc[u].y);
      }
    }
  }
}

template <int D, int NVH>
cudaError_t launch_vt_one(const VtPrepArgs &p, cudaStream_t stream) {
  constexpr int SMEM = (kTile + 2 * (11 / 2)) * (D + 8) * 2;
  auto kern = vt_prep_kernel<D, 6, 11, NVH>;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  kern<<<dim3(p.n_tiles, p.H, p.B), kPrepThreads, SMEM, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_vt_prep(const VtPrepArgs &p, cudaStream_t stream) {
  if (p.cq != 6 || p.ck != 11 || (p.nvh != 1 && p.nvh != 2)) return cudaErrorInvalidValue;
  if (p.d == 128) return p.nvh == 2 ? launch_vt_one<128, 2>(p, stream) : launch_vt_one<128, 1>(p, stream);
  if (p.d == 96) return p.nvh == 2 ? launch_vt_one<96, 2>(p, stream) : launch_vt_one<96, 1>(p, stream);
  if (p.d == 64) return p.nvh == 2 ? launch_vt_one<64, 2>(p, stream) : launch_vt_one<64, 1>(p, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_kq_prep(const KqPrepArgs &p, cudaStream_t stream) {
  if (p.cq != 6 || p.ck != 11 || p.M != PrepGeo<128, 6, 11, false>::M) return cudaErrorInvalidValue;
  auto go = [&](auto d_tag) -> cudaError_t {
    constexpr int DD = decltype(d_tag)::value;
    return p.exact ? launch_prep_one<DD, 6, 11, true>(p, stream) : launch_prep_one<DD, 6, 11, false>(p, stream);
  };
  if (p.d == 128) return go(std::integral_constant<int, 128>{});
  if (p.d == 96) return go(std::integral_constant<int, 96>{});
  if (p.d == 64) return go(std::integral_constant<int, 64>{});
  return cudaErrorInvalidValue;
}

}  // namespace mta
