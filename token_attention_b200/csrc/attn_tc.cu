// attn_tc.cu -- fused MTA attention on the sm_100a tensor cores (bf16 in/out).
//
// What it computes ("Multi-Token Attention | Summary" (greeksharifa)):
//   section 2  : logits A_hat = Q K^T / sqrt(d), causal softmax, A V;
//   section 3.1: A = Softmax(Mask_-inf(Conv2d_theta(Mask_0(A_hat)))), a c_q x c_k
//                kernel per head over (current and previous queries, keys
//                centred on the key);
//   section 3.2: post-softmax head mixing inside groups of 2 heads;
//   section 3.3: optional group norm + depth scale of each head's output
//                (fused epilogue of the layer).
// Appendix B of the same page: post-softmax mixing acts through the values, so
// O^h = sum_s w[h][s] (A^s V^h) -- the kernel never forms a mixed L x L map.
//
// Design (one CTA = one (batch, head, tile of BR = 128-(c_q-1) queries)):
//   * TMA loads the query rows i0-(c_q-1) .. i0+BR-1 (the c_q-1 row halo the
//     convolution reads) and, per key tile of 128, the key rows j0-c .. j0+128+c
//     (c = c_k/2 column halo), 128-byte swizzled.
//   * One thread issues tcgen05.mma: S = Q K^T (M=128, N=144, fp32 in tensor
//     memory), then Z_hd += P V^hd for every destination head hd of the group,
//     with P read from tensor memory.
//   * Four warpgroups of 128 threads (one TMEM lane = one query row per thread,
//     one warpgroup per 32 output keys) read S with tcgen05.ld, apply Mask_0,
//     publish their columns to a shared-memory copy of the masked tile (the
//     convolution needs the c_q-1 rows above and c columns on each side),
//     convolve with theta (fp32 FMA, 1/sqrt(d) and log2(e) folded into theta),
//     apply Mask_-inf, keep an exact online softmax (the convolution is local
//     and precedes the row max; the running max is only moved when it grows by
//     more than 2^8, and the accumulators are rescaled then), and write P
//     (bf16, two keys per 32-bit column) into tensor memory for the next MMA.
//   * Post-softmax mixing (c_h = 2): the two heads of a group run as a 2-CTA
//     cluster.  CTA s accumulates Z_{s->h} = P^s V^h for both destination heads h
//     and, at the end, sends Z_{s->peer} / l_s to the peer through distributed
//     shared memory; each CTA then forms O^h = sum_s w[h][s] Z_{s->h} / l_s.
//   * The L x L maps exist only as 128 x 144 tiles in tensor memory and shared
//     memory.  Every mbarrier wait is bounded (error word + early exit).
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace mta {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;  // move the running max only when it grows by > 2^8
constexpr int kConvWarps = 16;        // four warpgroups
constexpr int kThreads = 64 + 32 * kConvWarps;  // warp 0 TMA, warp 1 MMA, warps 2..17 softmax/conv
constexpr int kConvThreads = 32 * kConvWarps;

// named barriers (0 is __syncthreads)
constexpr int kBarScratch = 1;  // masked S tile published to shared memory
constexpr int kBarMax = 2;      // row maxima exchanged between warpgroups
constexpr int kBarSum = 3;      // row sums exchanged (end of the key loop)

// ---------------------------------------------------------------------------
// compile-time geometry
// ---------------------------------------------------------------------------
// MIX: 0 = no head mixing, 1 = pre-softmax (group of 2), 2 = post-softmax (group of 2)
template <int D, int CQ, int CK, int MIX>
struct Geo {
  static constexpr int CH = MIX ? 2 : 1;              // heads per group
  static constexpr int NH = MIX == 1 ? 2 : 1;         // source heads whose logits this CTA convolves
  static constexpr int NV = MIX == 2 ? 2 : 1;         // destination heads (V tiles, Z accumulators)
  static constexpr int CLUSTER = MIX == 2 ? 2 : 1;
  static constexpr int C = CK / 2;
  static constexpr int HALO = CQ - 1;
  static constexpr int BM = 128;                      // S rows = queries incl. halo
  static constexpr int BR = BM - HALO;                // output queries per CTA
  static constexpr int BN = 128;                      // output keys per key tile
  static constexpr int NS = (BN + 2 * C + 15) / 16 * 16;  // S columns (MMA N)
  static constexpr int NDC = D / 64;                  // 64-element (128-byte) d chunks
  static constexpr int KW = 32;                       // output keys per warpgroup
  static constexpr int WIN = KW + 2 * C;              // convolution window of a warpgroup
  static constexpr int SCOLS = BN + 2 * C;            // columns of the shared masked tile
  static constexpr int SSTR0 = (SCOLS + 3) / 4 * 4;
  static constexpr int SSTR = (SSTR0 % 8 == 0) ? SSTR0 + 4 : SSTR0;  // conflict-free rows
  static constexpr int DQ = D / 4;                    // output columns per warpgroup
  // shared memory (bytes)
  static constexpr int Q_HEAD = BM * D * 2;
  static constexpr int Q_BYTES = NH * Q_HEAD;
  static constexpr int Q_CHUNK = BM * 128;
  static constexpr int K_CHUNK = NS * 128;
  static constexpr int K_BYTES = NS * D * 2;
  static constexpr int V_CHUNK = BN * 128;
  static constexpr int V_HEAD = BN * D * 2;
  static constexpr int V_BYTES = NV * V_HEAD;
  static constexpr int SCR_BYTES = (CQ > 1 || MIX == 2) ? BM * SSTR * 4 : 0;  // also the exchange buffer
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + K_BYTES;
  static constexpr int OFF_SCR = OFF_V + V_BYTES;
  static constexpr int OFF_SMALL = (OFF_SCR + SCR_BYTES + 1023) / 1024 * 1024;
  static constexpr int SMALL_BYTES = 10240;
  static constexpr int SMEM_USED = OFF_SMALL + SMALL_BYTES + 1024;
  // at least half the SM's shared memory, so that one CTA runs per SM and the
  // 512-column TMEM allocation never waits for another CTA
  static constexpr int SMEM = SMEM_USED > 232448 / 2 + 1024 ? SMEM_USED : 232448 / 2 + 1024;
  // exchange buffer for the post-softmax mix (reuses V and the scratch after the loop)
  static constexpr int XSTR = D + 4;
  // tensor memory columns
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL0 = 0;
  static constexpr uint32_t S_COL1 = 224;  // second source head (pre-softmax mixing)
  static constexpr uint32_t P_COL = 160;   // 64 columns: 128 keys of bf16, two per column
  static constexpr uint32_t Z_COL0 = NH == 2 ? 384 : 256;
  static_assert(NS <= 160 && NS % 16 == 0, "S tile");
  static_assert(Z_COL0 + 128 * (NV - 1) + D <= TMEM_COLS, "tensor memory");
  static_assert(NH == 1 || (S_COL1 + NS <= Z_COL0 && P_COL + 64 <= S_COL1), "tensor memory (two S)");
  static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0, "swizzle alignment");
  static_assert(MIX != 2 || BM * XSTR * 4 <= V_BYTES + SCR_BYTES, "exchange buffer");
  static_assert(SMEM <= 232448, "shared memory");
};

struct TcParams {
  const float *theta;   // [H][CQ][CK]; null = 1x1 identity kernel (no convolution)
  const float *w;       // [H/CH][CH][CH]
  __nv_bfloat16 *out;   // [B][L][H][D]
  const float *gamma, *beta;
  float eps, lam;
  const float *gate;    // [H] sigmoid gate logits (replace lam) or null
  int gn;               // fuse group norm + depth scale
  int L, H, n_qtiles;
  float qk_scale;       // logit scale (1/sqrt(d) unless the caller chose another)
  unsigned *err;
};

// One query row of the key-query convolution for 32 output keys:
//   acc[jj] += sum_t th[t] * X[jj + 2C - t]      (key j - (t - C) of the row)
template <int CK, int WIN>
__device__ __forceinline__ void conv_row(float (&acc)[32], const float (&X)[WIN], const float *th) {
  constexpr int C = CK / 2;
#pragma unroll
  for (int t = 0; t < CK; ++t) {
    const float k = th[t];
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) acc[jj] = fmaf(k, X[jj + 2 * C - t], acc[jj]);
  }
}

template <int N>
__device__ __forceinline__ float tree_max(const float (&x)[N]) {
  float m[N / 2];
#pragma unroll
  for (int i = 0; i < N / 2; ++i) m[i] = fmaxf(x[2 * i], x[2 * i + 1]);
#pragma unroll
  for (int s = N / 4; s >= 1; s >>= 1)
#pragma unroll
    for (int i = 0; i < s; ++i) m[i] = fmaxf(m[i], m[i + s]);
  return m[0];
}

template <int D, int CQ, int CK, int MIX>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const TcParams p) {
  using G = Geo<D, CQ, CK, MIX>;
  constexpr int CH = G::CH, NH = G::NH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *Qs = smem + G::OFF_Q;
  uint8_t *Ks = smem + G::OFF_K;
  uint8_t *Vs = smem + G::OFF_V;
  float *Scr = reinterpret_cast<float *>(smem + G::OFF_SCR);
  uint8_t *small = smem + G::OFF_SMALL;
  float *th_s = reinterpret_cast<float *>(small);             // [NH][CQ*CK], scaled
  float *w_s = reinterpret_cast<float *>(small + 1024);       // [CH*CH]
  float *redmax = reinterpret_cast<float *>(small + 1088);    // [2 parity][4 wg][128]
  float *redsum = reinterpret_cast<float *>(small + 5184);    // [4 wg][128]
  float *redgn = reinterpret_cast<float *>(small + 7232);     // [4 wg][128]
  uint64_t *bars = reinterpret_cast<uint64_t *>(small + 9280);
  uint64_t *q_full = bars + 0, *k_full = bars + 1, *k_empty = bars + 2, *v_full = bars + 3;
  uint64_t *v_empty = bars + 4, *s_full = bars + 5, *s_free = bars + 7, *p_full = bars + 9;
  uint64_t *mma_done = bars + 10;   // s_full[NH], s_free[NH]: one per source head
  uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 11);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 12);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x;
  const int b = blockIdx.y;
  const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.z);  // longest tiles first
  const int g = h / CH, hr = h % CH;
  const int L = p.L;
  const int i0 = qt * G::BR;
  const int row0 = i0 - G::HALO;  // query index of S row 0
  const int last_q = min(L - 1, i0 + G::BR - 1);
  const int n_kv = last_q / G::BN + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1); mbar_init(k_full, 1); mbar_init(k_empty, 1); mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    for (int hh = 0; hh < NH; ++hh) { mbar_init(s_full + hh, 1); mbar_init(s_free + hh, kConvWarps); }
    mbar_init(p_full, kConvWarps); mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x >= 64 && threadIdx.x < 64 + NH * CQ * CK) {
    // key-query kernels, scaled by 1/sqrt(d) and log2(e).  Pre-softmax mixing is
    // linear after the convolution, so w[h][s] is folded into source head s's
    // kernel: C'_h = sum_s (w[h][s] theta_s) * Mask_0(A_hat_s).
    const int i = threadIdx.x - 64, hh = i / (CQ * CK), e = i % (CQ * CK);
    const int hs = NH == 2 ? g * CH + hh : h;
    float th = (p.theta ? p.theta[static_cast<long long>(hs) * CQ * CK + e] : 1.f) * (p.qk_scale * kLog2e);
    if (NH == 2) th *= p.w[(static_cast<long long>(g) * CH + hr) * CH + hh];
    th_s[i] = th;
  }
  if (threadIdx.x >= 256 && threadIdx.x < 256 + CH * CH)
    w_s[threadIdx.x - 256] = p.w[static_cast<long long>(g) * CH * CH + (threadIdx.x - 256)];
  if (warp == 1) { tmem_alloc(tslot, G::TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    // Two independent streams: lane 0 loads Q and the key tiles (a key tile is
    // requested as soon as the previous QK^T has consumed the buffer), lane 1
    // loads the value tiles (after the previous P V has consumed theirs).
    if (lane == 0) {
      prefetch_tmap(&tmQ); prefetch_tmap(&tmK);
      mbar_arrive_expect_tx(q_full, G::Q_BYTES);
#pragma unroll
      for (int hh = 0; hh < NH; ++hh)
#pragma unroll
        for (int dc = 0; dc < G::NDC; ++dc)
          tma_load_4d(Qs + hh * G::Q_HEAD + dc * G::Q_CHUNK, &tmQ, q_full, dc * 64,
                      NH == 2 ? g * CH + hh : h, row0, b);
      int nk = 0;
      for (int u = 0; u < n_kv * NH; ++u) {  // key tiles, source heads alternating
        const int t = u / NH, hh = u % NH;
        if (!mbar_wait(k_empty, (u & 1) ^ 1, abort_flag, p.err)) break;
        mbar_arrive_expect_tx(k_full, G::K_BYTES);
#pragma unroll
        for (int dc = 0; dc < G::NDC; ++dc)
          tma_load_4d(Ks + dc * G::K_CHUNK, &tmK, k_full, dc * 64, NH == 2 ? g * CH + hh : h,
                      t * G::BN - G::C, b);
        ++nk;
      }
      drain_wait(q_full, 0);
      if (*abort_flag && nk) drain_wait(k_full, (nk - 1) & 1);  // copies in flight land first
    } else if (lane == 1) {
      prefetch_tmap(&tmV);
      int nv = 0;
      for (int t = 0; t < n_kv; ++t) {
        if (!mbar_wait(v_empty, (t & 1) ^ 1, abort_flag, p.err)) break;
        mbar_arrive_expect_tx(v_full, G::V_BYTES);
#pragma unroll
        for (int hd = 0; hd < G::NV; ++hd) {
          const int hv = (G::NV == 1) ? h : g * CH + hd;
#pragma unroll
          for (int dc = 0; dc < G::NDC; ++dc)
            tma_load_4d(Vs + hd * G::V_HEAD + dc * G::V_CHUNK, &tmV, v_full, dc * 64, hv, t * G::BN, b);
        }
        ++nv;
      }
      if (*abort_flag && nv) drain_wait(v_full, (nv - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, G::NS, 0, 0);
      const uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_base = smem_u32(Qs), k_base = smem_u32(Ks), v_base = smem_u32(Vs);
      bool ok = mbar_wait(q_full, 0, abort_flag, p.err);
      auto issue_qk = [&](int t, int hh) -> bool {
        const int u = t * NH + hh;
        if (!mbar_wait(k_full, u & 1, abort_flag, p.err)) return false;
        if (t > 0 && !mbar_wait(s_free + hh, (t - 1) & 1, abort_flag, p.err)) return false;
        tc_fence_after();
        const uint32_t qh = q_base + hh * G::Q_HEAD;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tmem + (hh ? G::S_COL1 : G::S_COL0),
                      sdesc_sw128(qh + (kk >> 2) * G::Q_CHUNK + (kk & 3) * 32, 16, 1024),
                      sdesc_sw128(k_base + (kk >> 2) * G::K_CHUNK + (kk & 3) * 32, 16, 1024), idesc_qk,
                      kk > 0);
        mma_commit(k_empty);
        mma_commit(s_full + hh);
        return true;
      };
      for (int hh = 0; ok && hh < NH; ++hh) ok = issue_qk(0, hh);
      for (int t = 0; ok && t < n_kv; ++t) {
        bool next_ok = true;
        for (int hh = 0; next_ok && hh < NH && t + 1 < n_kv; ++hh) next_ok = issue_qk(t + 1, hh);
        if (!next_ok) break;
        if (!mbar_wait(p_full, t & 1, abort_flag, p.err)) break;
        if (!mbar_wait(v_full, t & 1, abort_flag, p.err)) break;
        tc_fence_after();
#pragma unroll
        for (int hd = 0; hd < G::NV; ++hd)
#pragma unroll
          for (int kk = 0; kk < G::BN / 16; ++kk)
            mma_f16_ts(tmem + G::Z_COL0 + 128 * hd, tmem + G::P_COL + 8 * kk,
                        sdesc_sw128(v_base + hd * G::V_HEAD + kk * 16 * 128, G::V_CHUNK, 1024),
                        idesc_pv, (t > 0 || kk > 0));
        mma_commit(v_empty);
      }
      mma_commit(mma_done);
      drain_wait(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------- softmax / conv
    const int wg = (warp - 2) >> 2;      // warpgroup: output keys 32*wg .. 32*wg+31 of a tile
    const int q4 = warp & 3;             // TMEM lane quadrant of this warp
    const int r = 32 * q4 + lane;        // S row = TMEM lane
    const int qrow = row0 + r;           // query index of this row
    const bool out_row = r >= G::HALO;   // rows below the halo produce outputs
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q4) << 16);
    const int cb = G::KW * wg;           // first output key (tile-relative) of this warpgroup
    float m_run = -INFINITY, l_part = 0.f;

    for (int t = 0; t < n_kv; ++t) {
      const int j0 = t * G::BN;
      float acc[32];
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) acc[jj] = 0.f;
      // a warp whose 32 rows all precede the chunk's first key has nothing to compute
      const bool live = (j0 + cb) <= (row0 + 32 * q4 + 31);
#pragma unroll 1
      for (int hh = 0; hh < NH; ++hh) {  // source heads (two when mixing before the softmax)
        mbar_wait(s_full + hh, t & 1, abort_flag, p.err);
        tc_fence_after();
        const uint32_t scol = hh ? G::S_COL1 : G::S_COL0;
        uint32_t u0[32], u1[16];
        tmem_ld32(tl + scol + cb, u0);
        if (G::WIN > 32) tmem_ld16(tl + scol + cb + 32, u1);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free + hh);
        float X[G::WIN];
#pragma unroll
        for (int k = 0; k < G::WIN; ++k) X[k] = __uint_as_float(k < 32 ? u0[k] : u1[(k - 32) & 15]);
        // Mask_0: keys after this row's query count as 0 inside the convolution
        const int key0 = j0 - G::C + cb;  // key of window element 0
        if (key0 + G::WIN - 1 > qrow) {
#pragma unroll
          for (int k = 0; k < G::WIN; ++k)
            if (key0 + k > qrow) X[k] = 0.f;
        }
        if (CQ > 1) {  // publish this warpgroup's columns of the masked tile
          if (hh > 0) named_bar_sync(kBarScratch, kConvThreads);  // previous head's tile fully read
          float *my = Scr + r * G::SSTR + cb;
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            *reinterpret_cast<float4 *>(my + k) = make_float4(X[k], X[k + 1], X[k + 2], X[k + 3]);
          if (wg == 3) {
#pragma unroll
            for (int k = 32; k + 4 <= G::WIN; k += 4)
              *reinterpret_cast<float4 *>(my + k) = make_float4(X[k], X[k + 1], X[k + 2], X[k + 3]);
#pragma unroll
            for (int k = 32 + (G::WIN - 32) / 4 * 4; k < G::WIN; ++k) my[k] = X[k];
          }
          named_bar_sync(kBarScratch, kConvThreads);
        }
        if (out_row && live) {
          const float *th = th_s + hh * CQ * CK;
          conv_row<CK, G::WIN>(acc, X, th);
#pragma unroll
          for (int a = 1; a < CQ; ++a) {
            const float *src = Scr + (r - a) * G::SSTR + cb;
            float Y[G::WIN];
#pragma unroll
            for (int k = 0; k + 4 <= G::WIN; k += 4) {
              const float4 f = *reinterpret_cast<const float4 *>(src + k);
              Y[k] = f.x; Y[k + 1] = f.y; Y[k + 2] = f.z; Y[k + 3] = f.w;
            }
#pragma unroll
            for (int k = G::WIN / 4 * 4; k < G::WIN; ++k) Y[k] = src[k];
            conv_row<CK, G::WIN>(acc, Y, th + a * CK);
          }
        }
      }
      // Mask_-inf and the tile's row max (log2 units)
      const int kbase = j0 + cb;
#pragma unroll
      for (int jj = 0; jj < 32; ++jj)
        if (kbase + jj > qrow) acc[jj] = -INFINITY;
      float mt = out_row ? tree_max<32>(acc) : -INFINITY;
      float *rm = redmax + (t & 1) * 512;
      rm[wg * 128 + r] = mt;
      named_bar_sync(kBarMax, kConvThreads);  // also: every read of the shared tile is done
      mt = fmaxf(fmaxf(rm[r], rm[128 + r]), fmaxf(rm[256 + r], rm[384 + r]));
      const float m_new = fmaxf(m_run, mt);
      bool resc = false;
      float alpha = 1.f;
      if (t == 0) {
        m_run = m_new;
      } else if (m_new > m_run + kRescaleLog2) {
        resc = true;
        alpha = ex2(m_run - m_new);
        m_run = m_new;
      }
      // P = 2^(C - m) (bf16), row sums
      uint32_t pk[16];
      float ps[16];
#pragma unroll
      for (int jj = 0; jj < 32; jj += 2) {
        const float p0 = out_row ? ex2(acc[jj] - m_run) : 0.f;
        const float p1 = out_row ? ex2(acc[jj + 1] - m_run) : 0.f;
        ps[jj >> 1] = p0 + p1;
        pk[jj >> 1] = pack_bf16x2(p0, p1);
      }
#pragma unroll
      for (int s = 8; s >= 1; s >>= 1)
#pragma unroll
        for (int i = 0; i < s; ++i) ps[i] += ps[i + s];
      if (t > 0) {  // P(t-1) consumed and Z(t-1) complete
        mbar_wait(v_empty, (t - 1) & 1, abort_flag, p.err);
        tc_fence_after();
      }
      // tcgen05.ld/st are warp-collective: rescale for the whole warp when any
      // row needs it (alpha = 1 on the other rows)
      if (__any_sync(0xffffffffu, resc)) {
        l_part *= alpha;
#pragma unroll
        for (int hd = 0; hd < G::NV; ++hd)
#pragma unroll
          for (int c0 = 0; c0 < G::DQ; c0 += 16) {
            uint32_t z[16];
            const uint32_t ad = tl + G::Z_COL0 + 128 * hd + wg * G::DQ + c0;
            tmem_ld16(ad, z);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) z[i] = __float_as_uint(__uint_as_float(z[i]) * alpha);
            tmem_st16(ad, z);
          }
      }
      l_part += ps[0];
      tmem_st16(tl + G::P_COL + (cb >> 1), pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // all P V products of the last tile are in Z
    mbar_wait(v_empty, (n_kv - 1) & 1, abort_flag, p.err);
    tc_fence_after();
    redsum[wg * 128 + r] = l_part;
    named_bar_sync(kBarSum, kConvThreads);
  }

  // ------------------------------------------------------------- epilogue
  const bool conv_thread = warp >= 2;
  const int wg = conv_thread ? (warp - 2) >> 2 : 0;
  const int q4 = warp & 3;
  const int r = 32 * q4 + lane;
  const int qrow = row0 + r;
  const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q4) << 16);
  const int cbase = wg * G::DQ;
  float o[G::DQ];
  float inv_l = 0.f;
  if (conv_thread) {
    inv_l = redsum[r] + redsum[128 + r] + redsum[256 + r] + redsum[384 + r];
    inv_l = (r >= G::HALO && inv_l > 0.f) ? 1.f / inv_l : 0.f;
  }
  if constexpr (MIX == 2) {
    float *xbuf = reinterpret_cast<float *>(Vs);  // [BM][XSTR] fp32, reuses V and the scratch
    cluster_sync_all();                           // both CTAs are done with V and the scratch
    if (conv_thread) {
      const uint32_t peer = static_cast<uint32_t>(hr ^ 1);
      const uint32_t dst = map_peer(smem_u32(xbuf + r * G::XSTR + cbase), peer);
#pragma unroll
      for (int c0 = 0; c0 < G::DQ; c0 += 16) {
        uint32_t z[16];
        tmem_ld16(tl + G::Z_COL0 + 128 * (hr ^ 1) + cbase + c0, z);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; i += 4)
          st_cluster_v4(dst + 4 * (c0 + i), __uint_as_float(z[i]) * inv_l, __uint_as_float(z[i + 1]) * inv_l,
                        __uint_as_float(z[i + 2]) * inv_l, __uint_as_float(z[i + 3]) * inv_l);
      }
    }
    cluster_sync_all();  // the peer's Z_{peer->h} / l_peer is in xbuf
    if (conv_thread) {
      const float w_own = w_s[hr * CH + hr], w_peer = w_s[hr * CH + (hr ^ 1)];
      const float *xr = xbuf + r * G::XSTR + cbase;
#pragma unroll
      for (int c0 = 0; c0 < G::DQ; c0 += 16) {
        uint32_t z[16];
        tmem_ld16(tl + G::Z_COL0 + 128 * hr + cbase + c0, z);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          o[c0 + i] = w_own * (__uint_as_float(z[i]) * inv_l) + w_peer * xr[c0 + i];
      }
    }
  } else {
    if (conv_thread) {
#pragma unroll
      for (int c0 = 0; c0 < G::DQ; c0 += 16) {
        uint32_t z[16];
        tmem_ld16(tl + G::Z_COL0 + cbase + c0, z);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) o[c0 + i] = __uint_as_float(z[i]) * inv_l;
      }
    }
  }
  if (p.gn) {  // group norm over the D channels of (token, head), then depth scale
    float s = 0.f;
    if (conv_thread) {
#pragma unroll
      for (int i = 0; i < G::DQ; ++i) s += o[i];
      redgn[wg * 128 + r] = s;
    }
    __syncthreads();
    float mu = 0.f, rstd = 0.f;
    if (conv_thread) {
      mu = (redgn[r] + redgn[128 + r] + redgn[256 + r] + redgn[384 + r]) * (1.f / D);
      float s2 = 0.f;
#pragma unroll
      for (int i = 0; i < G::DQ; ++i) { const float x = o[i] - mu; s2 += x * x; }
      s = s2;
    }
    __syncthreads();
    if (conv_thread) redgn[wg * 128 + r] = s;
    __syncthreads();
    if (conv_thread) {
      rstd = rsqrtf((redgn[r] + redgn[128 + r] + redgn[256 + r] + redgn[384 + r]) * (1.f / D) + p.eps);
      const float *gm = p.gamma + static_cast<long long>(h) * D + cbase;
      const float *bt = p.beta + static_cast<long long>(h) * D + cbase;
      const float mh = head_multiplier(p.gate, p.lam, h);
#pragma unroll
      for (int i = 0; i < G::DQ; ++i) o[i] = ((o[i] - mu) * rstd * gm[i] + bt[i]) * mh;
    }
  }
  if (conv_thread && r >= G::HALO && qrow < L) {
    __nv_bfloat16 *dst = p.out + ((static_cast<long long>(b) * L + qrow) * p.H + h) * D + cbase;
#pragma unroll
    for (int i = 0; i < G::DQ; i += 8) {
      uint4 v;
      v.x = pack_bf16x2(o[i], o[i + 1]);
      v.y = pack_bf16x2(o[i + 2], o[i + 3]);
      v.z = pack_bf16x2(o[i + 4], o[i + 5]);
      v.w = pack_bf16x2(o[i + 6], o[i + 7]);
      *reinterpret_cast<uint4 *>(dst + i) = v;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, G::TMEM_COLS);
  }
}

template <int D, int CQ, int CK, int MIX>
cudaError_t launch_one(const AttnArgs &a, const GnArgs *gn) {
  using G = Geo<D, CQ, CK, MIX>;
  alignas(64) CUtensorMap tq, tk, tv;
  const unsigned long long dims[4] = {static_cast<unsigned long long>(D), static_cast<unsigned long long>(a.H),
                                      static_cast<unsigned long long>(a.L), static_cast<unsigned long long>(a.B)};
  const unsigned long long str[3] = {static_cast<unsigned long long>(D) * 2,
                                     static_cast<unsigned long long>(a.rs) * 2,
                                     static_cast<unsigned long long>(a.rs) * 2 * a.L};
  const unsigned boxq[4] = {64, 1, G::BM, 1}, boxk[4] = {64, 1, G::NS, 1}, boxv[4] = {64, 1, G::BN, 1};
  if (!encode_tmap_bf16(&tq, a.q, 4, dims, str, boxq, true)) return cudaErrorInvalidValue;
  if (!encode_tmap_bf16(&tk, a.k, 4, dims, str, boxk, true)) return cudaErrorInvalidValue;
  if (!encode_tmap_bf16(&tv, a.v, 4, dims, str, boxv, true)) return cudaErrorInvalidValue;
  TcParams p;
  p.theta = a.theta;
  p.w = a.w;
  p.out = static_cast<__nv_bfloat16 *>(a.out);
  p.gn = gn != nullptr;
  p.gamma = gn ? gn->gamma : nullptr;
  p.beta = gn ? gn->beta : nullptr;
  p.eps = gn ? gn->eps : 0.f;
  p.lam = gn ? gn->lam : 1.f;
  p.gate = gn ? gn->gate : nullptr;
  p.L = a.L;
  p.H = a.H;
  p.n_qtiles = (a.L + G::BR - 1) / G::BR;
  p.qk_scale = a.scale;
  p.err = a.err;
  auto kern = attn_tc_kernel<D, CQ, CK, MIX>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.H, a.B, p.n_qtiles);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = G::SMEM;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = G::CLUSTER;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, p);
}

}  // namespace

bool attn_tc_supported(const AttnArgs &a) {
  if (a.dtype != 1 || a.kqp != 0) return false;
  if (a.d != 64 && a.d != 128) return false;
  const bool kq_std = a.kq == 1 && a.cq == 6 && a.ck == 11;
  const bool kq_off = a.kq == 0;
  if (!kq_std && !kq_off) return false;
  const bool mix_off = a.hp == 0;
  const bool mix_group2 = (a.hp == 1 || a.hp == 2) && a.ch == 2;  // pre- or post-softmax
  if (!mix_off && !mix_group2) return false;
  if (a.B > 65535 || a.H > 65535 || (a.L + 122) / 123 > 65535) return false;
  const uintptr_t al = reinterpret_cast<uintptr_t>(a.q) | reinterpret_cast<uintptr_t>(a.k) |
                       reinterpret_cast<uintptr_t>(a.v) | reinterpret_cast<uintptr_t>(a.out);
  if (al % 16 != 0 || a.rs % 8 != 0) return false;
  return true;
}

template <int D, int CQ, int CK>
cudaError_t launch_mix(const AttnArgs &a, const GnArgs *gn) {
  if (a.hp == 1) return launch_one<D, CQ, CK, 1>(a, gn);
  if (a.hp == 2) return launch_one<D, CQ, CK, 2>(a, gn);
  return launch_one<D, CQ, CK, 0>(a, gn);
}

cudaError_t launch_attn_tc(const AttnArgs &a0, const GnArgs *gn) {
  AttnArgs a = a0;
  if (a.kq == 1) return a.d == 128 ? launch_mix<128, 6, 11>(a, gn) : launch_mix<64, 6, 11>(a, gn);
  a.theta = nullptr;  // no key-query convolution: 1 x 1 identity kernel
  return a.d == 128 ? launch_mix<128, 1, 1>(a, gn) : launch_mix<64, 1, 1>(a, gn);
}

}  // namespace mta
