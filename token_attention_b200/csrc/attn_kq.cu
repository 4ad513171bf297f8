// attn_kq.cu -- fused MTA attention with the key-query convolution as a
// tensor-core contraction (bf16 in/out, fp16 contraction operands).
//
// What it computes ("Multi-Token Attention | Summary" (greeksharifa)):
//   section 2  : logits A_hat = Q K^T / sqrt(d), causal softmax, A V;
//   section 3.1: A = Softmax(Mask_-inf(Conv2d_theta(Mask_0(A_hat)))) (or the exact
//                causal indicator), and optionally the convolution after the
//                softmax, A' = Mask_0(Conv2d_theta_post(A));
//   section 3.2: head mixing inside groups of 2 heads, before the softmax or after
//                it (appendix B: through the values, O^h = sum_s w[h][s] A^s V^h);
//   section 3.3: optional group norm with a depth scale or sigmoid gate (fused
//                epilogue).
//
// The convolution is linear in the logits, and the logits are bilinear in q and
// k, so without the mask
//   C[i][j] = s * sum_a q[i-a] . Kt_a[j],   Kt_a[j] = sum_t theta[a][t] k[j-(t-c)],
// a contraction of length c_q*d between the c_q shifted query rows and the
// per-row-convolved keys (built by the prepass in kq_prep.cu).  Mask_0 zeroes
// the taps that read a key after the shifted query (key j-(t-c) > i-a); such taps
// only exist in the band 0 <= i-j < W = (c_q-1)+c, where the kernel replaces the
// contraction's value by the convolution taken tap by tap over the unmasked taps:
//   C[i][j] = s * sum_{a,t: m = (i-a) - (j-(t-c)) >= 0} theta[a][t] Vp[i-a][m],
// with the prepass's past dot products Vp[i][m] = q[i] . k[i-m].  Nothing the
// kernel reads for query i depends on an input after position i, so outputs are
// exactly causal (the query tile's fp16 scale only scales down, when |q| > 2^14).
//
// Design (persistent: one CTA, or a 2-CTA cluster with post-softmax mixing, per SM,
// walking (query tile of 128, batch, head group) work items longest first):
//   * Warp 10's TMA loads the query rows i0-(c_q-1) .. i0+127 of each item as
//     8-element strips in which consecutive rows are 16 bytes apart; the softmax
//     warps convert them in place to fp16 with a power-of-2 scale.  A row shift
//     by a is then a 16*a-byte offset of the MMA descriptor (SWIZZLE_NONE layout).
//   * Per key tile of 128: warp 8's TMA streams Kt (fp16, 128-byte swizzle)
//     through a ring whose stage is a whole tap row when d is a multiple of 64;
//     warp 9's single thread issues the contraction MMAs (M=128, N=128, K=16) of C
//     into tensor memory, then P V (P read from tensor memory; one N=256 MMA for
//     both heads' V with post-softmax mixing).
//   * Two softmax warpgroups (64 key columns and half of the output channels each,
//     a whole query row per thread) read C, scale it, apply the Mask_0 correction
//     near the diagonal and Mask_-inf, keep an exact online softmax (the running
//     max moves only when it grows by more than 2^8, then Z is rescaled) and write
//     P (bf16) to tensor memory.
//   * Post-softmax mixing runs as a 2-CTA cluster exchanging Z_{s->peer}/l_s through
//     an L2 buffer in the workspace once per item, handshaked by cluster mbarriers.
//   * With the post-softmax convolution (POST) each item makes two passes (exact
//     row statistics, then normalised weights in shared memory times the values
//     convolved by the post-softmax kernels, c_q row-shifted products), with the c
//     keys ending at each diagonal added on the CUDA cores (see POST below).
//   * Every mbarrier wait is bounded (error word + early exit).
#include <cuda.h>

#include <algorithm>
#include <type_traits>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace mta {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;
// warps 0-7: two softmax warpgroups (warpgroup w takes key columns 64w .. 64w+63 of
// every tile and half of the output channels); warp 8: TMA of the convolved keys
// (and values); warp 9: MMA; warp 10: TMA of V and of the query rows (a warp of its
// own, so that these waits never hold up the busier key stream)
constexpr int kThreads = 352;
constexpr int kSmThreads = 256;
constexpr int kTmaWarp = 8, kMmaWarp = 9, kTma2Warp = 10;
constexpr int kBarAll = 1;      // named barrier over both softmax warpgroups
constexpr int kKqMaxClusters = 160;  // persistent grid: at most this many CTAs (>= SM count)
constexpr int kItemSlots = 4;        // item ring: indices taken from the queue ahead of their use

template <int D, int CQ, int CK, int MIX, bool EXACT, bool POST>
struct KGeo {
  // band 0 <= i-j < W where taps are masked: keys after the shifted query (Mask_0)
  // or after the output query (exact indicator); Vp[i][m] = q[i] . k[i-m+OFF]
  static constexpr int C = CK / 2, HALO = CQ - 1, W = EXACT ? C : HALO + C, M = HALO + 2 * C;
  static constexpr int OFF = EXACT ? HALO : 0;
  static constexpr int BM = 128, BN = 128, HALF = BN / 2;
  // output channels: warpgroup 0 takes DH (a multiple of 32), warpgroup 1 the other DH1
  static constexpr int DH = (D / 2 + 31) / 32 * 32, DH1 = D - DH;
  static constexpr int QROWS = (BM + HALO + 7) / 8 * 8;  // query rows staged (with halo)
  static constexpr int NSTRIP = D / 8;
  static constexpr int STRIP = QROWS * 16;               // bytes of one 8-element strip
  static constexpr int Q_BYTES = NSTRIP * STRIP;
  static constexpr int NDC = (D + 63) / 64;              // 64-channel blocks of a V row
  // Kt row of a key = the c_q*D contraction operand, in 64-element chunks
  static constexpr int NCH = CQ * D / 64;                // Kt chunks per key tile
  static constexpr int KCHUNK = BN * 128;                // 128 keys x 64 elements, fp16

  static constexpr int NV = MIX == 2 ? 2 : 1;            // V heads per CTA (post-softmax mixing: both)
  static constexpr int NSRC = MIX == 1 ? 2 : 1;          // heads whose C a CTA computes (pre-softmax mixing: both)
  static constexpr int CLUSTER = MIX == 2 ? 2 : 1;       // CTAs of a cluster: the heads of a group
  static constexpr int V_CHUNK = BN * 128;
  static constexpr int V_HEAD = NDC * V_CHUNK;            // a V tile: 64-channel boxes (the last may pass D)
  // with the post-softmax convolution the convolved values stream through the Kt
  // ring, and the normalised weights go to shared memory (8-key strips, 16-byte
  // rows, PS_PAD rows of padding above row 0 for the row shifts)
  static constexpr int V_BYTES = POST ? 0 : NV * V_HEAD;
  static constexpr int RSH = POST ? HALO : 0;            // rows of a tile above its output rows
  static constexpr int BMO = BM - RSH;                   // output rows per query tile
  static constexpr int PS_PAD = 8;
  static constexpr int PS_STRIP = (BM + PS_PAD) * 16;
  static constexpr int PS_BYTES = POST ? (BN / 8) * PS_STRIP : 0;
  static constexpr int DG_BYTES = POST ? BM * C * 4 : 0;   // weights of the c keys ending at the diagonal
  static constexpr int NVCH = NV * CQ * NDC;              // convolved-value chunks per key tile
  static constexpr int UB = HALO + 2 * C;                 // diagonals of the near-diagonal value band
  static constexpr int UROWS = BM + HALO;
  static constexpr int U_BYTES = (UROWS * M * 4 + 15) / 16 * 16;
  static constexpr int CS_BYTES = 2 * BM * W * 4;        // band values, one block per warpgroup
  static constexpr int RED_BYTES = 10 * BM * 4;          // row maxima (2 tiles x 2 groups), l, norm sums
  static constexpr int FAC_BYTES = NSRC * 2 * BN * 4;    // column factors of two key tiles, per source head
  static constexpr int Q_ALLOC = Q_BYTES;                              // query tiles of the sources, back to back
  static constexpr int Q_AREA = (NSRC * Q_ALLOC + 1023) / 1024 * 1024;  // up to the 1024-aligned ring
  // small area: taps [2 items][NSRC][128], per-warp |q| maxima, barriers, TMEM slot, abort flag
  static constexpr int TH_OFF = 0, THP_OFF = 2 * NSRC * 128 * 4;
  static constexpr int QRED_OFF = THP_OFF + (POST ? 2 * 128 * 4 : 0), BAR_OFF = QRED_OFF + 64;
  static constexpr int TSLOT_OFF = BAR_OFF + 8 * 40, ABORT_OFF = TSLOT_OFF + 8;
  static constexpr int ITEMS_OFF = ABORT_OFF + 8;         // the item ring: kItemSlots item indices
  static constexpr int SMALL_BYTES = (ITEMS_OFF + 16 + 255) / 256 * 256;
  // Kt ring: as many 16 KB stages as the shared memory left over holds (at most 8)
  static constexpr int REST = Q_AREA + V_BYTES + PS_BYTES + DG_BYTES + NSRC * U_BYTES + CS_BYTES +
                              RED_BYTES + FAC_BYTES + SMALL_BYTES + 1024;
  // a ring stage holds SB boxes: a whole tap row when d is a multiple of 64 and at
  // least three such stages fit, else one box
  static constexpr int SB = (D % 64 == 0 && (232448 - REST) / (NDC * KCHUNK) >= 3) ? NDC : 1;
  static constexpr int KSTAGE = SB * KCHUNK;
  static constexpr int NS = (232448 - REST) / KSTAGE < 8 ? (232448 - REST) / KSTAGE : 8;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_AREA;
  static constexpr int OFF_V = OFF_K + NS * KSTAGE;
  static constexpr int OFF_PS = OFF_V + V_BYTES;
  static constexpr int OFF_DG = OFF_PS + PS_BYTES;
  static constexpr int OFF_U = OFF_DG + DG_BYTES;
  static constexpr int OFF_CS = OFF_U + NSRC * U_BYTES;
  static constexpr int OFF_RED = OFF_CS + CS_BYTES;
  static constexpr int OFF_FAC = OFF_RED + RED_BYTES;
  static constexpr int OFF_SMALL = OFF_FAC + FAC_BYTES;
  static constexpr int SMEM_USED = OFF_SMALL + SMALL_BYTES + 1024;
  // at least half the SM's shared memory: one CTA per SM, so the 512-column TMEM
  // allocation never waits for another CTA
  static constexpr int SMEM = SMEM_USED > 232448 / 2 + 1024 ? SMEM_USED : 232448 / 2 + 1024;
  // tensor memory.  DB (one source head, no post-softmax convolution): C in two
  // 128-column buffers used by alternate key tiles, each tile's P (bf16, 64
  // columns) written over its own C, then Z.  Otherwise: C of each source head (128
  // columns each), P (64), Z (P lives in shared memory with POST).
  static constexpr bool DB = !POST && NSRC == 1;
  // DEFER (DB with post-softmax mixing): an item's epilogue releases Z, parks both
  // halves (for the peer head and for its own) in the L2 exchange buffer, and
  // finishes (mixing, group norm, store) only after the next item's first tile
  static constexpr bool DEFER = DB && MIX == 2;
  static constexpr uint32_t TMEM_COLS = 512, C_COL = 0, P_COL = DB ? 0 : 128 * NSRC;
  static constexpr uint32_t Z_COL0 = DB ? 256 : POST ? P_COL : P_COL + 128;
  static_assert(Z_COL0 + 128 * (NV - 1) + D <= TMEM_COLS, "tensor memory");
  // C double-buffered (tile T in buffer T & 1): DB, and the post-softmax variant when
  // a second C fits after Z (its weights are in shared memory, not over C); buffer 1
  // starts at column CB1
  static constexpr bool CDB = DB || (POST && Z_COL0 + 128 * (NV - 1) + D + 128 * NSRC <= TMEM_COLS);
  static constexpr uint32_t CB1 = DB ? 128 : TMEM_COLS - 128 * NSRC;
  static_assert(5 + 2 * NS + 10 <= 32, "barriers before the item ring");
  static_assert(MIX != 1 || NV == 1, "pre-softmax mixing uses the destination head's V only");
  static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0, "swizzle alignment");
  static_assert(OFF_PS % 16 == 0 && OFF_DG % 16 == 0 && OFF_U % 16 == 0, "alignment");
  static_assert(OFF_SMALL % 16 == 0, "alignment");
  static_assert(NS >= 3, "Kt ring");
  static_assert(NCH % SB == 0 && NDC % SB == 0, "whole stages");
  static_assert(15 + 2 * NS <= 32, "barrier slots (32 .. 39: the item ring)");
  static_assert(SMEM <= 232448, "shared memory");
  static_assert(CQ * CK <= 120, "kernel taps");
  static_assert(CQ * D % 64 == 0 && D % 16 == 0, "contraction chunks");
};

struct KqParams {
  const float *theta;   // [H][CQ][CK]
  const float *w;       // [H/2][2][2]
  __nv_bfloat16 *out;   // [B][L][H][D]
  const float *gamma, *beta;
  float eps, lam;
  const float *gate;    // [H] sigmoid gate logits (replace lam) or null
  int gn;
  int B, L, H, n_qtiles, lpad;
  float qk_scale;
  const float *fac;     // [B][H][lpad] s*log2(e)*2^-e_j per convolved key row (0 past L)
  const float *vp;      // [B][H][L][M] past dot products
  float *xg;            // post-softmax mixing exchange: [CTA][2 parities][2 parts][D/4][BM] float4
  unsigned *err;
  // post-softmax convolution: its kernels and the values (for the band near the diagonal)
  const float *theta_post;    // [H][CQ][CK]
  const __nv_bfloat16 *v;     // [B][L][H][D], token stride rs
  long long rs;
  unsigned *queue;            // work-queue counter (zero when the launch starts)
  int wave;                   // units (batch, head group) per wave of the item order
};

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

// Work item k of the launch: (query tile qt, batch b, head group g).  The units
// (b, g) are taken in waves of `wave` units (as many as keep their convolved keys
// resident in L2 together); inside a wave, items go longest first (query tile
// descending), then by unit.  The clusters take items from a queue in this order,
// so the clusters running at any time read the keys of a few units, and the
// shortest items come last.
struct Item {
  int qt, b, g;
};
__device__ __forceinline__ Item item_of(int k, int B, int G, int n_qtiles, int wave) {
  const int per_wave = wave * n_qtiles;
  const int w = k / per_wave, r = k - w * per_wave;
  const int nu = min(wave, B * G - w * wave);  // units of this wave (the last may have fewer)
  const int unit = w * wave + r % nu;
  Item it;
  it.qt = n_qtiles - 1 - r / nu;
  it.b = unit / G;
  it.g = unit % G;
  return it;
}

template <int D, int CQ, int CK, int MIX, bool EXACT, bool POST>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmVt,
                   const KqParams p) {
  using G = KGeo<D, CQ, CK, MIX, EXACT, POST>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *Qs = smem + G::OFF_Q;
  uint8_t *Ks = smem + G::OFF_K;
  uint8_t *Vs = smem + G::OFF_V;
  uint8_t *Ps = smem + G::OFF_PS;                                // normalised weights (POST)
  float *Dg = reinterpret_cast<float *>(smem + G::OFF_DG);       // [BM][C] near-diagonal weights (POST)
  float *Us = reinterpret_cast<float *>(smem + G::OFF_U);
  float *Cs = reinterpret_cast<float *>(smem + G::OFF_CS);
  float *red = reinterpret_cast<float *>(smem + G::OFF_RED);
  float *facs = reinterpret_cast<float *>(smem + G::OFF_FAC);  // [NSRC][2][BN]
  uint8_t *small = smem + G::OFF_SMALL;
  float *th_s = reinterpret_cast<float *>(small + G::TH_OFF);   // [2 items][NSRC][128]
  float *thp_s = reinterpret_cast<float *>(small + G::THP_OFF); // [2 items][128] post-softmax taps
  float *qred = reinterpret_cast<float *>(small + G::QRED_OFF); // [8] per-warp max |q|
  uint64_t *bars = reinterpret_cast<uint64_t *>(small + G::BAR_OFF);
  uint64_t *q_full = bars + 0, *q_ready = bars + 1, *q_free = bars + 2, *z_free = bars + 3;
  uint64_t *x_ready = bars + 4, *k_full = bars + 5, *k_empty = bars + 5 + G::NS;
  uint64_t *v_full = bars + 5 + 2 * G::NS, *v_empty = v_full + 1, *c_full = v_full + 2;
  uint64_t *c_free = v_full + 3, *p_full = v_full + 4, *mma_done = v_full + 5;
  // DB: C complete and P written, per buffer (tile T uses buffer T & 1)
  uint64_t *const c_fullb[2] = {c_full, v_full + 6};
  uint64_t *const p_fullb[2] = {p_full, v_full + 7};
  // CDB without DB (post-softmax variant): C of buffer b has been read by the softmax
  uint64_t *const c_freeb[2] = {c_free, v_full + 8};
  // post-softmax mixing: the peer's exchange data of item r is in place, one barrier
  // per item parity.  With one barrier the peer, one short item ahead, could complete
  // a second phase before this CTA waited for the first, and the parity wait then
  // waited for a phase that needs this CTA's own progress.  The peer cannot get two
  // items ahead: its item r+2 needs this CTA's arrival for r+1, which follows the wait
  // for r.
  uint64_t *const x_readyb[2] = {x_ready, v_full + 9};
  uint32_t *tslot = reinterpret_cast<uint32_t *>(small + G::TSLOT_OFF);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(small + G::ABORT_OFF);
  // item ring: it_full[s] completes when slot s holds the next item index (or -1 at
  // the end); it_empty[s] (in the cluster's first CTA) when every consumer of both
  // CTAs has read it
  uint64_t *it_full = bars + 32, *it_empty = bars + 36;
  volatile int *item_slot = reinterpret_cast<volatile int *>(small + G::ITEMS_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // cluster c (the two heads of a group with post-softmax mixing, else one CTA)
  const int hr = MIX == 2 ? static_cast<int>(blockIdx.x) : 0;
  const int c = static_cast<int>(blockIdx.y);  // this cluster's slot of the exchange buffer
  constexpr int CL = MIX == 2 ? 2 : 1;
  const int n_groups = p.H / CL;
  const int n_items = p.B * n_groups * p.n_qtiles;
  const int L = p.L;
  // Consumers of the item ring: the r-th item of this cluster (r = 0, 1, ...), or
  // false at the end of the queue (or after an abort).  Every consumer thread waits;
  // one arrival per consumer (lane 0 of a warp, or a single thread) frees the slot.
  auto take_item = [&](int r, Item &it, bool arrive) -> bool {
    const int s = r % kItemSlots;
    const bool ok = mbar_wait_cluster(it_full + s, (r / kItemSlots) & 1, abort_flag, p.err);
    const int k = ok ? item_slot[s] : -1;
    if (ok && arrive) {
      if (CL == 2 && hr != 0)
        mbar_arrive_cluster(map_peer(smem_u32(it_empty + s), 0u));
      else
        mbar_arrive(it_empty + s);
    }
    if (k < 0) return false;
    it = item_of(k, p.B, n_groups, p.n_qtiles, p.wave);
    return true;
  };
  // The producer (the cluster's first CTA, TMA warp lane 0): takes the next index
  // from the queue and publishes it to both CTAs' rings; -1 once the queue is empty.
  auto publish_item = [&](int r, Item &it) -> bool {
    const int s = r % kItemSlots;
    if (!mbar_wait_cluster(it_empty + s, ((r / kItemSlots) & 1) ^ 1, abort_flag, p.err)) return false;
    int k = static_cast<int>(atomicAdd(p.queue, 1u));
    if (k >= n_items) k = -1;
    item_slot[s] = k;
    if (CL == 2) {
      st_cluster_s32(map_peer(smem_u32(const_cast<int *>(item_slot + s)), 1u), k);
      mbar_arrive_cluster(map_peer(smem_u32(it_full + s), 1u));  // releases the store above
    }
    mbar_arrive(it_full + s);
    if (k < 0) return false;
    it = item_of(k, p.B, n_groups, p.n_qtiles, p.wave);
    return true;
  };
  // first query row of an item's tile (with POST, its c_q-1 rows above the output rows)
  auto row_start = [&](const Item &it) { return it.qt * G::BMO - G::RSH; };
  auto kv_tiles = [&](const Item &it) { return min(L - 1, row_start(it) + G::BM - 1) / G::BN + 1; };
  // key-tile passes of an item: one, or two with POST (exact row statistics first)
  auto n_slots = [&](const Item &it) { return POST ? 2 * kv_tiles(it) : kv_tiles(it); };
  // the head whose C is accumulated as source s of destination head h
  auto src_head = [&](int h, int s) { return G::NSRC == 2 ? (h & ~1) + s : h; };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1); mbar_init(q_ready, 8); mbar_init(q_free, 1); mbar_init(z_free, 8);
    mbar_init(x_readyb[0], kSmThreads); mbar_init(x_readyb[1], kSmThreads);
    for (int s = 0; s < G::NS; ++s) { mbar_init(k_full + s, 1); mbar_init(k_empty + s, 1); }
    mbar_init(v_full, 1); mbar_init(v_empty, 1); mbar_init(c_full, 1); mbar_init(c_free, 8);
    mbar_init(p_full, 8); mbar_init(mma_done, 1);
    mbar_init(c_fullb[1], 1); mbar_init(p_fullb[1], 8); mbar_init(c_freeb[1], 8);
    // consumers per item: the V and query loaders, the MMA thread and the 8 softmax
    // warps of each CTA, and the second CTA's key loader (no V loader with POST)
    constexpr int per_cta = (POST ? 1 : 2) + 1 + 8;
    for (int s = 0; s < kItemSlots; ++s) {
      mbar_init(it_full + s, 1);
      mbar_init(it_empty + s, CL == 2 ? 2 * per_cta + 1 : per_cta);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if constexpr (POST) {  // padding rows above the weights (read only for rows that are not output)
    for (int i = threadIdx.x; i < (G::BN / 8) * G::PS_PAD * 4; i += kThreads)
      reinterpret_cast<uint32_t *>(Ps + (i / (G::PS_PAD * 4)) * G::PS_STRIP)[i % (G::PS_PAD * 4)] = 0u;
  }
  if (warp == kMmaWarp) { tmem_alloc(tslot, G::TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  if (MIX == 2) cluster_sync_all();  // the peer's barriers are initialised before remote arrivals
  tc_fence_after();
  const uint32_t tmem = *tslot;
  // launched as the prepasses' programmatic dependent: everything above overlapped
  // their tail; from here on their outputs (convolved keys and values, column
  // factors, dot products) are complete and visible
  pdl_wait_primary();

  if (warp == kTmaWarp || warp == kTma2Warp) {
    // -------------------------------------------------------------- TMA
    if (warp == kTmaWarp && lane == 0) {  // Kt chunks (and with POST the convolved values), through the ring
      prefetch_tmap(&tmK);
      if (POST) prefetch_tmap(&tmVt);
      int cnt = 0;
      // one ring stage: SB boxes, box bx at (x[bx], y, z[bx])
      auto push = [&](const CUtensorMap *map, const int (&x)[G::SB], int y, const int (&z)[G::SB]) -> bool {
        const int st = cnt % G::NS;
        if (!mbar_wait(k_empty + st, ((cnt / G::NS) & 1) ^ 1, abort_flag, p.err)) return false;
        mbar_arrive_expect_tx(k_full + st, G::KSTAGE);
#pragma unroll
        for (int bx = 0; bx < G::SB; ++bx)
          tma_load_3d(Ks + st * G::KSTAGE + bx * G::KCHUNK, map, k_full + st, x[bx], y, z[bx]);
        ++cnt;
        return true;
      };
      Item it;
      bool ok = true;
      // the cluster's first CTA takes the items from the queue; the second reads them
      for (int r = 0; ok && !*abort_flag && (hr == 0 ? publish_item(r, it) : take_item(r, it, true)); ++r) {
        const int h = it.g * CL + hr, n_kv = kv_tiles(it), nsl = n_slots(it);
        auto load_c = [&](int t) -> bool {
          for (int ch = 0; ch < G::NSRC * G::NCH; ch += G::SB) {
            const int sc = ch / G::NCH, zh = it.b * p.H + src_head(h, sc);
            int x[G::SB], z[G::SB];
#pragma unroll
            for (int bx = 0; bx < G::SB; ++bx) {
              const int cs = ch % G::NCH + bx;
              x[bx] = D % 64 == 0 ? (cs % G::NDC) * 64 : 0;
              z[bx] = D % 64 == 0 ? zh * CQ + cs / G::NDC : zh * G::NCH + cs;
            }
            if (!push(&tmK, x, t * G::BN, z)) return false;
          }
          return true;
        };
        auto load_pv = [&](int t) -> bool {  // chunk (value head hd, tap row a, 64-channel block dc)
          for (int ch = 0; ch < G::NVCH; ch += G::SB) {
            int x[G::SB], z[G::SB];
#pragma unroll
            for (int bx = 0; bx < G::SB; ++bx) {
              const int c2 = ch + bx, hd = c2 / (CQ * G::NDC), a = (c2 / G::NDC) % CQ, dc = c2 % G::NDC;
              x[bx] = dc * 64;
              z[bx] = ((it.b * p.H + h) * G::NV + hd) * CQ + a;
            }
            if (!push(&tmVt, x, t * G::BN, z)) return false;
          }
          return true;
        };
        // the order the MMA issuer consumes: C of slot s+1 before P V of slot s
        for (int sl = 0; ok && sl < nsl && !*abort_flag; ++sl) {
          ok = load_c(sl % n_kv);
          if (POST && ok && sl >= n_kv + 1) ok = load_pv(sl - 1 - n_kv);
        }
        if (POST && ok && !*abort_flag) ok = load_pv(n_kv - 1);
      }
      if (*abort_flag)  // copies still in flight land before the CTA exits
        for (int c2 = (cnt > G::NS ? cnt - G::NS : 0); c2 < cnt; ++c2)
          drain_wait(k_full + c2 % G::NS, (c2 / G::NS) & 1);
    } else if (warp == kTma2Warp && lane == 0 && !POST) {  // V of both heads of the group, per key tile
      prefetch_tmap(&tmV);
      int nv = 0;
      Item it;
      for (int r = 0; !*abort_flag && take_item(r, it, true); ++r) {
        const int h = it.g * CL + hr, n_kv = kv_tiles(it);
        for (int t = 0; t < n_kv; ++t, ++nv) {
          if (!mbar_wait(v_empty, (nv & 1) ^ 1, abort_flag, p.err)) break;
          mbar_arrive_expect_tx(v_full, G::V_BYTES);
#pragma unroll
          for (int hd = 0; hd < G::NV; ++hd)
#pragma unroll
            for (int dc = 0; dc < G::NDC; ++dc)
              tma_load_4d(Vs + hd * G::V_HEAD + dc * G::V_CHUNK, &tmV, v_full, dc * 64,
                          G::NV == 2 ? 2 * it.g + hd : h, t * G::BN, it.b);
        }
      }
      if (*abort_flag && nv) drain_wait(v_full, (nv - 1) & 1);
    } else if (warp == kTma2Warp && lane == 1) {  // the query rows of each item, once the previous item's C is done
      prefetch_tmap(&tmQ);
      int nq = 0;
      Item it;
      for (int r = 0; !*abort_flag && take_item(r, it, true); ++r, ++nq) {
        if (r > 0 && !mbar_wait(q_free, (r - 1) & 1, abort_flag, p.err)) break;
        const int h = it.g * CL + hr, row0 = row_start(it) - G::HALO;
        mbar_arrive_expect_tx(q_full, G::NSRC * G::Q_BYTES);
#pragma unroll 1
        for (int sc = 0; sc < G::NSRC; ++sc)
#pragma unroll 1
          for (int s2 = 0; s2 < G::NSTRIP; ++s2)
            tma_load_4d(Qs + sc * G::Q_ALLOC + s2 * G::STRIP, &tmQ, q_full, 8 * s2, src_head(h, sc), row0, it.b);
      }
      if (nq) drain_wait(q_full, (nq - 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // -------------------------------------------------------------- MMA
    // The whole warp runs the issuing loop; one elected lane issues the instructions.
    {
      const bool issuer = elect_one();
      // waits of the issuing loop, made warp-uniform (all lanes poll the same barrier)
      auto wwait = [&](uint64_t *bar, uint32_t ph) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, ph, abort_flag, p.err));
      };
      auto take_mma = [&](int r, Item &x) -> bool {
        const bool got = __all_sync(0xffffffffu, take_item(r, x, lane == 0));
        __syncwarp();
        return got;
      };
      const uint32_t idesc_c = idesc_f16_f32(128, G::BN);
      const uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      // descriptors of the first operand tiles; every other tile differs only in its
      // start address (field bits 0-13, address / 16), added below
      const uint64_t qdesc0 = sdesc_noswz(smem_u32(Qs), G::STRIP, 128);
      const uint64_t kdesc0 = sdesc_sw128(smem_u32(Ks), 16, 1024);
      const uint64_t vdesc0 = sdesc_sw128(smem_u32(Vs), G::V_CHUNK, 1024);
      // POST: weights in shared memory (row shift a = 16a bytes earlier) times the
      // convolved values in the ring (N = 64 channels per chunk)
      const uint32_t idesc_pv64 = idesc_bf16_f32(128, 64, 0, 1);
      const uint64_t psdesc0 = sdesc_noswz(smem_u32(Ps), G::PS_STRIP, 128);
      const uint64_t vtdesc0 = sdesc_sw128(smem_u32(Ks), G::KCHUNK, 1024);  // a ring stage as MN-major B
      int cnt = 0, T = 0;  // ring chunks and C tiles issued so far (all items)
      int npv = 0;         // P V tiles issued (POST)
      bool ok = true;
      // C of global key tile T = sum over the NCH 64-element chunks of the c_q*D
      // contraction; element kappa = a*D + e pairs Q shifted by a rows with Kt_a
      // DB: into buffer T & 1 without waiting for the softmax (the buffer's previous
      // tile, T - 2, had its P V issued before, and MMAs run in issue order)
      auto issue_c = [&](bool last_of_item) -> bool {
        if constexpr (!G::DB) {
          if constexpr (G::CDB) {  // the softmax has read the buffer's previous tile, T - 2
            if (T >= 2 && !wwait(c_freeb[T & 1], ((T - 2) >> 1) & 1)) return false;
          } else if (T > 0 && !wwait(c_free, (T - 1) & 1)) {
            return false;
          }
        }
        const uint32_t c_dst = tmem + G::C_COL + ((G::CDB && (T & 1)) ? G::CB1 : 0u);
        for (int ch = 0; ch < G::NSRC * G::NCH; ch += G::SB, ++cnt) {
          const int st = cnt % G::NS;
          // source head sc (its own accumulator and query rows); the 16 elements
          // kappa = 64 cs + 16 kk of step kk: tap row a, channels e0 .. e0+15 (D is a
          // multiple of 16, so a step never straddles two tap rows); Q rows shifted up
          // by a (16 bytes per row), 8-channel strips e0/8 and e0/8 + 1
          if constexpr (D % 64 == 0) {
            if (!wwait(k_full + st, (cnt / G::NS) & 1)) return false;
            tc_fence_after();
            // box bx of the stage is chunk cs: tap row a = cs / NDC, channels 64 dc ..
            // 64 dc + 63 (a stage is a whole tap row when SB = NDC)
            const int sc = ch / G::NCH;
            const uint64_t kd = kdesc0 + static_cast<uint32_t>((st * G::KSTAGE) >> 4);
#pragma unroll
            for (int bx = 0; bx < G::SB; ++bx) {
              const int cs = ch % G::NCH + bx, a = cs / G::NDC, dc = cs % G::NDC;
              const uint64_t qd = qdesc0 + static_cast<uint32_t>((sc * G::Q_ALLOC + 8 * dc * G::STRIP + 16 * (G::HALO - a)) >> 4);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ss_if(issuer, c_dst + 128 * sc, qd + (2 * kk * G::STRIP >> 4),
                            kd + (bx * G::KCHUNK >> 4) + 2 * kk, idesc_c, (cs > 0 || kk > 0));
            }
          } else {
            const int sc = ch / G::NCH, cs = ch % G::NCH;
            const uint64_t kd = kdesc0 + static_cast<uint32_t>((st * G::KSTAGE) >> 4);
            uint64_t qd[4];
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const int kap = 64 * cs + 16 * kk, a = kap / D, e0 = kap % D;
              qd[kk] = qdesc0 + static_cast<uint32_t>((sc * G::Q_ALLOC + (e0 / 8) * G::STRIP + 16 * (G::HALO - a)) >> 4);
            }
            if (!wwait(k_full + st, (cnt / G::NS) & 1)) return false;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss_if(issuer, c_dst + 128 * sc, qd[kk], kd + 2 * kk, idesc_c, (cs > 0 || kk > 0));
          }
          mma_commit_if(issuer, k_empty + st);
        }
        mma_commit_if(issuer, G::CDB ? c_fullb[T & 1] : c_full);
        if (last_of_item) mma_commit_if(issuer, q_free);  // the query buffer may take the next item
        return true;
      };
      // Z_hd += sum_a (weights shifted down by a rows) x Vt_{hd,a}, from the ring
      auto issue_pv = [&](bool first_of_item) -> bool {
        for (int ch = 0; ch < G::NVCH; ch += G::SB, ++cnt) {
          const int st = cnt % G::NS;
          if (!wwait(k_full + st, (cnt / G::NS) & 1)) return false;
          tc_fence_after();
          if constexpr (G::SB == 2) {
            // the stage holds both 64-channel boxes of (hd, a): one N = 128 MMA per key step
            const int hd = ch / (CQ * G::NDC), a = (ch / G::NDC) % CQ;
            const uint64_t pd = psdesc0 + static_cast<uint32_t>(G::PS_PAD - a);
            const uint64_t vd = vtdesc0 + static_cast<uint32_t>((st * G::KSTAGE) >> 4);
#pragma unroll
            for (int kk = 0; kk < G::BN / 16; ++kk)
              mma_ss_if(issuer, tmem + G::Z_COL0 + 128 * hd, pd + static_cast<uint32_t>((2 * kk * G::PS_STRIP) >> 4),
                          vd + static_cast<uint32_t>((kk * 16 * 128) >> 4), idesc_bf16_f32(128, 128, 0, 1),
                          !(first_of_item && a == 0 && kk == 0));
          } else {
#pragma unroll
            for (int bx = 0; bx < G::SB; ++bx) {
              const int c2 = ch + bx, hd = c2 / (CQ * G::NDC), a = (c2 / G::NDC) % CQ, dc = c2 % G::NDC;
              const uint64_t pd = psdesc0 + static_cast<uint32_t>(G::PS_PAD - a);
              const uint64_t vd = vtdesc0 + static_cast<uint32_t>((st * G::KSTAGE + bx * G::KCHUNK) >> 4);
#pragma unroll
              for (int kk = 0; kk < G::BN / 16; ++kk)
                mma_ss_if(issuer, tmem + G::Z_COL0 + 128 * hd + 64 * dc, pd + static_cast<uint32_t>((2 * kk * G::PS_STRIP) >> 4),
                            vd + static_cast<uint32_t>((kk * 16 * 128) >> 4), idesc_pv64,
                            !(first_of_item && a == 0 && kk == 0));
            }
          }
          mma_commit_if(issuer, k_empty + st);
        }
        mma_commit_if(issuer, v_empty);
        return true;
      };
      Item it;
      for (int r = 0; ok && take_mma(r, it); ++r) {
        const int n_kv = kv_tiles(it), nsl = n_slots(it);
        if (!wwait(q_ready, r & 1)) break;
        if constexpr (G::DB) {
          // C of the first two tiles, then per tile: P V, and C two tiles ahead into
          // the buffer that P V has just consumed
          const int T0 = T;
          ok = issue_c(nsl == 1);
          if (ok && nsl > 1) {
            T = T0 + 1;
            ok = issue_c(nsl == 2);
          }
          for (int sl = 0; ok && sl < nsl; ++sl) {
            const int Tt = T0 + sl;
            if (!wwait(p_fullb[Tt & 1], (Tt >> 1) & 1)) { ok = false; break; }
            if (!wwait(v_full, Tt & 1)) { ok = false; break; }
            if (sl == 0 && r > 0 && !wwait(z_free, (r - 1) & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t pcol = tmem + 128u * (Tt & 1);
            if constexpr (G::NV * G::NDC * 64 == 256) {
#pragma unroll
              for (int kk = 0; kk < G::BN / 16; ++kk)
                mma_ts_if(issuer, tmem + G::Z_COL0, pcol + 8 * kk, vdesc0 + ((kk * 16 * 128) >> 4),
                           idesc_bf16_f32(128, 256, 0, 1), (sl > 0 || kk > 0));
            } else {
#pragma unroll
              for (int hd = 0; hd < G::NV; ++hd)
#pragma unroll
                for (int kk = 0; kk < G::BN / 16; ++kk)
                  mma_ts_if(issuer, tmem + G::Z_COL0 + 128 * hd, pcol + 8 * kk,
                             vdesc0 + ((hd * G::V_HEAD + kk * 16 * 128) >> 4), idesc_pv, (sl > 0 || kk > 0));
            }
            mma_commit_if(issuer, v_empty);
            if (sl + 2 < nsl) {
              T = Tt + 2;
              ok = issue_c(sl + 3 == nsl);
            }
          }
          T = T0 + nsl;
          continue;
        }
        const int T0 = T;
        ok = issue_c(nsl == 1);
        for (int sl = 0; ok && sl < nsl; ++sl) {
          const int Tt = T0 + sl;
          if (sl + 1 < nsl) {
            T = Tt + 1;
            if (!issue_c(sl + 2 == nsl)) { ok = false; break; }
          }
          if constexpr (POST) {
            if (sl < n_kv) continue;  // first pass: statistics only
            if (!wwait(p_full, npv & 1)) { ok = false; break; }
            if (sl == n_kv && r > 0 && !wwait(z_free, (r - 1) & 1)) { ok = false; break; }
            tc_fence_after();
            if (!issue_pv(sl == n_kv)) { ok = false; break; }
            ++npv;
          } else {
            const int t = sl;
            if (!wwait(p_full, Tt & 1)) { ok = false; break; }
            if (!wwait(v_full, Tt & 1)) { ok = false; break; }
            // Z is overwritten (accumulate off) by the first P V of an item: the previous
            // item's epilogue must have read it
            if (t == 0 && r > 0 && !wwait(z_free, (r - 1) & 1)) { ok = false; break; }
            tc_fence_after();
            if constexpr (G::NV * G::NDC * 64 == 256) {
              // both heads' V tiles are four consecutive 64-channel boxes and both Z
              // accumulators 256 consecutive columns: one N = 256 MMA per key step
#pragma unroll
              for (int kk = 0; kk < G::BN / 16; ++kk)
                mma_ts_if(issuer, tmem + G::Z_COL0, tmem + G::P_COL + 8 * kk, vdesc0 + ((kk * 16 * 128) >> 4),
                           idesc_bf16_f32(128, 256, 0, 1), (t > 0 || kk > 0));
            } else {
#pragma unroll
              for (int hd = 0; hd < G::NV; ++hd)
#pragma unroll
                for (int kk = 0; kk < G::BN / 16; ++kk)
                  mma_ts_if(issuer, tmem + G::Z_COL0 + 128 * hd, tmem + G::P_COL + 8 * kk,
                             vdesc0 + ((hd * G::V_HEAD + kk * 16 * 128) >> 4), idesc_pv, (t > 0 || kk > 0));
            }
            mma_commit_if(issuer, v_empty);
          }
        }
        T = T0 + nsl;
      }
      mma_commit_if(issuer, mma_done);
      drain_wait(mma_done, 0);
    }
  } else {
    // ---------------------------------------------- softmax warpgroups
    const int wg = warp >> 2, q4 = warp & 3;
    const int r_ = 32 * q4 + lane;           // query row of this thread = TMEM lane
    const int st_id = threadIdx.x;           // 0..255
    const int cb = G::HALF * wg;             // key columns of this warpgroup
    const int zc = G::DH * wg;               // output channels of this warpgroup: zc .. zc+zn-1
    const int zn = G::DH1 == G::DH ? G::DH : (wg ? G::DH1 : G::DH);  // a constant unless d = 96
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q4) << 16);
    const float sc0 = p.qk_scale * kLog2e;
    float *brow = Cs + r_ * G::W;             // this row of the item's band table

    // Stage item r: its query rows in fp16 (scaled down by a power of 2 only if
    // |q| > 2^14), the past dot products of its staged rows and its kernel taps.
    // Returns the query exponent.
    auto prepare = [&](int r, const Item &it) -> int {
      const int h = it.g * CL + hr, row0 = row_start(it) - G::HALO;
      mbar_wait(q_full, r & 1, abort_flag, p.err);
      float qmax = 0.f;
      // (the query tiles of the source heads lie Q_ALLOC = Q_BYTES apart)
      static_assert(G::Q_ALLOC == G::Q_BYTES, "contiguous query tiles");
      for (int c16 = st_id; c16 < G::NSRC * G::Q_BYTES / 16; c16 += kSmThreads) {
        const uint4 raw = *reinterpret_cast<const uint4 *>(Qs + 16 * c16);
        const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          qmax = fmaxf(qmax, fmaxf(fabsf(__low2float(p2[u])), fabsf(__high2float(p2[u]))));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, o));
      if (lane == 0) qred[warp] = qmax;
      named_bar_sync(kBarAll, kSmThreads);
#pragma unroll
      for (int i = 0; i < 8; ++i) qmax = fmaxf(qmax, qred[i]);
      int eq = 0;
      if (qmax > 16384.f) eq = max(-60, static_cast<int>(floorf(log2f(16384.f / qmax))));
      const float qsc = exp2f(static_cast<float>(eq));
      for (int c16 = st_id; c16 < G::NSRC * G::Q_BYTES / 16; c16 += kSmThreads) {
        uint4 raw = *reinterpret_cast<const uint4 *>(Qs + 16 * c16);
        __nv_bfloat162 *p2 = reinterpret_cast<__nv_bfloat162 *>(&raw);
        uint4 o;
        uint32_t *ow = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          __half2 hv = __floats2half2_rn(__low2float(p2[u]) * qsc, __high2float(p2[u]) * qsc);
          ow[u] = *reinterpret_cast<uint32_t *>(&hv);
        }
        *reinterpret_cast<uint4 *>(Qs + 16 * c16) = o;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
#pragma unroll 1
      for (int sc = 0; sc < G::NSRC; ++sc) {
        const int hs = src_head(h, sc);
        const long long bh = static_cast<long long>(it.b) * p.H + hs;
        float *us = Us + sc * (G::U_BYTES / 4);
        // the staged rows are contiguous in Vp: every load of a thread is issued
        // before any of them is stored, so their latencies overlap
        constexpr int NU = (G::UROWS * G::M + kSmThreads - 1) / kSmThreads;
        const float *vsrc = p.vp + (bh * L + row0) * G::M;
        float vt[NU];
#pragma unroll
        for (int u = 0; u < NU; ++u) {
          const int e = st_id + u * kSmThreads, iq = row0 + e / G::M;
          vt[u] = (e < G::UROWS * G::M && iq >= 0 && iq < L) ? vsrc[e] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < NU; ++u) {
          const int e = st_id + u * kSmThreads;
          if (e < G::UROWS * G::M) us[e] = vt[u];
        }
        if (st_id < CQ * CK)
          th_s[((r & 1) * G::NSRC + sc) * 128 + st_id] = p.theta[static_cast<long long>(hs) * CQ * CK + st_id];
      }
      if (POST && st_id < CQ * CK)  // the post-softmax kernel of this CTA's head
        thp_s[(r & 1) * 128 + st_id] = p.theta_post[static_cast<long long>(h) * CQ * CK + st_id];
      return eq;
    };

    // exchange buffer slot of CTA (cluster cc, head rank hh) for items of parity par:
    // part 0 = for the peer head, part 1 (DEFER) = its own head's part
    auto xslot = [&](int cc, int hh, int par, int part) -> float4 * {
      return reinterpret_cast<float4 *>(p.xg) +
             ((static_cast<long long>(2 * cc + hh) * 2 + par) * 2 + part) * (G::BM * D / 4);
    };
    // DEFER: the item whose epilogue is still to be finished
    bool pend = false;
    int pend_r = 0;
    Item pend_it{0, 0, 0};
    // the rest of item pr's epilogue: its own part plus the peer's, group norm and
    // depth scale (or gate), bf16 store
    auto finish = [&](int pr, const Item &pi) {
      const int ph = pi.g * CL + hr, pg = pi.g;
      const int pq = row_start(pi) + r_;
      const bool pout = pq >= 0 && pq < L && r_ >= G::RSH;
      mbar_wait_cluster(x_readyb[pr & 1], (pr >> 1) & 1, abort_flag, p.err);
      const float4 *own = xslot(c, hr, pr & 1, 1);
      const float4 *theirs = xslot(c, hr ^ 1, pr & 1, 0);
      const float w_peer = p.w[pg * 4 + hr * 2 + (hr ^ 1)];
      float o[G::DH];
#pragma unroll
      for (int c4 = 0; c4 < G::DH / 4; ++c4) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f), y = x;
        if (4 * c4 < zn) {
          x = own[(zc / 4 + c4) * G::BM + r_];
          y = theirs[(zc / 4 + c4) * G::BM + r_];
        }
        o[4 * c4] = x.x + w_peer * y.x;
        o[4 * c4 + 1] = x.y + w_peer * y.y;
        o[4 * c4 + 2] = x.z + w_peer * y.z;
        o[4 * c4 + 3] = x.w + w_peer * y.w;
      }
      if (p.gn) {
        float s1 = 0.f;
#pragma unroll
        for (int i = 0; i < G::DH; ++i) s1 += o[i];  // channels past zn are 0
        red[(6 + wg) * G::BM + r_] = s1;
        named_bar_sync(kBarAll, kSmThreads);
        const float mu = (s1 + red[(6 + (wg ^ 1)) * G::BM + r_]) * (1.f / D);
        float s2 = 0.f;
#pragma unroll
        for (int i = 0; i < G::DH; ++i) { const float x = i < zn ? o[i] - mu : 0.f; s2 += x * x; }
        red[(8 + wg) * G::BM + r_] = s2;
        named_bar_sync(kBarAll, kSmThreads);
        const float rstd = rsqrtf((s2 + red[(8 + (wg ^ 1)) * G::BM + r_]) * (1.f / D) + p.eps);
        const float *gm = p.gamma + static_cast<long long>(ph) * D + zc;
        const float *bt = p.beta + static_cast<long long>(ph) * D + zc;
        const float mh = head_multiplier(p.gate, p.lam, ph);
#pragma unroll
        for (int i = 0; i < G::DH; ++i)
          if (i < zn) o[i] = ((o[i] - mu) * rstd * gm[i] + bt[i]) * mh;
      }
      if (pout) {
        __nv_bfloat16 *dst = p.out + ((static_cast<long long>(pi.b) * L + pq) * p.H + ph) * D + zc;
#pragma unroll
        for (int i = 0; i < G::DH; i += 8) {
          if (i >= zn) break;
          uint4 v;
          v.x = pack_bf16x2(o[i], o[i + 1]);
          v.y = pack_bf16x2(o[i + 2], o[i + 3]);
          v.z = pack_bf16x2(o[i + 4], o[i + 5]);
          v.w = pack_bf16x2(o[i + 6], o[i + 7]);
          *reinterpret_cast<uint4 *>(dst + i) = v;
        }
      }
    };

    int T = 0;   // C tiles processed so far (all items, both passes with POST)
    int NP = 0;  // weight tiles handed to the P V issuer so far (POST)
    Item it, nx;
    // every softmax thread reads the ring; lane 0 of each warp frees the slot
    auto take_sm = [&](int r, Item &x) -> bool {
      const bool got = take_item(r, x, false);
      __syncwarp();
      if (lane == 0) {
        const int s = r % kItemSlots;
        if (CL == 2 && hr != 0)
          mbar_arrive_cluster(map_peer(smem_u32(it_empty + s), 0u));
        else
          mbar_arrive(it_empty + s);
      }
      return got;
    };
    bool have = take_sm(0, it);
    int eq = 0;
    if (have) {
      eq = prepare(0, it);
      const int h0 = it.g * CL + hr;
      if (st_id < G::BN)
#pragma unroll
        for (int sc = 0; sc < G::NSRC; ++sc)
          facs[sc * 2 * G::BN + st_id] = p.fac[(static_cast<long long>(it.b) * p.H + src_head(h0, sc)) * p.lpad + st_id];
      named_bar_sync(kBarAll, kSmThreads);
    }
    for (int r = 0; have; ++r) {
      const int h = it.g * CL + hr, g = it.g;
      const int R0 = row_start(it), qi = R0 + r_;
      const bool row_ok = qi >= 0 && qi < L;          // a query of the sequence
      const bool out_row = row_ok && r_ >= G::RSH;     // an output row of this tile
      const int n_kv = kv_tiles(it), nsl = n_slots(it);
      // the next item, read from the ring at this item's last key tile
      bool more = false, nx_known = false;
      auto fetch_next = [&]() {
        if (!nx_known) {
          more = take_sm(r + 1, nx);
          nx_known = true;
        }
      };
      // column factors of source s for the key tile of the slot after sl (this item's;
      // the next item's first tile's are loaded after the slot loop)
      auto fac_next = [&](int sc, int sl) -> float {
        if (sl + 1 < nsl)
          return p.fac[(static_cast<long long>(it.b) * p.H + src_head(h, sc)) * p.lpad +
                       (POST ? (sl + 1) % n_kv : sl + 1) * G::BN + st_id];
        return 0.f;
      };
      const float qinv = exp2f(static_cast<float>(-eq));
      // pre-softmax mixing weights of the sources: w[g][destination][source]
      float wmix[G::NSRC];
#pragma unroll
      for (int sc = 0; sc < G::NSRC; ++sc) wmix[sc] = G::NSRC == 2 ? p.w[(h >> 1) * 4 + (h & 1) * 2 + sc] : 1.f;
      // the band 0 <= i-j < W, where the mask removes taps: the convolution tap by
      // tap over the kept taps, from the dot products (key (i-a) - m, m = dd - a + t - c):
      //   Mask_0: taps with m >= 0; exact indicator: taps with key <= i, i.e. t >= c - dd
      //   C[i][i-dd] = s * sum_{kept a,t} theta[a][t] q[i-a] . k[i-a-m]   (acc[dd] / s)
      // Each warpgroup takes half of the W diagonals of its row, once per item, into
      // the band table brow[dd] (log2 units; read by both warpgroups after a barrier).
      auto band_part = [&](auto lo_c) {
        constexpr int LO = decltype(lo_c)::value, NB = LO == 0 ? (G::W + 1) / 2 : G::W - (G::W + 1) / 2;
        float acc[NB];
#pragma unroll
        for (int e = 0; e < NB; ++e) acc[e] = 0.f;
#pragma unroll
        for (int sc = 0; sc < G::NSRC; ++sc)
#pragma unroll
        for (int a = 0; a < CQ; ++a) {
          // rows before query 0 are zero; the source's taps carry its mixing weight
          const float *vrow = Us + sc * (G::U_BYTES / 4) + (r_ + G::HALO - a) * G::M;
          const float *th = th_s + ((r & 1) * G::NSRC + sc) * 128;
          float vr[G::M];
#pragma unroll
          for (int m = 0; m < G::M; ++m) vr[m] = vrow[m];
#pragma unroll
          for (int tp = 0; tp < CK; ++tp) {
            const float thv = th[a * CK + tp] * wmix[sc];
#pragma unroll
            for (int e = 0; e < NB; ++e) {
              const int dd = LO + e, m = dd - a + tp - G::C;
              const bool kept = EXACT ? tp >= G::C - dd : m >= 0;
              if (kept && m + G::OFF >= 0 && m + G::OFF < G::M) acc[e] = fmaf(thv, vr[m + G::OFF], acc[e]);
            }
          }
        }
#pragma unroll
        for (int e = 0; e < NB; ++e) brow[LO + e] = acc[e] * sc0;
      };
      float m_run = -INFINITY, l_run = 0.f;
      float mm = INFINITY;  // POST: log2 of (row max x row sum), final after the first pass
      // column factors two slots ahead: loaded a whole tile before they are stored
      float fpre[G::NSRC];
#pragma unroll
      for (int sc = 0; sc < G::NSRC; ++sc) fpre[sc] = st_id < G::BN ? fac_next(sc, 0) : 0.f;
      for (int sl = 0; sl < nsl; ++sl, ++T) {
        const int t = POST ? sl % n_kv : sl;
        const bool pass2 = POST && sl >= n_kv;
        const int j0 = t * G::BN;
        if (POST && sl == n_kv) {  // exact statistics of the row: one normaliser for the second pass
          red[(4 + wg) * G::BM + r_] = l_run;
          named_bar_sync(kBarAll, kSmThreads);
          const float l_tot = l_run + red[(4 + (wg ^ 1)) * G::BM + r_];
          mm = (row_ok && l_tot > 0.f) ? m_run + log2f(l_tot) : INFINITY;
        }
        // the band table of the item, while the first C is computed
        if (sl == 0) {
          if (row_ok) {
            if (wg == 0)
              band_part(std::integral_constant<int, 0>());
            else
              band_part(std::integral_constant<int, (G::W + 1) / 2>());
          }
          named_bar_sync(kBarAll, kSmThreads);
        }
        // next key tile's column factors (stored before this tile's barrier, read after
        // it), and the load of the one after
        float fnext[G::NSRC];
#pragma unroll
        for (int sc = 0; sc < G::NSRC; ++sc) {
          fnext[sc] = fpre[sc];
          fpre[sc] = st_id < G::BN ? fac_next(sc, sl + 1) : 0.f;
        }
        if constexpr (G::CDB)
          mbar_wait(c_fullb[T & 1], (T >> 1) & 1, abort_flag, p.err);
        else
          mbar_wait(c_full, T & 1, abort_flag, p.err);
        tc_fence_after();
        const uint32_t cbuf = (G::CDB && (T & 1)) ? G::CB1 : 0u;  // this tile's C (and, with DB, P) buffer
        // C' = sum over source heads of w * (C_s x its column factors); one source without mixing
        float cv[G::HALF];
#pragma unroll
        for (int sc = 0; sc < G::NSRC; ++sc) {
          const float4 *f4 = reinterpret_cast<const float4 *>(facs + (sc * 2 + (T & 1)) * G::BN + cb);
          // both 32-column halves in flight before one wait
          uint32_t u32[2][32];
          tmem_ld32(tl + G::C_COL + cbuf + 128 * sc + cb, u32[0]);
          tmem_ld32(tl + G::C_COL + cbuf + 128 * sc + cb + 32, u32[1]);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < G::HALF / 4; ++i) {
            float4 f = f4[i];
            if (G::NSRC == 2) { f.x *= wmix[sc]; f.y *= wmix[sc]; f.z *= wmix[sc]; f.w *= wmix[sc]; }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float fe = e == 0 ? f.x : e == 1 ? f.y : e == 2 ? f.z : f.w;
              const float x = __uint_as_float(u32[i / 8][4 * (i % 8) + e]) * fe;
              cv[4 * i + e] = sc == 0 ? x : cv[4 * i + e] + x;
            }
          }
        }
        tc_fence_before();  // (with DB: orders the C reads before the barrier that precedes the P writes)
        if constexpr (!G::DB) {  // with DB the buffer is reused only after this tile's P V
          __syncwarp();
          if (lane == 0) mbar_arrive(G::CDB ? c_freeb[T & 1] : c_free);
        }
        if (eq != 0) {  // queries were scaled down (|q| > 2^14)
#pragma unroll
          for (int jj = 0; jj < G::HALF; ++jj) cv[jj] *= qinv;
        }
        const int dmax = qi - j0 - cb;  // i - j for this warpgroup's first column
        if (row_ok && dmax >= 0 && dmax - (G::W - 1) < G::HALF) {
#pragma unroll
          for (int jj = 0; jj < G::HALF; ++jj) {
            const int dd = dmax - jj;
            if (static_cast<unsigned>(dd) < static_cast<unsigned>(G::W)) cv[jj] = brow[dd];
          }
        }
        // Mask_-inf: keys after the query (only tiles reaching past the tile's first row)
        if (j0 + G::BN - 1 > R0) {
#pragma unroll
          for (int jj = 0; jj < G::HALF; ++jj)
            if (j0 + cb + jj > qi) cv[jj] = -INFINITY;
        }
        if (!pass2) {
          // the row max over both warpgroups' columns (log2 units)
          float *rmx = red + (T & 1) * 2 * G::BM;
          rmx[wg * G::BM + r_] = row_ok ? tree_max<G::HALF>(cv) : -INFINITY;
          if (st_id < G::BN)
#pragma unroll
            for (int sc = 0; sc < G::NSRC; ++sc) facs[(sc * 2 + ((T + 1) & 1)) * G::BN + st_id] = fnext[sc];
          named_bar_sync(kBarAll, kSmThreads);
          tc_fence_after();  // both warpgroups have read this tile's C (P may overwrite it)
          const float mt = fmaxf(rmx[r_], rmx[G::BM + r_]);
          const float m_new = fmaxf(m_run, mt);
          if constexpr (POST) {  // first pass: row sums only
            if (m_new != -INFINITY) {
              float ls = 0.f;
#pragma unroll
              for (int jj = 0; jj < G::HALF; ++jj) ls += ex2(cv[jj] - m_new);
              l_run = l_run * ex2(m_run - m_new) + ls;
              m_run = m_new;
            }
          } else {
            bool resc = false;
            float alpha = 1.f;
            if (t == 0) {
              m_run = m_new;
            } else if (m_new > m_run + kRescaleLog2) {
              resc = true;
              alpha = ex2(m_run - m_new);
              m_run = m_new;
            }
            if (T > 0) {  // P and Z of the previous key tile are consumed / complete
              mbar_wait(v_empty, (T - 1) & 1, abort_flag, p.err);
              tc_fence_after();
            }
            if (__any_sync(0xffffffffu, resc)) {  // warp-collective tensor-memory access
              l_run *= alpha;
#pragma unroll 1
              for (int hd = 0; hd < G::NV; ++hd)
#pragma unroll 1
                for (int c0 = 0; c0 < G::DH; c0 += 32) {
                  if (c0 >= zn) break;
                  uint32_t z[32];
                  const uint32_t za = tl + G::Z_COL0 + 128 * hd + zc + c0;
                  tmem_ld32(za, z);
                  tmem_wait_ld();
#pragma unroll
                  for (int i = 0; i < 32; ++i) z[i] = __float_as_uint(__uint_as_float(z[i]) * alpha);
                  tmem_st32(za, z);
                }
            }
            float ls = 0.f;
            uint32_t pk[32];
#pragma unroll
            for (int q2 = 0; q2 < 32; ++q2) {
              const float p0 = row_ok ? ex2(cv[2 * q2] - m_run) : 0.f;
              const float p1 = row_ok ? ex2(cv[2 * q2 + 1] - m_run) : 0.f;
              ls += p0 + p1;
              pk[q2] = pack_bf16x2(p0, p1);
            }
            // (with DB, over this tile's C: both warpgroups have read it, see the barrier above)
            tmem_st32(tl + G::P_COL + cbuf + 32 * wg, pk);
            l_run += ls;
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(G::DB ? p_fullb[T & 1] : p_full);
            if constexpr (G::DEFER) {
              // the previous item's epilogue, while this tile's P V and the next C run
              if (pend && sl == 0) {
                finish(pend_r, pend_it);
                pend = false;
              }
            }
          }
        } else {
          // second pass: normalised weights A = 2^(C - mm); the c keys ending at the
          // diagonal go through the band below (their convolved values would reach
          // past the query), so they are 0 here
          if (st_id < G::BN)
#pragma unroll
            for (int sc = 0; sc < G::NSRC; ++sc) facs[(sc * 2 + ((T + 1) & 1)) * G::BN + st_id] = fnext[sc];
          named_bar_sync(kBarAll, kSmThreads);
          const bool cut = j0 + G::BN - 1 > R0 - G::C;
          uint32_t pk[32];
#pragma unroll
          for (int q2 = 0; q2 < 32; ++q2) {
            float p0 = ex2(cv[2 * q2] - mm), p1 = ex2(cv[2 * q2 + 1] - mm);
            if (cut) {
              if (j0 + cb + 2 * q2 > qi - G::C) p0 = 0.f;
              if (j0 + cb + 2 * q2 + 1 > qi - G::C) p1 = 0.f;
            }
            pk[q2] = pack_bf16x2(p0, p1);
          }
          if (NP > 0) mbar_wait(v_empty, (NP - 1) & 1, abort_flag, p.err);  // the previous P V read the buffer
          uint8_t *prow = Ps + (cb / 8) * G::PS_STRIP + 16 * (r_ + G::PS_PAD);
#pragma unroll
          for (int k8 = 0; k8 < G::HALF / 8; ++k8)
            *reinterpret_cast<uint4 *>(prow + k8 * G::PS_STRIP) =
                make_uint4(pk[4 * k8], pk[4 * k8 + 1], pk[4 * k8 + 2], pk[4 * k8 + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_full);
          ++NP;
        }
      }
      if constexpr (POST) {
        // normalised weights of the c keys ending at each row's diagonal, for the band
        if (wg == 0) {
#pragma unroll
          for (int dl = 0; dl < G::C; ++dl)
            Dg[r_ * G::C + dl] = (row_ok && qi - dl >= 0) ? ex2(brow[dl] - mm) : 0.f;
        }
      }
      // the next item's queries, dot products and taps, while this item's last P V runs
      // The next item, taken from the ring only now: its index may be published only
      // after the key loader has issued this item's last loads, which (with POST) are
      // the convolved values its last weights are multiplied by.  Its first key
      // tile's column factors go to the factor buffer of tile T (the barriers of
      // prepare() and of the epilogue order them before that tile reads them).
      fetch_next();
      if (more && st_id < G::BN)
#pragma unroll
        for (int sc = 0; sc < G::NSRC; ++sc)
          facs[(sc * 2 + (T & 1)) * G::BN + st_id] =
              p.fac[(static_cast<long long>(nx.b) * p.H + src_head(nx.g * CL + hr, sc)) * p.lpad + st_id];
      const int eq_next = more ? prepare(r + 1, nx) : 0;

      // ---------------------------------------------------------- epilogue
      mbar_wait(v_empty, ((POST ? NP : T) - 1) & 1, abort_flag, p.err);
      tc_fence_after();
      float inv_l = 1.f;
      // POST: the band near the diagonal, sum_u Gb[u] v[i-u] (u < UB), with
      //   Gb[u] = sum over tap rows a, diagonal offsets dl < c and taps t with
      //           a + dl + c - t = u of theta_post[a][t] A[i-a][i-a-dl]
      float Gb[G::UB];
#pragma unroll
      for (int u = 0; u < G::UB; ++u) Gb[u] = 0.f;
      if constexpr (POST) {
        named_bar_sync(kBarAll, kSmThreads);  // every row's Dg is written
        if (out_row) {
          const float *tp = thp_s + (r & 1) * 128;
#pragma unroll
          for (int a = 0; a < CQ; ++a)
#pragma unroll
            for (int dl = 0; dl < G::C; ++dl) {
              const float pv = Dg[(r_ - a) * G::C + dl];
#pragma unroll
              for (int tq = 0; tq < CK; ++tq) {
                const int u = a + dl + G::C - tq;
                if (u >= 0 && u < G::UB) Gb[u] = fmaf(tp[a * CK + tq], pv, Gb[u]);
              }
            }
        }
      } else {
        red[(4 + wg) * G::BM + r_] = l_run;
        named_bar_sync(kBarAll, kSmThreads);
        const float l_tot = l_run + red[(4 + (wg ^ 1)) * G::BM + r_];
        inv_l = (out_row && l_tot > 0.f) ? 1.f / l_tot : 0.f;
      }
      // 32 output channels zc+c0 .. of head vh: Z (times 1/l) plus, with POST, the band
      auto z_chunk = [&](int hd, int vh, int c0, float (&zo)[32]) {
        uint32_t z[32];
        tmem_ld32(tl + G::Z_COL0 + 128 * hd + zc + c0, z);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) zo[i] = __uint_as_float(z[i]) * inv_l;
        if constexpr (POST) {
          if (out_row) {
#pragma unroll
            for (int u = 0; u < G::UB; ++u) {
              if (qi - u < 0) break;
              const uint4 *vr = reinterpret_cast<const uint4 *>(
                  p.v + (static_cast<long long>(it.b) * L + (qi - u)) * p.rs + static_cast<long long>(vh) * D + zc + c0);
#pragma unroll
              for (int q8 = 0; q8 < 4; ++q8) {
                const uint4 w4 = vr[q8];
                const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  zo[8 * q8 + 2 * e] = fmaf(Gb[u], __uint_as_float(wv[e] << 16), zo[8 * q8 + 2 * e]);
                  zo[8 * q8 + 2 * e + 1] = fmaf(Gb[u], __uint_as_float(wv[e] & 0xffff0000u), zo[8 * q8 + 2 * e + 1]);
                }
              }
            }
          }
        }
      };
      float o[G::DH];
      if constexpr (G::DEFER) {
        // Z_{h->peer} / l_h and w_own * Z_{h->h} / l_h go to the L2 exchange buffer;
        // Z is released at once, the rest of the epilogue waits for finish()
        float4 *mine = xslot(c, hr, r & 1, 0), *own = xslot(c, hr, r & 1, 1);
        const float w_own = p.w[g * 4 + hr * 2 + hr];
#pragma unroll
        for (int c0 = 0; c0 < G::DH; c0 += 32) {
          if (c0 >= zn) break;
          float zo[32];
          z_chunk(hr ^ 1, 2 * g + (hr ^ 1), c0, zo);
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            mine[((zc + c0 + i) / 4) * G::BM + r_] = make_float4(zo[i], zo[i + 1], zo[i + 2], zo[i + 3]);
          z_chunk(hr, 2 * g + hr, c0, zo);
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            own[((zc + c0 + i) / 4) * G::BM + r_] =
                make_float4(w_own * zo[i], w_own * zo[i + 1], w_own * zo[i + 2], w_own * zo[i + 3]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(z_free);  // the next item's first P V may overwrite Z
        // every thread's stores are released to the peer by its own arrival
        mbar_arrive_cluster(map_peer(smem_u32(x_readyb[r & 1]), static_cast<uint32_t>(hr ^ 1)));
        pend = true;
        pend_r = r;
        pend_it = it;
        have = more;
        it = nx;
        eq = eq_next;
        continue;
      } else if constexpr (MIX == 2) {
        // Z_{h->peer} / l_h goes to the peer through L2: [parity][column/4][row] float4
        float4 *mine = xslot(c, hr, r & 1, 0);
        const float4 *theirs = xslot(c, hr ^ 1, r & 1, 0);
#pragma unroll
        for (int c0 = 0; c0 < G::DH; c0 += 32) {
          if (c0 >= zn) break;
          float zo[32];
          z_chunk(hr ^ 1, 2 * g + (hr ^ 1), c0, zo);
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            mine[((zc + c0 + i) / 4) * G::BM + r_] = make_float4(zo[i], zo[i + 1], zo[i + 2], zo[i + 3]);
        }
        const float w_own = p.w[g * 4 + hr * 2 + hr], w_peer = p.w[g * 4 + hr * 2 + (hr ^ 1)];
#pragma unroll
        for (int c0 = 0; c0 < G::DH; c0 += 32) {
          float zo[32];
          if (c0 < zn) z_chunk(hr, 2 * g + hr, c0, zo);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[c0 + i] = c0 < zn ? w_own * zo[i] : 0.f;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(z_free);  // the next item's first P V may overwrite Z
        // every thread's stores are released to the peer by its own arrival
        mbar_arrive_cluster(map_peer(smem_u32(x_readyb[r & 1]), static_cast<uint32_t>(hr ^ 1)));
        mbar_wait_cluster(x_readyb[r & 1], (r >> 1) & 1, abort_flag, p.err);
#pragma unroll
        for (int c4 = 0; c4 < G::DH / 4; ++c4) {
          if (4 * c4 >= zn) break;
          const float4 x = theirs[(zc / 4 + c4) * G::BM + r_];
          o[4 * c4] += w_peer * x.x;
          o[4 * c4 + 1] += w_peer * x.y;
          o[4 * c4 + 2] += w_peer * x.z;
          o[4 * c4 + 3] += w_peer * x.w;
        }
      } else {
#pragma unroll
        for (int c0 = 0; c0 < G::DH; c0 += 32) {
          float zo[32];
          if (c0 < zn) z_chunk(0, h, c0, zo);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[c0 + i] = c0 < zn ? zo[i] : 0.f;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(z_free);
      }
      if (p.gn) {  // group norm over the D channels of (token, head), then depth scale
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < G::DH; ++i) s += o[i];  // channels past zn are 0
        red[(6 + wg) * G::BM + r_] = s;
        named_bar_sync(kBarAll, kSmThreads);
        const float mu = (s + red[(6 + (wg ^ 1)) * G::BM + r_]) * (1.f / D);
        float s2 = 0.f;
#pragma unroll
        for (int i = 0; i < G::DH; ++i) { const float x = i < zn ? o[i] - mu : 0.f; s2 += x * x; }
        red[(8 + wg) * G::BM + r_] = s2;
        named_bar_sync(kBarAll, kSmThreads);
        const float rstd = rsqrtf((s2 + red[(8 + (wg ^ 1)) * G::BM + r_]) * (1.f / D) + p.eps);
        const float *gm = p.gamma + static_cast<long long>(h) * D + zc;
        const float *bt = p.beta + static_cast<long long>(h) * D + zc;
        const float mh = head_multiplier(p.gate, p.lam, h);
#pragma unroll
        for (int i = 0; i < G::DH; ++i)
          if (i < zn) o[i] = ((o[i] - mu) * rstd * gm[i] + bt[i]) * mh;
      }
      if (out_row) {
        __nv_bfloat16 *dst = p.out + ((static_cast<long long>(it.b) * L + qi) * p.H + h) * D + zc;
#pragma unroll
        for (int i = 0; i < G::DH; i += 8) {
          if (i >= zn) break;
          uint4 v;
          v.x = pack_bf16x2(o[i], o[i + 1]);
          v.y = pack_bf16x2(o[i + 2], o[i + 3]);
          v.z = pack_bf16x2(o[i + 4], o[i + 5]);
          v.w = pack_bf16x2(o[i + 6], o[i + 7]);
          *reinterpret_cast<uint4 *>(dst + i) = v;
        }
      }
      have = more;
      it = nx;
      eq = eq_next;
    }
    if constexpr (G::DEFER) {
      if (pend) finish(pend_r, pend_it);  // the last item's epilogue
    }
  }
  tc_fence_before();
  __syncthreads();
  if (MIX == 2) cluster_sync_all();  // no remote arrival reaches a CTA that has exited
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, G::TMEM_COLS);
  }
}

template <int D, int CQ, int CK, int MIX, bool EXACT, bool POST>
cudaError_t launch_kq_one(const AttnArgs &a, const GnArgs *gn, const KqPrepArgs &pa, float *xg, void *vt) {
  using G = KGeo<D, CQ, CK, MIX, EXACT, POST>;
  alignas(64) CUtensorMap tq, tk, tv, tvt;
  const unsigned long long dims[4] = {static_cast<unsigned long long>(D), static_cast<unsigned long long>(a.H),
                                      static_cast<unsigned long long>(a.L), static_cast<unsigned long long>(a.B)};
  const unsigned long long str[3] = {static_cast<unsigned long long>(D) * 2,
                                     static_cast<unsigned long long>(a.rs) * 2,
                                     static_cast<unsigned long long>(a.rs) * 2 * a.L};
  const unsigned boxq[4] = {8, 1, G::QROWS, 1}, boxv[4] = {64, 1, G::BN, 1};
  if (!encode_tmap_bf16(&tq, a.q, 4, dims, str, boxq, false)) return cudaErrorInvalidValue;
  if (!encode_tmap_bf16(&tv, a.v, 4, dims, str, boxv, true)) return cudaErrorInvalidValue;
  // Kt (16-bit elements; the copy moves bytes, fp16 as 16-bit): [B*H*CQ][L][D] when D is
  // a multiple of 64, else [B*H*NCH][L][64]
  const bool krows = D % 64 == 0;
  const unsigned long long kdims[3] = {krows ? static_cast<unsigned long long>(D) : 64ull,
                                       static_cast<unsigned long long>(a.L),
                                       static_cast<unsigned long long>(a.B) * a.H * (krows ? CQ : G::NCH)};
  const unsigned long long kstr[2] = {krows ? static_cast<unsigned long long>(D) * 2 : 128ull,
                                      static_cast<unsigned long long>(a.L) * (krows ? D * 2 : 128)};
  const unsigned boxk[3] = {64, G::BN, 1};
  if (!encode_tmap_bf16(&tk, pa.kt, 3, kdims, kstr, boxk, true)) return cudaErrorInvalidValue;
  tvt = tk;
  if (POST) {  // convolved values: [B*H*NV*CQ][L][D] bf16, 64-channel x 128-key boxes
    const unsigned long long vdims[3] = {static_cast<unsigned long long>(D), static_cast<unsigned long long>(a.L),
                                         static_cast<unsigned long long>(a.B) * a.H * G::NV * CQ};
    const unsigned long long vstr[2] = {static_cast<unsigned long long>(D) * 2,
                                        static_cast<unsigned long long>(a.L) * D * 2};
    if (!encode_tmap_bf16(&tvt, vt, 3, vdims, vstr, boxk, true)) return cudaErrorInvalidValue;
  }
  KqParams p;
  p.theta = a.theta;
  p.w = a.w;
  p.out = static_cast<__nv_bfloat16 *>(a.out);
  p.gn = gn != nullptr;
  p.gamma = gn ? gn->gamma : nullptr;
  p.beta = gn ? gn->beta : nullptr;
  p.eps = gn ? gn->eps : 0.f;
  p.lam = gn ? gn->lam : 1.f;
  p.gate = gn ? gn->gate : nullptr;
  p.B = a.B;
  p.L = a.L;
  p.H = a.H;
  p.n_qtiles = (a.L + G::BMO - 1) / G::BMO;
  p.qk_scale = a.scale;
  p.lpad = pa.lpad;
  p.fac = pa.fac;
  p.vp = pa.vp;
  p.xg = xg;
  p.err = a.err;
  p.theta_post = a.theta_post;
  p.v = static_cast<const __nv_bfloat16 *>(a.v);
  p.rs = a.rs;
  p.queue = a.err + 3;  // zeroed with the error word before every call
  {
    // units (batch, head group) per wave: as many as keep the convolved keys they read
    // (c_q*L*d fp16 per source head, both heads of a group) within a quarter of L2
    const long long unit_bytes = static_cast<long long>(CQ) * a.L * D * 2 * (G::CLUSTER == 2 || G::NSRC == 2 ? 2 : 1);
    const long long units = static_cast<long long>(a.B) * (a.H / G::CLUSTER);
    const long long w = (32ll << 20) / unit_bytes;
    p.wave = static_cast<int>(std::max<long long>(1, std::min<long long>(w, units)));
  }
  auto kern = attn_kq_kernel<D, CQ, CK, MIX, EXACT, POST>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  // persistent: as many clusters as can be resident at once (at most one per work
  // item and kKqMaxClusters), each walking its share of the work items
  const long long n_items = static_cast<long long>(a.B) * (a.H / G::CLUSTER) * p.n_qtiles;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = G::SMEM;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = G::CLUSTER;  // the two heads of a group
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent of the prepass launched just before it on this stream
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(G::CLUSTER, kKqMaxClusters / G::CLUSTER);
  int resident = 0;
  e = cudaOccupancyMaxActiveClusters(&resident, kern, &cfg);
  if (e != cudaSuccess) return e;
  if (resident < 1) return cudaErrorInvalidConfiguration;
  const long long nc = std::min<long long>(std::min<long long>(resident, n_items), kKqMaxClusters / G::CLUSTER);
  cfg.gridDim = dim3(G::CLUSTER, static_cast<unsigned>(nc));
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, tvt, p);
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

bool attn_kq_supported(const AttnArgs &a) {
  if (a.dtype != 1 || (a.d != 64 && a.d != 96 && a.d != 128)) return false;
  if ((a.kq != 1 && a.kq != 3) || a.cq != 6 || a.ck != 11) return false;
  if (!(a.hp == 0 || ((a.hp == 1 || a.hp == 2) && a.ch == 2))) return false;
  if (a.B > 65535 || a.H > 65535 || (a.L + 127) / 128 > 65535) return false;
  const uintptr_t al = reinterpret_cast<uintptr_t>(a.q) | reinterpret_cast<uintptr_t>(a.k) |
                       reinterpret_cast<uintptr_t>(a.v) | reinterpret_cast<uintptr_t>(a.out);
  return al % 16 == 0 && a.rs % 8 == 0;
}

namespace {
// rows of the query tiles: 128, or 123 output rows with the post-softmax convolution
size_t kq_items(int B, int H, int L, int kqp) {
  const size_t bmo = kqp ? 128 - 5 : 128;
  return static_cast<size_t>(B) * (H / 2) * ((static_cast<size_t>(L) + bmo - 1) / bmo);
}
}  // namespace

// Workspace of the contraction path: Kt [B][H][c_q*d/64][L][64] fp16 | fac [B][H][Lpad] fp32 |
// Vp [B][H][L][M] fp32 | (post-softmax mixing) the exchange buffer of the persistent
// CTAs, [CTAs][2 parities][2 parts][d][128] fp32 | (post-softmax convolution) the convolved values
// Vt [B][H][nvh][c_q][L][d] bf16, nvh = 2 with post-softmax mixing, else 1;
// Lpad = L rounded up to 128, M = (c_q-1) + 2*(c_k/2); each part 256-byte aligned.
size_t attn_kq_workspace_bytes(int B, int H, int L, int d, int cq, int ck, int hp, int kqp) {
  const size_t BH = static_cast<size_t>(B) * H, BHL = BH * L;
  const size_t lpad = (static_cast<size_t>(L) + 127) / 128 * 128;
  const size_t M = static_cast<size_t>(cq - 1 + 2 * (ck / 2));
  // the CTA-pair kernel's mixing scratch, or one exchange slot pair per persistent CTA
  // of this kernel (at most kKqMaxClusters CTAs, and at most two per work item)
  const size_t items = kq_items(B, H, L, kqp);
  const size_t ctas = std::min<size_t>(kKqMaxClusters, 2 * items);
  const size_t xg = attn_kq_pair_applies(d, 1, hp, kqp, L) ? attn_kq_pair_scratch_bytes(B, H, L, d, hp)
                    : hp == 2                           ? ctas * 2 * 2 * d * 128 * 4
                                                        : 0;
  const size_t vt = kqp ? align256(BHL * (hp == 2 ? 2 : 1) * cq * d * 2) : 0;
  return align256(BHL * cq * d * 2) + align256(BH * lpad * 4) + align256(BHL * M * 4) + xg + vt;
}

cudaError_t launch_attn_kq(const AttnArgs &a, const GnArgs *gn, void *ws) {
  KqPrepArgs pa;
  pa.q = a.q;
  pa.k = a.k;
  pa.rs = a.rs;
  pa.theta = a.theta;
  pa.B = a.B; pa.H = a.H; pa.L = a.L; pa.d = a.d; pa.cq = a.cq; pa.ck = a.ck;
  pa.M = a.cq - 1 + 2 * (a.ck / 2);
  pa.n_tiles = (a.L + 127) / 128;
  pa.lpad = pa.n_tiles * 128;
  pa.scale_log2 = a.scale * 1.4426950408889634f;
  pa.exact = a.kq == 3;
  const size_t BH = static_cast<size_t>(a.B) * a.H, BHL = BH * a.L;
  char *base = static_cast<char *>(ws);
  pa.kt = base;
  pa.fac = reinterpret_cast<float *>(base + align256(BHL * a.cq * a.d * 2));
  pa.vp = reinterpret_cast<float *>(reinterpret_cast<char *>(pa.fac) + align256(BH * pa.lpad * 4));
  float *xg = reinterpret_cast<float *>(reinterpret_cast<char *>(pa.vp) + align256(BHL * pa.M * 4));
  const size_t items = kq_items(a.B, a.H, a.L, a.kqp);
  const bool pair = attn_kq_pair_applies(a.d, a.kq, a.hp, a.kqp, a.L);
  const size_t xg_bytes = pair ? attn_kq_pair_scratch_bytes(a.B, a.H, a.L, a.d, a.hp)
                          : a.hp == 2 ? std::min<size_t>(kKqMaxClusters, 2 * items) * 2 * 2 * a.d * 128 * 4
                                      : 0;
  void *vt = reinterpret_cast<char *>(xg) + xg_bytes;
  pa.zero = nullptr;
  pa.n_zero = 0;
  if (pair && a.hp == 2) {  // the pair kernel's mixing counters, after its scratch slots
    const size_t slots = static_cast<size_t>(a.B) * (a.H / 2) * ((static_cast<size_t>(a.L) + 127) / 128);
    pa.zero = reinterpret_cast<unsigned *>(reinterpret_cast<char *>(xg) + slots * 2 * 2 * a.d * 128 * 4);
    pa.n_zero = static_cast<int>(slots);
  }
  cudaError_t e = launch_kq_prep(pa, a.stream);
  if (e != cudaSuccess || (e = mark(a)) != cudaSuccess) return e;
  if (a.kqp) {
    VtPrepArgs va;
    va.v = a.v;
    va.rs = a.rs;
    va.theta_post = a.theta_post;
    va.vt = vt;
    va.B = a.B; va.H = a.H; va.L = a.L; va.d = a.d; va.cq = a.cq; va.ck = a.ck;
    va.nvh = a.hp == 2 ? 2 : 1;
    va.n_tiles = pa.n_tiles;
    if ((e = launch_vt_prep(va, a.stream)) != cudaSuccess || (e = mark(a)) != cudaSuccess) return e;
  }
  if (pair) {
    e = launch_attn_kq_pair(a, gn, pa, xg);
    return e != cudaSuccess ? e : mark(a);
  }
  // MIX: 0 no head mixing, 1 pre-softmax mixing (both C of a group per CTA), 2 post-softmax
  auto go = [&](auto d_tag, auto mix_tag) -> cudaError_t {
    constexpr int DD = decltype(d_tag)::value, MX = decltype(mix_tag)::value;
    if (a.kqp)
      return pa.exact ? launch_kq_one<DD, 6, 11, MX, true, true>(a, gn, pa, xg, vt)
                      : launch_kq_one<DD, 6, 11, MX, false, true>(a, gn, pa, xg, vt);
    return pa.exact ? launch_kq_one<DD, 6, 11, MX, true, false>(a, gn, pa, xg, vt)
                    : launch_kq_one<DD, 6, 11, MX, false, false>(a, gn, pa, xg, vt);
  };
  using D64 = std::integral_constant<int, 64>;
  using D96 = std::integral_constant<int, 96>;
  using D128 = std::integral_constant<int, 128>;
  using M0 = std::integral_constant<int, 0>;
  using M1 = std::integral_constant<int, 1>;
  using M2 = std::integral_constant<int, 2>;
  if (a.d == 128) e = a.hp == 2 ? go(D128{}, M2{}) : a.hp == 1 ? go(D128{}, M1{}) : go(D128{}, M0{});
  else if (a.d == 96) e = a.hp == 2 ? go(D96{}, M2{}) : a.hp == 1 ? go(D96{}, M1{}) : go(D96{}, M0{});
  else e = a.hp == 2 ? go(D64{}, M2{}) : a.hp == 1 ? go(D64{}, M1{}) : go(D64{}, M0{});
  return e != cudaSuccess ? e : mark(a);
}

}  // namespace mta
