// attn_kq_pair.cu -- the contraction form of MTA attention on CTA pairs.
//
// Same computation as attn_kq.cu ("Multi-Token Attention | Summary"
// (greeksharifa), sections 2, 3.1, 3.2, 3.3): the key-query convolution as the
// contraction C[i][j] = s * sum_a q[i-a] . Kt_a[j] (length c_q*d) against the
// prepass's per-row-convolved keys, Mask_0 taken tap by tap in the band near the
// diagonal, exact online softmax, head mixing after the softmax through the
// values (appendix B: O_h = sum_s w[h][s] Z_{s->h} / l_s), group norm with a
// depth scale or gate.  This variant serves the recipe without pre-softmax mixing
// and without the post-softmax convolution (d = 128, or d = 64 with post-softmax
// mixing).
//
// Why pairs: with one CTA per 128-row query tile, every 128x128x16 MMA reads 8 KB
// of operands from shared memory while the convolved keys stream in at 4 KB per
// MMA; shared memory, not the tensor pipe, then sets the MMA rate (about 100
// cycles per MMA against 64 at the tensor peak).  Here two CTAs on two SMs take
// two adjacent query tiles of one head, and the pair's first CTA issues
// cta_group::2 MMAs of M = 256: each CTA supplies its own 128 query rows and half
// of each key tile (64 keys) and half of the value columns, so each SM's shared
// memory moves 6 KB of operands and 2 KB of convolved keys per MMA.
//
// Roles (352 threads per CTA, as in attn_kq.cu): warps 0-7 softmax (both CTAs,
// their own rows), warp 8 TMA of the convolved keys (each CTA its half; the first
// CTA also takes the work items from the queue), warp 9 the MMA issuer (first CTA
// only), warp 10 TMA of V (each CTA its half) and of the query rows (each CTA its
// own tile).  Barriers that collect both CTAs' data or arrivals live in the first
// CTA; MMA completions are multicast to both CTAs.
//
// Post-softmax mixing pairs heads 2g and 2g+1, which different CTA pairs compute.
// Each CTA writes its two parts (Z_{s->peer}/l_s and w[s][s] Z_{s->s}/l_s) of each
// query row to an L2 scratch slot of its (batch, group, query tile) and counts
// itself in; the second of the two finishes both heads (mixing, group norm, store).
// Nobody waits for the other head: the kernel never relies on two pairs being
// resident at once.
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
constexpr int kThreads = 352;
constexpr int kSmThreads = 256;
constexpr int kTmaWarp = 8, kMmaWarp = 9, kTma2Warp = 10;
constexpr int kBarAll = 1;
constexpr int kBarP = 2;   // the softmax warps of a CTA, before its one arrival on P
constexpr int kItemSlots = 4;
constexpr int kMaxPairs = 80;  // persistent grid: at most this many CTA pairs (>= SM count / 2)
// Sequences at least this long use this kernel for the shapes below (measured on
// B200, one call, d = 128, groups of 2 mixed after the softmax: the one-CTA kernel
// is faster at L = 2048 (309 vs 326 us: this kernel's per-item exchange between
// the two heads' pairs weighs more on short items), this one at L = 4096 (459 vs
// 465 us) and L = 16384 (3.04 vs 3.53 ms))
constexpr int kPairMinL = 4096;

template <int D, int MIX, bool EXACT>
struct PGeo {
  static constexpr int CQ = 6, CK = 11;
  static constexpr int C = CK / 2, HALO = CQ - 1, W = EXACT ? C : HALO + C, M = HALO + 2 * C;
  static constexpr int OFF = EXACT ? HALO : 0;
  static constexpr int BM = 128, BN = 128, HALF = BN / 2;
  static constexpr int DH = D / 2;                        // output channels per softmax warpgroup
  static constexpr int QROWS = (BM + HALO + 7) / 8 * 8;   // query rows staged (with halo)
  static constexpr int NSTRIP = D / 8, STRIP = QROWS * 16, Q_BYTES = NSTRIP * STRIP;
  static constexpr int NDC = D / 64;                      // 64-channel blocks of a tap row
  static constexpr int KBOX = 64 * 128;                   // this CTA's half of a key tile: 64 keys x 64 channels
  static constexpr int SB = NDC, KSTAGE = SB * KBOX;      // a ring stage: this CTA's half of one tap row
  static constexpr int NCH = CQ * NDC;                    // 64-channel chunks of a key tile's operand
  static constexpr int NV = MIX == 2 ? 2 : 1;             // value heads in the P V product
  static constexpr int NPV = NV * D;                      // its N (this CTA holds NPV/2 columns)
  static constexpr int VBOXES = NPV / 2 / 64;             // 64-channel V boxes per CTA
  static constexpr int V_BYTES = VBOXES * BN * 128;
  static constexpr int UROWS = BM + HALO;
  static constexpr int U_BYTES = (UROWS * M * 4 + 15) / 16 * 16;
  static constexpr int CS_BYTES = 2 * BM * W * 4;
  static constexpr int RED_BYTES = 10 * BM * 4;
  static constexpr int FAC_BYTES = 2 * BN * 4;
  static constexpr int Q_AREA = (Q_BYTES + 1023) / 1024 * 1024;
  // small area: taps [2 items][128], per-warp |q| maxima, 40 barriers, TMEM slot,
  // abort flag, the item ring, the finish flag
  static constexpr int TH_OFF = 0, QRED_OFF = 2 * 128 * 4, BAR_OFF = QRED_OFF + 64;
  static constexpr int TSLOT_OFF = BAR_OFF + 8 * 40, ABORT_OFF = TSLOT_OFF + 8, ITEMS_OFF = ABORT_OFF + 8;
  static constexpr int XFLAG_OFF = ITEMS_OFF + 16;
  static constexpr int SMALL_BYTES = (XFLAG_OFF + 16 + 255) / 256 * 256;
  static constexpr int REST = Q_AREA + V_BYTES + U_BYTES + CS_BYTES + RED_BYTES + FAC_BYTES + SMALL_BYTES + 1024;
  static constexpr int NS = (232448 - REST) / KSTAGE < 8 ? (232448 - REST) / KSTAGE : 8;
  static constexpr int OFF_Q = 0, OFF_K = Q_AREA, OFF_V = OFF_K + NS * KSTAGE;
  static constexpr int OFF_U = OFF_V + V_BYTES, OFF_CS = OFF_U + U_BYTES, OFF_RED = OFF_CS + CS_BYTES;
  static constexpr int OFF_FAC = OFF_RED + RED_BYTES, OFF_SMALL = OFF_FAC + FAC_BYTES;
  static constexpr int SMEM = OFF_SMALL + SMALL_BYTES + 1024;
  // tensor memory: C in two 128-column buffers (alternate key tiles; each tile's P,
  // bf16, written over its own C), then Z (NPV columns)
  static constexpr uint32_t TMEM_COLS = 512, Z_COL0 = 256;
  static_assert(Z_COL0 + NPV <= TMEM_COLS, "tensor memory");
  static_assert(NPV / 2 % 64 == 0, "whole 64-channel value boxes per CTA");
  static_assert(NS >= 3, "key ring");
  static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0, "swizzle alignment");
  static_assert(OFF_U % 16 == 0 && OFF_SMALL % 16 == 0, "alignment");
  static_assert(SMEM <= 232448, "shared memory");
  static_assert(11 + 2 * NS + 2 * kItemSlots <= 40, "barrier slots");
};

struct PairParams {
  const float *theta;   // [H][CQ][CK]
  const float *w;       // [H/2][2][2]
  __nv_bfloat16 *out;   // [B][L][H][D]
  const float *gamma, *beta;
  float eps, lam;
  const float *gate;
  int gn;
  int B, L, H, n_qtiles, n_qpairs, lpad;
  float qk_scale;
  const float *fac;     // [B][H][lpad]
  const float *vp;      // [B][H][L][M]
  float *xs;            // post-softmax mixing: [B][H/2][n_qtiles][2 heads][2 parts][D/4][BM] float4
  unsigned *xcnt;       // [B][H/2][n_qtiles] parts counted in (zeroed by the prepass)
  unsigned *err;
  unsigned *queue;      // work-queue counter (zero when the launch starts)
  int wave;             // units (batch, head) per wave of the item order
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

// Work item k: (query-tile pair kp, batch b, head h).  Units (b, h) in waves of
// `wave` units; inside a wave the longest pairs first, then by unit.
struct PItem {
  int kp, b, h;
};
__device__ __forceinline__ PItem pitem_of(int k, int B, int H, int n_qpairs, int wave) {
  const int per_wave = wave * n_qpairs;
  const int w = k / per_wave, r = k - w * per_wave;
  const int nu = min(wave, B * H - w * wave);
  const int unit = w * wave + r % nu;
  PItem it;
  it.kp = n_qpairs - 1 - r / nu;
  it.b = unit / H;
  it.h = unit % H;
  return it;
}

template <int D, int MIX, bool EXACT>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kq_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const PairParams p) {
  using G = PGeo<D, MIX, EXACT>;
  constexpr int CQ = G::CQ, CK = G::CK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *Qs = smem + G::OFF_Q;
  uint8_t *Ks = smem + G::OFF_K;
  uint8_t *Vs = smem + G::OFF_V;
  float *Us = reinterpret_cast<float *>(smem + G::OFF_U);
  float *Cs = reinterpret_cast<float *>(smem + G::OFF_CS);
  float *red = reinterpret_cast<float *>(smem + G::OFF_RED);
  float *facs = reinterpret_cast<float *>(smem + G::OFF_FAC);  // [2][BN]
  uint8_t *small = smem + G::OFF_SMALL;
  float *th_s = reinterpret_cast<float *>(small + G::TH_OFF);    // [2 items][128]
  float *qred = reinterpret_cast<float *>(small + G::QRED_OFF);
  uint64_t *bars = reinterpret_cast<uint64_t *>(small + G::BAR_OFF);
  // local: q_full; first CTA: q_ready, z_free, v_full, p_full[2], mma_done, k_full[],
  // it_empty[]; both (multicast or written by the first CTA): q_free, v_empty,
  // c_full[2], k_empty[], it_full[]
  uint64_t *q_full = bars + 0, *q_ready = bars + 1, *q_free = bars + 2, *z_free = bars + 3;
  uint64_t *v_full = bars + 4, *v_empty = bars + 5, *c_full = bars + 6, *p_full = bars + 8, *mma_done = bars + 10;
  uint64_t *k_full = bars + 11, *k_empty = bars + 11 + G::NS;
  uint64_t *it_full = bars + 11 + 2 * G::NS, *it_empty = it_full + kItemSlots;
  uint32_t *tslot = reinterpret_cast<uint32_t *>(small + G::TSLOT_OFF);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(small + G::ABORT_OFF);
  volatile int *item_slot = reinterpret_cast<volatile int *>(small + G::ITEMS_OFF);
  volatile int *xflag = reinterpret_cast<volatile int *>(small + G::XFLAG_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: takes the items and issues the MMAs
  const int rk = static_cast<int>(rank);
  const int L = p.L, n_items = p.B * p.H * p.n_qpairs;
  // an address in the first CTA (shared::cluster) of a barrier of this CTA's layout
  auto first = [&](uint64_t *bar) { return map_peer(smem_u32(bar), 0u); };
  // arrive on a barrier of the first CTA (release at cluster scope)
  auto arrive_first = [&](uint64_t *bar) { mbar_arrive_cluster(first(bar)); };

  // this CTA's query tile of item it (the pair's tiles are 2 kp and 2 kp + 1)
  auto qtile = [&](const PItem &it) { return 2 * it.kp + rk; };
  // key tiles of the pair: those of its longer (valid) query tile
  auto kv_tiles = [&](const PItem &it) {
    const int last = min(2 * it.kp + 1, p.n_qtiles - 1);
    return min(L - 1, last * G::BM + G::BM - 1) / G::BN + 1;
  };

  // ---- the item ring (as in attn_kq.cu): the first CTA's key loader takes
  // indices from the queue and publishes them to both CTAs
  auto take_item = [&](int r, PItem &it, bool arrive) -> bool {
    const int s = r % kItemSlots;
    const bool ok = mbar_wait_cluster(it_full + s, (r / kItemSlots) & 1, abort_flag, p.err);
    const int k = ok ? item_slot[s] : -1;
    if (ok && arrive) arrive_first(it_empty + s);
    if (k < 0) return false;
    it = pitem_of(k, p.B, p.H, p.n_qpairs, p.wave);
    return true;
  };
  auto publish_item = [&](int r, PItem &it) -> bool {
    const int s = r % kItemSlots;
    if (!mbar_wait_cluster(it_empty + s, ((r / kItemSlots) & 1) ^ 1, abort_flag, p.err)) return false;
    int k = static_cast<int>(atomicAdd(p.queue, 1u));
    if (k >= n_items) k = -1;
    item_slot[s] = k;
    st_cluster_s32(map_peer(smem_u32(const_cast<int *>(item_slot + s)), 1u), k);
    mbar_arrive_cluster(map_peer(smem_u32(it_full + s), 1u));  // releases the store above
    mbar_arrive(it_full + s);
    if (k < 0) return false;
    it = pitem_of(k, p.B, p.H, p.n_qpairs, p.wave);
    return true;
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_ready, 16);  // 8 softmax warps of each CTA
    mbar_init(q_free, 1);
    mbar_init(z_free, 16);
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    for (int b = 0; b < 2; ++b) { mbar_init(c_full + b, 1); mbar_init(p_full + b, 2); }
    mbar_init(mma_done, 1);
    for (int s = 0; s < G::NS; ++s) { mbar_init(k_full + s, 1); mbar_init(k_empty + s, 1); }
    // consumers per item: both CTAs' V and query loaders and 8 softmax warps, the
    // MMA thread, and the second CTA's key loader
    for (int s = 0; s < kItemSlots; ++s) { mbar_init(it_full + s, 1); mbar_init(it_empty + s, 2 * (2 + 8) + 2); }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) { tmem_alloc_pair(tslot, G::TMEM_COLS); tmem_relinquish_pair(); }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tslot;
  pdl_wait_primary();  // the prepass's outputs are complete and visible from here on

  if (warp == kTmaWarp || warp == kTma2Warp) {
    // -------------------------------------------------------------- TMA
    if (warp == kTmaWarp && lane == 0) {  // this CTA's half of the convolved keys
      prefetch_tmap(&tmK);
      int cnt = 0;
      PItem it;
      bool ok = true;
      for (int r = 0; ok && !*abort_flag && (rank == 0 ? publish_item(r, it) : take_item(r, it, true)); ++r) {
        const int n_kv = kv_tiles(it);
        const int zh = it.b * p.H + it.h;
        for (int t = 0; ok && t < n_kv && !*abort_flag; ++t)
          for (int a = 0; a < CQ; ++a) {  // one stage per tap row: this CTA's 64 keys x d
            const int st = cnt % G::NS;
            if (!mbar_wait_cluster(k_empty + st, ((cnt / G::NS) & 1) ^ 1, abort_flag, p.err)) { ok = false; break; }
            if (rank == 0) mbar_arrive_expect_tx(k_full + st, 2 * G::KSTAGE);  // both CTAs' halves
            const uint32_t kf = first(k_full + st);
#pragma unroll
            for (int dc = 0; dc < G::NDC; ++dc)
              tma_load_3d_pair(Ks + st * G::KSTAGE + dc * G::KBOX, &tmK, kf, 64 * dc, t * G::BN + 64 * rk,
                               zh * CQ + a);
            ++cnt;
          }
      }
      if (*abort_flag && rank == 0)  // copies in flight (both CTAs', counted here) land first
        for (int c2 = (cnt > G::NS ? cnt - G::NS : 0); c2 < cnt; ++c2)
          drain_wait(k_full + c2 % G::NS, (c2 / G::NS) & 1);
    } else if (warp == kTma2Warp && lane == 0) {  // this CTA's half of the value columns, per key tile
      prefetch_tmap(&tmV);
      int nv = 0;
      PItem it;
      for (int r = 0; !*abort_flag && take_item(r, it, true); ++r) {
        const int n_kv = kv_tiles(it);
        for (int t = 0; t < n_kv; ++t, ++nv) {
          if (!mbar_wait_cluster(v_empty, (nv & 1) ^ 1, abort_flag, p.err)) break;
          if (rank == 0) mbar_arrive_expect_tx(v_full, 2 * G::V_BYTES);
          const uint32_t vf = first(v_full);
#pragma unroll
          for (int vb = 0; vb < G::VBOXES; ++vb) {
            // post-softmax mixing: CTA rank r holds head 2g+r's values; else half of d
            const int vh = MIX == 2 ? (it.h & ~1) + rk : it.h;
            const int ch = MIX == 2 ? 64 * vb : 64 * (G::VBOXES * rk + vb);
            tma_load_4d_pair(Vs + vb * G::BN * 128, &tmV, vf, ch, vh, t * G::BN, it.b);
          }
        }
      }
      if (*abort_flag && rank == 0 && nv) drain_wait(v_full, (nv - 1) & 1);
    } else if (warp == kTma2Warp && lane == 1) {  // this CTA's query rows of each item
      prefetch_tmap(&tmQ);
      int nq = 0;
      PItem it;
      for (int r = 0; !*abort_flag && take_item(r, it, true); ++r, ++nq) {
        if (r > 0 && !mbar_wait_cluster(q_free, (r - 1) & 1, abort_flag, p.err)) break;
        const int row0 = qtile(it) * G::BM - G::HALO;
        mbar_arrive_expect_tx(q_full, G::Q_BYTES);
#pragma unroll 1
        for (int s2 = 0; s2 < G::NSTRIP; ++s2)
          tma_load_4d(Qs + s2 * G::STRIP, &tmQ, q_full, 8 * s2, it.h, row0, it.b);
      }
      if (nq) drain_wait(q_full, (nq - 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // -------------------------------------------------------------- MMA (first CTA)
    // The whole warp runs the issuing loop; one elected lane issues the instructions.
    if (rank == 0) {
      const bool issuer = elect_one();
      // waits of the issuing loop, made warp-uniform (all lanes poll the same barrier)
      auto wwait = [&](uint64_t *bar, uint32_t ph) -> bool {
        return __all_sync(0xffffffffu, mbar_wait_cluster(bar, ph, abort_flag, p.err));
      };
      const uint32_t idesc_c = idesc_f16_f32(256, G::BN);
      const uint32_t idesc_pv = idesc_bf16_f32(256, G::NPV, 0, 1);
      const uint64_t qdesc0 = sdesc_noswz(smem_u32(Qs), G::STRIP, 128);
      const uint64_t kdesc0 = sdesc_sw128(smem_u32(Ks), 16, 1024);
      const uint64_t vdesc0 = sdesc_sw128(smem_u32(Vs), G::BN * 128, 1024);
      int cnt = 0, T = 0;
      bool ok = true;
      // C of global key tile T into buffer T & 1: per tap row a, this CTA's 64 keys
      // of the stage (the other CTA's 64 keys at the same offsets); Q shifted up by a rows
      auto issue_c = [&](bool last_of_item) -> bool {
        const uint32_t c_dst = tmem + 128u * (T & 1);
        for (int a = 0; a < CQ; ++a, ++cnt) {
          const int st = cnt % G::NS;
          if (!wwait(k_full + st, (cnt / G::NS) & 1)) return false;
          tc_fence_after();
          const uint64_t kd = kdesc0 + static_cast<uint32_t>((st * G::KSTAGE) >> 4);
#pragma unroll
          for (int dc = 0; dc < G::NDC; ++dc) {
            const uint64_t qd = qdesc0 + static_cast<uint32_t>((8 * dc * G::STRIP + 16 * (G::HALO - a)) >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss_pair_if(issuer, c_dst, qd + (2 * kk * G::STRIP >> 4), kd + (dc * G::KBOX >> 4) + 2 * kk,
                             idesc_c, (a > 0 || dc > 0 || kk > 0));
          }
          mma_commit_pair_if(issuer, k_empty + st, 0x3);
        }
        mma_commit_pair_if(issuer, c_full + (T & 1), 0x3);
        if (last_of_item) mma_commit_pair_if(issuer, q_free, 0x3);  // both query buffers may take the next item
        return true;
      };
      PItem it;
      // (one arrival per item on the ring: this warp counts as one consumer)
      auto take_mma = [&](int r, PItem &x) -> bool {
        const bool got = __all_sync(0xffffffffu, take_item(r, x, false));
        if (lane == 0) arrive_first(it_empty + r % kItemSlots);
        return got;
      };
      for (int r = 0; ok && take_mma(r, it); ++r) {
        const int nsl = kv_tiles(it);
        if (!wwait(q_ready, r & 1)) break;
        const int T0 = T;
        ok = issue_c(nsl == 1);
        if (ok && nsl > 1) {
          T = T0 + 1;
          ok = issue_c(nsl == 2);
        }
        for (int sl = 0; ok && sl < nsl; ++sl) {
          const int Tt = T0 + sl;
          if (!wwait(p_full + (Tt & 1), (Tt >> 1) & 1)) { ok = false; break; }
          if (!wwait(v_full, Tt & 1)) { ok = false; break; }
          if (sl == 0 && r > 0 && !wwait(z_free, (r - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t pcol = tmem + 128u * (Tt & 1);
#pragma unroll
          for (int kk = 0; kk < G::BN / 16; ++kk)
            mma_ts_pair_if(issuer, tmem + G::Z_COL0, pcol + 8 * kk, vdesc0 + ((kk * 16 * 128) >> 4), idesc_pv,
                           (sl > 0 || kk > 0));
          mma_commit_pair_if(issuer, v_empty, 0x3);
          if (sl + 2 < nsl) {
            T = Tt + 2;
            ok = issue_c(sl + 3 == nsl);
          }
        }
        T = T0 + nsl;
      }
      mma_commit_pair_if(issuer, mma_done, 0x1);
      drain_wait(mma_done, 0);
    }
  } else {
    // ---------------------------------------------- softmax warpgroups (both CTAs)
    const int wg = warp >> 2, q4 = warp & 3;
    const int r_ = 32 * q4 + lane;   // query row of this thread = TMEM lane
    const int st_id = threadIdx.x;
    const int cb = G::HALF * wg;     // key columns of this warpgroup
    const int zc = G::DH * wg;       // output channels of this warpgroup
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q4) << 16);
    const float sc0 = p.qk_scale * kLog2e;
    float *brow = Cs + r_ * G::W;             // this row of the item's band table

    auto arrive_all = [&](uint64_t *bar) {  // one arrival per warp on a barrier of the first CTA
      __syncwarp();
      if (lane == 0) arrive_first(bar);
    };
    auto take_sm = [&](int r, PItem &x) -> bool {
      const bool got = take_item(r, x, false);
      arrive_all(it_empty + r % kItemSlots);
      return got;
    };
    // Stage item r: this CTA's query rows in fp16 (scaled down by a power of 2 only
    // if |q| > 2^14), the past dot products of its staged rows and the head's taps.
    auto prepare = [&](int r, const PItem &it) -> int {
      const int row0 = qtile(it) * G::BM - G::HALO;
      mbar_wait(q_full, r & 1, abort_flag, p.err);
      float qmax = 0.f;
      for (int c16 = st_id; c16 < G::Q_BYTES / 16; c16 += kSmThreads) {
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
      for (int c16 = st_id; c16 < G::Q_BYTES / 16; c16 += kSmThreads) {
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
      arrive_all(q_ready);
      const long long bh = static_cast<long long>(it.b) * p.H + it.h;
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
        if (e < G::UROWS * G::M) Us[e] = vt[u];
      }
      if (st_id < CQ * CK) th_s[(r & 1) * 128 + st_id] = p.theta[static_cast<long long>(it.h) * CQ * CK + st_id];
      return eq;
    };

    // post-softmax mixing: scratch slot of (batch, group, query tile), source head s, part
    // (0: for the peer head, 1: the head's own, mixing weight applied)
    auto xslot = [&](int b, int g, int qt, int s, int part) -> float4 * {
      return reinterpret_cast<float4 *>(p.xs) +
             ((((static_cast<long long>(b) * (p.H / 2) + g) * p.n_qtiles + qt) * 2 + s) * 2 + part) *
                 (G::BM * D / 4);
    };
    // group norm (or not) of this thread's DH channels o of head hh at query row qrow, and store
    auto norm_store = [&](float (&o)[G::DH], int b, int hh, int qrow, bool store) {
      if (p.gn) {
        float s1 = 0.f;
#pragma unroll
        for (int i = 0; i < G::DH; ++i) s1 += o[i];
        red[(6 + wg) * G::BM + r_] = s1;
        named_bar_sync(kBarAll, kSmThreads);
        const float mu = (s1 + red[(6 + (wg ^ 1)) * G::BM + r_]) * (1.f / D);
        float s2 = 0.f;
#pragma unroll
        for (int i = 0; i < G::DH; ++i) { const float x = o[i] - mu; s2 += x * x; }
        red[(8 + wg) * G::BM + r_] = s2;
        named_bar_sync(kBarAll, kSmThreads);
        const float rstd = rsqrtf((s2 + red[(8 + (wg ^ 1)) * G::BM + r_]) * (1.f / D) + p.eps);
        const float *gm = p.gamma + static_cast<long long>(hh) * D + zc;
        const float *bt = p.beta + static_cast<long long>(hh) * D + zc;
        const float mh = head_multiplier(p.gate, p.lam, hh);
#pragma unroll
        for (int i = 0; i < G::DH; ++i) o[i] = ((o[i] - mu) * rstd * gm[i] + bt[i]) * mh;
        named_bar_sync(kBarAll, kSmThreads);  // red is free for the next head's statistics
      }
      if (store) {
        __nv_bfloat16 *dst = p.out + ((static_cast<long long>(b) * L + qrow) * p.H + hh) * D + zc;
#pragma unroll
        for (int i = 0; i < G::DH; i += 8) {
          uint4 v;
          v.x = pack_bf16x2(o[i], o[i + 1]);
          v.y = pack_bf16x2(o[i + 2], o[i + 3]);
          v.z = pack_bf16x2(o[i + 4], o[i + 5]);
          v.w = pack_bf16x2(o[i + 6], o[i + 7]);
          *reinterpret_cast<uint4 *>(dst + i) = v;
        }
      }
    };
    // the item whose mixing is still to be finished by this CTA (the second of the
    // two heads of its (batch, group, query tile) to count in)
    bool pend = false;
    PItem pend_it{0, 0, 0};
    auto finish = [&](const PItem &pi) {
      const int qt = qtile(pi), g = pi.h >> 1, qrow = qt * G::BM + r_;
      const bool store = qrow < L;
      __threadfence();  // the other head's parts, counted in before ours, are visible
#pragma unroll 1
      for (int s = 0; s < 2; ++s) {  // destination head 2g + s: its own part + w * the other's part for it
        const float4 *own = xslot(pi.b, g, qt, s, 1);
        const float4 *oth = xslot(pi.b, g, qt, s ^ 1, 0);
        const float wx = p.w[g * 4 + s * 2 + (s ^ 1)];
        float o[G::DH];
#pragma unroll
        for (int c4 = 0; c4 < G::DH / 4; ++c4) {
          const float4 x = __ldcg(own + (zc / 4 + c4) * G::BM + r_);
          const float4 y = __ldcg(oth + (zc / 4 + c4) * G::BM + r_);
          o[4 * c4] = x.x + wx * y.x;
          o[4 * c4 + 1] = x.y + wx * y.y;
          o[4 * c4 + 2] = x.z + wx * y.z;
          o[4 * c4 + 3] = x.w + wx * y.w;
        }
        norm_store(o, pi.b, 2 * g + s, qrow, store);
      }
    };

    int T = 0;
    PItem it, nx;
    bool have = take_sm(0, it);
    int eq = 0;
    if (have) {
      eq = prepare(0, it);
      if (st_id < G::BN) facs[st_id] = p.fac[(static_cast<long long>(it.b) * p.H + it.h) * p.lpad + st_id];
      named_bar_sync(kBarAll, kSmThreads);
    }
    for (int r = 0; have; ++r) {
      const int h = it.h, qt = qtile(it);
      const int R0 = qt * G::BM, qi = R0 + r_;
      const bool row_ok = qi < L;   // a query of the sequence (R0 >= 0)
      const int nsl = kv_tiles(it);
      const long long fbase = (static_cast<long long>(it.b) * p.H + h) * p.lpad;
      const float qinv = exp2f(static_cast<float>(-eq));
      // the band 0 <= i-j < W, where the mask removes taps (see attn_kq.cu)
      // (each warpgroup takes half of the W diagonals of its row, once per item, into
      // the band table brow[dd], log2 units, read by both after a barrier)
      auto band_part = [&](auto lo_c) {
        constexpr int LO = decltype(lo_c)::value, NB = LO == 0 ? (G::W + 1) / 2 : G::W - (G::W + 1) / 2;
        float acc[NB];
#pragma unroll
        for (int e = 0; e < NB; ++e) acc[e] = 0.f;
#pragma unroll
        for (int a = 0; a < CQ; ++a) {
          const float *vrow = Us + (r_ + G::HALO - a) * G::M;
          const float *th = th_s + (r & 1) * 128;
          float vr[G::M];
#pragma unroll
          for (int m = 0; m < G::M; ++m) vr[m] = vrow[m];
#pragma unroll
          for (int tp = 0; tp < CK; ++tp) {
            const float thv = th[a * CK + tp];
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
      // column factors two tiles ahead: loaded a whole tile before they are stored
      float fpre = (st_id < G::BN && 1 < nsl) ? p.fac[fbase + G::BN + st_id] : 0.f;
      for (int sl = 0; sl < nsl; ++sl, ++T) {
        const int j0 = sl * G::BN;
        if (sl == 0) {  // the band table of the item, while the first C is computed
          if (row_ok) {
            if (wg == 0)
              band_part(std::integral_constant<int, 0>());
            else
              band_part(std::integral_constant<int, (G::W + 1) / 2>());
          }
          named_bar_sync(kBarAll, kSmThreads);
        }
        const float fnext = fpre;
        fpre = (st_id < G::BN && sl + 2 < nsl) ? p.fac[fbase + (sl + 2) * G::BN + st_id] : 0.f;
        mbar_wait_cluster(c_full + (T & 1), (T >> 1) & 1, abort_flag, p.err);
        tc_fence_after();
        const uint32_t cbuf = 128u * (T & 1);
        float cv[G::HALF];
        {
          const float4 *f4 = reinterpret_cast<const float4 *>(facs + (T & 1) * G::BN + cb);
          // both 32-column halves in flight before one wait
          uint32_t u32[2][32];
          tmem_ld32(tl + cbuf + cb, u32[0]);
          tmem_ld32(tl + cbuf + cb + 32, u32[1]);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < G::HALF / 4; ++i) {
            const float4 f = f4[i];
            cv[4 * i] = __uint_as_float(u32[i / 8][4 * (i % 8)]) * f.x;
            cv[4 * i + 1] = __uint_as_float(u32[i / 8][4 * (i % 8) + 1]) * f.y;
            cv[4 * i + 2] = __uint_as_float(u32[i / 8][4 * (i % 8) + 2]) * f.z;
            cv[4 * i + 3] = __uint_as_float(u32[i / 8][4 * (i % 8) + 3]) * f.w;
          }
        }
        tc_fence_before();  // orders the C reads before the barrier that precedes the P writes
        if (eq != 0) {
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
        if (j0 + G::BN - 1 > R0) {  // Mask_-inf: keys after the query
#pragma unroll
          for (int jj = 0; jj < G::HALF; ++jj)
            if (j0 + cb + jj > qi) cv[jj] = -INFINITY;
        }
        float *rmx = red + (T & 1) * 2 * G::BM;
        rmx[wg * G::BM + r_] = row_ok ? tree_max<G::HALF>(cv) : -INFINITY;
        if (st_id < G::BN) facs[((T + 1) & 1) * G::BN + st_id] = fnext;
        named_bar_sync(kBarAll, kSmThreads);
        tc_fence_after();  // both warpgroups have read this tile's C (P may overwrite it)
        const float mt = fmaxf(rmx[r_], rmx[G::BM + r_]);
        const float m_new = fmaxf(m_run, mt);
        bool resc = false;
        float alpha = 1.f;
        if (sl == 0) {
          m_run = m_new;
        } else if (m_new > m_run + kRescaleLog2) {
          resc = true;
          alpha = ex2(m_run - m_new);
          m_run = m_new;
        }
        if (T > 0) {  // the previous tile's P V is complete (Z may be rescaled)
          mbar_wait_cluster(v_empty, (T - 1) & 1, abort_flag, p.err);
          tc_fence_after();
        }
        if (__any_sync(0xffffffffu, resc)) {  // warp-collective tensor-memory access
          l_run *= alpha;
#pragma unroll 1
          for (int hd = 0; hd < G::NV; ++hd)
#pragma unroll 1
            for (int c0 = 0; c0 < G::DH; c0 += 32) {
              uint32_t z[32];
              const uint32_t za = tl + G::Z_COL0 + D * hd + zc + c0;
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
        tmem_st32(tl + cbuf + 32 * wg, pk);  // over this tile's C (both warpgroups have read it)
        l_run += ls;
        tmem_wait_st();
        tc_fence_before();
        // one arrival per CTA: the TMEM stores of all eight warps are ordered before it
        // by their fences and the barrier (a release at cluster scope per warp cost
        // about as much as the tile's exponentials)
        named_bar_sync(kBarP, kSmThreads);
        if (st_id == 0) {
          tc_fence_after();
          arrive_first(p_full + (T & 1));
        }
        if (pend && sl == 0) {  // the previous item's mixing, while this tile's P V and the next C run
          finish(pend_it);
          pend = false;
        }
      }
      // the next item (its index may be published only after the key loader issued
      // this item's last loads) and its first key tile's column factors
      const bool more = take_sm(r + 1, nx);
      if (more && st_id < G::BN)
        facs[(T & 1) * G::BN + st_id] = p.fac[(static_cast<long long>(nx.b) * p.H + nx.h) * p.lpad + st_id];
      const int eq_next = more ? prepare(r + 1, nx) : 0;

      // ---------------------------------------------------------- epilogue
      mbar_wait_cluster(v_empty, (T - 1) & 1, abort_flag, p.err);
      tc_fence_after();
      red[(4 + wg) * G::BM + r_] = l_run;
      named_bar_sync(kBarAll, kSmThreads);
      const float l_tot = l_run + red[(4 + (wg ^ 1)) * G::BM + r_];
      const float inv_l = (row_ok && l_tot > 0.f) ? 1.f / l_tot : 0.f;
      const bool tile_ok = qt < p.n_qtiles;  // the pair's second tile may lie past the sequence
      if constexpr (MIX == 2) {
        // both parts of this head's rows to the scratch slot; Z is then free
        const int s = h & 1, g = h >> 1;
        const float w_own = p.w[g * 4 + s * 2 + s];
        float4 *oth = tile_ok ? xslot(it.b, g, qt, s, 0) : nullptr, *own = tile_ok ? xslot(it.b, g, qt, s, 1) : nullptr;
#pragma unroll
        for (int c0 = 0; c0 < G::DH; c0 += 32) {
          uint32_t z[32];
          tmem_ld32(tl + G::Z_COL0 + D * (s ^ 1) + zc + c0, z);
          tmem_wait_ld();
          if (tile_ok)
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              __stcg(oth + ((zc + c0 + i) / 4) * G::BM + r_,
                     make_float4(__uint_as_float(z[i]) * inv_l, __uint_as_float(z[i + 1]) * inv_l,
                                 __uint_as_float(z[i + 2]) * inv_l, __uint_as_float(z[i + 3]) * inv_l));
          tmem_ld32(tl + G::Z_COL0 + D * s + zc + c0, z);
          tmem_wait_ld();
          const float fo = w_own * inv_l;
          if (tile_ok)
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              __stcg(own + ((zc + c0 + i) / 4) * G::BM + r_,
                     make_float4(__uint_as_float(z[i]) * fo, __uint_as_float(z[i + 1]) * fo,
                                 __uint_as_float(z[i + 2]) * fo, __uint_as_float(z[i + 3]) * fo));
        }
        tc_fence_before();
        arrive_all(z_free);  // the next item's first P V may overwrite Z
        if (tile_ok) {
          // count this head in; the second of the pair of heads finishes both
          __threadfence();
          named_bar_sync(kBarAll, kSmThreads);
          if (st_id == 0)
            *xflag = static_cast<int>(atomicAdd(p.xcnt + (static_cast<long long>(it.b) * (p.H / 2) + g) * p.n_qtiles + qt, 1u));
          named_bar_sync(kBarAll, kSmThreads);
          if (*xflag == 1) {
            pend = true;
            pend_it = it;
          }
          named_bar_sync(kBarAll, kSmThreads);  // everyone has read the flag before it is reused
        }
      } else {
        float o[G::DH];
#pragma unroll
        for (int c0 = 0; c0 < G::DH; c0 += 32) {
          uint32_t z[32];
          tmem_ld32(tl + G::Z_COL0 + zc + c0, z);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[c0 + i] = __uint_as_float(z[i]) * inv_l;
        }
        tc_fence_before();
        arrive_all(z_free);
        norm_store(o, it.b, h, qi, tile_ok && row_ok);
      }
      have = more;
      it = nx;
      eq = eq_next;
    }
    if (pend) finish(pend_it);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no remote arrival reaches a CTA that has exited; TMEM is no longer used
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, G::TMEM_COLS);
  }
}

template <int D, int MIX, bool EXACT>
cudaError_t launch_pair_one(const AttnArgs &a, const GnArgs *gn, const KqPrepArgs &pa, float *xs, unsigned *xcnt) {
  using G = PGeo<D, MIX, EXACT>;
  alignas(64) CUtensorMap tq, tk, tv;
  const unsigned long long dims[4] = {static_cast<unsigned long long>(D), static_cast<unsigned long long>(a.H),
                                      static_cast<unsigned long long>(a.L), static_cast<unsigned long long>(a.B)};
  const unsigned long long str[3] = {static_cast<unsigned long long>(D) * 2,
                                     static_cast<unsigned long long>(a.rs) * 2,
                                     static_cast<unsigned long long>(a.rs) * 2 * a.L};
  const unsigned boxq[4] = {8, 1, G::QROWS, 1}, boxv[4] = {64, 1, G::BN, 1};
  if (!encode_tmap_bf16(&tq, a.q, 4, dims, str, boxq, false)) return cudaErrorInvalidValue;
  if (!encode_tmap_bf16(&tv, a.v, 4, dims, str, boxv, true)) return cudaErrorInvalidValue;
  // Kt [B*H*CQ][L][D] (16-bit elements), boxes of 64 keys x 64 channels
  const unsigned long long kdims[3] = {static_cast<unsigned long long>(D), static_cast<unsigned long long>(a.L),
                                       static_cast<unsigned long long>(a.B) * a.H * G::CQ};
  const unsigned long long kstr[2] = {static_cast<unsigned long long>(D) * 2, static_cast<unsigned long long>(a.L) * D * 2};
  const unsigned boxk[3] = {64, 64, 1};
  if (!encode_tmap_bf16(&tk, pa.kt, 3, kdims, kstr, boxk, true)) return cudaErrorInvalidValue;
  PairParams p;
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
  p.n_qtiles = (a.L + G::BM - 1) / G::BM;
  p.n_qpairs = (p.n_qtiles + 1) / 2;
  p.lpad = pa.lpad;
  p.qk_scale = a.scale;
  p.fac = pa.fac;
  p.vp = pa.vp;
  p.xs = xs;
  p.xcnt = xcnt;
  p.err = a.err;
  p.queue = a.err + 3;  // zeroed with the error word before every call
  {
    // units (batch, head) per wave: as many as keep their convolved keys within a
    // quarter of L2, an even number so that the two heads of a group share a wave
    const long long unit_bytes = static_cast<long long>(G::CQ) * a.L * D * 2;
    const long long units = static_cast<long long>(a.B) * a.H;
    long long w = std::max<long long>(2, ((32ll << 20) / unit_bytes) & ~1ll);
    p.wave = static_cast<int>(std::min<long long>(w, units));
  }
  auto kern = attn_kq_pair_kernel<D, MIX, EXACT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  const long long n_items = static_cast<long long>(a.B) * a.H * p.n_qpairs;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = G::SMEM;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(2 * kMaxPairs);
  int resident = 0;
  if ((e = cudaOccupancyMaxActiveClusters(&resident, kern, &cfg)) != cudaSuccess) return e;
  if (resident < 1) return cudaErrorInvalidConfiguration;
  const long long np = std::min<long long>(std::min<long long>(resident, n_items), kMaxPairs);
  cfg.gridDim = dim3(static_cast<unsigned>(2 * np));
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, p);
}

}  // namespace

bool attn_kq_pair_applies(int d, int kq, int hp, int kqp, int L) {
  return L >= kPairMinL && kqp == 0 && (kq == 1 || kq == 3) && ((d == 128 && (hp == 0 || hp == 2)) || (d == 64 && hp == 2));
}

size_t attn_kq_pair_scratch_bytes(int B, int H, int L, int d, int hp) {
  if (hp != 2) return 0;
  const size_t nqt = (static_cast<size_t>(L) + 127) / 128;
  const size_t slots = static_cast<size_t>(B) * (H / 2) * nqt;
  // [slots][2 heads][2 parts][d][128] fp32, then the counters [slots] (256-byte aligned)
  return slots * 2 * 2 * d * 128 * 4 + (slots * 4 + 255) / 256 * 256;
}

cudaError_t launch_attn_kq_pair(const AttnArgs &a, const GnArgs *gn, const KqPrepArgs &pa, void *scratch) {
  float *xs = static_cast<float *>(scratch);
  const size_t nqt = (static_cast<size_t>(a.L) + 127) / 128;
  unsigned *xcnt = reinterpret_cast<unsigned *>(static_cast<char *>(scratch) +
                                                static_cast<size_t>(a.B) * (a.H / 2) * nqt * 2 * 2 * a.d * 128 * 4);
  const bool ex = a.kq == 3;
  if (a.d == 128) {
    if (a.hp == 2) return ex ? launch_pair_one<128, 2, true>(a, gn, pa, xs, xcnt) : launch_pair_one<128, 2, false>(a, gn, pa, xs, xcnt);
    return ex ? launch_pair_one<128, 0, true>(a, gn, pa, xs, xcnt) : launch_pair_one<128, 0, false>(a, gn, pa, xs, xcnt);
  }
  return ex ? launch_pair_one<64, 2, true>(a, gn, pa, xs, xcnt) : launch_pair_one<64, 2, false>(a, gn, pa, xs, xcnt);
}

}  // namespace mta
