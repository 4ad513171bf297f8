// gemm_tc.cu -- bf16 GEMM on the sm_100a tensor cores: C[M][N] = A[M][K] B[N][K]^T.
//
// Used for the two projections of the MTA layer ("Multi-Token Attention |
// Summary" (greeksharifa), section 2): QKV = x Wqkv^T and out = Y Wo^T, and for
// their gradients in the layer's backward pass (dY = dOut Wo, dWo = dOut^T Y,
// dx = dQKV Wqkv, dWqkv = dQKV^T x).  Either operand may be stored K-major
// ([rows][K], the forward's case) or MN-major ([K][rows], a transposed operand,
// read as such by the MMA: no transpose pass); C is bf16 or fp32.
//
// Persistent: one CTA per SM walks the 128 x 256 tiles of C (t = blockIdx.x,
// + gridDim.x, ...).  Warp 0 streams 64-wide K slices of A and B with TMA
// (128-byte swizzle) through a 4-stage shared-memory ring that runs on across
// tiles; warp 1 issues tcgen05.mma (M=128, N=256, K=16) into one of two 128 x 256
// fp32 accumulators in tensor memory (alternate tiles), so that warps 2..5 read
// one tile back with tcgen05.ld and store bf16 while the next tile's MMAs run.
// Every mbarrier wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace mta {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BYTES = BN * BK * 2;            // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 48 KB
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t TMEM_COLS = 512;             // two 256-column accumulators
constexpr int PANEL_BYTES = 64 * BK * 2;        // MN-major operand: 64 rows x 64 K, 8 KB

// Operand staging.  K-major: one TMA box {64 K, R rows} per stage, 128-byte rows
// (64 K elements), swizzled.  MN-major ([K][rows] in memory): R/64 boxes {64 rows,
// 64 K}, each a panel of 64 K-rows of 128 bytes (64 operand rows).
template <bool MN>
__device__ __forceinline__ void load_operand(uint8_t *dst, const CUtensorMap *map, uint64_t *bar, int k0, int r0,
                                             int R) {
  if constexpr (!MN) {
    tma_load_2d(dst, map, bar, k0, r0);
  } else {
    for (int p = 0; p < R / 64; ++p) tma_load_2d(dst + p * PANEL_BYTES, map, bar, r0 + 64 * p, k0);
  }
}
template <bool MN>
__device__ __forceinline__ void load_operand_pair(uint8_t *dst, const CUtensorMap *map, uint32_t bar_cluster, int k0,
                                                  int r0, int R) {
  if constexpr (!MN) {
    tma_load_2d_pair(dst, map, bar_cluster, k0, r0);
  } else {
    for (int p = 0; p < R / 64; ++p) tma_load_2d_pair(dst + p * PANEL_BYTES, map, bar_cluster, r0 + 64 * p, k0);
  }
}
// Shared-memory descriptor of K step k (16 elements) of a staged operand.
// K-major: +32 bytes inside the swizzled 128-byte row.  MN-major: +16 K-rows
// (2048 bytes); the 64-row panels lie PANEL_BYTES apart (leading offset), 8-row
// groups of K 1024 bytes apart (stride offset).
template <bool MN>
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int k) {
  if constexpr (!MN)
    return sdesc_sw128(base + 32 * k, 16, 1024);
  else
    return sdesc_sw128(base + 2048 * k, PANEL_BYTES, 1024);
}

// Stores 32 consecutive fp32 accumulator columns of one row of C.
template <bool F32>
__device__ __forceinline__ void store_row32(void *C, int row, int col, int M, int N, const uint32_t *r) {
  if (row >= M || col >= N) return;
  if constexpr (F32) {
    float *dst = static_cast<float *>(C) + static_cast<long long>(row) * N + col;
    if ((N % 4) == 0 && col + 32 <= N) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        reinterpret_cast<float4 *>(dst)[i] = make_float4(__uint_as_float(r[4 * i + 0]), __uint_as_float(r[4 * i + 1]),
                                                         __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (col + i < N) dst[i] = __uint_as_float(r[i]);
    }
  } else {
    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(C) + static_cast<long long>(row) * N + col;
    if ((N % 8) == 0 && col + 32 <= N) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(r[8 * i + 0]), __uint_as_float(r[8 * i + 1]));
        w.y = pack_bf16x2(__uint_as_float(r[8 * i + 2]), __uint_as_float(r[8 * i + 3]));
        w.z = pack_bf16x2(__uint_as_float(r[8 * i + 4]), __uint_as_float(r[8 * i + 5]));
        w.w = pack_bf16x2(__uint_as_float(r[8 * i + 6]), __uint_as_float(r[8 * i + 7]));
        reinterpret_cast<uint4 *>(dst)[i] = w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (col + i < N) dst[i] = __float2bfloat16_rn(__uint_as_float(r[i]));
    }
  }
}

template <bool AT, bool BT, bool F32>
__global__ void __launch_bounds__(192, 1)
    gemm_bf16_nt_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        void *__restrict__ C, int M, int N, int K, unsigned *err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
  uint64_t *empty = full + STAGES;
  uint64_t *acc_full = empty + STAGES;  // [2] accumulator b holds a finished tile
  uint64_t *acc_empty = acc_full + 2;   // [2] the epilogue has read accumulator b
  uint32_t *tslot = reinterpret_cast<uint32_t *>(acc_empty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tn = (N + BN - 1) / BN, n_tiles = ((M + BM - 1) / BM) * n_tn;
  const int nk = (K + BK - 1) / BK;
  // tile t of this CTA's walk: row block t / n_tn, column block t % n_tn
  auto tile_m0 = [&](int t) { return (t / n_tn) * BM; };
  auto tile_n0 = [&](int t) { return (t % n_tn) * BN; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 4); }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) { tmem_alloc(tslot, TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;  // K slices loaded so far (all tiles)
      for (int t = blockIdx.x; t < n_tiles && !*abort_flag; t += gridDim.x) {
        const int m0 = tile_m0(t), n0 = tile_n0(t);
        for (int kt = 0; kt < nk; ++kt, ++issued) {
          const int s = issued % STAGES;
          const uint32_t ph = (issued / STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, err)) break;
          uint8_t *a_s = smem + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          load_operand<AT>(a_s, &tmA, &full[s], kt * BK, m0, BM);
          load_operand<BT>(a_s + A_BYTES, &tmB, &full[s], kt * BK, n0, BN);
        }
      }
      if (*abort_flag)  // let copies in flight land before the CTA exits
        for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
          drain_wait(&full[i % STAGES], (i / STAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, BN, AT ? 1 : 0, BT ? 1 : 0);
      int used = 0;  // K slices consumed so far (all tiles)
      int local = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++local) {
        const int b = local & 1;
        // the epilogue has read this accumulator's previous tile (two tiles ago)
        if (local >= 2 && !mbar_wait(&acc_empty[b], ((local >> 1) - 1) & 1, abort_flag, err)) break;
        tc_fence_after();
        for (int kt = 0; kt < nk; ++kt, ++used) {
          const int s = used % STAGES;
          const uint32_t ph = (used / STAGES) & 1;
          if (!mbar_wait(&full[s], ph, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)  // K=16 per MMA
            mma_bf16_ss(tmem + 256u * b, operand_desc<AT>(a_base, k), operand_desc<BT>(b_base, k), idesc,
                        (kt | k) != 0);
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&acc_full[b]);
      }
    }
  } else {
    const int qd = warp & 3;  // TMEM lane quadrant this warp may access
    int local = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++local) {
      const int b = local & 1;
      if (!mbar_wait(&acc_full[b], (local >> 1) & 1, abort_flag, err)) break;
      tc_fence_after();
      const int row = tile_m0(t) + 32 * qd + lane, n0 = tile_n0(t);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + 256u * b + (static_cast<uint32_t>(32 * qd) << 16) + c0, r);
        tmem_wait_ld();
        store_row32<F32>(C, row, n0 + c0, M, N, r);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);  // the MMA may overwrite this accumulator
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, TMEM_COLS); }
}

// CTA pairs: the pair computes 256 x 256 tiles of C with one cta_group::2 MMA
// (M=256, N=256, K=16) per K step, issued by the pair's first CTA.  Each CTA
// loads its own 128 rows of A and its half (128 rows) of B, so each SM's shared
// memory supplies 8 KB per MMA instead of 12 KB with a 128 x 256 tile per CTA
// (that memory's bandwidth, not the tensor pipe, bounds the one-CTA kernel).
// The loads of both CTAs are counted on the first CTA's full barrier; the MMA
// commits arrive on both CTAs' barriers; each CTA stores its own 128 rows.
constexpr bool kPairs = true;  // launch the CTA-pair kernel for M >= 256
constexpr int P_STAGES = 6;
constexpr int P_A_BYTES = 128 * BK * 2;                 // 16 KB
constexpr int P_B_BYTES = 128 * BK * 2;                 // 16 KB (half of the 256 columns)
constexpr int P_STAGE_BYTES = P_A_BYTES + P_B_BYTES;    // 32 KB
constexpr int P_SMEM_BYTES = P_STAGES * P_STAGE_BYTES + 1024 + 256;

template <bool AT, bool BT, bool F32>
__global__ void __launch_bounds__(192, 1)
    gemm_bf16_nt_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             void *__restrict__ C, int M, int N, int K, unsigned *err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + P_STAGES * P_STAGE_BYTES);  // used in the first CTA
  uint64_t *empty = full + P_STAGES;
  uint64_t *acc_full = empty + P_STAGES;  // [2]
  uint64_t *acc_empty = acc_full + 2;     // [2], used in the first CTA
  uint32_t *tslot = reinterpret_cast<uint32_t *>(acc_empty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs
  const int pair = static_cast<int>(blockIdx.x >> 1), n_pairs = static_cast<int>(gridDim.x >> 1);
  const int n_tn = (N + 255) / 256, n_tiles = ((M + 255) / 256) * n_tn;
  const int nk = (K + BK - 1) / BK;
  auto tile_m0 = [&](int t) { return (t / n_tn) * 256; };
  auto tile_n0 = [&](int t) { return (t % n_tn) * 256; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 8); }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) { tmem_alloc_pair(tslot, TMEM_COLS); tmem_relinquish_pair(); }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int t = pair; t < n_tiles && !*abort_flag; t += n_pairs) {
        const int am = tile_m0(t) + 128 * static_cast<int>(rank), bn = tile_n0(t) + 128 * static_cast<int>(rank);
        for (int kt = 0; kt < nk; ++kt, ++issued) {
          const int s = issued % P_STAGES;
          const uint32_t ph = (issued / P_STAGES) & 1;
          if (!mbar_wait_cluster(&empty[s], ph ^ 1, abort_flag, err)) break;
          // the first CTA's full barrier counts both CTAs' bytes of this stage
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * P_STAGE_BYTES);
          const uint32_t fb = map_peer(smem_u32(&full[s]), 0u);
          uint8_t *a_s = smem + s * P_STAGE_BYTES;
          load_operand_pair<AT>(a_s, &tmA, fb, kt * BK, am, 128);
          load_operand_pair<BT>(a_s + P_A_BYTES, &tmB, fb, kt * BK, bn, 128);
        }
      }
      // copies still in flight land before the CTA exits: both CTAs' loads are counted
      // on the first CTA's barriers, so the first CTA drains them
      if (*abort_flag && rank == 0)
        for (int i = (issued > P_STAGES ? issued - P_STAGES : 0); i < issued; ++i)
          drain_wait(&full[i % P_STAGES], (i / P_STAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_bf16_f32(256, 256, AT ? 1 : 0, BT ? 1 : 0);
      int used = 0, local = 0;
      bool ok = true;
      for (int t = pair; ok && t < n_tiles; t += n_pairs, ++local) {
        const int b = local & 1;
        if (local >= 2 && !mbar_wait_cluster(&acc_empty[b], ((local >> 1) - 1) & 1, abort_flag, err)) break;
        tc_fence_after();
        for (int kt = 0; kt < nk; ++kt, ++used) {
          const int s = used % P_STAGES;
          if (!mbar_wait_cluster(&full[s], (used / P_STAGES) & 1, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * P_STAGE_BYTES);
          const uint32_t b_base = a_base + P_A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16_ss_pair(tmem + 256u * b, operand_desc<AT>(a_base, k), operand_desc<BT>(b_base, k), idesc,
                             (kt | k) != 0);
          mma_commit_pair(&empty[s], 0x3);  // both CTAs' loaders may refill stage s
        }
        if (ok) mma_commit_pair(&acc_full[b], 0x3);
      }
    }
  } else {
    const int qd = warp & 3;
    const uint32_t acc_empty_first = map_peer(smem_u32(&acc_empty[0]), 0u);
    int local = 0;
    for (int t = pair; t < n_tiles; t += n_pairs, ++local) {
      const int b = local & 1;
      if (!mbar_wait_cluster(&acc_full[b], (local >> 1) & 1, abort_flag, err)) break;
      tc_fence_after();
      const int row = tile_m0(t) + 128 * static_cast<int>(rank) + 32 * qd + lane, n0 = tile_n0(t);
#pragma unroll 1
      for (int c0 = 0; c0 < 256; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + 256u * b + (static_cast<uint32_t>(32 * qd) << 16) + c0, r);
        tmem_wait_ld();
        store_row32<F32>(C, row, n0 + c0, M, N, r);
      }
      tc_fence_before();
      __syncwarp();
      // the first CTA's MMA thread may overwrite accumulator b once both CTAs have read it
      if (lane == 0) mbar_arrive_cluster(acc_empty_first + 8u * static_cast<uint32_t>(b));
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no arrival reaches a CTA that has exited; both CTAs are done with TMEM
  if (warp == 1) { tc_fence_after(); tmem_dealloc_pair(tmem, TMEM_COLS); }
}

template <bool AT, bool BT, bool F32>
cudaError_t launch_gemm_impl(const void *A, const void *B, void *C, int M, int N, int K, unsigned *err,
                             cudaStream_t stream) {
  alignas(64) CUtensorMap ta, tb;
  // K-major operand [rows][K]: dims {K, rows}, box {64, R}; MN-major [K][rows]:
  // dims {rows, K}, box {64, 64}
  auto encode = [&](CUtensorMap *map, const void *base, bool mn, int rows, int R) {
    const unsigned long long dims[2] = {static_cast<unsigned long long>(mn ? rows : K),
                                        static_cast<unsigned long long>(mn ? K : rows)};
    const unsigned long long st[1] = {static_cast<unsigned long long>(mn ? rows : K) * 2};
    const unsigned box[2] = {64u, mn ? 64u : static_cast<unsigned>(R)};
    return encode_tmap_bf16(map, base, 2, dims, st, box, true);
  };
  int dev = 0, sms = 148;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if (kPairs && M >= 256) {
    // CTA pairs, persistent: as many pairs as are resident (at most one per 256 x 256 tile)
    if (!encode(&ta, A, AT, M, 128) || !encode(&tb, B, BT, N, 128)) return cudaErrorInvalidValue;
    auto kern = gemm_bf16_nt_pair_kernel<AT, BT, F32>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM_BYTES)) != cudaSuccess)
      return e;
    const long long tiles2 = static_cast<long long>((N + 255) / 256) * ((M + 255) / 256);
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(192);
    cfg.dynamicSmemBytes = P_SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(2 * (sms / 2));
    int pairs = 0;
    if ((e = cudaOccupancyMaxActiveClusters(&pairs, kern, &cfg)) != cudaSuccess) return e;
    if (pairs < 1) return cudaErrorInvalidConfiguration;
    const long long np = std::min<long long>(pairs, tiles2);
    cfg.gridDim = dim3(static_cast<unsigned>(2 * np));
    return cudaLaunchKernelEx(&cfg, kern, ta, tb, C, M, N, K, err);
  }
  if (!encode(&ta, A, AT, M, BM) || !encode(&tb, B, BT, N, BN)) return cudaErrorInvalidValue;
  auto kern = gemm_bf16_nt_kernel<AT, BT, F32>;
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) != cudaSuccess)
    return e;
  const long long tiles = static_cast<long long>((N + BN - 1) / BN) * ((M + BM - 1) / BM);
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  kern<<<grid, 192, SMEM_BYTES, stream>>>(ta, tb, C, M, N, K, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const void *A, const void *B, void *C, int M, int N, int K, bool a_mn, bool b_mn,
                        bool f32_out, unsigned *err, cudaStream_t stream) {
  const int sel = (a_mn ? 4 : 0) | (b_mn ? 2 : 0) | (f32_out ? 1 : 0);
  switch (sel) {
    case 0: return launch_gemm_impl<false, false, false>(A, B, C, M, N, K, err, stream);
    case 1: return launch_gemm_impl<false, false, true>(A, B, C, M, N, K, err, stream);
    case 3: return launch_gemm_impl<false, true, true>(A, B, C, M, N, K, err, stream);
    case 7: return launch_gemm_impl<true, true, true>(A, B, C, M, N, K, err, stream);
    case 2: return launch_gemm_impl<false, true, false>(A, B, C, M, N, K, err, stream);
    case 4: return launch_gemm_impl<true, false, false>(A, B, C, M, N, K, err, stream);
    case 5: return launch_gemm_impl<true, false, true>(A, B, C, M, N, K, err, stream);
    default: return launch_gemm_impl<true, true, false>(A, B, C, M, N, K, err, stream);
  }
}

cudaError_t launch_gemm_bf16_nt(const void *A, const void *B, void *C, int M, int N, int K, unsigned *err,
                                cudaStream_t stream) {
  return launch_gemm(A, B, C, M, N, K, false, false, false, err, stream);
}

}  // namespace mta
