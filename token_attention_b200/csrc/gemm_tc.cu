// gemm_tc.cu -- bf16 GEMM on the sm_100a tensor cores: C[M][N] = A[M][K] B[N][K]^T.
//
// Used for the two projections of the MTA layer ("Multi-Token Attention |
// Summary" (greeksharifa), section 2): QKV = x Wqkv^T and out = Y Wo^T.
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

__global__ void __launch_bounds__(192, 1)
    gemm_bf16_nt_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        __nv_bfloat16 *__restrict__ C, int M, int N, int K, unsigned *err) {
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
          tma_load_2d(a_s, &tmA, &full[s], kt * BK, m0);
          tma_load_2d(a_s + A_BYTES, &tmB, &full[s], kt * BK, n0);
        }
      }
      if (*abort_flag)  // let copies in flight land before the CTA exits
        for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
          drain_wait(&full[i % STAGES], (i / STAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 0);
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
          for (int k = 0; k < BK / 16; ++k)  // K=16 per MMA: +32 bytes inside the 128-byte swizzle row
            mma_bf16_ss(tmem + 256u * b, sdesc_sw128(a_base + 32 * k, 16, 1024),
                        sdesc_sw128(b_base + 32 * k, 16, 1024), idesc, (kt | k) != 0);
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&acc_full[b]);
      }
    }
  } else {
    const int qd = warp & 3;  // TMEM lane quadrant this warp may access
    const bool vec = (N % 8) == 0;
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
        const int col = n0 + c0;
        if (row < M && col < N) {
          __nv_bfloat16 *dst = C + static_cast<long long>(row) * N + col;
          if (vec && col + 32 <= N) {
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

__global__ void __launch_bounds__(192, 1)
    gemm_bf16_nt_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             __nv_bfloat16 *__restrict__ C, int M, int N, int K, unsigned *err) {
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
          tma_load_2d_pair(a_s, &tmA, fb, kt * BK, am);
          tma_load_2d_pair(a_s + P_A_BYTES, &tmB, fb, kt * BK, bn);
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
      const uint32_t idesc = idesc_bf16_f32(256, 256, 0, 0);
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
            mma_bf16_ss_pair(tmem + 256u * b, sdesc_sw128(a_base + 32 * k, 16, 1024),
                             sdesc_sw128(b_base + 32 * k, 16, 1024), idesc, (kt | k) != 0);
          mma_commit_pair(&empty[s], 0x3);  // both CTAs' loaders may refill stage s
        }
        if (ok) mma_commit_pair(&acc_full[b], 0x3);
      }
    }
  } else {
    const int qd = warp & 3;
    const bool vec = (N % 8) == 0;
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
        const int col = n0 + c0;
        if (row < M && col < N) {
          __nv_bfloat16 *dst = C + static_cast<long long>(row) * N + col;
          if (vec && col + 32 <= N) {
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

}  // namespace

cudaError_t launch_gemm_bf16_nt(const void *A, const void *B, void *C, int M, int N, int K, unsigned *err,
                                cudaStream_t stream) {
  alignas(64) CUtensorMap ta, tb;
  const unsigned long long dA[2] = {static_cast<unsigned long long>(K), static_cast<unsigned long long>(M)};
  const unsigned long long dB[2] = {static_cast<unsigned long long>(K), static_cast<unsigned long long>(N)};
  const unsigned long long st[1] = {static_cast<unsigned long long>(K) * 2};
  const unsigned boxA[2] = {BK, BM}, boxB[2] = {BK, BN};
  if (!encode_tmap_bf16(&ta, A, 2, dA, st, boxA, true)) return cudaErrorInvalidValue;
  if (!encode_tmap_bf16(&tb, B, 2, dB, st, boxB, true)) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if (kPairs && M >= 256) {
    // CTA pairs, persistent: as many pairs as are resident (at most one per 256 x 256 tile)
    const unsigned boxB2[2] = {BK, 128};
    if (!encode_tmap_bf16(&tb, B, 2, dB, st, boxB2, true)) return cudaErrorInvalidValue;
    if ((e = cudaFuncSetAttribute(gemm_bf16_nt_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  P_SMEM_BYTES)) != cudaSuccess)
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
    if ((e = cudaOccupancyMaxActiveClusters(&pairs, gemm_bf16_nt_pair_kernel, &cfg)) != cudaSuccess) return e;
    if (pairs < 1) return cudaErrorInvalidConfiguration;
    const long long np = std::min<long long>(pairs, tiles2);
    cfg.gridDim = dim3(static_cast<unsigned>(2 * np));
    return cudaLaunchKernelEx(&cfg, gemm_bf16_nt_pair_kernel, ta, tb, static_cast<__nv_bfloat16 *>(C), M, N, K, err);
  }
  if ((e = cudaFuncSetAttribute(gemm_bf16_nt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) !=
      cudaSuccess)
    return e;
  const long long tiles = static_cast<long long>((N + BN - 1) / BN) * ((M + BM - 1) / BM);
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  gemm_bf16_nt_kernel<<<grid, 192, SMEM_BYTES, stream>>>(ta, tb, static_cast<__nv_bfloat16 *>(C), M, N, K, err);
  return cudaGetLastError();
}

}  // namespace mta
