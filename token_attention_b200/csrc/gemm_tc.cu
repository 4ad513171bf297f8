// gemm_tc.cu -- bf16 GEMM on the sm_100a tensor cores: C[M][N] = A[M][K] B[N][K]^T.
//
// Used for the two projections of the MTA layer ("Multi-Token Attention |
// Summary" (greeksharifa), section 2): QKV = x Wqkv^T and out = Y Wo^T.
//
// One CTA computes one 128 x 256 tile of C.  Warp 0 streams 64-wide K slices of
// A and B with TMA (128-byte swizzle) into a 4-stage shared-memory ring; warp 1
// issues tcgen05.mma (M=128, N=256, K=16) into a 128 x 256 fp32 accumulator in
// tensor memory; warps 2..5 read the accumulator back with tcgen05.ld and store
// bf16.  Every mbarrier wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace mta {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BYTES = BN * BK * 2;            // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 48 KB
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t TMEM_COLS = 256;

__global__ void __launch_bounds__(192, 1)
    gemm_bf16_nt_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        __nv_bfloat16 *__restrict__ C, int M, int N, int K, unsigned *err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
  uint64_t *empty = full + STAGES;
  uint64_t *accum = empty + STAGES;
  uint32_t *tslot = reinterpret_cast<uint32_t *>(accum + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int nk = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(accum, 1);
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
      int issued = 0;
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % STAGES;
        const uint32_t ph = (kt / STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, err)) break;
        uint8_t *a_s = smem + s * STAGE_BYTES;
        mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
        tma_load_2d(a_s, &tmA, &full[s], kt * BK, m0);
        tma_load_2d(a_s + A_BYTES, &tmB, &full[s], kt * BK, n0);
        ++issued;
      }
      if (*abort_flag)  // let copies in flight land before the CTA exits
        for (int kt = (issued > STAGES ? issued - STAGES : 0); kt < issued; ++kt)
          drain_wait(&full[kt % STAGES], (kt / STAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 0);
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % STAGES;
        const uint32_t ph = (kt / STAGES) & 1;
        if (!mbar_wait(&full[s], ph, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + s * STAGE_BYTES);
        const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)  // K=16 per MMA: +32 bytes inside the 128-byte swizzle row
          mma_bf16_ss(tmem, sdesc_sw128(a_base + 32 * k, 16, 1024), sdesc_sw128(b_base + 32 * k, 16, 1024),
                      idesc, (kt | k) != 0);
        mma_commit(&empty[s]);
      }
      mma_commit(accum);
    }
  } else {
    mbar_wait(accum, 0, abort_flag, err);
    tc_fence_after();
    const int qd = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = m0 + 32 * qd + lane;
    const bool vec = (N % 8) == 0;
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * qd) << 16) + c0, r);
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
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, TMEM_COLS); }
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
  cudaError_t e = cudaFuncSetAttribute(gemm_bf16_nt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  gemm_bf16_nt_kernel<<<grid, 192, SMEM_BYTES, stream>>>(ta, tb, static_cast<__nv_bfloat16 *>(C), M, N, K, err);
  return cudaGetLastError();
}

}  // namespace mta
