// gemm_batched.cu -- batched bf16 GEMM on the sm_100a tensor cores for the
// attention backward: C[z][m][n] = alpha * sum_k A[z][m][k] B[z][n][k]
// (+ C[z][m][n] when accumulating), z = b * H + h over the batch and the heads.
//
// The operands are read in place from the attention's own tensors through
// four-dimensional TMA maps (a [B][L][H][d] tensor with its token stride, or a
// [B][H][rows][pitch] strip of the backward), each either K-major (its rows are
// M or N, its contiguous dimension K) or MN-major (contiguous M or N, rows K),
// with a coordinate offset on both indices, so that a query block's rows of Q or
// dO, or the hi / lo half of a strip, are addressed without a copy.  C is fp32
// with arbitrary element strides (rows of dq, dk, dv in [B][L][H][d], or a strip).
//
// Persistent: one CTA per SM walks the (z, 128-row, BN-column) tiles.  Warp 0
// streams 64-wide K slices of A and B with TMA (128-byte swizzle) through a
// 4-stage ring; warp 1 runs the MMA loop in all lanes and issues tcgen05.mma
// (M=128, N=BN, K=16) from one elected lane into one of two BN-column fp32
// accumulators in tensor memory; warps 2..5 read a finished tile back with
// tcgen05.ld while the next tile's MMAs run, 32 rows x 32 columns at a time, into
// a 128-byte-swizzled shared-memory box that one lane writes out with a TMA store
// (or, accumulating, a TMA add into the fp32 output).  A warp's 32 rows then
// leave as whole 128-byte lines, not as 32 scattered 16-byte pieces per
// instruction.  Every mbarrier wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace mta {
namespace {

constexpr int BM = 128, BK = 64, STAGES = 4;
constexpr int PANEL = 64 * BK * 2;  // an MN-major box: 64 rows x 64 K, 8 KB

constexpr int EBOX = 32 * 32 * 4;  // an epilogue box: 32 rows x 32 fp32, 4 KB

template <int BN>
struct BG {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int EPI = 4 * 2 * EBOX;  // two boxes per epilogue warp
  static constexpr int SMEM = STAGES * STAGE + EPI + 1024 + 256;
  static constexpr uint32_t TMEM_COLS = 2 * BN;
  static_assert(SMEM <= 232448, "shared memory");
};

// Loads rows [r, r + R) x K slice [k, k + 64) of operand `o` for batch (b, h).
// The map's coordinates are (c0 contiguous, c1, c2, c3 = b) with the row index at
// position o.pos_row and the head at the other of 1 and 2.
template <int R>
__device__ __forceinline__ void load_op(uint8_t *dst, const CUtensorMap *map, const BgOperand &o, uint64_t *bar,
                                        int r, int k, int b, int h) {
  auto load = [&](uint8_t *d, int c0, int row) {
    if (o.pos_row == 1)
      tma_load_4d(d, map, bar, c0, row, h, b);
    else
      tma_load_4d(d, map, bar, c0, h, row, b);
  };
  if (o.k_period) {
    r += (k / o.k_period) * o.period_shift;
    k %= o.k_period;
  }
  if (!o.mn) {
    load(dst, k + o.off_k, r + o.off_mn);
  } else {
#pragma unroll
    for (int p = 0; p < R / 64; ++p) load(dst + p * PANEL, r + o.off_mn + 64 * p, k + o.off_k);
  }
}

__device__ __forceinline__ uint64_t op_desc(bool mn, uint32_t base, int k) {
  return mn ? sdesc_sw128(base + 2048 * k, PANEL, 1024) : sdesc_sw128(base + 32 * k, 16, 1024);
}

template <int BN>
__global__ void __launch_bounds__(192, 1)
    gemm_batched_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmC, const BgArgs p) {
  using G = BG<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *epi = smem + STAGES * G::STAGE;  // 1024-aligned: STAGE is a multiple of 8 KB
  uint64_t *full = reinterpret_cast<uint64_t *>(epi + G::EPI);
  uint64_t *empty = full + STAGES;
  uint64_t *acc_full = empty + STAGES;  // [2]
  uint64_t *acc_empty = acc_full + 2;   // [2]
  uint32_t *tslot = reinterpret_cast<uint32_t *>(acc_empty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tm = (p.M + BM - 1) / BM, n_tn = (p.N + BN - 1) / BN;
  const int per_z = n_tm * n_tn * p.ksplit, n_tiles = p.Z * per_z;
  const int nk_all = (p.K + BK - 1) / BK, nkc = (nk_all + p.ksplit - 1) / p.ksplit;
  // tile t: batch z, output block (m0, n0), K slices [k0, k1) (every range non-empty)
  auto tile_of = [&](int t, int &z, int &m0, int &n0, int &k0, int &k1) {
    z = t / per_z;
    int r = t - z * per_z;
    const int ks = r % p.ksplit;
    r /= p.ksplit;
    m0 = (r / n_tn) * BM;
    n0 = (r % n_tn) * BN;
    k0 = ks * nkc;
    k1 = min(nk_all, k0 + nkc);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 4); }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
  }
  if (warp == 1) { tmem_alloc(tslot, G::TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int t = blockIdx.x; t < n_tiles && !*abort_flag; t += gridDim.x) {
        int z, m0, n0, k0, k1;
        tile_of(t, z, m0, n0, k0, k1);
        const int b = z / p.H, h = z - b * p.H;
        for (int kt = k0; kt < k1; ++kt, ++issued) {
          const int s = issued % STAGES;
          if (!mbar_wait(&empty[s], ((issued / STAGES) & 1) ^ 1, abort_flag, p.err)) break;
          uint8_t *a_s = smem + s * G::STAGE;
          mbar_arrive_expect_tx(&full[s], G::STAGE);
          load_op<BM>(a_s, &tmA, p.a, &full[s], m0, kt * BK, b, h);
          load_op<BN>(a_s + G::A_BYTES, &tmB, p.b, &full[s], n0, kt * BK, b, h);
        }
      }
      if (*abort_flag)  // let copies in flight land before the CTA exits
        for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
          drain_wait(&full[i % STAGES], (i / STAGES) & 1);
    }
  } else if (warp == 1) {
    // the whole warp runs the loop; one elected lane issues
    const bool issuer = elect_one();
    auto wwait = [&](uint64_t *bar, uint32_t ph) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, ph, abort_flag, p.err));
    };
    const uint32_t idesc = idesc_bf16_f32(BM, BN, p.a.mn, p.b.mn);
    int used = 0, local = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++local) {
      const int ab = local & 1;
      if (local >= 2 && !wwait(&acc_empty[ab], ((local >> 1) - 1) & 1)) break;
      tc_fence_after();
      int z, m0, n0, k0, k1;
      tile_of(t, z, m0, n0, k0, k1);
      for (int kt = k0; kt < k1; ++kt, ++used) {
        const int s = used % STAGES;
        if (!wwait(&full[s], (used / STAGES) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + s * G::STAGE);
        const uint32_t b_base = a_base + G::A_BYTES;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          mma_ss_if(issuer, tmem + BN * ab, op_desc(p.a.mn, a_base, k), op_desc(p.b.mn, b_base, k), idesc,
                    (kt - k0) + k != 0);
        mma_commit_if(issuer, &empty[s]);
      }
      if (ok) mma_commit_if(issuer, &acc_full[ab]);
    }
  } else {
    // warp 2 + q takes TMEM lanes (tile rows) 32 qd .. 32 qd + 31, qd = warp & 3
    const int qd = warp & 3;
    uint8_t *ebox = epi + qd * 2 * EBOX;
    int local = 0, nbox = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++local) {
      const int ab = local & 1;
      if (!mbar_wait(&acc_full[ab], (local >> 1) & 1, abort_flag, p.err)) break;
      tc_fence_after();
      int z, m0, n0, k0, k1;
      tile_of(t, z, m0, n0, k0, k1);
      const int b = z / p.H, h = z - b * p.H;
      const int r0 = m0 + 32 * qd;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32, ++nbox) {
        uint32_t r[32];
        tmem_ld32(tmem + BN * ab + (static_cast<uint32_t>(32 * qd) << 16) + c0, r);
        tmem_wait_ld();
        // the box written two boxes ago has been read by its store
        uint8_t *box = ebox + (nbox & 1) * EBOX;
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        // row `lane` of the box; its 16-byte chunk i sits at i ^ (row & 7) (128-byte swizzle)
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<float4 *>(box + lane * 128 + ((i ^ (lane & 7)) << 4)) =
              make_float4(p.alpha * __uint_as_float(r[4 * i]), p.alpha * __uint_as_float(r[4 * i + 1]),
                          p.alpha * __uint_as_float(r[4 * i + 2]), p.alpha * __uint_as_float(r[4 * i + 3]));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // rows past M and columns past N are clipped by the map
          if (r0 < p.M && n0 + c0 < p.N) {
            const int c1 = p.c_pos_row == 1 ? r0 : h, c2 = p.c_pos_row == 1 ? h : r0;
            if (p.accumulate)
              tma_reduce_add_4d(&tmC, box, n0 + c0, c1, c2, b);
            else
              tma_store_4d(&tmC, box, n0 + c0, c1, c2, b);
          }
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
    if (lane == 0) bulk_wait_all();  // the output is written before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, G::TMEM_COLS); }
}

}  // namespace

bool make_bg_map(void *map, const BgTensor &t, bool mn, int rows) {
  unsigned box[4] = {64u, 1u, 1u, 1u};
  box[t.pos_row] = mn ? 64u : static_cast<unsigned>(rows);
  return encode_tmap_bf16(map, t.base, 4, t.dims, t.strides, box, true);
}

// The output as a 4-D fp32 map (n, m or h, h or m, b), the two middle dimensions in
// increasing stride order; boxes of 32 columns x 32 rows, 128-byte swizzle.
static bool make_c_map(CUtensorMap *map, BgArgs &a) {
  if ((reinterpret_cast<uintptr_t>(a.C) & 15) || ((a.sm | a.sh | a.sb) & 3) || a.Z % a.H) return false;
  const bool m_first = a.sm <= a.sh;
  a.c_pos_row = m_first ? 1 : 2;
  const unsigned long long B = static_cast<unsigned long long>(a.Z / a.H);
  unsigned long long dims[4] = {static_cast<unsigned long long>(a.N), 0, 0, B};
  unsigned long long str[3] = {0, 0, static_cast<unsigned long long>(a.sb) * 4};
  dims[1] = m_first ? static_cast<unsigned long long>(a.M) : static_cast<unsigned long long>(a.H);
  dims[2] = m_first ? static_cast<unsigned long long>(a.H) : static_cast<unsigned long long>(a.M);
  str[0] = static_cast<unsigned long long>(m_first ? a.sm : a.sh) * 4;
  str[1] = static_cast<unsigned long long>(m_first ? a.sh : a.sm) * 4;
  unsigned box[4] = {32u, 1u, 1u, 1u};
  box[a.c_pos_row] = 32u;
  return encode_tmap_f32(map, a.C, 4, dims, str, box, true);
}

cudaError_t launch_gemm_batched(const BgTensor &A, const BgTensor &B, const BgArgs &args_in, cudaStream_t stream) {
  BgArgs args = args_in;
  if (args.Z < 1 || args.M < 1 || args.N < 1 || args.K < 1) return cudaSuccess;
  // the contiguous coordinate of every TMA box must start on 16 bytes
  if ((args.a.mn ? args.a.off_mn : args.a.off_k) % 8 != 0 || (args.b.mn ? args.b.off_mn : args.b.off_k) % 8 != 0)
    return cudaErrorInvalidValue;
  if (A.pos_row != args.a.pos_row || B.pos_row != args.b.pos_row) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  alignas(64) CUtensorMap ta, tb, tc;
  if (!make_c_map(&tc, args)) return cudaErrorInvalidValue;
  args.ksplit = 1;
  auto run = [&](auto kern, int bn, int smem) -> cudaError_t {
    if (!make_bg_map(&ta, A, args.a.mn, BM) || !make_bg_map(&tb, B, args.b.mn, bn)) return cudaErrorInvalidValue;
    cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e2 != cudaSuccess) return e2;
    const long long tiles =
        static_cast<long long>(args.Z) * ((args.M + BM - 1) / BM) * ((args.N + bn - 1) / bn) * args.ksplit;
    const int grid = static_cast<int>(std::min<long long>(tiles, sms));
    kern<<<grid, 192, smem, stream>>>(ta, tb, tc, args);
    return cudaGetLastError();
  };
  if (args.N > 128) return run(gemm_batched_kernel<256>, 256, BG<256>::SMEM);
  // narrow outputs: when 128-column tiles would leave SMs idle, K in two halves
  // (added into the zeroed output: with exactly two partial sums the result does not
  // depend on their order) or else 64-column tiles
  const long long t128 = static_cast<long long>(args.Z) * ((args.M + BM - 1) / BM) * ((args.N + 127) / 128);
  if (args.N > 64 && t128 < sms && args.split_ok && args.accumulate && (args.K + BK - 1) / BK >= 2) {
    args.ksplit = 2;
    return run(gemm_batched_kernel<128>, 128, BG<128>::SMEM);
  }
  if (args.N <= 64 || t128 < sms) return run(gemm_batched_kernel<64>, 64, BG<64>::SMEM);
  return run(gemm_batched_kernel<128>, 128, BG<128>::SMEM);
}

}  // namespace mta
