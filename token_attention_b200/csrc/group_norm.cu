// group_norm.cu -- depth-scaled group normalisation of head outputs.
//
// "Multi-Token Attention | Summary" (greeksharifa), section 3.3: each head's
// output is group-normalised before the heads are concatenated; "Multi-Token
// Attention" (bycloud), mechanism item 3: group normalisation with depth scaling.
// y = lambda * ((o - mean) / sqrt(var + eps) * gamma + beta), statistics over the
// d channels of one (token, head), biased variance.
//
// HBM-bound (2 bytes read and 2 written per element): at d = 128 half a warp per
// (token, head) row with 16-byte loads, several rows in flight per warp; other d
// one warp per row.  Used by the layer when the attention epilogue does not fuse it.
#include <cuda_bf16.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace mta {
namespace {

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// d = 128: 16 lanes per (token, head) row, 8 channels (16 bytes) per lane, so a
// warp covers two rows; a block of 8 warps covers 16 consecutive rows per step and
// kRowsAhead steps.  Every load of a thread is issued before it reduces any row,
// so that enough bytes are in flight to keep HBM busy; one block per 16*kRowsAhead
// rows, no grid-stride loop, 32-bit row indices.
constexpr int kRowsAhead = 8;

__device__ __forceinline__ float half_warp_sum(float x) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__global__ void __launch_bounds__(256, 4) group_norm_d128_kernel(const __nv_bfloat16 *__restrict__ o,
                                                                 GnArgs gn, int rows, int H,
                                                                 __nv_bfloat16 *__restrict__ y) {
  const int lane = threadIdx.x & 31, hl = lane & 15;
  const int row0 = blockIdx.x * 16 * kRowsAhead + 2 * (threadIdx.x >> 5) + (lane >> 4);
  uint4 raw[kRowsAhead];
#pragma unroll
  for (int u = 0; u < kRowsAhead; ++u) {
    const int r = row0 + 16 * u;
    raw[u] = r < rows ? reinterpret_cast<const uint4 *>(o + static_cast<long long>(r) * 128)[hl]
                      : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int u = 0; u < kRowsAhead; ++u) {
    const int r = row0 + 16 * u;
    const uint32_t wv[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
    float x[8];
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(wv[i] << 16);
      x[2 * i + 1] = __uint_as_float(wv[i] & 0xffff0000u);
      s += x[2 * i] + x[2 * i + 1];
    }
    // both halves of the warp take every shuffle (a row past the end works on zeros)
    const float mu = half_warp_sum(s) * (1.f / 128.f);
    float s2 = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) { x[i] -= mu; s2 += x[i] * x[i]; }
    const float rstd = rsqrtf(half_warp_sum(s2) * (1.f / 128.f) + gn.eps);
    if (r >= rows) continue;
    const int h = r % H;
    const float4 *g4 = reinterpret_cast<const float4 *>(gn.gamma + h * 128 + 8 * hl);
    const float4 *b4 = reinterpret_cast<const float4 *>(gn.beta + h * 128 + 8 * hl);
    const float4 ga = __ldg(g4), gb = __ldg(g4 + 1), ba = __ldg(b4), bb = __ldg(b4 + 1);
    const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
    const float b[8] = {ba.x, ba.y, ba.z, ba.w, bb.x, bb.y, bb.z, bb.w};
    const float m = head_multiplier(gn.gate, gn.lam, h);
    uint4 outw;
    uint32_t *ow = reinterpret_cast<uint32_t *>(&outw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 q = __floats2bfloat162_rn((x[2 * i] * rstd * g[2 * i] + b[2 * i]) * m,
                                               (x[2 * i + 1] * rstd * g[2 * i + 1] + b[2 * i + 1]) * m);
      ow[i] = *reinterpret_cast<uint32_t *>(&q);
    }
    reinterpret_cast<uint4 *>(y + static_cast<long long>(r) * 128)[hl] = outw;
  }
}

__global__ void __launch_bounds__(256) group_norm_any_kernel(const __nv_bfloat16 *__restrict__ o,
                                                             GnArgs gn, long long rows, int H, int d,
                                                             __nv_bfloat16 *__restrict__ y) {
  const int lane = threadIdx.x & 31;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long r = warp; r < rows; r += nwarps) {
    const int h = static_cast<int>(r % H);
    const __nv_bfloat16 *src = o + r * d;
    float x[4];
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = lane + 32 * i;
      x[i] = e < d ? __bfloat162float(src[e]) : 0.f;
      s += x[i];
    }
    const float mu = warp_sum(s) / d;
    float s2 = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = lane + 32 * i;
      x[i] = e < d ? x[i] - mu : 0.f;
      s2 += x[i] * x[i];
    }
    const float rstd = rsqrtf(warp_sum(s2) / d + gn.eps);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = lane + 32 * i;
      if (e < d)
        y[r * d + e] = __float2bfloat16_rn((x[i] * rstd * gn.gamma[h * d + e] + gn.beta[h * d + e]) *
                                           head_multiplier(gn.gate, gn.lam, h));
    }
  }
}

// Backward of the scaled group norm, for (token, head) rows of head h = blockIdx.x:
// given dy, recomputes xhat = (o - mean) * rstd and returns
//   y  = m (xhat gamma + beta)                        (bf16, the output projection's operand)
//   do = rstd (g - mean(g) - xhat mean(g xhat)),  g = m gamma dy   (bf16)
// and adds the block's sums of dgamma = m dy xhat, dbeta = m dy and, with a gate,
// dgate_h = m (1 - m) sum dy (xhat gamma + beta) to the fp32 outputs (zeroed by the
// caller).  A warp per row, channel e = lane + 32 c in lane `lane`, CPL = d / 32
// channels per lane; 8 warps take kGnBwdRows consecutive tokens of the head, so a
// block adds 2 d (+1) values instead of 2 d per row.
constexpr int kGnBwdRows = 64;

template <int CPL>
__global__ void __launch_bounds__(256) group_norm_bwd_kernel(const __nv_bfloat16 *__restrict__ o,
                                                             const float *__restrict__ dy, GnArgs gn, int tokens,
                                                             int H, __nv_bfloat16 *__restrict__ y,
                                                             __nv_bfloat16 *__restrict__ dout, float *dgamma,
                                                             float *dbeta, float *dgate) {
  constexpr int d = 32 * CPL;
  __shared__ float red[8][2 * d + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x;
  const float m = head_multiplier(gn.gate, gn.lam, h);
  float gam[CPL], bet[CPL], dga[CPL], dbe[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    gam[c] = gn.gamma[h * d + lane + 32 * c];
    bet[c] = gn.beta[h * d + lane + 32 * c];
    dga[c] = 0.f;
    dbe[c] = 0.f;
  }
  float dgt = 0.f;
  const int t_end = min(tokens, (blockIdx.y + 1) * kGnBwdRows);
  for (int t = blockIdx.y * kGnBwdRows + warp; t < t_end; t += 8) {
    const long long base = (static_cast<long long>(t) * H + h) * d;
    float x[CPL], g[CPL];
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      x[c] = __bfloat162float(o[base + lane + 32 * c]);
      g[c] = dy[base + lane + 32 * c];
      s += x[c];
    }
    const float mu = warp_sum(s) * (1.f / d);
    float s2 = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      x[c] -= mu;
      s2 += x[c] * x[c];
    }
    const float rstd = rsqrtf(warp_sum(s2) * (1.f / d) + gn.eps);
    float sg = 0.f, sgx = 0.f, sdg = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const float xh = x[c] * rstd, aff = xh * gam[c] + bet[c];
      y[base + lane + 32 * c] = __float2bfloat16_rn(m * aff);
      dga[c] += m * g[c] * xh;
      dbe[c] += m * g[c];
      sdg += g[c] * aff;
      const float gx = m * gam[c] * g[c];
      g[c] = gx;
      x[c] = xh;
      sg += gx;
      sgx += gx * xh;
    }
    const float mg = warp_sum(sg) * (1.f / d), mgx = warp_sum(sgx) * (1.f / d);
#pragma unroll
    for (int c = 0; c < CPL; ++c)
      dout[base + lane + 32 * c] = __float2bfloat16_rn(rstd * (g[c] - mg - x[c] * mgx));
    dgt += sdg;
  }
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    red[warp][lane + 32 * c] = dga[c];
    red[warp][d + lane + 32 * c] = dbe[c];
  }
  dgt = warp_sum(dgt);
  if (lane == 0) red[warp][2 * d] = dgt;
  __syncthreads();
  for (int i = threadIdx.x; i < 2 * d + 1; i += blockDim.x) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += red[w][i];
    if (i < d)
      atomicAdd(dgamma + h * d + i, v);
    else if (i < 2 * d)
      atomicAdd(dbeta + h * d + (i - d), v);
    else if (gn.gate && dgate)
      atomicAdd(dgate + h, v * m * (1.f - m));
  }
}

}  // namespace

cudaError_t launch_group_norm_bwd(const void *o, const float *dy, const GnArgs &gn, int tokens, int H, int d,
                                  void *y, void *dout, float *dgamma, float *dbeta, float *dgate,
                                  cudaStream_t stream) {
  if (tokens == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(H), static_cast<unsigned>((tokens + kGnBwdRows - 1) / kGnBwdRows));
  const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(o);
  __nv_bfloat16 *yb = static_cast<__nv_bfloat16 *>(y), *db = static_cast<__nv_bfloat16 *>(dout);
  switch (d) {
    case 32: group_norm_bwd_kernel<1><<<grid, 256, 0, stream>>>(src, dy, gn, tokens, H, yb, db, dgamma, dbeta, dgate); break;
    case 64: group_norm_bwd_kernel<2><<<grid, 256, 0, stream>>>(src, dy, gn, tokens, H, yb, db, dgamma, dbeta, dgate); break;
    case 96: group_norm_bwd_kernel<3><<<grid, 256, 0, stream>>>(src, dy, gn, tokens, H, yb, db, dgamma, dbeta, dgate); break;
    case 128: group_norm_bwd_kernel<4><<<grid, 256, 0, stream>>>(src, dy, gn, tokens, H, yb, db, dgamma, dbeta, dgate); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_group_norm(const void *o, const GnArgs &gn, int tokens, int H, int d, void *y,
                              cudaStream_t stream) {
  const long long rows = static_cast<long long>(tokens) * H;
  if (rows == 0) return cudaSuccess;
  const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(o);
  __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(y);
  const bool vec = d == 128 && rows < (1ll << 31) - 16 * kRowsAhead &&
                   ((reinterpret_cast<uintptr_t>(gn.gamma) | reinterpret_cast<uintptr_t>(gn.beta)) & 15) == 0 &&
                   ((reinterpret_cast<uintptr_t>(o) | reinterpret_cast<uintptr_t>(y)) & 15) == 0;
  if (vec) {
    const long long blocks = (rows + 16 * kRowsAhead - 1) / (16 * kRowsAhead);
    group_norm_d128_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(src, gn, static_cast<int>(rows), H,
                                                                             dst);
  } else {
    // a warp per row, grid-stride; at most 8 blocks of 8 warps per SM
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long want = (rows + 7) / 8;
    const int blocks = static_cast<int>(want < 8LL * sms ? want : 8LL * sms);
    group_norm_any_kernel<<<blocks, 256, 0, stream>>>(src, gn, rows, H, d, dst);
  }
  return cudaGetLastError();
}

}  // namespace mta
