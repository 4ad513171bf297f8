// group_norm.cu -- depth-scaled group normalisation of head outputs.
//
// "Multi-Token Attention | Summary" (greeksharifa), section 3.3: each head's
// output is group-normalised before the heads are concatenated; "Multi-Token
// Attention" (bycloud), mechanism item 3: group normalisation with depth scaling.
// y = lambda * ((o - mean) / sqrt(var + eps) * gamma + beta), statistics over the
// d channels of one (token, head), biased variance.
//
// HBM-bound: one warp per (token, head) row, grid-stride over rows, vector loads
// when d == 128.  Used by the layer when the attention epilogue does not fuse it.
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

__global__ void __launch_bounds__(256) group_norm_d128_kernel(const __nv_bfloat16 *__restrict__ o,
                                                              GnArgs gn, long long rows, int H,
                                                              __nv_bfloat16 *__restrict__ y) {
  const int lane = threadIdx.x & 31;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long r = warp; r < rows; r += nwarps) {
    const int h = static_cast<int>(r % H);
    const uint2 raw = reinterpret_cast<const uint2 *>(o + r * 128)[lane];
    const __nv_bfloat162 p0 = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
    const __nv_bfloat162 p1 = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
    float x[4] = {__low2float(p0), __high2float(p0), __low2float(p1), __high2float(p1)};
    const float mu = warp_sum(x[0] + x[1] + x[2] + x[3]) * (1.f / 128.f);
    float s2 = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) { x[i] -= mu; s2 += x[i] * x[i]; }
    const float rstd = rsqrtf(warp_sum(s2) * (1.f / 128.f) + gn.eps);
    const float4 g4 = reinterpret_cast<const float4 *>(gn.gamma + h * 128)[lane];
    const float4 b4 = reinterpret_cast<const float4 *>(gn.beta + h * 128)[lane];
    const float m = head_multiplier(gn.gate, gn.lam, h);
    const float y0 = (x[0] * rstd * g4.x + b4.x) * m, y1 = (x[1] * rstd * g4.y + b4.y) * m;
    const float y2 = (x[2] * rstd * g4.z + b4.z) * m, y3 = (x[3] * rstd * g4.w + b4.w) * m;
    __nv_bfloat162 q0 = __floats2bfloat162_rn(y0, y1), q1 = __floats2bfloat162_rn(y2, y3);
    uint2 outw;
    outw.x = *reinterpret_cast<uint32_t *>(&q0);
    outw.y = *reinterpret_cast<uint32_t *>(&q1);
    reinterpret_cast<uint2 *>(y + r * 128)[lane] = outw;
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

}  // namespace

cudaError_t launch_group_norm(const void *o, const GnArgs &gn, int tokens, int H, int d, void *y,
                              cudaStream_t stream) {
  const long long rows = static_cast<long long>(tokens) * H;
  if (rows == 0) return cudaSuccess;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (rows + 7) / 8;  // 8 warps per block
  const int blocks = static_cast<int>(want < 8LL * sms ? want : 8LL * sms);
  const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(o);
  __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(y);
  const bool vec = d == 128 &&
                   ((reinterpret_cast<uintptr_t>(gn.gamma) | reinterpret_cast<uintptr_t>(gn.beta)) & 15) == 0 &&
                   ((reinterpret_cast<uintptr_t>(o) | reinterpret_cast<uintptr_t>(y)) & 7) == 0;
  if (vec)
    group_norm_d128_kernel<<<blocks, 256, 0, stream>>>(src, gn, rows, H, dst);
  else
    group_norm_any_kernel<<<blocks, 256, 0, stream>>>(src, gn, rows, H, d, dst);
  return cudaGetLastError();
}

}  // namespace mta
