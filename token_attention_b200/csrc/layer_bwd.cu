// layer_bwd.cu -- the one elementwise step of the layer's backward pass that is
// not part of another kernel: packing the attention core's fp32 gradients of
// q, k and v into the bf16 [tokens][3 D] operand of the two projection-gradient
// GEMMs (dx = dQKV Wqkv and dWqkv = dQKV^T x; "Multi-Token Attention | Summary"
// (greeksharifa), section 2: Q, K and V are projections of the same input).
//
// HBM-bound: 12 bytes read and 6 written per element of each of dq, dk, dv;
// four consecutive channels per thread (16-byte loads, 8-byte stores).
#include <cuda_bf16.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace mta {
namespace {

__global__ void __launch_bounds__(256) pack_qkv_grad_kernel(const float *__restrict__ dq, const float *__restrict__ dk,
                                                            const float *__restrict__ dv, long long n4, int hd4,
                                                            uint2 *__restrict__ out) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    // i: group of 4 channels of one source; token t, channel group c of that source
    const long long t = i / hd4;
    const int c = static_cast<int>(i - t * hd4);
    const long long o = t * 3 * hd4 + c;
    const float4 a = reinterpret_cast<const float4 *>(dq)[i];
    const float4 b = reinterpret_cast<const float4 *>(dk)[i];
    const float4 v = reinterpret_cast<const float4 *>(dv)[i];
    out[o] = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
    out[o + hd4] = make_uint2(pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
    out[o + 2 * hd4] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

}  // namespace

cudaError_t launch_pack_qkv_grad(const float *dq, const float *dk, const float *dv, long long tokens, int hd,
                                 void *dqkv, cudaStream_t stream) {
  if (hd % 4 != 0) return cudaErrorInvalidValue;
  const long long n4 = tokens * (hd / 4);
  if (n4 == 0) return cudaSuccess;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (n4 + 255) / 256;
  const int blocks = static_cast<int>(want < 8LL * sms ? want : 8LL * sms);
  pack_qkv_grad_kernel<<<blocks, 256, 0, stream>>>(dq, dk, dv, n4, hd / 4, static_cast<uint2 *>(dqkv));
  return cudaGetLastError();
}

}  // namespace mta
