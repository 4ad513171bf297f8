// bwd_common.cuh -- shared-memory helpers of the CUDA-core backward kernels.
#pragma once

namespace mta {

// out(r, s, A[r] . Bm[s]) for r < nr, s < ns, dot products of length d whose rows lie
// dp floats apart in shared memory.  Each thread takes four consecutive rows of one
// column: the warp's lanes share the four row loads (broadcasts) and read distinct
// columns (dp = d + 1 keeps them in distinct banks), so the loop issues 5 loads per 4
// FMAs instead of 2 per FMA.
template <int NT, typename Out>
__device__ __forceinline__ void dot_rows4(const float *A, const float *Bm, int nr, int ns, int d, int dp,
                                          Out out) {
  const int nrb = (nr + 3) / 4;
  for (int i = threadIdx.x; i < nrb * ns; i += NT) {
    const int rb = i / ns, s = i % ns, r0 = 4 * rb;
    const float *b = Bm + s * dp;
    const float *a0 = A + min(r0, nr - 1) * dp, *a1 = A + min(r0 + 1, nr - 1) * dp;
    const float *a2 = A + min(r0 + 2, nr - 1) * dp, *a3 = A + min(r0 + 3, nr - 1) * dp;
    float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
    for (int e = 0; e < d; ++e) {
      const float x = b[e];
      v0 = fmaf(a0[e], x, v0);
      v1 = fmaf(a1[e], x, v1);
      v2 = fmaf(a2[e], x, v2);
      v3 = fmaf(a3[e], x, v3);
    }
    out(r0, s, v0);
    if (r0 + 1 < nr) out(r0 + 1, s, v1);
    if (r0 + 2 < nr) out(r0 + 2, s, v2);
    if (r0 + 3 < nr) out(r0 + 3, s, v3);
  }
}

}  // namespace mta
