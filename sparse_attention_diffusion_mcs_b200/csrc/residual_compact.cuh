// residual_compact.cuh -- the cached residual ("the residual between the
// dense and sparse attention outputs", cnshai.top post, section "MC-Sparse:
// three failure modes, one fix") stored compactly: fp32 -> bf16, rounded to
// nearest with ties to even.  The reused step then reads half the bytes per
// row in its epilogue.  One pass per plan, HBM-bound: 6 bytes per element.
#pragma once

#include "mcs_common.cuh"

namespace mcs {

constexpr int kCompactThreads = 256;

// out[i] = bf16_rn(r[i]); eight elements per thread and iteration (two float4
// loads, one 16-byte store), grid-stride; the n % 8 tail by the first threads.
__global__ void __launch_bounds__(kCompactThreads) residual_compact_kernel(const float *__restrict__ r, size_t n,
                                                                           bf16 *__restrict__ out) {
  const size_t n8 = n / 8;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t t0 = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const float4 *src = reinterpret_cast<const float4 *>(r);
  uint4 *dst = reinterpret_cast<uint4 *>(out);
  for (size_t i = t0; i < n8; i += stride) {
    const float4 a = __ldcs(src + 2 * i), b = __ldcs(src + 2 * i + 1);
    const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 p = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);   // .x low half
      w[e] = *reinterpret_cast<const uint32_t *>(&p);
    }
    dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (t0 < n % 8) out[n8 * 8 + t0] = __float2bfloat16_rn(r[n8 * 8 + t0]);
}

}  // namespace mcs
