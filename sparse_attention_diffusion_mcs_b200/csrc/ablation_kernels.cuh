// ablation_kernels.cuh -- the selection rules MC-Sparse replaces, for the
// controlled comparisons of its three failure modes (aiqbench.com abstract:
// "constraints imposed by token grouping, inaccurate interaction selection,
// and the attention contributions lost"; cnshai.top post, section "MC-Sparse:
// three failure modes, one fix").  Not on the hot path: the reused step and
// the residual pass consume whatever key lists these produce.
//
//  block_sum_kernel     block-granular scores: the sum of a group's exact
//                       probability sums over aligned blocks of keys (only
//                       full blocks); a block selection then keeps the
//                       highest blocks (topk_kernel over block scores) and
//                       expand_blocks_kernel lists their keys.
//  pooled_scores_kernel a heuristic score: the group's queries averaged into
//                       one query, and the probability that pooled query
//                       gives each key, softmax_j(scale qbar . K_j).
#pragma once

#include "mcs_common.cuh"

namespace mcs {

// bs[r, b] = sum_{t < block} scores[r, b*block + t], b < N / block; one warp
// per block score, lanes striding the block.
__global__ void block_sum_kernel(const float *__restrict__ scores, int rows, int N, int block,
                                 float *__restrict__ bs) {
  const int nb = N / block;
  const size_t n = static_cast<size_t>(rows) * nb;
  const int lane = threadIdx.x & 31;
  const size_t warps = static_cast<size_t>(gridDim.x) * (blockDim.x >> 5);
  for (size_t w = blockIdx.x * static_cast<size_t>(blockDim.x >> 5) + (threadIdx.x >> 5); w < n; w += warps) {
    const size_t r = w / nb, b = w % nb;
    const float *src = scores + r * N + b * block;
    float acc = 0.f;
    for (int t = lane; t < block; t += 32) acc += src[t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) bs[w] = acc;
  }
}

// kv[r, i*block + t] = blk[r, i]*block + t: the keys of the selected blocks,
// ascending because blk is ascending.
__global__ void expand_blocks_kernel(const int32_t *__restrict__ blk, int rows, int kb, int block,
                                     int32_t *__restrict__ kv) {
  const size_t n = static_cast<size_t>(rows) * kb * block;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t r = i / (static_cast<size_t>(kb) * block);
    const int rem = static_cast<int>(i % (static_cast<size_t>(kb) * block));
    kv[i] = blk[r * kb + rem / block] * block + rem % block;
  }
}

constexpr int kPooledThreads = 256;

// One CTA per (group, head): out[bh, g, j] = softmax_j(scale qbar_g . K_j)
// with qbar_g the mean of the group's query rows (fp32 from bf16).
template <int D>
__global__ void __launch_bounds__(kPooledThreads) pooled_scores_kernel(const bf16 *__restrict__ Q,
                                                                       const bf16 *__restrict__ K,
                                                                       const int32_t *__restrict__ perm, int N,
                                                                       int G, int n_groups, float scale_log2,
                                                                       float *__restrict__ out, unsigned *status) {
  __shared__ float qbar[D];
  __shared__ float red[kPooledThreads / 32];
  const int g = blockIdx.x, bh = blockIdx.y;
  const size_t head = static_cast<size_t>(bh) * N;
  const int r0 = g * G;
  const int rows = min(G, N - r0);
  if (threadIdx.x < D) {
    float acc = 0.f;
    for (int r = 0; r < rows; ++r) {
      int q = perm[head + r0 + r];
      if (static_cast<unsigned>(q) >= static_cast<unsigned>(N)) {   // corrupt grouping: never read past the head
        record_status(status, kStatusBadMeta);
        q = 0;
      }
      acc += __bfloat162float(Q[(head + q) * D + threadIdx.x]);
    }
    qbar[threadIdx.x] = acc / static_cast<float>(rows);
  }
  __syncthreads();
  float *row = out + (static_cast<size_t>(bh) * n_groups + g) * N;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  auto reduce = [&](float v, bool is_max) -> float {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float x = __shfl_xor_sync(0xffffffffu, v, o);
      v = is_max ? fmaxf(v, x) : v + x;
    }
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = red[0];
    for (int w = 1; w < kPooledThreads / 32; ++w) t = is_max ? fmaxf(t, red[w]) : t + red[w];
    __syncthreads();
    return t;
  };
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < N; j += kPooledThreads) {
    const uint4 *kr = reinterpret_cast<const uint4 *>(K + (head + j) * D);
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const uint4 u = kr[c];
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        s = fmaf(qbar[8 * c + 2 * e], __uint_as_float(w4[e] << 16), s);
        s = fmaf(qbar[8 * c + 2 * e + 1], __uint_as_float(w4[e] & 0xFFFF0000u), s);
      }
    }
    s *= scale_log2;
    row[j] = s;
    mx = fmaxf(mx, s);
  }
  mx = reduce(mx, true);
  float sum = 0.f;
  for (int j = threadIdx.x; j < N; j += kPooledThreads) {
    const float e = ex2_approx(row[j] - mx);
    row[j] = e;
    sum += e;
  }
  const float inv = 1.f / reduce(sum, false);
  for (int j = threadIdx.x; j < N; j += kPooledThreads) row[j] *= inv;
}

}  // namespace mcs
