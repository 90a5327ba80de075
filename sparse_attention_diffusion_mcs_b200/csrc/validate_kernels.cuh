// validate_kernels.cuh -- metadata checks that never trap, and a self-test of
// the bounded mbarrier wait used by every pipelined kernel.
#pragma once

#include "mcs_common.cuh"

namespace mcs {

// Bit (bh*N + value) of `seen` is set for every perm entry; a second hit or an
// out-of-range value records code 1.  `bad` keeps the smallest failing check
// code (INT_MAX = none).  `seen` must be zeroed and hold BH*N bits.
__global__ void perm_mark_kernel(const int32_t *__restrict__ perm, int N, int BH,
                                 unsigned *__restrict__ seen, int *__restrict__ bad) {
  const size_t n = static_cast<size_t>(BH) * N;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t bh = i / N;
    const int v = perm[i];
    if (v < 0 || v >= N) {
      atomicMin(bad, 1);
      continue;
    }
    const size_t bit = bh * N + v;
    const unsigned m = 1u << (bit & 31);
    const unsigned prev = atomicOr(seen + (bit >> 5), m);
    if (prev & m) atomicMin(bad, 1);
  }
}

__global__ void kv_check_kernel(const int32_t *__restrict__ kv, int N, int k, size_t rows,
                                int *__restrict__ bad) {
  const size_t n = rows * k;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int v = kv[i];
    if (v < 0 || v >= N) atomicMin(bad, 2);
    if (i % k != 0 && kv[i - 1] >= v) atomicMin(bad, 3);
  }
}

__global__ void residual_check_kernel(const float *__restrict__ r, size_t n, int *__restrict__ bad) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    if (!isfinite(r[i])) atomicMin(bad, 4);
  }
}

// Pair union lists (pair_kernel.cuh): every length in [k, 2k] (exactly k for
// a lone last group) and every listed entry in [0, N); else code 5.
__global__ void pair_check_kernel(const int32_t *__restrict__ pair_idx, const int32_t *__restrict__ pair_len,
                                  int N, int kk, int n_groups, int n_pairs, size_t items, int *__restrict__ bad) {
  for (size_t it = blockIdx.x; it < items; it += gridDim.x) {
    const int p = static_cast<int>(it % n_pairs);
    const int umax = 2 * p + 1 < n_groups ? 2 * kk : kk;
    const int u = pair_len[it];
    if (u < kk || u > umax) {
      if (threadIdx.x == 0) atomicMin(bad, 5);
      continue;
    }
    const int32_t *L = pair_idx + it * 2 * static_cast<size_t>(kk);
    for (int i = threadIdx.x; i < u; i += blockDim.x) {
      const int v = L[i];
      if (v < 0 || v >= N) atomicMin(bad, 5);
    }
  }
}

// Waits on an mbarrier that nothing ever arrives on.  The bounded wait gives
// up after limit_ns and records the timeout in the status word; the kernel
// then returns normally.
__global__ void wait_selftest_kernel(uint64_t limit_ns, unsigned *status) {
  __shared__ alignas(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    abort_flag = 0;
    mbar_init_fence();
  }
  __syncthreads();
  const bool ok = mbar_wait(b, 0, limit_ns, &abort_flag);
  if (!ok) record_status(status, kStatusTimeout);
}

}  // namespace mcs
