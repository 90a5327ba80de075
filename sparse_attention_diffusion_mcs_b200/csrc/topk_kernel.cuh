// topk_kernel.cuh -- per-group selection of individual KV tokens, step a4.
//
// For one (head, group) row of N non-negative fp32 scores, keep the k largest
// (ties towards the lower key index) and write their key indices ascending
// ("selects individual key-value (KV) tokens", aiqbench.com abstract;
// cctest.ai "Individual KV selection").
//
// Non-negative IEEE floats order like their bit patterns as uint32, so the
// k-th largest value T is found by a most-significant-digit radix select over
// 4 x 8-bit digits (histograms in shared memory, warp-aggregated atomics).
// A final pass in index order keeps every key with bits > T and the first
// (k - #greater) keys with bits == T, so the output comes out ascending
// without a sort.  One CTA per row; the row streams from L2/HBM 5 times.
#pragma once

#include "mcs_common.cuh"

namespace mcs {

constexpr int kTopkThreads = 1024;

// exclusive block scan of one int per thread; returns the prefix, *total gets the sum
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_sums, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (blockDim.x >> 5) ? warp_sums[lane] : 0;
    int inc = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    warp_sums[lane] = inc - w;          // exclusive prefix of warp totals
    if (lane == 31) warp_sums[32] = inc;
  }
  __syncthreads();
  const int res = warp_sums[warp] + x - v;
  *total = warp_sums[32];
  __syncthreads();
  return res;
}

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float *__restrict__ colsum, int N,
                                                            int k, int32_t *__restrict__ kv_idx) {
  __shared__ unsigned hist[256];
  __shared__ int warp_sums[33];
  __shared__ unsigned sel_digit;
  __shared__ int sel_rank;

  const size_t row = blockIdx.x;
  const unsigned *u = reinterpret_cast<const unsigned *>(colsum + row * N);
  int32_t *out = kv_idx + row * k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (k >= N) {
    for (int j = tid; j < N; j += blockDim.x) out[j] = j;
    return;
  }

  unsigned prefix = 0, mask = 0;
  int kk = k;   // rank from the top, among candidates, of the value sought
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int base = 0; base < N; base += blockDim.x) {
      const int j = base + tid;
      unsigned x = 0;
      bool cand = false;
      if (j < N) {
        x = __ldg(u + j);
        cand = (x & mask) == prefix;
      }
      const unsigned digit = (x >> shift) & 255u;
      const unsigned cm = __ballot_sync(0xffffffffu, cand);
      if (cand) {
        const unsigned peers = __match_any_sync(cm, digit);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
      }
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds bins 255-8l .. 248-8l (descending)
      unsigned cnt[8];
      unsigned lsum = 0;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        cnt[b] = hist[255 - 8 * lane - b];
        lsum += cnt[b];
      }
      unsigned inc = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const unsigned before = inc - lsum;
      const bool here = before < static_cast<unsigned>(kk) && inc >= static_cast<unsigned>(kk);
      if (here) {
        unsigned acc = before;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          if (acc + cnt[b] >= static_cast<unsigned>(kk)) {
            sel_digit = 255u - 8u * lane - b;
            sel_rank = kk - static_cast<int>(acc);
            break;
          }
          acc += cnt[b];
        }
      }
    }
    __syncthreads();
    prefix |= sel_digit << shift;
    mask |= 255u << shift;
    kk = sel_rank;
    __syncthreads();
  }
  const unsigned Tbits = prefix;
  const int need_eq = kk;        // how many keys equal to the threshold to keep

  int written = 0, eq_seen = 0;
  for (int base = 0; base < N; base += blockDim.x) {
    const int j = base + tid;
    unsigned x = 0;
    if (j < N) x = __ldg(u + j);
    const int gt = (j < N && x > Tbits) ? 1 : 0;
    const int eq = (j < N && x == Tbits) ? 1 : 0;
    int eq_total;
    const int eq_rank = block_exclusive_scan(eq, warp_sums, &eq_total);
    const int take = gt | (eq && (eq_seen + eq_rank) < need_eq);
    int take_total;
    const int pos = block_exclusive_scan(take, warp_sums, &take_total);
    if (take) out[written + pos] = j;
    written += take_total;
    eq_seen += eq_total;
  }
}

}  // namespace mcs
