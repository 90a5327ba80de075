// topk_kernel.cuh -- per-group selection of individual KV tokens, step a4.
//
// For one (head, group) row of N non-negative fp32 scores, keep the k largest
// (ties towards the lower key index) and write their key indices ascending
// ("selects individual key-value (KV) tokens", aiqbench.com abstract;
// cctest.ai "Individual KV selection").
//
// Non-negative IEEE floats order like their bit patterns as uint32, so the
// k-th largest value T is found by a most-significant-digit radix select over
// the 31 magnitude bits, in digits of 12, 11 and 8 bits.  The first digit
// (exponent plus four mantissa bits) is counted over the whole row; the keys
// whose first digit equals the threshold's are then copied into a shared
// memory candidate list, and the two remaining digits are resolved on that
// list alone.  Every key with bits > T and the first (k - #greater) keys with
// bits == T are kept.  Each warp owns a contiguous slice of the row, so the
// per-warp counts give every warp its output offset and the warps write their
// selections in index order: the output comes out ascending without a sort.
//
// One CTA per row.  The row is read from global memory once, with 16-byte
// loads four deep per lane, and kept in shared memory when it fits; longer
// rows are re-read (from L2) by the two later passes.  If the candidate list
// overflows (a near-constant row), the remaining digits are resolved by
// passes over the whole row instead.
#pragma once

#include "mcs_common.cuh"

namespace mcs {

constexpr int kTopkThreads = 1024;
constexpr int kTopkCandCap = 6144;                 // candidate list entries (bits + index)
constexpr int kTopkRowCacheBytes = 160 * 1024;     // rows up to 40,960 keys are kept in shared memory
constexpr int kTopkFixedSmem = (4096 + 2 * kTopkCandCap) * 4;   // histogram + candidate list
constexpr unsigned kTopkMagnitude = 0x7fffffffu;   // scores are >= 0; the sign bit is ignored

// exclusive scan of one int per thread over a 1024-thread block; *total gets the sum
__device__ __forceinline__ int topk_block_scan(int v, int *wsum, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const int w = wsum[lane];
    int x = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    wsum[lane] = x - w;
    if (lane == 31) wsum[32] = x;
  }
  __syncthreads();
  const int res = wsum[warp] + inc - v;
  *total = wsum[32];
  __syncthreads();
  return res;
}

// Find the bin (of nb, counted from the top) holding the kk-th largest
// candidate; returns it and replaces kk by the rank inside that bin.
__device__ __forceinline__ unsigned topk_select_bin(const unsigned *hist, int nb, int &kk, int *wsum,
                                                    unsigned *s_bin, int *s_rank) {
  const int per = nb >= kTopkThreads ? nb / kTopkThreads : 1;
  const int t = threadIdx.x;
  const bool holds = t * per < nb;
  const int top = nb - 1 - t * per;          // this thread's bins, descending: top .. top-per+1
  int lsum = 0;
  if (holds)
    for (int b = 0; b < per; ++b) lsum += static_cast<int>(hist[top - b]);
  int total;
  const int before = topk_block_scan(lsum, wsum, &total);
  if (holds && before < kk && before + lsum >= kk) {
    int acc = before;
    for (int b = 0; b < per; ++b) {
      const int c = static_cast<int>(hist[top - b]);
      if (acc + c >= kk) {
        *s_bin = static_cast<unsigned>(top - b);
        *s_rank = kk - acc;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
  kk = *s_rank;
  const unsigned bin = *s_bin;
  __syncthreads();
  return bin;
}

// Walk this warp's slice [lo, hi) of the row in index order, VEC keys per lane
// per step and four steps of loads in flight; f(j0, keys, valid) is called by
// every lane of the warp for every step (it may use warp votes).
template <int VEC, class F>
__device__ __forceinline__ void topk_walk(const unsigned *__restrict__ src, bool from_smem, int lo, int hi,
                                          F &&f) {
  constexpr int STEP = 32 * VEC;
  const int lane = threadIdx.x & 31;
  for (int b = lo; b < hi; b += 4 * STEP) {
    unsigned x[4][VEC];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j0 = b + u * STEP + VEC * lane;
      if (j0 < hi) {
        if constexpr (VEC == 4) {
          const uint4 v = from_smem ? *reinterpret_cast<const uint4 *>(src + j0)
                                    : __ldg(reinterpret_cast<const uint4 *>(src + j0));
          x[u][0] = v.x;
          x[u][1] = v.y;
          x[u][2] = v.z;
          x[u][3] = v.w;
        } else {
          x[u][0] = from_smem ? src[j0] : __ldg(src + j0);
        }
      } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) x[u][e] = 0u;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (b + u * STEP >= hi) break;   // warp-uniform
      const int j0 = b + u * STEP + VEC * lane;
      unsigned key[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) key[e] = x[u][e] & kTopkMagnitude;
      f(j0, key, j0 < hi);
    }
  }
}

// VEC = 4 needs N % 4 == 0 and a 16-byte aligned score array.
template <int VEC>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float *__restrict__ colsum, int N, int k,
                                                            int cache_row, int32_t *__restrict__ kv_idx) {
  // dynamic shared memory: histogram, candidate list, then the row when cache_row
  extern __shared__ __align__(16) unsigned topk_sm[];
  unsigned *hist = topk_sm;
  unsigned *cand_bits = hist + 4096;
  int *cand_idx = reinterpret_cast<int *>(cand_bits + kTopkCandCap);
  unsigned *row_sm = reinterpret_cast<unsigned *>(cand_idx + kTopkCandCap);
  __shared__ int wsum[33];
  __shared__ int gt_cnt[32], eq_cnt[32], w_take[32], w_base[32];
  __shared__ unsigned s_bin;
  __shared__ int s_rank, s_ncand;

  const size_t row = blockIdx.x;
  const unsigned *ug = reinterpret_cast<const unsigned *>(colsum + row * N);
  int32_t *out = kv_idx + row * k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;

  if (k >= N) {
    for (int j = tid; j < N; j += blockDim.x) out[j] = j;
    return;
  }
  constexpr int STEP = 32 * VEC;
  const int span = ((N + 31) / 32 + STEP - 1) / STEP * STEP;
  const int lo = min(N, warp * span), hi = min(N, lo + span);
  const bool cached = cache_row != 0;
  const unsigned *src = cached ? row_sm : ug;

  for (int i = tid; i < 4096; i += kTopkThreads) hist[i] = 0;
  if (tid < 32) gt_cnt[tid] = eq_cnt[tid] = 0;
  if (tid == 0) s_ncand = 0;
  __syncthreads();

  // ---- pass 1 (global): cache the row, count the first digit (bits 30..19)
  topk_walk<VEC>(ug, false, lo, hi, [&](int j0, const unsigned *key, bool valid) {
    if (!valid) return;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      if (cached) row_sm[j0 + e] = key[e];
      atomicAdd(&hist[key[e] >> 19], 1u);
    }
  });
  __syncthreads();
  int kk = k;
  const unsigned b1 = topk_select_bin(hist, 4096, kk, wsum, &s_bin, &s_rank);
  for (int i = tid; i < 4096; i += kTopkThreads) hist[i] = 0;

  // ---- pass 2: per-warp count above the threshold's bin; candidates into the list
  int above = 0;
  topk_walk<VEC>(src, cached, lo, hi, [&](int j0, const unsigned *key, bool valid) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const unsigned d = key[e] >> 19;
      above += (valid && d > b1) ? 1 : 0;
      const bool c = valid && d == b1;
      const unsigned bal = __ballot_sync(0xffffffffu, c);
      if (bal == 0u) continue;
      int base = 0;
      if (lane == 0) base = atomicAdd(&s_ncand, __popc(bal));
      base = __shfl_sync(0xffffffffu, base, 0);
      const int pos = base + __popc(bal & lt);
      if (c && pos < kTopkCandCap) {
        cand_bits[pos] = key[e];
        cand_idx[pos] = j0 + e;
      }
    }
  });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
  if (lane == 0) gt_cnt[warp] = above;
  __syncthreads();
  const int ncand = s_ncand;
  const bool listed = ncand <= kTopkCandCap;

  // ---- passes 3, 4: bits 18..8, then 7..0, over the candidates
  unsigned prefix = b1 << 19, mask = 0xfffu << 19;
  for (int pass = 0; pass < 2; ++pass) {
    const int shift = pass == 0 ? 8 : 0;
    const int nb = pass == 0 ? 2048 : 256;
    const unsigned dm = static_cast<unsigned>(nb - 1);
    if (listed) {
      for (int i = tid; i < ncand; i += kTopkThreads) {
        const unsigned x = cand_bits[i];
        if ((x & mask) == prefix) atomicAdd(&hist[(x >> shift) & dm], 1u);
      }
    } else {
      topk_walk<VEC>(src, cached, lo, hi, [&](int, const unsigned *key, bool valid) {
        if (!valid) return;
#pragma unroll
        for (int e = 0; e < VEC; ++e)
          if ((key[e] & mask) == prefix) atomicAdd(&hist[(key[e] >> shift) & dm], 1u);
      });
    }
    __syncthreads();
    const unsigned bin = topk_select_bin(hist, nb, kk, wsum, &s_bin, &s_rank);
    prefix |= bin << shift;
    mask |= dm << shift;
    for (int i = tid; i < nb; i += kTopkThreads) hist[i] = 0;
  }
  const unsigned T = prefix;
  const int need_eq = kk;   // keys equal to T to keep: the first need_eq of them in index order

  // ---- per-warp counts of keys above T and equal to T
  if (listed) {
    for (int i = tid; i < ncand; i += kTopkThreads) {
      const unsigned x = cand_bits[i];
      const int w = cand_idx[i] / span;
      if (x > T) atomicAdd(&gt_cnt[w], 1);
      else if (x == T) atomicAdd(&eq_cnt[w], 1);
    }
  } else {
    int g = 0, q = 0;
    topk_walk<VEC>(src, cached, lo, hi, [&](int, const unsigned *key, bool valid) {
      if (!valid) return;
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        if ((key[e] >> 19) != b1) continue;
        g += key[e] > T ? 1 : 0;
        q += key[e] == T ? 1 : 0;
      }
    });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      g += __shfl_xor_sync(0xffffffffu, g, o);
      q += __shfl_xor_sync(0xffffffffu, q, o);
    }
    if (lane == 0) {
      gt_cnt[warp] += g;
      eq_cnt[warp] = q;
    }
  }
  __syncthreads();
  if (warp == 0) {
    const int e = eq_cnt[lane];
    int x = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    const int take = max(0, min(e, need_eq - (x - e)));
    const int sel = gt_cnt[lane] + take;
    int s = sel;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    w_take[lane] = take;
    w_base[lane] = s - sel;
  }
  __syncthreads();

  // ---- pass 5: each warp writes its selected keys in index order
  const int eq_take = w_take[warp];
  int written = w_base[warp], eq_seen = 0;
  topk_walk<VEC>(src, cached, lo, hi, [&](int j0, const unsigned *key, bool valid) {
    unsigned beq[VEC];
    int own_eq = 0;
#pragma unroll
    for (int e = 0; e < VEC; ++e) beq[e] = __ballot_sync(0xffffffffu, valid && key[e] == T);
    int eq_lanes_before = 0;
#pragma unroll
    for (int e = 0; e < VEC; ++e) eq_lanes_before += __popc(beq[e] & lt);
    bool take[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const bool is_eq = valid && key[e] == T;
      take[e] = valid && (key[e] > T || (is_eq && eq_seen + eq_lanes_before + own_eq < eq_take));
      own_eq += is_eq ? 1 : 0;
    }
    unsigned bsel[VEC];
    int sel_lanes_before = 0, step_sel = 0;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      bsel[e] = __ballot_sync(0xffffffffu, take[e]);
      sel_lanes_before += __popc(bsel[e] & lt);
      step_sel += __popc(bsel[e]);
      eq_seen += __popc(beq[e]);
    }
    int own_sel = 0;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      if (take[e]) {
        const int pos = written + sel_lanes_before + own_sel;
        if (pos < k) out[pos] = j0 + e;
        ++own_sel;
      }
    }
    written += step_sel;
  });
}

}  // namespace mcs
