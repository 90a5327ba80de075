// topk_kernel.cuh -- per-group selection of individual KV tokens, step a4.
//
// For one (head, group) row of N non-negative fp32 scores, keep the k largest
// (ties towards the lower key index) and write their key indices ascending
// ("selects individual key-value (KV) tokens", aiqbench.com abstract;
// cctest.ai "Individual KV selection").
//
// Non-negative IEEE floats order like their bit patterns as uint32, so the
// k-th largest value T is found by a most-significant-digit radix select over
// the 31 magnitude bits in three digits (D1 bits, then the rest in two).  The
// first digit is counted over the whole row; the keys whose first digit
// equals the threshold's are then copied into a shared memory candidate list,
// and the two remaining digits are resolved on that list alone.  Every key
// with bits > T and the first (k - #greater) keys with bits == T are kept.
// Each warp owns a contiguous slice of the row, so the per-warp counts give
// every warp its output offset and the warps write their selections in index
// order: the output comes out ascending without a sort.
//
// topk_row is that selection for one row by one CTA of NT threads;
// topk_kernel runs it with one CTA of 512 threads per row of a score matrix:
// pass 1 reads the row from HBM with 16-byte loads four deep per lane, and
// the candidate and output passes read it again, from L2; with 64 KB of
// shared memory per CTA, several rows are in flight per SM (a 1024-thread
// CTA caching the row in 160 KB of shared memory, one per SM, took 40 % more
// time on the 32K-token layer's 6144 rows).  If the candidate list overflows
// (a near-constant row), the remaining digits are resolved by passes over the
// whole row instead.
#pragma once

#include "mcs_common.cuh"

namespace mcs {

constexpr int kTopkThreads = 512;
constexpr int kTopkCandCap = 6144;                 // candidate list entries (bits + index)
constexpr int kTopkRowCacheBytes = 0;             // rows are not kept in shared memory (see above)
constexpr int kTopkFixedSmem = (4096 + 2 * kTopkCandCap) * 4;   // histogram + candidate list
constexpr unsigned kTopkMagnitude = 0x7fffffffu;   // scores are >= 0; the sign bit is ignored

// The statically sized scratch of one row selection.
struct TopkShared {
  int wsum[33];
  int gt_cnt[32], eq_cnt[32], w_take[32], w_base[32];
  unsigned s_bin;
  int s_rank, s_ncand;
};

// exclusive scan of one int per thread over an NT-thread block; *total gets the sum
template <int NT>
__device__ __forceinline__ int topk_block_scan(int v, int *wsum, int *total) {
  constexpr int NW = NT / 32;
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
    const int w = lane < NW ? wsum[lane] : 0;
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
template <int NT>
__device__ __forceinline__ unsigned topk_select_bin(const unsigned *hist, int nb, int &kk, TopkShared &sh) {
  const int per = (nb + NT - 1) / NT;
  const int t = threadIdx.x;
  const int top = nb - 1 - t * per;          // this thread's bins, descending: top .. top-per+1 (>= 0)
  int lsum = 0;
  for (int b = 0; b < per && top - b >= 0; ++b) lsum += static_cast<int>(hist[top - b]);
  int total;
  const int before = topk_block_scan<NT>(lsum, sh.wsum, &total);
  if (lsum > 0 && before < kk && before + lsum >= kk) {
    int acc = before;
    for (int b = 0; b < per && top - b >= 0; ++b) {
      const int c = static_cast<int>(hist[top - b]);
      if (acc + c >= kk) {
        sh.s_bin = static_cast<unsigned>(top - b);
        sh.s_rank = kk - acc;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
  kk = sh.s_rank;
  const unsigned bin = sh.s_bin;
  __syncthreads();
  return bin;
}

// Walk this warp's slice [lo, hi) of the row in index order, VEC keys per lane
// per step and four steps of loads in flight; f(j0, keys, valid) is called by
// every lane of the warp for every step (it may use warp votes).
template <int VEC, class F>
__device__ __forceinline__ void topk_walk(const unsigned *src, bool from_smem, int lo, int hi, F &&f) {
  constexpr int STEP = 32 * VEC;
  const int lane = threadIdx.x & 31;
  for (int b = lo; b < hi; b += 4 * STEP) {
    unsigned x[4][VEC];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j0 = b + u * STEP + VEC * lane;
      if (j0 < hi) {
        if constexpr (VEC == 4) {
          const uint4 *p = reinterpret_cast<const uint4 *>(src + j0);
          const uint4 v = from_smem ? *p : __ldg(p);
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

// The k largest of the row's N scores (row_g: their bit patterns), ties to the
// lower index, written ascending to out[0, k), by the NT threads of the CTA
// (all of them call it).  row_g is read-only for the whole kernel.  hist:
// 2^D1 zeroed bins (D1: the first digit's width).  cand_bits / cand_idx:
// cand_cap entries each.  row_sm: a shared copy of the row (N entries) to
// fill in pass 1 and read later, or nullptr.  Every thread of the CTA must
// reach this call (it synchronises the block).
template <int VEC, int NT, int D1>
__device__ void topk_row(const unsigned *row_g, int N, int k, unsigned *hist, unsigned *cand_bits, int *cand_idx,
                         int cand_cap, unsigned *row_sm, TopkShared &sh, int32_t *out) {
  static_assert(NT % 32 == 0 && NT / 32 <= 32, "whole warps, at most 32");
  constexpr int NW = NT / 32;
  constexpr int D2 = (32 - D1) / 2, D3 = 31 - D1 - D2;   // the two remaining digits
  constexpr int S1 = 31 - D1;                           // shift of the first digit
  constexpr int NB1 = 1 << D1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;

  if (k >= N) {
    for (int j = tid; j < N; j += NT) out[j] = j;
    return;
  }
  constexpr int STEP = 32 * VEC;
  const int span = ((N + NW - 1) / NW + STEP - 1) / STEP * STEP;
  const int lo = min(N, warp * span), hi = min(N, lo + span);
  const bool cached = row_sm != nullptr;
  const unsigned *src = cached ? row_sm : row_g;

  if (tid < 32) sh.gt_cnt[tid] = sh.eq_cnt[tid] = 0;
  if (tid == 0) sh.s_ncand = 0;
  __syncthreads();

  // ---- pass 1 (global): cache the row, count the first digit
  topk_walk<VEC>(row_g, false, lo, hi, [&](int j0, const unsigned *key, bool valid) {
    if (!valid) return;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      if (cached) row_sm[j0 + e] = key[e];
      atomicAdd(&hist[key[e] >> S1], 1u);
    }
  });
  __syncthreads();
  int kk = k;
  const unsigned b1 = topk_select_bin<NT>(hist, NB1, kk, sh);
  for (int i = tid; i < NB1; i += NT) hist[i] = 0;

  // ---- pass 2: per-warp count above the threshold's bin; candidates into the list
  int above = 0;
  topk_walk<VEC>(src, cached, lo, hi, [&](int j0, const unsigned *key, bool valid) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const unsigned d = key[e] >> S1;
      above += (valid && d > b1) ? 1 : 0;
      const bool c = valid && d == b1;
      const unsigned bal = __ballot_sync(0xffffffffu, c);
      if (bal == 0u) continue;
      int base = 0;
      if (lane == 0) base = atomicAdd(&sh.s_ncand, __popc(bal));
      base = __shfl_sync(0xffffffffu, base, 0);
      const int pos = base + __popc(bal & lt);
      if (c && pos < cand_cap) {
        cand_bits[pos] = key[e];
        cand_idx[pos] = j0 + e;
      }
    }
  });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
  if (lane == 0) sh.gt_cnt[warp] = above;
  __syncthreads();
  const int ncand = sh.s_ncand;
  const bool listed = ncand <= cand_cap;

  // ---- passes 3, 4: the second and third digits, over the candidates
  unsigned prefix = b1 << S1, mask = static_cast<unsigned>(NB1 - 1) << S1;
  for (int pass = 0; pass < 2; ++pass) {
    const int shift = pass == 0 ? D3 : 0;
    const int nb = pass == 0 ? (1 << D2) : (1 << D3);
    const unsigned dm = static_cast<unsigned>(nb - 1);
    if (listed) {
      for (int i = tid; i < ncand; i += NT) {
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
    const unsigned bin = topk_select_bin<NT>(hist, nb, kk, sh);
    prefix |= bin << shift;
    mask |= dm << shift;
    for (int i = tid; i < nb; i += NT) hist[i] = 0;
    __syncthreads();   // the next digit's counts start only once every bin is clear
  }
  const unsigned T = prefix;
  const int need_eq = kk;   // keys equal to T to keep: the first need_eq of them in index order

  // ---- per-warp counts of keys above T and equal to T
  if (listed) {
    for (int i = tid; i < ncand; i += NT) {
      const unsigned x = cand_bits[i];
      const int w = cand_idx[i] / span;
      if (x > T) atomicAdd(&sh.gt_cnt[w], 1);
      else if (x == T) atomicAdd(&sh.eq_cnt[w], 1);
    }
  } else {
    int g = 0, q = 0;
    topk_walk<VEC>(src, cached, lo, hi, [&](int, const unsigned *key, bool valid) {
      if (!valid) return;
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        if ((key[e] >> S1) != b1) continue;
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
      sh.gt_cnt[warp] += g;
      sh.eq_cnt[warp] = q;
    }
  }
  __syncthreads();
  if (warp == 0) {
    const int e = lane < NW ? sh.eq_cnt[lane] : 0;
    int x = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    const int take = max(0, min(e, need_eq - (x - e)));
    const int sel = (lane < NW ? sh.gt_cnt[lane] : 0) + take;
    int s = sel;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    sh.w_take[lane] = take;
    sh.w_base[lane] = s - sel;
  }
  __syncthreads();

  // ---- pass 5: each warp writes its selected keys in index order
  const int eq_take = sh.w_take[warp];
  int written = sh.w_base[warp], eq_seen = 0;
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

// One CTA per row of a read-only score matrix.  VEC = 4 needs N % 4 == 0 and
// a 16-byte aligned score array.
template <int VEC>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float *__restrict__ colsum, int N, int k,
                                                            int cache_row, int32_t *__restrict__ kv_idx) {
  // dynamic shared memory: histogram, candidate list, then the row when cache_row
  extern __shared__ __align__(16) unsigned topk_sm[];
  unsigned *hist = topk_sm;
  unsigned *cand_bits = hist + 4096;
  int *cand_idx = reinterpret_cast<int *>(cand_bits + kTopkCandCap);
  unsigned *row_sm = reinterpret_cast<unsigned *>(cand_idx + kTopkCandCap);
  __shared__ TopkShared sh;
  const size_t row = blockIdx.x;
  for (int i = threadIdx.x; i < 4096; i += kTopkThreads) hist[i] = 0;
  topk_row<VEC, kTopkThreads, 12>(reinterpret_cast<const unsigned *>(colsum + row * N), N, k, hist,
                                        cand_bits, cand_idx, kTopkCandCap, cache_row ? row_sm : nullptr, sh,
                                        kv_idx + row * k);
}

}  // namespace mcs
