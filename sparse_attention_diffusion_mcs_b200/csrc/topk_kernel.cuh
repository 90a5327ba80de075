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
// keys whose first digit is at least b1 (the threshold's) go to a shared
// memory candidate list, and the digits are resolved on that list alone.
// Every key with bits > T and the first (k - #greater) keys with bits == T
// are kept, written ascending.
//
// A CTA takes a contiguous run of rows, i.e. adjacent query groups of one
// head, whose score rows are alike (on the 32K-token video layer b1 moves by
// at most one of 4096 bins between adjacent groups).  So the walk that reads
// a row from HBM only lists the keys whose first digit is at least a guess,
// the previous row's b1 less one bin, with no per-key histogram.  If at least
// k keys were listed (and the list did not overflow), the k-th largest key
// and every key above it are on the list, and all three digits are resolved
// there.  Otherwise (the run's first row, or a miss) the first digit is
// counted over the whole row, a further walk lists the keys with first digit
// >= b1, and if even those overflow the list (a near-constant row, a large k)
// the remaining digits are resolved by walks over the whole row.
//
// Output: when no key equal to T has to be dropped, the selected keys are
// marked in a bitmap of the row (in the histogram's memory, N <= 131072), and
// a block scan over the bitmap's word counts gives every thread the output
// offset of its words: ascending without a sort and without walking the row.
// Otherwise each warp owns a contiguous slice of the row, per-warp counts
// above and equal to T give every warp its output offset and its share of the
// ties (the first ones in index order), and the warps walk their slices and
// write their selections in index order.
//
// topk_row is that selection for one row by one CTA of NT threads;
// topk_kernel runs it with 512-thread CTAs, three per SM (64 KB of shared
// memory each), each over a contiguous run of rows.  On the 32K-token video
// layer (6144 rows of 32,760 scores) DRAM runs at about a quarter of its peak
// while the SMs issue about 2.8 instructions per cycle of 4: the pace is set
// by each row's chain of walk and barrier-separated candidate phases, of
// which three CTAs per SM overlap only three.
#pragma once

#include "mcs_common.cuh"

namespace mcs {

constexpr int kTopkThreads = 512;
constexpr int kTopkCtasPerSm = 3;
constexpr int kTopkCandCap = 6144;                 // candidate list entries (bits + index)
constexpr int kTopkHistWords = 4096;               // first-digit histogram, later the output bitmap
constexpr int kTopkSmem = (kTopkHistWords + 2 * kTopkCandCap) * 4;   // histogram + candidate list
constexpr unsigned kTopkGuessMargin = 1;           // bins below the previous row's b1 listed in pass 1
constexpr unsigned kTopkMagnitude = 0x7fffffffu;   // scores are >= 0; the sign bit is ignored

// The statically sized scratch of one row selection.
struct TopkShared {
  int wsum[33];
  int gt_cnt[32], eq_cnt[32], w_take[32], w_base[32];
  unsigned s_bin;
  int s_rank, s_ncand, s_eq;
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
__device__ __forceinline__ void topk_walk(const unsigned *src, int lo, int hi, F &&f) {
  constexpr int STEP = 32 * VEC;
  const int lane = threadIdx.x & 31;
  for (int b = lo; b < hi; b += 4 * STEP) {
    unsigned x[4][VEC];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j0 = b + u * STEP + VEC * lane;
      if (j0 < hi) {
        if constexpr (VEC == 4) {
          const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src + j0));
          x[u][0] = v.x;
          x[u][1] = v.y;
          x[u][2] = v.z;
          x[u][3] = v.w;
        } else {
          x[u][0] = __ldg(src + j0);
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

// List the keys of this warp's slice [lo, hi) whose magnitude bits are >= thr
// (bits and index) on the candidate list; entries past cap are counted but
// not stored.  Per lane, 4 steps of VEC keys are loaded at once; the lane
// counts its candidates among them, and one warp scan of those counts plus
// one shared-memory atomic per warp give every lane its list positions (the
// list's order is free: the selection is sorted by the output bitmap or by
// the per-warp walk).
template <int VEC>
__device__ __forceinline__ void topk_list_walk(const unsigned *src, int lo, int hi, unsigned thr, unsigned *cand_bits,
                                               int *cand_idx, int cap, int *ncand) {
  constexpr int STEP = 32 * VEC;
  const int lane = threadIdx.x & 31;
  for (int b = lo; b < hi; b += 4 * STEP) {
    unsigned x[4][VEC];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j0 = b + u * STEP + VEC * lane;
      if (j0 < hi) {
        if constexpr (VEC == 4) {
          const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src + j0));
          x[u][0] = v.x;
          x[u][1] = v.y;
          x[u][2] = v.z;
          x[u][3] = v.w;
        } else {
          x[u][0] = __ldg(src + j0);
        }
      } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) x[u][e] = 0u;
      }
    }
    // sel bit (u * VEC + e): key x[u][e] is in the slice and listed
    unsigned sel = 0u;
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        x[u][e] &= kTopkMagnitude;
        const bool in = b + u * STEP + VEC * lane + e < hi;
        sel |= (in && x[u][e] >= thr) ? 1u << (u * VEC + e) : 0u;
      }
    const int m = __popc(sel);
    int incl = m;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (total > 0) {   // warp-uniform
      int base = 0;
      if (lane == 31) base = atomicAdd(ncand, total);
      int pos = __shfl_sync(0xffffffffu, base, 31) + incl - m;
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          if ((sel >> (u * VEC + e)) & 1u) {
            if (pos < cap) {
              cand_bits[pos] = x[u][e];
              cand_idx[pos] = b + u * STEP + VEC * lane + e;
            }
            ++pos;
          }
        }
    }
  }
}

// The k largest of the row's N scores (row_g: their bit patterns), ties to the
// lower index, written ascending to out[0, k), by the NT threads of the CTA
// (all of them call it; it synchronises the block).  row_g is read-only for
// the whole kernel.  hist: kTopkHistWords zeroed words (left zeroed on
// return).  cand_bits / cand_idx: cand_cap entries each.  guess: pass 1 lists
// the keys whose first digit is >= guess (1 << D1 or more: no guess, the
// first digit is counted over the row).  Returns the first digit of the
// row's threshold (the next row's guess is derived from it), or 1 << D1 when
// every key is kept.
template <int VEC, int NT, int D1>
__device__ unsigned topk_row(const unsigned *row_g, int N, int k, unsigned *hist, unsigned *cand_bits, int *cand_idx,
                             int cand_cap, unsigned guess, TopkShared &sh, int32_t *out) {
  static_assert(NT % 32 == 0 && NT / 32 <= 32, "whole warps, at most 32");
  constexpr int NW = NT / 32;
  constexpr int D2 = (32 - D1) / 2, D3 = 31 - D1 - D2;   // the two remaining digits
  constexpr int S1 = 31 - D1;                           // shift of the first digit
  constexpr int NB1 = 1 << D1;
  static_assert(NB1 <= kTopkHistWords && (1 << D2) <= kTopkHistWords, "digits fit the histogram");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (k >= N) {
    for (int j = tid; j < N; j += NT) out[j] = j;
    return static_cast<unsigned>(NB1);
  }
  constexpr int STEP = 32 * VEC;
  const int span = ((N + NW - 1) / NW + STEP - 1) / STEP * STEP;
  const int lo = min(N, warp * span), hi = min(N, lo + span);

  if (tid < 32) sh.gt_cnt[tid] = sh.eq_cnt[tid] = 0;
  if (tid == 0) {
    sh.s_ncand = 0;
    sh.s_eq = 0;
  }
  __syncthreads();

  int kk = k;
  unsigned b1 = 0;
  bool listed = false;
  if (guess < static_cast<unsigned>(NB1)) {
    // ---- pass 1 (HBM): list the keys whose first digit is >= guess
    topk_list_walk<VEC>(row_g, lo, hi, guess << S1, cand_bits, cand_idx, cand_cap, &sh.s_ncand);
    __syncthreads();
    const int n1 = sh.s_ncand;
    // at least k keys listed: the k-th largest is among them, and so is every
    // key at or above it; the first digit is then counted over the list alone
    listed = n1 >= k && n1 <= cand_cap;
    if (listed) {
      for (int i = tid; i < n1; i += NT) atomicAdd(&hist[cand_bits[i] >> S1], 1u);
      __syncthreads();
      b1 = topk_select_bin<NT>(hist, NB1, kk, sh);
      for (int i = static_cast<int>(guess) + tid; i < NB1; i += NT) hist[i] = 0;
      __syncthreads();
    }
  }
  if (!listed) {
    // ---- no guess, or it missed: count the first digit over the row (from
    // HBM, or from L2 after a pass 1), then list the keys with first digit >= b1
    topk_walk<VEC>(row_g, lo, hi, [&](int, const unsigned *key, bool valid) {
      if (!valid) return;
#pragma unroll
      for (int e = 0; e < VEC; ++e) atomicAdd(&hist[key[e] >> S1], 1u);
    });
    __syncthreads();
    b1 = topk_select_bin<NT>(hist, NB1, kk, sh);
    const int in_bin = static_cast<int>(hist[b1]);
    const int n_above = k - kk;             // keys whose first digit is above b1
    __syncthreads();                        // every thread has read hist[b1]
    for (int i = tid; i < NB1; i += NT) hist[i] = 0;
    const bool relist = n_above + in_bin <= cand_cap;
    if (relist && tid == 0) sh.s_ncand = 0;
    __syncthreads();                        // histogram clear and list reset seen by all
    if (relist) {
      topk_list_walk<VEC>(row_g, lo, hi, b1 << S1, cand_bits, cand_idx, cand_cap, &sh.s_ncand);
      __syncthreads();
      listed = true;
    }
  }
  const int ncand = listed ? sh.s_ncand : 0;

  // ---- passes 3, 4: the second and third digits, over the candidates (or the row)
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
      topk_walk<VEC>(row_g, lo, hi, [&](int, const unsigned *key, bool valid) {
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

  // ---- keys equal to T: if all of them are kept, mark the selection in a bitmap
  const int W = (N + 31) / 32;
  if (listed) {
    int q = 0;
    for (int i = tid; i < ncand; i += NT) q += cand_bits[i] == T ? 1 : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    if (lane == 0 && q > 0) atomicAdd(&sh.s_eq, q);
    __syncthreads();
  }
  if (listed && sh.s_eq == need_eq && W <= kTopkHistWords) {
    for (int i = tid; i < ncand; i += NT)
      if (cand_bits[i] >= T) atomicOr(&hist[cand_idx[i] >> 5], 1u << (cand_idx[i] & 31));
    __syncthreads();
    const int per = (W + NT - 1) / NT;
    const int w0 = min(W, tid * per), w1 = min(W, w0 + per);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(hist[w]);
    int total;
    int pos = topk_block_scan<NT>(cnt, sh.wsum, &total);
    for (int w = w0; w < w1; ++w) {
      unsigned bits = hist[w];
      while (bits != 0u) {
        const int b = __ffs(bits) - 1;
        if (pos < k) out[pos] = w * 32 + b;
        ++pos;
        bits &= bits - 1u;
      }
    }
    __syncthreads();   // every word read before the bitmap is cleared
    for (int i = tid; i < W; i += NT) hist[i] = 0;
    return b1;
  }

  // ---- otherwise per-warp counts of keys above T and equal to T
  if (listed) {
    for (int i = tid; i < ncand; i += NT) {
      const unsigned x = cand_bits[i];
      const int w = cand_idx[i] / span;
      if (x > T) atomicAdd(&sh.gt_cnt[w], 1);
      else if (x == T) atomicAdd(&sh.eq_cnt[w], 1);
    }
  } else {
    int g = 0, q = 0;
    topk_walk<VEC>(row_g, lo, hi, [&](int, const unsigned *key, bool valid) {
      if (!valid) return;
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
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
      sh.gt_cnt[warp] = g;
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

  // ---- each warp writes its selected keys in index order
  const unsigned lt = (1u << lane) - 1u;
  const int eq_take = sh.w_take[warp];
  int written = sh.w_base[warp], eq_seen = 0;
  topk_walk<VEC>(row_g, lo, hi, [&](int j0, const unsigned *key, bool valid) {
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
  return b1;
}

// Rows [r0, r1) of a read-only score matrix per CTA, a contiguous run so
// that each row's guess comes from its neighbour.  VEC = 4 needs N % 4 == 0
// and a 16-byte aligned score array.
template <int VEC>
__global__ void __launch_bounds__(kTopkThreads, kTopkCtasPerSm)
    topk_kernel(const float *__restrict__ colsum, long long rows, int N, int k, int32_t *__restrict__ kv_idx) {
  // dynamic shared memory: histogram (later the output bitmap), candidate list
  extern __shared__ __align__(16) unsigned topk_sm[];
  unsigned *hist = topk_sm;
  unsigned *cand_bits = hist + kTopkHistWords;
  int *cand_idx = reinterpret_cast<int *>(cand_bits + kTopkCandCap);
  __shared__ TopkShared sh;
  for (int i = threadIdx.x; i < kTopkHistWords; i += kTopkThreads) hist[i] = 0;
  const long long r0 = rows * blockIdx.x / gridDim.x, r1 = rows * (blockIdx.x + 1) / gridDim.x;
  unsigned guess = 1u << 12;   // the first row lists nothing in pass 1
  for (long long r = r0; r < r1; ++r) {
    const unsigned b1 = topk_row<VEC, kTopkThreads, 12>(reinterpret_cast<const unsigned *>(colsum + r * N), N, k,
                                                        hist, cand_bits, cand_idx, kTopkCandCap, guess, sh,
                                                        kv_idx + r * k);
    guess = b1 > kTopkGuessMargin ? b1 - kTopkGuessMargin : 0u;
  }
}

}  // namespace mcs
