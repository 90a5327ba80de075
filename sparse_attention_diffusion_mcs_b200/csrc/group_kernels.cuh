// group_kernels.cuh -- tile-aligned grouping of similar queries, step a1.
//
// "organizing similar queries into tile-aligned groups for efficient GPU
// execution" (aiqbench.com abstract; cctest.ai "Hardware-aware query
// organization").  The pages do not say how similarity is measured; this
// library orders each head's queries by their projection on the first
// principal direction of Q and cuts the order into contiguous runs of G.
//
// Everything runs in fp64 (bf16 inputs are exact in fp64), so the order is
// the order of the exact projections up to fp64 rounding:
//   mean_kernel       per (head, chunk of rows): column sums of Q
//   cov_kernel        per (head, chunk): sum of (q - mu)(q - mu)^T
//   cov_reduce_kernel per head: C = sum of the chunk partials / N
//   eig_kernel        per head: top eigenvector of C by repeated
//                     squaring + power iteration, sign fixed so the
//                     largest-magnitude component is positive
//   project_kernel    p_n = (q_n - mu) . v  -> order-preserving uint64 key
//   sort_hist_kernel, sort_scatter_kernel
//                     per head, over several CTAs: stable LSD radix sort of
//                     (key, n) -> perm
#pragma once

#include "mcs_common.cuh"

namespace mcs {

constexpr int kGroupChunk = 1024;     // rows per chunk of the mean / covariance passes
constexpr int kSortThreads = 1024;

// ---------------------------------------------------------------- mean
template <int D>
__global__ void __launch_bounds__(256) mean_kernel(const bf16 *__restrict__ Q, int N, int n_chunks,
                                                   double *__restrict__ part) {
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int r0 = chunk * kGroupChunk;
  const int r1 = min(N, r0 + kGroupChunk);
  constexpr int RSTEP = 256 / D;
  const int col = threadIdx.x % D;
  const int rr = threadIdx.x / D;
  const bf16 *q = Q + static_cast<size_t>(bh) * N * D;
  double acc = 0.0;
  for (int r = r0 + rr; r < r1; r += RSTEP) acc += __bfloat162float(q[static_cast<size_t>(r) * D + col]);
  __shared__ double red[256];
  red[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x < D) {
    double sum = 0.0;
    for (int i = 0; i < RSTEP; ++i) sum += red[i * D + threadIdx.x];
    part[(static_cast<size_t>(bh) * n_chunks + chunk) * D + threadIdx.x] = sum;
  }
}

template <int D>
__global__ void mean_finalize_kernel(const double *__restrict__ part, int N, int n_chunks,
                                     double *__restrict__ mean) {
  const int bh = blockIdx.x, c = threadIdx.x;
  if (c >= D) return;
  double sum = 0.0;
  for (int i = 0; i < n_chunks; ++i) sum += part[(static_cast<size_t>(bh) * n_chunks + i) * D + c];
  mean[bh * D + c] = sum / N;
}

// ---------------------------------------------------------------- covariance
// 256 threads as a 16 x 16 grid; thread (ti, tj) accumulates C[ti + 16a][tj + 16b]
// in fp64 registers (columns interleaved so the shared memory reads of one
// warp hit distinct banks) for the block pairs a <= b < R = D/16 only, and
// writes each a < b entry twice, at (i, j) and at its mirror (j, i): the
// mirror would be the same sequence of fma(x_i, x_j, .) in the same row order
// (the product commutes), so the partial matrices are exactly symmetric and
// the lower block triangle (R(R-1)/2 of the R^2 block pairs) is not computed.
// Rows are centred and staged through a double-buffered shared tile, the next
// tile's 16-byte loads in flight while the current one is consumed.
template <int D>
__global__ void __launch_bounds__(256) cov_kernel(const bf16 *__restrict__ Q, const double *__restrict__ mean,
                                                  int N, int n_chunks, double *__restrict__ part) {
  constexpr int R = D / 16;
  constexpr int ROWS = 16;
  constexpr int VPR = D / 8;             // 16-byte vectors per row
  constexpr int NV = ROWS * VPR;         // vectors per staged tile (<= 256)
  __shared__ double xs[2][ROWS][D];
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int r0 = chunk * kGroupChunk;
  const int r1 = min(N, r0 + kGroupChunk);
  const int tid = threadIdx.x, ti = tid / 16, tj = tid % 16;
  const bf16 *q = Q + static_cast<size_t>(bh) * N * D;
  const double *mu = mean + bh * D;
  const bool stager = tid < NV;
  const int srow = tid / VPR, scol = (tid % VPR) * 8;
  double mus[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) mus[e] = stager ? mu[scol + e] : 0.0;
  auto fetch = [&](int rb) -> uint4 {
    const int r = rb + srow;
    if (stager && r < r1) return __ldg(reinterpret_cast<const uint4 *>(q + static_cast<size_t>(r) * D + scol));
    return make_uint4(0u, 0u, 0u, 0u);
  };
  auto stage = [&](int buf, int rb, uint4 v) {
    if (!stager) return;
    const bool live = rb + srow < r1;
    const bf16 *h = reinterpret_cast<const bf16 *>(&v);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      xs[buf][srow][scol + e] = live ? static_cast<double>(__bfloat162float(h[e])) - mus[e] : 0.0;
  };
  double acc[R][R];   // only a <= b is used
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = a; b < R; ++b) acc[a][b] = 0.0;
  int buf = 0;
  stage(0, r0, fetch(r0));
  __syncthreads();
  for (int rb = r0; rb < r1; rb += ROWS) {
    const bool more = rb + ROWS < r1;
    const uint4 nxt = more ? fetch(rb + ROWS) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 4
    for (int rr = 0; rr < ROWS; ++rr) {
      double xi[R], xj[R];
#pragma unroll
      for (int a = 0; a < R; ++a) {
        xi[a] = xs[buf][rr][ti + 16 * a];
        xj[a] = xs[buf][rr][tj + 16 * a];
      }
#pragma unroll
      for (int a = 0; a < R; ++a)
#pragma unroll
        for (int b = a; b < R; ++b) acc[a][b] = fma(xi[a], xj[b], acc[a][b]);
    }
    if (more) stage(buf ^ 1, rb + ROWS, nxt);
    __syncthreads();
    buf ^= 1;
  }
  double *out = part + (static_cast<size_t>(bh) * n_chunks + chunk) * D * D;
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = a; b < R; ++b) {
      out[(ti + 16 * a) * D + tj + 16 * b] = acc[a][b];
      if (b > a) out[(tj + 16 * b) * D + ti + 16 * a] = acc[a][b];
    }
}

// C = (sum of the chunk partials, in chunk order) / N; one thread per entry.
template <int D>
__global__ void __launch_bounds__(256) cov_reduce_kernel(const double *__restrict__ part, int N, int n_chunks,
                                                         double *__restrict__ cov) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * 256 + threadIdx.x;
  if (e >= D * D) return;
  const double *p = part + static_cast<size_t>(bh) * n_chunks * D * D + e;
  double sum = 0.0;
  for (int i = 0; i < n_chunks; ++i) sum += p[static_cast<size_t>(i) * D * D];
  cov[static_cast<size_t>(bh) * D * D + e] = sum / N;
}

// ---------------------------------------------------------------- eigenvector
// One CTA of 256 threads per head.  M, a normalised power of C obtained by
// repeated squaring, lives in shared memory; squaring separates the top
// eigenvector even for small spectral gaps.  A few power iterations with M
// and then with C itself (copied into the same shared buffer) give v.
// M stays exactly symmetric (T[i][j] and T[j][i] are the same fma sequence),
// so T = M.M is formed as sum_t M[t][i] M[t][j]: both operands are read from
// row t, and thread (ti, tj) keeps its blocks a <= b of T in registers and
// writes each a < b entry also at its mirror (as the covariance does).
template <int D>
__global__ void __launch_bounds__(256) eig_kernel(const double *__restrict__ cov, double *__restrict__ vdir,
                                                  float *__restrict__ lambda) {
  constexpr int R = D / 16;
  extern __shared__ double dsm[];
  double *M = dsm;               // D*D
  double *vec = M + D * D;       // D
  double *tmp = vec + D;         // 2*D
  __shared__ double red[256];
  const int bh = blockIdx.x, tid = threadIdx.x, ti = tid / 16, tj = tid % 16;
  const double *Cm = cov + static_cast<size_t>(bh) * D * D;

  auto block_sum = [&](double x) -> double {
    red[tid] = x;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
      if (tid < o) red[tid] += red[tid + o];
      __syncthreads();
    }
    const double r = red[0];
    __syncthreads();
    return r;
  };

  const double tr = block_sum(tid < D ? Cm[tid * D + tid] : 0.0);
  if (!(tr > 0.0)) {   // all queries identical: every direction is principal; take e_0
    if (tid < D) vdir[bh * D + tid] = tid == 0 ? 1.0 : 0.0;
    if (tid == 0) lambda[bh] = 0.f;
    return;
  }
  for (int e = tid; e < D * D; e += 256) M[e] = Cm[e] / tr;
  __syncthreads();
  for (int sq = 0; sq < 10; ++sq) {        // M <- M^2 / trace(M^2)  ->  C^(2^10), normalised
    double acc[R][R];   // only a <= b is used
#pragma unroll
    for (int a = 0; a < R; ++a)
#pragma unroll
      for (int b = a; b < R; ++b) acc[a][b] = 0.0;
#pragma unroll 2
    for (int t = 0; t < D; ++t) {
      double xi[R], xj[R];
#pragma unroll
      for (int a = 0; a < R; ++a) {
        xi[a] = M[t * D + ti + 16 * a];
        xj[a] = M[t * D + tj + 16 * a];
      }
#pragma unroll
      for (int a = 0; a < R; ++a)
#pragma unroll
        for (int b = a; b < R; ++b) acc[a][b] = fma(xi[a], xj[b], acc[a][b]);
    }
    double dsum = 0.0;
    if (ti == tj)
#pragma unroll
      for (int a = 0; a < R; ++a) dsum += acc[a][a];
    const double t2 = block_sum(dsum);     // its barriers also end every read of M
#pragma unroll
    for (int a = 0; a < R; ++a)
#pragma unroll
      for (int b = a; b < R; ++b) {
        const double x = acc[a][b] / t2;
        M[(ti + 16 * a) * D + tj + 16 * b] = x;
        if (b > a) M[(tj + 16 * b) * D + ti + 16 * a] = x;
      }
    __syncthreads();
  }
  // start from the column of M with the largest diagonal entry
  if (tid == 0) {
    int best = 0;
    for (int i = 1; i < D; ++i)
      if (M[i * D + i] > M[best * D + best]) best = i;
    red[0] = best;
  }
  __syncthreads();
  const int best = static_cast<int>(red[0]);
  __syncthreads();
  if (tid < D) vec[tid] = M[tid * D + best];
  __syncthreads();
  // y = A v for the symmetric A in shared memory: y_i = sum_t A[t][i] v_t, the
  // two halves of t on two threads, then normalise
  auto matvec_norm = [&]() {
    const int i = tid % D, h = tid / D;
    if (h < 2) {
      double a0 = 0.0, a1 = 0.0;
      const int t0 = h * (D / 2);
      for (int t = t0; t < t0 + D / 2; t += 2) {
        a0 = fma(M[t * D + i], vec[t], a0);
        a1 = fma(M[(t + 1) * D + i], vec[t + 1], a1);
      }
      tmp[h * D + i] = a0 + a1;
    }
    __syncthreads();
    const double y = tid < D ? tmp[tid] + tmp[D + tid] : 0.0;
    const double nn = block_sum(y * y);
    const double inv = nn > 0.0 ? 1.0 / sqrt(nn) : 0.0;
    if (tid < D) vec[tid] = y * inv;
    __syncthreads();
  };
  for (int it = 0; it < 8; ++it) matvec_norm();
  for (int e = tid; e < D * D; e += 256) M[e] = Cm[e];
  __syncthreads();
  for (int it = 0; it < 64; ++it) matvec_norm();
  // sign: the first component of largest magnitude is positive
  if (tid == 0) {
    int im = 0;
    for (int i = 1; i < D; ++i)
      if (fabs(vec[i]) > fabs(vec[im])) im = i;
    red[0] = vec[im] < 0.0 ? -1.0 : 1.0;
  }
  __syncthreads();
  const double sg = red[0];
  __syncthreads();
  // Rayleigh quotient v.C.v for the eigenvalue
  if (tid < D) {
    double acc = 0.0;
    for (int t = 0; t < D; ++t) acc = fma(M[t * D + tid], vec[t], acc);
    tmp[tid] = acc * vec[tid];
  }
  __syncthreads();
  const double lam = block_sum(tid < D ? tmp[tid] : 0.0);
  if (tid < D) vdir[bh * D + tid] = sg * vec[tid];
  if (tid == 0) lambda[bh] = static_cast<float>(lam);
}

// ---------------------------------------------------------------- projection
__device__ __forceinline__ unsigned long long double_order_key(double f) {
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(f));
  return (b & 0x8000000000000000ull) ? ~b : (b | 0x8000000000000000ull);
}

template <int D>
__global__ void __launch_bounds__(256) project_kernel(const bf16 *__restrict__ Q, const double *__restrict__ mean,
                                                      const double *__restrict__ vdir, int N,
                                                      unsigned long long *__restrict__ keys,
                                                      int32_t *__restrict__ vals) {
  // one warp per row; lanes split the columns
  const int bh = blockIdx.y;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const bf16 *q = Q + (static_cast<size_t>(bh) * N + row) * D;
  const double *mu = mean + bh * D;
  const double *v = vdir + bh * D;
  double acc = 0.0;
  for (int c = lane; c < D; c += 32) acc = fma(static_cast<double>(__bfloat162float(q[c])) - mu[c], v[c], acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    keys[static_cast<size_t>(bh) * N + row] = double_order_key(acc);
    vals[static_cast<size_t>(bh) * N + row] = row;
  }
}

// ---------------------------------------------------------------- stable LSD radix sort
// 8 passes of 8 bits over 64-bit keys.  A head's array is cut into `parts`
// contiguous chunks of whole 1024-key tiles, one CTA each, so a head's sort
// runs on several SMs.  Per pass, sort_hist_kernel counts each chunk's digits
// and sort_scatter_kernel places each chunk's keys from base[digit] = (the
// head's keys of smaller digits) + (keys of this digit in earlier chunks),
// scattering its tiles in index order and ranking equal digits inside a tile
// by (warp, lane): stable, exactly the order one CTA per head would give.
__global__ void __launch_bounds__(kSortThreads) sort_hist_kernel(const unsigned long long *__restrict__ keys, int N,
                                                                 int chunk, int shift, unsigned *__restrict__ ghist) {
  __shared__ unsigned bins[256];
  const int part = blockIdx.x, bh = blockIdx.y, parts = gridDim.x;
  for (int i = threadIdx.x; i < 256; i += kSortThreads) bins[i] = 0;
  __syncthreads();
  const unsigned long long *k = keys + static_cast<size_t>(bh) * N;
  const int j0 = part * chunk, j1 = min(N, j0 + chunk);
  for (int j = j0 + static_cast<int>(threadIdx.x); j < j1; j += kSortThreads)
    atomicAdd(&bins[static_cast<unsigned>(k[j] >> shift) & 255u], 1u);
  __syncthreads();
  for (int i = threadIdx.x; i < 256; i += kSortThreads) ghist[(static_cast<size_t>(bh) * parts + part) * 256 + i] = bins[i];
}

// vout_head: the pass's value output for this head (the next pass's input, or
// the final perm row)
__global__ void __launch_bounds__(kSortThreads) sort_scatter_kernel(const unsigned long long *__restrict__ kin,
                                                                    const int32_t *__restrict__ vin,
                                                                    unsigned long long *__restrict__ kout,
                                                                    int32_t *__restrict__ vout, int N, int chunk,
                                                                    int shift, const unsigned *__restrict__ ghist) {
  __shared__ unsigned base[256];
  __shared__ unsigned tile_tot[256];
  __shared__ unsigned short wcnt[32][256];   // per-warp digit counts, then exclusive prefixes
  const int part = blockIdx.x, bh = blockIdx.y, parts = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;
  if (warp == 0) {   // lane l owns digits 8l .. 8l+7
    unsigned tot[8], before[8], sum = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int d = lane * 8 + b;
      unsigned t = 0, e = 0;
      for (int pp = 0; pp < parts; ++pp) {
        const unsigned x = ghist[(static_cast<size_t>(bh) * parts + pp) * 256 + d];
        t += x;
        e += pp < part ? x : 0u;
      }
      tot[b] = t;
      before[b] = e;
      sum += t;
    }
    unsigned inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    unsigned run = inc - sum;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      base[lane * 8 + b] = run + before[b];
      run += tot[b];
    }
  }
  __syncthreads();
  const unsigned long long *ki = kin + static_cast<size_t>(bh) * N;
  const int32_t *vi = vin + static_cast<size_t>(bh) * N;
  unsigned long long *ko = kout + static_cast<size_t>(bh) * N;
  int32_t *vo = vout + static_cast<size_t>(bh) * N;
  const int j0 = part * chunk, j1 = min(N, j0 + chunk);
  for (int t0 = j0; t0 < j1; t0 += kSortThreads) {
    const int j = t0 + tid;
    const bool valid = j < j1;
    unsigned long long key = 0;
    int32_t val = 0;
    if (valid) {
      key = ki[j];
      val = vi[j];
    }
    const unsigned digit = valid ? (static_cast<unsigned>(key >> shift) & 255u) : 256u;
    for (int b = lane; b < 256; b += 32) wcnt[warp][b] = 0;
    __syncwarp();
    const unsigned peers = __match_any_sync(0xffffffffu, digit);
    const unsigned rank_in_warp = __popc(peers & lt_mask);
    if (valid && rank_in_warp == 0) wcnt[warp][digit] = static_cast<unsigned short>(__popc(peers));
    __syncthreads();
    if (tid < 256) {
      unsigned run = 0;
      for (int w = 0; w < 32; ++w) {
        const unsigned cnt = wcnt[w][tid];
        wcnt[w][tid] = static_cast<unsigned short>(run);
        run += cnt;
      }
      tile_tot[tid] = run;
    }
    __syncthreads();
    if (valid) {
      const unsigned pos = base[digit] + wcnt[warp][digit] + rank_in_warp;
      ko[pos] = key;
      vo[pos] = val;
    }
    __syncthreads();
    if (tid < 256) base[tid] += tile_tot[tid];
    __syncthreads();
  }
}

// chunks per head: about two CTAs per SM of a 148-SM B200 in all (a fixed
// figure, so the workspace size does not depend on the device), whole tiles,
// at most 64
constexpr int kSortSms = 148;
inline int sort_parts(int BH, int N, int sms = kSortSms) {
  const int tiles = (N + kSortThreads - 1) / kSortThreads;
  int parts = BH > 0 ? (2 * sms) / BH : 1;
  parts = parts < 1 ? 1 : (parts > 64 ? 64 : parts);
  if (parts > tiles) parts = tiles > 0 ? tiles : 1;
  const int chunk = ((tiles + parts - 1) / parts) * kSortThreads;
  return N > 0 ? (N + chunk - 1) / chunk : 1;
}
inline int sort_chunk(int N, int parts) {
  const int tiles = (N + kSortThreads - 1) / kSortThreads;
  return ((tiles + parts - 1) / parts) * kSortThreads;
}

}  // namespace mcs
