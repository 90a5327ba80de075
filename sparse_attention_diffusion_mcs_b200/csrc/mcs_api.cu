// mcs_api.cu -- host side of the C ABI declared in include/mcs.h: argument
// checks, workspace carving and kernel launches on the caller's stream.
#include <cudaTypedefs.h>

#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "../../include/mcs.h"
#include "ablation_kernels.cuh"
#include "attn_dual_kernel.cuh"
#include "attn_kernel.cuh"
#include "colsum_kernel.cuh"
#include "group_kernels.cuh"
#include "pair_kernel.cuh"
#include "residual_compact.cuh"
#include "topk_kernel.cuh"
#include "validate_kernels.cuh"

using namespace mcs;

namespace {

__device__ unsigned g_status_word;

constexpr int kMaxDevices = 64;
uint64_t g_wait_ns = 4000000000ull;
std::mutex g_mu;
unsigned *g_status_ptr[kMaxDevices];

unsigned *status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<unsigned *>(p);
  }
  return g_status_ptr[dev];
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool shape_ok(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1) return false;
  if (static_cast<long long>(B) * H > 65535) return false;
  if (N > (1 << 24)) return false;
  if (static_cast<long long>(B) * H * N >= (1ll << 31)) return false;   // TMA row coordinates are int32
  (void)d;
  return true;
}
bool d_ok(int d) { return d == 64 || d == 128; }
bool g_ok(int G) { return G == 64 || G == 128; }

// ---------------------------------------------------------------- TMA tensor maps
// cuTensorMapEncodeTiled is fetched through the runtime's driver entry point,
// so the library does not link the driver and still loads on hosts without it.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// rows x D bf16 rows, box of 64 columns (128 bytes) x box_rows rows; one
// row: the tile::gather4 source, 64 rows: contiguous key tiles
bool map_rows(CUtensorMap *m, const void *base, int D, size_t rows, unsigned box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map_gather(CUtensorMap *m, const void *base, int D, size_t rows) { return map_rows(m, base, D, rows, 1); }

// [BH, N, D] bf16, box of 128 rows x 64 columns of one head: rows past N read as zero
bool map_tile(CUtensorMap *m, const void *base, int D, int N, int BH) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(N) * D * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// SMs of the current device
cudaError_t sm_count(int *n) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  return cudaDeviceGetAttribute(n, cudaDevAttrMultiProcessorCount, dev);
}

template <typename F>
cudaError_t set_smem(F *fn, int bytes) {
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// ---------------------------------------------------------------- attention launches
struct QKV {
  const void *Q, *K, *V;
};

template <int D, int MODE>
cudaError_t launch_attn(AttnArgs &a, const QKV &t, int grid_x, int BH, cudaStream_t s) {
  a.BH = BH;
  const long items = static_cast<long>(grid_x) * BH;
  cudaError_t e;
  if constexpr (!is_sparse_mode(MODE)) {
    // Dense modes (long items, small epilogues): one CTA per (head, query
    // tile), two softmax warpgroups taking alternate key tiles.
    using C = DualCfg<D, MODE>;
    static_assert(C::SMEM <= 232448, "shared memory budget");
    if (!(map_tile(&a.tmQ, t.Q, D, a.N, BH) && map_tile(&a.tmK, t.K, D, a.N, BH) && map_tile(&a.tmV, t.V, D, a.N, BH)))
      return cudaErrorInvalidValue;
    if (items == 0) return cudaSuccess;
    if ((e = set_smem(attn_dual_kernel<D, MODE>, C::SMEM)) != cudaSuccess) return e;
    attn_dual_kernel<D, MODE><<<static_cast<unsigned>(items), C::THREADS, C::SMEM, s>>>(a);
  } else {
    // Sparse modes run persistent, one CTA per SM (the kernel takes all of an
    // SM's shared memory and TMEM) looping over (head, group) items, so each
    // item's gathers and first Q.K^T overlap the previous item's epilogue.
    using C = AttnCfg<D, MODE>;
    static_assert(C::SMEM <= 232448, "shared memory budget");
    const size_t rows = static_cast<size_t>(BH) * a.N;
    if (!(map_gather(&a.tmQ, t.Q, D, rows) && map_gather(&a.tmK, t.K, D, rows) && map_gather(&a.tmV, t.V, D, rows)))
      return cudaErrorInvalidValue;
    if (items == 0) return cudaSuccess;
    if ((e = set_smem(attn_kernel<D, MODE>, C::SMEM)) != cudaSuccess) return e;
    int sms = 0;
    if ((e = sm_count(&sms)) != cudaSuccess) return e;
    const long grid = items < sms ? items : sms;
    attn_kernel<D, MODE><<<static_cast<unsigned>(grid), C::THREADS, C::SMEM, s>>>(a);
  }
  return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_attn_d(int d, AttnArgs &a, const QKV &t, int grid_x, int BH, cudaStream_t s) {
  return d == 64 ? launch_attn<64, MODE>(a, t, grid_x, BH, s) : launch_attn<128, MODE>(a, t, grid_x, BH, s);
}

// The sparse modes over pairs of groups sharing one union list of keys
// (pair_kernel.cuh): persistent, one CTA per SM, items (head, pair).  With
// BLOCK the lists hold block indices and K/V tiles are contiguous 64-row boxes.
template <int D, int MODE, int BLOCK = 0>
cudaError_t launch_pair(AttnArgs &a, const QKV &t, int BH, cudaStream_t s) {
  using C = PairCfg<D>;
  a.BH = BH;
  const size_t rows = static_cast<size_t>(BH) * a.N;
  const unsigned kv_box = BLOCK ? C::BN : 1;
  if (!(map_gather(&a.tmQ, t.Q, D, rows) && map_rows(&a.tmK, t.K, D, rows, kv_box) &&
        map_rows(&a.tmV, t.V, D, rows, kv_box)))
    return cudaErrorInvalidValue;
  const long items = static_cast<long>(BH) * a.n_pairs;
  if (items == 0) return cudaSuccess;
  cudaError_t e;
  if ((e = set_smem(pair_kernel<D, MODE, BLOCK>, C::SMEM)) != cudaSuccess) return e;
  int sms = 0;
  if ((e = sm_count(&sms)) != cudaSuccess) return e;
  const long grid = items < sms ? items : sms;
  pair_kernel<D, MODE, BLOCK><<<static_cast<unsigned>(grid), C::THREADS, C::SMEM, s>>>(a);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_pair_d(int d, AttnArgs &a, const QKV &t, int BH, cudaStream_t s) {
  return d == 64 ? launch_pair<64, MODE>(a, t, BH, s) : launch_pair<128, MODE>(a, t, BH, s);
}

inline int pairs_of(int n_groups) { return (n_groups + 1) / 2; }

// union lists of group pairs (2p, 2p+1) from the groups' ascending kv lists
cudaError_t run_pairs(const int32_t *kv_idx, int BH, int n_groups, int kk, int32_t *pair_idx,
                      int32_t *pair_len, cudaStream_t s) {
  const int np = pairs_of(n_groups);
  if (np == 0 || BH == 0) return cudaSuccess;
  pair_build_kernel<<<dim3(np, BH), kPairThreads, 0, s>>>(kv_idx, n_groups, kk, np, pair_idx, pair_len);
  return cudaGetLastError();
}

AttnArgs base_args(int N, float scale) {
  AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  a.N = N;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.status = status_ptr();
  a.wait_ns = g_wait_ns;
  return a;
}

// ---------------------------------------------------------------- plan workspace
struct PlanWs {
  size_t mean_part, mean, cov_part, cov64, vdir, lambda, keys0, vals0, keys1, vals1, ghist;
  size_t row_m, row_l, O32, colsum, pair_idx, pair_len, total;
};

PlanWs plan_ws(int B, int H, int N, int d, int G, int k) {
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t nch = (N + kGroupChunk - 1) / kGroupChunk;
  const size_t ng = (N + G - 1) / G;
  PlanWs w;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  w.mean_part = take(BH * nch * d * 8);
  w.mean = take(BH * d * 8);
  w.cov_part = take(BH * nch * d * d * 8);
  w.cov64 = take(BH * d * d * 8);
  w.vdir = take(BH * d * 8);
  w.lambda = take(BH * 4);
  w.keys0 = take(BH * N * 8);
  w.vals0 = take(BH * N * 4);
  w.keys1 = take(BH * N * 8);
  w.vals1 = take(BH * N * 4);
  w.ghist = take(BH * static_cast<size_t>(sort_parts(static_cast<int>(BH), N)) * 256 * 4);
  w.row_m = take(BH * N * 4);
  w.row_l = take(BH * N * 4);
  w.O32 = take(BH * N * static_cast<size_t>(d) * 4);
  w.colsum = take(BH * ng * static_cast<size_t>(N) * 4);
  const size_t np = (ng + 1) / 2, kk = static_cast<size_t>(k < N ? k : N);
  w.pair_idx = take(BH * np * 2 * kk * 4);   // union lists for the residual pass (stage entry)
  w.pair_len = take(BH * np * 4);
  w.total = o;
  return w;
}

template <typename T>
T *at(void *ws, size_t off) {
  return reinterpret_cast<T *>(static_cast<uint8_t *>(ws) + off);
}

mcs_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MCS_OK : MCS_ERR_CUDA; }

// ---------------------------------------------------------------- stages
template <int D>
cudaError_t run_group(const void *Q, int BH, int N, int32_t *perm, void *ws, const PlanWs &w,
                      cudaStream_t s) {
  const int nch = (N + kGroupChunk - 1) / kGroupChunk;
  const bf16 *q = static_cast<const bf16 *>(Q);
  mean_kernel<D><<<dim3(nch, BH), 256, 0, s>>>(q, N, nch, at<double>(ws, w.mean_part));
  mean_finalize_kernel<D><<<BH, D, 0, s>>>(at<double>(ws, w.mean_part), N, nch, at<double>(ws, w.mean));
  cov_kernel<D><<<dim3(nch, BH), 256, 0, s>>>(q, at<double>(ws, w.mean), N, nch, at<double>(ws, w.cov_part));
  cov_reduce_kernel<D><<<dim3((D * D + 255) / 256, BH), 256, 0, s>>>(at<double>(ws, w.cov_part), N, nch,
                                                                      at<double>(ws, w.cov64));
  const int eig_smem = (D * D + 3 * D) * 8;
  cudaError_t e = set_smem(eig_kernel<D>, eig_smem);
  if (e != cudaSuccess) return e;
  eig_kernel<D><<<BH, 256, eig_smem, s>>>(at<double>(ws, w.cov64), at<double>(ws, w.vdir),
                                           at<float>(ws, w.lambda));
  project_kernel<D><<<dim3((N + 7) / 8, BH), 256, 0, s>>>(q, at<double>(ws, w.mean), at<double>(ws, w.vdir), N,
                                                           at<unsigned long long>(ws, w.keys0),
                                                           at<int32_t>(ws, w.vals0));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // stable LSD radix sort of (key, token) over several CTAs per head; the last
  // pass writes its tokens straight into perm
  const int parts = sort_parts(BH, N), chunk = sort_chunk(N, parts);
  unsigned *gh = at<unsigned>(ws, w.ghist);
  unsigned long long *ka = at<unsigned long long>(ws, w.keys0), *kb = at<unsigned long long>(ws, w.keys1);
  int32_t *va = at<int32_t>(ws, w.vals0), *vb = at<int32_t>(ws, w.vals1);
  const dim3 grid(parts, BH);
  for (int pass = 0; pass < 8; ++pass) {
    sort_hist_kernel<<<grid, kSortThreads, 0, s>>>(ka, N, chunk, 8 * pass, gh);
    sort_scatter_kernel<<<grid, kSortThreads, 0, s>>>(ka, va, kb, pass == 7 ? perm : vb, N, chunk, 8 * pass, gh);
    std::swap(ka, kb);
    std::swap(va, vb);
  }
  return cudaGetLastError();
}

cudaError_t run_plan_dense(const void *Q, const void *K, const void *V, int BH, int N, int d, float scale,
                           void *O_dense, void *ws, const PlanWs &w, cudaStream_t s) {
  AttnArgs a = base_args(N, scale);
  a.O = static_cast<bf16 *>(O_dense);
  a.O32 = at<float>(ws, w.O32);
  a.row_m = at<float>(ws, w.row_m);
  a.row_l = at<float>(ws, w.row_l);
  return launch_attn_d<kModePlanDense>(d, a, QKV{Q, K, V}, (N + 127) / 128, BH, s);
}

cudaError_t run_scores(const void *Q, const void *K, const int32_t *perm, int BH, int N, int d, int G,
                       float scale, void *ws, const PlanWs &w, cudaStream_t s) {
  const int ng = (N + G - 1) / G;
  ColsumArgs c;
  std::memset(&c, 0, sizeof(c));
  if (!map_gather(&c.tmQ, Q, d, static_cast<size_t>(BH) * N) || !map_tile(&c.tmK, K, d, N, BH))
    return cudaErrorInvalidValue;
  c.perm = perm;
  c.row_m = at<float>(ws, w.row_m);
  c.row_l = at<float>(ws, w.row_l);
  c.colsum = at<float>(ws, w.colsum);
  c.N = N;
  c.G = G;
  c.n_groups = ng;
  c.scale_log2 = scale * 1.4426950408889634f;
  c.status = status_ptr();
  c.wait_ns = g_wait_ns;
  cudaError_t e;
  if (d == 64) {
    e = set_smem(colsum_kernel<64>, ColsumCfg<64>::SMEM);
    if (e != cudaSuccess) return e;
    colsum_kernel<64><<<dim3(ng, BH), 224, ColsumCfg<64>::SMEM, s>>>(c);
  } else {
    e = set_smem(colsum_kernel<128>, ColsumCfg<128>::SMEM);
    if (e != cudaSuccess) return e;
    colsum_kernel<128><<<dim3(ng, BH), 224, ColsumCfg<128>::SMEM, s>>>(c);
  }
  return cudaGetLastError();
}

// top-k of `rows` rows of N scores each: as many CTAs as fit on the device at
// once (or one per row), each over a contiguous run of rows
template <int VEC>
cudaError_t launch_topk_vec(const float *scores, long long rows, int N, int k, int32_t *kv_idx, cudaStream_t s) {
  cudaError_t e = set_smem(topk_kernel<VEC>, kTopkSmem);
  if (e != cudaSuccess) return e;
  int sms = 0, per_sm = 0;
  if ((e = sm_count(&sms)) != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_kernel<VEC>, kTopkThreads, kTopkSmem);
  if (e != cudaSuccess) return e;
  const long long fit = static_cast<long long>(sms) * (per_sm > 0 ? per_sm : 1);
  const int grid = static_cast<int>(rows < fit ? rows : fit);
  topk_kernel<VEC><<<grid, kTopkThreads, kTopkSmem, s>>>(scores, rows, N, k, kv_idx);
  return cudaGetLastError();
}

cudaError_t launch_topk(const float *scores, long long rows, int N, int k, int32_t *kv_idx, cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  if (N % 4 == 0 && aligned16(scores)) return launch_topk_vec<4>(scores, rows, N, k, kv_idx, s);
  return launch_topk_vec<1>(scores, rows, N, k, kv_idx, s);
}

cudaError_t run_topk(int BH, int N, int G, int k, int32_t *kv_idx, void *ws, const PlanWs &w,
                     cudaStream_t s) {
  const int ng = (N + G - 1) / G;
  return launch_topk(at<float>(ws, w.colsum), BH * ng, N, k, kv_idx, s);
}

// a5 over pairs of groups: the union lists go to (pair_idx, pair_len), which
// are the metadata's own lists or the workspace's scratch
cudaError_t run_residual(const void *Q, const void *K, const void *V, const int32_t *perm,
                         const int32_t *kv_idx, int BH, int N, int d, int G, int k, float scale,
                         float *residual, void *ws, const PlanWs &w, int32_t *pair_idx, int32_t *pair_len,
                         cudaStream_t s) {
  const int ng = (N + G - 1) / G;
  if (!pair_idx || !pair_len) {
    pair_idx = at<int32_t>(ws, w.pair_idx);
    pair_len = at<int32_t>(ws, w.pair_len);
  }
  cudaError_t e = run_pairs(kv_idx, BH, ng, k, pair_idx, pair_len, s);
  if (e != cudaSuccess) return e;
  AttnArgs a = base_args(N, scale);
  a.G = G;
  a.k = k;
  a.n_groups = ng;
  a.n_pairs = pairs_of(ng);
  a.perm = perm;
  a.kv_idx = kv_idx;
  a.pair_idx = pair_idx;
  a.pair_len = pair_len;
  a.O32_in = at<float>(ws, w.O32);
  a.R_out = residual;
  return launch_pair_d<kModePlanResid>(d, a, QKV{Q, K, V}, BH, s);
}

mcs_status check_common(const void *Q, const void *K, const void *V, int B, int H, int N, int d,
                        float scale) {
  if (!Q || !K || !V) return MCS_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V)) return MCS_ERR_INVALID_ARG;
  if (!shape_ok(B, H, N, d)) return MCS_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !(scale < INFINITY)) return MCS_ERR_INVALID_ARG;
  if (!d_ok(d)) return MCS_ERR_UNSUPPORTED;
  return MCS_OK;
}

mcs_status check_ws(void *ws, size_t bytes, size_t need) {
  if (!ws || bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MCS_ERR_WORKSPACE;
  return MCS_OK;
}

// ---------------------------------------------------------------- allocation-free validation scratch
// Fixed scratch for mcs_validate_meta_noalloc: a 256-byte flag area followed
// by one bit per token.  Host code may not pass the symbol itself to a kernel
// (on the host it only names a stand-in); the device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
constexpr size_t kNoAllocScratchBytes = 256 + (static_cast<size_t>(MCS_NOALLOC_MAX_TOKENS) + 7) / 8;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
unsigned char *g_noalloc_ptr[kMaxDevices];

unsigned char *noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
    g_noalloc_ptr[dev] = static_cast<unsigned char *>(p);
  }
  return g_noalloc_ptr[dev];
}

// pair-list check of mcs_validate_meta(_noalloc), when the metadata has them
void launch_pair_check(const mcs_meta *meta, int *bad, cudaStream_t s) {
  if (!meta->pair_idx || !meta->pair_len) return;
  const int np = pairs_of(meta->n_groups);
  const size_t items = static_cast<size_t>(meta->B) * meta->H * np;
  const unsigned grid = static_cast<unsigned>(items < 148 * 8 ? items : 148 * 8);
  pair_check_kernel<<<grid, 256, 0, s>>>(meta->pair_idx, meta->pair_len, meta->N, meta->k, meta->n_groups, np,
                                          items, bad);
}

}  // namespace

// ============================================================================ C ABI

extern "C" {

int mcs_abi_version(void) { return MCS_ABI_VERSION; }

const char *mcs_status_string(mcs_status s) {
  switch (s) {
    case MCS_OK: return "MCS_OK";
    case MCS_ERR_INVALID_ARG: return "MCS_ERR_INVALID_ARG";
    case MCS_ERR_UNSUPPORTED: return "MCS_ERR_UNSUPPORTED";
    case MCS_ERR_WORKSPACE: return "MCS_ERR_WORKSPACE";
    case MCS_ERR_CUDA: return "MCS_ERR_CUDA";
    case MCS_ERR_TIMEOUT: return "MCS_ERR_TIMEOUT";
    case MCS_ERR_BAD_META: return "MCS_ERR_BAD_META";
    case MCS_ERR_TOO_LARGE: return "MCS_ERR_TOO_LARGE";
  }
  return "MCS_ERR_UNKNOWN";
}

mcs_status mcs_meta_init(mcs_meta *meta, int B, int H, int N, int d, int G, int k) {
  if (!meta) return MCS_ERR_INVALID_ARG;
  if (!shape_ok(B, H, N, d) || k < 1) return MCS_ERR_INVALID_ARG;
  if (!d_ok(d) || !g_ok(G)) return MCS_ERR_UNSUPPORTED;
  meta->B = B;
  meta->H = H;
  meta->N = N;
  meta->d = d;
  meta->G = G;
  meta->k = k < N ? k : N;
  meta->n_groups = (N + G - 1) / G;
  return MCS_OK;
}

size_t mcs_plan_workspace_size(int B, int H, int N, int d, int G, int k) {
  if (!shape_ok(B, H, N, d) || !d_ok(d) || !g_ok(G) || k < 1) return 0;
  return plan_ws(B, H, N, d, G, k).total;
}

mcs_status mcs_plan_workspace_offsets(int B, int H, int N, int d, int G, int k, size_t *row_m, size_t *row_l,
                                      size_t *O32, size_t *colsum) {
  if (!shape_ok(B, H, N, d) || !d_ok(d) || !g_ok(G) || k < 1) return MCS_ERR_INVALID_ARG;
  const PlanWs w = plan_ws(B, H, N, d, G, k);
  if (row_m) *row_m = w.row_m;
  if (row_l) *row_l = w.row_l;
  if (O32) *O32 = w.O32;
  if (colsum) *colsum = w.colsum;
  return MCS_OK;
}

mcs_status mcs_plan_group(const void *Q, int B, int H, int N, int d, int32_t *perm, void *workspace,
                          size_t workspace_bytes, mcs_stream_t stream) {
  mcs_status st = check_common(Q, Q, Q, B, H, N, d, 1.f);
  if (st != MCS_OK) return st;
  if (!perm) return MCS_ERR_INVALID_ARG;
  const PlanWs w = plan_ws(B, H, N, d, 128, 1);
  // grouping needs only the part of the workspace before the statistics
  if ((st = check_ws(workspace, workspace_bytes, w.row_m)) != MCS_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int BH = B * H;
  return cuda_status(d == 64 ? run_group<64>(Q, BH, N, perm, workspace, w, s)
                             : run_group<128>(Q, BH, N, perm, workspace, w, s));
}

mcs_status mcs_plan_stats(const void *Q, const void *K, const void *V, int B, int H, int N, int d, int G,
                          int k, float scale, void *O_dense, void *workspace, size_t workspace_bytes,
                          mcs_stream_t stream) {
  mcs_status st = check_common(Q, K, V, B, H, N, d, scale);
  if (st != MCS_OK) return st;
  if (k < 1 || (O_dense && !aligned16(O_dense))) return MCS_ERR_INVALID_ARG;
  if (!g_ok(G)) return MCS_ERR_UNSUPPORTED;
  const PlanWs w = plan_ws(B, H, N, d, G, k);
  if ((st = check_ws(workspace, workspace_bytes, w.total)) != MCS_OK) return st;
  return cuda_status(run_plan_dense(Q, K, V, B * H, N, d, scale, O_dense, workspace, w,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

mcs_status mcs_plan_scores(const void *Q, const void *K, const int32_t *perm, int B, int H, int N, int d,
                           int G, int k, float scale, void *workspace, size_t workspace_bytes,
                           mcs_stream_t stream) {
  mcs_status st = check_common(Q, K, K, B, H, N, d, scale);
  if (st != MCS_OK) return st;
  if (!perm || k < 1) return MCS_ERR_INVALID_ARG;
  if (!g_ok(G)) return MCS_ERR_UNSUPPORTED;
  const PlanWs w = plan_ws(B, H, N, d, G, k);
  if ((st = check_ws(workspace, workspace_bytes, w.total)) != MCS_OK) return st;
  return cuda_status(run_scores(Q, K, perm, B * H, N, d, G, scale, workspace, w,
                                reinterpret_cast<cudaStream_t>(stream)));
}

mcs_status mcs_plan_topk(int B, int H, int N, int d, int G, int k, int32_t *kv_idx, void *workspace,
                         size_t workspace_bytes, mcs_stream_t stream) {
  if (!shape_ok(B, H, N, d) || !kv_idx || k < 1) return MCS_ERR_INVALID_ARG;
  if (!d_ok(d) || !g_ok(G)) return MCS_ERR_UNSUPPORTED;
  const PlanWs w = plan_ws(B, H, N, d, G, k);
  mcs_status st = check_ws(workspace, workspace_bytes, w.total);
  if (st != MCS_OK) return st;
  return cuda_status(run_topk(B * H, N, G, k < N ? k : N, kv_idx, workspace, w,
                              reinterpret_cast<cudaStream_t>(stream)));
}

mcs_status mcs_select_topk(const float *scores, int rows, int N, int k, int32_t *kv_idx,
                           mcs_stream_t stream) {
  if (!scores || !kv_idx || rows < 0 || N < 1 || k < 1) return MCS_ERR_INVALID_ARG;
  return cuda_status(launch_topk(scores, rows, N, k < N ? k : N, kv_idx,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

mcs_status mcs_plan_residual(const void *Q, const void *K, const void *V, const int32_t *perm,
                             const int32_t *kv_idx, int B, int H, int N, int d, int G, int k, float scale,
                             float *residual, void *workspace, size_t workspace_bytes, mcs_stream_t stream) {
  mcs_status st = check_common(Q, K, V, B, H, N, d, scale);
  if (st != MCS_OK) return st;
  if (!perm || !kv_idx || !residual || k < 1 || !aligned16(residual)) return MCS_ERR_INVALID_ARG;
  if (!g_ok(G)) return MCS_ERR_UNSUPPORTED;
  const PlanWs w = plan_ws(B, H, N, d, G, k);
  if ((st = check_ws(workspace, workspace_bytes, w.total)) != MCS_OK) return st;
  return cuda_status(run_residual(Q, K, V, perm, kv_idx, B * H, N, d, G, k < N ? k : N, scale, residual,
                                  workspace, w, nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream)));
}

mcs_status mcs_plan(const void *Q, const void *K, const void *V, int B, int H, int N, int d, int G, int k,
                    float scale, mcs_meta *meta, void *O_dense, void *workspace, size_t workspace_bytes,
                    mcs_stream_t stream) {
  mcs_status st = check_common(Q, K, V, B, H, N, d, scale);
  if (st != MCS_OK) return st;
  if (!meta || !meta->perm || !meta->kv_idx || !meta->residual) return MCS_ERR_INVALID_ARG;
  if (!aligned16(meta->residual) || (O_dense && !aligned16(O_dense))) return MCS_ERR_INVALID_ARG;
  if ((st = mcs_meta_init(meta, B, H, N, d, G, k)) != MCS_OK) return st;
  const PlanWs w = plan_ws(B, H, N, d, G, k);
  if ((st = check_ws(workspace, workspace_bytes, w.total)) != MCS_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int BH = B * H;
  cudaError_t e = d == 64 ? run_group<64>(Q, BH, N, meta->perm, workspace, w, s)
                          : run_group<128>(Q, BH, N, meta->perm, workspace, w, s);
  if (e == cudaSuccess) e = run_plan_dense(Q, K, V, BH, N, d, scale, O_dense, workspace, w, s);
  if (e == cudaSuccess) e = run_scores(Q, K, meta->perm, BH, N, d, G, scale, workspace, w, s);
  if (e == cudaSuccess) e = run_topk(BH, N, G, meta->k, meta->kv_idx, workspace, w, s);
  if (e == cudaSuccess)
    e = run_residual(Q, K, V, meta->perm, meta->kv_idx, BH, N, d, G, meta->k, scale, meta->residual,
                     workspace, w, meta->pair_idx, meta->pair_len, s);
  return cuda_status(e);
}

mcs_status mcs_meta_pairs(const mcs_meta *meta, mcs_stream_t stream) {
  if (!meta || !meta->kv_idx || !meta->pair_idx || !meta->pair_len) return MCS_ERR_INVALID_ARG;
  if (!shape_ok(meta->B, meta->H, meta->N, meta->d) || !d_ok(meta->d) || !g_ok(meta->G))
    return MCS_ERR_INVALID_ARG;
  if (meta->k < 1 || meta->k > meta->N || meta->n_groups != (meta->N + meta->G - 1) / meta->G)
    return MCS_ERR_INVALID_ARG;
  return cuda_status(run_pairs(meta->kv_idx, meta->B * meta->H, meta->n_groups, meta->k, meta->pair_idx,
                               meta->pair_len, reinterpret_cast<cudaStream_t>(stream)));
}

mcs_status mcs_sparse_step(const void *Q, const void *K, const void *V, const mcs_meta *meta, float scale,
                           void *O, mcs_stream_t stream) {
  if (!meta) return MCS_ERR_INVALID_ARG;
  mcs_status st = check_common(Q, K, V, meta->B, meta->H, meta->N, meta->d, scale);
  if (st != MCS_OK) return st;
  if (!O || !aligned16(O) || !meta->perm || !meta->kv_idx || !meta->residual) return MCS_ERR_INVALID_ARG;
  if (!aligned16(meta->residual)) return MCS_ERR_INVALID_ARG;
  if (!g_ok(meta->G)) return MCS_ERR_UNSUPPORTED;
  if (meta->k < 1 || meta->k > meta->N || meta->n_groups != (meta->N + meta->G - 1) / meta->G)
    return MCS_ERR_INVALID_ARG;
  AttnArgs a = base_args(meta->N, scale);
  a.G = meta->G;
  a.k = meta->k;
  a.n_groups = meta->n_groups;
  a.perm = meta->perm;
  a.kv_idx = meta->kv_idx;
  a.residual = meta->residual;
  a.O = static_cast<bf16 *>(O);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (meta->pair_idx && meta->pair_len) {
    a.n_pairs = pairs_of(meta->n_groups);
    a.pair_idx = meta->pair_idx;
    a.pair_len = meta->pair_len;
    return cuda_status(launch_pair_d<kModeStep>(meta->d, a, QKV{Q, K, V}, meta->B * meta->H, s));
  }
  return cuda_status(launch_attn_d<kModeStep>(meta->d, a, QKV{Q, K, V}, meta->n_groups, meta->B * meta->H, s));
}

mcs_status mcs_residual_compact(const float *residual, size_t n, void *residual_bf16, mcs_stream_t stream) {
  if (n == 0) return MCS_OK;
  if (!residual || !residual_bf16 || !aligned16(residual) || !aligned16(residual_bf16)) return MCS_ERR_INVALID_ARG;
  int sms = 0;
  cudaError_t e = sm_count(&sms);
  if (e != cudaSuccess) return cuda_status(e);
  const size_t want = (n / 8 + kCompactThreads - 1) / kCompactThreads;
  const size_t cap = static_cast<size_t>(sms) * 8;
  const unsigned grid = static_cast<unsigned>(want < 1 ? 1 : (want < cap ? want : cap));
  residual_compact_kernel<<<grid, kCompactThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      residual, n, static_cast<bf16 *>(residual_bf16));
  return cuda_status(cudaGetLastError());
}

mcs_status mcs_sparse_step_compact(const void *Q, const void *K, const void *V, const mcs_meta *meta,
                                   const void *residual_bf16, float scale, void *O, mcs_stream_t stream) {
  if (!meta) return MCS_ERR_INVALID_ARG;
  mcs_status st = check_common(Q, K, V, meta->B, meta->H, meta->N, meta->d, scale);
  if (st != MCS_OK) return st;
  if (!O || !aligned16(O) || !meta->perm || !meta->kv_idx || !residual_bf16 || !aligned16(residual_bf16))
    return MCS_ERR_INVALID_ARG;
  if (!meta->pair_idx || !meta->pair_len) return MCS_ERR_INVALID_ARG;
  if (!g_ok(meta->G)) return MCS_ERR_UNSUPPORTED;
  if (meta->k < 1 || meta->k > meta->N || meta->n_groups != (meta->N + meta->G - 1) / meta->G)
    return MCS_ERR_INVALID_ARG;
  AttnArgs a = base_args(meta->N, scale);
  a.G = meta->G;
  a.k = meta->k;
  a.n_groups = meta->n_groups;
  a.perm = meta->perm;
  a.kv_idx = meta->kv_idx;
  a.residual16 = static_cast<const bf16 *>(residual_bf16);
  a.O = static_cast<bf16 *>(O);
  a.n_pairs = pairs_of(meta->n_groups);
  a.pair_idx = meta->pair_idx;
  a.pair_len = meta->pair_len;
  return cuda_status(launch_pair_d<kModeStep>(meta->d, a, QKV{Q, K, V}, meta->B * meta->H,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

mcs_status mcs_dense(const void *Q, const void *K, const void *V, int B, int H, int N, int d, float scale,
                     void *O, mcs_stream_t stream) {
  mcs_status st = check_common(Q, K, V, B, H, N, d, scale);
  if (st != MCS_OK) return st;
  if (!O || !aligned16(O)) return MCS_ERR_INVALID_ARG;
  AttnArgs a = base_args(N, scale);
  a.O = static_cast<bf16 *>(O);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return cuda_status(launch_attn_d<kModeDense>(d, a, QKV{Q, K, V}, (N + 127) / 128, B * H, s));
}

size_t mcs_validate_workspace_size(int B, int H, int N) {
  if (B < 1 || H < 1 || N < 1) return 0;
  const size_t bits = static_cast<size_t>(B) * H * N;
  return align256(256 + ((bits + 31) / 32) * 4);
}

mcs_status mcs_validate_meta(const mcs_meta *meta, void *workspace, size_t workspace_bytes, int *first_bad,
                             mcs_stream_t stream) {
  if (first_bad) *first_bad = 0;
  if (!meta || !meta->perm || !meta->kv_idx || !meta->residual) return MCS_ERR_INVALID_ARG;
  if (!shape_ok(meta->B, meta->H, meta->N, meta->d) || !d_ok(meta->d) || !g_ok(meta->G))
    return MCS_ERR_INVALID_ARG;
  if (meta->k < 1 || meta->k > meta->N || meta->n_groups != (meta->N + meta->G - 1) / meta->G)
    return MCS_ERR_INVALID_ARG;
  const size_t need = mcs_validate_workspace_size(meta->B, meta->H, meta->N);
  mcs_status st = check_ws(workspace, workspace_bytes, need);
  if (st != MCS_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int BH = meta->B * meta->H;
  int *bad = static_cast<int *>(workspace);
  unsigned *seen = reinterpret_cast<unsigned *>(static_cast<uint8_t *>(workspace) + 256);
  const int init = INT_MAX;
  cudaError_t e = cudaMemcpyAsync(bad, &init, sizeof(int), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(seen, 0, need - 256, s);
  if (e != cudaSuccess) return MCS_ERR_CUDA;
  const int grid = 148 * 8;
  perm_mark_kernel<<<grid, 256, 0, s>>>(meta->perm, meta->N, BH, seen, bad);
  kv_check_kernel<<<grid, 256, 0, s>>>(meta->kv_idx, meta->N, meta->k,
                                       static_cast<size_t>(BH) * meta->n_groups, bad);
  residual_check_kernel<<<grid, 256, 0, s>>>(meta->residual,
                                             static_cast<size_t>(BH) * meta->N * meta->d, bad);
  launch_pair_check(meta, bad, s);
  if (cudaGetLastError() != cudaSuccess) return MCS_ERR_CUDA;
  int h = INT_MAX;
  e = cudaMemcpyAsync(&h, bad, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return MCS_ERR_CUDA;
  if (h == INT_MAX) return MCS_OK;
  if (first_bad) *first_bad = h;
  return MCS_ERR_BAD_META;
}

mcs_status mcs_validate_meta_noalloc(const mcs_meta *meta, int *first_bad, mcs_stream_t stream) {
  if (first_bad) *first_bad = 0;
  if (!meta || !meta->perm || !meta->kv_idx || !meta->residual) return MCS_ERR_INVALID_ARG;
  if (!shape_ok(meta->B, meta->H, meta->N, meta->d) || !d_ok(meta->d) || !g_ok(meta->G))
    return MCS_ERR_INVALID_ARG;
  if (meta->k < 1 || meta->k > meta->N || meta->n_groups != (meta->N + meta->G - 1) / meta->G)
    return MCS_ERR_INVALID_ARG;
  const size_t tokens = static_cast<size_t>(meta->B) * meta->H * meta->N;
  if (tokens > MCS_NOALLOC_MAX_TOKENS) return MCS_ERR_TOO_LARGE;
  unsigned char *scratch = noalloc_scratch();
  if (!scratch) return MCS_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int BH = meta->B * meta->H;
  int *bad = reinterpret_cast<int *>(scratch);
  unsigned *seen = reinterpret_cast<unsigned *>(scratch + 256);
  const size_t bitmap_bytes = ((tokens + 31) / 32) * 4;
  // the array keeps the previous call's contents: clear the flag and every bit this call reads
  const int init = INT_MAX;
  cudaError_t e = cudaMemcpyAsync(bad, &init, sizeof(int), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(seen, 0, bitmap_bytes, s);
  if (e != cudaSuccess) return MCS_ERR_CUDA;
  const int grid = 148 * 8;
  perm_mark_kernel<<<grid, 256, 0, s>>>(meta->perm, meta->N, BH, seen, bad);
  kv_check_kernel<<<grid, 256, 0, s>>>(meta->kv_idx, meta->N, meta->k,
                                       static_cast<size_t>(BH) * meta->n_groups, bad);
  residual_check_kernel<<<grid, 256, 0, s>>>(meta->residual, tokens * meta->d, bad);
  launch_pair_check(meta, bad, s);
  if (cudaGetLastError() != cudaSuccess) return MCS_ERR_CUDA;
  int h = INT_MAX;
  e = cudaMemcpyAsync(&h, bad, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return MCS_ERR_CUDA;
  if (h == INT_MAX) return MCS_OK;
  if (first_bad) *first_bad = h;
  return MCS_ERR_BAD_META;
}

size_t mcs_select_blocks_workspace_size(int rows, int N, int block, int k_blocks) {
  if (rows < 0 || N < 1 || block < 1 || k_blocks < 1 || N / block < k_blocks) return 0;
  const size_t nb = N / block;
  return align256(static_cast<size_t>(rows) * nb * 4) + align256(static_cast<size_t>(rows) * k_blocks * 4);
}

mcs_status mcs_select_blocks(const float *scores, int rows, int N, int block, int k_blocks, int32_t *kv_idx,
                             void *workspace, size_t workspace_bytes, mcs_stream_t stream) {
  if (!scores || !kv_idx || rows < 0 || N < 1 || block < 1 || k_blocks < 1 || N / block < k_blocks)
    return MCS_ERR_INVALID_ARG;
  const size_t need = mcs_select_blocks_workspace_size(rows, N, block, k_blocks);
  if (rows == 0) return MCS_OK;
  mcs_status st = check_ws(workspace, workspace_bytes, need);
  if (st != MCS_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int nb = N / block;
  float *bs = static_cast<float *>(workspace);
  int32_t *blk = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(workspace) +
                                             align256(static_cast<size_t>(rows) * nb * 4));
  block_sum_kernel<<<148 * 8, 256, 0, s>>>(scores, rows, N, block, bs);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = launch_topk(bs, rows, nb, k_blocks, blk, s);
  if (e == cudaSuccess) {
    expand_blocks_kernel<<<148 * 8, 256, 0, s>>>(blk, rows, k_blocks, block, kv_idx);
    e = cudaGetLastError();
  }
  return cuda_status(e);
}

mcs_status mcs_select_block_indices(const float *scores, int rows, int N, int block, int k_blocks,
                                    int32_t *blk_idx, void *workspace, size_t workspace_bytes,
                                    mcs_stream_t stream) {
  if (!scores || !blk_idx || rows < 0 || N < 1 || block < 1 || k_blocks < 1 || N / block < k_blocks)
    return MCS_ERR_INVALID_ARG;
  const size_t need = mcs_select_blocks_workspace_size(rows, N, block, k_blocks);
  if (rows == 0) return MCS_OK;
  mcs_status st = check_ws(workspace, workspace_bytes, need);
  if (st != MCS_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float *bs = static_cast<float *>(workspace);
  block_sum_kernel<<<148 * 8, 256, 0, s>>>(scores, rows, N, block, bs);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = launch_topk(bs, rows, N / block, k_blocks, blk_idx, s);
  return cuda_status(e);
}

mcs_status mcs_union_pairs(const int32_t *lists, int B, int H, int n_groups, int k, int32_t *pair_idx,
                           int32_t *pair_len, mcs_stream_t stream) {
  if (!lists || !pair_idx || !pair_len || B < 0 || H < 0 || n_groups < 0 || k < 1) return MCS_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 65535) return MCS_ERR_UNSUPPORTED;
  return cuda_status(run_pairs(lists, B * H, n_groups, k, pair_idx, pair_len, reinterpret_cast<cudaStream_t>(stream)));
}

mcs_status mcs_sparse_step_blocks(const void *Q, const void *K, const void *V, int B, int H, int N, int d, int G,
                                  int block, int k_blocks, const int32_t *perm, const int32_t *pair_idx,
                                  const int32_t *pair_len, const float *residual, float scale, void *O,
                                  mcs_stream_t stream) {
  mcs_status st = check_common(Q, K, V, B, H, N, d, scale);
  if (st != MCS_OK) return st;
  if (!O || !aligned16(O) || !perm || !pair_idx || !pair_len) return MCS_ERR_INVALID_ARG;
  if (residual && !aligned16(residual)) return MCS_ERR_INVALID_ARG;
  if (!g_ok(G) || (block != 64 && block != 128)) return MCS_ERR_UNSUPPORTED;
  if (k_blocks < 1 || k_blocks > N / block) return MCS_ERR_INVALID_ARG;
  AttnArgs a = base_args(N, scale);
  a.G = G;
  a.k = k_blocks;
  a.n_groups = (N + G - 1) / G;
  a.perm = perm;
  a.residual = residual;
  a.O = static_cast<bf16 *>(O);
  a.n_pairs = pairs_of(a.n_groups);
  a.pair_idx = pair_idx;
  a.pair_len = pair_len;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const QKV t{Q, K, V};
  const int BH = B * H;
  cudaError_t e;
  if (d == 64)
    e = block == 64 ? launch_pair<64, kModeStep, 64>(a, t, BH, s) : launch_pair<64, kModeStep, 128>(a, t, BH, s);
  else
    e = block == 64 ? launch_pair<128, kModeStep, 64>(a, t, BH, s) : launch_pair<128, kModeStep, 128>(a, t, BH, s);
  return cuda_status(e);
}

mcs_status mcs_pooled_scores(const void *Q, const void *K, const int32_t *perm, int B, int H, int N, int d, int G,
                             float scale, float *scores, mcs_stream_t stream) {
  mcs_status st = check_common(Q, K, K, B, H, N, d, scale);
  if (st != MCS_OK) return st;
  if (!perm || !scores) return MCS_ERR_INVALID_ARG;
  if (!g_ok(G)) return MCS_ERR_UNSUPPORTED;
  const int ng = (N + G - 1) / G;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const float sl2 = scale * 1.4426950408889634f;
  const dim3 grid(ng, B * H);
  if (d == 64)
    pooled_scores_kernel<64><<<grid, kPooledThreads, 0, s>>>(static_cast<const bf16 *>(Q), static_cast<const bf16 *>(K),
                                                             perm, N, G, ng, sl2, scores, status_ptr());
  else
    pooled_scores_kernel<128><<<grid, kPooledThreads, 0, s>>>(static_cast<const bf16 *>(Q), static_cast<const bf16 *>(K),
                                                              perm, N, G, ng, sl2, scores, status_ptr());
  return cuda_status(cudaGetLastError());
}

mcs_status mcs_last_device_status(mcs_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned *p = status_ptr();
  if (!p) return MCS_ERR_CUDA;
  unsigned h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, p, sizeof(unsigned), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(p, 0, sizeof(unsigned), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return MCS_ERR_CUDA;
  return h == 0 ? MCS_OK : static_cast<mcs_status>(h);
}

void mcs_set_wait_limit_ns(uint64_t ns) { g_wait_ns = ns ? ns : 4000000000ull; }

// Self-test of the bounded wait (declared in mcs.h).
mcs_status mcs_selftest_wait_timeout(uint64_t limit_ns, mcs_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned *p = status_ptr();
  if (!p) return MCS_ERR_CUDA;
  wait_selftest_kernel<<<1, 32, 0, s>>>(limit_ns ? limit_ns : 1000000ull, p);
  return cuda_status(cudaGetLastError());
}

}  // extern "C"
