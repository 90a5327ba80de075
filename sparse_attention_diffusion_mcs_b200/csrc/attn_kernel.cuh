// attn_kernel.cuh -- the sparse tcgen05 / TMEM / TMA flash-attention kernel
// (two uses) and the argument block it shares with the dense kernel of
// attn_dual_kernel.cuh.
//
//  kModeStep      the reused denoising step (split-precision P, like the plan
//                 passes): each CTA owns one query group
//                 (rows gathered through perm), attends only to the group's
//                 cached KV indices (rows gathered through kv_idx), adds the
//                 cached residual in the epilogue and scatters bf16 rows back
//                 to the original token order (aiqbench.com abstract: query
//                 groups, KV indices and residuals "reused across subsequent
//                 denoising steps"; cnshai.top post, section "MC-Sparse:
//                 three failure modes, one fix").
//  kModePlanResid sparse pass of the plan with split-precision P (bf16 hi +
//                 lo parts, two P.V MMAs, ~2^-17 relative error instead of
//                 2^-9); the epilogue writes R = O_dense - O_sparse (the cached
//                 residual "between dense and sparse attention outputs").
// (kModeDense and kModePlanDense, the dense passes, run in attn_dual_kernel.cuh.)
//
// A persistent CTA per SM takes (head, query group) items; per item, 128
// query rows x all of the group's key tiles of 128 keys:
//   warps 0-3  softmax + epilogue; thread t owns query row t = TMEM lane t
//   warp  4    TMEM allocation and the single UMMA-issuing thread
//   warps 5-8  Q and K producers, 9-11 V producers (384 threads)
// Rows listed by index arrive through TMA tile::gather4, four
// 128-byte rows per instruction.  On B200 its throughput grows with the
// number of issuing warps (measured 2.1 TB/s from one warp, 3.4 from two, 5
// from four, 6.4 from eight), so the K ring has four issuing warps and the V
// ring three, each owning an interleaved share of the tile's gather4
// operations.  (A 288-thread CTA is register-allocated like 384 threads, so
// the extra warps cost no registers.)
// TMEM: S double buffer (2 x 128 fp32 columns) + O (D columns) + the lo part
// of P (2 x 64 columns).  P's hi part (bf16 pairs) is written over its own S
// buffer; P.V runs with A straight from TMEM, so shared memory holds only Q
// and the K and V rings.
// Synchronisation is mbarrier-only inside the loops; every wait is bounded.
#pragma once

#include <type_traits>

#include "mcs_common.cuh"

namespace mcs {

enum AttnMode : int { kModeDense = 0, kModeStep = 1, kModePlanDense = 2, kModePlanResid = 3 };

constexpr bool is_sparse_mode(int mode) { return mode == kModeStep || mode == kModePlanResid; }

struct alignas(64) AttnArgs {
  CUtensorMap tmQ, tmK, tmV;   // gather maps (2D, box {64,1}) or tile maps (3D, box {64,128,1})
  int N;                   // tokens per head
  int G;                   // query group size (sparse modes)
  int k;                   // kept keys per group (sparse modes), <= N
  int n_groups;            // ceil(N / G)
  float scale_log2;        // softmax scale * log2(e)
  const int32_t *perm;     // [BH, N]               sparse modes
  const int32_t *kv_idx;   // [BH, n_groups, k]     sparse modes
  const float *residual;   // [BH, N, D]            kModeStep
  bf16 *O;                 // [BH, N, D] bf16 out   dense / step / plan-dense (optional)
  float *O32;              // [BH, N, D]            kModePlanDense
  const float *O32_in;     // [BH, N, D]            kModePlanResid
  float *R_out;            // [BH, N, D]            kModePlanResid
  float *row_m, *row_l;    // [BH, N]               kModePlanDense (log2 domain)
  unsigned *status;        // device status word
  uint64_t wait_ns;        // bound on any single wait
  int BH;                  // heads; work items are (head, query tile or group) pairs
  const int32_t *pair_idx; // [BH, n_pairs, 2k]     pair kernel: union list of groups 2p, 2p+1
  const int32_t *pair_len; // [BH, n_pairs]         pair kernel: union sizes
  int n_pairs;             // ceil(n_groups / 2)
  const bf16 *residual16;  // [BH, N, D] bf16       pair kernel, kModeStep: compact residual (replaces residual)
};

template <int D, int MODE>
struct AttnCfg {
  static_assert(is_sparse_mode(MODE), "sparse modes only");
  static constexpr int BM = 128, BN = 128;
  // split-precision P (bf16 hi + lo, two P.V MMAs): the reused step adds a
  // residual that can nearly cancel the sparse output, so the sparse output
  // needs more than bf16's 2^-9
  static constexpr int NK = D == 64 ? 6 : 3;   // K ring depth
  static constexpr int NV = D == 64 ? 6 : 3;   // V ring depth
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + NV * KV_BYTES;
  static constexpr int N_BAR = 1 + 2 * NK + 2 * NV + 8;   // q, k/v full/empty, s_full[2], p[2], pv[2], drain, q_empty
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BAR;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;          // + slack to align the base to 1 KB
  static constexpr int KW = 4, VW = 3;   // issuing warps per ring
  static constexpr int THREADS = (5 + KW + VW) * 32;   // softmax 0-3, MMA 4, then the K and V warps
  // The softmax reference max trails the true row max by up to 2^kRaise (log2
  // units) before O and l are rescaled.  bf16 P and fp32 O, l keep their
  // relative precision at any scale, so the only bound is range: P <= 2^32
  // and l <= N 2^32 stay far from fp32 overflow for |V| < 2^64.
  static constexpr float kRaise = 32.f;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O = 256, COL_PLO = 384;
};

template <int D, int MODE>
__global__ void __launch_bounds__(AttnCfg<D, MODE>::THREADS, 1) attn_kernel(const __grid_constant__ AttnArgs a) {
  using C = AttnCfg<D, MODE>;
  constexpr int BM = C::BM, BN = C::BN, NK = C::NK, NV = C::NV;
  constexpr int NDB = D / 64;                       // 64-column (128-byte) blocks per row
  constexpr uint32_t TILE_TX = 128u * D * 2u;       // bytes of one 128-row tile

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sK0 = sbase + C::OFF_K;
  const uint32_t sV0 = sbase + C::OFF_V;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t b_q = bar0;
  auto b_kfull = [&](int s) { return bar0 + 8 * (1 + s); };
  auto b_kempty = [&](int s) { return bar0 + 8 * (1 + NK + s); };
  auto b_vfull = [&](int s) { return bar0 + 8 * (1 + 2 * NK + s); };
  auto b_vempty = [&](int s) { return bar0 + 8 * (1 + 2 * NK + NV + s); };
  const uint32_t b_sfull0 = bar0 + 8 * (1 + 2 * NK + 2 * NV);
  // "P ready" and "P.V done" alternate between two barriers each by tile
  // parity.  The softmax warps wait on P.V only now and then (a rescale, the
  // epilogue) and may publish P two tiles in a row before the MMA thread has
  // looked, so up to two completions of each kind can be outstanding; with
  // one barrier per parity each has at most one, and a parity wait cannot
  // alias (P of tile j+2 needs S of tile j+2, whose Q.K^T is issued after
  // the P.V of tile j, which needs P of tile j)
  auto b_p = [&](int gj) { return b_sfull0 + 16 + 8 * (gj & 1); };
  auto b_pv = [&](int gj) { return b_sfull0 + 32 + 8 * (gj & 1); };
  const uint32_t b_drain = b_sfull0 + 48;
  const uint32_t b_qempty = b_sfull0 + 56;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int N = a.N;
  // Work items are (head, query group) pairs, head-major; CTA c takes items c, c + grid,
  // c + 2 grid, ...  Every item has the same number of key tiles T, so the
  // rings, S buffers and barrier phases run on one tile counter per CTA and
  // the next item's loads and first Q.K^T overlap this item's epilogue.
  const int per_head = a.n_groups;
  const int n_items = a.BH * per_head;
  const int nkeys = a.k;
  const int T = (nkeys + BN - 1) / BN;
  struct Item {
    int tile, bh;
    size_t head;
    const int32_t *kv_list;
  };
  auto item_at = [&](int item) -> Item {
    Item w;
    w.tile = item % per_head;
    w.bh = item / per_head;
    w.head = static_cast<size_t>(w.bh) * N;
    w.kv_list = a.kv_idx + (static_cast<size_t>(w.bh) * a.n_groups + w.tile) * a.k;
    return w;
  };

  // query row r of an item -> token index, or -1 when the row is padding.
  // q_raw only loads (so the load can be issued long before its use);
  // q_check validates what it loaded.
  auto q_raw = [&](const Item &w, int r) -> int {
    const int gr = w.tile * a.G + r;
    return (r >= a.G || gr >= N) ? -1 : a.perm[w.head + gr];
  };
  auto q_check = [&](int q) -> int {
    if (q != -1 && static_cast<unsigned>(q) >= static_cast<unsigned>(N)) {
      record_status(a.status, kStatusBadMeta);   // corrupt metadata: never gather out of range
      return -1;
    }
    return q;
  };
  auto q_token = [&](const Item &w, int r) -> int { return q_check(q_raw(w, r)); };

  if (tid == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < NK; ++s) {
      mbar_init(b_kfull(s), 1);
      mbar_init(b_kempty(s), 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(b_vfull(s), 1);
      mbar_init(b_vempty(s), 1);
    }
    mbar_init(b_sfull0, 1);
    mbar_init(b_sfull0 + 8, 1);
    mbar_init(b_p(0), 128);
    mbar_init(b_p(1), 128);
    mbar_init(b_pv(0), 1);
    mbar_init(b_pv(1), 1);
    mbar_init(b_drain, 1);
    mbar_init(b_qempty, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 5 && lane == 0) {
    tma_prefetch_desc(&a.tmQ);
    tma_prefetch_desc(&a.tmK);
    tma_prefetch_desc(&a.tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp >= 5) {
    // ------------------------------------------------------------------ TMA producers
    const int pw = warp - 5;                  // 0..KW-1: K ring, KW..KW+VW-1: V ring
    const bool is_k = pw < C::KW;
    const int NW = is_k ? C::KW : C::VW;      // issuing warps of this ring
    const int h = is_k ? pw : pw - C::KW;     // this warp's share of the tile's operations
    const void *tm = is_k ? static_cast<const void *>(&a.tmK) : static_cast<const void *>(&a.tmV);
    const int NS = is_k ? NK : NV;
    const uint32_t ring = is_k ? sK0 : sV0;
    // gather4 operation o (4 rows x 128 bytes) of a tile belongs to
    // warp o % NW, lane o / NW; a tile has 32 row quads x NDB column blocks
    constexpr int OPS = 32 * NDB;
    const int op_raw = h + NW * lane;
    const bool active = op_raw < OPS;
    const int op = active ? op_raw : h;
    const int quad = op % 32, dbk = op / 32;
    bool ok = true;
    int issued = 0;                           // fills of this ring by this CTA
    int nq = 0;                               // Q tiles loaded (K ring warps)
    for (int item = blockIdx.x, it = 0; item < n_items && ok; item += gridDim.x, ++it) {
      const Item w = item_at(item);
      // global row indices of tile t for this lane's gather4
      auto tile_rows = [&](int t, int (&rows)[4]) {
        const int first = w.kv_list[0];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int pos = t * BN + 4 * quad + i;
          int key = pos < nkeys ? w.kv_list[pos] : first;   // padding keys re-read a valid key (masked later)
          if (static_cast<unsigned>(key) >= static_cast<unsigned>(N)) {   // corrupt metadata
            record_status(a.status, kStatusBadMeta);
            key = 0;
          }
          rows[i] = static_cast<int>(w.head) + key;
        }
      };
      int rows[4] = {0, 0, 0, 0}, next[4] = {0, 0, 0, 0};
      tile_rows(0, rows);
      if (is_k) {
        // the item's Q tile, once the previous item's last Q.K^T has read the buffer
        if (it > 0) {
          int got = 1;
          if (lane == 0) got = mbar_wait(b_qempty, (it - 1) & 1, a.wait_ns, abort_flag);
          got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) { ok = false; break; }
        }
        const int q0 = q_token(w, 0);
        const int fallback = q0 >= 0 ? q0 : 0;   // padding rows re-read a valid row
        int qrows[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int q = q_token(w, 4 * quad + i);
          qrows[i] = static_cast<int>(w.head) + (q >= 0 ? q : fallback);
        }
        if (h == 0 && lane == 0) mbar_arrive_expect_tx(b_q, TILE_TX);
        __syncwarp();
        if (active)
          tma_gather4(sQ + dbk * (BM * 128) + quad * 512, &a.tmQ, dbk * 64, qrows[0], qrows[1], qrows[2],
                      qrows[3], b_q);
        ++nq;
      }
      for (int j = 0; j < T; ++j) {
        const int s = issued % NS;
        if (j + 1 < T) tile_rows(j + 1, next);   // in flight while we wait for the slot
        int got = 1;
        if (lane == 0)
          got = mbar_wait(is_k ? b_kempty(s) : b_vempty(s), ((issued / NS) & 1) ^ 1, a.wait_ns, abort_flag);
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) { ok = false; break; }
        const uint32_t full = is_k ? b_kfull(s) : b_vfull(s);
        const uint32_t dst = ring + s * C::KV_BYTES;
        // one expect-tx arrival per phase; the other warps' bytes may land first
        if (h == 0 && lane == 0) mbar_arrive_expect_tx(full, TILE_TX);
        __syncwarp();
        if (active)
          tma_gather4(dst + dbk * (BN * 128) + quad * 512, tm, dbk * 64, rows[0], rows[1], rows[2], rows[3], full);
#pragma unroll
        for (int i = 0; i < 4; ++i) rows[i] = next[i];
        ++issued;
      }
    }
    if (!ok && lane == 0 && !*abort_flag) {
      *abort_flag = 1;
      record_status(a.status, kStatusTimeout);
    }
    // never leave the CTA with a copy still landing in its shared memory
    if (lane == 0) {
      volatile int never = 0;
      for (int t = (issued > NS ? issued - NS : 0); t < issued; ++t)
        mbar_wait(is_k ? b_kfull(t % NS) : b_vfull(t % NS), (t / NS) & 1, 2000000000ull, &never);
      if (is_k && nq > 0) mbar_wait(b_q, (nq - 1) & 1, 2000000000ull, &never);
    }
    __syncwarp();
  } else if (warp == 4) {
    // ------------------------------------------------------------------ UMMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, 1);
      const uint32_t tS0 = tbase + C::COL_S0, tS1 = tbase + C::COL_S1, tO = tbase + C::COL_O;
      bool ok = true;
      int g = 0;                               // this CTA's key tiles so far (all items)
      // tile j of the current item is global tile g + j: ring slot, S buffer and phases
      auto issue_qk = [&](int j) -> bool {
        const int gj = g + j;
        const int s = gj % NK;
        if (!mbar_wait(b_kfull(s), (gj / NK) & 1, a.wait_ns, abort_flag)) return false;
        tc_fence_after();
        const uint32_t kb = sK0 + s * C::KV_BYTES;
        const uint32_t tS = (gj & 1) ? tS1 : tS0;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          umma_bf16_ss(tS, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024),
                       idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(b_sfull0 + 8 * (gj & 1));
        umma_commit(b_kempty(s));
        if (j == T - 1) umma_commit(b_qempty);   // the item's last read of Q
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int gj = g + j;
        const int s = gj % NV;
        if (!mbar_wait(b_p(gj), (gj >> 1) & 1, a.wait_ns, abort_flag)) return false;
        if (!mbar_wait(b_vfull(s), (gj / NV) & 1, a.wait_ns, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vb = sV0 + s * C::KV_BYTES;
        const uint32_t tP = (gj & 1) ? tS1 : tS0;                              // hi part over S
        const uint32_t tPlo = tbase + C::COL_PLO + (gj & 1) * (BN / 2);        // lo part
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t bdesc = sdesc_sw128(vb + kk * 16 * 128, BN * 128, 1024);
          umma_bf16_ts(tO, tP + kk * 8, bdesc, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t bdesc = sdesc_sw128(vb + kk * 16 * 128, BN * 128, 1024);
          umma_bf16_ts(tO, tPlo + kk * 8, bdesc, idesc_pv, 1u);
        }
        umma_commit(b_pv(gj));
        umma_commit(b_vempty(s));
        return true;
      };
      // the next item's first P.V (accumulate = 0) overwrites O only after its
      // P is ready, which the softmax warps publish after reading this item's O
      for (int item = blockIdx.x, it = 0; item < n_items && ok; item += gridDim.x, ++it) {
        ok = mbar_wait(b_q, it & 1, a.wait_ns, abort_flag);
        if (ok) ok = issue_qk(0);
        if (ok && T > 1) ok = issue_qk(1);
        for (int j = 0; j < T && ok; ++j) {
          ok = issue_pv(j);
          if (ok && j + 2 < T) ok = issue_qk(j + 2);
        }
        g += T;
      }
      if (!ok && !*abort_flag) {
        *abort_flag = 1;
        record_status(a.status, kStatusTimeout);
      }
      // make sure nothing issued is still running before TMEM is released
      umma_commit(b_drain);
      volatile int never = 0;
      mbar_wait(b_drain, 0, 2000000000ull, &never);
    }
  } else {
    // ------------------------------------------------------------------ softmax
    const int r = tid;                           // query row == TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = a.scale_log2;
    bool ok = true;
    int g = 0;                                   // this CTA's key tiles so far (all items)
    // the epilogue's second input (residual, or the dense output), read per row
    const float *ep_in = MODE == kModeStep ? a.residual : a.O32_in;
    auto warm_row = [&](size_t head_, int q) {   // pull the row into L2 well before the epilogue
      if (q >= 0) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(ep_in + (head_ + q) * D + c * 32));
      }
    };
    int my_q = -1;
    if (static_cast<int>(blockIdx.x) < n_items) {
      const Item w0 = item_at(blockIdx.x);
      my_q = q_token(w0, r);
      warm_row(w0.head, my_q);
    }
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, g += T) {
    const Item w = item_at(item);
    const size_t head = w.head;
    // the next item's token, loaded now and used after this item's tiles
    const int nitem = item + static_cast<int>(gridDim.x);
    const bool has_next = nitem < n_items;
    const Item wn = item_at(has_next ? nitem : item);
    const int next_raw = has_next ? q_raw(wn, r) : -1;
    float m_run = -INFINITY, l_run = 0.f;
    for (int j = 0; j < T; ++j) {
      const int gj = g + j;
      if (!mbar_wait_warp(b_sfull0 + 8 * (gj & 1), (gj >> 1) & 1, a.wait_ns, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tS = tbase + lane_addr + ((gj & 1) ? C::COL_S1 : C::COL_S0);
      const uint32_t tPlo = tbase + lane_addr + C::COL_PLO + (gj & 1) * (BN / 2);
      const int nvalid = nkeys - j * BN;   // >= 1; only the last tile can be partial
      float alpha = 1.f;
      bool resc = false;
      float rs0 = 0.f, rs1 = 0.f;
      // new running max from this tile's max (scaled to the log2 domain)
      auto update_max = [&](float mx) {
        mx *= sl2;
        if (j == 0) {
          m_run = mx;
        } else if (mx > m_run + C::kRaise) {   // lazy rescale: only when the max grew by > 2^kRaise
          alpha = ex2_approx(m_run - mx);
          m_run = mx;
          resc = true;
        }
      };
      // P of 32 keys as 16 bf16 pairs over S; their lo parts in their own columns
      auto store_p = [&](const float (&pv)[32], uint32_t dst_hi, uint32_t dst_lo) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(pv[2 * i], pv[2 * i + 1]);
        tmem_st16u(dst_hi, pk);
        const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 h = make_float2(__uint_as_float(pk[i] << 16), __uint_as_float(pk[i] & 0xFFFF0000u));
          const float2 lo = __ffma2_rn(h, neg1, make_float2(pv[2 * i], pv[2 * i + 1]));   // exact v - h
          pk[i] = pack_bf16x2(lo.x, lo.y);
        }
        tmem_st16u(dst_lo, pk);
      };
      auto tile_body = [&](auto masked_tag) {
        constexpr bool kMask = decltype(masked_tag)::value;
        auto val = [&](float x, int col) -> float {
          if constexpr (kMask) return col < nvalid ? x : -INFINITY;
          else return x;
        };
        // pass 1: row max of this tile.  Both passes stay rolled: unrolled
        // over the four chunks they need more than the 168 registers a
        // thread of this CTA has, and the spills cost more than the loop.
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll 1
        for (int ch = 0; ch < BN / 64; ++ch) {
          float v[64];
          tmem_ld64(tS + ch * 64, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 64; i += 4) {
            m0 = fmax3(m0, val(v[i], ch * 64 + i), val(v[i + 1], ch * 64 + i + 1));
            m1 = fmax3(m1, val(v[i + 2], ch * 64 + i + 2), val(v[i + 3], ch * 64 + i + 3));
          }
        }
        update_max(fmaxf(m0, m1));
        // pass 2: P = 2^(s*scale*log2e - m); chunk cc lands on columns [16cc, 16cc+16),
        // all of them already read
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          float v[32];
          tmem_ld32(tS + cc * 32, v);
          tmem_wait_ld();
          // column pairs through the packed two-lane fp32 instructions
          const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-m_run, -m_run);
          float2 rs2 = make_float2(rs0, rs1);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 x = __ffma2_rn(make_float2(v[i], v[i + 1]), sc2, nm2);
            v[i] = ex2_approx(x.x);
            v[i + 1] = ex2_approx(x.y);
            if constexpr (kMask) {
              if (cc * 32 + i >= nvalid) v[i] = 0.f;
              if (cc * 32 + i + 1 >= nvalid) v[i + 1] = 0.f;
            }
            rs2 = __fadd2_rn(rs2, make_float2(v[i], v[i + 1]));
          }
          rs0 = rs2.x;
          rs1 = rs2.y;
          store_p(v, tS + cc * 16, tPlo + cc * 16);
        }
      };
      if (nvalid >= BN) tile_body(std::false_type{});
      else tile_body(std::true_type{});
      l_run = fmaf(l_run, alpha, rs0 + rs1);
      tmem_wait_st();
      // Only a warp with a row whose max moved by more than 2^kRaise waits for
      // the previous P.V (O then holds exactly the tiles before this one) and
      // rescales O; otherwise P is published at once and the P.V of this
      // tile queues behind the previous one in the tensor pipe.
      if (j > 0 && __any_sync(0xffffffffu, resc)) {
        if (!mbar_wait_warp(b_pv(gj - 1), ((gj - 1) >> 1) & 1, a.wait_ns, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tO = tbase + lane_addr + C::COL_O;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          float o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(tO + cc * 32, o);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(b_p(gj));
    }
    const int q = my_q;
    const size_t row = (head + (q >= 0 ? q : 0)) * D;
    // the epilogue input of the first chunk is in flight while the last P.V runs
    float4 ein[8];
    if (q >= 0) {
      const float4 *src = reinterpret_cast<const float4 *>(ep_in + row);
#pragma unroll
      for (int u = 0; u < 8; ++u) ein[u] = __ldg(src + u);
    }
    if (ok) {
      my_q = has_next ? q_check(next_raw) : -1;
      warm_row(wn.head, my_q);
    }
    // O is final once the item's last two P.V have completed (the earlier
    // ones completed before the last Q.K^T this thread has seen)
    for (int t = T >= 2 ? T - 2 : 0; t < T && ok; ++t)
      if (!mbar_wait_warp(b_pv(g + t), ((g + t) >> 1) & 1, a.wait_ns, abort_flag)) ok = false;
    if (ok) {
      // ------------------------------------------------------------------ epilogue
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      const uint32_t tO = tbase + lane_addr + C::COL_O;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        // next chunk's input in flight while this chunk is finished
        float4 enx[8];
        if (q >= 0 && cc + 1 < D / 32) {
          const float4 *src = reinterpret_cast<const float4 *>(ep_in + row + (cc + 1) * 32);
#pragma unroll
          for (int u = 0; u < 8; ++u) enx[u] = __ldg(src + u);
        }
        float o[32];
        tmem_ld32(tO + cc * 32, o);
        tmem_wait_ld();
        if (q >= 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= inv_l;
        if (MODE == kModeStep) {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            o[4 * u + 0] += ein[u].x;
            o[4 * u + 1] += ein[u].y;
            o[4 * u + 2] += ein[u].z;
            o[4 * u + 3] += ein[u].w;
          }
        }
        if (MODE == kModePlanResid) {
          float4 *rp = reinterpret_cast<float4 *>(a.R_out + row + cc * 32);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            rp[u] = make_float4(ein[u].x - o[4 * u], ein[u].y - o[4 * u + 1], ein[u].z - o[4 * u + 2],
                                ein[u].w - o[4 * u + 3]);
        }
        if (MODE == kModeStep) {
          uint4 *op = reinterpret_cast<uint4 *>(a.O + row + cc * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 w;
            w.x = pack_bf16x2(o[8 * u + 0], o[8 * u + 1]);
            w.y = pack_bf16x2(o[8 * u + 2], o[8 * u + 3]);
            w.z = pack_bf16x2(o[8 * u + 4], o[8 * u + 5]);
            w.w = pack_bf16x2(o[8 * u + 6], o[8 * u + 7]);
            op[u] = w;
          }
        }
        }   // q >= 0
        if (cc + 1 < D / 32) {
#pragma unroll
          for (int u = 0; u < 8; ++u) ein[u] = enx[u];
        }
      }
    }
    }   // items
    if (!ok && !*abort_flag) {
      *abort_flag = 1;
      record_status(a.status, kStatusTimeout);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace mcs
